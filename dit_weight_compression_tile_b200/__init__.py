"""B200-native fused decode of lattice-rANS compressed weights.

The library (``libeptile.so``, C ABI in ``include/eptile.h``) holds the host compressor,
the stream parser and the sm_100a decode kernel; ``binding`` marshals torch tensors to
it.  Importing the package loads nothing; the first use of a binding name imports
``binding``, whose ``lib()`` fails loudly when the built library is missing.
"""
_BINDING_NAMES = ("BF16", "FP16", "FP32", "INT8", "FP8E4M3", "EpError", "compress", "compress_device", "prepare",
                  "decompress", "decompress_host", "stream_info", "lib", "StreamInfo")


_COMPRESSED_NAMES = ("CompressedTensor", "LatticeRANSConfig", "TileANSConfig")
_LINEAR_NAMES = ("CompressedLinear", "CompressedFP8Linear", "CompressedINT8Linear")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    if name in _COMPRESSED_NAMES:
        from . import compressed
        return getattr(compressed, name)
    if name in _LINEAR_NAMES:
        from . import linear
        return getattr(linear, name)
    raise AttributeError(name)
