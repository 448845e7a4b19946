"""compress(tensor, config) -> CompressedTensor and decompress(compressed, config) -> tensor, the calls
of the API reference ("EntroPack API reference", Tensor encoding and decoding; CompressedTensor),
over the C ABI: ep_compress_device (a CUDA tensor) or ep_compress_host (a host tensor) builds the
stream, the same bytes either way; ep_prepare and the fused ep_decompress kernel decode it.  This module only keeps the pieces together (stream,
parsed plan, prepared tables, output dtype); it computes nothing itself.

Two schemes: the lossy lattice-rANS tile stream (LatticeRANSConfig) and the lossless Tile-ANS
stream (TileANSConfig: each element's top byte rANS-coded in the same lane tiles, the other bytes
kept as they are; ep_ans_compress_host, ep_ans_prepare, ep_ans_decompress).

Differences from the pages, by design: CompressedTensor is a plain object, not a torch.Tensor
subclass; decoding needs a CUDA device (no CPU decoder); DFloat11Config is not offered (Tile-ANS
covers BF16 losslessly); the "raw" container that the pages return when encoding fails is kept.
"""
import math
import warnings
from dataclasses import dataclass

import torch

from . import binding as B

STATE_VERSION = 1
_LATTICE, _RAW, _TILE_ANS = 0, 1, 2
_ELT = {torch.bfloat16: 2, torch.float16: 2, torch.float32: 4, torch.int8: 1, torch.float8_e4m3fn: 1}


@dataclass
class LatticeRANSConfig:
    """target_bpp: stored bits per element including metadata, in [0.001, 11] ([0.001, 8) for
    code containers).  container: None (the source dtype) or torch.int8 / torch.float8_e4m3fn
    (per-row absmax codes; the rate then counts the row scales).  blocks_per_lane: 0 picks it
    from the shape.  n_threads: host encoder threads (0: all cores).  coding: 0 automatic, 1 one
    token per coordinate, 2 coordinates 1..6 in pairs whenever their tokens allow (the decoder
    then does 5 table lookups per E8 block instead of 8).  layout: "rows" (the tiles follow the
    rows) or "gemm" (every tile one 128 x 64 operand tile of a consumer GEMM; rows a multiple of
    128, columns of 64; what CompressedLinear's fused forward reads)."""
    target_bpp: float = 4.0
    container: object = None
    blocks_per_lane: int = 0
    n_threads: int = 0
    coding: int = 0
    layout: str = "rows"


@dataclass
class TileANSConfig:
    """The lossless scheme: every bit of a BF16, FP16, FP32, INT8 or FP8 E4M3 tensor of any shape.
    blocks_per_lane: chunks of 8 elements per lane, 0 picks it from the size.  n_threads: host
    encoder threads (0: all cores)."""
    blocks_per_lane: int = 0
    n_threads: int = 0


class CompressedTensor:
    """One compressed tensor: the stream (a uint8 tensor on some device) and its parsed plan, or,
    for compress_method == "raw", the tensor itself.  ``ans`` marks a Tile-ANS stream."""

    def __init__(self, blob=None, info=None, out_dtype=None, raw=None, ans=False):
        self._blob, self._info, self._raw, self._ans = blob, info, raw, ans
        if out_dtype is None:
            out_dtype = raw.dtype if raw is not None else (info.torch_dtype if ans else info.dtype)
        self._dtype = out_dtype
        self._work = None  # (workspace, event) of the slot tables prepared for this device copy

    # ---- properties of the API reference
    @property
    def compress_method(self):
        return "raw" if self._raw is not None else ("tile_ans" if self._ans else "lattice_rans")

    @property
    def lossless(self):
        return self._raw is not None or self._ans

    @property
    def shape(self):
        return self._raw.shape if self._raw is not None else torch.Size(self._info.shape)

    @property
    def dtype(self):
        """dtype of the reconstructed tensor"""
        return self._dtype

    @property
    def encoded_dtype(self):
        if self._raw is not None:
            return self._raw.dtype
        return self._info.torch_dtype if self._ans else self._info.dtype

    @property
    def device(self):
        return (self._raw if self._raw is not None else self._blob).device

    @property
    def info(self):
        return self._info

    @property
    def blob(self):
        return self._blob

    def storage_nbytes(self, include_header=True):
        if self._raw is not None:
            return self._raw.numel() * _ELT[self._raw.dtype]
        header = 64 if self._ans else self._info.header_nbytes
        return self._info.storage_nbytes - (0 if include_header else header)

    @property
    def actual_bpp(self):
        """8 * storage_nbytes() / number of elements (API reference, CompressedTensor)"""
        return 8.0 * self.storage_nbytes() / math.prod(self.shape)

    # ---- methods of the API reference
    def to(self, device=None, dtype=None, copy=False):
        """another device and / or output dtype, without recompression.  A float container
        decodes to BF16, FP16 or FP32; a code container to its own dtype only."""
        if isinstance(device, torch.dtype):
            device, dtype = None, device
        dtype = self._dtype if dtype is None else dtype
        if self._ans and dtype != self._dtype:
            raise B.EpError(-1, "a lossless Tile-ANS stream decodes to its own dtype only")
        if self._raw is None and not self._ans and dtype != self._dtype:
            if B.dtype_code(dtype) not in _allowed_out(self._info.container_dtype):
                raise B.EpError(-1, f"a {self._info.dtype} container does not decode to {dtype}")
        dev = self.device if device is None else torch.device(device)
        if self._raw is not None:
            raw = self._raw.to(dev, copy=copy)
            return CompressedTensor(raw=raw, out_dtype=dtype)
        blob = self._blob.to(dev, copy=copy)
        ct = CompressedTensor(blob, self._info, dtype, ans=self._ans)
        if blob.data_ptr() == self._blob.data_ptr():
            ct._work = self._work  # same device copy: the prepared tables stay valid
        return ct

    def state_dict(self, prefix=""):
        """tensors only, so that torch.load(..., weights_only=True) restores it"""
        method = _RAW if self._raw is not None else (_TILE_ANS if self._ans else _LATTICE)
        meta = torch.tensor([STATE_VERSION, method, _dtype_tag(self._dtype)], dtype=torch.int64)
        if self._raw is not None:
            return {prefix + "ep_meta": meta, prefix + "ep_raw": self._raw}
        return {prefix + "ep_meta": meta, prefix + "ep_stream": self._blob}

    @classmethod
    def from_state_dict(cls, state, prefix=""):
        meta = state[prefix + "ep_meta"].tolist()
        if meta[0] != STATE_VERSION:
            raise B.EpError(-6, f"state version {meta[0]}")
        out_dtype = _TAG_DTYPE[meta[2]]
        if meta[1] == _RAW:
            return cls(raw=state[prefix + "ep_raw"], out_dtype=out_dtype)
        blob = state[prefix + "ep_stream"]
        if blob.dtype != torch.uint8 or blob.dim() != 1:
            raise B.EpError(-6, "stream tensor")
        if meta[1] == _TILE_ANS:
            info = B.ans_stream_info(_host_view(blob))
            if blob.numel() != info.storage_nbytes:
                raise B.EpError(-6, "stream length")
            return cls(blob, info, out_dtype, ans=True)
        if meta[1] != _LATTICE:
            raise B.EpError(-6, f"method tag {meta[1]}")
        info = B.stream_info(_host_view(blob))
        if blob.numel() != info.storage_nbytes:
            raise B.EpError(-6, "stream length")
        return cls(blob, info, out_dtype)

    def decompress(self, stream=None, out=None, status=None):
        return decompress(self, stream=stream, out=out, status=status)

    def __repr__(self):
        return (f"CompressedTensor(shape={tuple(self.shape)}, dtype={self.dtype}, method={self.compress_method}, "
                f"actual_bpp={self.actual_bpp:.3f}, device={self.device})")


_DTYPE_TAG = {torch.bfloat16: 1, torch.float16: 2, torch.float32: 3, torch.int8: 4, torch.float8_e4m3fn: 5}
_TAG_DTYPE = {v: k for k, v in _DTYPE_TAG.items()}


def _dtype_tag(d):
    if d not in _DTYPE_TAG:
        raise B.EpError(-1, f"dtype {d}")
    return _DTYPE_TAG[d]


def _allowed_out(container):
    return (B.BF16, B.FP16, B.FP32) if container in (B.BF16, B.FP16, B.FP32) else (container,)


def _host_view(blob):
    """a host copy of the stream's header, row factors, tables and directory is all that the
    parser reads; the whole stream is copied for simplicity"""
    return blob.detach().to("cpu")


def compress(tensor, config):
    """compress(tensor, config) -> CompressedTensor on the tensor's device.
    LatticeRANSConfig: a non-empty, 2-D, finite BF16 / FP16 / FP32 tensor; if even the coarsest
    resolution exceeds the target, a warning says so and the tensor is kept uncompressed
    (compress_method == "raw").  TileANSConfig: any non-empty BF16 / FP16 / FP32 / INT8 / FP8 E4M3
    tensor of 1 to 8 dims, every bit kept (the host compressor encodes a copy of a CUDA tensor)."""
    if isinstance(config, TileANSConfig):
        blob = B.ans_compress(tensor, blocks_per_lane=config.blocks_per_lane, n_threads=config.n_threads)
        info = B.ans_stream_info(blob)
        return CompressedTensor(blob.to(tensor.device), info, tensor.dtype, ans=True)
    if not isinstance(config, LatticeRANSConfig):
        raise B.EpError(-1, "config must be a LatticeRANSConfig or a TileANSConfig")
    container = 0 if config.container is None else config.container
    layouts = {"rows": B.LAYOUT_ROWS, "gemm": B.LAYOUT_GEMM}
    if config.layout not in layouts:
        raise B.EpError(-1, f"layout must be 'rows' or 'gemm', not {config.layout!r}")
    layout = layouts[config.layout]
    try:
        if tensor.is_cuda:  # the GPU compressor writes the host compressor's bytes
            blob = B.compress_device(tensor, config.target_bpp, container=container,
                                     blocks_per_lane=config.blocks_per_lane, coding=config.coding, layout=layout)
        else:
            blob = B.compress(tensor, config.target_bpp, container=container,
                              blocks_per_lane=config.blocks_per_lane, n_threads=config.n_threads,
                              coding=config.coding, layout=layout)
    except B.EpError as e:
        if e.status != -4:  # EP_ERR_TARGET_UNREACHABLE
            raise
        warnings.warn(f"target_bpp {config.target_bpp} is below what the stream's metadata alone needs for "
                      f"shape {tuple(tensor.shape)}; the tensor is stored uncompressed (compress_method='raw')")
        return CompressedTensor(raw=tensor.detach().clone(), out_dtype=tensor.dtype)
    info = B.stream_info(blob.cpu() if blob.is_cuda else blob)
    # by default the output has the input's dtype; code containers decode to their codes
    out_dtype = tensor.dtype if B.CODE_OF.get(tensor.dtype) in _allowed_out(info.container_dtype) else info.dtype
    return CompressedTensor(blob.to(tensor.device), info, out_dtype)


def _tables(ct, stream):
    """slot tables for this device copy, prepared once; later decodes on other streams wait for them"""
    if ct._work is None:
        work = (B.ans_prepare if ct._ans else B.prepare)(ct._blob, ct._info, stream=stream)
        ev = torch.cuda.Event()
        ev.record(stream)
        ct._work = (work, ev)
    else:
        stream.wait_event(ct._work[1])
    return ct._work[0]


def decompress(compressed, config=None, stream=None, out=None, status=None):
    """decompress(compressed, config) -> tensor of compressed.shape and compressed.dtype on
    compressed.device.  A lattice stream is always decoded by the GPU kernel: a stream held in
    host memory is copied to the current CUDA device, decoded there and the weights copied back
    (ep_decompress_host); without a CUDA device that raises.  ``config`` carries only encoding
    settings here, so it is accepted and not used."""
    ct = compressed
    if ct._raw is not None:
        return ct._raw.to(dtype=ct.dtype, copy=True)
    if ct._ans:
        if not ct._blob.is_cuda:
            # the GPU decodes a host-resident stream: copy in, decode, copy back
            if not torch.cuda.is_available():
                raise B.EpError(-1, "decompress decodes on a CUDA device and none is available")
            dev = torch.device("cuda", torch.cuda.current_device())
            s = stream or torch.cuda.current_stream(dev)
            with torch.cuda.stream(s):
                d = ct._blob.to(dev, non_blocking=False)
                res = B.ans_decompress(d, ct._info, status=status, stream=s)
                host = res.to("cpu") if out is None else out.copy_(res)
            s.synchronize()
            return host
        s = stream or torch.cuda.current_stream(ct._blob.device)
        work = _tables(ct, s)
        return B.ans_decompress(ct._blob, ct._info, workspace=work, out=out, status=status, stream=s)
    if not ct._blob.is_cuda:
        if out is not None and out.is_cuda:
            raise B.EpError(-1, "the output of a host-resident stream is a host tensor")
        return B.decompress_host(ct._blob.contiguous(), ct._info, out=out, out_dtype=ct.dtype, status=status,
                                 stream=stream)
    s = stream or torch.cuda.current_stream(ct._blob.device)
    work = _tables(ct, s)
    return B.decompress(ct._blob, ct._info, workspace=work, out=out, status=status, stream=s, out_dtype=ct.dtype)
