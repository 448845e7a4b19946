"""The C-ABI library loads without a GPU and exports every function include/eptile.h
declares; the host-side calls (compressor, parser) behave as documented."""
import ctypes as C

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth


def test_exports_every_declared_symbol():
    names = B.declared_functions()
    assert set(names) == {"ep_compress_bound", "ep_compress_host", "ep_compress_device_scratch",
                          "ep_compress_device", "ep_stream_info", "ep_prepare", "ep_decompress",
                          "ep_decompress_noalloc", "ep_decompress_host_scratch", "ep_decompress_host",
                          "ep_ans_compress_bound", "ep_ans_compress_host", "ep_ans_stream_info",
                          "ep_ans_prepare", "ep_ans_decompress", "ep_linear_fused_workspace", "ep_linear_fused", "ep_linear_fused_plan",
                          "ep_status_string"}
    lib = B.lib()
    for n in names:
        assert hasattr(lib, n), n
    # the symbols are plain C (unmangled) in the shared object's dynamic table
    raw = C.CDLL(B.LIB_PATH)
    for n in names:
        assert C.cast(getattr(raw, n), C.c_void_p).value


def test_device_compress_rejects_bad_arguments_before_any_launch():
    cfg = B._config(4.0)
    L = B.lib()
    fake = 1 << 20
    n = C.c_size_t(0)
    need = L.ep_compress_device_scratch(64, 256, C.byref(cfg))
    assert need >= 64 * 256 * 9  # symbols (5 bytes per weight) and the code matrix (4)
    assert L.ep_compress_device_scratch(0, 256, C.byref(cfg)) == 0
    assert L.ep_compress_device(None, B.BF16, 64, 256, C.byref(cfg), fake, 1 << 20, C.byref(n), fake, need, None) == -1
    assert L.ep_compress_device(fake, B.BF16, 64, 256, C.byref(cfg), fake, 1 << 20, C.byref(n), None, need, None) == -1
    assert L.ep_compress_device(fake, B.INT8, 64, 256, C.byref(cfg), fake, 1 << 20, C.byref(n), fake, need, None) == -8
    assert L.ep_compress_device(fake, B.BF16, 64, 256, C.byref(cfg), fake, 1 << 20, C.byref(n), fake + 16, need,
                                None) == -1  # scratch not 256-byte aligned
    assert L.ep_compress_device(fake, B.BF16, 64, 256, C.byref(cfg), fake, 1 << 20, C.byref(n), fake, need - 1,
                                None) == -1  # scratch too small


def test_status_strings():
    lib = B.lib()
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8, 99):
        assert lib.ep_status_string(code)


def test_info_fields_and_storage():
    w = synth.gaussian(256, 256, 0.02, 0)
    blob = B.compress(w, 3.5)
    info = B.stream_info(blob)
    assert info.shape == (256, 256) and info.dtype == torch.bfloat16
    assert info.storage_nbytes == blob.numel()
    assert info.actual_bpp == 8.0 * blob.numel() / w.numel() <= 3.5  # "actual_bpp" of the API reference
    assert info.storage_nbytes_(include_header=False) == blob.numel() - 64
    assert info.out_nbytes == 2 * w.numel()
    assert info.workspace_nbytes == 7 * 2048 * 4  # the decoder's slot tables


def test_errors():
    w = synth.gaussian(8, 64, 0.02, 1)
    with pytest.raises(B.EpError) as e:
        bad = w.clone()
        bad[0, 0] = float("nan")
        B.compress(bad, 4.0)
    assert e.value.status == -2
    with pytest.raises(B.EpError) as e:
        B.compress(w, 12.0)
    assert e.value.status == -3
    with pytest.raises(B.EpError) as e:
        B.compress(w, 8.0, container="int8")
    assert e.value.status == -3
    with pytest.raises(B.EpError) as e:
        B.compress(w, 0.01)
    assert e.value.status == -4
    # 8 x 12 at 4 bpp: the padded rows' metadata alone is over the target
    with pytest.raises(B.EpError) as e:
        B.compress(synth.gaussian(8, 12, 0.02, 1), 4.0)
    assert e.value.status == -4
    assert B.stream_info(B.compress(synth.gaussian(64, 12, 0.02, 1), 11.0)).cols == 12
    with pytest.raises(B.EpError):
        B.compress(torch.zeros(0, 8), 4.0)
    with pytest.raises(B.EpError):
        B.stream_info(torch.zeros(10, dtype=torch.uint8))


def test_coding_option_checked():
    w = synth.gaussian(64, 256, 0.02, 7)
    for bad in (-1, 3):
        with pytest.raises(B.EpError) as e:
            B.compress(w, 4.0, coding=bad)
        assert e.value.status == -1
    # the three codings decode to the same plan shape; paired streams need more table memory
    infos = [B.stream_info(B.compress(w, 4.0, coding=c)) for c in (0, 1, 2)]
    assert [i.paired for i in infos] == [0, 0, 1]
    assert infos[1].workspace_nbytes == 57344 and infos[2].workspace_nbytes == 108544


def test_malformed_paired_streams_rejected(oracle):
    """the library parser refuses what the oracle's parser refuses in a paired stream"""
    w = synth.row_lognormal(64, 512, 9)
    blob = B.compress(w, 4.0, coding=B.CODING_PAIRED)
    info = B.stream_info(blob)
    assert info.paired == 1
    q = info.off_freq + 2 * info.ntok[0]
    for off, val in ((43, 2), (39, 8), (43, 0), (q, None)):
        bad = blob.clone()
        bad[off] = (int(bad[off]) ^ 1) if val is None else val
        with pytest.raises(B.EpError) as e:
            B.stream_info(bad)
        assert e.value.status == -6, off
        assert oracle.parse(bad.numpy())[0] == oracle.ERR_CORRUPT


def test_corrupt_streams_rejected():
    w = synth.gaussian(64, 512, 0.02, 2)
    blob = B.compress(w, 4.0)
    info = B.stream_info(blob)
    with pytest.raises(B.EpError):
        B.stream_info(blob[:-16])
    # (a moved inner directory entry passes the parser; the decoder flags it)
    for off in (0, 4, 7, 34, info.off_freq, info.off_dir):
        bad = blob.clone()
        bad[off] ^= 0x5A
        with pytest.raises(B.EpError) as e:
            B.stream_info(bad)
        assert e.value.status == -6, off


def test_decompress_needs_device_memory():
    blob = B.compress(synth.gaussian(16, 64, 0.02, 3), 11.0, q_index=600)
    with pytest.raises(B.EpError):
        B.decompress(blob)


def test_compress_bound_holds():
    w = synth.gaussian(64, 256, 0.02, 4)
    for target in (0.5, 2.0, 4.0, 8.0):
        cfg = B._config(target)
        bound = B.lib().ep_compress_bound(64, 256, C.byref(cfg))
        try:
            blob = B.compress(w, target)
        except B.EpError:
            continue
        assert blob.numel() <= bound
    cfg = B._config(4.0, q_index=900)
    assert B.compress(w, 4.0, q_index=900).numel() <= B.lib().ep_compress_bound(64, 256, C.byref(cfg))


def test_decode_calls_reject_bad_arguments_before_any_launch():
    """argument checks of ep_prepare / ep_decompress / ep_decompress_noalloc happen on the host and
    need no device: null pointers, misaligned pointers, a container the stream does not hold, a
    damaged plan"""
    blob = B.compress(synth.gaussian(16, 64, 0.02, 5), 4.0)
    info = B.stream_info(blob)
    L = B.lib()
    fake, odd = 1 << 20, (1 << 20) + 8  # never dereferenced: every call below fails its checks first
    assert L.ep_prepare(None, fake, fake, None, None) == -1
    assert L.ep_prepare(C.byref(info), None, fake, None, None) == -1
    assert L.ep_prepare(C.byref(info), fake, None, None, None) == -1
    assert L.ep_prepare(C.byref(info), odd, fake, None, None) == -1
    assert L.ep_decompress(C.byref(info), fake, None, fake, info.container_dtype, None, None) == -1
    assert L.ep_decompress(C.byref(info), fake, fake, None, info.container_dtype, None, None) == -1
    assert L.ep_decompress(C.byref(info), fake, odd, fake, info.container_dtype, None, None) == -1
    assert L.ep_decompress(C.byref(info), fake, fake, odd, info.container_dtype, None, None) == -1
    assert L.ep_decompress(C.byref(info), fake, fake, fake, B.INT8, None, None) == -1  # a BF16 stream
    assert L.ep_decompress(C.byref(info), fake, fake, fake, 99, None, None) == -1
    assert L.ep_decompress_noalloc(None, fake, fake, info.container_dtype, None, None) == -1
    assert L.ep_decompress_noalloc(C.byref(info), fake, fake, B.INT8, None, None) == -1
    codes = B.stream_info(B.compress(synth.gaussian(64, 256, 0.02, 5), 6.0, container=B.INT8))
    for dt in (B.BF16, B.FP16, B.FP32, B.FP8E4M3):  # code containers decode to their own dtype only
        assert L.ep_decompress(C.byref(codes), fake, fake, fake, dt, None, None) == -1
    bad = B.StreamInfo.from_buffer_copy(info)
    bad.split[3] = 12  # beyond the largest split of its context
    assert L.ep_decompress(C.byref(bad), fake, fake, fake, info.container_dtype, None, None) == -6
    assert L.ep_prepare(C.byref(bad), fake, fake, None, None) == -6
    bad = B.StreamInfo.from_buffer_copy(info)
    bad.cols = 0
    assert L.ep_decompress(C.byref(bad), fake, fake, fake, info.container_dtype, None, None) == -1
    # a paired plan: alphabets above 256 tokens, splits beyond the narrow range, an unknown coding
    paired = B.stream_info(B.compress(synth.row_lognormal(64, 512, 5), 4.0, coding=B.CODING_PAIRED))
    assert paired.paired == 1
    for field, idx, val in (("ntok", 1, 300), ("split", 4, 8), ("paired", None, 2)):
        bad = B.StreamInfo.from_buffer_copy(paired)
        if idx is None:
            setattr(bad, field, val)
        else:
            getattr(bad, field)[idx] = val
        assert L.ep_decompress(C.byref(bad), fake, fake, fake, bad.container_dtype, None, None) == -6, field
        assert L.ep_prepare(C.byref(bad), fake, fake, None, None) == -6, field


def test_host_buffer_decode_checks_arguments_before_any_copy():
    """ep_decompress_host_scratch sums the 256-byte rounded stream, tables and output; the call
    rejects null pointers, misaligned or short scratch and an output dtype the stream cannot
    decode to, on the host"""
    blob = B.compress(synth.gaussian(40, 100, 0.02, 6), 4.0)
    info = B.stream_info(blob)
    L = B.lib()
    r = lambda n: (n + 255) // 256 * 256
    assert L.ep_decompress_host_scratch(C.byref(info), B.BF16) == \
        r(info.storage_nbytes) + r(info.workspace_nbytes) + r(40 * 100 * 2)
    assert L.ep_decompress_host_scratch(C.byref(info), B.FP32) == \
        r(info.storage_nbytes) + r(info.workspace_nbytes) + r(40 * 100 * 4)
    assert L.ep_decompress_host_scratch(C.byref(info), B.INT8) == 0
    assert L.ep_decompress_host_scratch(None, B.BF16) == 0
    need = L.ep_decompress_host_scratch(C.byref(info), info.container_dtype)
    fake = 1 << 20  # never dereferenced: every call below fails its checks first
    h = blob.data_ptr()
    dt = info.container_dtype
    assert L.ep_decompress_host(None, h, fake, dt, fake, need, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), None, fake, dt, fake, need, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), h, None, dt, fake, need, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), h, fake, dt, None, need, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), h, fake, dt, fake + 16, need, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), h, fake, dt, fake, need - 1, None, None) == -1
    assert L.ep_decompress_host(C.byref(info), h, fake, B.INT8, fake, need, None, None) == -1
    bad = B.StreamInfo.from_buffer_copy(info)
    bad.split[3] = 12
    assert L.ep_decompress_host(C.byref(bad), h, fake, dt, fake, need, None, None) == -6


def test_huge_header_shapes_rejected_without_overflow():
    """rows and cols near the parser's 2^40 bound make rows * cols overflow 64 bits: the parser
    refuses such headers as corrupt before it forms any product"""
    import struct
    blob = B.compress(synth.gaussian(64, 512, 0.02, 2), 4.0)
    for rows, cols in [((1 << 40) - 1, (1 << 40) - 1), ((1 << 39), (1 << 30)), ((1 << 35), (1 << 36))]:
        bad = bytearray(blob.numpy().tobytes())
        struct.pack_into("<qq", bad, 8, rows, cols)
        with pytest.raises(B.EpError) as e:
            B.stream_info(torch.frombuffer(bad, dtype=torch.uint8))
        assert e.value.status == -6, (rows, cols)
