"""The library's Tile-ANS lossless scheme ("EntroPack README", Configuration: TileANSConfig;
"EntroPack API reference", decompress restores every bit of a lossless scheme's input).

Host side (no GPU): the host compressor writes the oracle's bytes for every dtype, ragged element
counts, tile sizes and shapes; the parser reads the oracle's layout; bad arguments and damaged
streams are refused before anything runs.  GPU side (marked gpu): the sm_100a decode returns the
input bit for bit, for streams of the host compressor, damaged streams set status bits, and the
sizes span several tiles, a ragged last chunk and partial last tiles."""
import ctypes as C

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth


def bits(t):
    t = t.contiguous()
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy()
    if t.element_size() == 2:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.int32).numpy().view(np.uint32)


def tensors():
    g = torch.Generator().manual_seed(11)
    yield "bf16 lognormal", synth.row_lognormal(257, 1000, seed=12)
    yield "fp16 gaussian", synth.gaussian(64, 777, 0.02, seed=13).to(torch.float16)
    yield "fp32 student-t", synth.dit_layer(2, 1)[:40, :999].float().contiguous()
    yield "int8 codes", torch.clamp(torch.round(torch.randn(123, 457, generator=g) * 30), -127, 127).to(torch.int8)
    yield "fp8 codes", (torch.randn(99, 321, generator=g) * 40).to(torch.float8_e4m3fn)
    yield "bf16 all patterns", torch.from_numpy(np.arange(65536, dtype=np.int32).astype(np.int16)).view(torch.bfloat16)
    yield "fp32 random bits", torch.from_numpy(
        np.random.default_rng(14).integers(0, 2 ** 32, size=(3, 5, 1001), dtype=np.uint64).astype(np.uint32)
        .view(np.int32)).view(torch.float32)
    yield "bf16 one element", torch.tensor([-0.0], dtype=torch.bfloat16)
    yield "int8 constant", torch.full((3000,), 7, dtype=torch.int8)


@pytest.mark.parametrize("K", [0, 1, 5])
def test_host_bytes_equal_oracle(oracle, K):
    for name, t in tensors():
        blob = B.ans_compress(t, blocks_per_lane=K)
        rc, ref = oracle.ta_compress(bits(t), B.CODE_OF[t.dtype], shape=tuple(t.shape), blocks_per_lane=K)
        assert rc == 0 and np.array_equal(blob.numpy(), ref), (name, K)
        info = B.ans_stream_info(blob)
        rc, oi = oracle.ta_parse(ref)
        assert info.shape == tuple(t.shape) and info.dtype == B.CODE_OF[t.dtype]
        assert (info.n_tiles, info.blocks_per_lane, info.off_raw, info.off_tiles) == \
            (oi.n_tiles, oi.blocks_per_lane, oi.off_raw, oi.off_tiles)
        assert info.storage_nbytes == blob.numel() and info.out_nbytes == t.numel() * t.element_size()
        assert info.ratio == pytest.approx(blob.numel() / info.out_nbytes)


def test_threads_do_not_change_bytes():
    t = synth.row_lognormal(512, 2048, seed=15)
    one = B.ans_compress(t, n_threads=1)
    assert np.array_equal(one.numpy(), B.ans_compress(t, n_threads=7).numpy())


def test_ratio_on_weights():
    """the coded top bytes of Gaussian-like BF16 weights take about 3 bits: ~69 % of the input"""
    info = B.ans_stream_info(B.ans_compress(synth.row_lognormal(1024, 1024, seed=16)))
    assert 0.66 < info.ratio < 0.72


def test_bad_arguments_and_damage():
    L = B.lib()
    t = synth.gaussian(64, 256, 0.02, seed=17)
    src = bits(t)
    n = C.c_size_t(0)
    dims = (C.c_int64 * 8)(64, 256)
    cfg = B.AnsConfig(B.BF16, 0, 0, 0)
    out = np.zeros(L.ep_ans_compress_bound(src.size, B.BF16), np.uint8)
    p = lambda a: a.ctypes.data_as(C.c_void_p)
    assert L.ep_ans_compress_host(None, src.size, 2, dims, C.byref(cfg), p(out), out.size, C.byref(n)) == -1
    assert L.ep_ans_compress_host(p(src), src.size, 0, dims, C.byref(cfg), p(out), out.size, C.byref(n)) == -1
    bad_dims = (C.c_int64 * 8)(64, 255)
    assert L.ep_ans_compress_host(p(src), src.size, 2, bad_dims, C.byref(cfg), p(out), out.size, C.byref(n)) == -1
    bad_cfg = B.AnsConfig(6, 0, 0, 0)
    assert L.ep_ans_compress_host(p(src), src.size, 2, dims, C.byref(bad_cfg), p(out), out.size, C.byref(n)) == -1
    assert L.ep_ans_compress_host(p(src), src.size, 2, dims, C.byref(cfg), p(out), 100, C.byref(n)) == -5
    assert n.value > 100
    assert L.ep_ans_compress_bound(0, B.BF16) == 0 and L.ep_ans_compress_bound(10, 9) == 0
    blob = B.ans_compress(t)
    assert L.ep_ans_compress_bound(t.numel(), B.BF16) >= blob.numel()
    info = B.ans_stream_info(blob)
    with pytest.raises(B.EpError) as e:
        B.ans_stream_info(blob[:-16])
    assert e.value.status == -6
    for off in (0, 4, 6, 7, 24, info.off_freq + 2 * 0x3c, info.off_dir + 4 * info.n_tiles):
        bad = blob.clone()
        bad[off] ^= 0x5A
        with pytest.raises(B.EpError) as e:
            B.ans_stream_info(bad)
        assert e.value.status == -6, off


def test_decode_calls_check_arguments_before_any_launch():
    """null or misaligned pointers and an info that no parse produced are refused on the host"""
    L = B.lib()
    blob = B.ans_compress(synth.gaussian(8, 64, 0.02, seed=20))
    info = B.ans_stream_info(blob)
    fake = C.c_void_p(1 << 20)  # never dereferenced: every call below returns before a launch
    odd = C.c_void_p((1 << 20) + 8)
    assert L.ep_ans_prepare(None, fake, fake, None, None) == -1
    assert L.ep_ans_prepare(C.byref(info), None, fake, None, None) == -1
    assert L.ep_ans_prepare(C.byref(info), odd, fake, None, None) == -1
    assert L.ep_ans_decompress(C.byref(info), fake, fake, None, None, None) == -1
    assert L.ep_ans_decompress(C.byref(info), fake, odd, fake, None, None) == -1
    bad = B.AnsInfo.from_buffer_copy(info)
    bad.dtype = 9
    assert L.ep_ans_decompress(C.byref(bad), fake, fake, fake, None, None) == -6
    bad = B.AnsInfo.from_buffer_copy(info)
    bad.workspace_nbytes = 100
    assert L.ep_ans_prepare(C.byref(bad), fake, fake, None, None) == -1


def test_decode_needs_device_memory():
    blob = B.ans_compress(synth.gaussian(8, 64, 0.02, seed=18))
    with pytest.raises(B.EpError):
        B.ans_decompress(blob, B.ans_stream_info(blob))


# ---------------------------------------------------------------- GPU parity
def gpu_decode(blob, info):
    d = blob.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    work = B.ans_prepare(d, info, status=status)
    out = B.ans_decompress(d, info, workspace=work, status=status)
    torch.cuda.synchronize()
    return out, int(status.item())


@pytest.mark.gpu
@pytest.mark.parametrize("K", [0, 1, 5])
def test_gpu_decode_bit_exact(K):
    for name, t in tensors():
        blob = B.ans_compress(t, blocks_per_lane=K)
        info = B.ans_stream_info(blob)
        out, st = gpu_decode(blob, info)
        assert st == 0, name
        assert out.dtype == t.dtype and tuple(out.shape) == tuple(t.shape), name
        assert np.array_equal(bits(out.cpu()), bits(t)), (name, K)


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 7, 8, 9, 4095, 8192 * 32 - 3, 8192 * 32 + 11, 3 * 1024 * 1024 + 5])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32, torch.int8])
def test_gpu_ragged_and_many_tiles(n, dtype):
    g = torch.Generator().manual_seed(n)
    t = (torch.randn(n, generator=g) * (30 if dtype == torch.int8 else 0.02)).to(dtype)
    blob = B.ans_compress(t)
    info = B.ans_stream_info(blob)
    out, st = gpu_decode(blob, info)
    assert st == 0 and np.array_equal(bits(out.cpu()), bits(t))


@pytest.mark.gpu
def test_gpu_damaged_tiles_flagged(oracle):
    t = synth.row_lognormal(256, 1024, seed=19)
    blob = B.ans_compress(t)
    info = B.ans_stream_info(blob)
    import struct
    b = blob.numpy().tobytes()
    for tile in (0, info.n_tiles // 2, info.n_tiles - 1):
        bad = blob.clone()
        off = info.off_tiles + 16 * struct.unpack_from("<I", b, info.off_dir + 4 * tile)[0] + 192 + 40
        bad[off] ^= 0x40
        out, st = gpu_decode(bad, info)
        rc, ost, _ = oracle.ta_decode(bad.numpy())
        assert (st != 0) == (ost != 0) and st != 0, tile
