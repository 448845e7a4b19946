"""GPU parity: the sm_100a decode, called through the C ABI, against the oracle's decode of
the same stream -- bit-exact on the lattice points and on the container bytes, for every
container, ragged tails, every rate regime and damaged streams.  Streams here come from the
ORACLE's encoder, so no expected value depends on the product library."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

pytestmark = pytest.mark.gpu

TORCH_OF = {B.BF16: torch.bfloat16, B.FP16: torch.float16, B.FP32: torch.float32, B.INT8: torch.int8,
            B.FP8E4M3: torch.float8_e4m3fn}


def as_bytes(t):
    return t.contiguous().view(torch.uint8).cpu().numpy().reshape(-1)


def gpu_decode(blob_np, lattice=False, stream=None):
    blob = torch.from_numpy(np.ascontiguousarray(blob_np))
    info = B.stream_info(blob)
    d = blob.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = B.decompress(d, info, status=status, lattice=lattice, stream=stream)
    torch.cuda.synchronize()
    return info, out, int(status.item())


def check_parity(oracle, blob_np):
    rc, st, v_ref, out_ref = oracle.decode(blob_np)
    assert rc == 0 and st == 0
    info, out, status = gpu_decode(blob_np)
    assert status == 0
    assert out.dtype == TORCH_OF[info.container_dtype] and tuple(out.shape) == info.shape
    assert np.array_equal(as_bytes(out), out_ref.view(np.uint8).reshape(-1))
    _, v, status = gpu_decode(blob_np, lattice=True)
    assert status == 0
    assert np.array_equal(v.cpu().numpy(), v_ref)
    return info, out


def test_readme_example(oracle):
    """256x256 BF16 N(0, 0.02^2) at 3.5 bpp, the README's quick start: shape and dtype come
    back, stored rate at most the target"""
    w = synth.gaussian(256, 256, 0.02, 0)
    rc, blob = oracle.compress(w, 3.5)
    info, out = check_parity(oracle, blob)
    assert out.shape == w.shape and out.dtype == w.dtype and info.actual_bpp <= 3.5


@pytest.mark.parametrize("container", [B.BF16, B.FP16, B.FP32, B.INT8, B.FP8E4M3])
@pytest.mark.parametrize("shape,K", [((1, 8), 0), ((3, 24), 1), ((5, 40), 3), ((17, 64), 7), ((33, 512), 0),
                                     ((100, 808), 0), ((64, 1024), 16), ((300, 2048), 2),
                                     # rows zero-padded to whole E8 blocks (cols % 8 != 0)
                                     ((1, 1), 0), ((7, 13), 1), ((33, 255), 0), ((64, 1001), 2), ((5, 3), 0)])
def test_ragged_shapes_all_containers(oracle, container, shape, K):
    src_dtype = torch.float16 if container == B.FP16 else (torch.float32 if container == B.FP32 else torch.bfloat16)
    w = synth.row_lognormal(*shape, seed=shape[0] + shape[1], dtype=src_dtype)
    rc, blob = oracle.compress(w, 7.0, container=container, blocks_per_lane=K, q_override=700)
    assert rc == 0
    check_parity(oracle, blob)


@pytest.mark.parametrize("target", [0.5, 1.0, 2.0, 3.5, 5.0, 8.0, 11.0])
def test_rates(oracle, target):
    """low rates (single-token contexts with a phantom token), mid rates, and high rates (many
    escape tokens whose raw extra bits come from the back of the lane's region)"""
    w = synth.gaussian_outliers(256, 4096, seed=11)
    rc, blob = oracle.compress(w, target)
    assert rc == 0
    check_parity(oracle, blob)


@pytest.mark.parametrize("container,target", [(B.INT8, 3.0), (B.FP8E4M3, 3.0), (B.INT8, 7.9), (B.FP8E4M3, 6.0)])
def test_code_containers(oracle, container, target):
    w = synth.gaussian(512, 1024, 0.02, 12)
    rc, blob = oracle.compress(w, target, container=container)
    assert rc == 0
    check_parity(oracle, blob)


def test_dit_layer_slice(oracle):
    w = synth.dit_layer(5, 0)[:1024]
    for target in (2.5, 4.0):
        rc, blob = oracle.compress(w, target)
        check_parity(oracle, blob)


def test_repeat_and_streams(oracle):
    """same bytes on repeat; two decodes in flight on two streams do not interfere"""
    w1 = synth.row_lognormal(512, 2048, 13)
    w2 = synth.gaussian(1024, 1024, 0.02, 14)
    rc, b1 = oracle.compress(w1, 4.0)
    rc, b2 = oracle.compress(w2, 2.0)
    _, _, _, r1 = oracle.decode(b1)
    _, _, _, r2 = oracle.decode(b2)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    d1 = torch.from_numpy(b1).cuda()
    d2 = torch.from_numpy(b2).cuda()
    torch.cuda.synchronize()
    i1, i2 = B.stream_info(torch.from_numpy(b1)), B.stream_info(torch.from_numpy(b2))
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            o1 = B.decompress(d1, i1, stream=s1)
        with torch.cuda.stream(s2):
            o2 = B.decompress(d2, i2, stream=s2)
        outs.append((o1, o2))
    torch.cuda.synchronize()
    for o1, o2 in outs:
        assert np.array_equal(as_bytes(o1), r1.view(np.uint8).reshape(-1))
        assert np.array_equal(as_bytes(o2), r2.view(np.uint8).reshape(-1))


@pytest.mark.parametrize("target", [4.0, 8.0])
def test_damaged_streams_flagged(oracle, target):
    """damage found on the device goes to the status word; the decode stays in bounds (narrow
    value fields at 4 bpp, wide ones at 8 bpp)"""
    w = synth.gaussian(256, 1024, 0.02, 15)
    rc, blob = oracle.compress(w, target)
    rc, info = oracle.parse(blob)
    host_info = B.stream_info(torch.from_numpy(blob))
    rng = np.random.default_rng(1)
    flagged = 0
    for trial in range(12):
        bad = blob.copy()
        pos = int(rng.integers(info.off_tiles + 128, blob.size - 16))
        bad[pos] ^= np.uint8(1 << int(rng.integers(0, 8)))
        d = torch.from_numpy(bad).cuda()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.decompress(d, host_info, status=status)
        torch.cuda.synchronize()
        rc, st_or, _, _ = oracle.decode(bad)
        flagged += int(status.item()) != 0
        assert (int(status.item()) != 0) == (st_or != 0)
    assert flagged >= 10
    # directory entries pointing outside the tile section, or shrinking tiles
    bad = blob.copy()
    bad[info.off_dir + 8: info.off_dir + 12] = np.frombuffer(np.uint32(0xFFFFFFF0).tobytes(), np.uint8)
    bad[info.off_dir + 4: info.off_dir + 8] = np.frombuffer(np.uint32(3).tobytes(), np.uint8)
    d = torch.from_numpy(bad).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.decompress(d, host_info, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 16  # EP_DEC_BAD_TILE
    # frequency tables that no longer sum to 2^11 (device copy differs from the parsed one)
    bad = blob.copy()
    bad[info.off_freq] ^= np.uint8(0x40)
    d = torch.from_numpy(bad).cuda()
    status.zero_()
    B.decompress(d, host_info, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) != 0


@pytest.mark.parametrize("K,q", [(64, 900), (256, 760), (128, 1000), (1024, 900)])
def test_large_tiles(oracle, K, q):
    """tiles of tens of KB take fewer warps per CTA (their buffers fill shared memory); tiles
    beyond every buffer (K = 1024 at ~8 bits, ~260 KB) are decoded in place from global memory"""
    w = synth.gaussian_outliers(96, 4096, seed=K) if K < 1024 else synth.gaussian_outliers(128, 16384, seed=K)
    rc, blob = oracle.compress(w, 11.0, blocks_per_lane=K, q_override=q)
    assert rc == 0
    rc, info = oracle.parse(blob)
    sizes = np.diff(np.frombuffer(blob[info.off_dir: info.off_dir + 4 * (info.n_tiles + 1)].tobytes(), np.uint32))
    assert (16 * sizes > 6144).any()
    if K == 1024:
        assert (16 * sizes > 232448).any()
    check_parity(oracle, blob)


def _expected_tables(oracle, blob_np):
    """the decoder's slot tables as include/eptile.h documents them, from the oracle's parse of
    the stream: per context 2048 entries f << 21 | escape << 20 | field << 11 | (slot - cum);
    field = v + 256 for a direct token (v its lattice coordinate), the escape index d (2d + c for
    coordinates 1..6) otherwise; context 3 + 2c + p stored at position 3 + c + 2p.  When a split
    is beyond the narrow range (8 for contexts 1, 2, 7 for contexts 3..6) the tables are wide:
    coordinates 1..7 store y = (v - c) / 2 + 256 and escape index d"""
    rc, info = oracle.parse(blob_np)
    assert rc == 0
    wide = any(info.split[c] > m for c, m in enumerate((9, 8, 8, 7, 7, 7, 7)))
    b = blob_np.tobytes()
    tab = np.zeros((7, 2048), np.uint32)
    off = info.off_freq
    for ctx in range(7):
        n, m = info.ntok[ctx], info.split[ctx]
        f = np.frombuffer(b, np.uint16, count=n, offset=off).astype(np.int64)
        off += 2 * n
        pos = ctx if ctx < 3 else 3 + ((ctx - 3) >> 1) + 2 * ((ctx - 3) & 1)
        cum = 0
        for t in range(n):
            if t < (1 << m):
                if ctx == 0:
                    v = 4 * oracle.unzigzag(t >> 2) + (t & 3)
                elif ctx < 3:
                    y = 2 * oracle.unzigzag(t >> 1) + (t & 1)
                    v = y if wide else 2 * y + (ctx - 1)
                else:
                    y = 2 * oracle.unzigzag(t) + ((ctx - 3) & 1)
                    v = y if wide else 2 * y + ((ctx - 3) >> 1)
                head = (int(f[t]) << 21) | (((v + 256) & 0x1FF) << 11)
            else:
                d = t - (1 << m)
                fv = 2 * d + (ctx - 1) if ctx in (1, 2) and not wide else d
                head = (int(f[t]) << 21) | (1 << 20) | ((fv & 0x1FF) << 11)
            for s in range(cum, cum + int(f[t])):
                tab[pos, s] = head | (s - cum)
            cum += int(f[t])
    return tab


@pytest.mark.parametrize("target,container", [(4.0, 0), (0.5, 0), (8.0, 0), (11.0, 0), (3.0, B.INT8)])
def test_prepared_tables_match_documented_layout(oracle, target, container):
    w = synth.gaussian_outliers(128, 2048, seed=16)
    rc, blob = oracle.compress(w, target, container=container)
    assert rc == 0
    if target == 11.0:  # the wide layout is exercised
        rc, info = oracle.parse(blob)
        assert any(info.split[c] > m for c, m in enumerate((9, 8, 8, 7, 7, 7, 7)))
    d = torch.from_numpy(blob).cuda()
    info = B.stream_info(torch.from_numpy(blob))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    work = B.prepare(d, info, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = work.cpu().numpy().view(np.uint32).reshape(7, 2048)
    assert np.array_equal(got, _expected_tables(oracle, blob))
