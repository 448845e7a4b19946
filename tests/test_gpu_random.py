"""Seeded random sweep of GPU parity: shapes (ragged rows included), rates, containers, forced tile
sizes, output dtypes and (every third case) paired coding drawn from a fixed generator; every case is encoded by the ORACLE and the
GPU decode must equal the oracle's decode byte for byte (lattice points and container bytes), and
the GPU compressor must write the oracle's stream for the same tensor."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

pytestmark = pytest.mark.gpu

CONTAINERS = [B.BF16, B.FP16, B.FP32, B.INT8, B.FP8E4M3]
SRC = {B.BF16: torch.bfloat16, B.FP16: torch.float16, B.FP32: torch.float32, B.INT8: torch.bfloat16,
       B.FP8E4M3: torch.bfloat16}


def cases(n=40, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        rows = int(rng.integers(1, 300))
        cols = int(rng.choice([int(rng.integers(1, 64)), int(rng.integers(64, 2100)), 8 * int(rng.integers(1, 260))]))
        container = CONTAINERS[int(rng.integers(0, len(CONTAINERS)))]
        hi = 7.9 if container in (B.INT8, B.FP8E4M3) else 11.0
        target = float(np.round(rng.uniform(0.3, hi), 2))
        K = int(rng.choice([0, 0, 1, 2, 3, 8, 16, 64]))
        out.append((i, rows, cols, container, target, K, 2 if i % 3 == 1 else 0))
    return out


@pytest.mark.parametrize("i,rows,cols,container,target,K,coding", cases(), ids=lambda v: str(v))
def test_random_case(oracle, i, rows, cols, container, target, K, coding):
    w = synth.row_lognormal(rows, cols, seed=1000 + i, dtype=SRC[container])
    if i % 3 == 0:
        w = synth.gaussian_outliers(rows, cols, seed=1000 + i, dtype=SRC[container])
    rc, blob = oracle.compress(w, target, container=container, blocks_per_lane=K, coding=coding)
    if rc == oracle.ERR_TARGET_UNREACHABLE:
        with pytest.raises(B.EpError):
            B.compress_device(w.cuda(), target, container=container, blocks_per_lane=K, coding=coding)
        return
    assert rc == 0
    # the GPU compressor writes the same stream
    got = B.compress_device(w.cuda(), target, container=container, blocks_per_lane=K, coding=coding).cpu().numpy()
    assert np.array_equal(got, blob)
    # the GPU decode equals the oracle's, for the container and the lattice points
    d = torch.from_numpy(blob).cuda()
    info = B.stream_info(torch.from_numpy(blob))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = B.decompress(d, info, status=status)
    lat = B.decompress(d, info, status=status, lattice=True)
    rc, st, v_ref, out_ref = oracle.decode(blob)
    torch.cuda.synchronize()
    assert rc == 0 and st == 0 and int(status.item()) == 0
    assert np.array_equal(out.contiguous().view(torch.uint8).cpu().numpy().reshape(-1),
                          out_ref.view(np.uint8).reshape(-1))
    assert np.array_equal(lat.cpu().numpy(), v_ref)
    if container in (B.BF16, B.FP16, B.FP32):  # and an output dtype change
        other = {B.BF16: B.FP32, B.FP16: B.BF16, B.FP32: B.FP16}[container]
        got2 = B.decompress(d, info, out_dtype=other)
        rc, st, _, ref2 = oracle.decode(blob, out_dtype=other)
        assert np.array_equal(got2.contiguous().view(torch.uint8).cpu().numpy().reshape(-1),
                              ref2.view(np.uint8).reshape(-1))
