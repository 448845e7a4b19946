"""Pins for the oracle's output dtype change (CompressedTensor.to(dtype=...) of the API reference:
the output dtype changes without recompression).  Reading: the fp32 weight w = fp32(f_r v) is
rounded once into the requested float dtype.  Checked against library routines, not against the
oracle itself: numpy's float32 multiply gives w from the decoded lattice points and the stored
row factors, torch's and numpy's round-to-nearest-even casts give BF16 and FP16 from w."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import synth

BF16, FP16, FP32, INT8, FP8 = 1, 2, 3, 4, 5
SRC = {BF16: torch.bfloat16, FP16: torch.float16, FP32: torch.float32}


def row_factors(blob, info):
    return np.frombuffer(blob.tobytes(), np.float32, count=info.rows, offset=info.off_rowf)


@pytest.mark.parametrize("container", [BF16, FP16, FP32])
def test_float_containers_decode_to_every_float_dtype(oracle, container):
    w = synth.row_lognormal(40, 96, seed=container, dtype=SRC[container])
    rc, blob = oracle.compress(w, 4.0)
    assert rc == 0
    rc, info = oracle.parse(blob)
    fr = row_factors(blob, info)
    rc, st, v, w32 = oracle.decode(blob, out_dtype=FP32)
    assert rc == 0 and st == 0 and w32.dtype == np.float32
    # w = fp32(f_r v), one correctly rounded multiply (v is exact in fp32)
    assert np.array_equal(w32, fr[:, None] * v.astype(np.float32))
    rc, st, _, wb = oracle.decode(blob, out_dtype=BF16)
    ref_b = torch.from_numpy(w32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert rc == 0 and np.array_equal(wb, ref_b)
    rc, st, _, wh = oracle.decode(blob, out_dtype=FP16)
    assert rc == 0 and np.array_equal(wh, w32.astype(np.float16).view(np.uint16))
    # the container's own dtype is the default
    rc, st, _, wc = oracle.decode(blob)
    _, _, _, wsame = oracle.decode(blob, out_dtype=container)
    assert np.array_equal(wc, wsame)


@pytest.mark.parametrize("container", [INT8, FP8])
def test_code_containers_decode_to_their_own_dtype_only(oracle, container):
    w = synth.gaussian(64, 256, 0.02, 7)
    rc, blob = oracle.compress(w, 5.0, container=container)
    assert rc == 0
    for dt in (BF16, FP16, FP32, INT8, FP8):
        rc, st, _, out = oracle.decode(blob, out_dtype=dt)
        assert (rc == 0) == (dt == container)
