"""The library's multithreaded host compressor writes exactly the oracle's bytes, and its
parser reads exactly the oracle's plan.  The two encoders share no code: agreement byte for
byte pins the product encoder to the oracle (and so to the oracle's own pins)."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

CASES = [
    ("readme_256", lambda: synth.gaussian(256, 256, 0.02, 0), 3.5, 0, 0),
    ("lognormal_1024", lambda: synth.row_lognormal(1024, 1024, 1), 4.0, 0, 0),
    ("int8", lambda: synth.gaussian(256, 512, 0.02, 2), 3.0, B.INT8, 0),
    ("fp8", lambda: synth.gaussian(256, 512, 0.02, 2), 3.0, B.FP8E4M3, 0),
    ("int8_high", lambda: synth.gaussian(128, 512, 0.02, 2), 7.9, B.INT8, 0),
    ("outlier_0.5", lambda: synth.gaussian_outliers(256, 2048, 3), 0.5, 0, 0),
    ("outlier_8", lambda: synth.gaussian_outliers(256, 2048, 3), 8.0, 0, 0),
    ("outlier_11", lambda: synth.gaussian_outliers(64, 2048, 3), 11.0, 0, 0),
    ("fp16_src", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float16), 4.0, 0, 0),
    ("fp32_src", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float32), 5.0, 0, 0),
    ("fp32_to_bf16", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float32), 5.0, B.BF16, 0),
    ("dit_out_rows", lambda: synth.dit_layer(3, 1)[:512], 2.5, 0, 0),
    ("K1", lambda: synth.gaussian(40, 256, 0.02, 5), 11.0, 0, 1),
    ("K5", lambda: synth.gaussian(40, 256, 0.02, 5), 8.0, 0, 5),
    ("zero_rows", lambda: torch.cat([synth.gaussian(30, 512, 0.02, 6), torch.zeros(2, 512, dtype=torch.bfloat16)]),
     4.0, 0, 0),
    # rows zero-padded to whole E8 blocks (cols % 8 != 0)
    ("ragged_1001", lambda: synth.row_lognormal(96, 1001, 3), 4.0, 0, 0),
    ("ragged_int8", lambda: synth.gaussian(64, 523, 0.02, 4), 3.0, B.INT8, 0),
    ("ragged_K3", lambda: synth.row_lognormal(33, 13, 5, dtype=torch.float32), 9.0, 0, 3),
]


PAIRED_CASES = [
    ("paired_lognormal", lambda: synth.row_lognormal(300, 1000, 7), 3.0, 0, 0),
    ("paired_outliers", lambda: synth.gaussian_outliers(96, 2048, 2), 3.5, 0, 0),
    ("paired_outliers_low", lambda: synth.gaussian_outliers(96, 2048, 4), 2.0, 0, 0),
    ("paired_ragged_K3", lambda: synth.row_lognormal(137, 455, 5), 3.5, 0, 3),
    ("paired_int8", lambda: synth.gaussian(96, 808, 0.02, 3), 4.0, B.INT8, 0),
    ("paired_fp8", lambda: synth.gaussian(256, 512, 0.02, 2), 3.0, B.FP8E4M3, 0),
]


@pytest.mark.parametrize("name,make,target,container,K", PAIRED_CASES, ids=[c[0] for c in PAIRED_CASES])
def test_paired_bytes_identical_to_oracle(oracle, name, make, target, container, K):
    """paired coding asked for at sizes below the automatic threshold"""
    w = make()
    rc, ref = oracle.compress(w, target, container=container, blocks_per_lane=K, coding=oracle.CODING_PAIRED)
    assert rc == 0
    assert oracle.parse(ref)[1].paired == 1
    blob = B.compress(w, target, container=container, blocks_per_lane=K, coding=B.CODING_PAIRED).numpy()
    assert np.array_equal(blob, ref)
    assert B.stream_info(torch.from_numpy(blob)).paired == 1


@pytest.mark.parametrize("name,make,target,container,K", CASES, ids=[c[0] for c in CASES])
def test_bytes_identical_to_oracle(oracle, name, make, target, container, K):
    w = make()
    rc, ref = oracle.compress(w, target, container=container, blocks_per_lane=K)
    assert rc == 0
    blob = B.compress(w, target, container=container, blocks_per_lane=K).numpy()
    assert blob.size == ref.size
    assert np.array_equal(blob, ref)


def test_fixed_resolution_identical(oracle):
    w = synth.gaussian(17, 64, 0.02, 7)
    for k in (0, 300, 640, 900, 1279):
        rc, ref = oracle.compress(w, 11.0, q_override=k)
        assert np.array_equal(B.compress(w, 11.0, q_index=k).numpy(), ref)


def test_thread_count_independent():
    w = synth.row_lognormal(512, 1024, 8)
    blobs = [B.compress(w, 3.0, n_threads=n).numpy() for n in (1, 3, 8)]
    assert all(np.array_equal(blobs[0], b) for b in blobs[1:])


def test_parse_matches_oracle(oracle):
    w = synth.gaussian(256, 512, 0.02, 9)
    for container, coding in ((0, 0), (B.INT8, 0), (0, B.CODING_PAIRED), (B.INT8, B.CODING_PAIRED)):
        blob = B.compress(w, 3.0, container=container, coding=coding)
        info = B.stream_info(blob)
        rc, oi = oracle.parse(blob.numpy())
        assert rc == 0
        assert info.paired == oi.paired == (1 if coding else 0)
        for f in ("rows", "cols", "src_dtype", "container_dtype", "storage_nbytes", "header_nbytes",
                  "actual_bpp", "q_index", "n_tiles", "blocks_per_lane", "off_rowf", "off_scales",
                  "off_freq", "off_dir", "off_tiles"):
            assert getattr(info, f) == getattr(oi, f), f
        assert list(info.split)[:7] == list(oi.split) and list(info.ntok)[:7] == list(oi.ntok)


def test_same_error_codes(oracle):
    w = synth.gaussian(8, 64, 0.02, 10)
    for target, container in ((0.01, 0), (12.0, 0), (8.0, B.INT8), (0.0005, 0)):
        rc, _ = oracle.compress(w, target, container=container)
        with pytest.raises(B.EpError) as e:
            B.compress(w, target, container=container)
        assert e.value.status == rc
