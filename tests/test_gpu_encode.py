"""GPU compressor (ep_compress_device) parity: from a tensor in device memory it must write the
oracle's stream byte for byte (the oracle's encoder is the reference; the library's host
compressor is pinned to the same bytes elsewhere), for every container, ragged rows, forced tile
sizes and resolutions, zero rows, escapes at high rates; and fail like the host compressor on
invalid input.  The streams it writes also decode on the GPU to the oracle's weights."""
import ctypes as C

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [
    ("readme_256", lambda: synth.gaussian(256, 256, 0.02, 0), 3.5, 0, 0, -1),
    ("lognormal_1024", lambda: synth.row_lognormal(1024, 1024, 1), 4.0, 0, 0, -1),
    ("int8", lambda: synth.gaussian(256, 512, 0.02, 2), 3.0, B.INT8, 0, -1),
    ("fp8", lambda: synth.gaussian(256, 512, 0.02, 2), 3.0, B.FP8E4M3, 0, -1),
    ("int8_high", lambda: synth.gaussian(128, 512, 0.02, 2), 7.9, B.INT8, 0, -1),
    ("outlier_0.5", lambda: synth.gaussian_outliers(256, 2048, 3), 0.5, 0, 0, -1),
    ("outlier_8", lambda: synth.gaussian_outliers(256, 2048, 3), 8.0, 0, 0, -1),
    ("outlier_11", lambda: synth.gaussian_outliers(64, 2048, 3), 11.0, 0, 0, -1),
    ("fp16_src", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float16), 4.0, 0, 0, -1),
    ("fp32_src", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float32), 5.0, 0, 0, -1),
    ("fp32_to_bf16", lambda: synth.row_lognormal(128, 1024, 4, dtype=torch.float32), 5.0, B.BF16, 0, -1),
    ("dit_out_rows", lambda: synth.dit_layer(3, 1)[:512], 2.5, 0, 0, -1),
    ("K1", lambda: synth.gaussian(40, 256, 0.02, 5), 11.0, 0, 1, -1),
    ("K5", lambda: synth.gaussian(40, 256, 0.02, 5), 8.0, 0, 5, -1),
    ("q_forced", lambda: synth.row_lognormal(100, 808, 2), 6.0, 0, 3, 700),
    ("zero_rows", lambda: torch.cat([synth.gaussian(30, 512, 0.02, 6), torch.zeros(2, 512, dtype=torch.bfloat16)]),
     4.0, 0, 0, -1),
    ("ragged_1001", lambda: synth.row_lognormal(96, 1001, 3), 4.0, 0, 0, -1),
    ("ragged_int8", lambda: synth.gaussian(64, 523, 0.02, 4), 3.0, B.INT8, 0, -1),
    ("ragged_K3", lambda: synth.row_lognormal(33, 13, 5, dtype=torch.float32), 9.0, 0, 3, -1),
    ("five_cols", lambda: synth.gaussian(2000, 5, 0.02, 8), 11.0, 0, 0, -1),
]


@pytest.mark.parametrize("name,make,target,container,K,q", CASES, ids=[c[0] for c in CASES])
def test_device_stream_equals_oracle(oracle, name, make, target, container, K, q):
    w = make()
    rc, ref = oracle.compress(w, target, container=container, blocks_per_lane=K, q_override=q)
    assert rc == 0
    got = B.compress_device(w.cuda(), target, container=container, blocks_per_lane=K, q_index=q)
    assert got.is_cuda
    got = got.cpu().numpy()
    assert got.size == ref.size and np.array_equal(got, ref)


def test_device_stream_decodes(oracle):
    w = synth.row_lognormal(512, 2048, 9).cuda()
    d = B.compress_device(w, 4.0)
    info = B.stream_info(d.cpu())
    out = B.decompress(d, info)
    rc, st, _, ref = oracle.decode(d.cpu().numpy())
    torch.cuda.synchronize()
    assert rc == 0 and st == 0
    assert np.array_equal(out.view(torch.uint8).cpu().numpy().reshape(-1), ref.view(np.uint8).reshape(-1))


def test_device_errors_match_host():
    w = synth.gaussian(8, 64, 0.02, 1)
    bad = w.clone()
    bad[0, 0] = float("nan")
    for tensor, target, container, status in [(bad, 4.0, 0, -2), (w, 12.0, 0, -3), (w, 8.0, "int8", -3),
                                              (w, 0.01, 0, -4)]:
        with pytest.raises(B.EpError) as e:
            B.compress_device(tensor.cuda(), target, container=container)
        assert e.value.status == status
        with pytest.raises(B.EpError) as e:
            B.compress(tensor, target, container=container)
        assert e.value.status == status


def test_device_buffer_too_small_reports_the_size(oracle):
    w = synth.row_lognormal(128, 512, 4).cuda()
    rc, ref = oracle.compress(w.cpu(), 4.0)
    cfg = B._config(4.0)
    L = B.lib()
    scratch = torch.empty(L.ep_compress_device_scratch(128, 512, C.byref(cfg)), dtype=torch.uint8, device="cuda")
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    n = C.c_size_t(0)
    s = torch.cuda.current_stream().cuda_stream
    rc = L.ep_compress_device(w.data_ptr(), B.BF16, 128, 512, C.byref(cfg), small.data_ptr(), small.numel(),
                              C.byref(n), scratch.data_ptr(), scratch.numel(), s)
    assert rc == -5 and n.value == ref.size
    big = torch.empty(n.value, dtype=torch.uint8, device="cuda")
    rc = L.ep_compress_device(w.data_ptr(), B.BF16, 128, 512, C.byref(cfg), big.data_ptr(), big.numel(),
                              C.byref(n), scratch.data_ptr(), scratch.numel(), s)
    assert rc == 0 and np.array_equal(big.cpu().numpy(), ref)
