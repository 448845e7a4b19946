"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark times.
Every weight and every lattice point of every workload is compared with the oracle's decode of
the same stream (the oracle's tile decoder on every host core, tiles split among threads):

* 4096x4096 log-normal rows at 4 bpp, and 8192x8192 INT8 / FP8 codes at 3 bpp;
* the 8192x28672 outlier matrix at 0.5, 1, 2, 3.5, 5 and 8 bpp;
* all 112 tensors of the DiT weight set (28 blocks of hidden 3072) at 2.5 and 4 bpp.

The streams the GPU decodes come from the GPU compressor, as in the benchmark; its bytes equal the
host compressor's on every tensor checked here, and the host compressor's equal the oracle's on
the 4096x4096 matrix, on one DiT tensor of each shape and on the outlier matrix at 3.5 bpp."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def as_bytes(t):
    return t.contiguous().view(torch.uint8).cpu().numpy().reshape(-1)


def decode_gpu(d_blob, info):
    """container and lattice points of a device stream, with the decode's status checked"""
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    work = B.prepare(d_blob, info, status=status)
    out = B.decompress(d_blob, info, workspace=work, status=status)
    v = B.decompress(d_blob, info, workspace=work, status=status, lattice=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, v


def check_all(oracle, host_blob, out, v, what):
    """every container byte and every lattice point equal the oracle's decode of the stream"""
    rc, st, v_ref, out_ref = oracle.decode_parallel(host_blob.numpy())
    assert rc == 0 and st == 0, what
    assert np.array_equal(as_bytes(out), out_ref.view(np.uint8).reshape(-1)), what
    assert np.array_equal(v.cpu().numpy(), v_ref), what


def test_lognormal_4096_full(oracle):
    """4096x4096 BF16, per-row log-normal std, 4 bpp: encoder bytes, every weight and every
    lattice point bit-exact"""
    w = synth.row_lognormal(4096, 4096, 1)
    blob = B.compress(w, 4.0)
    rc, ref = oracle.compress(w, 4.0)
    assert rc == 0 and np.array_equal(blob.numpy(), ref)
    d = B.compress_device(w.cuda(), 4.0)
    assert np.array_equal(d.cpu().numpy(), ref)
    info = B.stream_info(blob)
    assert info.actual_bpp <= 4.0
    out, v = decode_gpu(d, info)
    check_all(oracle, blob, out, v, "4096x4096")


@pytest.mark.parametrize("container", [B.INT8, B.FP8E4M3])
def test_codes_8192_full(oracle, container):
    """8192x8192 N(0, 0.02^2) as per-row absmax INT8 / FP8 codes at 3 bpp, all weights"""
    w = synth.gaussian(8192, 8192, 0.02, 2)
    blob = B.compress(w, 3.0, container=container)
    d = B.compress_device(w.cuda(), 3.0, container=container)
    assert np.array_equal(d.cpu().numpy(), blob.numpy())
    info = B.stream_info(blob)
    assert info.actual_bpp <= 3.0 and info.container_dtype == container
    out, v = decode_gpu(d, info)
    check_all(oracle, blob, out, v, container)


@pytest.fixture(scope="module")
def outlier_matrix():
    return synth.gaussian_outliers(8192, 28672, 3)


@pytest.mark.parametrize("target", [0.5, 1.0, 2.0, 3.5, 5.0, 8.0])
def test_outlier_sweep_full(oracle, outlier_matrix, target):
    """8192x28672 with 0.1 % 8-sigma outliers across the bitrate sweep: every weight"""
    w = outlier_matrix
    d = B.compress_device(w.cuda(), target)
    host = d.cpu()
    assert np.array_equal(B.compress(w, target).numpy(), host.numpy())
    if target == 3.5:
        rc, ref = oracle.compress(w, target)
        assert rc == 0 and np.array_equal(ref, host.numpy())
    info = B.stream_info(host)
    assert info.actual_bpp <= target
    out, v = decode_gpu(d, info)
    check_all(oracle, host, out, v, target)


@pytest.mark.parametrize("target", [2.5, 4.0])
def test_dit_weight_set_full(oracle, target):
    """the DiT weight set (28 blocks x qkv 3072x9216, out 3072x3072, MLP 3072x12288 and
    12288x3072, Student-t entries with per-row log-normal scale): all 112 tensors, every weight"""
    for block in range(28):
        for layer in range(4):
            w = synth.dit_layer(block, layer)
            d = B.compress_device(w.cuda(), target)
            host = d.cpu()
            if block == 0:
                # one tensor of each shape: GPU compressor = host compressor = oracle
                assert np.array_equal(B.compress(w, target).numpy(), host.numpy()), layer
                if target == 4.0:
                    rc, ref = oracle.compress(w, target)
                    assert rc == 0 and np.array_equal(ref, host.numpy()), layer
            info = B.stream_info(host)
            assert info.actual_bpp <= target
            out, v = decode_gpu(d, info)
            check_all(oracle, host, out, v, (block, layer, target))
