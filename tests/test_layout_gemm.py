"""The GEMM block order of the tiles (EP_LAYOUT_GEMM: every tile one 128 x 64 operand tile of a
consumer GEMM) in the library: the host compressor writes the oracle's bytes, the parser reads the
layout and refuses what it cannot take, and (marked gpu) the GPU compressor writes the same bytes and
the decode kernel reproduces the oracle's weights and lattice points."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

CASES = [((256, 512), 4.0, 0, B.CODING_SINGLE), ((384, 1024), 3.0, 0, B.CODING_PAIRED),
         ((128, 192), 5.0, 0, B.CODING_AUTO), ((256, 256), 3.0, B.INT8, B.CODING_AUTO),
         ((128, 640), 8.0, 0, B.CODING_SINGLE), ((512, 3072), 4.0, B.FP8E4M3, B.CODING_PAIRED)]


def make(shape):
    return synth.row_lognormal(*shape, seed=shape[0] + shape[1])


@pytest.mark.parametrize("shape,target,container,coding", CASES)
def test_host_bytes_equal_oracle(oracle, shape, target, container, coding):
    w = make(shape)
    blob = B.compress(w, target, container=container, coding=coding, layout=B.LAYOUT_GEMM)
    rc, ref = oracle.compress(w, target, container=container, coding=coding, layout=1)
    assert rc == 0 and np.array_equal(blob.numpy(), ref)
    info = B.stream_info(blob)
    assert info.layout == 1 and info.blocks_per_lane == 32 and info.actual_bpp <= target


def test_layout_refused_where_it_does_not_fit():
    for shape, K in [((100, 128), 0), ((128, 100), 0), ((128, 128), 16)]:
        with pytest.raises(B.EpError) as e:
            B.compress(synth.gaussian(*shape, 0.02, seed=1), 4.0, blocks_per_lane=K, layout=B.LAYOUT_GEMM)
        assert e.value.status == -1
    with pytest.raises(B.EpError):
        B.compress(synth.gaussian(128, 128, 0.02, seed=1), 4.0, layout=2)
    blob = B.compress(synth.gaussian(128, 128, 0.02, seed=1), 4.0, layout=B.LAYOUT_GEMM)
    for byte, val in ((58, 2), (28, 16)):
        bad = blob.clone()
        bad[byte] = val
        with pytest.raises(B.EpError) as e:
            B.stream_info(bad)
        assert e.value.status == -6


@pytest.mark.gpu
@pytest.mark.parametrize("shape,target,container,coding", CASES)
def test_gpu_compressor_and_decode(oracle, shape, target, container, coding):
    w = make(shape)
    rc, ref = oracle.compress(w, target, container=container, coding=coding, layout=1)
    assert rc == 0
    d = B.compress_device(w.cuda(), target, container=container, coding=coding, layout=B.LAYOUT_GEMM)
    assert np.array_equal(d.cpu().numpy(), ref)
    info = B.stream_info(d.cpu())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    work = B.prepare(d, info, status=status)
    out = B.decompress(d, info, workspace=work, status=status)
    v = B.decompress(d, info, workspace=work, status=status, lattice=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rc, st, v_ref, out_ref = oracle.decode(ref)
    assert rc == 0 and st == 0
    assert np.array_equal(out.contiguous().view(torch.uint8).cpu().numpy().reshape(-1),
                          out_ref.view(np.uint8).reshape(-1))
    assert np.array_equal(v.cpu().numpy(), v_ref)
