"""The fused GEMM's launch plan as ep_linear_fused_plan computes it on the host, for the streams and
token counts the kernel takes: the shared-memory regions lie in order inside the per-CTA limit and
above half an SM (one CTA per SM, so no CTA waits for another's tensor memory), aligned as the bulk
copies and the operand descriptors need; the grid is one wave of CTAs and every K split has tiles;
the tensor memory holds the accumulator; the scratch holds the partial sums, the band counters and
(code containers) the activations' codes and scales.  Streams and counts it cannot take are refused."""
import pytest

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth

LIMIT = 232448


def stream(shape, container, coding, target=4.0):
    w = synth.row_lognormal(*shape, seed=shape[0] + shape[1])
    return B.stream_info(B.compress(w, target if container == 0 else 3.0, container=container, coding=coding,
                                    layout=B.LAYOUT_GEMM))


SHAPES = [(128, 64), (128, 1024), (384, 1024), (1024, 3072), (3072, 3072), (3072, 9216), (12288, 3072)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("container,coding", [(0, B.CODING_SINGLE), (0, B.CODING_PAIRED), (B.INT8, B.CODING_AUTO),
                                              (B.FP8E4M3, B.CODING_SINGLE)])
def test_plan_fits(shape, container, coding):
    info = stream(shape, container, coding)
    codes = container != 0
    KT = shape[1] // 64
    for sms in (148, 132, 20, 1):
        for m in (1, 16, 17, 64, 100, 128):
            rc, P = B.linear_fused_plan(info, m, sms)
            assert rc == 0, (shape, m, sms, rc)
            S = P.decoding_warps
            assert P.bands == shape[0] // 128
            assert P.splits * P.k_tiles_per_split >= KT > (P.splits - 1) * P.k_tiles_per_split
            assert P.bands * P.splits <= max(sms, P.bands)
            assert 1 <= S <= min(15, P.k_tiles_per_split) and P.threads == 32 * max(S + 1, 4)
            assert P.tokens_padded == -(-m // 16) * 16
            assert P.tmem_columns >= max(32, P.tokens_padded) and P.tmem_columns <= 512
            assert P.tmem_columns & (P.tmem_columns - 1) == 0
            assert P.tile_buffer_bytes >= info.max_tile_nbytes + 160 and P.tile_buffer_bytes % 16 == 0
            assert P.smem_tables_bytes == (108544 if info.paired else 57344) == P.smem_barriers_offset
            assert P.smem_barriers_offset % 8 == 0
            assert P.smem_barriers_offset + 40 * S + 24 <= P.smem_tiles_offset and P.smem_tiles_offset % 16 == 0
            assert P.smem_tiles_offset + S * P.tile_buffer_bytes <= P.smem_slices_offset
            assert P.smem_slices_offset % 128 == 0
            assert P.smem_slices_offset + S * 8192 == P.smem_x_offset
            assert P.smem_x_bytes_per_warp == P.tokens_padded * (64 if codes else 128)
            assert P.smem_x_offset + S * P.smem_x_bytes_per_warp <= P.smem_bytes <= LIMIT
            assert P.smem_bytes > LIMIT // 2
            parts = P.splits * m * shape[0] * 4 + P.bands * 4
            assert P.work_bytes >= parts + (m * shape[1] + m * 4 if codes else 0)


def test_more_warps_when_more_tiles():
    """a CTA with more K tiles gets more decoding warps, as many as its buffers allow"""
    info = stream((128, 3072), 0, B.CODING_SINGLE)
    rc, few = B.linear_fused_plan(info, 16, 148)   # 48 splits of one tile
    rc2, many = B.linear_fused_plan(info, 16, 1)   # one CTA with all 48 tiles
    assert rc == rc2 == 0
    assert few.decoding_warps == 1 and few.splits == 48
    assert many.splits == 1 and many.decoding_warps >= 8


def test_refused():
    info = stream((128, 128), 0, B.CODING_SINGLE)
    for m, sms in ((0, 148), (129, 148), (16, 0)):
        assert B.linear_fused_plan(info, m, sms)[0] == -1
    rows = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=2), 4.0))
    assert B.linear_fused_plan(rows, 16, 148)[0] == -1
    fp16 = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=3).half(), 3.0, layout=B.LAYOUT_GEMM))
    assert B.linear_fused_plan(fp16, 16, 148)[0] == -1
