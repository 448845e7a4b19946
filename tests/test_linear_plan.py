"""The fused GEMM's launch plan as ep_linear_fused_plan computes it on the host, for the streams and
token counts the kernel takes: the shared-memory regions lie in order inside the per-CTA limit and
above half an SM (one CTA per SM, so no CTA waits for another's tensor memory), aligned as the bulk
copies and the operand descriptors need; the tiles are spread evenly over one wave of CTAs (the
most tiles and bands per CTA recomputed here from the even split); the tensor memory holds one
accumulator per band a CTA touches; the scratch holds every CTA's partial sums, the band counters
and (code containers) the activations' codes and scales.  Streams and counts it cannot take are
refused.  The rule by which a band's last CTA knows how many CTAs touched the band is checked
against brute force over tile counts and grids."""
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
            T = P.bands * KT
            C = P.ctas
            # the CTAs' tile ranges, as the kernel maps them: cover every tile once, none empty
            starts = [map_first(P, c, T, KT) for c in range(C + 1)]
            assert starts[0] == 0 and starts[C] == T and all(a < b for a, b in zip(starts, starts[1:]))
            for t in range(T):
                c = map_cta_of(P, t, T, KT)
                assert starts[c] <= t < starts[c + 1]
            most_bands = max((starts[c + 1] - 1) // KT - starts[c] // KT + 1 for c in range(C))
            assert P.tiles_per_cta == max(b - a for a, b in zip(starts, starts[1:]))
            if P.spread:
                assert C >= min(sms, T) and most_bands * -(-m // 16) * 16 <= 512
            else:
                assert most_bands == 1 and C == P.bands * P.splits
            S = P.decoding_warps
            assert P.bands == shape[0] // 128
            assert P.accumulators == most_bands
            assert 1 <= S <= min(15, P.tiles_per_cta) and P.threads == 32 * max(S + 1, 4)
            assert P.tokens_padded == -(-m // 16) * 16
            assert P.tmem_columns >= max(32, P.accumulators * P.tokens_padded) and P.tmem_columns <= 512
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
            parts = P.ctas * P.accumulators * m * 128 * 4 + P.bands * 4
            assert P.work_bytes >= parts + (m * shape[1] + m * 4 if codes else 0)


def first(c, T, C):
    return c * T // C


def map_first(P, c, T, KT):
    """the first tile of CTA c (tiles spread evenly, or each band's K tiles in P.splits ranges)"""
    if P.spread:
        return first(c, T, P.ctas)
    ktps = -(-KT // P.splits)
    return (c // P.splits) * KT + min((c % P.splits) * ktps, KT)


def map_cta_of(P, t, T, KT):
    if P.spread:
        return cta_of(t, T, P.ctas)
    ktps = -(-KT // P.splits)
    return (t // KT) * P.splits + (t % KT) // ktps


def cta_of(t, T, C):
    """the CTA that holds tile t, the rule the kernel uses: the largest c with first(c) <= t"""
    return ((t + 1) * C - 1) // T


def test_band_contributors_rule():
    """for every band, the CTAs from the holder of its first tile to the holder of its last are
    exactly those whose tile range meets the band"""
    for KT in (1, 2, 3, 48, 144):
        for bands in (1, 2, 5, 24, 96, 150, 224):
            T = bands * KT
            for C in sorted({1, 2, 7, 96, 132, 148, min(148, T)}):
                C = min(C, T)
                for c in range(C):
                    assert first(c, T, C) < first(c + 1, T, C)  # no CTA without tiles
                    for t in range(first(c, T, C), first(c + 1, T, C)):
                        assert cta_of(t, T, C) == c
                for b in range(bands):
                    touching = [c for c in range(C) if first(c, T, C) < (b + 1) * KT and first(c + 1, T, C) > b * KT]
                    assert touching == list(range(cta_of(b * KT, T, C), cta_of((b + 1) * KT - 1, T, C) + 1))


def test_more_warps_when_more_tiles():
    """a CTA with more tiles gets more decoding warps, as many as its buffers allow; fewer bands than
    SMs still fill the SMs"""
    info = stream((128, 3072), 0, B.CODING_SINGLE)
    rc, few = B.linear_fused_plan(info, 16, 148)   # 48 CTAs of one tile
    rc2, many = B.linear_fused_plan(info, 16, 1)   # one CTA with all 48 tiles
    assert rc == rc2 == 0
    assert few.decoding_warps == 1 and few.ctas == 48
    assert many.ctas == 1 and many.decoding_warps >= 8
    # 96 bands of 48 tiles on 148 SMs: band-aligned CTAs would leave 52 SMs idle and take 4 rounds of
    # 12 tiles; spread evenly, 148 CTAs of at most 32 tiles, 3 rounds
    wide = stream((12288, 3072), 0, B.CODING_SINGLE)
    rc, P = B.linear_fused_plan(wide, 16, 148)
    assert rc == 0 and P.spread == 1 and P.ctas == 148 and P.tiles_per_cta == 32 and P.accumulators == 2
    # 24 bands of 144 tiles: 6 splits of 24 fill 144 SMs in 2 rounds, as the even spread would
    tall = stream((3072, 9216), 0, B.CODING_SINGLE)
    rc, P = B.linear_fused_plan(tall, 16, 148)
    assert rc == 0 and P.spread == 0 and P.splits == 6 and P.ctas == 144 and P.accumulators == 1


def test_refused():
    info = stream((128, 128), 0, B.CODING_SINGLE)
    for m, sms in ((0, 148), (129, 148), (16, 0)):
        assert B.linear_fused_plan(info, m, sms)[0] == -1
    rows = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=2), 4.0))
    assert B.linear_fused_plan(rows, 16, 148)[0] == -1
    fp16 = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=3).half(), 3.0, layout=B.LAYOUT_GEMM))
    assert B.linear_fused_plan(fp16, 16, 148)[0] == -1
