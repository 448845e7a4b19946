"""Pins for the oracle's container conversions against PyTorch's CPU casts (library
routines with the same rounding rule), over dense sweeps of fp32 inputs including the
exact rounding ties, plus the INT8/FP8 per-row code preparation."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import synth

BF16, FP16, FP32, INT8, FP8 = 1, 2, 3, 4, 5


def sweep(lo_exp, hi_exp, n=1 << 20, seed=0):
    """fp32 values spanning [2^lo_exp, 2^hi_exp) with random mantissas, both signs, plus ties."""
    rng = np.random.default_rng(seed)
    e = rng.integers(max(lo_exp, -127), min(hi_exp, 128), size=n)  # -127: fp32 subnormals
    m = rng.integers(0, 1 << 23, size=n)
    bits = ((e + 127).astype(np.uint32) << 23) | m.astype(np.uint32)
    bits[: n // 4] &= ~np.uint32(0xFFFF)  # exact bf16 values
    bits[n // 4: n // 2] = (bits[n // 4: n // 2] & ~np.uint32(0xFFFF)) | np.uint32(0x8000)  # bf16 ties
    x = bits.view(np.float32).copy()
    x[1::2] *= -1
    return np.concatenate([x, np.array([0.0, -0.0], np.float32)])


def test_bf16(oracle):
    x = sweep(-133, 127)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.convert(x, BF16), ref)


def test_fp16(oracle):
    x = sweep(-26, 17)
    ties = (np.arange(-4096, 4096, dtype=np.float32) + 0.5) * np.float32(2.0 ** -24)  # subnormal ties
    x = np.concatenate([x, ties, (np.arange(0, 2048, dtype=np.float32) + 0.5) * 32.0])
    ref = torch.from_numpy(x).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.convert(x, FP16), ref)


def test_e4m3(oracle):
    x = sweep(-12, 9)
    x = np.concatenate([x, (np.arange(-64, 64, dtype=np.float32) + 0.5) * np.float32(2.0 ** -9)])
    clamped = np.clip(x, -448.0, 448.0)
    ref = torch.from_numpy(clamped).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.convert(x, FP8), ref)  # saturating: beyond 448 -> +-448
    big = np.array([449.0, 464.0, 480.0, 1e30, -1e30, -500.0], np.float32)
    assert list(oracle.convert(big, FP8)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


def test_int8(oracle):
    x = np.concatenate([sweep(-3, 9), np.arange(-200, 200, 0.5, dtype=np.float32)])
    ref = torch.round(torch.from_numpy(x)).clamp(-127, 127).to(torch.int8).numpy()
    assert np.array_equal(oracle.convert(x, INT8), ref)


@pytest.mark.parametrize("container", [INT8, FP8])
def test_prequant_matches_torch(oracle, container):
    w = synth.gaussian(64, 256, 0.02, 9)
    w[3] = 0  # an all-zero row gets scale 1 and zero codes
    codes, scales = oracle.prequant(w, container)
    wd = w.double()
    amax = wd.abs().amax(1, keepdim=True)
    bound = 127.0 if container == INT8 else 448.0
    s = (amax / bound).float()
    s[amax == 0] = 1.0
    assert np.array_equal(scales, s.squeeze(1).numpy())
    if container == INT8:
        ref = torch.round(wd / s.double()).clamp(-127, 127)
    else:
        t = (wd / s.double()).float().clamp(-448, 448)
        ref = t.to(torch.float8_e4m3fn).double()
    assert np.array_equal(codes, ref.numpy())
    assert np.abs(codes).max() <= bound
