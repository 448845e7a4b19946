"""CompressedTensor on the host (no GPU needed): the properties and methods of the API reference's
CompressedTensor, the state_dict round trip through torch.save / torch.load(weights_only=True),
the "raw" container returned when the target cannot be met, and the loud failure of a decode
that has no GPU copy of the stream."""
import io
import math
import warnings

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth
from dit_weight_compression_tile_b200.compressed import CompressedTensor, LatticeRANSConfig, compress, decompress


def test_properties_follow_the_stream():
    w = synth.row_lognormal(64, 512, seed=3)
    ct = compress(w, LatticeRANSConfig(target_bpp=3.5))
    info = ct.info
    assert ct.compress_method == "lattice_rans" and not ct.lossless
    assert ct.shape == w.shape and ct.dtype == torch.bfloat16 and ct.encoded_dtype == torch.bfloat16
    assert ct.storage_nbytes() == info.storage_nbytes == ct.blob.numel()
    assert ct.storage_nbytes(include_header=False) == info.storage_nbytes - info.header_nbytes
    assert ct.actual_bpp == pytest.approx(8.0 * info.storage_nbytes / w.numel()) and ct.actual_bpp <= 3.5
    assert ct.actual_bpp == pytest.approx(info.actual_bpp)


def test_code_container_outputs_codes():
    w = synth.gaussian(128, 256, 0.02, 4)
    ct = compress(w, LatticeRANSConfig(target_bpp=4.0, container=torch.int8))
    assert ct.encoded_dtype == torch.int8 and ct.dtype == torch.int8
    with pytest.raises(B.EpError):
        ct.to(dtype=torch.bfloat16)
    f = compress(w, LatticeRANSConfig(target_bpp=4.0))
    assert f.to(dtype=torch.float32).dtype == torch.float32 and f.to(torch.float16).dtype == torch.float16
    with pytest.raises(B.EpError):
        f.to(dtype=torch.int8)


@pytest.mark.parametrize("prefix", ["", "layers.0.weight."])
def test_state_dict_round_trip_weights_only(prefix):
    w = synth.row_lognormal(48, 256, seed=5, dtype=torch.float16)
    ct = compress(w, LatticeRANSConfig(target_bpp=4.0)).to(dtype=torch.float32)
    buf = io.BytesIO()
    torch.save(ct.state_dict(prefix), buf)
    buf.seek(0)
    state = torch.load(buf, weights_only=True)
    assert all(k.startswith(prefix) for k in state)
    back = CompressedTensor.from_state_dict(state, prefix)
    assert torch.equal(back.blob, ct.blob)
    assert back.dtype == torch.float32 and back.encoded_dtype == torch.float16 and back.shape == w.shape
    assert back.actual_bpp == ct.actual_bpp


def test_damaged_state_is_rejected():
    ct = compress(synth.gaussian(32, 256, 0.02, 6), LatticeRANSConfig(target_bpp=4.0))
    state = ct.state_dict()
    state["ep_stream"] = state["ep_stream"][:-16]
    with pytest.raises(B.EpError):
        CompressedTensor.from_state_dict(state)


def test_unreachable_target_keeps_the_tensor_raw():
    w = synth.gaussian(8, 16, 0.02, 1)
    with warnings.catch_warnings(record=True) as caught:
        warnings.simplefilter("always")
        ct = compress(w, LatticeRANSConfig(target_bpp=0.01))
    assert any("uncompressed" in str(c.message) for c in caught)
    assert ct.compress_method == "raw" and ct.lossless and ct.actual_bpp == 16.0
    assert torch.equal(decompress(ct), w)
    state = ct.state_dict("x.")
    back = CompressedTensor.from_state_dict(state, "x.")
    assert back.compress_method == "raw" and torch.equal(back.to(dtype=torch.float32).decompress(), w.float())


def test_decode_without_a_cuda_device_fails_loudly(monkeypatch):
    """a host-resident lattice stream is decoded by the GPU kernel or not at all"""
    ct = compress(synth.gaussian(32, 256, 0.02, 2), LatticeRANSConfig(target_bpp=4.0))
    assert ct.device.type == "cpu"
    monkeypatch.setattr(torch.cuda, "is_available", lambda: False)
    with pytest.raises(B.EpError, match="CUDA device"):
        decompress(ct)


def test_invalid_inputs_raise():
    with pytest.raises(B.EpError):
        compress(torch.zeros(16), LatticeRANSConfig())
    bad = synth.gaussian(16, 64, 0.02, 1)
    bad[3, 5] = float("nan")
    with pytest.raises(B.EpError):
        compress(bad, LatticeRANSConfig())
    with pytest.raises(B.EpError):
        compress(bad, 4.0)
    assert math.isfinite(compress(synth.gaussian(16, 64, 0.02, 1), LatticeRANSConfig(target_bpp=8.0)).actual_bpp)


def test_config_coding_reaches_the_stream(oracle):
    """LatticeRANSConfig.coding selects paired or single coding of coordinates 1..6"""
    w = synth.row_lognormal(128, 1024, 3)
    paired = compress(w, LatticeRANSConfig(target_bpp=4.0, coding=2))
    single = compress(w, LatticeRANSConfig(target_bpp=4.0, coding=1))
    assert paired._info.paired == 1 and single._info.paired == 0
    rc, ref = oracle.compress(w, 4.0, coding=oracle.CODING_PAIRED)
    assert np.array_equal(paired.blob.numpy(), ref)


def test_tile_ans_container_host():
    """compress(tensor, TileANSConfig()): a lossless container of any shape and dtype; its
    properties, its state_dict round trip and the refusal to change dtype"""
    from dit_weight_compression_tile_b200.compressed import TileANSConfig
    for t in (synth.row_lognormal(64, 256, seed=30), synth.gaussian(4, 8, 0.02, seed=31).float().reshape(2, 2, 8),
              torch.clamp(torch.round(torch.randn(1000) * 20), -127, 127).to(torch.int8)):
        ct = compress(t, TileANSConfig())
        assert ct.compress_method == "tile_ans" and ct.lossless
        assert ct.shape == t.shape and ct.dtype == t.dtype and ct.encoded_dtype == t.dtype
        assert ct.storage_nbytes() == ct.blob.numel() and ct.storage_nbytes(include_header=False) == ct.blob.numel() - 64
        assert ct.actual_bpp == pytest.approx(8.0 * ct.blob.numel() / t.numel())
        with pytest.raises(B.EpError):
            ct.to(dtype=torch.float16 if t.dtype != torch.float16 else torch.float32)
        buf = io.BytesIO()
        torch.save(ct.state_dict("w."), buf)
        buf.seek(0)
        back = CompressedTensor.from_state_dict(torch.load(buf, weights_only=True), "w.")
        assert back.compress_method == "tile_ans" and torch.equal(back.blob, ct.blob) and back.shape == t.shape
    bf16 = compress(synth.row_lognormal(512, 512, seed=32), TileANSConfig())
    assert 0.66 * 16 < bf16.actual_bpp < 0.72 * 16
