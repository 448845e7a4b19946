"""CompressedLinear on the host (no GPU): construction, storage properties of the API reference,
checkpoints through state_dict / load_state_dict (torch.load with weights_only=True), and the loud
failure of a forward call without a GPU copy of the stream."""
import io

import pytest
import torch
import torch.nn as nn

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200.compressed import LatticeRANSConfig
from dit_weight_compression_tile_b200.linear import CompressedINT8Linear, CompressedLinear


def source(in_f=256, out_f=128, seed=0):
    torch.manual_seed(seed)
    lin = nn.Linear(in_f, out_f, dtype=torch.bfloat16)
    return lin


def test_from_linear_properties():
    lin = source()
    layer = CompressedLinear.from_linear(lin, config=LatticeRANSConfig(target_bpp=4.0))
    assert layer.container_dtype == torch.bfloat16 and layer.weight.shape == (128, 256)
    assert layer.stored_nbytes == layer.weight.blob.numel()
    assert layer.compressed_bits == pytest.approx(8.0 * layer.stored_nbytes / (128 * 256)) and layer.compressed_bits <= 4.0
    assert torch.equal(layer.bias, lin.bias)
    codes = CompressedINT8Linear.from_linear(lin, config=LatticeRANSConfig(target_bpp=5.0))
    assert codes.container_dtype == torch.int8 and codes.compressed_bits <= 5.0


def test_checkpoint_round_trip():
    model = nn.Sequential(CompressedLinear.from_linear(source(seed=1), config=LatticeRANSConfig(3.0)),
                          CompressedINT8Linear.from_linear(source(128, 64, seed=2), config=LatticeRANSConfig(4.0)))
    buf = io.BytesIO()
    torch.save(model.state_dict(), buf)
    buf.seek(0)
    state = torch.load(buf, weights_only=True)
    fresh = nn.Sequential(CompressedLinear(256, 128), CompressedINT8Linear(128, 64))
    res = fresh.load_state_dict(state)
    assert not res.missing_keys and not res.unexpected_keys
    for a, b in zip(model, fresh):
        assert torch.equal(a.weight.blob, b.weight.blob) and torch.equal(a.bias, b.bias)
        assert b.compressed_bits == a.compressed_bits


def test_mismatched_checkpoint_is_an_error():
    state = CompressedLinear.from_linear(source(), config=LatticeRANSConfig(4.0)).state_dict()
    with pytest.raises(RuntimeError):
        CompressedLinear(128, 256).load_state_dict(state)
    with pytest.raises(RuntimeError):
        CompressedINT8Linear(256, 128).load_state_dict(state)  # BF16 weights, INT8 layer


def test_layer_without_weight_or_gpu_fails_loudly():
    with pytest.raises(B.EpError):
        CompressedLinear(256, 128)(torch.zeros(2, 256, dtype=torch.bfloat16))
    layer = CompressedLinear.from_linear(source(), config=LatticeRANSConfig(4.0))
    with pytest.raises(B.EpError):
        layer(torch.zeros(2, 256, dtype=torch.bfloat16))  # the stream is on the host
    with pytest.raises(B.EpError):
        layer.compress_weight(torch.zeros(3, 3))
