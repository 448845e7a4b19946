"""CompressedLinear / CompressedINT8Linear / CompressedFP8Linear on the GPU.  The weight each forward
call uses is the oracle's decode of the layer's stream, and the products are checked against
references computed separately: the same library call on the oracle's weight (BF16, bit for
bit), an int64 matmul on the host (INT8: the int32 accumulation is exact, the scaling elementwise),
an fp64 matmul (FP8, within the fp32 accumulation's rounding)."""
import io

import numpy as np
import pytest
import torch
import torch.nn as nn
import torch.nn.functional as F

from dit_weight_compression_tile_b200.compressed import LatticeRANSConfig
from dit_weight_compression_tile_b200.linear import CompressedFP8Linear, CompressedINT8Linear, CompressedLinear

pytestmark = pytest.mark.gpu


def source(in_f, out_f, seed, dtype=torch.bfloat16):
    torch.manual_seed(seed)
    lin = nn.Linear(in_f, out_f, dtype=dtype)
    with torch.no_grad():
        lin.weight.mul_(torch.exp(0.3 * torch.randn(out_f, 1, dtype=dtype)))
    return lin.cuda()


def oracle_weight(oracle, layer, torch_dtype):
    rc, st, _, out = oracle.decode(layer.weight.blob.cpu().numpy())
    assert rc == 0 and st == 0
    if torch_dtype in (torch.bfloat16, torch.float16):
        return torch.from_numpy(out.view(np.int16)).view(torch_dtype).cuda()
    if torch_dtype == torch.float8_e4m3fn:
        return torch.from_numpy(out).view(torch.float8_e4m3fn).cuda()
    return torch.from_numpy(out).cuda()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_compressed_linear_matches_library_call_on_oracle_weight(oracle, dtype):
    lin = source(1024, 768, 1, dtype)
    layer = CompressedLinear.from_linear(lin, config=LatticeRANSConfig(target_bpp=4.0))
    assert layer.weight.device.type == "cuda" and layer.compressed_bits <= 4.0
    w = oracle_weight(oracle, layer, dtype)
    x = torch.randn(4, 37, 1024, dtype=dtype, device="cuda")
    for _ in range(2):  # the buffer is reused
        y = layer(x)
        assert torch.equal(y, F.linear(x, w, lin.bias))
    assert torch.equal(layer.dequantize(), w)
    # relative L2 of the weight against the source
    rel = (w.float() - lin.weight.detach().float()).norm() / lin.weight.detach().float().norm()
    assert float(rel) < 0.12


def test_checkpoint_on_the_gpu(oracle):
    layer = CompressedLinear.from_linear(source(512, 256, 2), config=LatticeRANSConfig(3.0))
    buf = io.BytesIO()
    torch.save(layer.state_dict(), buf)
    buf.seek(0)
    fresh = CompressedLinear(512, 256, device="cuda")
    fresh.load_state_dict(torch.load(buf, weights_only=True, map_location="cuda"))
    x = torch.randn(8, 512, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(fresh(x), layer(x))
    moved = fresh.to("cpu").to("cuda")
    assert torch.equal(moved(x), layer(x))


def quantized_x(x, bound, dtype):
    amax = x.abs().amax(dim=1, keepdim=True).float()
    sx = torch.where(amax > 0, amax / torch.full_like(amax, bound), torch.ones_like(amax))  # rounded division
    q = x.float() / sx
    q = q.round().clamp(-127, 127).to(torch.int8) if dtype == torch.int8 else q.clamp(-448, 448).to(dtype)
    return q, sx


def test_int8_linear(oracle):
    lin = source(1024, 512, 3)
    layer = CompressedINT8Linear.from_linear(lin, config=LatticeRANSConfig(target_bpp=4.0))
    codes = oracle_weight(oracle, layer, torch.int8)
    assert torch.equal(layer.codes(), codes)
    sw = layer._scales()
    assert torch.equal(layer.dequantize(), (codes.float() * sw[:, None]).to(torch.bfloat16))
    x = torch.randn(64, 1024, dtype=torch.bfloat16, device="cuda")
    q, sx = quantized_x(x, 127.0, torch.int8)
    acc = (q.cpu().long() @ codes.cpu().long().T).cuda()  # exact
    ref = ((acc.float() * sx * sw[None, :]).to(torch.bfloat16) + lin.bias.detach())
    assert torch.equal(layer(x), ref)


def test_fp8_linear(oracle):
    lin = source(1024, 512, 4)
    layer = CompressedFP8Linear.from_linear(lin, config=LatticeRANSConfig(target_bpp=4.0))
    codes = oracle_weight(oracle, layer, torch.float8_e4m3fn)
    assert torch.equal(layer.codes().view(torch.uint8), codes.view(torch.uint8))
    sw = layer._scales()
    x = torch.randn(64, 1024, dtype=torch.bfloat16, device="cuda")
    q, sx = quantized_x(x, 448.0, torch.float8_e4m3fn)
    ref = (q.double() @ codes.double().T) * sx.double() * sw.double()[None, :] + lin.bias.detach().double()
    y = layer(x).double()
    assert float((y - ref).norm() / ref.norm()) < 1e-2
