"""The decode fused into a tcgen05 GEMM (ep_linear_fused; "EntroPack API reference",
CompressedLinear: the weight is reconstructed on every forward call).

Host side: the entry point refuses what it cannot take before any launch (a row-ordered stream, an
FP16 / FP32 container, m outside [1, 128], null or misaligned pointers).  GPU side (marked gpu): the
output equals the library GEMM applied to the oracle's decoded weight, within the tolerance of two
fp32 sums of the same BF16 products taken in different orders and rounded once to BF16 (the bound
below), for single and paired streams, with and without bias, several m and K splits."""
import ctypes as C

import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth


def gemm_stream(shape, target=4.0, coding=B.CODING_AUTO, container=0, seed=1):
    w = synth.row_lognormal(*shape, seed=seed)
    blob = B.compress(w, target, coding=coding, container=container, layout=B.LAYOUT_GEMM)
    return w, blob, B.stream_info(blob)


def test_refused_before_any_launch():
    L = B.lib()
    _, blob, info = gemm_stream((128, 128))
    fake = C.c_void_p(1 << 20)  # never dereferenced: every call below returns before a launch
    assert L.ep_linear_fused_workspace(C.byref(info), 0) == 0
    assert L.ep_linear_fused_workspace(C.byref(info), 129) == 0
    assert L.ep_linear_fused(C.byref(info), fake, fake, fake, 0, None, fake, fake, 1 << 20, None, None) == -1
    assert L.ep_linear_fused(C.byref(info), None, fake, fake, 4, None, fake, fake, 1 << 20, None, None) == -1
    assert L.ep_linear_fused(C.byref(info), C.c_void_p((1 << 20) + 4), fake, fake, 4, None, fake, fake, 1 << 20,
                             None, None) == -1
    rows = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=2), 4.0))
    assert rows.layout == 0
    assert L.ep_linear_fused_workspace(C.byref(rows), 4) == 0
    assert L.ep_linear_fused(C.byref(rows), fake, fake, fake, 4, None, fake, fake, 1 << 20, None, None) == -1
    # an FP16 container: the fused GEMM takes BF16 weights or INT8 / FP8 codes
    fp16 = B.stream_info(B.compress(synth.gaussian(128, 128, 0.02, seed=3).half(), 3.0, layout=B.LAYOUT_GEMM))
    assert fp16.container_dtype == B.FP16
    assert L.ep_linear_fused_workspace(C.byref(fp16), 4) == 0
    assert L.ep_linear_fused(C.byref(fp16), fake, fake, fake, 4, None, fake, fake, 1 << 20, None, None) == -1


def reference(oracle, blob, x, bias):
    """the library GEMM (fp32) on the oracle's decoded weight, and the bound on the fused result:
    both sum the same exact BF16 x BF16 products in fp32, in different orders; the difference is at
    most K u sum |x_k w_k| (u = 2^-24, a standard bound for two recursive sums), and one BF16
    rounding (half an ulp, 2^-9 relative) of each"""
    rc, st, _, wd = oracle.decode(blob.numpy())
    assert rc == 0 and st == 0
    wf = torch.from_numpy(wd.view(np.int16)).view(torch.bfloat16).float()
    xf = x.float().cpu()
    y = xf @ wf.T + (bias.float().cpu() if bias is not None else 0.0)
    mag = xf.abs() @ wf.abs().T + (bias.float().cpu().abs() if bias is not None else 0.0)
    K = xf.shape[1]
    tol = K * 2.0 ** -24 * mag + 2.0 ** -8 * y.abs() + 1e-30
    return y, tol


@pytest.mark.gpu
@pytest.mark.parametrize("shape,m,coding,with_bias", [((128, 128), 1, B.CODING_SINGLE, False),
                                                      ((256, 512), 16, B.CODING_SINGLE, True),
                                                      ((384, 1024), 64, B.CODING_PAIRED, True),
                                                      ((128, 3072), 128, B.CODING_AUTO, False),
                                                      ((1024, 3072), 7, B.CODING_PAIRED, True),
                                                      # DiT shapes: 8 and 10 decoding warps per CTA, 3 and 5
                                                      # rounds of tiles; the largest token count paired
                                                      ((3072, 9216), 16, B.CODING_AUTO, True),
                                                      ((12288, 3072), 3, B.CODING_SINGLE, False),
                                                      ((3072, 3072), 128, B.CODING_PAIRED, True)])
def test_fused_equals_gemm_on_decoded_weight(oracle, shape, m, coding, with_bias):
    w, blob, info = gemm_stream(shape, coding=coding, seed=shape[1] + m)
    g = torch.Generator().manual_seed(m)
    x = (torch.randn(m, shape[1], generator=g) * 0.5).to(torch.bfloat16)
    bias = (torch.randn(shape[0], generator=g) * 0.1).to(torch.bfloat16) if with_bias else None
    d = blob.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = B.prepare(d, info, status=status)
    work = torch.zeros(B.linear_fused_workspace(info, m), dtype=torch.uint8, device="cuda")
    y = B.linear_fused(x.cuda(), d, info, tables, bias=bias.cuda() if bias is not None else None, work=work,
                       status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, tol = reference(oracle, blob, x, bias)
    got = y.float().cpu()
    assert got.shape == ref.shape
    bad = (got - ref).abs() > tol
    assert not bad.any(), (float((got - ref).abs().max()), int(bad.sum()))
    # a second call on the same tables and scratch gives the same bits (the band counters in the
    # scratch are back at zero after every call)
    y2 = B.linear_fused(x.cuda(), d, info, tables, bias=bias.cuda() if bias is not None else None, work=work)
    assert torch.equal(y2, y)
    nb = info.rows // 128
    assert int(work[-4 * nb:].view(torch.int32).abs().sum()) == 0


def test_layer_takes_the_fused_path_only_where_it_applies():
    from dit_weight_compression_tile_b200 import CompressedLinear, LatticeRANSConfig
    lin = torch.nn.Linear(128, 256, dtype=torch.bfloat16)
    gemm = CompressedLinear.from_linear(lin, config=LatticeRANSConfig(4.0, layout="gemm"))
    rows = CompressedLinear.from_linear(lin, config=LatticeRANSConfig(4.0))
    assert gemm.weight.info.layout == B.LAYOUT_GEMM and rows.weight.info.layout == B.LAYOUT_ROWS
    x = torch.zeros(3, 128, dtype=torch.bfloat16)
    assert not gemm.fused_for(x)  # a host tensor
    with pytest.raises(B.EpError):
        CompressedLinear.from_linear(lin, config=LatticeRANSConfig(4.0, layout="columns"))
    with pytest.raises(B.EpError):  # 100 output features are not whole 128-row bands
        CompressedLinear.from_linear(torch.nn.Linear(128, 100), config=LatticeRANSConfig(4.0, layout="gemm"))


@pytest.mark.gpu
@pytest.mark.parametrize("tokens", [(1,), (2, 8), (4, 7), (3, 50)])
def test_layer_forward(oracle, tokens):
    from dit_weight_compression_tile_b200 import CompressedLinear, LatticeRANSConfig
    from dit_weight_compression_tile_b200.linear import FUSED_MAX_TOKENS
    torch.manual_seed(3)
    lin = torch.nn.Linear(1024, 384, dtype=torch.bfloat16)
    layer = CompressedLinear.from_linear(lin, config=LatticeRANSConfig(4.0, layout="gemm")).cuda()
    x = (torch.randn(*tokens, 1024) * 0.5).to(torch.bfloat16)
    y = layer(x.cuda())
    m = x.numel() // 1024
    assert layer.fused_for(x.cuda()) == (m <= FUSED_MAX_TOKENS)
    blob = layer.weight.blob.cpu()
    ref, tol = reference(oracle, blob, x.reshape(-1, 1024), layer.bias.detach().cpu())
    got = y.float().cpu().reshape(-1, 384)
    assert y.shape == (*tokens, 384)
    # above FUSED_MAX_TOKENS the layer decodes and calls the library GEMM: summed in another order, same bound
    assert torch.all((got - ref).abs() <= tol), float((got - ref).abs().max())


def w8a8_reference(oracle, blob, x, bias, container):
    """the per-row-quantized layers' arithmetic on the CPU with the oracle's decoded codes: the
    activations quantized per token (scale amax / 127 or / 448), the codes multiplied (INT8 exactly
    in int64, FP8 in fp64), y = RNE_bf16(fp32(fp32(sum) s_x) s_w), then RNE_bf16(y + bias).  Returns
    y and, for FP8, the bound on the fused result (fp32 sums in another order: K 2^-23 sum |x w|
    scaled, plus two BF16 roundings)"""
    b = blob.numpy()
    rc, st, _, wq = oracle.decode(b)
    assert rc == 0 and st == 0
    rc, info = oracle.parse(b)
    sw = torch.from_numpy(np.frombuffer(b.tobytes(), np.float32, count=info.rows, offset=info.off_scales).copy())
    xf = x.float().cpu()
    bound = 127.0 if container == B.INT8 else 448.0
    amax = xf.abs().amax(dim=1, keepdim=True)
    sx = torch.where(amax > 0, amax / torch.full_like(amax, bound), torch.ones_like(amax))  # rounded division
    q = xf / sx
    if container == B.INT8:
        xq = q.round().clamp(-127, 127).to(torch.int64)
        acc = (xq @ torch.from_numpy(wq.astype(np.int64)).T).float()
        mag = None
    else:
        xq = q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).double()
        wf = torch.from_numpy(wq.view(np.uint8).copy()).view(torch.float8_e4m3fn).double()
        acc = (xq @ wf.T).float()
        mag = (xq.abs() @ wf.abs().T).float()
    y0 = acc * sx * sw[None, :]
    y = y0.to(torch.bfloat16)
    if bias is not None:
        y = y + bias.to(torch.bfloat16).cpu()
    if mag is None:
        return y, None
    K = xf.shape[1]
    tol = K * 2.0 ** -23 * mag * sx * sw[None, :] + 2.0 ** -8 * (y0.abs() + y.float().abs()) + 1e-30
    return y, tol


@pytest.mark.gpu
@pytest.mark.parametrize("shape,m,container,coding,with_bias", [((256, 512), 16, B.INT8, B.CODING_SINGLE, True),
                                                                ((1024, 3072), 5, B.INT8, B.CODING_PAIRED, False),
                                                                ((3072, 3072), 16, B.INT8, B.CODING_AUTO, True),
                                                                ((384, 1024), 7, B.FP8E4M3, B.CODING_SINGLE, True),
                                                                ((3072, 9216), 16, B.FP8E4M3, B.CODING_AUTO, False),
                                                                ((128, 1024), 128, B.INT8, B.CODING_SINGLE, True),
                                                                # 2 and 3 rounds of tiles per decoding warp
                                                                ((3072, 9216), 16, B.INT8, B.CODING_AUTO, True),
                                                                ((3072, 12288), 3, B.INT8, B.CODING_SINGLE, False)])
def test_fused_w8a8(oracle, shape, m, container, coding, with_bias):
    """INT8: every output bit equals the CPU arithmetic on the oracle's codes; FP8: within the bound"""
    w = synth.row_lognormal(*shape, seed=shape[0] + m)
    blob = B.compress(w, 3.0, container=container, coding=coding, layout=B.LAYOUT_GEMM)
    info = B.stream_info(blob)
    g = torch.Generator().manual_seed(m + 1)
    x = (torch.randn(m, shape[1], generator=g) * 0.5).to(torch.bfloat16)
    x[0, :7] = 0.0  # a token with zeros, and (below) an all-zero token: scale 1
    if m > 2:
        x[2] = 0.0
    bias = (torch.randn(shape[0], generator=g) * 0.1).to(torch.bfloat16) if with_bias else None
    d = blob.cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    tables = B.prepare(d, info, status=status)
    work = torch.zeros(B.linear_fused_workspace(info, m), dtype=torch.uint8, device="cuda")
    y = B.linear_fused(x.cuda(), d, info, tables, bias=bias.cuda() if bias is not None else None, work=work,
                       status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, tol = w8a8_reference(oracle, blob, x, bias, container)
    got = y.cpu()
    if tol is None:
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), \
            (float((got.float() - ref.float()).abs().max()), int((got != ref).sum()))
    else:
        assert bool(((got.float() - ref.float()).abs() <= tol).all()), float((got.float() - ref.float()).abs().max())
    y2 = B.linear_fused(x.cuda(), d, info, tables, bias=bias.cuda() if bias is not None else None, work=work)
    assert torch.equal(y2, y)


@pytest.mark.gpu
@pytest.mark.parametrize("cls", ["CompressedINT8Linear", "CompressedFP8Linear"])
def test_code_layers_fused_forward(cls):
    """the W8A8 layers of a GEMM-ordered stream: fused up to FUSED_MAX_TOKENS tokens, library GEMM
    above, the same per-token quantization either way (INT8: the same bits)"""
    from dit_weight_compression_tile_b200 import linear as Lm
    from dit_weight_compression_tile_b200.compressed import LatticeRANSConfig
    torch.manual_seed(4)
    lin = torch.nn.Linear(1024, 256, dtype=torch.bfloat16)
    layer = getattr(Lm, cls).from_linear(lin, config=LatticeRANSConfig(3.0, layout="gemm")).cuda()
    x = (torch.randn(2, 6, 1024) * 0.5).to(torch.bfloat16).cuda()
    assert layer.fused_for(x)
    y = layer(x)
    x2 = x.reshape(-1, 1024)
    # the library path on the same layer: call it with more tokens than the fused path takes (32,
    # zero-padded: a multiple of 16 for the library GEMMs) and compare the first rows
    big = torch.cat([x2, torch.zeros(32 - x2.shape[0], 1024, dtype=torch.bfloat16, device="cuda")])
    assert not layer.fused_for(big)
    yb = layer(big)[: x2.shape[0]].reshape(2, 6, 256)
    assert y.shape == (2, 6, 256)
    if cls == "CompressedINT8Linear":
        assert torch.equal(y, yb)
    else:
        assert torch.allclose(y.float(), yb.float(), rtol=2 ** -6, atol=1e-3)
