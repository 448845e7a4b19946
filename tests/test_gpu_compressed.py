"""GPU parity of the output dtype change (CompressedTensor.to(dtype=...) of the API reference) and of
the CompressedTensor calls: the fused decode into BF16, FP16 and FP32 from every float container,
through the C ABI and through CompressedTensor, equal byte for byte to the oracle's decode of the
same oracle-encoded stream (the fp32 weight rounded once into the requested dtype)."""
import numpy as np
import pytest
import torch

from dit_weight_compression_tile_b200 import binding as B
from dit_weight_compression_tile_b200 import synth
from dit_weight_compression_tile_b200.compressed import CompressedTensor, LatticeRANSConfig, compress, decompress

pytestmark = pytest.mark.gpu

SRC = {B.BF16: torch.bfloat16, B.FP16: torch.float16, B.FP32: torch.float32}


def as_bytes(t):
    return t.contiguous().view(torch.uint8).cpu().numpy().reshape(-1)


@pytest.mark.parametrize("container", [B.BF16, B.FP16, B.FP32])
@pytest.mark.parametrize("shape,K", [((100, 808), 0), ((512, 2048), 0), ((64, 1024), 4), ((33, 1001), 2)])
def test_float_containers_to_every_float_dtype(oracle, container, shape, K):
    w = synth.row_lognormal(*shape, seed=shape[0] + container, dtype=SRC[container])
    rc, blob = oracle.compress(w, 4.5, blocks_per_lane=K)
    assert rc == 0
    d = torch.from_numpy(blob).cuda()
    info = B.stream_info(torch.from_numpy(blob))
    ct = CompressedTensor(d, info)
    for out_dt in (B.BF16, B.FP16, B.FP32):
        rc, st, _, ref = oracle.decode(blob, out_dtype=out_dt)
        assert rc == 0 and st == 0
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = B.decompress(d, info, status=status, out_dtype=out_dt)
        via_ct = ct.to(dtype=B.TORCH_DTYPE[out_dt]).decompress()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert got.dtype == B.TORCH_DTYPE[out_dt] and via_ct.dtype == got.dtype
        assert np.array_equal(as_bytes(got), ref.view(np.uint8).reshape(-1))
        assert np.array_equal(as_bytes(via_ct), ref.view(np.uint8).reshape(-1))


def test_compressed_tensor_on_the_gpu(oracle):
    """compress on the GPU tensor's device, decompress on two streams, restore from a state_dict
    on the GPU: all equal the oracle's decode of the stream the product encoder wrote"""
    w = synth.row_lognormal(256, 1024, seed=9).cuda()
    ct = compress(w, LatticeRANSConfig(target_bpp=4.0))
    assert ct.device.type == "cuda" and ct.dtype == torch.bfloat16
    blob = ct.blob.cpu().numpy()
    rc, st, _, ref = oracle.decode(blob)
    assert rc == 0 and st == 0
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        a = decompress(ct, stream=s1)
    with torch.cuda.stream(s2):
        b = ct.decompress(stream=s2)  # waits for the tables prepared on s1
    torch.cuda.synchronize()
    assert np.array_equal(as_bytes(a), ref.view(np.uint8).reshape(-1))
    assert np.array_equal(as_bytes(b), ref.view(np.uint8).reshape(-1))
    back = CompressedTensor.from_state_dict(ct.state_dict("m."), "m.")
    assert back.device.type == "cuda"
    rc, st, _, ref32 = oracle.decode(blob, out_dtype=B.FP32)
    got32 = back.to(dtype=torch.float32).decompress()
    assert np.array_equal(got32.cpu().numpy(), ref32)
    # relative L2 against the source, reported by the pages for lossy schemes
    rel = (got32 - w.float()).norm() / w.float().norm()
    assert float(rel) < 0.12


def test_cpu_copy_moves_to_the_gpu(oracle):
    w = synth.gaussian(128, 512, 0.02, 11)
    ct = compress(w, LatticeRANSConfig(target_bpp=3.0, container=torch.float8_e4m3fn))
    assert ct.device.type == "cpu" and ct.dtype == torch.float8_e4m3fn
    g = ct.to("cuda")
    rc, st, _, ref = oracle.decode(ct.blob.numpy())
    out = g.decompress()
    assert out.dtype == torch.float8_e4m3fn
    assert np.array_equal(as_bytes(out), ref.view(np.uint8).reshape(-1))


@pytest.mark.parametrize("container,out_dt,shape", [(B.BF16, None, (300, 1000)), (B.FP16, B.FP32, (64, 2048)),
                                                    (B.FP32, B.BF16, (17, 37)), (B.INT8, None, (128, 512)),
                                                    (B.FP8E4M3, None, (96, 808))])
def test_host_buffer_decode(oracle, container, out_dt, shape):
    """ep_decompress_host: the stream in host memory, the weights back in host memory, equal byte
    for byte to the oracle's decode; also through CompressedTensor.decompress on a CPU copy"""
    src = {B.INT8: torch.bfloat16, B.FP8E4M3: torch.bfloat16}.get(container, SRC.get(container))
    w = synth.row_lognormal(*shape, seed=shape[1], dtype=src)
    target = 6.0 if container in (B.INT8, B.FP8E4M3) else 5.0
    rc, blob = oracle.compress(w, target, container=container)
    assert rc == 0
    h = torch.from_numpy(blob).pin_memory()
    info = B.stream_info(h)
    rc, st, _, ref = oracle.decode(blob, out_dtype=out_dt or 0)
    assert rc == 0 and st == 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = B.decompress_host(h, info, out_dtype=out_dt, status=status)
    assert not got.is_cuda and int(status.item()) == 0
    assert np.array_equal(as_bytes(got), ref.view(np.uint8).reshape(-1))
    # caller-owned scratch and output, asynchronous on a side stream
    s = torch.cuda.Stream()
    scratch = torch.empty(B.decompress_host_scratch(info, out_dt), dtype=torch.uint8, device="cuda")
    out = torch.empty(info.shape, dtype=got.dtype).pin_memory()
    B.decompress_host(h, info, out=out, out_dtype=out_dt, scratch=scratch, stream=s, sync=False)
    s.synchronize()
    assert np.array_equal(as_bytes(out), ref.view(np.uint8).reshape(-1))
    if out_dt is None:
        ct = CompressedTensor(torch.from_numpy(blob), info)
        via_ct = ct.decompress()
        assert via_ct.device.type == "cpu"
        assert np.array_equal(as_bytes(via_ct), ref.view(np.uint8).reshape(-1))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32, torch.int8, torch.float8_e4m3fn])
def test_tile_ans_round_trip(dtype):
    """compress(tensor, TileANSConfig()) and decompress on the GPU, from a CUDA tensor and from a
    host-resident stream: every bit of the input, in its shape and dtype"""
    from dit_weight_compression_tile_b200.compressed import TileANSConfig
    g = torch.Generator().manual_seed(40)
    t = (torch.randn(3, 257, 129, generator=g) * (20 if dtype in (torch.int8, torch.float8_e4m3fn) else 0.02)).to(dtype)
    view = torch.int16 if t.element_size() == 2 else (torch.int32 if t.element_size() == 4 else torch.uint8)
    for src in (t, t.cuda()):
        ct = compress(src, TileANSConfig())
        assert ct.device == src.device and ct.lossless
        out = decompress(ct)
        assert out.device == src.device and out.dtype == dtype and out.shape == t.shape
        assert torch.equal(out.cpu().view(view), t.view(view))
        # a second decode reuses the prepared table
        assert torch.equal(ct.decompress().cpu().view(view), t.view(view))
