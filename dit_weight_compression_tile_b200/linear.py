"""CompressedLinear, CompressedFP8Linear and CompressedINT8Linear of the API reference
("EntroPack API reference", CompressedLinear / CompressedFP8Linear and CompressedINT8Linear):
linear layers whose weight is held as a lattice-rANS stream and reconstructed for every forward
call.  The reconstruction is the fused decode kernel (ep_decompress) into a buffer the layer
keeps; the product is the library GEMM (cuBLAS through torch: F.linear, torch._scaled_mm for
FP8, torch._int_mm for INT8).  A BF16 layer whose stream is GEMM-ordered (LatticeRANSConfig(layout=
"gemm")) instead decodes inside its own tcgen05 GEMM (ep_linear_fused) when the call has at most
FUSED_MAX_TOKENS BF16 tokens: the weight then never passes through memory (the FP8 / INT8 layers
quantize the activations per token the same way and multiply codes with kind::f8f6f4 / kind::i8).  Above that the decode
into a buffer plus the library GEMM is faster (the fused kernel's decoding warps share each SM with
the operand buffers and go no faster with more tokens, while its X slices grow).

The FP8 / INT8 layers hold per-row absmax codes (the stream's code container) and quantize the
activations per row of x the same way (E4M3 with scale amax / 448, INT8 with amax / 127, RNE);
the GEMM multiplies codes and applies both scales to the fp32 / int32 products.
"""
import dataclasses

import torch
import torch.nn as nn
import torch.nn.functional as F

from . import binding as B
from .compressed import CompressedTensor, LatticeRANSConfig, _tables, compress, decompress

FUSED_MAX_TOKENS = 16


class CompressedLinear(nn.Module):
    """y = x W^T + b with W held compressed (lossy lattice-rANS, `config`) and decoded per call.
    A layer built by the constructor holds no weight until compress_weight runs or a checkpoint
    is loaded."""

    code_dtype = None  # the FP8 / INT8 layers store codes of this dtype

    def __init__(self, in_features, out_features, bias=True, *, config=None, device=None, dtype=torch.bfloat16):
        super().__init__()
        self.in_features, self.out_features = in_features, out_features
        self.config = config if config is not None else LatticeRANSConfig()
        if self.code_dtype is not None:
            self.config = dataclasses.replace(self.config, container=self.code_dtype)
        self.init_dtype = dtype
        self.bias = nn.Parameter(torch.zeros(out_features, device=device, dtype=dtype), requires_grad=False) \
            if bias else None
        self._weight = None
        self._buf = None  # decoded weight (or codes), reused across calls
        self._work = None  # fp32 partial sums of the fused GEMM, reused across calls

    # ---- construction
    @classmethod
    def from_linear(cls, linear, **kwargs):
        if linear.weight.is_meta:
            raise B.EpError(-1, "the source weights must be loaded (not on the meta device)")
        kwargs.setdefault("dtype", linear.weight.dtype)
        layer = cls(linear.in_features, linear.out_features, bias=linear.bias is not None,
                    device=linear.weight.device, **kwargs)
        layer.compress_weight(linear.weight.detach())
        if linear.bias is not None:
            layer.bias.data.copy_(linear.bias.detach().to(layer.bias.dtype))
        return layer

    def compress_weight(self, weight):
        if tuple(weight.shape) != (self.out_features, self.in_features):
            raise B.EpError(-1, f"weight shape {tuple(weight.shape)} is not {(self.out_features, self.in_features)}")
        src = weight.detach()
        if src.dtype not in (torch.bfloat16, torch.float16, torch.float32):
            src = src.to(self.init_dtype)
        self._weight = compress(src, self.config)
        self._buf = None

    # ---- properties of the API reference
    @property
    def weight(self):
        return self._weight

    @property
    def container_dtype(self):
        return self._weight.encoded_dtype

    @property
    def stored_nbytes(self):
        """weight storage including metadata and code scales, excluding the bias"""
        return self._weight.storage_nbytes()

    @property
    def compressed_bits(self):
        return 8.0 * self.stored_nbytes / (self.in_features * self.out_features)

    def _need(self):
        if self._weight is None:
            raise B.EpError(-1, "the layer has no weight: call compress_weight or load a checkpoint")
        return self._weight

    def _decoded(self):
        """the reconstruction of this call, into the layer's buffer"""
        w = self._need()
        if self._buf is None or self._buf.device != w.device:
            self._buf = torch.empty(tuple(w.shape), dtype=w.dtype, device=w.device)
        return decompress(w, out=self._buf)

    def dequantize(self, device=None):
        w = self._need()
        out = decompress(w).to(self.init_dtype)
        return out if device is None else out.to(device)

    def fused_for(self, x):
        """whether forward(x) decodes inside the fused GEMM (ep_linear_fused): a GEMM-ordered BF16
        stream on x's CUDA device, x BF16 with 1..FUSED_MAX_TOKENS tokens"""
        w = self._weight
        if w is None or w.compress_method != "lattice_rans" or not x.is_cuda or x.dtype != torch.bfloat16:
            return False
        info = w.info
        tokens = x.numel() // self.in_features if x.dim() else 0
        return (info.layout == B.LAYOUT_GEMM and info.container_dtype in (B.BF16, B.INT8, B.FP8E4M3)
                and w.device == x.device and 1 <= tokens <= FUSED_MAX_TOKENS)

    def _fused_forward(self, x):
        """the weight decoded inside the tcgen05 GEMM (ep_linear_fused); the FP8 / INT8 layers'
        activations are quantized per token inside the same call"""
        w = self._weight
        s = torch.cuda.current_stream(x.device)
        tables = _tables(w, s)
        bias = None if self.bias is None else self.bias.to(torch.bfloat16)
        if self._work is None or self._work.device != x.device:
            self._work = torch.zeros(B.linear_fused_workspace(w.info, FUSED_MAX_TOKENS), dtype=torch.uint8,
                                     device=x.device)
        y = B.linear_fused(x.reshape(-1, self.in_features), w.blob, w.info, tables, bias=bias, work=self._work,
                           stream=s)
        return y.reshape(*x.shape[:-1], self.out_features)

    def forward(self, x):
        if self.fused_for(x):
            return self._fused_forward(x)
        w = self._decoded()
        return F.linear(x, w.to(x.dtype) if w.dtype != x.dtype else w, self.bias)

    # ---- moving and checkpoints
    def _apply(self, fn, recurse=True):
        super()._apply(fn, recurse)
        if self._weight is not None:
            probe = fn(torch.empty(0, device=self._weight.device))
            if probe.device != self._weight.device:  # .to(device) moves the stream; dtypes stay as encoded
                self._weight = self._weight.to(probe.device)
                self._buf = self._work = None
        return self

    def _save_to_state_dict(self, destination, prefix, keep_vars):
        super()._save_to_state_dict(destination, prefix, keep_vars)
        if self._weight is not None:
            destination.update(self._weight.state_dict(prefix + "weight."))

    def _load_from_state_dict(self, state_dict, prefix, local_metadata, strict, missing_keys, unexpected_keys,
                              error_msgs):
        mine = [k for k in state_dict if k.startswith(prefix + "weight.")]
        if mine:
            w = CompressedTensor.from_state_dict({k: state_dict[k] for k in mine}, prefix + "weight.")
            if tuple(w.shape) != (self.out_features, self.in_features):
                error_msgs.append(f"{prefix}weight: shape {tuple(w.shape)} does not match the layer")
            elif self.code_dtype is not None and w.encoded_dtype != self.code_dtype:
                error_msgs.append(f"{prefix}weight: codes are {w.encoded_dtype}, the layer holds {self.code_dtype}")
            else:
                dev = self.bias.device if self.bias is not None else w.device
                self._weight = w.to(dev)
                self._buf = self._work = None
        elif strict:
            missing_keys.append(prefix + "weight.ep_meta")
        rest = {k: v for k, v in state_dict.items() if not k.startswith(prefix + "weight.")}
        super()._load_from_state_dict(rest, prefix, local_metadata, strict, missing_keys, unexpected_keys,
                                      error_msgs)
        for k in mine:
            if k in unexpected_keys:
                unexpected_keys.remove(k)

    def extra_repr(self):
        bits = f", compressed_bits={self.compressed_bits:.3f}" if self._weight is not None else ""
        return f"in_features={self.in_features}, out_features={self.out_features}, bias={self.bias is not None}{bits}"


class _CodeLinear(CompressedLinear):
    """W8A8: per-row codes of W from the stream, activations quantized per row of x"""

    def _scales(self):
        w = self._need()
        info = w.info
        return w.blob[info.off_scales: info.off_scales + 4 * info.rows].view(torch.float32)

    def codes(self, device=None):
        w = self._need()
        out = decompress(w)
        return out if device is None else out.to(device)

    def dequantize(self, device=None):
        out = (self.codes().float() * self._scales()[:, None]).to(self.init_dtype)
        return out if device is None else out.to(device)

    def _quantize_x(self, x2):
        amax = x2.abs().amax(dim=1, keepdim=True).float()
        bound = 448.0 if self.code_dtype == torch.float8_e4m3fn else 127.0
        # a correctly rounded division (tensor by tensor: torch divides by a Python number as a
        # multiplication by its reciprocal, which can differ in the last bit)
        scale = torch.where(amax > 0, amax / torch.full_like(amax, bound), torch.ones_like(amax))
        q = x2.float() / scale
        if self.code_dtype == torch.int8:
            q = q.round().clamp(-127, 127).to(torch.int8)
        else:
            q = q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
        return q, scale


class CompressedFP8Linear(_CodeLinear):
    code_dtype = torch.float8_e4m3fn

    def forward(self, x):
        if self.fused_for(x):
            return self._fused_forward(x)
        shape = x.shape
        x2 = x.reshape(-1, self.in_features)
        q, sx = self._quantize_x(x2)
        wc = self._decoded()
        y = torch._scaled_mm(q, wc.t(), scale_a=sx, scale_b=self._scales()[None, :].contiguous(),
                             out_dtype=torch.bfloat16 if x.dtype == torch.float32 else x.dtype)
        y = y.to(x.dtype)
        if self.bias is not None:
            y = y + self.bias.to(y.dtype)
        return y.reshape(*shape[:-1], self.out_features)


class CompressedINT8Linear(_CodeLinear):
    code_dtype = torch.int8

    def forward(self, x):
        if self.fused_for(x):
            return self._fused_forward(x)
        shape = x.shape
        x2 = x.reshape(-1, self.in_features)
        q, sx = self._quantize_x(x2)
        wc = self._decoded()
        acc = torch._int_mm(q, wc.t())  # int32, exact
        y = (acc.float() * sx * self._scales()[None, :]).to(x.dtype)
        if self.bias is not None:
            y = y + self.bias.to(y.dtype)
        return y.reshape(*shape[:-1], self.out_features)
