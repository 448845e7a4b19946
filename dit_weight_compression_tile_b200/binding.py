"""Thin ctypes binding of libeptile.so (include/eptile.h): argument marshalling only.

Every step of compression runs in the library's C++ and every step of decompression in
its sm_100a kernel; this module passes torch tensors' pointers, sizes and streams.
There is no fallback: a missing library or a missing GPU raises ``EpError``.
"""
import ctypes as C
import os
import re

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libeptile.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "eptile.h")

BF16, FP16, FP32, INT8, FP8E4M3, LATTICE_I32 = 1, 2, 3, 4, 5, 6
TORCH_DTYPE = {BF16: torch.bfloat16, FP16: torch.float16, FP32: torch.float32, INT8: torch.int8,
               FP8E4M3: torch.float8_e4m3fn}
CODE_OF = {v: k for k, v in TORCH_DTYPE.items()}
NAMES = {"bf16": BF16, "fp16": FP16, "fp32": FP32, "int8": INT8, "fp8_e4m3": FP8E4M3}


class EpError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        msg = lib().ep_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{what}: {msg} ({status})" if what else f"{msg} ({status})")


class Config(C.Structure):
    _fields_ = [("target_bpp", C.c_double), ("container_dtype", C.c_int32), ("blocks_per_lane", C.c_uint32),
                ("q_index", C.c_int32), ("n_threads", C.c_int32), ("coding", C.c_int32), ("layout", C.c_int32)]


class StreamInfo(C.Structure):
    _fields_ = [
        ("rows", C.c_int64), ("cols", C.c_int64),
        ("src_dtype", C.c_int32), ("container_dtype", C.c_int32),
        ("storage_nbytes", C.c_uint64), ("header_nbytes", C.c_uint64),
        ("actual_bpp", C.c_double), ("q_index", C.c_int32),
        ("n_tiles", C.c_uint32), ("blocks_per_lane", C.c_uint32),
        ("split", C.c_uint8 * 8), ("ntok", C.c_uint16 * 8),
        ("off_rowf", C.c_uint64), ("off_scales", C.c_uint64), ("off_freq", C.c_uint64),
        ("off_dir", C.c_uint64), ("off_tiles", C.c_uint64), ("out_nbytes", C.c_uint64),
        ("max_tile_nbytes", C.c_uint64), ("workspace_nbytes", C.c_uint64), ("paired", C.c_uint32),
        ("layout", C.c_uint32),
    ]

    @property
    def shape(self):
        return (self.rows, self.cols)

    @property
    def dtype(self):
        return TORCH_DTYPE[self.container_dtype]

    def storage_nbytes_(self, include_header=True):
        return self.storage_nbytes - (0 if include_header else self.header_nbytes)


class AnsConfig(C.Structure):
    _fields_ = [("dtype", C.c_int32), ("blocks_per_lane", C.c_uint32), ("n_threads", C.c_int32),
                ("reserved", C.c_int32)]


class AnsInfo(C.Structure):
    _fields_ = [
        ("n_elems", C.c_int64), ("dtype", C.c_int32), ("ndim", C.c_int32), ("shape_", C.c_int64 * 8),
        ("storage_nbytes", C.c_uint64), ("ratio", C.c_double), ("n_tiles", C.c_uint32),
        ("blocks_per_lane", C.c_uint32), ("off_freq", C.c_uint64), ("off_dir", C.c_uint64),
        ("off_raw", C.c_uint64), ("off_tiles", C.c_uint64), ("out_nbytes", C.c_uint64),
        ("max_tile_nbytes", C.c_uint64), ("workspace_nbytes", C.c_uint64),
    ]

    @property
    def shape(self):
        return tuple(self.shape_[: self.ndim])

    @property
    def torch_dtype(self):
        return TORCH_DTYPE[self.dtype]


_lib = None


def declared_functions():
    """names of the functions include/eptile.h declares"""
    text = open(HEADER).read()
    return re.findall(r"^(?:int|size_t|const char \*)\s*\*?\s*(ep_\w+)\(", text, flags=re.M)


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m dit_weight_compression_tile_b200.build`")
        L = C.CDLL(LIB_PATH)
        p = C.c_void_p
        L.ep_compress_bound.restype = C.c_size_t
        L.ep_compress_bound.argtypes = [C.c_int64, C.c_int64, C.POINTER(Config)]
        L.ep_compress_device_scratch.restype = C.c_size_t
        L.ep_compress_device_scratch.argtypes = [C.c_int64, C.c_int64, C.POINTER(Config)]
        L.ep_compress_device.restype = C.c_int
        L.ep_compress_device.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.POINTER(Config), p, C.c_size_t,
                                         C.POINTER(C.c_size_t), p, C.c_size_t, p]
        L.ep_compress_host.restype = C.c_int
        L.ep_compress_host.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.POINTER(Config), p, C.c_size_t,
                                       C.POINTER(C.c_size_t)]
        L.ep_stream_info.restype = C.c_int
        L.ep_stream_info.argtypes = [p, C.c_size_t, C.POINTER(StreamInfo)]
        L.ep_prepare.restype = C.c_int
        L.ep_prepare.argtypes = [C.POINTER(StreamInfo), p, p, p, p]
        L.ep_decompress.restype = C.c_int
        L.ep_decompress.argtypes = [C.POINTER(StreamInfo), p, p, p, C.c_int32, p, p]
        L.ep_decompress_noalloc.restype = C.c_int
        L.ep_decompress_noalloc.argtypes = [C.POINTER(StreamInfo), p, p, C.c_int32, p, p]
        L.ep_decompress_host_scratch.restype = C.c_size_t
        L.ep_decompress_host_scratch.argtypes = [C.POINTER(StreamInfo), C.c_int32]
        L.ep_decompress_host.restype = C.c_int
        L.ep_decompress_host.argtypes = [C.POINTER(StreamInfo), p, p, C.c_int32, p, C.c_size_t, p, p]
        L.ep_linear_fused_workspace.restype = C.c_size_t
        L.ep_linear_fused_workspace.argtypes = [C.POINTER(StreamInfo), C.c_int64]
        L.ep_linear_fused_plan.restype = C.c_int
        L.ep_linear_fused_plan.argtypes = [C.POINTER(StreamInfo), C.c_int64, C.c_int32, C.POINTER(LinearPlan)]
        L.ep_linear_fused.restype = C.c_int
        L.ep_linear_fused.argtypes = [C.POINTER(StreamInfo), p, p, p, C.c_int64, p, p, p, C.c_size_t, p, p]
        L.ep_ans_compress_bound.restype = C.c_size_t
        L.ep_ans_compress_bound.argtypes = [C.c_int64, C.c_int32]
        L.ep_ans_compress_host.restype = C.c_int
        L.ep_ans_compress_host.argtypes = [p, C.c_int64, C.c_int32, p, C.POINTER(AnsConfig), p, C.c_size_t,
                                           C.POINTER(C.c_size_t)]
        L.ep_ans_stream_info.restype = C.c_int
        L.ep_ans_stream_info.argtypes = [p, C.c_size_t, C.POINTER(AnsInfo)]
        L.ep_ans_prepare.restype = C.c_int
        L.ep_ans_prepare.argtypes = [C.POINTER(AnsInfo), p, p, p, p]
        L.ep_ans_decompress.restype = C.c_int
        L.ep_ans_decompress.argtypes = [C.POINTER(AnsInfo), p, p, p, p, p]
        L.ep_status_string.restype = C.c_char_p
        L.ep_status_string.argtypes = [C.c_int]
        _lib = L
    return _lib


CODING_AUTO, CODING_SINGLE, CODING_PAIRED = 0, 1, 2
LAYOUT_ROWS, LAYOUT_GEMM = 0, 1


def _config(target_bpp, container=0, blocks_per_lane=0, q_index=-1, n_threads=0, coding=CODING_AUTO,
            layout=LAYOUT_ROWS):
    if isinstance(container, str):
        container = NAMES[container]
    if isinstance(container, torch.dtype):
        container = CODE_OF[container]
    return Config(float(target_bpp), int(container or 0), int(blocks_per_lane), int(q_index), int(n_threads),
                  int(coding), int(layout))


def compress(tensor, target_bpp, container=0, blocks_per_lane=0, q_index=-1, n_threads=0, coding=CODING_AUTO,
             layout=LAYOUT_ROWS):
    """compress(tensor, config) on the host: returns the stream as a CPU uint8 tensor.

    ``tensor``: 2-D BF16/FP16/FP32 (moved to the CPU if needed).  ``container``: 0 (same as
    the source), a dtype code / name / torch dtype; INT8 and FP8 store per-row absmax codes.
    ``coding``: CODING_AUTO, CODING_SINGLE or CODING_PAIRED (ep_config.coding).  ``layout``:
    LAYOUT_ROWS, or LAYOUT_GEMM for tiles that are a consumer GEMM's 128 x 64 operand tiles."""
    if tensor.dim() != 2 or tensor.numel() == 0:
        raise EpError(-1, "compress needs a non-empty 2-D tensor")
    src = tensor.detach().to("cpu").contiguous()
    if src.dtype not in (torch.bfloat16, torch.float16, torch.float32):
        raise EpError(-8, f"source dtype {src.dtype}")
    cfg = _config(target_bpp, container, blocks_per_lane, q_index, n_threads, coding, layout)
    L = lib()
    cap = L.ep_compress_bound(src.shape[0], src.shape[1], C.byref(cfg))
    out = torch.empty(max(cap, 64), dtype=torch.uint8)
    n = C.c_size_t(0)
    rc = L.ep_compress_host(src.data_ptr(), CODE_OF[src.dtype], src.shape[0], src.shape[1], C.byref(cfg),
                            out.data_ptr(), out.numel(), C.byref(n))
    if rc == -5:  # the bound is a guarantee; this is a second chance, not the normal path
        out = torch.empty(n.value, dtype=torch.uint8)
        rc = L.ep_compress_host(src.data_ptr(), CODE_OF[src.dtype], src.shape[0], src.shape[1], C.byref(cfg),
                                out.data_ptr(), out.numel(), C.byref(n))
    if rc != 0:
        raise EpError(rc, "ep_compress_host")
    return out[: n.value].clone()


def compress_device(tensor, target_bpp, container=0, blocks_per_lane=0, q_index=-1, stream=None,
                    coding=CODING_AUTO, layout=LAYOUT_ROWS):
    """compress(tensor, config) for a CUDA tensor (ep_compress_device): the same stream as
    ``compress`` byte for byte, built on the GPU.  Returns a CUDA uint8 tensor."""
    if tensor.dim() != 2 or tensor.numel() == 0:
        raise EpError(-1, "compress needs a non-empty 2-D tensor")
    if not tensor.is_cuda:
        raise EpError(-1, "compress_device needs a CUDA tensor")
    src = tensor.detach().contiguous()
    if src.dtype not in (torch.bfloat16, torch.float16, torch.float32):
        raise EpError(-8, f"source dtype {src.dtype}")
    cfg = _config(target_bpp, container, blocks_per_lane, q_index, 0, coding, layout)
    L = lib()
    R, Cc = src.shape
    scratch = torch.empty(max(1, L.ep_compress_device_scratch(R, Cc, C.byref(cfg))), dtype=torch.uint8,
                          device=src.device)
    cap = L.ep_compress_bound(R, Cc, C.byref(cfg))
    out = torch.empty(max(cap, 64), dtype=torch.uint8, device=src.device)
    n = C.c_size_t(0)
    s = (stream or torch.cuda.current_stream(src.device)).cuda_stream
    rc = L.ep_compress_device(src.data_ptr(), CODE_OF[src.dtype], R, Cc, C.byref(cfg), out.data_ptr(), out.numel(),
                              C.byref(n), scratch.data_ptr(), scratch.numel(), s)
    if rc != 0:
        raise EpError(rc, "ep_compress_device")
    return out[: n.value].clone()


def stream_info(blob):
    """CompressedTensor properties from a host copy of the stream (CPU uint8 tensor)."""
    b = blob.detach().to("cpu").contiguous()
    info = StreamInfo()
    rc = lib().ep_stream_info(b.data_ptr(), b.numel(), C.byref(info))
    if rc != 0:
        raise EpError(rc, "ep_stream_info")
    return info


def prepare(d_blob, info=None, workspace=None, status=None, stream=None):
    """The decoder's slot tables for one device copy of a stream (ep_prepare): run once when the
    stream lands on the device.  Returns the workspace (CUDA uint8 tensor of
    ``info.workspace_nbytes``), allocated here unless ``workspace`` is given."""
    if not d_blob.is_cuda:
        raise EpError(-1, "prepare needs the stream in device memory")
    if info is None:
        info = stream_info(d_blob.cpu())
    if workspace is None:
        workspace = torch.empty(info.workspace_nbytes, dtype=torch.uint8, device=d_blob.device)
    if (not workspace.is_cuda or workspace.dtype != torch.uint8 or workspace.numel() < info.workspace_nbytes
            or not workspace.is_contiguous()):
        raise EpError(-1, "workspace does not match the stream")
    st = status.data_ptr() if status is not None else None
    s = (stream or torch.cuda.current_stream(d_blob.device)).cuda_stream
    rc = lib().ep_prepare(C.byref(info), d_blob.data_ptr(), workspace.data_ptr(), st, s)
    if rc != 0:
        raise EpError(rc, "ep_prepare")
    return workspace


def dtype_code(d):
    """EP_* dtype code of a torch dtype, a name ("bf16", ...) or a code"""
    if isinstance(d, torch.dtype):
        if d not in CODE_OF:
            raise EpError(-1, f"no container dtype for {d}")
        return CODE_OF[d]
    if isinstance(d, str):
        return NAMES[d]
    return int(d)


def decompress(d_blob, info=None, workspace=None, out=None, status=None, stream=None, lattice=False,
               out_dtype=None):
    """decompress(compressed): the fused GPU decode of a device-resident stream.

    ``d_blob``: CUDA uint8 tensor holding the whole stream.  ``info``: from ``stream_info``
    (parsed from ``d_blob`` through a host copy when omitted).  ``workspace``: from ``prepare``
    on this ``d_blob``.  When omitted, every call allocates a workspace and runs ``prepare``
    again on the same stream (a few microseconds of table building per call); callers that
    decode one stream repeatedly should prepare once and pass the workspace, as
    ``CompressedTensor`` does.  ``out``: optional CUDA
    tensor of ``info.shape`` / ``info.dtype``.  ``status``: optional CUDA int32 tensor of one
    element into which damage flags are ORed.  Launches on ``stream`` (default: the current
    stream).  ``lattice=True`` returns the decoded lattice points v = 2z (int32) instead of
    weights.  ``out_dtype``: for a BF16 / FP16 / FP32 container, any of the three (the fp32
    weight rounded once into it); default the container's dtype."""
    if not d_blob.is_cuda:
        raise EpError(-1, "decompress needs the stream in device memory")
    if info is None:
        info = stream_info(d_blob.cpu())
    if workspace is None:
        workspace = prepare(d_blob, info, status=status, stream=stream)
    dt = LATTICE_I32 if lattice else (info.container_dtype if out_dtype is None else dtype_code(out_dtype))
    want = torch.int32 if lattice else TORCH_DTYPE.get(dt)
    if want is None:
        raise EpError(-1, f"output dtype code {dt}")
    if out is None:
        out = torch.empty(info.shape, dtype=want, device=d_blob.device)
    if not out.is_cuda or out.dtype != want or tuple(out.shape) != info.shape or not out.is_contiguous():
        raise EpError(-1, "output tensor does not match the stream")
    st = status.data_ptr() if status is not None else None
    s = (stream or torch.cuda.current_stream(d_blob.device)).cuda_stream
    rc = lib().ep_decompress(C.byref(info), d_blob.data_ptr(), workspace.data_ptr(), out.data_ptr(), dt, st, s)
    if rc != 0:
        raise EpError(rc, "ep_decompress")
    return out


def decompress_host_scratch(info, out_dtype=None):
    """bytes of device scratch that ``decompress_host`` needs (ep_decompress_host_scratch)"""
    dt = info.container_dtype if out_dtype is None else dtype_code(out_dtype)
    return int(lib().ep_decompress_host_scratch(C.byref(info), dt))


def decompress_host(h_blob, info=None, out=None, out_dtype=None, scratch=None, status=None, stream=None,
                    device=None, sync=True):
    """decompress(compressed) for a stream in host memory (ep_decompress_host): the stream is
    copied to the GPU, decoded by the fused kernel there and the weights copied back into a host
    tensor, all on one CUDA stream.  ``h_blob``: CPU uint8 tensor (pinned memory lets the copies
    run without staging).  ``out``: optional CPU tensor of ``info.shape`` and the output dtype.
    ``scratch``: optional CUDA uint8 tensor of ``decompress_host_scratch`` bytes, allocated on
    ``device`` (default: the current CUDA device) when omitted.  With ``sync`` the call waits for
    the stream before returning; otherwise ``out`` is valid once ``stream`` has been synchronised."""
    if h_blob.is_cuda or h_blob.dtype != torch.uint8 or not h_blob.is_contiguous():
        raise EpError(-1, "decompress_host takes the stream as a contiguous CPU uint8 tensor")
    if not torch.cuda.is_available():
        raise EpError(-1, "decompress_host decodes on a CUDA device and none is available")
    if info is None:
        info = stream_info(h_blob)
    dt = info.container_dtype if out_dtype is None else dtype_code(out_dtype)
    want = TORCH_DTYPE.get(dt)
    if want is None:
        raise EpError(-1, f"output dtype code {dt}")
    if out is None:
        out = torch.empty(info.shape, dtype=want, pin_memory=True)
    if out.is_cuda or out.dtype != want or tuple(out.shape) != info.shape or not out.is_contiguous():
        raise EpError(-1, "output tensor does not match the stream")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    need = decompress_host_scratch(info, dt)
    if scratch is None:
        scratch = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if not scratch.is_cuda or scratch.dtype != torch.uint8 or scratch.numel() < need:
        raise EpError(-1, "scratch does not match the stream")
    st = status.data_ptr() if status is not None else None
    cs = stream or torch.cuda.current_stream(scratch.device)
    with torch.cuda.device(scratch.device):
        rc = lib().ep_decompress_host(C.byref(info), h_blob.data_ptr(), out.data_ptr(), dt, scratch.data_ptr(),
                                      scratch.numel(), st, cs.cuda_stream)
    if rc != 0:
        raise EpError(rc, "ep_decompress_host")
    if sync:
        cs.synchronize()
    return out


# ---------------------------------------------------------------- the Tile-ANS lossless scheme
def ans_compress(tensor, blocks_per_lane=0, n_threads=0):
    """compress(tensor, TileANSConfig()) on the host (ep_ans_compress_host): every bit of a BF16,
    FP16, FP32, INT8 or FP8 E4M3 tensor of any shape (1 to 8 dims).  Returns the stream as a CPU
    uint8 tensor."""
    if tensor.dtype not in CODE_OF:
        raise EpError(-1, f"Tile-ANS takes BF16, FP16, FP32, INT8 or FP8 E4M3, not {tensor.dtype}")
    if tensor.numel() == 0 or tensor.dim() < 1 or tensor.dim() > 8:
        raise EpError(-1, "Tile-ANS needs a non-empty tensor of 1 to 8 dims")
    src = tensor.detach().to("cpu").contiguous()
    cfg = AnsConfig(CODE_OF[src.dtype], int(blocks_per_lane), int(n_threads), 0)
    dims = (C.c_int64 * 8)(*src.shape)
    L = lib()
    cap = L.ep_ans_compress_bound(src.numel(), cfg.dtype)
    out = torch.empty(max(cap, 1024), dtype=torch.uint8)
    n = C.c_size_t(0)
    rc = L.ep_ans_compress_host(src.data_ptr(), src.numel(), src.dim(), dims, C.byref(cfg), out.data_ptr(),
                                out.numel(), C.byref(n))
    if rc == -5:
        out = torch.empty(n.value, dtype=torch.uint8)
        rc = L.ep_ans_compress_host(src.data_ptr(), src.numel(), src.dim(), dims, C.byref(cfg), out.data_ptr(),
                                    out.numel(), C.byref(n))
    if rc != 0:
        raise EpError(rc, "ep_ans_compress_host")
    return out[: n.value].clone()


def ans_stream_info(blob):
    b = blob.detach().to("cpu").contiguous()
    info = AnsInfo()
    rc = lib().ep_ans_stream_info(b.data_ptr(), b.numel(), C.byref(info))
    if rc != 0:
        raise EpError(rc, "ep_ans_stream_info")
    return info


def ans_prepare(d_blob, info, workspace=None, status=None, stream=None):
    """the decoder's slot table for one device copy of a Tile-ANS stream (ep_ans_prepare)"""
    if not d_blob.is_cuda:
        raise EpError(-1, "ans_prepare needs the stream in device memory")
    if workspace is None:
        workspace = torch.empty(info.workspace_nbytes, dtype=torch.uint8, device=d_blob.device)
    if not workspace.is_cuda or workspace.numel() < info.workspace_nbytes:
        raise EpError(-1, "workspace does not match the stream")
    st = status.data_ptr() if status is not None else None
    s = (stream or torch.cuda.current_stream(d_blob.device)).cuda_stream
    rc = lib().ep_ans_prepare(C.byref(info), d_blob.data_ptr(), workspace.data_ptr(), st, s)
    if rc != 0:
        raise EpError(rc, "ep_ans_prepare")
    return workspace


def ans_decompress(d_blob, info, workspace=None, out=None, status=None, stream=None):
    """decompress of a device-resident Tile-ANS stream (ep_ans_decompress): the tensor, bit for bit.
    Without ``workspace`` the table is prepared here on every call."""
    if not d_blob.is_cuda:
        raise EpError(-1, "ans_decompress needs the stream in device memory")
    if workspace is None:
        workspace = ans_prepare(d_blob, info, status=status, stream=stream)
    want = TORCH_DTYPE[info.dtype]
    if out is None:
        out = torch.empty(info.shape, dtype=want, device=d_blob.device)
    if not out.is_cuda or out.dtype != want or tuple(out.shape) != info.shape or not out.is_contiguous():
        raise EpError(-1, "output tensor does not match the stream")
    st = status.data_ptr() if status is not None else None
    s = (stream or torch.cuda.current_stream(d_blob.device)).cuda_stream
    rc = lib().ep_ans_decompress(C.byref(info), d_blob.data_ptr(), workspace.data_ptr(), out.data_ptr(), st, s)
    if rc != 0:
        raise EpError(rc, "ep_ans_decompress")
    return out


# ---------------------------------------------------------------- the decode fused into a GEMM
class LinearPlan(C.Structure):
    """ep_linear_plan: the launch ep_linear_fused would make (grid, warps, shared-memory layout)"""
    _fields_ = [(n, C.c_uint32) for n in ("bands", "ctas", "tiles_per_cta", "accumulators", "spread", "splits",
                                          "decoding_warps", "threads",
                                          "tokens_padded", "tmem_columns", "tile_buffer_bytes", "smem_tables_bytes",
                                          "smem_barriers_offset", "smem_tiles_offset", "smem_slices_offset",
                                          "smem_x_offset", "smem_x_bytes_per_warp")] + \
               [("smem_bytes", C.c_uint64), ("work_bytes", C.c_uint64)]


def linear_fused_plan(info, m, sms):
    """(status, LinearPlan) of ep_linear_fused for m tokens on a GPU with `sms` multiprocessors,
    computed on the host"""
    plan = LinearPlan()
    rc = lib().ep_linear_fused_plan(C.byref(info), m, sms, C.byref(plan))
    return rc, plan


def linear_fused_workspace(info, m):
    """bytes of scratch ep_linear_fused needs for m tokens (0: the stream or m is not one it takes)"""
    return int(lib().ep_linear_fused_workspace(C.byref(info), m))


def linear_fused(x, d_blob, info, tables, bias=None, out=None, work=None, status=None, stream=None):
    """Y = X W^T (+ bias) with W decoded inside the tcgen05 GEMM (ep_linear_fused).  ``x``: CUDA
    BF16 (m, K) with 1 <= m <= 128; ``d_blob``: a GEMM-ordered (LAYOUT_GEMM) BF16, INT8 or FP8
    stream on the device (INT8 / FP8: the activations are quantized per token and the codes
    multiplied); ``tables``: from ``prepare``; ``work``: scratch of linear_fused_workspace bytes,
    zero-filled before its first use (the call leaves it reusable; a new one is zero-allocated
    when absent or too small).  Returns the BF16 (m, N) output."""
    if not (x.is_cuda and d_blob.is_cuda and tables.is_cuda):
        raise EpError(-1, "linear_fused works on CUDA tensors")
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[1] != info.cols:
        raise EpError(-1, "x must be a BF16 (m, in_features) tensor")
    x = x.contiguous()
    m = x.shape[0]
    L = lib()
    need = linear_fused_workspace(info, m)
    if need == 0:
        raise EpError(-1, "ep_linear_fused takes a GEMM-ordered BF16 / INT8 / FP8 stream and 1 <= m <= 128")
    if work is None or work.numel() * work.element_size() < need:
        work = torch.zeros(need, dtype=torch.uint8, device=x.device)
    elif not (work.is_cuda and work.is_contiguous()):
        raise EpError(-1, "work must be a contiguous CUDA tensor")
    if out is None:
        out = torch.empty((m, info.rows), dtype=torch.bfloat16, device=x.device)
    elif not (out.is_cuda and out.dtype == torch.bfloat16 and out.is_contiguous() and out.numel() == m * info.rows):
        raise EpError(-1, "out must be a contiguous CUDA BF16 tensor of m x out_features elements")
    if bias is not None:
        bias = bias.contiguous()
        if not bias.is_cuda or bias.dtype != torch.bfloat16 or bias.numel() != info.rows:
            raise EpError(-1, "bias must be a CUDA BF16 tensor with out_features elements")
    st = status.data_ptr() if status is not None else None
    s = (stream or torch.cuda.current_stream(x.device)).cuda_stream
    rc = L.ep_linear_fused(C.byref(info), d_blob.data_ptr(), tables.data_ptr(), x.data_ptr(), m,
                           bias.data_ptr() if bias is not None else None, out.data_ptr(), work.data_ptr(),
                           work.numel() * work.element_size(), st, s)
    if rc != 0:
        raise EpError(rc, "ep_linear_fused")
    return out
