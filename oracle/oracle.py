"""ctypes binding of the C oracle (oracle/ep_oracle.c) -- test infrastructure only.

Argument marshalling between numpy arrays and the C functions; no arithmetic of the
method lives here.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
leg may import this module.
"""
import ctypes as C

import numpy as np

from . import build as _build

BF16, FP16, FP32, INT8, FP8E4M3 = 1, 2, 3, 4, 5
OK, ERR_INVALID_ARG, ERR_NONFINITE, ERR_TARGET_RANGE, ERR_TARGET_UNREACHABLE = 0, -1, -2, -3, -4
ERR_BUFFER_TOO_SMALL, ERR_CORRUPT, ERR_UNSUPPORTED = -5, -6, -8
CODING_AUTO, CODING_SINGLE, CODING_PAIRED = 0, 1, 2
ELT = {BF16: 2, FP16: 2, FP32: 4, INT8: 1, FP8E4M3: 1}
NP_DTYPE = {BF16: np.uint16, FP16: np.uint16, FP32: np.float32, INT8: np.int8, FP8E4M3: np.uint8}


class Info(C.Structure):
    _fields_ = [
        ("rows", C.c_int64), ("cols", C.c_int64),
        ("src_dtype", C.c_int32), ("container_dtype", C.c_int32),
        ("storage_nbytes", C.c_uint64), ("header_nbytes", C.c_uint64),
        ("actual_bpp", C.c_double), ("q_index", C.c_int32),
        ("n_tiles", C.c_uint32), ("blocks_per_lane", C.c_uint32),
        ("split", C.c_uint8 * 7), ("ntok", C.c_uint16 * 7),
        ("off_rowf", C.c_uint64), ("off_scales", C.c_uint64), ("off_freq", C.c_uint64),
        ("off_dir", C.c_uint64), ("off_tiles", C.c_uint64), ("paired", C.c_uint32), ("layout", C.c_uint32),
    ]


class TAInfo(C.Structure):
    _fields_ = [
        ("n", C.c_int64), ("dtype", C.c_int32), ("ndim", C.c_int32), ("shape", C.c_int64 * 8),
        ("n_tiles", C.c_uint32), ("blocks_per_lane", C.c_uint32),
        ("off_freq", C.c_uint64), ("off_dir", C.c_uint64), ("off_raw", C.c_uint64), ("off_tiles", C.c_uint64),
        ("storage_nbytes", C.c_uint64),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(_build.build())
        p = C.c_void_p
        L.or_q_of_k.restype = C.c_double
        L.or_q_of_k.argtypes = [C.c_int32]
        L.or_k_max.restype = C.c_int32
        L.or_k_max.argtypes = [C.c_int64]
        L.or_d8_nearest.argtypes = [p, p]
        L.or_e8_nearest.argtypes = [p, p]
        L.or_e8_nearest_batch.argtypes = [p, C.c_int64, p]
        L.or_zigzag.restype = C.c_uint32
        L.or_zigzag.argtypes = [C.c_int32]
        L.or_unzigzag.restype = C.c_int32
        L.or_unzigzag.argtypes = [C.c_uint32]
        L.or_tokenize_batch.argtypes = [p, C.c_int64, C.c_int32, C.c_int32, p, p, p]
        L.or_detokenize.restype = C.c_uint32
        L.or_detokenize.argtypes = [C.c_uint32, C.c_int32, C.c_int32, C.c_uint32]
        L.or_detokenize_batch.argtypes = [p, C.c_int64, C.c_int32, C.c_int32, p, p]
        L.or_alphabet_size.restype = C.c_uint32
        L.or_alphabet_size.argtypes = [C.c_int32, C.c_int32]
        L.or_block_symbols.argtypes = [p, p, p]
        L.or_block_values.argtypes = [p, p, p]
        L.or_normalize_freqs.restype = C.c_int32
        L.or_normalize_freqs.argtypes = [p, C.c_int32, p]
        L.or_normalize_freqs_to.restype = C.c_int32
        L.or_normalize_freqs_to.argtypes = [p, C.c_int32, C.c_int32, p]
        L.or_pair_table.argtypes = [p, C.c_uint32, C.c_uint64, p, p]
        L.or_choose_blocks_per_lane.restype = C.c_uint32
        L.or_choose_blocks_per_lane.argtypes = [C.c_int64, C.c_double]
        L.or_convert_batch.argtypes = [p, C.c_int64, C.c_int32, p]
        L.or_prequant.restype = C.c_int
        L.or_prequant.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_int32, p, p]
        L.or_row_factors.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_int32, C.c_int32, p, p]
        L.or_quantize.restype = C.c_int
        L.or_quantize.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_int32, C.c_int32, p]
        L.or_estimate_bpp.restype = C.c_double
        L.or_estimate_bpp.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_int32, C.c_int32, C.c_uint32,
                                      C.c_int32]
        L.or_compress.restype = C.c_int
        L.or_compress.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_double, C.c_int32, C.c_uint32,
                                  C.c_int32, C.c_int32, p, C.c_size_t, C.POINTER(C.c_size_t)]
        L.or_parse.restype = C.c_int
        L.or_parse.argtypes = [p, C.c_size_t, C.POINTER(Info)]
        L.or_decode.restype = C.c_int
        L.or_decode.argtypes = [p, C.c_size_t, C.c_uint32, C.c_uint32, p, p, C.POINTER(C.c_uint32)]
        L.or_decode_as.restype = C.c_int
        L.or_decode_as.argtypes = [p, C.c_size_t, C.c_uint32, C.c_uint32, p, p, C.c_int32, C.POINTER(C.c_uint32)]
        L.or_code_stats.restype = C.c_int
        L.or_code_stats.argtypes = [p, C.c_size_t, C.POINTER(C.c_double), C.POINTER(C.c_double),
                                    C.POINTER(C.c_double), C.POINTER(C.c_uint64), C.POINTER(C.c_uint64)]
        L.or_compress_layout.argtypes = [p, C.c_int32, C.c_int64, C.c_int64, C.c_double, C.c_int32, C.c_uint32,
                                         C.c_int32, C.c_int32, C.c_int32, p, C.c_size_t, C.POINTER(C.c_size_t)]
        L.ota_blocks_per_lane.restype = C.c_uint32
        L.ota_blocks_per_lane.argtypes = [C.c_int64]
        L.ota_compress.argtypes = [p, C.c_int32, C.c_int64, C.c_int32, p, C.c_uint32, p, C.c_size_t,
                                   C.POINTER(C.c_size_t)]
        L.ota_parse.argtypes = [p, C.c_size_t, C.POINTER(TAInfo)]
        L.ota_decode.argtypes = [p, C.c_size_t, C.c_uint32, C.c_uint32, p, C.POINTER(C.c_uint32)]
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p)


def _src(src):
    """(pointer-able contiguous array, dtype code) for a numpy array or a CPU torch tensor."""
    try:
        import torch
        if isinstance(src, torch.Tensor):
            if src.dtype == torch.bfloat16:
                return src.contiguous().view(torch.int16).numpy().view(np.uint16), BF16
            if src.dtype == torch.float16:
                return src.contiguous().view(torch.int16).numpy().view(np.uint16), FP16
            if src.dtype == torch.float32:
                return src.contiguous().numpy(), FP32
            raise TypeError(f"unsupported dtype {src.dtype}")
    except ImportError:
        pass
    a = np.ascontiguousarray(src)
    if a.dtype == np.float32:
        return a, FP32
    raise TypeError("pass a torch tensor (bf16/fp16/fp32) or a float32 array")


# ---- scalar pieces ----
def q_of_k(k):
    return lib().or_q_of_k(int(k))


def k_max(cols):
    return lib().or_k_max(int(cols))


def d8_nearest(y):
    y = np.ascontiguousarray(y, dtype=np.float64)
    r = np.zeros(8, np.float64)
    lib().or_d8_nearest(_ptr(y), _ptr(r))
    return r


def e8_nearest(x):
    """Lattice points v = 2z for blocks x of shape (..., 8)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    shp = x.shape
    x2 = x.reshape(-1, 8)
    v = np.zeros(x2.shape, np.int32)
    lib().or_e8_nearest_batch(_ptr(x2), x2.shape[0], _ptr(v))
    return v.reshape(shp)


def zigzag(y):
    return lib().or_zigzag(int(y))


def unzigzag(u):
    return lib().or_unzigzag(int(u))


# low bits kept in every token, and the largest split, per context
CTX_LOW = (2, 1, 1, 0, 0, 0, 0)
CTX_MAX_SPLIT = (9, 9, 9, 8, 8, 8, 8)


def tokenize(s, m, low):
    s = np.ascontiguousarray(s, dtype=np.uint32)
    tok = np.zeros_like(s)
    nb = np.zeros_like(s)
    ex = np.zeros_like(s)
    lib().or_tokenize_batch(_ptr(s), s.size, int(m), int(low), _ptr(tok), _ptr(nb), _ptr(ex))
    return tok, nb, ex


def detokenize(tok, m, low, extra):
    return lib().or_detokenize(int(tok), int(m), int(low), int(extra))


def detokenize_batch(tok, m, low, extra):
    tok = np.ascontiguousarray(tok, dtype=np.uint32)
    extra = np.ascontiguousarray(extra, dtype=np.uint32)
    s = np.zeros_like(tok)
    lib().or_detokenize_batch(_ptr(tok), tok.size, int(m), int(low), _ptr(extra), _ptr(s))
    return s


def alphabet_size(m, low):
    return lib().or_alphabet_size(int(m), int(low))


def block_symbols(v):
    """contexts and coded values of one block of 8 lattice coordinates v = 2z"""
    v = np.ascontiguousarray(v, dtype=np.int32)
    ctx = np.zeros(8, np.uint32)
    s = np.zeros(8, np.uint32)
    lib().or_block_symbols(_ptr(v), _ptr(ctx), _ptr(s))
    return ctx, s


def block_values(s):
    s = np.ascontiguousarray(s, dtype=np.uint32)
    v = np.zeros(8, np.int32)
    ctx = np.zeros(8, np.uint32)
    lib().or_block_values(_ptr(s), _ptr(v), _ptr(ctx))
    return v, ctx


def normalize_freqs(counts, bits=11):
    c = np.ascontiguousarray(counts, dtype=np.uint64)
    f = np.zeros(c.size, np.uint32)
    n = lib().or_normalize_freqs_to(_ptr(c), c.size, int(bits), _ptr(f))
    return f, n


def blocks_per_lane(nblocks, target_bpp):
    return lib().or_choose_blocks_per_lane(int(nblocks), float(target_bpp))


def convert(w, dtype):
    w = np.ascontiguousarray(w, dtype=np.float32)
    out = np.zeros(w.shape, NP_DTYPE[dtype])
    lib().or_convert_batch(_ptr(w), w.size, dtype, _ptr(out))
    return out


def prequant(src, container):
    a, dt = _src(src)
    R, Cc = a.shape
    codes = np.zeros((R, Cc), np.float64)
    scales = np.zeros(R, np.float32)
    lib().or_prequant(_ptr(a), dt, R, Cc, container, _ptr(codes), _ptr(scales))
    return codes, scales


def row_factors(src, k, container=0):
    a, dt = _src(src)
    R, Cc = a.shape
    s = np.zeros(R, np.float32)
    f = np.zeros(R, np.float32)
    lib().or_row_factors(_ptr(a), dt, R, Cc, container or dt, int(k), _ptr(s), _ptr(f))
    return s, f


def quantize(src, k, container=0):
    a, dt = _src(src)
    R, Cc = a.shape
    v = np.zeros((R, Cc), np.int32)
    lib().or_quantize(_ptr(a), dt, R, Cc, container or dt, int(k), _ptr(v))
    return v


def pair_table(inside, A, N):
    """(frequencies, rare flags) of a pair table: ``inside`` the B * B pair counts inside the base"""
    B = min(int(A), 40)
    c = np.ascontiguousarray(inside, dtype=np.uint64)
    assert c.size == B * B
    f = np.zeros(B * B + 1, np.uint32)
    r = np.zeros(max(B * B, 1), np.uint8)
    lib().or_pair_table(_ptr(c), int(A), int(N), _ptr(f), _ptr(r))
    return f, r[: B * B]


def estimate_bpp(src, k, container=0, blocks_per_lane=0, coding=CODING_AUTO):
    a, dt = _src(src)
    R, Cc = a.shape
    return lib().or_estimate_bpp(_ptr(a), dt, R, Cc, container or dt, int(k), blocks_per_lane, int(coding))


# ---- the stream ----
def compress(src, target_bpp, container=0, blocks_per_lane=0, q_override=-1, coding=CODING_AUTO, layout=0):
    """Returns (rc, blob as a uint8 numpy array).  ``coding``: CODING_AUTO, CODING_SINGLE or
    CODING_PAIRED (coordinates 1..6 paired whenever the alphabets allow, at any size).  ``layout``:
    0 (lanes along rows) or 1 (tiles of 128 rows x 64 columns, the block order of a consumer GEMM)."""
    a, dt = _src(src)
    R, Cc = a.shape
    n = C.c_size_t(0)
    rc = lib().or_compress_layout(_ptr(a), dt, R, Cc, float(target_bpp), container, blocks_per_lane, q_override,
                                  int(coding), int(layout), None, 0, C.byref(n))
    if rc not in (OK, ERR_BUFFER_TOO_SMALL):
        return rc, None
    out = np.zeros(n.value, np.uint8)
    rc = lib().or_compress_layout(_ptr(a), dt, R, Cc, float(target_bpp), container, blocks_per_lane, q_override,
                                  int(coding), int(layout), _ptr(out), out.size, C.byref(n))
    return rc, (out[: n.value] if rc == OK else None)


def parse(blob):
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    info = Info()
    rc = lib().or_parse(_ptr(blob), blob.size, C.byref(info))
    return rc, info


def decode(blob, t0=0, t1=None, want_v=True, want_out=True, out_buf=None, out_dtype=0):
    """Returns (rc, status, v (rows, cols) int32 or None, out (rows, cols) container array or None).
    ``out_buf``: optional preallocated container array to decode into.  ``out_dtype``: 0 (the
    container's dtype) or, for a float container, BF16 / FP16 / FP32 (to(dtype=...) of the API
    reference: the fp32 weight rounded once into that dtype)."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rc, info = parse(blob)
    if rc != OK:
        return rc, 0, None, None
    R, Cc = info.rows, info.cols
    v = np.zeros((R, Cc), np.int32) if want_v else None
    if out_buf is not None:
        out = out_buf
    else:
        out = np.zeros((R, Cc), NP_DTYPE[out_dtype or info.container_dtype]) if want_out else None
    st = C.c_uint32(0)
    t1 = info.n_tiles if t1 is None else t1
    rc = lib().or_decode_as(_ptr(blob), blob.size, t0, t1, _ptr(v) if v is not None else None,
                            _ptr(out) if out is not None else None, int(out_dtype), C.byref(st))
    return rc, st.value, v, out


def decode_parallel(blob, threads=None, want_v=True, out_dtype=0):
    """``decode`` of the whole stream with the oracle's tile decoder on several host threads:
    the tiles are independent, so each thread decodes its own contiguous range of them into the
    shared output arrays (ctypes releases the GIL during the C call).  Same results as
    ``decode``; returns (rc, status, v or None, out)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rc, info = parse(blob)
    if rc != OK:
        return rc, 0, None, None
    R, Cc = info.rows, info.cols
    v = np.zeros((R, Cc), np.int32) if want_v else None
    out = np.zeros((R, Cc), NP_DTYPE[out_dtype or info.container_dtype])
    if threads is None:
        try:
            threads = len(os.sched_getaffinity(0))
        except AttributeError:
            threads = os.cpu_count() or 1
    T = info.n_tiles
    n = max(1, min(int(threads), T))
    cuts = [(T * i) // n for i in range(n + 1)]

    def one(i):
        st = C.c_uint32(0)
        r = lib().or_decode_as(_ptr(blob), blob.size, cuts[i], cuts[i + 1], _ptr(v) if v is not None else None,
                               _ptr(out), int(out_dtype), C.byref(st))
        return r, st.value

    with ThreadPoolExecutor(n) as ex:
        res = list(ex.map(one, range(n)))
    rc = next((r for r, _ in res if r != OK), OK)
    st = 0
    for _, s_ in res:
        st |= s_
    return rc, st, v, out


def code_stats(blob):
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    ideal, H, extra = C.c_double(), C.c_double(), C.c_double()
    ns, pb = C.c_uint64(), C.c_uint64()
    rc = lib().or_code_stats(_ptr(blob), blob.size, C.byref(ideal), C.byref(H), C.byref(extra),
                             C.byref(ns), C.byref(pb))
    return rc, dict(ideal_bits=ideal.value, entropy_bits=H.value, extra_bits=extra.value,
                    n_symbols=ns.value, payload_bytes=pb.value)


# ---- the Tile-ANS lossless stream ----
TA_NP = {BF16: np.uint16, FP16: np.uint16, FP32: np.uint32, INT8: np.uint8, FP8E4M3: np.uint8}


def ta_compress(bits, dtype, shape=None, blocks_per_lane=0):
    """Tile-ANS stream of the elements ``bits`` (a numpy array of the dtype's raw bit patterns:
    uint16 for BF16 / FP16, uint32 for FP32, uint8 for INT8 / FP8).  Returns (rc, blob)."""
    a = np.ascontiguousarray(bits)
    shape = tuple(a.shape) if shape is None else tuple(shape)
    dims = (C.c_int64 * 8)(*shape)
    n = C.c_size_t(0)
    rc = lib().ota_compress(_ptr(a), dtype, a.size, len(shape), dims, blocks_per_lane, None, 0, C.byref(n))
    if rc not in (OK, ERR_BUFFER_TOO_SMALL):
        return rc, None
    out = np.zeros(n.value, np.uint8)
    rc = lib().ota_compress(_ptr(a), dtype, a.size, len(shape), dims, blocks_per_lane, _ptr(out), out.size,
                            C.byref(n))
    return rc, (out if rc == OK else None)


def ta_parse(blob):
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    info = TAInfo()
    rc = lib().ota_parse(_ptr(blob), blob.size, C.byref(info))
    return rc, info


def ta_decode(blob, t0=0, t1=None):
    """(rc, status, elements as a numpy array of the dtype's bit patterns in the stream's shape)"""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rc, info = ta_parse(blob)
    if rc != OK:
        return rc, 0, None
    out = np.zeros(info.n, TA_NP[info.dtype])
    st = C.c_uint32(0)
    t1 = info.n_tiles if t1 is None else t1
    rc = lib().ota_decode(_ptr(blob), blob.size, t0, t1, _ptr(out), C.byref(st))
    return rc, st.value, out.reshape(tuple(info.shape[: info.ndim]))
