"""ctypes front end of the CPU oracle (``moe_oracle.c``) — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg use this package.  It shares no code with the CUDA path and never imports
it.  Arrays are numpy; bf16 tensors travel as their uint16 bit patterns.
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

_i64 = ctypes.c_int64
_dbl = ctypes.c_double
_p = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP); returns the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_capacity.restype = _i64
        _lib.oracle_capacity.argtypes = [_i64, _i64, _i64, _dbl]
        _lib.oracle_num_threads.restype = ctypes.c_int
        _lib.oracle_permute.restype = _i64
        _lib.oracle_moe_forward.restype = _i64
        _lib.oracle_round_bf16.restype = _dbl
        _lib.oracle_round_bf16.argtypes = [_dbl]
        _lib.oracle_e4m3_encode.restype = ctypes.c_ubyte
        _lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_decode.restype = _dbl
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_ubyte]
    return _lib


def _ptr(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """Threads the calling host thread's oracle calls use (per host thread)."""
    lib().oracle_set_num_threads(ctypes.c_int(int(n)))


def capacity(T, E, k, cf) -> int:
    return int(lib().oracle_capacity(T, E, k, float(cf)))


def router_logits(x_bits, w_router, bias=None):
    x_bits = _c(x_bits, np.uint16)
    w_router = _c(w_router, np.float32)
    bias = _c(bias, np.float32)
    T, d = x_bits.shape
    E = w_router.shape[1]
    out = np.empty((T, E), np.float64)
    lib().oracle_router_logits(_ptr(x_bits), _ptr(w_router), _ptr(bias), _i64(T), _i64(d),
                               _i64(E), _ptr(out))
    return out


def topk(logits32, k):
    logits32 = _c(logits32, np.float32)
    T, E = logits32.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    lib().oracle_topk(_ptr(logits32), _i64(T), _i64(E), _i64(k), _ptr(idx), _ptr(w))
    return idx, w


def permute(topk_idx, E, C):
    """Returns (counts[E], offsets[E+1], slot[T,k], row_src[N], n_dropped)."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    slot = np.empty((T, k), np.int32)
    row_src = np.full(T * k, -1, np.int32)
    n_drop = lib().oracle_permute(_ptr(topk_idx), _i64(T), _i64(E), _i64(k), _i64(C),
                                  _ptr(counts), _ptr(offsets), _ptr(slot), _ptr(row_src))
    return counts, offsets, slot, row_src[: offsets[E]].copy(), int(n_drop)


def dispatch(x_bits, row_src):
    x_bits = _c(x_bits, np.uint16)
    row_src = _c(row_src, np.int32)
    N = row_src.shape[0]
    d = x_bits.shape[1]
    out = np.empty((N, d), np.uint16)
    lib().oracle_dispatch(_ptr(x_bits), _ptr(row_src), _i64(N), _i64(d), _ptr(out))
    return out


def dispatch_padded(x_bits, topk_idx, slot, E, C):
    """The padded [E*C, d] buffer and its row_src (-1 on padding rows)."""
    x_bits = _c(x_bits, np.uint16)
    topk_idx, slot = _c(topk_idx, np.int32), _c(slot, np.int32)
    T, d = x_bits.shape
    k = topk_idx.shape[1]
    out = np.empty((E * C, d), np.uint16)
    row_src = np.empty(E * C, np.int32)
    lib().oracle_dispatch_padded(_ptr(x_bits), _ptr(topk_idx), _ptr(slot), _i64(T), _i64(d),
                                 _i64(k), _i64(E), _i64(C), _ptr(out), _ptr(row_src))
    return out, row_src


def round_bf16(v):
    """Nearest bf16 value (ties to even) of a double, as the oracle rounds h."""
    return lib().oracle_round_bf16(float(v))


def swiglu_rows(x_rows_bits, wg_bits, wu_bits, wd_bits, want_h=False, h_bf16=True):
    """One expert: x_rows [n,d], wg/wu [d,f], wd [f,d] (bf16 bits).  Returns
    (h [n,f] or None, o [n,d]) in fp64.  h_bf16: round h to bf16 before the
    down projection (the expert GEMMs take bf16 operands)."""
    x_rows_bits = _c(x_rows_bits, np.uint16)
    wg_bits, wu_bits, wd_bits = (_c(a, np.uint16) for a in (wg_bits, wu_bits, wd_bits))
    n, d = x_rows_bits.shape
    f = wg_bits.shape[1]
    h = np.empty((n, f), np.float64) if want_h else None
    o = np.empty((n, d), np.float64)
    lib().oracle_swiglu_rows(_ptr(x_rows_bits), _i64(n), _i64(d), _i64(f), _ptr(wg_bits),
                             _ptr(wu_bits), _ptr(wd_bits), ctypes.c_int(int(h_bf16)), _ptr(h),
                             _ptr(o))
    return h, o


def expert_mlp(x_perm_bits, offsets, w_gate_bits, w_up_bits, w_down_bits, want_h=False,
               h_bf16=True):
    x_perm_bits = _c(x_perm_bits, np.uint16)
    offsets = _c(offsets, np.int32)
    wg, wu, wd = (_c(a, np.uint16) for a in (w_gate_bits, w_up_bits, w_down_bits))
    E, d, f = wg.shape
    N = int(offsets[E])
    h = np.empty((N, f), np.float64) if want_h else None
    y = np.empty((N, d), np.float64)
    lib().oracle_expert_mlp(_ptr(x_perm_bits), _ptr(offsets), _i64(E), _i64(d), _i64(f),
                            _ptr(wg), _ptr(wu), _ptr(wd), ctypes.c_int(int(h_bf16)), _ptr(h),
                            _ptr(y))
    return h, y


def combine(y_perm, x_bits, topk_idx, topk_w, slot, offsets):
    y_perm = _c(y_perm, np.float64)
    x_bits = _c(x_bits, np.uint16)
    topk_idx = _c(topk_idx, np.int32)
    topk_w = _c(topk_w, np.float64)
    slot = _c(slot, np.int32)
    offsets = _c(offsets, np.int32)
    T, d = x_bits.shape
    k = topk_idx.shape[1]
    y = np.empty((T, d), np.float64)
    lib().oracle_combine(_ptr(y_perm), _ptr(x_bits), _ptr(topk_idx), _ptr(topk_w), _ptr(slot),
                         _ptr(offsets), _i64(T), _i64(d), _i64(k), _ptr(y))
    return y


def moe_forward(x_bits, w_router, bias, w_gate_bits, w_up_bits, w_down_bits, k, cf,
                decision_logits=None, h_bf16=True):
    """The whole layer.  Returns a dict with y [T,d] fp64 and the routing
    intermediates (logits64, topk_idx, topk_w, slot, counts, offsets, n_dropped).
    h_bf16: round h to bf16 before the down projection (default: the expert
    GEMMs take bf16 operands); False keeps the MLP entirely in fp64."""
    x_bits = _c(x_bits, np.uint16)
    w_router = _c(w_router, np.float32)
    bias = _c(bias, np.float32)
    wg, wu, wd = (_c(a, np.uint16) for a in (w_gate_bits, w_up_bits, w_down_bits))
    decision_logits = _c(decision_logits, np.float32)
    T, d = x_bits.shape
    E, _, f = wg.shape
    out = {
        "y": np.empty((T, d), np.float64),
        "logits64": np.empty((T, E), np.float64),
        "topk_idx": np.empty((T, k), np.int32),
        "topk_w": np.empty((T, k), np.float64),
        "slot": np.empty((T, k), np.int32),
        "counts": np.empty(E, np.int32),
        "offsets": np.empty(E + 1, np.int32),
    }
    n_drop = lib().oracle_moe_forward(
        _ptr(x_bits), _ptr(w_router), _ptr(bias), _ptr(wg), _ptr(wu), _ptr(wd), _i64(T), _i64(d),
        _i64(E), _i64(k), _i64(f), _dbl(cf), ctypes.c_int(int(h_bf16)), _ptr(decision_logits),
        _ptr(out["y"]),
        _ptr(out["logits64"]), _ptr(out["topk_idx"]), _ptr(out["topk_w"]), _ptr(out["slot"]),
        _ptr(out["counts"]), _ptr(out["offsets"]))
    out["n_dropped"] = int(n_drop)
    return out


def e4m3_encode(v):
    """Nearest e4m3 code (ties to even, saturating at +-448) of a float."""
    return int(lib().oracle_e4m3_encode(float(v)))


def e4m3_decode(q):
    return float(lib().oracle_e4m3_decode(int(q)))


def quantize_fp8(w_bits):
    """bf16 weights [E,K,N] (bits) -> (e4m3 codes uint8 [E,K,N], fp32 scales [E,N])."""
    w_bits = _c(w_bits, np.uint16)
    E, K, N = w_bits.shape
    q = np.empty((E, K, N), np.uint8)
    s = np.empty((E, N), np.float32)
    lib().oracle_quantize_fp8(_ptr(w_bits), _i64(E), _i64(K), _i64(N), _ptr(q), _ptr(s))
    return q, s


def dequant_fp8(q, scale):
    q = _c(q, np.uint8)
    scale = _c(scale, np.float32)
    E, K, N = q.shape
    out = np.empty((E, K, N), np.float64)
    lib().oracle_dequant_fp8(_ptr(q), _ptr(scale), _i64(E), _i64(K), _i64(N), _ptr(out))
    return out


def swiglu_rows_f64w(x_rows_bits, wg, wu, wd, want_h=False, h_bf16=True):
    """One expert with fp64 weights (e.g. dequantized FP8): x_rows [n,d] bf16
    bits, wg/wu [d,f], wd [f,d] fp64.  Returns (h or None, o) in fp64."""
    x_rows_bits = _c(x_rows_bits, np.uint16)
    wg, wu, wd = (_c(a, np.float64) for a in (wg, wu, wd))
    n, d = x_rows_bits.shape
    f = wg.shape[1]
    h = np.empty((n, f), np.float64) if want_h else None
    o = np.empty((n, d), np.float64)
    lib().oracle_swiglu_rows_f64w(_ptr(x_rows_bits), _i64(n), _i64(d), _i64(f), _ptr(wg), _ptr(wu),
                                  _ptr(wd), ctypes.c_int(int(h_bf16)), _ptr(h), _ptr(o))
    return h, o


def quantize_rows_fp8(x_bits):
    """bf16 rows [R,K] (bits) -> (e4m3 codes uint8 [R,K], fp32 row scales [R])."""
    x_bits = _c(x_bits, np.uint16)
    R, K = x_bits.shape
    q = np.empty((R, K), np.uint8)
    s = np.empty(R, np.float32)
    lib().oracle_quantize_rows_fp8(_ptr(x_bits), _i64(R), _i64(K), _ptr(q), _ptr(s))
    return q, s


def dequant_rows_fp8(q, scale):
    q = _c(q, np.uint8)
    scale = _c(scale, np.float32)
    R, K = q.shape
    out = np.empty((R, K), np.float64)
    lib().oracle_dequant_rows_fp8(_ptr(q), _ptr(scale), _i64(R), _i64(K), _ptr(out))
    return out


def gate_up_f64(a, wg, wu, h_bf16=True):
    """h = silu(a wg) * (a wu) in fp64 for a [n,d], wg/wu [d,f]; rounded to
    bf16 when h_bf16."""
    a, wg, wu = (_c(t, np.float64) for t in (a, wg, wu))
    n, d = a.shape
    f = wg.shape[1]
    h = np.empty((n, f), np.float64)
    lib().oracle_gate_up_f64(_ptr(a), _i64(n), _i64(d), _i64(f), _ptr(wg), _ptr(wu),
                             ctypes.c_int(int(h_bf16)), _ptr(h))
    return h


def matmul_f64(a, w):
    a, w = _c(a, np.float64), _c(w, np.float64)
    n, K = a.shape
    N = w.shape[1]
    out = np.empty((n, N), np.float64)
    lib().oracle_matmul_f64(_ptr(a), _i64(n), _i64(K), _ptr(w), _i64(N), _ptr(out))
    return out


def bf16_bits(t):
    """torch bf16 tensor -> numpy uint16 bit patterns (no arithmetic)."""
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(a):
    """uint16 bf16 bit patterns -> exact fp64 values."""
    a = np.asarray(a, np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
