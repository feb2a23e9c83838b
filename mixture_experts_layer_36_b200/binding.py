"""Python binding of libmoe (sparse MoE layer forward on one B200).

Thin ctypes marshalling over the C ABI declared in ``include/moe.h``: the
functions below carry the same names, check dtypes / devices / shapes, pass
raw device pointers and torch's current CUDA stream, and raise on any non-OK
status.  Every step of the layer runs in the library's CUDA kernels; nothing
here computes.  If ``libmoe.so`` is missing the import fails loudly — there is
no fallback path.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_WORKSPACE", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_UNSUPPORTED", 5: "MOE_ERR_DEVICE_CHECK"}
DEV_ERR_WAIT_TIMEOUT = 1
DEV_ERR_BAD_OFFSETS = 2

# workspace fields of moe_layer_forward (enum moe_ws_field)
WS_FIELDS = ["status", "logits", "topk_idx", "topk_w", "slot", "counts", "offsets", "n_dropped",
             "row_src", "permute", "x_perm", "h", "y_perm", "route", "xq", "sx", "hq", "sh",
             "xq_tok", "sx_tok", "row_pair", "y32"]

EXPORTED = ["moe_status_string", "moe_version", "moe_selftest_bounded_wait", "moe_capacity",
            "moe_max_rows",
            "moe_route_workspace_size", "moe_permute_workspace_size", "moe_workspace_size", "moe_workspace_field_offset",
            "moe_route", "moe_permute", "moe_permute_noalloc", "moe_expert_gate_up", "moe_expert_down", "moe_expert_mlp",
            "moe_combine", "moe_combine_bf16rows", "moe_rows_to_bf16", "moe_layer_forward", "moe_quantize_weights_fp8",
            "moe_quantize_rows_fp8", "moe_permute_fp8", "moe_expert_gate_up_fp8", "moe_expert_down_fp8",
            "moe_workspace_size_fp8", "moe_layer_forward_fp8", "moe_padded_rows",
            "moe_permute_padded", "moe_permute_fused", "moe_expert_gate_up_gather",
            "moe_expert_down_scatter", "moe_combine_finalize", "moe_workspace_size_fused",
            "moe_layer_forward_fused", "moe_expert_mlp_buckets", "moe_layer_forward_ex"]


class MoEError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe.so not built at {LIB_PATH}; run "
                          "`python -m mixture_experts_layer_36_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    i64, dbl, p, sz = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_version": (ctypes.c_int, []),
        "moe_selftest_bounded_wait": (ctypes.c_int, [p, i64, p]),
        "moe_capacity": (i64, [i64, i64, i64, dbl]),
        "moe_max_rows": (i64, [i64, i64, i64, dbl]),
        "moe_route_workspace_size": (sz, [i64, i64, i64, i64]),
        "moe_permute_workspace_size": (sz, [i64, i64, i64]),
        "moe_workspace_size": (sz, [i64, i64, i64, i64, i64, dbl]),
        "moe_workspace_field_offset": (i64, [ctypes.c_int, i64, i64, i64, i64, i64, dbl]),
        "moe_route": (ctypes.c_int, [p, p, p, i64, i64, i64, i64, p, p, p, p, sz, p, p]),
        "moe_permute": (ctypes.c_int, [p, p, i64, i64, i64, i64, dbl, p, p, p, p, p, p, p, sz, p,
                                       p]),
        "moe_permute_noalloc": (ctypes.c_int, [p, p, i64, i64, i64, i64, dbl, p, p, p, p, p, p, p,
                                               p]),
        "moe_expert_gate_up": (ctypes.c_int, [p, p, i64, i64, i64, i64, p, p, p, p, p]),
        "moe_expert_down": (ctypes.c_int, [p, p, i64, i64, i64, i64, p, p, p, p]),
        "moe_expert_mlp": (ctypes.c_int, [p, p, i64, i64, i64, i64, p, p, p, p, p, p, p]),
        "moe_combine": (ctypes.c_int, [p, p, p, p, p, p, i64, i64, i64, p, p]),
        "moe_combine_bf16rows": (ctypes.c_int, [p, p, p, p, p, p, i64, i64, i64, p, p]),
        "moe_rows_to_bf16": (ctypes.c_int, [p, p, i64, i64, p]),
        "moe_layer_forward": (ctypes.c_int, [p, p, p, p, p, p, i64, i64, i64, i64, i64, dbl, p, p,
                                             sz, p]),
        "moe_layer_forward_ex": (ctypes.c_int, [p, p, p, p, p, p, i64, i64, i64, i64, i64, dbl, p,
                                                p, p, p, p, p, p, sz, p]),
        "moe_quantize_weights_fp8": (ctypes.c_int, [p, i64, i64, i64, p, p, p]),
        "moe_quantize_rows_fp8": (ctypes.c_int, [p, i64, i64, p, p, p, p]),
        "moe_permute_fp8": (ctypes.c_int, [p, p, p, i64, i64, i64, i64, dbl, p, p, p, p, p, p, p,
                                           p, sz, p, p]),
        "moe_expert_gate_up_fp8": (ctypes.c_int, [p, p, p, i64, i64, i64, i64, p, p, p, p, p, p,
                                                  p]),
        "moe_expert_down_fp8": (ctypes.c_int, [p, p, p, i64, i64, i64, i64, p, p, p, p, p]),
        "moe_workspace_size_fp8": (sz, [i64, i64, i64, i64, i64, dbl]),
        "moe_padded_rows": (i64, [i64, i64, i64, dbl]),
        "moe_expert_mlp_buckets": (ctypes.c_int, [p, p, p, i64, i64, i64, i64, i64, p, p, p, p, p,
                                                  p, p]),
        "moe_permute_fused": (ctypes.c_int, [p, p, i64, i64, i64, i64, dbl, p, p, p, p, p, p, p,
                                             p, p, sz, p, p]),
        "moe_expert_gate_up_gather": (ctypes.c_int, [p, i64, p, p, i64, i64, i64, i64, p, p, p, p,
                                                     p]),
        "moe_expert_down_scatter": (ctypes.c_int, [p, p, i64, i64, i64, i64, p, p, p, i64, p, p,
                                                   p]),
        "moe_combine_finalize": (ctypes.c_int, [p, p, p, i64, i64, i64, p, p]),
        "moe_workspace_size_fused": (sz, [i64, i64, i64, i64, i64, dbl]),
        "moe_layer_forward_fused": (ctypes.c_int, [p, p, p, p, p, p, i64, i64, i64, i64, i64, dbl,
                                                   p, p, sz, p]),
        "moe_permute_padded": (ctypes.c_int, [p, p, i64, i64, i64, i64, dbl, p, p, p, p, p, p, p,
                                              sz, p, p]),
        "moe_layer_forward_fp8": (ctypes.c_int, [p, p, p, p, p, p, p, p, p, i64, i64, i64, i64, i64,
                                                 dbl, p, p, sz, p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, st):
    if st != MOE_OK:
        raise MoEError(name, st)


def _want(t, name, dtype, shape=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


# ----------------------------------------------------------------- size queries

def moe_capacity(T, E, k, cf):
    return int(_lib.moe_capacity(T, E, k, float(cf)))


def moe_max_rows(T, E, k, cf):
    return int(_lib.moe_max_rows(T, E, k, float(cf)))


def moe_route_workspace_size(T, d, E, k):
    return int(_lib.moe_route_workspace_size(T, d, E, k))


def moe_permute_workspace_size(T, E, k):
    return int(_lib.moe_permute_workspace_size(T, E, k))


def moe_workspace_size(T, d, E, k, f, cf):
    return int(_lib.moe_workspace_size(T, d, E, k, f, float(cf)))


def moe_workspace_field_offset(field, T, d, E, k, f, cf):
    if isinstance(field, str):
        field = WS_FIELDS.index(field)
    return int(_lib.moe_workspace_field_offset(field, T, d, E, k, f, float(cf)))


def moe_version():
    return int(_lib.moe_version())


def moe_selftest_bounded_wait(dev_status, limit_ns, stream=None):
    """Run the bounded-wait self-test kernel (see include/moe.h)."""
    _want(dev_status, "dev_status", torch.int32, (1,))
    _check("moe_selftest_bounded_wait",
           _lib.moe_selftest_bounded_wait(_ptr(dev_status), int(limit_ns), _stream(stream)))


def moe_status_string(status):
    return _lib.moe_status_string(status).decode()


# ----------------------------------------------------------------- stages

def moe_route(x, w_router, bias, k, logits=None, topk_idx=None, topk_w=None, ws=None,
              dev_status=None, stream=None):
    """Router + top-k gating.  Returns (logits f32 [T,E], topk_idx i32 [T,k], topk_w f32 [T,k])."""
    T, d = x.shape
    E = w_router.shape[1]
    _want(x, "x", torch.bfloat16)
    _want(w_router, "w_router", torch.float32, (d, E))
    if bias is not None:
        _want(bias, "bias", torch.float32, (E,))
    dev = x.device
    logits = torch.empty(T, E, dtype=torch.float32, device=dev) if logits is None else logits
    topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty(T, k, dtype=torch.float32, device=dev) if topk_w is None else topk_w
    _want(logits, "logits", torch.float32, (T, E))
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    _want(topk_w, "topk_w", torch.float32, (T, k))
    if ws is None:
        ws = torch.empty(max(moe_route_workspace_size(T, d, E, k), 16), dtype=torch.uint8,
                         device=dev)
    _want(ws, "ws", torch.uint8)
    _check("moe_route", _lib.moe_route(_ptr(x), _ptr(w_router), _ptr(bias), T, d, E, k,
                                       _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(ws),
                                       ws.numel(), _ptr(dev_status), _stream(stream)))
    return logits, topk_idx, topk_w


def moe_permute(x, topk_idx, E, cf, out=None, ws=None, dev_status=None, stream=None):
    """Capacity-limited permutation.  Returns a dict with counts, offsets, slot,
    row_src, x_perm (max_rows rows; rows >= offsets[E] untouched), n_dropped."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    rows = moe_max_rows(T, E, k, cf)
    dev = x.device
    if out is None:
        out = {
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "slot": torch.empty(T, k, dtype=torch.int32, device=dev),
            "row_src": torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
            "x_perm": torch.empty(max(rows, 1), d, dtype=torch.bfloat16, device=dev),
            "n_dropped": torch.empty(1, dtype=torch.int32, device=dev),
        }
    nbytes = moe_permute_workspace_size(T, E, k)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    _want(ws, "ws", torch.uint8)
    _check("moe_permute", _lib.moe_permute(
        _ptr(x), _ptr(topk_idx), T, d, E, k, float(cf), _ptr(out["counts"]),
        _ptr(out["offsets"]), _ptr(out["slot"]), _ptr(out["row_src"]), _ptr(out["x_perm"]),
        _ptr(out["n_dropped"]), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))
    return out


def moe_permute_noalloc(x, topk_idx, E, cf, out, dev_status=None, stream=None):
    """moe_permute for callers that cannot provide scratch memory: the library
    uses a fixed array of its own (shared by every call; see include/moe.h).
    `out` holds the caller's output tensors, as returned by moe_permute."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    _check("moe_permute_noalloc", _lib.moe_permute_noalloc(
        _ptr(x), _ptr(topk_idx), T, d, E, k, float(cf), _ptr(out["counts"]),
        _ptr(out["offsets"]), _ptr(out["slot"]), _ptr(out["row_src"]), _ptr(out["x_perm"]),
        _ptr(out["n_dropped"]), _ptr(dev_status), _stream(stream)))
    return out


def moe_expert_gate_up(x_perm, offsets, w_gate, w_up, h=None, dev_status=None, stream=None):
    rows, d = x_perm.shape
    E, _, f = w_gate.shape
    _want(x_perm, "x_perm", torch.bfloat16)
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=x_perm.device) if h is None else h
    _want(h, "h", torch.bfloat16, (rows, f))
    _check("moe_expert_gate_up", _lib.moe_expert_gate_up(
        _ptr(x_perm), _ptr(offsets), E, d, f, rows, _ptr(w_gate), _ptr(w_up), _ptr(h),
        _ptr(dev_status), _stream(stream)))
    return h


def moe_expert_down(h, offsets, w_down, y_perm=None, dev_status=None, stream=None):
    rows, f = h.shape
    E, _, d = w_down.shape
    _want(h, "h", torch.bfloat16)
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    y_perm = torch.empty(rows, d, dtype=torch.float32, device=h.device) if y_perm is None \
        else y_perm
    _want(y_perm, "y_perm", torch.float32, (rows, d))
    _check("moe_expert_down", _lib.moe_expert_down(
        _ptr(h), _ptr(offsets), E, d, f, rows, _ptr(w_down), _ptr(y_perm), _ptr(dev_status),
        _stream(stream)))
    return y_perm


def moe_expert_mlp(x_perm, offsets, w_gate, w_up, w_down, h=None, y_perm=None, dev_status=None,
                   stream=None):
    rows, d = x_perm.shape
    E, _, f = w_gate.shape
    _want(x_perm, "x_perm", torch.bfloat16)
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    dev = x_perm.device
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=dev) if h is None else h
    y_perm = torch.empty(rows, d, dtype=torch.float32, device=dev) if y_perm is None else y_perm
    _want(h, "h", torch.bfloat16, (rows, f))
    _want(y_perm, "y_perm", torch.float32, (rows, d))
    _check("moe_expert_mlp", _lib.moe_expert_mlp(
        _ptr(x_perm), _ptr(offsets), E, d, f, rows, _ptr(w_gate), _ptr(w_up), _ptr(w_down),
        _ptr(h), _ptr(y_perm), _ptr(dev_status), _stream(stream)))
    return h, y_perm


def moe_combine(y_perm, x, topk_idx, topk_w, slot, offsets, y=None, stream=None):
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(y_perm, "y_perm", torch.float32)
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    _want(topk_w, "topk_w", torch.float32, (T, k))
    _want(slot, "slot", torch.int32, (T, k))
    _want(offsets, "offsets", torch.int32)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_combine", _lib.moe_combine(
        _ptr(y_perm), _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(slot), _ptr(offsets), T, d, k,
        _ptr(y), _stream(stream)))
    return y


def moe_combine_bf16rows(y_rows, x, topk_idx, topk_w, slot, offsets, y=None, stream=None):
    """moe_combine on bf16 expert-output rows (the expert-parallel return)."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(y_rows, "y_rows", torch.bfloat16)
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    _want(topk_w, "topk_w", torch.float32, (T, k))
    _want(slot, "slot", torch.int32, (T, k))
    _want(offsets, "offsets", torch.int32)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_combine_bf16rows", _lib.moe_combine_bf16rows(
        _ptr(y_rows), _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(slot), _ptr(offsets), T, d, k,
        _ptr(y), _stream(stream)))
    return y


def moe_rows_to_bf16(src, dst=None, stream=None):
    """bf16 copy (round to nearest even) of fp32 rows src [rows, d]."""
    rows, d = src.shape
    _want(src, "src", torch.float32)
    dst = torch.empty(rows, d, dtype=torch.bfloat16, device=src.device) if dst is None else dst
    _want(dst, "dst", torch.bfloat16, (rows, d))
    _check("moe_rows_to_bf16", _lib.moe_rows_to_bf16(_ptr(src), _ptr(dst), rows, d,
                                                     _stream(stream)))
    return dst


def moe_layer_forward(x, w_router, bias, w_gate, w_up, w_down, k, cf, y=None, ws=None,
                      stream=None):
    """The whole layer in one call.  Returns (y bf16 [T,d], ws uint8 workspace)."""
    T, d = x.shape
    E, _, f = w_gate.shape
    _want(x, "x", torch.bfloat16)
    _want(w_router, "w_router", torch.float32, (d, E))
    if bias is not None:
        _want(bias, "bias", torch.float32, (E,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    nbytes = moe_workspace_size(T, d, E, k, f, cf)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _want(ws, "ws", torch.uint8)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_layer_forward", _lib.moe_layer_forward(
        _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k,
        f, float(cf), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y, ws


def moe_layer_forward_ex(x, w_router, bias, w_gate, w_up, w_down, k, cf, y=None, logits=None,
                         topk_idx=None, topk_w=None, slot=None, counts=None, ws=None,
                         stream=None):
    """moe_layer_forward with optional caller tensors for the routing results
    (each one given is written in place of its workspace field).  Returns
    (y, ws)."""
    T, d = x.shape
    E, _, f = w_gate.shape
    _want(x, "x", torch.bfloat16)
    _want(w_router, "w_router", torch.float32, (d, E))
    if bias is not None:
        _want(bias, "bias", torch.float32, (E,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    for t, name, dt, shape in ((logits, "logits", torch.float32, (T, E)),
                               (topk_idx, "topk_idx", torch.int32, (T, k)),
                               (topk_w, "topk_w", torch.float32, (T, k)),
                               (slot, "slot", torch.int32, (T, k)),
                               (counts, "counts", torch.int32, (E,))):
        if t is not None:
            _want(t, name, dt, shape)
    nbytes = moe_workspace_size(T, d, E, k, f, cf)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _want(ws, "ws", torch.uint8)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_layer_forward_ex", _lib.moe_layer_forward_ex(
        _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k,
        f, float(cf), _ptr(y), _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(slot),
        _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)))
    return y, ws


# ----------------------------------------------------------------- buckets

def moe_expert_mlp_buckets(x_rows, offsets, bucket_rows, w_gate, w_up, w_down, h=None,
                           y_rows=None, dev_status=None, stream=None):
    """Grouped SwiGLU MLP over B buckets, bucket b through expert b % E_w,
    only its first bucket_rows[b] rows.  Returns (h, y_rows)."""
    rows, d = x_rows.shape
    B = offsets.shape[0] - 1
    E_w, _, f = w_gate.shape
    _want(x_rows, "x_rows", torch.bfloat16)
    _want(offsets, "offsets", torch.int32, (B + 1,))
    if bucket_rows is not None:
        _want(bucket_rows, "bucket_rows", torch.int32, (B,))
    _want(w_gate, "w_gate", torch.bfloat16, (E_w, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E_w, d, f))
    _want(w_down, "w_down", torch.bfloat16, (E_w, f, d))
    dev = x_rows.device
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=dev) if h is None else h
    y_rows = torch.empty(rows, d, dtype=torch.float32, device=dev) if y_rows is None else y_rows
    _check("moe_expert_mlp_buckets", _lib.moe_expert_mlp_buckets(
        _ptr(x_rows), _ptr(offsets), _ptr(bucket_rows), B, E_w, d, f, rows, _ptr(w_gate),
        _ptr(w_up), _ptr(w_down), _ptr(h), _ptr(y_rows), _ptr(dev_status), _stream(stream)))
    return h, y_rows


# ----------------------------------------------------------------- fused path

def moe_permute_fused(x, topk_idx, E, cf, copy_rows=True, out=None, ws=None, dev_status=None,
                      stream=None):
    """The permutation for the fused path.  Returns a dict with counts, offsets,
    slot, row_src, row_pair, n_dropped, a zeroed fp32 token accumulator "y32"
    [T, d] and, with copy_rows, "x_perm"."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    rows = moe_max_rows(T, E, k, cf)
    dev = x.device
    if out is None:
        out = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
               "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
               "slot": torch.empty(T, k, dtype=torch.int32, device=dev),
               "row_src": torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
               "row_pair": torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
               "n_dropped": torch.empty(1, dtype=torch.int32, device=dev),
               "y32": torch.empty(T, d, dtype=torch.float32, device=dev)}
        if copy_rows:
            out["x_perm"] = torch.empty(max(rows, 1), d, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = torch.empty(max(moe_permute_workspace_size(T, E, k), 16), dtype=torch.uint8,
                         device=dev)
    xp = out.get("x_perm") if copy_rows else None
    _check("moe_permute_fused", _lib.moe_permute_fused(
        _ptr(x) if copy_rows else None, _ptr(topk_idx), T, d, E, k, float(cf),
        _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(out["slot"]), _ptr(out["row_src"]),
        _ptr(out["row_pair"]), _ptr(xp), _ptr(out["n_dropped"]), _ptr(out.get("y32")), _ptr(ws),
        ws.numel(), _ptr(dev_status), _stream(stream)))
    return out


def moe_expert_gate_up_gather(x, row_src, offsets, w_gate, w_up, max_rows, h=None,
                              dev_status=None, stream=None):
    T, d = x.shape
    E, _, f = w_gate.shape
    _want(x, "x", torch.bfloat16)
    _want(row_src, "row_src", torch.int32)
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    h = torch.empty(max_rows, f, dtype=torch.bfloat16, device=x.device) if h is None else h
    _want(h, "h", torch.bfloat16, (max_rows, f))
    _check("moe_expert_gate_up_gather", _lib.moe_expert_gate_up_gather(
        _ptr(x), T, _ptr(row_src), _ptr(offsets), E, d, f, max_rows, _ptr(w_gate), _ptr(w_up),
        _ptr(h), _ptr(dev_status), _stream(stream)))
    return h


def moe_expert_down_scatter(h, offsets, w_down, row_pair, topk_w, y32, dev_status=None,
                            stream=None):
    rows, f = h.shape
    E, _, d = w_down.shape
    k = topk_w.shape[1]
    _want(h, "h", torch.bfloat16)
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    _want(row_pair, "row_pair", torch.int32)
    _want(topk_w, "topk_w", torch.float32)
    _want(y32, "y32", torch.float32, (topk_w.shape[0], d))
    _check("moe_expert_down_scatter", _lib.moe_expert_down_scatter(
        _ptr(h), _ptr(offsets), E, d, f, rows, _ptr(w_down), _ptr(row_pair), _ptr(topk_w), k,
        _ptr(y32), _ptr(dev_status), _stream(stream)))
    return y32


def moe_combine_finalize(y32, x, slot, y=None, stream=None):
    T, d = x.shape
    k = slot.shape[1]
    _want(y32, "y32", torch.float32, (T, d))
    _want(x, "x", torch.bfloat16)
    _want(slot, "slot", torch.int32, (T, k))
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_combine_finalize", _lib.moe_combine_finalize(
        _ptr(y32), _ptr(x), _ptr(slot), T, d, k, _ptr(y), _stream(stream)))
    return y


def moe_workspace_size_fused(T, d, E, k, f, cf):
    return int(_lib.moe_workspace_size_fused(T, d, E, k, f, float(cf)))


def moe_layer_forward_fused(x, w_router, bias, w_gate, w_up, w_down, k, cf, y=None, ws=None,
                            stream=None):
    """The whole layer on the fused path.  Returns (y, ws)."""
    T, d = x.shape
    E, _, f = w_gate.shape
    _want(x, "x", torch.bfloat16)
    _want(w_router, "w_router", torch.float32, (d, E))
    if bias is not None:
        _want(bias, "bias", torch.float32, (E,))
    _want(w_gate, "w_gate", torch.bfloat16, (E, d, f))
    _want(w_up, "w_up", torch.bfloat16, (E, d, f))
    _want(w_down, "w_down", torch.bfloat16, (E, f, d))
    nbytes = moe_workspace_size_fused(T, d, E, k, f, cf)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _want(ws, "ws", torch.uint8)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_layer_forward_fused", _lib.moe_layer_forward_fused(
        _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k,
        f, float(cf), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))
    return y, ws


# ----------------------------------------------------------------- padded layout

def moe_padded_rows(T, E, k, cf):
    return int(_lib.moe_padded_rows(T, E, k, float(cf)))


def moe_permute_padded(x, topk_idx, E, cf, out=None, ws=None, dev_status=None, stream=None):
    """moe_permute into the padded [E*C, d] layout.  Returns a dict like
    moe_permute's with "x_pad" in place of "x_perm" (offsets[e] = e*C)."""
    T, d = x.shape
    k = topk_idx.shape[1]
    _want(x, "x", torch.bfloat16)
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    rows = moe_padded_rows(T, E, k, cf)
    if rows < 0:
        raise ValueError("padded layout too large")
    dev = x.device
    if out is None:
        out = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
               "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
               "slot": torch.empty(T, k, dtype=torch.int32, device=dev),
               "row_src": torch.empty(max(rows, 1), dtype=torch.int32, device=dev),
               "x_pad": torch.empty(max(rows, 1), d, dtype=torch.bfloat16, device=dev),
               "n_dropped": torch.empty(1, dtype=torch.int32, device=dev)}
    if ws is None:
        ws = torch.empty(max(moe_permute_workspace_size(T, E, k), 16), dtype=torch.uint8,
                         device=dev)
    _check("moe_permute_padded", _lib.moe_permute_padded(
        _ptr(x), _ptr(topk_idx), T, d, E, k, float(cf), _ptr(out["counts"]), _ptr(out["offsets"]),
        _ptr(out["slot"]), _ptr(out["row_src"]), _ptr(out["x_pad"]), _ptr(out["n_dropped"]),
        _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))
    return out


# ----------------------------------------------------------------- FP8 experts

def moe_quantize_weights_fp8(w, stream=None):
    """bf16 weights [E,K,N] -> (e4m3 codes uint8 [E,N,K] (K-major), fp32 scales [E,N])."""
    E, K, N = w.shape
    _want(w, "w", torch.bfloat16)
    q = torch.empty(E, N, K, dtype=torch.uint8, device=w.device)
    sc = torch.empty(E, N, dtype=torch.float32, device=w.device)
    _check("moe_quantize_weights_fp8",
           _lib.moe_quantize_weights_fp8(_ptr(w), E, K, N, _ptr(q), _ptr(sc), _stream(stream)))
    return q, sc


def moe_quantize_rows_fp8(x, n_rows=None, q=None, scale=None, stream=None):
    """bf16 rows [R,K] -> (e4m3 codes uint8 [R,K], fp32 row scales [R])."""
    R, K = x.shape
    _want(x, "x", torch.bfloat16)
    q = torch.empty(R, K, dtype=torch.uint8, device=x.device) if q is None else q
    scale = torch.empty(R, dtype=torch.float32, device=x.device) if scale is None else scale
    _want(q, "q", torch.uint8, (R, K))
    _want(scale, "scale", torch.float32, (R,))
    if n_rows is not None:
        _want(n_rows, "n_rows", torch.int32)
    _check("moe_quantize_rows_fp8", _lib.moe_quantize_rows_fp8(
        _ptr(x), R, K, _ptr(n_rows), _ptr(q), _ptr(scale), _stream(stream)))
    return q, scale


def moe_permute_fp8(xq, sx, topk_idx, E, cf, out=None, ws=None, dev_status=None, stream=None):
    """moe_permute on e4m3 token rows (codes + row scales).  Returns a dict
    like moe_permute's, with "xq" / "sx" in place of "x_perm"."""
    T, d = xq.shape
    k = topk_idx.shape[1]
    _want(xq, "xq", torch.uint8)
    _want(sx, "sx", torch.float32, (T,))
    _want(topk_idx, "topk_idx", torch.int32, (T, k))
    rows = moe_max_rows(T, E, k, cf)
    dev = xq.device
    if out is None:
        out = {"counts": torch.empty(E, dtype=torch.int32, device=dev),
               "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
               "slot": torch.empty(T, k, dtype=torch.int32, device=dev),
               "row_src": torch.empty(rows, dtype=torch.int32, device=dev),
               "xq": torch.empty(rows, d, dtype=torch.uint8, device=dev),
               "sx": torch.empty(rows, dtype=torch.float32, device=dev),
               "n_dropped": torch.empty(1, dtype=torch.int32, device=dev)}
    if ws is None:
        ws = torch.empty(max(moe_permute_workspace_size(T, E, k), 16), dtype=torch.uint8,
                         device=dev)
    _check("moe_permute_fp8", _lib.moe_permute_fp8(
        _ptr(xq), _ptr(sx), _ptr(topk_idx), T, d, E, k, float(cf), _ptr(out["counts"]),
        _ptr(out["offsets"]), _ptr(out["slot"]), _ptr(out["row_src"]), _ptr(out["xq"]),
        _ptr(out["sx"]), _ptr(out["n_dropped"]), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))
    return out


def moe_expert_gate_up_fp8(xq, sx, offsets, wq_gate, s_gate, wq_up, s_up, h=None,
                           dev_status=None, stream=None):
    rows, d = xq.shape
    E, f, _ = wq_gate.shape
    _want(xq, "xq", torch.uint8)
    _want(sx, "sx", torch.float32, (rows,))
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(wq_gate, "wq_gate", torch.uint8, (E, f, d))
    _want(wq_up, "wq_up", torch.uint8, (E, f, d))
    _want(s_gate, "s_gate", torch.float32, (E, f))
    _want(s_up, "s_up", torch.float32, (E, f))
    h = torch.empty(rows, f, dtype=torch.bfloat16, device=xq.device) if h is None else h
    _want(h, "h", torch.bfloat16, (rows, f))
    _check("moe_expert_gate_up_fp8", _lib.moe_expert_gate_up_fp8(
        _ptr(xq), _ptr(sx), _ptr(offsets), E, d, f, rows, _ptr(wq_gate), _ptr(s_gate),
        _ptr(wq_up), _ptr(s_up), _ptr(h), _ptr(dev_status), _stream(stream)))
    return h


def moe_expert_down_fp8(hq, sh, offsets, wq_down, s_down, y_perm=None, dev_status=None,
                        stream=None):
    rows, f = hq.shape
    E, d, _ = wq_down.shape
    _want(hq, "hq", torch.uint8)
    _want(sh, "sh", torch.float32, (rows,))
    _want(offsets, "offsets", torch.int32, (E + 1,))
    _want(wq_down, "wq_down", torch.uint8, (E, d, f))
    _want(s_down, "s_down", torch.float32, (E, d))
    y_perm = torch.empty(rows, d, dtype=torch.float32, device=hq.device) if y_perm is None \
        else y_perm
    _want(y_perm, "y_perm", torch.float32, (rows, d))
    _check("moe_expert_down_fp8", _lib.moe_expert_down_fp8(
        _ptr(hq), _ptr(sh), _ptr(offsets), E, d, f, rows, _ptr(wq_down), _ptr(s_down),
        _ptr(y_perm), _ptr(dev_status), _stream(stream)))
    return y_perm


def moe_workspace_size_fp8(T, d, E, k, f, cf):
    return int(_lib.moe_workspace_size_fp8(T, d, E, k, f, float(cf)))


def moe_layer_forward_fp8(x, w_router, bias, wq_gate, s_gate, wq_up, s_up, wq_down, s_down, k, cf,
                          y=None, ws=None, stream=None):
    """The whole layer with FP8 experts.  Returns (y, ws)."""
    T, d = x.shape
    E, f, _ = wq_gate.shape
    _want(x, "x", torch.bfloat16)
    _want(w_router, "w_router", torch.float32, (d, E))
    if bias is not None:
        _want(bias, "bias", torch.float32, (E,))
    for name, t, shape in (("wq_gate", wq_gate, (E, f, d)), ("wq_up", wq_up, (E, f, d)),
                           ("wq_down", wq_down, (E, d, f))):
        _want(t, name, torch.uint8, shape)
    for name, t, shape in (("s_gate", s_gate, (E, f)), ("s_up", s_up, (E, f)),
                           ("s_down", s_down, (E, d))):
        _want(t, name, torch.float32, shape)
    nbytes = moe_workspace_size_fp8(T, d, E, k, f, cf)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
    _want(ws, "ws", torch.uint8)
    y = torch.empty_like(x) if y is None else y
    _want(y, "y", torch.bfloat16, (T, d))
    _check("moe_layer_forward_fp8", _lib.moe_layer_forward_fp8(
        _ptr(x), _ptr(w_router), _ptr(bias), _ptr(wq_gate), _ptr(s_gate), _ptr(wq_up), _ptr(s_up),
        _ptr(wq_down), _ptr(s_down), T, d, E, k, f, float(cf), _ptr(y), _ptr(ws), ws.numel(),
        _stream(stream)))
    return y, ws


def workspace_view(ws, field, T, d, E, k, f, cf):
    """A typed view of one intermediate inside a moe_layer_forward workspace."""
    rows = moe_max_rows(T, E, k, cf)
    spec = {
        "status": (torch.int32, (1,)), "logits": (torch.float32, (T, E)),
        "topk_idx": (torch.int32, (T, k)), "topk_w": (torch.float32, (T, k)),
        "slot": (torch.int32, (T, k)), "counts": (torch.int32, (E,)),
        "offsets": (torch.int32, (E + 1,)), "n_dropped": (torch.int32, (1,)),
        "row_src": (torch.int32, (rows,)), "x_perm": (torch.bfloat16, (rows, d)),
        "h": (torch.bfloat16, (rows, f)), "y_perm": (torch.float32, (rows, d)),
        "xq": (torch.uint8, (rows, d)), "sx": (torch.float32, (rows,)),
        "hq": (torch.uint8, (rows, f)), "sh": (torch.float32, (rows,)),
        "xq_tok": (torch.uint8, (T, d)), "sx_tok": (torch.float32, (T,)),
        "row_pair": (torch.int32, (rows,)), "y32": (torch.float32, (T, d)),
    }[field]
    dtype, shape = spec
    off = moe_workspace_field_offset(field, T, d, E, k, f, cf)
    n = 1
    for s in shape:
        n *= s
    nbytes = n * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype).view(shape)
