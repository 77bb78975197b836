"""ctypes binding of libnmoe (include/nmoe.h). Argument marshalling only.

Every function here hands device pointers, sizes and the current CUDA stream to the
C ABI; all of the layer's arithmetic runs in the library's CUDA kernels. There is no
fallback: if the shared library is missing, or a call fails, an error is raised.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# NMOE_DEBUG=1 loads the debug build (index and span checks in the kernels, reported
# through the error word); both are this package's own CUDA library.
DEBUG = os.environ.get("NMOE_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libnmoe_debug.so" if DEBUG else "libnmoe.so")

NMOE_BF16, NMOE_F32 = 0, 1
SCORE = {"softmax": 0, "sigmoid": 1}
COMBINE = {"raw": 0, "normalized": 1}
INTERMEDIATE = {"split": 0, "bf16": 1}
N_STAGES = 6
STATUS = {
    0: "NMOE_OK", 1: "NMOE_ERR_INVALID_ARG", 2: "NMOE_ERR_UNSUPPORTED",
    3: "NMOE_ERR_WORKSPACE", 4: "NMOE_ERR_CUDA", 5: "NMOE_ERR_TIMEOUT",
    6: "NMOE_ERR_DEVICE_CHECK", 7: "NMOE_ERR_NO_DEVICE",
}

# Every symbol include/nmoe.h declares.
EXPORTS = (
    "nmoe_options_init", "nmoe_router", "nmoe_select", "nmoe_forward", "nmoe_forward_ex",
    "nmoe_workspace_size", "nmoe_get_last_error", "nmoe_status_str", "nmoe_trace_create",
    "nmoe_trace_read", "nmoe_trace_reset", "nmoe_trace_destroy", "nmoe_stage_name",
    "nmoe_build_info", "nmoe_forward_noalloc", "nmoe_kernels_per_call",
    "nmoe_workspace_offsets", "nmoe_ep_rows", "nmoe_rows_gather", "nmoe_rows_scatter",
    "nmoe_combine_tokens",
)


class NmoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class Options(C.Structure):
    _fields_ = [
        ("dtype", C.c_int), ("score_fn", C.c_int), ("combine", C.c_int),
        ("route_scale", C.c_float), ("n_segments", C.c_int64), ("router_bias", C.c_void_p),
        ("workspace", C.c_void_p), ("workspace_bytes", C.c_size_t),
        ("scores_out", C.c_void_p), ("idx_out", C.c_void_p), ("host_io", C.c_int),
        ("trace", C.c_void_p), ("intermediate", C.c_int), ("out_f32", C.c_int),
        ("tma_gather", C.c_int), ("shared_w1", C.c_void_p), ("shared_w3", C.c_void_p),
        ("shared_w2", C.c_void_p), ("shared_f", C.c_int64), ("residual", C.c_void_p),
        ("gate2", C.c_void_p), ("expert_begin", C.c_int64), ("expert_end", C.c_int64),
        ("skip_combine", C.c_int), ("router_x", C.c_void_p),
        ("wait_budget_ns", C.c_uint64),
    ]


_lib = None
_lock = threading.Lock()
_i64 = C.c_int64
_vp = C.c_void_p


def lib() -> C.CDLL:
    """The loaded shared library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m diffusion_transformer_moe_b200.build`")
            L = C.CDLL(LIB_PATH)
            L.nmoe_options_init.argtypes = [C.POINTER(Options)]
            L.nmoe_options_init.restype = None
            L.nmoe_router.argtypes = [_vp, _vp, _i64, _i64, _i64, C.c_int, C.c_int, _vp, _i64,
                                      _vp, _vp, _vp]
            L.nmoe_router.restype = C.c_int
            L.nmoe_select.argtypes = [_vp, _i64, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]
            L.nmoe_select.restype = C.c_int
            L.nmoe_forward.argtypes = [_vp] * 5 + [_i64] * 5 + [_vp, _vp]
            L.nmoe_forward.restype = C.c_int
            L.nmoe_forward_ex.argtypes = [_vp] * 5 + [_i64] * 5 + [_vp, _vp,
                                                                  C.POINTER(Options)]
            L.nmoe_forward_ex.restype = C.c_int
            L.nmoe_workspace_size.argtypes = [_i64] * 5 + [C.POINTER(Options)]
            L.nmoe_workspace_size.restype = C.c_size_t
            L.nmoe_get_last_error.argtypes = [_vp]
            L.nmoe_get_last_error.restype = C.c_int
            L.nmoe_status_str.argtypes = [C.c_int]
            L.nmoe_status_str.restype = C.c_char_p
            L.nmoe_trace_create.argtypes = [C.c_int, C.POINTER(_vp)]
            L.nmoe_trace_create.restype = C.c_int
            L.nmoe_trace_read.argtypes = [_vp, C.POINTER(C.c_double), C.POINTER(C.c_int)]
            L.nmoe_trace_read.restype = C.c_int
            L.nmoe_trace_reset.argtypes = [_vp]
            L.nmoe_trace_reset.restype = C.c_int
            L.nmoe_trace_destroy.argtypes = [_vp]
            L.nmoe_trace_destroy.restype = None
            L.nmoe_stage_name.argtypes = [C.c_int]
            L.nmoe_stage_name.restype = C.c_char_p
            L.nmoe_build_info.argtypes = []
            L.nmoe_build_info.restype = C.c_char_p
            L.nmoe_forward_noalloc.argtypes = [_vp] * 5 + [_i64] * 5 + [_vp, _vp]
            L.nmoe_forward_noalloc.restype = C.c_int
            L.nmoe_kernels_per_call.argtypes = [_i64] * 5 + [C.POINTER(Options)]
            L.nmoe_kernels_per_call.restype = C.c_int
            L.nmoe_workspace_offsets.argtypes = [_i64] * 5 + [C.POINTER(Options)] + [
                C.POINTER(C.c_size_t)] * 3
            L.nmoe_workspace_offsets.restype = C.c_int
            L.nmoe_ep_rows.argtypes = [_vp, _vp] + [_i64] * 7 + [_vp, _i64, _vp, _vp]
            L.nmoe_ep_rows.restype = C.c_int
            L.nmoe_rows_gather.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp]
            L.nmoe_rows_gather.restype = C.c_int
            L.nmoe_rows_scatter.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp]
            L.nmoe_rows_scatter.restype = C.c_int
            L.nmoe_combine_tokens.argtypes = [_vp, _vp] + [_i64] * 4 + [C.c_int, C.c_int, _vp,
                                                                         _vp]
            L.nmoe_combine_tokens.restype = C.c_int
            _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise NmoeError(status, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return NMOE_BF16
    if t.dtype == torch.float32:
        return NMOE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dt_code(dtype: torch.dtype) -> int:
    if dtype == torch.bfloat16:
        return NMOE_BF16
    if dtype == torch.float32:
        return NMOE_F32
    raise TypeError(f"unsupported dtype {dtype}")


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _dev(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def options(dtype=NMOE_BF16, score_fn="softmax", combine="raw", route_scale=1.0,
            n_segments=1, router_bias=None, workspace=None, scores_out=None, idx_out=None,
            host_io=False, trace=None, intermediate="split", out_f32=False,
            tma_gather=False, shared=None, shared_f=None, residual=None,
            gate2=None, expert_begin=0, expert_end=0, skip_combine=False,
            router_x=None, wait_budget_ns=0) -> Options:
    """nmoe_options from keyword arguments. ``shared`` = (Ws1 [d,Fs], Ws3 [d,Fs],
    Ws2 [Fs,d]) device tensors adds the shared expert; ``shared_f`` alone (no tensors)
    only sizes a workspace for one. ``residual`` [T,d] and ``gate2`` fp32
    [n_segments,d] add the block's gated residual. ``router_x`` [T,d] is what the
    router scores instead of x (on the host with ``host_io``). ``wait_budget_ns`` bounds
    every device-side pipeline wait (0: the library's default)."""
    o = Options()
    lib().nmoe_options_init(C.byref(o))
    o.dtype = dtype
    o.score_fn = SCORE[score_fn]
    o.combine = COMBINE[combine]
    o.route_scale = float(route_scale)
    o.n_segments = int(n_segments)
    o.router_bias = _ptr(router_bias)
    if workspace is not None:
        o.workspace = workspace.data_ptr()
        o.workspace_bytes = workspace.numel() * workspace.element_size()
    o.scores_out = _ptr(scores_out)
    o.idx_out = _ptr(idx_out)
    o.host_io = 1 if host_io else 0
    o.trace = None if trace is None else trace.handle
    o.intermediate = INTERMEDIATE[intermediate]
    o.out_f32 = 1 if out_f32 else 0
    o.tma_gather = 1 if tma_gather else 0
    if shared is not None:
        Ws1, Ws3, Ws2 = shared
        for n, t in (("shared Ws1", Ws1), ("shared Ws3", Ws3), ("shared Ws2", Ws2)):
            _dev(t, n)
        o.shared_w1, o.shared_w3, o.shared_w2 = Ws1.data_ptr(), Ws3.data_ptr(), Ws2.data_ptr()
        o.shared_f = int(Ws1.shape[1])
    elif shared_f is not None:
        # sizing only (nmoe_workspace_size reads no weight): non-null placeholders
        o.shared_w1 = o.shared_w3 = o.shared_w2 = 256
        o.shared_f = int(shared_f)
    o.residual = _ptr(residual)
    o.gate2 = _ptr(gate2)
    o.expert_begin = int(expert_begin)
    o.expert_end = int(expert_end)
    o.skip_combine = 1 if skip_combine else 0
    o.router_x = _ptr(router_x)
    o.wait_budget_ns = int(wait_budget_ns)
    return o


def router(x, W_r, score_fn="softmax", router_bias=None, n_segments=1, stream=None):
    """scores [T,E], scores_t [E,T] (fp32) for x [T,d], W_r [d,E]."""
    _dev(x, "x"); _dev(W_r, "W_r")
    T, d = x.shape
    E = W_r.shape[1]
    scores = torch.empty(T, E, device=x.device, dtype=torch.float32)
    scores_t = torch.empty(E, T, device=x.device, dtype=torch.float32)
    _check(lib().nmoe_router(x.data_ptr(), W_r.data_ptr(), T, d, E, _dt(x), SCORE[score_fn],
                             _ptr(router_bias), n_segments, scores.data_ptr(),
                             scores_t.data_ptr(), _stream(stream)), "nmoe_router")
    return scores, scores_t


def select(scores_t, C_: int, n_segments=1, csr=True, stream=None):
    """idx [E, n_segments*C] int32, gate fp32, and (if csr) tok_ptr [T+1], tok_ent."""
    _dev(scores_t, "scores_t")
    E, T = scores_t.shape
    Ce = n_segments * C_
    dev = scores_t.device
    idx = torch.empty(E, Ce, device=dev, dtype=torch.int32)
    gate = torch.empty(E, Ce, device=dev, dtype=torch.float32)
    tok_ptr = torch.empty(T + 1, device=dev, dtype=torch.int32) if csr else None
    tok_ent = torch.empty(E * Ce, device=dev, dtype=torch.int32) if csr else None
    _check(lib().nmoe_select(scores_t.data_ptr(), T, E, C_, n_segments, idx.data_ptr(),
                             gate.data_ptr(), _ptr(tok_ptr), _ptr(tok_ent), _stream(stream)),
           "nmoe_select")
    return idx, gate, tok_ptr, tok_ent


def gather_rows(src, rows, out=None, stream=None):
    """out[i] = src[rows[i]] (a zero row where rows[i] < 0): rows of a 2-D device tensor
    whose row is a multiple of 16 bytes; rows is device int32 (any shape, read flat).
    With src = x and rows = idx, out holds each expert's chosen rows as one block."""
    _dev(src, "src"); _dev(rows, "rows")
    if src.dim() != 2 or not src.is_contiguous() or rows.dtype != torch.int32 \
            or not rows.is_contiguous():
        raise ValueError("src must be a contiguous 2-D tensor and rows contiguous int32")
    n = rows.numel()
    if out is None:
        out = torch.empty(n, src.shape[1], dtype=src.dtype, device=src.device)
    _check(lib().nmoe_rows_gather(src.data_ptr(), rows.data_ptr(), n,
                                  src.shape[1] * src.element_size(), out.data_ptr(),
                                  _stream(stream)), "nmoe_rows_gather")
    return out


def forward(x, W_r, W1, W3, W2, C_: int, out=None, stream=None, **opts):
    """The whole layer. ``opts`` are the nmoe_options fields (score_fn, combine,
    route_scale, n_segments, router_bias, workspace, scores_out, idx_out, trace,
    intermediate, out_f32, tma_gather, shared=(Ws1, Ws3, Ws2), residual, gate2, router_x).
    With ``host_io=True`` x, router_x and out are pinned CPU tensors."""
    host_io = bool(opts.get("host_io", False))
    for n, t in (("W_r", W_r), ("W1", W1), ("W3", W3), ("W2", W2)):
        _dev(t, n)
    rx = opts.get("router_x")
    if rx is not None and (rx.shape != x.shape or rx.dtype != x.dtype
                           or not rx.is_contiguous()):
        raise ValueError("router_x must be a contiguous tensor of x's shape and dtype")
    if not host_io:
        _dev(x, "x")
        if rx is not None:
            _dev(rx, "router_x")
    T, d = x.shape
    E, _, F = W1.shape
    if out is None:
        odt = torch.float32 if opts.get("out_f32", False) else x.dtype
        out = torch.empty(T, d, dtype=odt, device="cpu" if host_io else x.device,
                          pin_memory=host_io)
    o = options(dtype=_dt(x), **opts)
    if opts or x.dtype != torch.bfloat16:
        st = lib().nmoe_forward_ex(x.data_ptr(), W_r.data_ptr(), W1.data_ptr(), W3.data_ptr(),
                                   W2.data_ptr(), T, d, E, F, C_, out.data_ptr(),
                                   _stream(stream), C.byref(o))
    else:
        st = lib().nmoe_forward(x.data_ptr(), W_r.data_ptr(), W1.data_ptr(), W3.data_ptr(),
                                W2.data_ptr(), T, d, E, F, C_, out.data_ptr(), _stream(stream))
    _check(st, "nmoe_forward")
    return out


def workspace_size(T, d, E, F, C_, **opts) -> int:
    o = options(**opts)
    return int(lib().nmoe_workspace_size(T, d, E, F, C_, C.byref(o)))


def kernels_per_call(T, d, E, F, C_, **opts) -> int:
    """How many kernels one layer call with these sizes and options launches."""
    o = options(**opts)
    return int(lib().nmoe_kernels_per_call(T, d, E, F, C_, C.byref(o)))


def get_last_error(stream=None) -> int:
    return int(lib().nmoe_get_last_error(_stream(stream)))


def build_info() -> str:
    return lib().nmoe_build_info().decode()


class Trace:
    """Per-stage CUDA-event timer of nmoe_forward_ex calls (include/nmoe.h nmoe_trace)."""

    def __init__(self, max_calls: int):
        h = _vp()
        _check(lib().nmoe_trace_create(max_calls, C.byref(h)), "nmoe_trace_create")
        self.handle = h.value

    def read(self):
        ms = (C.c_double * N_STAGES)()
        n = C.c_int()
        _check(lib().nmoe_trace_read(self.handle, ms, C.byref(n)), "nmoe_trace_read")
        names = [lib().nmoe_stage_name(i).decode() for i in range(N_STAGES)]
        return dict(zip(names, list(ms))), n.value

    def reset(self):
        _check(lib().nmoe_trace_reset(self.handle), "nmoe_trace_reset")

    def close(self):
        if self.handle:
            lib().nmoe_trace_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
