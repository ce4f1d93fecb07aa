"""Python binding of librmm: Reduced Matrix Multiplication on B200 (sm_100a).

Argument marshalling only.  Every step of the op (column scores, TopK,
staging, the tensor-core product) runs in the CUDA kernels of librmm.so behind
the C ABI of include/rmm.h; PyTorch supplies device memory and streams.  There
is no CPU fallback: importing this package fails when librmm.so is missing,
and every call raises RmmError on a non-OK status.

Method: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (arXiv 2608.13426), §3.2-§3.3.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading
import weakref

__all__ = [
    "RMM_OK", "RMM_ERR_INVALID_ARG", "RMM_ERR_UNSUPPORTED", "RMM_ERR_WORKSPACE", "RMM_ERR_CUDA",
    "RMM_ERR_TIMEOUT", "RMM_BF16", "RMM_F32", "RMM_FP8_E4M3", "RMM_LINEAR", "RMM_QK", "RMM_PV", "RMM_FLAG_CAUSAL",
    "RMM_FLAG_USE_GIVEN_INDICES", "RmmError", "rmm_problem", "Plan", "lib", "library_path",
    "rmm_problem_init", "rmm_plan_create", "rmm_select", "rmm_matmul", "rmm_matmul_batched",
    "rmm_workspace_init", "rmm_workspace_status", "rmm_status_string", "rmm_version",
    "EXPORTED_SYMBOLS", "select", "matmul", "qk", "pv", "workspace_for", "check_workspaces",
    "rmm_plan_set_product_events", "rmm_plan_kernel_launches", "rmm_select_no_alloc",
    "rmm_selftest_wait_timeout", "RMM_FLAG_GIVEN_SCORES", "RMM_FLAG_EMIT_SCORES", "rmm_matmul_ex",
    "rmm_softmax_scores", "rmm_softmax_workspace_size", "softmax_scores", "rmm_attn_problem",
    "rmm_attention", "rmm_attention_workspace_size", "attention",
]

RMM_OK, RMM_ERR_INVALID_ARG, RMM_ERR_UNSUPPORTED, RMM_ERR_WORKSPACE, RMM_ERR_CUDA, RMM_ERR_TIMEOUT = range(6)
RMM_BF16, RMM_F32, RMM_FP8_E4M3 = 0, 1, 2
RMM_LINEAR, RMM_QK, RMM_PV = 0, 1, 2
RMM_FLAG_CAUSAL = 1
RMM_FLAG_USE_GIVEN_INDICES = 2
RMM_FLAG_GIVEN_SCORES = 4
RMM_FLAG_EMIT_SCORES = 8

EXPORTED_SYMBOLS = (
    "rmm_problem_init", "rmm_plan_create", "rmm_plan_destroy", "rmm_plan_k", "rmm_plan_workspace_size",
    "rmm_select", "rmm_matmul", "rmm_matmul_batched", "rmm_workspace_init", "rmm_workspace_status",
    "rmm_status_string", "rmm_version", "rmm_plan_set_product_events", "rmm_plan_kernel_launches",
    "rmm_select_no_alloc", "rmm_selftest_wait_timeout", "rmm_matmul_ex", "rmm_softmax_workspace_size",
    "rmm_softmax_scores", "rmm_attention_workspace_size", "rmm_attention",
)

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librmm.so")


class RmmError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_status_name(status)}")


class rmm_problem(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("n", ctypes.c_int64), ("d", ctypes.c_int64), ("m", ctypes.c_int64),
        ("lda", ctypes.c_int64), ("ldb", ctypes.c_int64), ("ldy", ctypes.c_int64),
        ("heads", ctypes.c_int64), ("kv_heads", ctypes.c_int64),
        ("stride_a", ctypes.c_int64), ("stride_b", ctypes.c_int64), ("stride_y", ctypes.c_int64),
        ("rho", ctypes.c_double), ("k", ctypes.c_int64), ("alpha", ctypes.c_float),
        ("flags", ctypes.c_uint32),
    ]


class rmm_attn_problem(ctypes.Structure):
    _fields_ = [
        ("heads", ctypes.c_int64), ("kv_heads", ctypes.c_int64), ("n", ctypes.c_int64),
        ("d_h", ctypes.c_int64), ("d_v", ctypes.c_int64),
        ("ldq", ctypes.c_int64), ("ldk", ctypes.c_int64), ("ldv", ctypes.c_int64), ("ldo", ctypes.c_int64),
        ("stride_q", ctypes.c_int64), ("stride_k", ctypes.c_int64), ("stride_v", ctypes.c_int64),
        ("stride_o", ctypes.c_int64), ("rho_d", ctypes.c_double), ("rho_t", ctypes.c_double),
        ("alpha", ctypes.c_float), ("flags", ctypes.c_uint32),
    ]


def _load_library():
    from . import build as _build
    if _build.stale():
        try:
            _build.build()
        except Exception as exc:  # no compiler, no sources: there is no other path
            raise ImportError(f"librmm.so is missing or stale and could not be built ({exc}); "
                              "this package has no CPU fallback") from exc
    if not os.path.exists(library_path):
        raise ImportError("librmm.so is not built; this package has no CPU fallback")
    L = ctypes.CDLL(library_path)
    vp, sz, i64, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64, ctypes.c_int
    pp = ctypes.POINTER(rmm_problem)
    L.rmm_problem_init.restype = None
    L.rmm_problem_init.argtypes = [pp, ctypes.c_int32, ctypes.c_int32, i64, i64, i64]
    L.rmm_plan_create.restype = st
    L.rmm_plan_create.argtypes = [ctypes.POINTER(vp), pp, ctypes.POINTER(sz)]
    L.rmm_plan_destroy.restype = st
    L.rmm_plan_destroy.argtypes = [vp]
    L.rmm_plan_k.restype = i64
    L.rmm_plan_k.argtypes = [vp]
    L.rmm_plan_workspace_size.restype = sz
    L.rmm_plan_workspace_size.argtypes = [vp]
    L.rmm_select.restype = st
    L.rmm_select.argtypes = [vp, vp, vp, vp, vp, sz, vp]
    L.rmm_matmul.restype = st
    L.rmm_matmul.argtypes = [vp, vp, vp, vp, vp, vp, sz, vp]
    L.rmm_matmul_batched.restype = st
    L.rmm_matmul_batched.argtypes = [vp, vp, vp, vp, vp, vp, sz, vp]
    L.rmm_workspace_init.restype = st
    L.rmm_workspace_init.argtypes = [vp, vp, sz, vp]
    L.rmm_workspace_status.restype = st
    L.rmm_workspace_status.argtypes = [vp, vp, vp]
    L.rmm_selftest_wait_timeout.restype = st
    L.rmm_selftest_wait_timeout.argtypes = [vp, vp, sz, vp]
    L.rmm_plan_set_product_events.restype = st
    L.rmm_plan_set_product_events.argtypes = [vp, vp, vp]
    L.rmm_plan_kernel_launches.restype = ctypes.c_int32
    L.rmm_plan_kernel_launches.argtypes = [vp]
    L.rmm_matmul_ex.restype = st
    L.rmm_matmul_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.rmm_softmax_workspace_size.restype = sz
    L.rmm_softmax_workspace_size.argtypes = [i64, i64, i64]
    L.rmm_softmax_scores.restype = st
    L.rmm_softmax_scores.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, ctypes.c_uint32, vp, sz, vp]
    L.rmm_attention_workspace_size.restype = sz
    L.rmm_attention_workspace_size.argtypes = [ctypes.POINTER(rmm_attn_problem)]
    L.rmm_attention.restype = st
    L.rmm_attention.argtypes = [ctypes.POINTER(rmm_attn_problem), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.rmm_select_no_alloc.restype = st
    L.rmm_select_no_alloc.argtypes = [vp, vp, vp, vp, vp]
    L.rmm_status_string.restype = ctypes.c_char_p
    L.rmm_status_string.argtypes = [st]
    L.rmm_version.restype = ctypes.c_char_p
    L.rmm_version.argtypes = []
    return L


lib = _load_library()


def _status_name(s: int) -> str:
    return lib.rmm_status_string(int(s)).decode()


def rmm_status_string(s: int) -> str:
    return _status_name(s)


def rmm_version() -> str:
    return lib.rmm_version().decode()


def _check(status: int, what: str):
    if status != RMM_OK:
        raise RmmError(status, what)


def rmm_problem_init(mode: int, dtype: int, n: int, d: int, m: int) -> rmm_problem:
    p = rmm_problem()
    lib.rmm_problem_init(ctypes.byref(p), mode, dtype, n, d, m)
    return p


class Plan:
    """Owns an rmm_plan (host memory) created from an rmm_problem."""

    def __init__(self, problem: rmm_problem):
        self.problem = problem
        h = ctypes.c_void_p()
        ws = ctypes.c_size_t()
        _check(lib.rmm_plan_create(ctypes.byref(h), ctypes.byref(problem), ctypes.byref(ws)),
               "rmm_plan_create")
        self.handle = h
        self.workspace_bytes = int(ws.value)
        self.k = int(lib.rmm_plan_k(h))
        self.kernel_launches = int(lib.rmm_plan_kernel_launches(h))
        self._ws = {}  # (device index, stream) -> workspace; released with the plan

    def set_product_events(self, start=None, stop=None):
        """Bracket the reduced-product kernel of later calls with torch.cuda.Event
        objects (created with enable_timing=True); None clears the hook."""
        def raw(e):
            if e is None:
                return None
            if not e.cuda_event:
                e.record()  # torch creates the event lazily on its first record
            return ctypes.c_void_p(e.cuda_event)
        _check(lib.rmm_plan_set_product_events(self.handle, raw(start), raw(stop)),
               "rmm_plan_set_product_events")

    def __del__(self):
        h = getattr(self, "handle", None)
        L = globals().get("lib")
        if h is not None and h.value and L is not None:  # lib is gone at interpreter exit
            L.rmm_plan_destroy(h)
            self.handle = None


def rmm_plan_create(problem: rmm_problem) -> Plan:
    return Plan(problem)


def rmm_plan_set_product_events(plan: Plan, start=None, stop=None):
    plan.set_product_events(start, stop)


def rmm_plan_kernel_launches(plan: Plan) -> int:
    return int(lib.rmm_plan_kernel_launches(plan.handle))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size()


def rmm_workspace_init(plan: Plan, workspace, stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_workspace_init(plan.handle, wp, wb, _stream(stream)), "rmm_workspace_init")


def rmm_selftest_wait_timeout(plan: Plan, workspace, stream=None):
    """Make one bounded wait run out on purpose (see include/rmm.h); the next
    rmm_workspace_status then reports RMM_ERR_TIMEOUT."""
    wp, wb = _ws(workspace)
    _check(lib.rmm_selftest_wait_timeout(plan.handle, wp, wb, _stream(stream)), "rmm_selftest_wait_timeout")


def rmm_workspace_status(plan: Plan, workspace, stream=None) -> int:
    return int(lib.rmm_workspace_status(plan.handle, _ptr(workspace), _stream(stream)))


def rmm_select(plan: Plan, A, I, s2=None, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_select(plan.handle, _ptr(A), _ptr(I), _ptr(s2), wp, wb, _stream(stream)), "rmm_select")


def rmm_select_no_alloc(plan: Plan, A, I, s2=None, stream=None):
    """rmm_select without a workspace: scratch lives in a static device array
    inside librmm (see include/rmm.h for the size limit and the rules on
    overlapping calls)."""
    _check(lib.rmm_select_no_alloc(plan.handle, _ptr(A), _ptr(I), _ptr(s2), _stream(stream)),
           "rmm_select_no_alloc")


def rmm_matmul(plan: Plan, A, B, Y, I=None, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_matmul(plan.handle, _ptr(A), _ptr(B), _ptr(Y), _ptr(I), wp, wb, _stream(stream)),
           "rmm_matmul")


def rmm_matmul_batched(plan: Plan, A, B, Y, I=None, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_matmul_batched(plan.handle, _ptr(A), _ptr(B), _ptr(Y), _ptr(I), wp, wb,
                                  _stream(stream)), "rmm_matmul_batched")


def rmm_matmul_ex(plan: Plan, A, B, Y, I=None, s2_in=None, s2_out=None, workspace=None, stream=None):
    """rmm_matmul_batched with producer-fused scoring: s2_in (fp32 [heads][d])
    with RMM_FLAG_GIVEN_SCORES, s2_out (fp32 [heads][m]) with RMM_FLAG_EMIT_SCORES."""
    wp, wb = _ws(workspace)
    _check(lib.rmm_matmul_ex(plan.handle, _ptr(A), _ptr(B), _ptr(Y), _ptr(I), _ptr(s2_in), _ptr(s2_out), wp, wb,
                             _stream(stream)), "rmm_matmul_ex")


def rmm_softmax_workspace_size(heads: int, n: int, t: int) -> int:
    return int(lib.rmm_softmax_workspace_size(heads, n, t))


def rmm_softmax_scores(S, P, s2, heads, n, t, lds, stride_s, ldp, stride_p, flags=0, workspace=None,
                       stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_softmax_scores(_ptr(S), _ptr(P), _ptr(s2), heads, n, t, lds, stride_s, ldp, stride_p,
                                  int(flags), wp, wb, _stream(stream)), "rmm_softmax_scores")


def rmm_attention_workspace_size(problem: rmm_attn_problem) -> int:
    return int(lib.rmm_attention_workspace_size(ctypes.byref(problem)))


def rmm_attention(problem: rmm_attn_problem, Q, K, V, O, I=None, T=None, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(lib.rmm_attention(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(I), _ptr(T), wp, wb,
                             _stream(stream)), "rmm_attention")


# ----------------------------------------------------------------------------
# Convenience layer over torch tensors (still marshalling only).
# ----------------------------------------------------------------------------
_cache_lock = threading.Lock()
_plans: dict = {}
_ws_plans = weakref.WeakSet()  # plans that own a workspace (for check_workspaces)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return RMM_BF16
    if t.dtype == torch.float32:
        return RMM_F32
    if t.dtype == torch.float8_e4m3fn:
        return RMM_FP8_E4M3
    raise TypeError(f"RMM supports bfloat16, float32 and float8_e4m3fn tensors, not {t.dtype}")


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("RMM tensors must live on a CUDA device (there is no CPU path)")


def _row_stride(t) -> int:
    if t.numel() == 0:
        return t.shape[-1]
    if t.stride(-1) != 1:
        raise ValueError("the last dimension must be contiguous")
    return t.stride(-2) if t.dim() >= 2 and t.shape[-2] > 1 else t.shape[-1]


def _plan_for(p: rmm_problem) -> Plan:
    key = tuple(getattr(p, f) for f, _ in rmm_problem._fields_)
    import torch
    key = key + (torch.cuda.current_device(),)
    with _cache_lock:
        plan = _plans.get(key)
        if plan is None:
            plan = Plan(p)
            _plans[key] = plan
    return plan


def workspace_for(plan: Plan, device=None, stream=None):
    """A zero-initialised workspace for a plan, kept on the plan per (device,
    stream): it lives as long as the plan, and a later plan never inherits it
    (its counters are laid out for this plan)."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    s = torch.cuda.current_stream(dev) if stream is None else stream
    key = (dev.index, s.cuda_stream)
    with _cache_lock:
        ws = plan._ws.get(key)
    if ws is None or ws.numel() < plan.workspace_bytes:
        ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device=dev)
        ws.record_stream(s)  # used on s: not reused before s's work on it is done
        rmm_workspace_init(plan, ws, s)
        with _cache_lock:
            plan._ws[key] = ws
            _ws_plans.add(plan)
    return ws


def check_workspaces():
    """Synchronise and read the error word of every workspace this module
    allocated; raise RmmError(RMM_ERR_TIMEOUT) if a kernel gave up on a wait."""
    import torch
    with _cache_lock:
        items = [(p, ws) for p in list(_ws_plans) for ws in list(p._ws.values())]
        raw = [ws for key, ws in _plans.items() if key[0] in ("softmax", "attention")]
    for plan, ws in items:
        _check(rmm_workspace_status(plan, ws), "kernel wait")
    if raw:
        torch.cuda.synchronize()
    for ws in raw:  # the softmax and attention workspaces keep their error word in the first 4 bytes
        if int(ws[:4].view(torch.int32).item()) != 0:
            raise RmmError(RMM_ERR_TIMEOUT, "kernel wait")


def _k_fields(p: rmm_problem, rho, k):
    if k is not None:
        p.k = int(k)
    elif rho is not None:
        p.rho = float(rho)
    else:
        raise ValueError("give rho or k")


def select(A, rho=None, k=None, return_scores=False):
    """I (and optionally fp32 s^2) for activations A [n, d] or [heads, n, d]."""
    import torch
    _require_cuda(A)
    heads = A.shape[0] if A.dim() == 3 else 1
    n, d = A.shape[-2], A.shape[-1]
    p = rmm_problem_init(RMM_LINEAR, _dtype_code(A), n, d, 8)
    p.lda = _row_stride(A)
    p.heads = heads
    p.kv_heads = 1
    p.stride_a = A.stride(0) if A.dim() == 3 else 0
    p.ldy, p.stride_y = 8, n * 8  # no product: the output layout only has to be valid
    _k_fields(p, rho, k)
    plan = _plan_for(p)
    I = torch.empty((heads, plan.k) if A.dim() == 3 else (plan.k,), dtype=torch.int32, device=A.device)
    s2 = torch.empty((heads, d) if A.dim() == 3 else (d,), dtype=torch.float32, device=A.device) \
        if return_scores else None
    rmm_select(plan, A, I, s2, workspace_for(plan))
    return (I, s2) if return_scores else I


def matmul(A, B, rho=None, k=None, indices=None, return_indices=False, out=None, scores=None,
           emit_scores=False, alpha=1.0):
    """RMM_rho(A, B) = alpha A[:, I] B[I, :] for A [n, d], B [d, m] (§3.2).
    scores: A's column scores from the op that produced A (fp32 [d]); the op
    then selects from them instead of reading A for them.  emit_scores=True
    also returns Y's column scores (fp32 [m]) for the op that takes Y next.
    float8_e4m3fn A and B (the low-bit form) give a bf16 Y; pass their
    per-tensor scales as alpha = scale_A * scale_B."""
    import torch
    _require_cuda(A, B, out, indices, scores)
    n, d = A.shape
    m = B.shape[1]
    if B.shape[0] != d or B.dtype != A.dtype:
        raise ValueError("A is n x d and B is d x m with the same dtype")
    p = rmm_problem_init(RMM_LINEAR, _dtype_code(A), n, d, m)
    p.lda, p.ldb = _row_stride(A), _row_stride(B)
    p.alpha = float(alpha)
    if indices is not None:
        p.k = indices.numel()
        p.flags |= RMM_FLAG_USE_GIVEN_INDICES
    else:
        _k_fields(p, rho, k)
    if scores is not None:
        p.flags |= RMM_FLAG_GIVEN_SCORES
    if emit_scores:
        p.flags |= RMM_FLAG_EMIT_SCORES
    y_dtype = torch.bfloat16 if A.dtype == torch.float8_e4m3fn else A.dtype
    Y = torch.empty((n, m), dtype=y_dtype, device=A.device) if out is None else out
    p.ldy = _row_stride(Y)
    plan = _plan_for(p)
    I = indices
    if I is None and return_indices:
        I = torch.empty(plan.k, dtype=torch.int32, device=A.device)
    if scores is None and not emit_scores:
        rmm_matmul(plan, A, B, Y, I, workspace_for(plan))
        return (Y, I) if return_indices else Y
    s2 = torch.empty(m, dtype=torch.float32, device=A.device) if emit_scores else None
    rmm_matmul_ex(plan, A, B, Y, I, scores, s2, workspace_for(plan))
    out_t = (Y,) + ((I,) if return_indices else ()) + ((s2,) if emit_scores else ())
    return out_t if len(out_t) > 1 else Y


def qk(Q, K, rho, alpha=None, causal=True, return_indices=False):
    """Reduced attention scores S[h] = alpha Q[h][:, I_h] K[g][:, I_h]^T (+ causal
    mask) for Q [H, n, d_h] and K [H_kv, m, d_h] (§3.3 "Attention")."""
    import torch
    _require_cuda(Q, K)
    H, n, dh = Q.shape
    Hkv, m, _ = K.shape
    p = rmm_problem_init(RMM_QK, _dtype_code(Q), n, dh, m)
    p.lda, p.ldb = _row_stride(Q), _row_stride(K)
    p.heads, p.kv_heads = H, Hkv
    p.stride_a, p.stride_b = Q.stride(0), K.stride(0)
    p.alpha = 1.0 / math.sqrt(dh) if alpha is None else float(alpha)
    p.flags = RMM_FLAG_CAUSAL if causal else 0
    _k_fields(p, rho, None)
    S = torch.empty((H, n, m), dtype=Q.dtype, device=Q.device)
    p.ldy, p.stride_y = m, n * m
    plan = _plan_for(p)
    I = torch.empty((H, plan.k), dtype=torch.int32, device=Q.device) if return_indices else None
    rmm_matmul_batched(plan, Q, K, S, I, workspace_for(plan))
    return (S, I) if return_indices else S


def softmax_scores(S, causal=False):
    """Attention weights P = softmax(S) over each row of S [H, n, t] (bf16,
    -inf = masked), with the token scores s2[h][t] = sum_i P[h][i][t]^2 of the
    stored weights (the op producing P scores its columns, §3.3 "Attention").
    Returns (P, s2)."""
    import torch
    _require_cuda(S)
    if S.dtype != torch.bfloat16:
        raise TypeError("softmax_scores takes bf16 scores")
    H, n, t = S.shape
    P = torch.empty_like(S)
    s2 = torch.empty((H, t), dtype=torch.float32, device=S.device)
    key = ("softmax", H, n, t, S.device.index)
    with _cache_lock:
        ws = _plans.get(key)
    if ws is None:
        ws = torch.zeros(max(rmm_softmax_workspace_size(H, n, t), 256), dtype=torch.uint8, device=S.device)
        with _cache_lock:
            _plans[key] = ws
    rmm_softmax_scores(S, P, s2, H, n, t, _row_stride(S), S.stride(0), _row_stride(P), P.stride(0),
                       RMM_FLAG_CAUSAL if causal else 0, ws)
    return P, s2


def attention(Q, K, V, rho_d, rho_t, causal=True, alpha=None, return_sets=False):
    """Fused RMM attention (§3.3 "Attention"): features of Q per head (rho_d),
    softmax of the reduced scores, tokens by P's column norms (rho_t), output
    over the kept tokens -- without writing S or P.  Q [H, n, 128],
    K and V [H_kv, n, 128], bf16.  Returns O (and I, T with return_sets)."""
    import torch
    _require_cuda(Q, K, V)
    H, n, dh = Q.shape
    Hkv, _, dv = V.shape
    p = rmm_attn_problem()
    p.heads, p.kv_heads, p.n, p.d_h, p.d_v = H, Hkv, n, dh, dv
    p.ldq, p.ldk, p.ldv = _row_stride(Q), _row_stride(K), _row_stride(V)
    p.stride_q, p.stride_k, p.stride_v = Q.stride(0), K.stride(0), V.stride(0)
    O = torch.empty((H, n, dv), dtype=Q.dtype, device=Q.device)
    p.ldo, p.stride_o = dv, n * dv
    p.rho_d, p.rho_t = float(rho_d), float(rho_t)
    p.alpha = 1.0 / math.sqrt(dh) if alpha is None else float(alpha)
    p.flags = RMM_FLAG_CAUSAL if causal else 0
    size = rmm_attention_workspace_size(p)
    if size == 0:
        raise RmmError(RMM_ERR_INVALID_ARG, "rmm_attention_workspace_size")
    key = ("attention", H, Hkv, n, float(rho_d), float(rho_t), Q.device.index)
    with _cache_lock:
        ws = _plans.get(key)
    if ws is None or ws.numel() < size:
        ws = torch.zeros(max(size, 256), dtype=torch.uint8, device=Q.device)
        with _cache_lock:
            _plans[key] = ws
    kd = _retained(float(rho_d), dh)
    kt = _retained(float(rho_t), n)
    I = torch.empty((H, kd), dtype=torch.int32, device=Q.device) if return_sets else None
    T = torch.empty((H, kt), dtype=torch.int32, device=Q.device) if return_sets else None
    rmm_attention(p, Q, K, V, O, I, T, ws)
    return (O, I, T) if return_sets else O


def attention_status(Q, K, V, rho_d, rho_t) -> int:
    """The error word of the workspace attention() used for these sizes: 0, or
    the code of a kernel that gave up on a wait (synchronises)."""
    import torch
    H, n = Q.shape[0], Q.shape[1]
    key = ("attention", H, K.shape[0], n, float(rho_d), float(rho_t), Q.device.index)
    with _cache_lock:
        ws = _plans.get(key)
    if ws is None:
        return 0
    torch.cuda.synchronize()
    return int(ws[:4].view(torch.int32).item())


def _retained(rho: float, d: int) -> int:
    x = rho * d
    r = round(x)
    k = r if abs(x - r) <= 1e-9 * d else math.ceil(x)
    return max(1, min(d, int(k)))


def pv(P, V, rho, return_indices=False, causal=False, scores=None):
    """Token-reduced value product O[h] = P[h][:, T_h] V[g][T_h, :] for
    P [H, n, n_k] and V [H_kv, n_k, d_v] (§3.3 "Attention", last sentence).
    causal=True states that P[h][i][t] = 0 for t > i (n = n_k): the op then
    skips the blocks of P above the diagonal (same result).  scores: P's token
    scores from the op that produced P (softmax_scores), fp32 [H, n_k]; the
    op then selects from them instead of reading P for them."""
    import torch
    _require_cuda(P, V)
    H, n, nk = P.shape
    Hkv, _, dv = V.shape
    p = rmm_problem_init(RMM_PV, _dtype_code(P), n, nk, dv)
    p.lda, p.ldb = _row_stride(P), _row_stride(V)
    p.heads, p.kv_heads = H, Hkv
    p.stride_a, p.stride_b = P.stride(0), V.stride(0)
    p.flags = RMM_FLAG_CAUSAL if causal else 0
    if scores is not None:
        _require_cuda(scores)
        p.flags |= RMM_FLAG_GIVEN_SCORES
    _k_fields(p, rho, None)
    O = torch.empty((H, n, dv), dtype=P.dtype, device=P.device)
    p.ldy, p.stride_y = dv, n * dv
    plan = _plan_for(p)
    T = torch.empty((H, plan.k), dtype=torch.int32, device=P.device) if return_indices else None
    if scores is None:
        rmm_matmul_batched(plan, P, V, O, T, workspace_for(plan))
    else:
        rmm_matmul_ex(plan, P, V, O, T, scores, None, workspace_for(plan))
    return (O, T) if return_indices else O
