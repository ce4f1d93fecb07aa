"""CPU oracle for Reduced Matrix Multiplication -- TEST INFRASTRUCTURE ONLY.

Plain fp64 statement of what the CUDA path computes, written from
"Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
LLM Inference" (arXiv 2608.13426), called "the RMM paper" below.  The
arithmetic lives in ``rmm_oracle.c`` (plain C, fp64); this module loads it with
ctypes and composes the per-head forms.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  It shares no code with the CUDA library and never
calls it.  Every function pins to the paper as follows (tests/test_oracle_pins.py):
  retained_count      -- k values worked out by hand from ceil(rho*d) (golden file)
  column_scores_sq    -- n=1 closed form, 2^p scaling, exact small-integer sums
  topk_indices        -- brute force over all subsets (Theorem 1 / Eq. 18)
  reduced_product     -- rho=1 equals numpy's dense product; Prop. 1 / Cor. 1 /
                         Eq. 17 bounds; equality in the rank-one construction;
                         sampled rows equal the full result's rows
  reduced_scores      -- rho=1 equals alpha*Q K^T; causal entries are -inf;
                         sampled rows masked by their own position
  rmm_qk / rmm_pv     -- rho=1 dense special cases; below rho = 1 the sets are
                         the largest column norms of Q (QK) and P (PV) by
                         enumeration over every subset, within Proposition 1
  decode_e4m3         -- hand-worked codes (golden file) and every code against
                         torch's float8_e4m3fn conversion
  rmm_attention       -- rho = 1 equals scipy's softmax attention; I is Q's
                         largest column norms and P scipy's softmax over I
                         alone; the token step obeys Proposition 1 on P V; its
                         sets are the TopK of the oracle's own column norms
  softmax_rows        -- closed forms (uniform row, two-key logistic), masked
                         entries exactly 0, rows sum to 1 and not columns,
                         per-row shift invariance, large logits stay finite
No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rmm_oracle.c")
_LIB = os.path.join(_HERE, "librmm_oracle.so")
_lock = threading.Lock()
_lib = None

_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile rmm_oracle.c into librmm_oracle.so with gcc (fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.rmm_oracle_retained_count.restype = _i64
            lib.rmm_oracle_retained_count.argtypes = [ctypes.c_double, _i64]
            lib.rmm_oracle_column_scores_sq.restype = None
            lib.rmm_oracle_column_scores_sq.argtypes = [_f64p, _i64, _i64, _i64, _f64p]
            lib.rmm_oracle_topk_indices.restype = ctypes.c_int
            lib.rmm_oracle_topk_indices.argtypes = [_f64p, _i64, _i64, _i32p]
            lib.rmm_oracle_reduced_product.restype = None
            lib.rmm_oracle_reduced_product.argtypes = [_f64p, _i64, _f64p, _i64, _i64, _i64,
                                                       _i32p, _i64, _f64p, _i64]
            lib.rmm_oracle_decode_e4m3.restype = ctypes.c_int
            lib.rmm_oracle_decode_e4m3.argtypes = [ctypes.POINTER(ctypes.c_uint8), _i64, _f64p]
            lib.rmm_oracle_softmax_rows.restype = ctypes.c_int
            lib.rmm_oracle_softmax_rows.argtypes = [_f64p, _i64, _i64, _i64, _f64p, _i64]
            lib.rmm_oracle_reduced_scores.restype = None
            lib.rmm_oracle_reduced_scores.argtypes = [_f64p, _i64, _f64p, _i64, _i64, _i64, _i64,
                                                      _i32p, _i64, ctypes.c_double, ctypes.c_int,
                                                      _f64p, _i64]
            _lib = lib
    return _lib


def as_f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (bf16/fp32/fp64) or array to C-contiguous fp64."""
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def retained_count(rho: float, d: int) -> int:
    """k = ceil(rho*d) [RMM paper, §3.2]; see rmm_oracle.c for the rounding reading."""
    k = _load().rmm_oracle_retained_count(float(rho), int(d))
    if k < 0:
        raise ValueError("rho must lie in (0, 1] and d >= 1")
    return int(k)


def column_scores_sq(A) -> np.ndarray:
    """s2[j] = ||A[:, j]||_2^2 in fp64 [RMM paper, §3.2]."""
    A = as_f64(A)
    n, d = A.shape
    s2 = np.empty(d, dtype=np.float64)
    _load().rmm_oracle_column_scores_sq(_p(A, _f64p), n, d, d, _p(s2, _f64p))
    return s2


def topk_indices(s2, k: int) -> np.ndarray:
    """Ascending int32 I = TopK(s, k), ties to the lower index [RMM paper, §3.2]."""
    s2 = as_f64(s2).ravel()
    I = np.empty(int(k), dtype=np.int32)
    if _load().rmm_oracle_topk_indices(_p(s2, _f64p), s2.size, int(k), _p(I, _i32p)) != 0:
        raise ValueError("bad k for TopK")
    return I


def select(A, rho: float | None = None, k: int | None = None):
    """(I, s2) for activations A: scores, then TopK [RMM paper, §3.2]."""
    A = as_f64(A)
    if k is None:
        k = retained_count(rho, A.shape[1])
    s2 = column_scores_sq(A)
    return topk_indices(s2, k), s2


def reduced_product(A, B, I, rows=None) -> np.ndarray:
    """Y = A[:, I] B[I, :] in fp64 [RMM paper, §3.2].  ``rows`` restricts the
    output to a subset of A's rows (for sampled checks at full size)."""
    A = as_f64(A)
    B = as_f64(B)
    if rows is not None:
        A = np.ascontiguousarray(A[np.asarray(rows)])
    I = np.ascontiguousarray(np.asarray(I, dtype=np.int32))
    n, m = A.shape[0], B.shape[1]
    Y = np.empty((n, m), dtype=np.float64)
    _load().rmm_oracle_reduced_product(_p(A, _f64p), A.shape[1], _p(B, _f64p), B.shape[1],
                                       n, m, _p(I, _i32p), I.size, _p(Y, _f64p), m)
    return Y


def rmm(A, B, rho: float | None = None, k: int | None = None):
    """RMM_rho(A, B) = A[:, I] B[I, :] with I from A's column norms [RMM paper, §3.2].
    Returns (Y fp64, I int32 ascending)."""
    I, _ = select(A, rho=rho, k=k)
    return reduced_product(A, B, I), I


def reduced_scores(Q, K, I, alpha: float, causal: bool, rows=None) -> np.ndarray:
    """S = alpha * Q[:, I] K[:, I]^T with the optional causal mask [RMM paper, §3.3].
    ``rows`` restricts to a subset of query rows (their true row index is kept
    for the mask)."""
    Q = as_f64(Q)
    K = as_f64(K)
    I = np.ascontiguousarray(np.asarray(I, dtype=np.int32))
    nq, nk = Q.shape[0], K.shape[0]
    lib = _load()
    if rows is None:
        S = np.empty((nq, nk), dtype=np.float64)
        lib.rmm_oracle_reduced_scores(_p(Q, _f64p), Q.shape[1], _p(K, _f64p), K.shape[1],
                                      nq, nk, 0, _p(I, _i32p), I.size, float(alpha),
                                      int(bool(causal)), _p(S, _f64p), nk)
        return S
    out = np.empty((len(rows), nk), dtype=np.float64)
    for r_out, r in enumerate(rows):
        q = np.ascontiguousarray(Q[int(r)][None, :])
        lib.rmm_oracle_reduced_scores(_p(q, _f64p), Q.shape[1], _p(K, _f64p), K.shape[1],
                                      1, nk, int(r), _p(I, _i32p), I.size, float(alpha),
                                      int(bool(causal)), _p(out[r_out:], _f64p), nk)
    return out


def decode_e4m3(codes) -> np.ndarray:
    """Exact fp64 values of E4M3 (OCP 8-bit float, e4m3fn) codes: uint8 array
    or a torch float8_e4m3fn tensor (its bytes).  The low-bit form of RMM
    stores A and B in this format (see rmm_oracle.c)."""
    if hasattr(codes, "detach"):
        codes = codes.detach().to("cpu").contiguous().view(__import__("torch").uint8).numpy()
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    if _load().rmm_oracle_decode_e4m3(c.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), c.size,
                                      _p(out, _f64p)) != 0:
        raise ValueError("NaN code in an E4M3 operand")
    return out


def softmax_rows(S) -> np.ndarray:
    """Attention weights P = softmax(S + M) over the key axis of each row, the
    mask M given as -inf entries of S [RMM paper, §3.3 "Attention"].  S is
    [n, t] or [heads, n, t]; fp64 out."""
    S = as_f64(S)
    if S.ndim == 3:
        return np.stack([softmax_rows(S[h]) for h in range(S.shape[0])])
    n, t = S.shape
    P = np.empty((n, t), dtype=np.float64)
    if _load().rmm_oracle_softmax_rows(_p(S, _f64p), t, n, t, _p(P, _f64p), t) != 0:
        raise ValueError("a row of S has no finite entry")
    return P


def kv_head_of(h: int, heads: int, kv_heads: int) -> int:
    """Grouped-query attention: query head h reads shared K/V head h // (heads/kv_heads)
    [RMM paper, §3.3: selection per query head, matching dims gathered from shared K, V]."""
    return h // (heads // kv_heads)


def rmm_qk(Q, K, rho: float, alpha: float, causal: bool = True, heads=None, rows=None):
    """Per-head reduced scores [RMM paper, §3.3 "Attention"].

    Q: [H, nq, d_h], K: [H_kv, nk, d_h].  For each query head h the index set
    I_h = TopK of Q_h's column norms over the d_h features, the same features
    of K's shared head are used, and S_h = alpha * Q_h[:, I_h] K_g[:, I_h]^T with
    the causal mask.  Returns (S [len(heads), rows, nk] fp64, I [H, k] int32);
    I is always computed for every head, S only for ``heads`` (default all).
    """
    Q = as_f64(Q)
    K = as_f64(K)
    H, _, dh = Q.shape
    Hkv = K.shape[0]
    k = retained_count(rho, dh)
    I = np.stack([select(Q[h], k=k)[0] for h in range(H)])
    hs = range(H) if heads is None else heads
    S = np.stack([reduced_scores(Q[h], K[kv_head_of(h, H, Hkv)], I[h], alpha, causal, rows)
                  for h in hs])
    return S, I


def rmm_attention(Q, K, V, rho_d: float, rho_t: float, alpha: float, causal: bool = True):
    """RMM attention of every head [RMM paper, §3.3 "Attention"], the three steps
    in the paper's order: features I_h = TopK of Q_h's column norms (rho_d)
    and S_h = alpha Q_h[:, I_h] K_g[:, I_h]^T + M; P_h = softmax(S_h) over each
    row; tokens T_h = TopK of P_h's column norms (rho_t) and
    O_h = P_h[:, T_h] V_g[T_h, :].  Q [H, n, d_h], K [H_kv, n_k, d_h],
    V [H_kv, n_k, d_v].  Returns (O [H, n, d_v], I [H, k_d], T [H, k_t], P [H, n, n_k]),
    all fp64 (I, T int32)."""
    Q, K, V = as_f64(Q), as_f64(K), as_f64(V)
    H = Q.shape[0]
    Hkv = K.shape[0]
    S, I = rmm_qk(Q, K, rho=rho_d, alpha=alpha, causal=causal)
    P = softmax_rows(S)
    kt = retained_count(rho_t, P.shape[2])
    T = np.stack([select(P[h], k=kt)[0] for h in range(H)])
    O = np.stack([reduced_product(P[h], V[kv_head_of(h, H, Hkv)], T[h]) for h in range(H)])
    return O, I, T, P


def rmm_pv(P, V, rho: float, heads=None, rows=None):
    """Per-head token-selected value product [RMM paper, §3.3 "Attention", last
    sentence; Appendix D.1, Eq. (2)].

    P: [H, nq, nk] attention weights, V: [H_kv, nk, d_v].  For each head h the
    token set T_h = TopK of P_h's column norms over the nk token positions and
    O_h = P_h[:, T_h] V_g[T_h, :].  Returns (O fp64, T [H, k] int32).
    """
    P = as_f64(P)
    V = as_f64(V)
    H, _, nk = P.shape
    Hkv = V.shape[0]
    k = retained_count(rho, nk)
    T = np.stack([select(P[h], k=k)[0] for h in range(H)])
    hs = range(H) if heads is None else heads
    O = np.stack([reduced_product(P[h], V[kv_head_of(h, H, Hkv)], T[h], rows) for h in hs])
    return O, T
