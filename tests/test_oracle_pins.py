"""Pins of the CPU oracle to the RMM paper (no GPU).

The oracle is the definition of the method written out in fp64; these tests
tie it to things other than itself (see oracle_checks.py for each pin and the
passage of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" it follows).
"""
import math

import numpy as np
import pytest

import oracle
from tests import oracle_checks as oc


@pytest.mark.parametrize("check", oc.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check):
    check(oracle)


def _qk_inputs(seed, H=4, Hkv=2, n=24, dh=16):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((H, n, dh)) * np.exp(rng.standard_normal((H, 1, dh)))
    K = rng.standard_normal((Hkv, n, dh)) * np.exp(rng.standard_normal((Hkv, 1, dh)))
    return Q, K


def test_qk_dense_special_case_and_mask():
    """§3.3 Attention: at rho_d = 1, S_h = (1/sqrt(d_h)) Q_h K_g^T with the
    grouped-query head g = h // (H/H_kv); the causal mask M puts -inf where the
    key index exceeds the query index.  Dense reference from numpy."""
    Q, K = _qk_inputs(1)
    H, n, dh = Q.shape
    alpha = 1.0 / math.sqrt(dh)
    S, I = oracle.rmm_qk(Q, K, rho=1.0, alpha=alpha, causal=True)
    assert np.array_equal(I, np.tile(np.arange(dh, dtype=np.int32), (H, 1)))
    upper = np.triu(np.ones((n, n), dtype=bool), 1)
    for h in range(H):
        ref = alpha * Q[h] @ K[h // 2].T
        assert np.all(np.isneginf(S[h][upper]))
        assert np.allclose(S[h][~upper], ref[~upper], rtol=1e-12, atol=1e-12)
    S_nc, _ = oracle.rmm_qk(Q, K, rho=1.0, alpha=alpha, causal=False)
    for h in range(H):
        assert np.allclose(S_nc[h], alpha * Q[h] @ K[h // 2].T, rtol=1e-12, atol=1e-12)


def test_qk_per_head_selection_and_bound():
    """§3.3 Attention: selection is per query head on Q's feature norms, and the
    same features of the shared K head are used; Proposition 1 bounds each
    head's error with B = K_g^T."""
    Q, K = _qk_inputs(2)
    H, n, dh = Q.shape
    for rho in (0.5, 0.8):
        S, I = oracle.rmm_qk(Q, K, rho=rho, alpha=1.0, causal=False)
        k = math.ceil(rho * dh)
        assert I.shape == (H, k)
        for h in range(H):
            s2 = (Q[h] ** 2).sum(axis=0)
            order = sorted(range(dh), key=lambda j: (-s2[j], j))
            assert I[h].tolist() == sorted(order[:k])
            full = Q[h] @ K[h // 2].T
            drop = np.setdiff1d(np.arange(dh), I[h])
            bound = np.sum(np.linalg.norm(Q[h][:, drop], axis=0) *
                           np.linalg.norm(K[h // 2][:, drop], axis=0))
            assert np.linalg.norm(full - S[h]) <= bound * (1 + 1e-12)
    rows = [0, 5, 23]
    S_all, _ = oracle.rmm_qk(Q, K, rho=0.5, alpha=0.25, causal=True)
    S_rows, _ = oracle.rmm_qk(Q, K, rho=0.5, alpha=0.25, causal=True, rows=rows)
    assert np.array_equal(S_rows, S_all[:, rows])


def test_pv_dense_special_case_and_bound():
    """§3.3 Attention (token selection) and Appendix D.1 Eq. (2): at rho_t = 1
    the product is the dense P_h V_g; below 1, Proposition 1 bounds the error
    with A = P_h (token columns) and B = V_g (token rows)."""
    rng = np.random.default_rng(3)
    H, Hkv, n, dv = 4, 2, 20, 8
    logits = rng.standard_normal((H, n, n)) * 2.0
    logits[:, np.triu(np.ones((n, n), dtype=bool), 1)] = -np.inf
    P = np.exp(logits - logits.max(-1, keepdims=True))
    P /= P.sum(-1, keepdims=True)
    V = rng.standard_normal((Hkv, n, dv))
    O, T = oracle.rmm_pv(P, V, rho=1.0)
    for h in range(H):
        assert np.allclose(O[h], P[h] @ V[h // 2], rtol=1e-12, atol=1e-14)
    for rho in (0.5, 0.8):
        O, T = oracle.rmm_pv(P, V, rho=rho)
        for h in range(H):
            drop = np.setdiff1d(np.arange(n), T[h])
            bound = np.sum(np.linalg.norm(P[h][:, drop], axis=0) *
                           np.linalg.norm(V[h // 2][drop, :], axis=1))
            assert np.linalg.norm(P[h] @ V[h // 2] - O[h]) <= bound * (1 + 1e-12) + 1e-15


def test_decode_one_row_selection_is_a_magnitude_sort():
    """Appendix D.1, the decode case: one query row per head.  With n = 1 the
    column norm of column j is |a_j|, so the oracle's TopK must equal the k
    largest magnitudes in a stable library sort (equal magnitudes in index
    order, which is the lower-index tie rule), returned ascending.  Values of
    both signs, zeros and exact ties."""
    rng = np.random.default_rng(17)
    vals = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 2.0, -3.0, 0.25])
    for d in (7, 64, 1000):
        a = vals[rng.integers(0, len(vals), size=(1, d))]
        for k in sorted({1, 3, d // 2, d - 1}):
            order = np.argsort(-np.abs(a[0]), kind="stable")
            expect = np.sort(order[:k]).astype(np.int32)
            got, _ = oracle.select(a, k=k)
            assert np.array_equal(np.asarray(got), expect), (d, k)


def test_decode_group_scores_and_values():
    """Decode-step forms on the oracle's per-head functions: with one query row,
    QK's scores at rho = 1 equal alpha * q K^T (numpy) for every KV head's
    query heads, and PV's output at rho = 1 equals P V (numpy); below rho = 1
    the PV error obeys the bound of Prop. 1 per head."""
    rng = np.random.default_rng(23)
    H, Hkv, t, dh = 8, 2, 40, 16
    q = rng.standard_normal((H, 1, dh))
    K = rng.standard_normal((Hkv, t, dh))
    V = rng.standard_normal((Hkv, t, dh))
    P = rng.random((H, 1, t))
    S, _ = oracle.rmm_qk(q, K, rho=1.0, alpha=0.25, causal=False)
    O, _ = oracle.rmm_pv(P, V, rho=1.0)
    for h in range(H):
        g = h // (H // Hkv)
        np.testing.assert_allclose(S[h], 0.25 * q[h] @ K[g].T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(O[h], P[h] @ V[g], rtol=1e-12, atol=1e-12)
    O5, T5 = oracle.rmm_pv(P, V, rho=0.5)
    for h in range(H):
        g = h // (H // Hkv)
        drop = np.setdiff1d(np.arange(t), T5[h])
        bound = sum(np.abs(P[h][0, j]) * np.linalg.norm(V[g][j]) for j in drop)
        assert np.linalg.norm(P[h] @ V[g] - O5[h]) <= bound * (1 + 1e-12) + 1e-12
