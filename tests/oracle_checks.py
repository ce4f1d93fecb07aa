"""Checks that pin the CPU oracle to what the RMM paper fixes.

Each check takes an implementation object with the oracle's interface
(``retained_count``, ``column_scores_sq``, ``topk_indices``,
``reduced_product``) and raises AssertionError when it disagrees with
something other than itself: brute-force enumeration, a closed form, a
theorem's bound, or numpy's dense product.  The real oracle must pass all of
them (test_oracle_pins.py); deliberately broken copies of it must each fail at
least one (test_oracle_mutants.py).

Paper: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
Reduction for LLM Inference" (arXiv 2608.13426).
"""
from __future__ import annotations

import itertools
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def check_retained_counts(impl):
    """k = ceil(rho d) [§3.2] against counts worked out by hand."""
    with open(os.path.join(GOLDEN, "retained_counts.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            rho, d, k = line.split()
            got = impl.retained_count(float(rho), int(d))
            assert got == int(k), f"retained_count({rho}, {d}) = {got}, want {k}"


def check_scores_closed_forms(impl):
    """s_j^2 = sum_i A[i,j]^2 [§3.2]: small integer matrices with sums done by
    hand, and the one-row case s_j = |a_j|."""
    A = np.array([[1.0, 2.0, 0.0, -3.0], [3.0, -4.0, 0.0, 1.0], [0.0, 1.0, 5.0, 1.0]])
    want = np.array([10.0, 21.0, 25.0, 11.0])
    got = impl.column_scores_sq(A)
    assert np.array_equal(got, want), (got, want)
    row = np.array([[-0.5, 0.25, 3.0, -3.0, 0.0]])
    assert np.array_equal(impl.column_scores_sq(row), np.array([0.25, 0.0625, 9.0, 9.0, 0.0]))


def _brute_force_topk(A_int: np.ndarray, k: int):
    """Lexicographically smallest index tuple among those maximising the kept
    energy sum_{j in I} ||A[:, j]||^2, in exact integer arithmetic."""
    energy = [int(sum(int(v) * int(v) for v in A_int[:, j])) for j in range(A_int.shape[1])]
    best, best_set = None, None
    for subset in itertools.combinations(range(A_int.shape[1]), k):
        e = sum(energy[j] for j in subset)
        if best is None or e > best:  # combinations() yields lexicographic order
            best, best_set = e, subset
    return np.array(best_set, dtype=np.int32)


def check_topk_brute_force(impl, cases=60, seed=11):
    """Theorem 1 and Eq. (18) [Appendix E.1, E.4]: TopK by column norm keeps the
    most energy of any index set of the same size; among equal-energy sets the
    tie reading keeps lower indices (= the lexicographically smallest set).
    Small integer entries make exact ties frequent."""
    rng = _rng(seed)
    for _ in range(cases):
        n = int(rng.integers(1, 5))
        d = int(rng.integers(1, 11))
        A = rng.integers(-3, 4, size=(n, d)).astype(np.float64)
        for k in range(1, d + 1):
            want = _brute_force_topk(A.astype(np.int64), k)
            got = impl.topk_indices(impl.column_scores_sq(A), k)
            assert np.array_equal(np.asarray(got), want), (A, k, got, want)


def check_dense_special_case(impl, seed=12):
    """rho = 1 keeps every index [§3.2: |I| = ceil(1*d) = d], so the product is
    the dense A B, computed here independently with numpy."""
    rng = _rng(seed)
    for n, d, m in [(1, 1, 1), (3, 5, 2), (17, 33, 9), (64, 256, 40)]:
        A = rng.standard_normal((n, d))
        B = rng.standard_normal((d, m))
        k = impl.retained_count(1.0, d)
        assert k == d
        I = impl.topk_indices(impl.column_scores_sq(A), k)
        assert np.array_equal(np.asarray(I), np.arange(d))
        Y = impl.reduced_product(A, B, I)
        ref = A @ B
        err = np.linalg.norm(Y - ref) / max(np.linalg.norm(ref), 1e-300)
        assert err <= 1e-12, err


def _error_and_bounds(A, B, I):
    d = A.shape[1]
    keep = np.zeros(d, dtype=bool)
    keep[np.asarray(I)] = True
    drop = ~keep
    a_norm = np.linalg.norm(A, axis=0)
    b_norm = np.linalg.norm(B, axis=1)
    prop1 = float(np.sum(a_norm[drop] * b_norm[drop]))                          # Eq. (12)
    cor1 = float(np.linalg.norm(A[:, drop]) * np.linalg.norm(B[drop, :]))        # Eq. (14)
    fa, fb = np.linalg.norm(A), np.linalg.norm(B)
    eps_a = np.linalg.norm(A[:, drop]) ** 2 / fa ** 2                           # Eq. (16)
    eps_b = np.linalg.norm(B[drop, :]) ** 2 / fb ** 2
    rel = float(np.sqrt(eps_a * eps_b))                                         # Eq. (17)
    return prop1, cor1, rel, fa * fb


def check_error_bounds(impl, seed=13):
    """Proposition 1 (Eq. 12), Corollary 1 (Eq. 14) and the relative bound
    (Eq. 17) [Appendix E.2-E.4] hold for the oracle's output at every rho.
    The dense product comes from numpy, not from the oracle."""
    rng = _rng(seed)
    for n, d, m in [(4, 16, 8), (32, 64, 24), (64, 256, 64)]:
        A = rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))
        B = rng.standard_normal((d, m)) * 0.02
        full = A @ B
        for rho in (0.1, 0.25, 0.5, 0.8, 1.0):
            k = impl.retained_count(rho, d)
            I = impl.topk_indices(impl.column_scores_sq(A), k)
            Y = impl.reduced_product(A, B, I)
            err = float(np.linalg.norm(full - Y))
            prop1, cor1, rel, scale = _error_and_bounds(A, B, I)
            slack = 1e-12 * scale + 1e-300
            assert err <= prop1 * (1 + 1e-12) + slack, (rho, err, prop1)
            assert prop1 <= cor1 * (1 + 1e-12) + slack, (rho, prop1, cor1)
            assert err / scale <= rel * (1 + 1e-12) + 1e-14, (rho, err / scale, rel)


def check_rank_one_equality(impl, seed=14):
    """Equality case of Eq. (12): when every term A[:,j] B[j,:] is a positive
    multiple of the same rank-one matrix u v^T, the triangle inequality in the
    proof of Proposition 1 is tight, so the error equals the bound exactly."""
    rng = _rng(seed)
    n, d, m = 6, 20, 5
    u = rng.standard_normal(n)
    v = rng.standard_normal(m)
    c = rng.uniform(0.1, 3.0, d)
    b = rng.uniform(0.1, 3.0, d)
    A = np.outer(u, c)
    B = np.outer(b, v)
    for rho in (0.2, 0.5, 0.75):
        k = impl.retained_count(rho, d)
        I = impl.topk_indices(impl.column_scores_sq(A), k)
        Y = impl.reduced_product(A, B, I)
        err = np.linalg.norm(A @ B - Y)
        drop = np.setdiff1d(np.arange(d), I)
        want = np.sum(c[drop] * b[drop]) * np.linalg.norm(u) * np.linalg.norm(v)
        assert abs(err - want) <= 1e-12 * want, (err, want)


def check_minimax_worst_case(impl, seed=15):
    """Theorem 1's inner problem and Remark 1 [Appendix E.1, Eq. (8)-(9)]: for
    the oracle's I, the adversarial row energies b_j = alpha_j / ||A[:,Ibar]||_F
    on the dropped set give sum alpha_j b_j = ||A[:,Ibar]||_F, and no other set
    of the same size leaves less energy behind (Eq. 18, by enumeration)."""
    rng = _rng(seed)
    n, d = 5, 9
    A = rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))
    alpha = np.linalg.norm(A, axis=0)
    for k in range(1, d):
        I = np.asarray(impl.topk_indices(impl.column_scores_sq(A), k))
        drop = np.setdiff1d(np.arange(d), I)
        resid = np.linalg.norm(A[:, drop])
        bj = alpha[drop] / resid
        assert abs(np.sum(bj ** 2) - 1.0) < 1e-12
        assert abs(np.sum(alpha[drop] * bj) - resid) <= 1e-12 * resid
        for other in itertools.combinations(range(d), k):
            odrop = np.setdiff1d(np.arange(d), other)
            assert np.linalg.norm(A[:, odrop]) >= resid * (1 - 1e-12)


def check_invariants(impl, seed=16):
    """Determinism [§3.2], nesting of the kept sets as rho grows, invariance of
    I under scaling A by a power of two, and equivariance of (I, Y) under a
    joint permutation of A's columns and B's rows."""
    rng = _rng(seed)
    n, d, m = 24, 96, 12
    A = rng.standard_normal((n, d)) * np.exp(rng.standard_normal(d))
    B = rng.standard_normal((d, m))
    s2 = impl.column_scores_sq(A)
    prev = set()
    for rho in (0.1, 0.3, 0.5, 0.7, 0.9, 1.0):
        k = impl.retained_count(rho, d)
        I1 = np.asarray(impl.topk_indices(s2, k))
        I2 = np.asarray(impl.topk_indices(impl.column_scores_sq(A.copy()), k))
        assert np.array_equal(I1, I2)
        assert np.all(np.diff(I1) > 0), "I must be strictly ascending"
        assert prev <= set(I1.tolist())
        prev = set(I1.tolist())
        I3 = np.asarray(impl.topk_indices(impl.column_scores_sq(A * 2.0 ** -7), k))
        assert np.array_equal(I1, I3)
        perm = rng.permutation(d)
        Ap, Bp = A[:, perm], B[perm, :]
        Ip = np.asarray(impl.topk_indices(impl.column_scores_sq(Ap), k))
        assert np.array_equal(np.sort(perm[Ip]), I1)
        Y = impl.reduced_product(A, B, I1)
        Yp = impl.reduced_product(Ap, Bp, Ip)
        assert np.allclose(Y, Yp, rtol=1e-12, atol=1e-12 * np.abs(Y).max())


def check_one_row_ties(impl):
    """n = 1: s_j = |a_j|, so +x and -x tie and the lower index is kept."""
    a = np.array([[0.5, -2.0, 2.0, 1.0, -0.5, 3.0, -3.0, 1.0]])
    s2 = impl.column_scores_sq(a)
    want = {1: [5], 2: [5, 6], 3: [1, 5, 6], 4: [1, 2, 5, 6], 5: [1, 2, 3, 5, 6],
            6: [1, 2, 3, 5, 6, 7], 7: [0, 1, 2, 3, 5, 6, 7]}
    for k, w in want.items():
        assert np.asarray(impl.topk_indices(s2, k)).tolist() == w, k


def check_grouped_heads(impl, seed=17):
    """§3.3 Attention with grouped-query heads: query head h reads K / V head
    h // (H / H_kv).  At rho = 1 the per-head forms equal numpy's products with
    that mapping (QK: alpha Q_h K_g^T; PV: P_h V_g)."""
    rng = _rng(seed)
    H, Hkv, n, t, dh = 8, 2, 3, 20, 16
    Q = rng.standard_normal((H, n, dh))
    K = rng.standard_normal((Hkv, t, dh))
    P = rng.random((H, n, t))
    V = rng.standard_normal((Hkv, t, dh))
    S, _ = impl.rmm_qk(Q, K, 1.0, 0.5, causal=False)
    O, _ = impl.rmm_pv(P, V, 1.0)
    for h in range(H):
        g = h // (H // Hkv)
        np.testing.assert_allclose(S[h], 0.5 * Q[h] @ K[g].T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(O[h], P[h] @ V[g], rtol=1e-12, atol=1e-12)


def _best_subset(norms_sq, k):
    """The k-subset with the largest sum of squared norms, by enumeration."""
    best = max(itertools.combinations(range(len(norms_sq)), k), key=lambda c: sum(norms_sq[j] for j in c))
    return np.array(best)


def check_grouped_heads_reduced(impl, seed=20):
    """§3.3 "Attention" below rho = 1, per head with grouped-query K/V: the QK
    form keeps the features of Q_h (not of K_g) whose column norms are largest
    (enumeration over every feature subset), the PV form keeps the tokens of
    P_h whose column norms are largest (enumeration over every token subset),
    and each result's error against the dense product obeys Proposition 1
    (Eq. 12): ||X Y - X_I Y_I||_F <= sum over dropped j of ||X_:j|| ||Y_j:||."""
    rng = _rng(seed)
    H, Hkv, n, t, dh = 4, 2, 5, 8, 6
    # Q's feature norms are ordered against K's, so the two choices differ
    Q = rng.standard_normal((H, n, dh)) * np.geomspace(4.0, 0.25, dh)
    K = rng.standard_normal((Hkv, t, dh)) * np.geomspace(0.25, 4.0, dh)
    P = rng.random((H, n, t)) * np.geomspace(3.0, 0.3, t)
    V = rng.standard_normal((Hkv, t, dh)) * np.geomspace(0.3, 3.0, t)[:, None]
    alpha = 0.5
    S, I = impl.rmm_qk(Q, K, 0.5, alpha, causal=False)
    O, T = impl.rmm_pv(P, V, 0.5)
    kd, kt = impl.retained_count(0.5, dh), impl.retained_count(0.5, t)
    for h in range(H):
        g = h // (H // Hkv)
        qn = (Q[h] ** 2).sum(axis=0)
        assert np.array_equal(np.sort(I[h]), _best_subset(qn, kd)), h
        dropped = np.setdiff1d(np.arange(dh), I[h])
        bound = alpha * sum(np.sqrt(qn[j]) * np.linalg.norm(K[g][:, j]) for j in dropped)
        assert np.linalg.norm(alpha * Q[h] @ K[g].T - S[h]) <= bound * (1 + 1e-12) + 1e-15, h
        pn = (P[h] ** 2).sum(axis=0)
        assert np.array_equal(np.sort(T[h]), _best_subset(pn, kt)), h
        dropped = np.setdiff1d(np.arange(t), T[h])
        bound = sum(np.sqrt(pn[j]) * np.linalg.norm(V[g][j]) for j in dropped)
        assert np.linalg.norm(P[h] @ V[g] - O[h]) <= bound * (1 + 1e-12) + 1e-15, h


def check_row_subsets(impl, seed=21):
    """The sampled-row forms used at full size give exactly the rows of the full
    result (whose values the other checks pin): the reduced product's rows, and
    the causal scores' rows with each row's own position deciding its mask."""
    rng = _rng(seed)
    A, B = rng.standard_normal((9, 12)), rng.standard_normal((12, 7))
    I = np.array([1, 2, 5, 7, 8, 11], dtype=np.int32)
    rows = [8, 0, 4, 3]
    assert np.array_equal(impl.reduced_product(A, B, I, rows=rows), impl.reduced_product(A, B, I)[rows])
    Q, K = rng.standard_normal((9, 8)), rng.standard_normal((11, 8))
    Iq = np.array([0, 3, 4, 6], dtype=np.int32)
    full = impl.reduced_scores(Q, K, Iq, 0.25, True)
    assert np.array_equal(impl.reduced_scores(Q, K, Iq, 0.25, True, rows=[5, 2, 8]), full[[5, 2, 8]])
    assert np.isneginf(full[2, 3]) and np.isfinite(full[2, 2]), "key t > row i is masked"


def check_softmax(impl, seed=18):
    """P = softmax(S + M) over the key axis of each row [§3.3 "Attention"]:
    a constant row gives 1/t; two keys give the logistic function of their
    difference; -inf (masked) entries weigh exactly 0 and a causal first row is
    one-hot; every row sums to 1 while columns of a wide S do not; adding a
    constant to a row changes nothing; logits of 1000 stay finite."""
    sm = impl.softmax_rows
    t = 7
    got = sm(np.full((3, t), 2.5))
    assert np.array_equal(got, np.full((3, t), 1.0 / t)), got
    for x in (-3.0, 0.0, 0.7, 5.0):
        got = sm(np.array([[0.0, x]]))
        lo = 1.0 / (1.0 + np.exp(x))
        assert abs(got[0, 0] - lo) <= 1e-15 and abs(got[0, 1] - (1.0 - lo)) <= 1e-15, (x, got)
    rng = _rng(seed)
    n, w = 6, 10
    S = rng.standard_normal((n, w)) * 3.0
    causal = np.triu(np.ones((n, w), dtype=bool), 1)
    Sm = np.where(causal, -np.inf, S)
    P = sm(Sm)
    assert np.all(P[causal] == 0.0)
    assert P[0, 0] == 1.0 and np.all(P[~causal] > 0.0)
    assert np.allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    Pw = sm(S)
    assert np.allclose(Pw.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert not np.allclose(Pw.sum(axis=0), 1.0, atol=1e-3)
    shift = rng.standard_normal((n, 1)) * 50.0
    assert np.allclose(sm(S + shift), Pw, rtol=1e-12, atol=1e-15)
    big = sm(np.array([[1000.0, 999.0, 0.0]]))
    assert np.all(np.isfinite(big))
    assert abs(big[0, 0] - 1.0 / (1.0 + np.exp(-1.0) + np.exp(-1000.0))) <= 1e-15


def check_e4m3_decoding(impl):
    """Exact E4M3 values (the low-bit operand format) against codes worked by
    hand from the OCP 8-bit floating point layout, and every non-NaN code
    against torch's float8_e4m3fn conversion (a library routine)."""
    import torch
    with open(os.path.join(GOLDEN, "e4m3_codes.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            code, want = line.split()
            got = impl.decode_e4m3(np.array([int(code, 16)], dtype=np.uint8))[0]
            assert got == float(want) and np.signbit(got) == np.signbit(float(want)), (code, got, want)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(impl.decode_e4m3(codes), lib)


def check_attention(impl, seed=19):
    """RMM attention [§3.3 "Attention"]: with every feature and token kept it is
    softmax(alpha Q K^T + M) V per head with grouped-query K/V (scipy's softmax,
    a library routine); with features and tokens dropped, I_h holds Q_h's
    largest column norms, P_h is scipy's row softmax of the scores over I_h
    alone, the error of O_h obeys Proposition 1 (Eq. 12) for the product
    P_h V_g, and T_h is the TopK of P_h's column norms."""
    import scipy.special
    rng = _rng(seed)
    H, Hkv, n, dh, dv = 4, 2, 12, 8, 6
    Q = rng.standard_normal((H, n, dh)) * np.exp(rng.standard_normal((H, 1, dh)))
    K = rng.standard_normal((Hkv, n, dh))
    V = rng.standard_normal((Hkv, n, dv))
    alpha = 1.0 / np.sqrt(dh)
    mask = np.triu(np.ones((n, n), dtype=bool), 1)
    O, I, T, P = impl.rmm_attention(Q, K, V, 1.0, 1.0, alpha, True)
    for h in range(H):
        g = h // (H // Hkv)
        logits = np.where(mask, -np.inf, alpha * Q[h] @ K[g].T)
        ref = scipy.special.softmax(logits, axis=1) @ V[g]
        assert np.allclose(O[h], ref, rtol=1e-12, atol=1e-14), h
    O, I, T, P = impl.rmm_attention(Q, K, V, 0.5, 0.5, alpha, True)
    kt = impl.retained_count(0.5, n)
    kd = impl.retained_count(0.5, dh)
    for h in range(H):
        g = h // (H // Hkv)
        # the features are Q_h's top column norms (brute force over all subsets
        # of size kd would pick the same set: the norms here are distinct), and
        # P_h is the row softmax of the scores over those features only
        q2 = (Q[h] ** 2).sum(axis=0)
        assert np.array_equal(np.sort(I[h]), np.sort(np.argsort(-q2, kind="stable")[:kd])), h
        feats = np.sort(I[h])
        logits = np.where(mask, -np.inf, alpha * Q[h][:, feats] @ K[g][:, feats].T)
        assert np.allclose(P[h], scipy.special.softmax(logits, axis=1), rtol=1e-12, atol=1e-15), h
        s2 = (P[h] ** 2).sum(axis=0)
        assert np.array_equal(T[h], impl.topk_indices(s2, kt))
        full = P[h] @ V[g]
        dropped = np.setdiff1d(np.arange(n), T[h])
        bound = sum(np.linalg.norm(P[h][:, j]) * np.linalg.norm(V[g][j]) for j in dropped)
        assert np.linalg.norm(full - O[h]) <= bound * (1 + 1e-12) + 1e-15


ALL_CHECKS = [
    check_retained_counts,
    check_scores_closed_forms,
    check_topk_brute_force,
    check_dense_special_case,
    check_error_bounds,
    check_rank_one_equality,
    check_minimax_worst_case,
    check_invariants,
    check_one_row_ties,
    check_grouped_heads,
    check_grouped_heads_reduced,
    check_row_subsets,
    check_softmax,
    check_e4m3_decoding,
    check_attention,
]
