"""Planted mistakes in the oracle must be caught by its pins (no GPU).

Each mutant is the oracle with one plausible error planted in it, on the CPU.
If the pin suite in oracle_checks.py lets any of them through, the pins are
too weak to trust the oracle they vouch for.
"""
import math
import types

import numpy as np
import pytest

import oracle
from tests import oracle_checks as oc


def _mutant(**overrides):
    m = types.SimpleNamespace(
        retained_count=oracle.retained_count,
        column_scores_sq=oracle.column_scores_sq,
        topk_indices=oracle.topk_indices,
        reduced_product=oracle.reduced_product,
        reduced_scores=oracle.reduced_scores,
        rmm_qk=oracle.rmm_qk,
        rmm_pv=oracle.rmm_pv,
        softmax_rows=oracle.softmax_rows,
        decode_e4m3=oracle.decode_e4m3,
        rmm_attention=oracle.rmm_attention,
    )
    for k, v in overrides.items():
        setattr(m, k, v)
    return m


def _topk_ties_high(s2, k):
    order = sorted(range(len(s2)), key=lambda j: (-s2[j], -j))
    return np.array(sorted(order[:k]), dtype=np.int32)


def _topk_smallest(s2, k):
    order = sorted(range(len(s2)), key=lambda j: (s2[j], j))
    return np.array(sorted(order[:k]), dtype=np.int32)


def _topk_unsorted(s2, k):
    order = sorted(range(len(s2)), key=lambda j: (-s2[j], j))
    return np.array(order[:k], dtype=np.int32)


def _scores_l1(A):
    return np.abs(oracle.as_f64(A)).sum(axis=0)


def _scores_rows(A):
    A = oracle.as_f64(A)
    s = (A ** 2).sum(axis=1)
    return np.resize(s, A.shape[1])


def _product_drops_last(A, B, I, rows=None):
    return oracle.reduced_product(A, B, np.asarray(I)[:-1] if len(I) > 1 else I, rows)


def _product_shifted_rows(A, B, I, rows=None):
    A = oracle.as_f64(A)
    B = oracle.as_f64(B)
    d = B.shape[0]
    Bs = np.ascontiguousarray(np.roll(B, -1, axis=0)) if d > 1 else B * 2
    return oracle.reduced_product(A, Bs, I, rows)


def _product_wrong_sign(A, B, I, rows=None):
    Y = oracle.reduced_product(A, B, I, rows)
    I = np.asarray(I)
    if len(I):
        A = oracle.as_f64(A)
        B = oracle.as_f64(B)
        j = int(I[0])
        Y = Y - 2.0 * np.outer(A[:, j] if rows is None else A[rows, j], B[j])
    return Y


def _qk_interleaved(Q, K, rho, alpha, causal=True, heads=None, rows=None):
    """Grouped-query heads mapped h -> h % H_kv instead of h // (H / H_kv)."""
    Q, K = oracle.as_f64(Q), oracle.as_f64(K)
    H, Hkv = Q.shape[0], K.shape[0]
    k = oracle.retained_count(rho, Q.shape[2])
    I = np.stack([oracle.select(Q[h], k=k)[0] for h in range(H)])
    S = np.stack([oracle.reduced_scores(Q[h], K[h % Hkv], I[h], alpha, causal) for h in range(H)])
    return S, I


def _pv_interleaved(P, V, rho, heads=None, rows=None):
    P, V = oracle.as_f64(P), oracle.as_f64(V)
    H, Hkv = P.shape[0], V.shape[0]
    k = oracle.retained_count(rho, P.shape[2])
    T = np.stack([oracle.select(P[h], k=k)[0] for h in range(H)])
    O = np.stack([oracle.reduced_product(P[h], V[h % Hkv], T[h]) for h in range(H)])
    return O, T


def _qk_features_from_keys(Q, K, rho, alpha, causal=True, heads=None, rows=None):
    """Each query head's features chosen by its K head's column norms."""
    Q, K = oracle.as_f64(Q), oracle.as_f64(K)
    H, Hkv = Q.shape[0], K.shape[0]
    k = oracle.retained_count(rho, Q.shape[2])
    I = np.stack([oracle.select(K[h // (H // Hkv)], k=k)[0] for h in range(H)])
    S = np.stack([oracle.reduced_scores(Q[h], K[h // (H // Hkv)], I[h], alpha, causal) for h in range(H)])
    return S, I


def _pv_tokens_by_value_norms(P, V, rho, heads=None, rows=None):
    """Each head's tokens chosen by the row norms of V instead of P's column norms."""
    P, V = oracle.as_f64(P), oracle.as_f64(V)
    H, Hkv = P.shape[0], V.shape[0]
    k = oracle.retained_count(rho, P.shape[2])
    T = np.stack([oracle.topk_indices((V[h // (H // Hkv)] ** 2).sum(axis=1), k) for h in range(H)])
    O = np.stack([oracle.reduced_product(P[h], V[h // (H // Hkv)], T[h]) for h in range(H)])
    return O, T


def _scores_rows_masked_by_position_in_sample(Q, K, I, alpha, causal, rows=None):
    """Sampled rows masked by their position in the sample, not their own row."""
    if rows is None:
        return oracle.reduced_scores(Q, K, I, alpha, causal)
    Q, K = oracle.as_f64(Q), oracle.as_f64(K)
    I = np.asarray(I)
    S = alpha * Q[np.asarray(rows)][:, I] @ K[:, I].T
    if causal:
        S = np.where(np.arange(K.shape[0])[None, :] > np.arange(len(rows))[:, None], -np.inf, S)
    return S


def _product_rows_from_the_top(A, B, I, rows=None):
    """Sampled rows taken as the first len(rows) rows."""
    if rows is None:
        return oracle.reduced_product(A, B, I)
    return oracle.reduced_product(A, B, I)[: len(rows)]


def _softmax_no_max_shift(S):
    with np.errstate(over="ignore", invalid="ignore"):
        E = np.exp(oracle.as_f64(S))
        return E / E.sum(axis=1, keepdims=True)


def _softmax_over_columns(S):
    S = oracle.as_f64(S)
    E = np.exp(S - S.max(axis=0, keepdims=True))
    return E / E.sum(axis=0, keepdims=True)


def _softmax_mask_as_zero_logit(S):
    S = oracle.as_f64(S)
    return oracle.softmax_rows(np.where(np.isneginf(S), 0.0, S))


def _softmax_linear(S):
    S = oracle.as_f64(S)
    E = np.where(np.isneginf(S), 0.0, S - S.min(axis=1, keepdims=True, initial=np.inf, where=~np.isneginf(S)) + 1.0)
    return E / E.sum(axis=1, keepdims=True)


def _e4m3_bias_8(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return oracle.decode_e4m3(c) / 2.0


def _e4m3_no_subnormals(codes):
    c = np.asarray(codes, dtype=np.uint8)
    v = oracle.decode_e4m3(c)
    return np.where((c & 0x78) == 0, 0.0 * v, v)


def _attention_tokens_from_scores(Q, K, V, rho_d, rho_t, alpha, causal=True):
    """Token set chosen from the column norms of the scores S instead of P."""
    Q, K, V = oracle.as_f64(Q), oracle.as_f64(K), oracle.as_f64(V)
    H, Hkv = Q.shape[0], K.shape[0]
    S, I = oracle.rmm_qk(Q, K, rho=rho_d, alpha=alpha, causal=causal)
    P = oracle.softmax_rows(S)
    kt = oracle.retained_count(rho_t, P.shape[2])
    Sf = np.where(np.isneginf(S), 0.0, S)
    T = np.stack([oracle.topk_indices((Sf[h] ** 2).sum(axis=0), kt) for h in range(H)])
    O = np.stack([oracle.reduced_product(P[h], V[h // (H // Hkv)], T[h]) for h in range(H)])
    return O, I, T, P


def _attention_unscaled(Q, K, V, rho_d, rho_t, alpha, causal=True):
    return oracle.rmm_attention(Q, K, V, rho_d, rho_t, 1.0, causal)


def _attention_features_from_keys(Q, K, V, rho_d, rho_t, alpha, causal=True):
    """Feature set chosen from the column norms of the head's K instead of Q."""
    Q, K, V = oracle.as_f64(Q), oracle.as_f64(K), oracle.as_f64(V)
    H, Hkv, n = Q.shape[0], K.shape[0], Q.shape[1]
    kd = oracle.retained_count(rho_d, Q.shape[2])
    I = np.stack([oracle.topk_indices(oracle.column_scores_sq(K[h // (H // Hkv)]), kd) for h in range(H)])
    mask = np.triu(np.ones((n, K.shape[1]), dtype=bool), 1) if causal else np.zeros((n, K.shape[1]), dtype=bool)
    S = np.stack([np.where(mask, -np.inf, alpha * Q[h][:, I[h]] @ K[h // (H // Hkv)][:, I[h]].T) for h in range(H)])
    P = oracle.softmax_rows(S)
    kt = oracle.retained_count(rho_t, P.shape[2])
    T = np.stack([oracle.select(P[h], k=kt)[0] for h in range(H)])
    O = np.stack([oracle.reduced_product(P[h], V[h // (H // Hkv)], T[h]) for h in range(H)])
    return O, I, T, P


def _attention_scores_over_all_features(Q, K, V, rho_d, rho_t, alpha, causal=True):
    """I reported, but the scores taken over every feature of Q and K."""
    _, I, _, _ = oracle.rmm_attention(Q, K, V, rho_d, rho_t, alpha, causal)
    O, _, T, P = oracle.rmm_attention(Q, K, V, 1.0, rho_t, alpha, causal)
    return O, I, T, P


def _count_floor(rho, d):
    return max(1, int(math.floor(rho * d)))


def _count_no_snap(rho, d):
    return min(d, max(1, int(math.ceil(rho * d))))


MUTANTS = {
    "ties_to_higher_index": _mutant(topk_indices=_topk_ties_high),
    "keeps_smallest": _mutant(topk_indices=_topk_smallest),
    "index_set_not_sorted": _mutant(topk_indices=_topk_unsorted),
    "l1_scores": _mutant(column_scores_sq=_scores_l1),
    "row_norms_not_column_norms": _mutant(column_scores_sq=_scores_rows),
    "product_drops_an_index": _mutant(reduced_product=_product_drops_last),
    "product_off_by_one_row": _mutant(reduced_product=_product_shifted_rows),
    "product_sign_error": _mutant(reduced_product=_product_wrong_sign),
    "k_floor_not_ceil": _mutant(retained_count=_count_floor),
    "k_no_rounding_snap": _mutant(retained_count=_count_no_snap),
    "gqa_heads_interleaved": _mutant(rmm_qk=_qk_interleaved, rmm_pv=_pv_interleaved),
    "qk_features_from_keys": _mutant(rmm_qk=_qk_features_from_keys),
    "sampled_score_rows_masked_by_sample_position": _mutant(reduced_scores=_scores_rows_masked_by_position_in_sample),
    "sampled_product_rows_from_the_top": _mutant(reduced_product=_product_rows_from_the_top),
    "pv_tokens_by_value_norms": _mutant(rmm_pv=_pv_tokens_by_value_norms),
    "softmax_without_max_shift": _mutant(softmax_rows=_softmax_no_max_shift),
    "softmax_over_the_query_axis": _mutant(softmax_rows=_softmax_over_columns),
    "softmax_mask_as_zero_logit": _mutant(softmax_rows=_softmax_mask_as_zero_logit),
    "softmax_without_exp": _mutant(softmax_rows=_softmax_linear),
    "e4m3_exponent_bias_8": _mutant(decode_e4m3=_e4m3_bias_8),
    "e4m3_subnormals_flushed": _mutant(decode_e4m3=_e4m3_no_subnormals),
    "attention_tokens_from_scores": _mutant(rmm_attention=_attention_tokens_from_scores),
    "attention_without_scale": _mutant(rmm_attention=_attention_unscaled),
    "attention_features_from_keys": _mutant(rmm_attention=_attention_features_from_keys),
    "attention_scores_over_all_features": _mutant(rmm_attention=_attention_scores_over_all_features),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    impl = MUTANTS[name]
    caught = []
    for check in oc.ALL_CHECKS:
        try:
            check(impl)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake '{name}'"
