"""GPU parity of the fused RMM attention (rmm_attention: features of Q, the
row softmax of the reduced scores, tokens by P's column norms, the output over
the kept tokens, without writing S or P) against the oracle's three steps.

I is bit-exact (Q's feature scores are opened at the boundary as in the QK
tests); T is bit-exact on seeds whose token scores the oracle finds separated
at the boundary by more than fp32 error (the kernel sums fp32 weights).  O
meets the per-element bound of every form, 1e-2 (|P_T| |V_T|), on the oracle's
P and V.  Its Frobenius bound differs from the forms whose operands arrive as
bf16: this op computes P and rounds it to bf16 (2^-9 relative per weight)
before its product and rounds O again, so |O - O_ref| <= 2^-8 (|P_T| |V_T|)
per element up to fp32 terms, and the relative Frobenius error is bounded by
2^-8 ||(|P_T| |V_T|)|| / ||O_ref|| (at least the common 2e-3)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap
from tests.parity import assert_indices_equal, assert_product_close

pytestmark = pytest.mark.gpu

TOKEN_GAP = 3e-4  # fp32 sums of ~n squared weights stay within n * 2^-24 of fp64


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


def _inputs(H, Hkv, n, rho_d, rho_t, causal, seed0):
    dh = 128
    kd = oracle.retained_count(rho_d, dh)
    alpha = 1.0 / math.sqrt(dh)
    for seed in range(seed0, seed0 + 12):
        (Q, K), _ = gap.enforce_boundary_gaps(
            lambda g: W.attn_qk(seed, n=n, heads=H, kv_heads=Hkv, head_dim=dh, col_gain=g),
            lambda x: gap.scores_per_head(x[0]), [kd])
        V = (torch.randn((Hkv, n, 128), generator=W.gen(seed + 1000)) ).to(torch.bfloat16)
        O, I, T, P = oracle.rmm_attention(Q, K, V, rho_d, rho_t, alpha, causal)
        kt = oracle.retained_count(rho_t, n)
        if min(gap.boundary_gap((P[h] ** 2).sum(axis=0), kt) for h in range(H)) >= TOKEN_GAP:
            return Q, K, V, O, I, T, P, alpha
    pytest.fail("no seed with the token scores separated at the boundary")


@pytest.mark.parametrize("H,Hkv,n,rho_d,rho_t,causal", [
    (4, 2, 256, 0.8, 0.8, True),      # two 128-row blocks
    (4, 2, 264, 0.5, 0.6, True),      # a ragged third block
    (2, 1, 384, 0.8, 0.5, False),     # every key block for every query block
    (8, 2, 1024, 0.8, 0.5, True),     # eight blocks; late key blocks lose every token
    (2, 2, 256, 1.0, 1.0, True),      # every feature and token kept: softmax attention
])
def test_fused_attention(rmm, H, Hkv, n, rho_d, rho_t, causal):
    Q, K, V, O_ref, I_ref, T_ref, P_ref, alpha = _inputs(H, Hkv, n, rho_d, rho_t, causal, 91)
    dev = torch.device("cuda")
    O, I, T = rmm.attention(Q.to(dev), K.to(dev), V.to(dev), rho_d, rho_t, causal=causal, alpha=alpha,
                            return_sets=True)
    O2, I2, T2 = rmm.attention(Q.to(dev), K.to(dev), V.to(dev), rho_d, rho_t, causal=causal, alpha=alpha,
                               return_sets=True)
    torch.cuda.synchronize()
    assert rmm.attention_status(Q, K, V, rho_d, rho_t) == 0
    assert_indices_equal(I, I_ref)
    assert_indices_equal(T, T_ref)
    assert torch.equal(O, O2) and torch.equal(T, T2), "the same bits on every call"
    V64 = oracle.as_f64(V)
    for h in range(H):
        g = oracle.kv_head_of(h, H, Hkv)
        absP, absV = np.abs(P_ref[h][:, T_ref[h]]), np.abs(V64[g][T_ref[h]])
        fro = max(2e-3, 2.0 ** -8 * np.linalg.norm(absP @ absV) / max(np.linalg.norm(O_ref[h]), 1e-300))
        assert_product_close(O[h], O_ref[h], absP, absV, rel_fro=fro)


def test_fused_attention_matches_the_unfused_ops(rmm):
    """The same I as the library's separate ops (QK with feature selection,
    the softmax with token scores, PV taking those scores), and token sets
    that differ from theirs only where the roundings of the separate path can
    swap them.  That path stores S in bf16 (each score within 2^-9 |S| of its
    value), so each of its weights lies within a factor e^(+-2c) of the exact
    one, c = 2^-9 max |S|, and its token scores (of bf16 weights, another
    2^-8) within r = e^(4c + 2^-7) of the exact ones; a token in one top-k and
    not the other then has an exact score within a factor r^2 of the k-th
    largest.  On heads whose sets agree the outputs agree within the two
    roundings of P and the rounding of S."""
    H, Hkv, n, rho_d, rho_t = 4, 2, 512, 0.8, 0.6
    Q, K, V, O_ref, I_ref, T_ref, P_ref, alpha = _inputs(H, Hkv, n, rho_d, rho_t, True, 120)
    dev = torch.device("cuda")
    Qg, Kg, Vg = Q.to(dev), K.to(dev), V.to(dev)
    O, I, T = rmm.attention(Qg, Kg, Vg, rho_d, rho_t, causal=True, alpha=alpha, return_sets=True)
    S, Iq = rmm.qk(Qg, Kg, rho=rho_d, alpha=alpha, causal=True, return_indices=True)
    P, s2 = rmm.softmax_scores(S, causal=True)
    O3, T3 = rmm.pv(P, Vg, rho=rho_t, return_indices=True, causal=True, scores=s2)
    torch.cuda.synchronize()
    assert torch.equal(I, Iq)
    assert_indices_equal(T, T_ref)
    S_ref, _ = oracle.rmm_qk(Q, K, rho_d, alpha, causal=True)
    kt = oracle.retained_count(rho_t, n)
    Tg, T3g = T.cpu().numpy(), T3.cpu().numpy()
    for h in range(H):
        c = 2.0 ** -9 * np.abs(S_ref[h][np.isfinite(S_ref[h])]).max()
        r2 = math.exp(2 * (4 * c + 2.0 ** -7)) * (1 + 1e-5)
        a2 = (P_ref[h] ** 2).sum(axis=0)
        kth = np.sort(a2)[::-1][kt - 1]
        for t in np.setxor1d(Tg[h], T3g[h]):
            assert kth / r2 <= a2[t] <= kth * r2, (h, int(t), a2[t] / kth, r2)
        if np.array_equal(Tg[h], T3g[h]):
            g = oracle.kv_head_of(h, H, Hkv)
            absPV = np.abs(P_ref[h][:, T_ref[h]]) @ np.abs(oracle.as_f64(V)[g][T_ref[h]])
            bound = (2.0 ** -7 + 4 * c) * np.linalg.norm(absPV) / np.linalg.norm(O_ref[h])
            rel = ((O[h].double() - O3[h].double()).norm() / O3[h].double().norm()).item()
            assert rel <= max(bound, 4e-3), (h, rel, bound)
