"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times: the index sets are compared in full (every head), the
products on two seeded rows of every 128-row tile (all rows when n <= 16)
against the oracle computed row by row."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap
from tests.parity import assert_indices_equal, assert_product_close, np64, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


def _linear_full(rmm, gen, n, rhos, seed, **kw):
    d = gen(seed, n=1, m=8, **kw)[0].shape[1] if "shape" not in kw else W.LLAMA70B_LINEAR[kw["shape"]][0]
    ks = [oracle.retained_count(r, d) for r in rhos]
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: gen(seed, n=n, col_gain=g, **kw),
                                          lambda x: gap.scores_2d(x[0]), ks)
    Ag, Bg = A.cuda(), B.cuda()
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    rows = list(range(n)) if n <= 16 else sample_rows(n, seed)
    for rho in rhos:
        Y, I = rmm.matmul(Ag, Bg, rho=rho, return_indices=True)
        torch.cuda.synchronize()
        rmm.check_workspaces()
        I_ref, _ = oracle.select(A64, rho=rho)
        assert_indices_equal(I, I_ref)
        Y_ref = oracle.reduced_product(A64, B64, I_ref, rows)
        assert_product_close(Y[rows], Y_ref, np.abs(A64[rows][:, I_ref]), np.abs(B64[I_ref]))


@pytest.mark.parametrize("n,rhos", [(1024, [0.7]), (2048, [0.8]), (4096, [0.5, 0.8])])
def test_llama8b_up_gate(rmm, n, rhos):
    _linear_full(rmm, W.mlp_up, n, rhos, seed=101)


@pytest.mark.parametrize("n,rhos", [(2048, [0.5, 0.8]), (4096, [0.7, 0.8])])
def test_llama8b_down(rmm, n, rhos):
    """n = 4096, rho = 0.8 is the benchmark's down-projection point."""
    _linear_full(rmm, W.mlp_down, n, rhos, seed=102)


@pytest.mark.parametrize("shape,n,rhos", [
    ("up", 1, [0.5, 0.8]), ("up", 16, [0.6, 1.0]), ("down", 16, [0.7]), ("qkv", 16, [0.8]),
    ("down", 1, [0.6]), ("qkv", 512, [0.5, 0.7]), ("up", 2048, [0.8]),
    # the longest K loops (k up to 22938) and the largest A packs of the suite
    ("down", 512, [0.5, 0.8]), ("down", 2048, [0.5, 0.8]), ("down", 4096, [0.5, 0.8]),
    ("up", 4096, [0.8]), ("qkv", 4096, [0.8]),
])
def test_llama70b_linear(rmm, shape, n, rhos):
    _linear_full(rmm, W.linear_70b, n, rhos, seed=103, shape=shape)


@pytest.mark.parametrize("n", [1024, 2048, 4096])
def test_attention_qk_full(rmm, n):
    H, Hkv, dh = 32, 8, 128
    rhos = [0.5, 0.8]
    ks = [oracle.retained_count(r, dh) for r in rhos]
    (Q, K), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(104, n=n, col_gain=g), lambda x: gap.scores_per_head(x[0]), ks)
    Qg, Kg = Q.cuda(), K.cuda()
    alpha = 1.0 / math.sqrt(dh)
    Q64, K64 = oracle.as_f64(Q), oracle.as_f64(K)
    rows = sample_rows(n, 7)
    heads = [0, 13, 31]
    for rho in rhos:
        S, I = rmm.qk(Qg, Kg, rho=rho, alpha=alpha, causal=True, return_indices=True)
        torch.cuda.synchronize()
        rmm.check_workspaces()
        S_ref, I_ref = oracle.rmm_qk(Q64, K64, rho=rho, alpha=alpha, causal=True, heads=heads, rows=rows)
        assert_indices_equal(I, I_ref)
        mask = np.arange(n)[None, :] > np.asarray(rows)[:, None]
        for i, h in enumerate(heads):
            g = oracle.kv_head_of(h, H, Hkv)
            assert_product_close(S[h][rows], S_ref[i], np.abs(Q64[h][rows][:, I_ref[h]]),
                                 np.abs(K64[g][:, I_ref[h]]).T, alpha=alpha, mask=mask)
        # every masked entry of every head is -inf; no unmasked entry is
        upper = torch.ones(n, n, dtype=torch.bool, device="cuda").triu_(1)
        assert bool(torch.isneginf(S[:, upper]).all())
        assert not bool(torch.isinf(S[:, ~upper]).any())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [2048, 4096])
def test_attention_pv_full(rmm, n, causal):
    H, Hkv, dv = 32, 8, 128
    rhos = [0.5, 0.8]
    ks = [oracle.retained_count(r, n) for r in rhos]
    dev = torch.device("cuda")
    (P, V), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_pv(105, n=n, col_gain=g, device=dev),
        lambda x: [oracle.column_scores_sq(x[0][h]) for h in range(H)], ks)
    rows = sample_rows(n, 9)
    heads = [0, 17, 31]
    P64 = {h: oracle.as_f64(P[h]) for h in heads}
    V64 = oracle.as_f64(V)
    for rho in rhos:
        O, T = rmm.pv(P, V, rho=rho, return_indices=True, causal=causal)
        torch.cuda.synchronize()
        rmm.check_workspaces()
        k = oracle.retained_count(rho, n)
        T_ref = np.stack([oracle.select(P[h], k=k)[0] for h in range(H)])
        assert_indices_equal(T, T_ref)
        for h in heads:
            g = oracle.kv_head_of(h, H, Hkv)
            O_ref = oracle.reduced_product(P64[h], V64[g], T_ref[h], rows)
            assert_product_close(O[h][rows], O_ref, np.abs(P64[h][rows][:, T_ref[h]]),
                                 np.abs(V64[g][T_ref[h]]))


@pytest.mark.parametrize("rho", [0.5, 0.8])
def test_decode_full(rmm, rho):
    """Decode step at the largest measured point: 16 sequences x 32768 cached
    tokens, Llama-3.1-8B heads (512 query heads, 128 KV heads).  The index
    sets of every head are compared with the oracle's (n = 1: exact squares of
    bf16 values on both sides); scores and outputs of 16 sampled heads in full."""
    from tests.parity import assert_heads_close
    dev = torch.device("cuda")
    q, K, V, P = W.attn_decode(111, t=32768, batch=16, device=dev)
    H, Hkv = q.shape[0], K.shape[0]
    alpha = 1.0 / math.sqrt(128)
    S, I = rmm.qk(q, K, rho=rho, alpha=alpha, causal=False, return_indices=True)
    O, T = rmm.pv(P, V, rho=rho, return_indices=True)
    torch.cuda.synchronize()
    rmm.check_workspaces()
    q64, P64 = oracle.as_f64(q.cpu()), oracle.as_f64(P.cpu())
    kf, kt = oracle.retained_count(rho, 128), oracle.retained_count(rho, 32768)
    I_ref = np.stack([oracle.select(q64[h], k=kf)[0] for h in range(H)])
    T_ref = np.stack([oracle.select(P64[h], k=kt)[0] for h in range(H)])
    assert_indices_equal(I, I_ref)
    assert_indices_equal(T, T_ref)
    heads = sorted(np.random.default_rng(7).choice(H, size=16, replace=False).tolist())
    S_ref, O_ref, aS, bS, aO, bO = [], [], [], [], [], []
    for h in heads:
        g = oracle.kv_head_of(h, H, Hkv)
        K64, V64 = oracle.as_f64(K[g].cpu()), oracle.as_f64(V[g].cpu())
        S_ref.append(oracle.reduced_scores(q64[h], K64, I_ref[h], alpha, False))
        aS.append(np.abs(q64[h][:, I_ref[h]]))
        bS.append(np.abs(K64[:, I_ref[h]]).T)
        O_ref.append(oracle.reduced_product(P64[h], V64, T_ref[h]))
        aO.append(np.abs(P64[h][:, T_ref[h]]))
        bO.append(np.abs(V64[T_ref[h]]))
    idx = torch.tensor(heads, device=dev)
    assert_heads_close(S[idx], np.stack(S_ref), aS, bS, alpha=alpha)
    assert_heads_close(O[idx], np.stack(O_ref), aO, bO)


@pytest.mark.parametrize("n", [2048, 4096])
def test_fused_attention_full(rmm, n):
    """The fused RMM attention at the bench's attention point (32 query / 8 KV
    heads, causal, rho_d = rho_t = 0.8): I bit-exact on every head; on three
    heads the oracle's three steps in full, T bit-exact where the oracle's
    token scores are separated at the boundary by more than the fp32 sums'
    error (n 2^-24 relative) and otherwise differing only in tokens that close
    to the k-th score, and O on sampled rows within the bound the op derives
    for its bf16 weights."""
    H, Hkv, dh, rho = 32, 8, 128, 0.8
    kd, kt = oracle.retained_count(rho, dh), oracle.retained_count(rho, n)
    (Q, K), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(106, n=n, col_gain=g), lambda x: gap.scores_per_head(x[0]), [kd])
    V = torch.randn((Hkv, n, 128), generator=W.gen(107)).to(torch.bfloat16)
    alpha = 1.0 / math.sqrt(dh)
    dev = torch.device("cuda")
    O, I, T = rmm.attention(Q.to(dev), K.to(dev), V.to(dev), rho, rho, causal=True, alpha=alpha,
                            return_sets=True)
    torch.cuda.synchronize()
    rmm.check_workspaces()
    I_all = np.stack([oracle.select(Q[h], k=kd)[0] for h in range(H)])
    assert_indices_equal(I, I_all)
    Tg = T.cpu().numpy()
    rows = sample_rows(n, 5)
    err = n * 2.0 ** -24
    compared = 0
    for h in (0, 13, 31):
        g = oracle.kv_head_of(h, H, Hkv)
        O_ref, I_ref, T_ref, P_ref = oracle.rmm_attention(Q[h:h + 1], K[g:g + 1], V[g:g + 1], rho, rho, alpha,
                                                          True)
        assert np.array_equal(I_ref[0], I_all[h])
        a2 = (P_ref[0] ** 2).sum(axis=0)
        if gap.boundary_gap(a2, kt) >= 2 * err:
            assert np.array_equal(Tg[h], T_ref[0]), h
        else:
            kth = np.sort(a2)[::-1][kt - 1]
            for t in np.setxor1d(Tg[h], T_ref[0]):
                assert abs(a2[t] - kth) <= 4 * err * kth, (h, int(t))
        if not np.array_equal(Tg[h], T_ref[0]):
            continue  # the output is the oracle's only over the same token set
        V64 = oracle.as_f64(V[g])
        absP, absV = np.abs(P_ref[0][rows][:, T_ref[0]]), np.abs(V64[T_ref[0]])
        fro = max(2e-3, 2.0 ** -8 * np.linalg.norm(absP @ absV) / max(np.linalg.norm(O_ref[0][rows]), 1e-300))
        assert_product_close(O[h][rows], O_ref[0][rows], absP, absV, rel_fro=fro)
        compared += 1
    assert compared >= 1, "no sampled head kept the oracle's token set"
