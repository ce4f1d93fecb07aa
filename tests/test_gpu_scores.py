"""GPU parity of producer-fused scoring: column scores written by the op that
produces an RMM input (the product's epilogue, RMM_FLAG_EMIT_SCORES; the
attention softmax, rmm_softmax_scores) and taken as given by the next op
(RMM_FLAG_GIVEN_SCORES), against the CPU oracle.

The scores are defined on the stored (rounded) output, so they are checked
against the oracle's column scores of the GPU's own output; the index set the
next op takes from them is checked bit-exactly against the oracle's selection
on that output, on inputs whose boundary gap exceeds fp32 summation error."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap
from tests.parity import assert_indices_equal, assert_product_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


def _scores_close(s2_gpu, s2_ref, rows):
    """fp32 sums of exactly squared stored values: relative error <= rows * 2^-24."""
    g = np64(s2_gpu)
    ref = np.asarray(s2_ref, dtype=np.float64)
    rel = np.abs(g - ref) / np.maximum(ref, 1e-30)
    assert rel.max() <= rows * 2.0 ** -24 + 1e-7, f"column scores off by {rel.max():.3e}"


# (n, d, m, dtype): the CTA-pair product (epilogue form, ragged tiles), the
# few-row and the single-CTA products (a score pass over Y), fp32 pairs
EMIT_SHAPES = [(300, 1024, 520, torch.bfloat16), (1100, 2048, 776, torch.bfloat16), (48, 1024, 264, torch.bfloat16),
               (100, 512, 264, torch.bfloat16), (300, 512, 264, torch.float32)]


@pytest.mark.parametrize("n,d,m,dtype", EMIT_SHAPES)
def test_emitted_scores_are_the_outputs_column_scores(rmm, n, d, m, dtype):
    rho = 0.6
    k = oracle.retained_count(rho, d)
    (A, B), _ = gap.enforce_boundary_gaps(
        lambda g: W.mlp_up(71, n=n, d=d, m=m, col_gain=g, dtype=dtype), lambda x: gap.scores_2d(x[0]), [k])
    Ag, Bg = A.cuda(), B.cuda()
    Y, I, s2 = rmm.matmul(Ag, Bg, rho=rho, return_indices=True, emit_scores=True)
    Y2, _, s2b = rmm.matmul(Ag, Bg, rho=rho, return_indices=True, emit_scores=True)
    torch.cuda.synchronize()
    rmm.check_workspaces()
    I_ref, _ = oracle.select(A, rho=rho)
    assert_indices_equal(I, I_ref)
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    rows = list(range(0, n, 3))
    assert_product_close(Y[rows], oracle.reduced_product(A64, B64, I_ref, rows), np.abs(A64[rows][:, I_ref]),
                         np.abs(B64[I_ref]))
    _scores_close(s2, oracle.column_scores_sq(Y.cpu()), n)
    assert torch.equal(s2, s2b) and torch.equal(Y, Y2), "emitted scores must be the same bits on every call"


@pytest.mark.parametrize("n2_rows", [300, 40])
def test_given_scores_chain_two_linear_ops(rmm, n2_rows):
    """op 1: Y = RMM(A, B1) writes Y's column scores; op 2: RMM(Y, B2) takes
    them and skips its score pass.  I of op 2 is the TopK of the given scores
    and the oracle's selection on the stored Y (B1's column gains open the
    boundary gap of Y's scores)."""
    n, d, m, m2, rho1, rho2 = n2_rows, 1024, 776, 520, 0.7, 0.5
    k2 = oracle.retained_count(rho2, m)

    def make(g):
        A, B1 = W.mlp_up(72, n=n, d=d, m=m)
        B1 = B1.float() if g is None else (B1.double() * torch.as_tensor(g)).float()
        return A, B1.to(torch.bfloat16).contiguous()

    def y_scores(x):
        A64, B64 = oracle.as_f64(x[0]), oracle.as_f64(x[1])
        return [oracle.column_scores_sq(A64 @ B64)]

    (A, B1), _ = gap.enforce_boundary_gaps(make, y_scores, [k2])
    _, B2 = W.mlp_down(73, n=1, d=m, m=m2)
    Ag, B1g, B2g = A.cuda(), B1.cuda(), B2.cuda()
    Y, s2 = rmm.matmul(Ag, B1g, rho=rho1, emit_scores=True)
    Z, I2 = rmm.matmul(Y, B2g, rho=rho2, return_indices=True, scores=s2)
    Z0, I0 = rmm.matmul(Y, B2g, rho=rho2, return_indices=True)  # the same op scoring Y itself
    torch.cuda.synchronize()
    rmm.check_workspaces()
    Yc = Y.cpu()
    _scores_close(s2, oracle.column_scores_sq(Yc), n)
    assert np.array_equal(I2.cpu().numpy(), oracle.topk_indices(np64(s2), k2))
    I_ref, _ = oracle.select(Yc, rho=rho2)
    assert_indices_equal(I2, I_ref)
    assert torch.equal(I2, I0)
    Y64, B64 = oracle.as_f64(Yc), oracle.as_f64(B2)
    assert_product_close(Z, oracle.reduced_product(Y64, B64, I_ref), np.abs(Y64[:, I_ref]), np.abs(B64[I_ref]))


def _causal_logits(seed, H, n, t, causal, device):
    """bf16 scores [H, n, t] = N(0, 2) logits plus a per-(head, key) bias
    N(0, 1.5) (keys of different weight, as attention has), -inf above the
    diagonal when causal."""
    g = W.gen(seed, device)
    S = torch.randn((H, n, t), generator=g, device=device) * 2.0
    S += torch.randn((H, 1, t), generator=g, device=device) * 1.5
    if causal:
        S.masked_fill_(torch.ones((n, t), dtype=torch.bool, device=device).triu_(1), -math.inf)
    return S.to(torch.bfloat16)


@pytest.mark.parametrize("H,n,t,causal", [(4, 512, 512, True), (2, 300, 4096, False), (2, 64, 8192, False),
                                          (3, 1000, 1000, True), (2, 1100, 1536, True), (1, 2048, 2048, True)])
def test_softmax_scores(rmm, H, n, t, causal):
    dev = torch.device("cuda")
    S = _causal_logits(74, H, n, t, causal, dev)
    P, s2 = rmm.softmax_scores(S, causal=causal)
    P2, s2b = rmm.softmax_scores(S, causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(P, P2) and torch.equal(s2, s2b), "same bits on every call"
    P_ref = oracle.softmax_rows(S.cpu())
    Pg = np64(P)
    # bf16 rounding of the weights (2^-9 relative) plus fp32 exponentials and sums
    err = np.abs(Pg - P_ref)
    assert np.all(err <= 2.0 ** -8 * P_ref + 1e-7), f"max error {err.max():.3e}"
    if causal:
        assert np.all(Pg[:, np.triu(np.ones((n, t), dtype=bool), 1)] == 0.0)
    for h in range(H):
        _scores_close(s2[h], oracle.column_scores_sq(P[h].cpu()), n)


def test_pv_with_scores_from_the_softmax(rmm):
    """QK -> softmax_scores -> PV with the given token scores: T is the TopK
    of the softmax's scores and the oracle's selection on the stored P; the
    product matches the oracle on that T.  Seeds are taken in order until the
    boundary gap of every head exceeds fp32 summation error."""
    H, Hkv, n, dv, rho = 4, 2, 512, 128, 0.6
    k = oracle.retained_count(rho, n)
    dev = torch.device("cuda")
    for seed in range(75, 95):
        S = _causal_logits(seed, H, n, n, True, dev)
        P, s2 = rmm.softmax_scores(S, causal=True)
        torch.cuda.synchronize()
        Pc = P.cpu()
        sc = [oracle.column_scores_sq(Pc[h]) for h in range(H)]
        if min(gap.boundary_gap(x, k) for x in sc) >= 1e-3:
            break
    else:
        pytest.fail("no seed with an open boundary gap")
    g = W.gen(seed + 100, dev)
    V = (torch.randn((Hkv, n, dv), generator=g, device=dev)).to(torch.bfloat16)
    O, T = rmm.pv(P, V, rho=rho, return_indices=True, causal=True, scores=s2)
    O0, T0 = rmm.pv(P, V, rho=rho, return_indices=True, causal=True)
    torch.cuda.synchronize()
    rmm.check_workspaces()
    T_top = np.stack([oracle.topk_indices(np64(s2[h]), k) for h in range(H)])
    assert np.array_equal(T.cpu().numpy(), T_top)
    T_ref = np.stack([oracle.select(Pc[h], k=k)[0] for h in range(H)])
    assert_indices_equal(T, T_ref)
    assert torch.equal(T, T0)
    P64, V64 = oracle.as_f64(Pc), oracle.as_f64(V)
    for h in range(H):
        gv = oracle.kv_head_of(h, H, Hkv)
        assert_product_close(O[h], oracle.reduced_product(P64[h], V64[gv], T_ref[h]), np.abs(P64[h][:, T_ref[h]]),
                             np.abs(V64[gv][T_ref[h]]))


def test_given_scores_on_every_selection_path(rmm):
    """Given scores replace each selection kernel (one-row, few-row, small
    head, score pass + radix select): the index set is the TopK of the given
    scores, the same as the op computing them itself."""
    dev = torch.device("cuda")
    cases = [(1, 4096), (4, 128), (200, 512), (600, 4096)]
    for n, d in cases:
        rho = 0.5
        k = oracle.retained_count(rho, d)
        (A, B), _ = gap.enforce_boundary_gaps(lambda g: W.mlp_up(76, n=n, d=d, m=136, col_gain=g),
                                              lambda x: gap.scores_2d(x[0]), [k])
        Ag, Bg = A.to(dev), B.to(dev)
        I_self, s2 = rmm.select(Ag, rho=rho, return_scores=True)
        Y, I = rmm.matmul(Ag, Bg, rho=rho, return_indices=True, scores=s2)
        torch.cuda.synchronize()
        assert torch.equal(I, I_self), (n, d)
        assert np.array_equal(I.cpu().numpy(), oracle.topk_indices(np64(s2), k))
