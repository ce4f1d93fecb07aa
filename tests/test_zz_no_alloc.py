"""rmm_select_no_alloc: index selection for callers that cannot allocate
device memory (frozen or captured pools, plugins inside another allocator,
fixed-budget processes).  It must give the same index set as rmm_select
(which uses a caller-provided workspace) and the same scores within the fp32
summation tolerance, on repeated calls that reuse its static scratch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


@pytest.mark.parametrize("gen,n,d,rho", [(W.mlp_up, 1024, 4096, 0.8), (W.mlp_down, 256, 14336, 0.5)])
def test_no_alloc_select_matches_workspace_select(rmm, gen, n, d, rho):
    ks = [oracle.retained_count(rho, d)]
    (A, _), _ = gap.enforce_boundary_gaps(lambda g: gen(41, n=n, d=d, m=8, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), ks)
    Ag = A.cuda()
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, n, d, 8)
    p.rho = rho
    plan = rmm.Plan(p)
    ws = rmm.workspace_for(plan)
    I_ref = torch.empty(plan.k, dtype=torch.int32, device="cuda")
    s2_ref = torch.empty(d, dtype=torch.float32, device="cuda")
    rmm.rmm_select(plan, Ag, I_ref, s2_ref, ws)
    torch.cuda.synchronize()
    tol = n * 2.0 ** -24 + 1e-7
    for call in range(2):
        I = torch.full((plan.k,), -1, dtype=torch.int32, device="cuda")
        s2 = torch.full((d,), -1.0, dtype=torch.float32, device="cuda")
        rmm.rmm_select_no_alloc(plan, Ag, I, s2)
        torch.cuda.synchronize()
        assert torch.equal(I, I_ref), f"call {call}: index sets differ"
        rel = ((s2.double() - s2_ref.double()).abs() / s2_ref.double().clamp_min(1e-30)).max().item()
        assert rel <= tol, f"call {call}: scores differ by {rel:.3e}"
        # and the index set is the oracle's
        assert np.array_equal(I.cpu().numpy(), oracle.select(A, rho=rho)[0])
        # scores only: I still written
        I2 = torch.full((plan.k,), -1, dtype=torch.int32, device="cuda")
        rmm.rmm_select_no_alloc(plan, Ag, I2, None)
        torch.cuda.synchronize()
        assert torch.equal(I2, I_ref)


def test_no_alloc_rejects_problems_beyond_its_scratch(rmm):
    # 22 heads x d = 49152: one row split per column block, so the scratch needs
    # 22 * 49152 * 4 * (1 + 1) bytes plus counters > 8 MiB.  The input is
    # allocated at its full size, so the call would stay in bounds even if it
    # were (wrongly) accepted.
    heads, n, d = 22, 8, 49152
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, n, d, 8)
    p.heads, p.kv_heads = heads, 1
    p.stride_a, p.stride_y = n * d, n * 8
    p.rho = 0.5
    plan = rmm.Plan(p)
    A = torch.zeros((heads, n, d), dtype=torch.bfloat16, device="cuda")
    I = torch.empty((heads, plan.k), dtype=torch.int32, device="cuda")
    with pytest.raises(rmm.RmmError) as e:
        rmm.rmm_select_no_alloc(plan, A, I)
    assert e.value.status == rmm.RMM_ERR_UNSUPPORTED


@pytest.mark.parametrize("case", ["pv_causal_heads", "qk_few_rows", "one_row"])
def test_no_alloc_select_per_head(rmm, case):
    """Several heads: per-head scratch offsets of the score pass (a causal PV
    plan, 4 heads of 512 tokens), and the one-kernel selections that need no
    scratch (QK heads of 4 rows, and one bf16 row per head), each against
    rmm_select on a workspace on two calls in a row."""
    dev = torch.device("cuda")
    if case == "pv_causal_heads":
        H, n = 4, 512
        ks = [oracle.retained_count(0.8, n)]
        (P, _), _ = gap.enforce_boundary_gaps(
            lambda g: W.attn_pv(42, n=n, heads=H, kv_heads=2, col_gain=g),
            lambda x: gap.scores_per_head(x[0]), ks)
        X = P.to(dev)
        p = rmm.rmm_problem_init(rmm.RMM_PV, rmm.RMM_BF16, n, n, 128)
        p.flags = rmm.RMM_FLAG_CAUSAL
        p.rho = 0.8
    elif case == "qk_few_rows":
        H, n = 8, 4
        ks = [oracle.retained_count(0.5, 128)]
        (Q, _), _ = gap.enforce_boundary_gaps(
            lambda g: W.attn_qk(43, n=n, heads=H, kv_heads=2, col_gain=g),
            lambda x: gap.scores_per_head(x[0]), ks)
        X = Q.to(dev)
        p = rmm.rmm_problem_init(rmm.RMM_QK, rmm.RMM_BF16, n, 128, 64)
        p.rho = 0.5
    else:  # one bf16 row per head over 4096 tokens (decode-step PV weights)
        H, n, t = 8, 1, 4096
        ks = [oracle.retained_count(0.5, t)]
        (_, _, _, P), _ = gap.enforce_boundary_gaps(
            lambda g: W.attn_decode(44, t=t, heads=H, kv_heads=2, p_gain=g),
            lambda x: gap.scores_per_head(x[3]), ks)
        X = P.to(dev)
        p = rmm.rmm_problem_init(rmm.RMM_PV, rmm.RMM_BF16, n, t, 128)
        p.rho = 0.5
    d = X.shape[2]
    p.lda = d
    p.heads, p.kv_heads = H, H
    p.stride_a = X.stride(0)
    p.ldb, p.stride_b = (d if p.mode == rmm.RMM_QK else 128), 0
    p.ldy = p.m
    p.stride_y = n * p.m
    plan = rmm.Plan(p)
    ws = rmm.workspace_for(plan)
    I_ref = torch.empty((H, plan.k), dtype=torch.int32, device=dev)
    s2_ref = torch.empty((H, d), dtype=torch.float32, device=dev)
    rmm.rmm_select(plan, X, I_ref, s2_ref, ws)
    torch.cuda.synchronize()
    assert np.array_equal(I_ref.cpu().numpy(),
                          np.stack([oracle.select(X[h].cpu(), k=plan.k)[0] for h in range(H)]))
    tol = n * 2.0 ** -24 + 1e-7
    for call in range(2):
        I = torch.full((H, plan.k), -1, dtype=torch.int32, device=dev)
        s2 = torch.full((H, d), -1.0, dtype=torch.float32, device=dev)
        rmm.rmm_select_no_alloc(plan, X, I, s2)
        torch.cuda.synchronize()
        assert torch.equal(I, I_ref), f"call {call}: index sets differ"
        rel = ((s2.double() - s2_ref.double()).abs() / s2_ref.double().clamp_min(1e-30)).max().item()
        assert rel <= tol, f"call {call}: scores differ by {rel:.3e}"
