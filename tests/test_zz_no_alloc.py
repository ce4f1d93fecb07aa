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
