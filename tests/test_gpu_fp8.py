"""GPU parity of the low-bit form of RMM (8-bit E4M3 operands with per-tensor
scales folded into alpha, bf16 output; tcgen05 kind::f8f6f4) against the CPU
oracle on the exactly decoded codes.

The index set is bit-exact (scores are sums of squares of the decoded codes,
exact per term in fp32); the product on that index set meets the same bounds
as the bf16 form (its operands are exact, fp32 accumulation, bf16 rounding of
the output), scaled by alpha."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap
from tests.parity import assert_indices_equal, assert_product_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


def _quantized(gen, seed, n, d, m, ks, **kw):
    """E4M3 codes of a bf16 workload, with the boundary gaps opened on the
    decoded codes' scores (gains applied before the quantization)."""
    def make(g):
        A, B = gen(seed, n=n, d=d, m=m, col_gain=g, **kw)
        Aq, sa = W.quantize_e4m3(A)
        Bq, sb = W.quantize_e4m3(B)
        return Aq, Bq, sa, sb
    (Aq, Bq, sa, sb), _ = gap.enforce_boundary_gaps(
        make, lambda x: [oracle.column_scores_sq(oracle.decode_e4m3(x[0]))], ks)
    return Aq, Bq, sa, sb


def _check(rmm, Aq, Bq, sa, sb, rho, rows=None):
    dev = torch.device("cuda")
    alpha = sa * sb
    Y, I = rmm.matmul(Aq.to(dev), Bq.to(dev), rho=rho, return_indices=True, alpha=alpha)
    torch.cuda.synchronize()
    rmm.check_workspaces()
    assert Y.dtype == torch.bfloat16
    A64, B64 = oracle.decode_e4m3(Aq), oracle.decode_e4m3(Bq)
    I_ref, _ = oracle.select(A64, rho=rho)
    assert_indices_equal(I, I_ref)
    r = list(range(A64.shape[0])) if rows is None else rows
    Y_ref = alpha * oracle.reduced_product(A64, B64, I_ref, r)
    assert_product_close(Y[r], Y_ref, np.abs(A64[r][:, I_ref]), np.abs(B64[I_ref]), alpha=alpha)
    return Y, I


# ragged row / column tiles and k, a split tail, the bench's shapes
@pytest.mark.parametrize("gen,n,d,m", [(W.mlp_up, 300, 1024, 528), (W.mlp_down, 1100, 2048, 784),
                                       (W.mlp_up, 200, 4096, 14336)])
def test_fp8_linear(rmm, gen, n, d, m):
    rhos = [0.5, 0.8, 1.0]
    ks = [oracle.retained_count(r, d) for r in rhos]
    Aq, Bq, sa, sb = _quantized(gen, 81, n, d, m, ks)
    for rho in rhos:
        _check(rmm, Aq, Bq, sa, sb, rho, rows=None if n <= 300 else list(range(0, n, 5)))


@pytest.mark.parametrize("kind", ["up", "down"])
def test_fp8_llama8b_mlp_full_size(rmm, kind):
    """The benchmark's MLP shapes at n = 4096, rho = 0.8: the index set in
    full, the product on two seeded rows of every 128-row tile."""
    from tests.parity import sample_rows
    n, rho = 4096, 0.8
    d, m = W.LLAMA8B_MLP[kind]
    gen = W.mlp_up if kind == "up" else W.mlp_down
    Aq, Bq, sa, sb = _quantized(gen, 82, n, d, m, [oracle.retained_count(rho, d)])
    _check(rmm, Aq, Bq, sa, sb, rho, rows=sample_rows(n, 3))


def test_fp8_given_indices_and_determinism(rmm):
    n, d, m = 260, 1024, 528
    Aq, Bq, sa, sb = _quantized(W.mlp_up, 83, n, d, m, [oracle.retained_count(0.6, d)])
    dev = torch.device("cuda")
    Y1, I1 = rmm.matmul(Aq.to(dev), Bq.to(dev), rho=0.6, return_indices=True, alpha=sa * sb)
    Y2 = rmm.matmul(Aq.to(dev), Bq.to(dev), indices=I1, alpha=sa * sb)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)


def test_fp8_rejects_what_it_does_not_run(rmm):
    """Few rows (no CTA-pair tile) and attention modes: RMM_ERR_UNSUPPORTED on
    the host, before anything is launched."""
    for mode, n in ((rmm.RMM_LINEAR, 64), (rmm.RMM_QK, 256), (rmm.RMM_PV, 256)):
        p = rmm.rmm_problem_init(mode, rmm.RMM_FP8_E4M3, n, 256, 256)
        p.rho = 0.5
        with pytest.raises(rmm.RmmError) as e:
            rmm.Plan(p)
        assert e.value.status == rmm.RMM_ERR_UNSUPPORTED
