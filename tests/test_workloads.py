"""The seeded generators: reproducible, right shapes and dtypes, and the
gap enforcement that the parity tests rely on (no GPU)."""
import numpy as np
import torch

import oracle
import workloads as W
from tests import gap


def test_seeded_and_shaped():
    A1, B1 = W.linear_small(7)
    A2, B2 = W.linear_small(7)
    assert torch.equal(A1, A2) and torch.equal(B1, B2)
    assert A1.shape == (64, 256) and B1.shape == (256, 256) and A1.dtype == torch.float32
    A, B = W.mlp_up(3, n=8)
    assert A.shape == (8, 4096) and B.shape == (4096, 14336) and A.dtype == torch.bfloat16
    A, B = W.mlp_down(3, n=8)
    assert A.shape == (8, 14336) and B.shape == (14336, 4096)
    assert float(A.float().min()) >= -0.28  # SiLU bottoms out near -0.2785 (bf16: -0.2793)
    Q, K = W.attn_qk(1, n=16)
    assert Q.shape == (32, 16, 128) and K.shape == (8, 16, 128)
    P, V = W.attn_pv(1, n=16, heads=4, kv_heads=2)
    assert P.shape == (4, 16, 16) and V.shape == (2, 16, 128)
    Pf = P.float()
    assert torch.all(Pf.triu(1) == 0)
    assert torch.allclose(Pf.sum(-1), torch.ones(4, 16), atol=2e-2)
    for shape, (d, m) in W.LLAMA70B_LINEAR.items():
        A, B = W.linear_70b(5, n=2, shape=shape)
        assert A.shape == (2, d) and B.shape == (d, m)


def test_outlier_channels():
    g = W.gen(9)
    A, _ = W.mlp_up(9, n=256, m=8)
    s = A.float().pow(2).mean(0).sqrt()
    assert int((s > 10 * s.median()).sum()) >= 20  # ~41 channels carry a x20 scale


def test_all_gaps_construction():
    A, _ = W.linear_small(21)
    g = gap.all_gaps_gain(oracle.column_scores_sq(A))
    A2, _ = W.linear_small(21, col_gain=g)
    assert gap.min_adjacent_gap(oracle.column_scores_sq(A2)) >= 1e-3


def test_boundary_gap_enforcement():
    ks = [oracle.retained_count(r, 4096) for r in (0.5, 0.7, 0.8)]
    (A, B), gain = gap.enforce_boundary_gaps(
        lambda g: W.mlp_up(4, n=32, m=8, col_gain=g), lambda x: gap.scores_2d(x[0]), ks)
    s2 = oracle.column_scores_sq(A)
    for k in ks:
        assert gap.boundary_gap(s2, k) >= 1e-3
