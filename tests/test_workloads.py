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


def test_attn_decode_shapes_and_structure():
    """The decode-step generator: shapes for `batch` sequences, seeded, P rows
    summing to one, the gains applied where documented, and the query heads of
    one KV head weighing tokens more alike than heads of different KV heads
    (the shared half of their logits)."""
    q, K, V, P = W.attn_decode(3, t=512, batch=2, n=1, heads=8, kv_heads=2, head_dim=64, v_dim=32)
    assert q.shape == (16, 1, 64) and K.shape == (4, 512, 64) and V.shape == (4, 512, 32)
    assert P.shape == (16, 1, 512) and P.dtype == torch.bfloat16
    q2, K2, V2, P2 = W.attn_decode(3, t=512, batch=2, n=1, heads=8, kv_heads=2, head_dim=64, v_dim=32)
    assert all(torch.equal(a, b) for a, b in ((q, q2), (K, K2), (V, V2), (P, P2)))
    assert torch.allclose(P.float().sum(-1), torch.ones(16, 1), atol=2e-2)
    # logits' correlation: heads 0-3 share KV head 0, heads 4-7 KV head 1
    lg = torch.log(P.float().clamp_min(1e-30))[:, 0]
    lg = lg - lg.mean(-1, keepdim=True)
    c = (lg @ lg.T) / (lg.norm(dim=-1)[:, None] * lg.norm(dim=-1)[None, :])
    same = float(c[0, 1:4].mean())
    other = float(c[0, 4:8].mean())
    assert same > 0.35 and abs(other) < 0.2, (same, other)
    g = np.ones((16, 64))
    g[:, 5] = 4.0
    qg = W.attn_decode(3, t=512, batch=2, n=1, heads=8, kv_heads=2, head_dim=64, v_dim=32, q_gain=g)[0]
    assert torch.allclose(qg.float()[:, :, 5], (4.0 * q.float()[:, :, 5]).to(torch.bfloat16).float())
    assert torch.equal(qg[:, :, 6], q[:, :, 6])
    gp = np.ones((16, 512))
    gp[:, 7] = 0.5
    Pg = W.attn_decode(3, t=512, batch=2, n=1, heads=8, kv_heads=2, head_dim=64, v_dim=32, p_gain=gp)[3]
    assert torch.equal(Pg[:, :, 8], P[:, :, 8])
    assert torch.allclose(Pg.float()[:, :, 7], 0.5 * P.float()[:, :, 7], rtol=1e-2)
