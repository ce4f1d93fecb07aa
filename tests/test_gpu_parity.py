"""GPU parity of the CUDA path (through the C ABI) against the CPU oracle on
oracle-scale inputs: several tiles and ragged tails, every mode, the
tie-break, given index sets, empty and degenerate shapes.

Inputs come from workloads/ with the oracle-measured score gap of
tests/gap.py, so that fp32 (GPU) and fp64 (oracle) scores order the
boundary the same way."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gap
from tests.parity import assert_heads_close, assert_indices_equal, assert_product_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rmm(cuda_device):
    import input_adaptive_reduced_b200 as r
    return r


def _linear_case(rmm, A, B, rho, rows=None):
    dev = torch.device("cuda")
    Ag, Bg = A.to(dev), B.to(dev)
    Y, I = rmm.matmul(Ag, Bg, rho=rho, return_indices=True)
    torch.cuda.synchronize()
    I_ref, _ = oracle.select(A, rho=rho)
    assert_indices_equal(I, I_ref)
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    r = slice(None) if rows is None else rows
    Y_ref = oracle.reduced_product(A64, B64, I_ref, rows)
    assert_product_close(Y[r] if rows is None else Y[rows], Y_ref,
                         np.abs(A64[r][:, I_ref]), np.abs(B64[I_ref, :]))
    return Y, I


@pytest.mark.parametrize("rho", [0.25, 0.5, 1.0])
@pytest.mark.parametrize("seed", [1, 2])
def test_linear_fp32_tiny(rmm, rho, seed):
    """64 x 256 x 256 fp32 (the one-launch tiny kernel: scores, TopK and an fp32
    FMA product), all sorted scores >= 1e-3 apart."""
    A, B = W.linear_small(seed)
    g = gap.all_gaps_gain(oracle.column_scores_sq(A))
    A, B = W.linear_small(seed, col_gain=g)
    assert gap.min_adjacent_gap(oracle.column_scores_sq(A)) >= 1e-3
    _linear_case(rmm, A, B, rho)


@pytest.mark.parametrize("n,d,m,rho", [(1, 100, 72, 0.5), (17, 256, 300, 0.8), (64, 64, 4, 0.9),
                                       (64, 252, 132, 0.3), (40, 4, 8, 0.5)])
def test_tiny_fp32_shapes(rmm, n, d, m, rho):
    """The one-launch fp32 kernel across its limits: one row, d up to 256 with
    ragged 32-column words, one 16-byte group of output columns, several
    32-column and 16-row CTAs, k = 2; then with a given index set, a scale and
    a padded row stride of A."""
    k = oracle.retained_count(rho, d)
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: W.linear_small(61, n=n, d=d, m=m, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), [k])
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_F32, n, d, m)
    p.rho = rho
    assert rmm.Plan(p).kernel_launches == 1
    _linear_case(rmm, A, B, rho)
    dev = torch.device("cuda")
    I = torch.from_numpy(np.sort(np.random.default_rng(d).choice(d, size=k, replace=False)).astype(np.int32))
    Apad = torch.zeros((n, d + 4), dtype=torch.float32)
    Apad[:, :d] = A
    Y = rmm.matmul(Apad.to(dev)[:, :d], B.to(dev), indices=I.to(dev), alpha=0.375)
    torch.cuda.synchronize()
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    I64 = I.numpy()
    assert_product_close(Y, 0.375 * oracle.reduced_product(A64, B64, I64), np.abs(A64[:, I64]), np.abs(B64[I64]),
                         alpha=0.375)


@pytest.mark.parametrize("direction", ["copy_up", "copy_down"])
@pytest.mark.parametrize("rho", [0.25, 0.5])
def test_exact_tie_lower_index_wins(rmm, rho, direction):
    """Duplicated columns straddling the k-th rank: equal scores, lower index kept."""
    A, B = W.linear_small(5)
    A, B = W.linear_small(5, col_gain=gap.all_gaps_gain(oracle.column_scores_sq(A)))
    s2 = oracle.column_scores_sq(A)
    order = gap.descending_order(s2)
    k = oracle.retained_count(rho, A.shape[1])
    src = int(order[k - 1])  # the last kept column
    dropped = order[k:].tolist()
    # copy it over a dropped column above it (src stays kept) or below it (the copy wins)
    cands = [j for j in dropped if (j > src if direction == "copy_up" else j < src)]
    if not cands:
        pytest.skip("no dropped column on that side of the boundary column")
    dst = cands[0]
    A2 = W.duplicate_columns(A, [(src, dst)])
    s2b = oracle.column_scores_sq(A2)
    assert s2b[src] == s2b[dst]
    Y, I = _linear_case(rmm, A2, B, rho)
    lo, hi = min(src, dst), max(src, dst)
    got = set(I.cpu().tolist())
    assert lo in got and hi not in got


def _tie_pair(s2, k, direction, other_block_of=None):
    """(src, dst): src is the last kept column; dst a dropped column above
    (copy_up) or below (copy_down) it, in another 256-column block when
    other_block_of is set.  None when there is no such column."""
    order = gap.descending_order(s2)
    src = int(order[k - 1])
    for j in order[k:].tolist():
        if (j > src) != (direction == "copy_up"):
            continue
        if other_block_of is not None and j // other_block_of == src // other_block_of:
            continue
        return src, int(j)
    return None


@pytest.mark.parametrize("direction", ["copy_up", "copy_down"])
@pytest.mark.parametrize("kind,d", [("up", 4096), ("down", 14336)])
def test_exact_tie_across_column_blocks(rmm, kind, d, direction):
    """Duplicated bf16 columns in different 256-column blocks of the score pass,
    at n = 1024 where every column block is summed in several row splits (16 at
    d = 4096, 6 at d = 14336) and the last CTA of the block adds the split
    partials: equal columns must get bit-equal scores wherever they sit, and
    the lower index of the tied pair is the one kept."""
    n, m, rho = 1024, 264, 0.8
    k = oracle.retained_count(rho, d)
    gen = W.mlp_up if kind == "up" else W.mlp_down
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: gen(21, n=n, d=d, m=m, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), [k])
    pair = _tie_pair(oracle.column_scores_sq(A), k, direction, other_block_of=256)
    if pair is None:
        pytest.skip("no dropped column on that side in another column block")
    src, dst = pair
    A2 = W.duplicate_columns(A, [(src, dst)])
    s2b = oracle.column_scores_sq(A2)
    assert s2b[src] == s2b[dst]
    Y, I = _linear_case(rmm, A2, B, rho, rows=list(range(0, n, 37)))
    got = set(I.cpu().tolist())
    assert min(src, dst) in got and max(src, dst) not in got


@pytest.mark.parametrize("n", [2, 4, 512, 1024])
def test_exact_tie_per_head_features(rmm, n):
    """Per-head feature selection with the boundary feature of every head
    duplicated over a dropped one (even heads above it, odd heads below it),
    through each selection path the heads take: n = 2 the decode QK kernel
    selects in-kernel, n = 4 the one-warp-per-head select (select() on
    [heads, 4, 128]), n = 512 and n = 1024 the QK op's cluster selection
    (eight CTAs per head adding their column sums in rank order)."""
    H, Hkv, dh, rho = 8, 2, 128, 0.8
    k = oracle.retained_count(rho, dh)
    nk = max(n, 64)  # keys: a multiple of 8

    def make(g):
        Qf, Kf = W.attn_qk(22, n=nk, heads=H, kv_heads=Hkv, head_dim=dh, col_gain=g)
        return Qf[:, :n].contiguous(), Kf

    (Q, K), _ = gap.enforce_boundary_gaps(make, lambda x: gap.scores_per_head(x[0]), [k])
    pairs = []
    for h in range(H):
        pr = _tie_pair(oracle.column_scores_sq(Q[h]), k, "copy_up" if h % 2 == 0 else "copy_down")
        if pr is None:
            pr = _tie_pair(oracle.column_scores_sq(Q[h]), k, "copy_down" if h % 2 == 0 else "copy_up")
        pairs.append(pr)
        Q[h] = W.duplicate_columns(Q[h], [pr])
    dev = torch.device("cuda")
    if n == 4:
        I = rmm.select(Q.to(dev), rho=rho)
    else:
        causal = n > 8  # the decode kernels take the non-causal form
        S, I = rmm.qk(Q.to(dev), K.to(dev), rho=rho, causal=causal, return_indices=True)
    torch.cuda.synchronize()
    I_ref = np.stack([oracle.select(Q[h], k=k)[0] for h in range(H)])
    assert_indices_equal(I, I_ref)
    for h, (src, dst) in enumerate(pairs):
        got = set(I[h].cpu().tolist())
        assert min(src, dst) in got and max(src, dst) not in got, h
    if n != 4:
        alpha = 1.0 / math.sqrt(dh)
        rows = list(range(n)) if n <= 8 else list(range(0, n, 61))
        S_ref, _ = oracle.rmm_qk(Q, K, rho=rho, alpha=alpha, causal=causal, heads=[0, 5], rows=rows)
        Q64, K64 = oracle.as_f64(Q), oracle.as_f64(K)
        mask = (np.arange(nk)[None, :] > np.asarray(rows)[:, None]) if causal else None
        for i, h in enumerate([0, 5]):
            g = oracle.kv_head_of(h, H, Hkv)
            assert_product_close(S[h][rows], S_ref[i], np.abs(Q64[h][rows][:, I_ref[h]]),
                                 np.abs(K64[g][:, I_ref[h]]).T, alpha=alpha, mask=mask)


LINEAR_SHAPES = [
    ("up", 200, 4096, 520),
    ("down", 136, 14336, 264),
    ("up", 1, 8192, 264),
    ("up", 16, 8192, 776),
    ("down", 130, 136, 24),
]


@pytest.mark.parametrize("kind,n,d,m", LINEAR_SHAPES)
def test_linear_bf16(rmm, kind, n, d, m):
    rhos = [0.5, 0.7, 0.8, 1.0]
    ks = [oracle.retained_count(r, d) for r in rhos]
    gen = W.mlp_up if kind == "up" else W.mlp_down
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: gen(11, n=n, d=d, m=m, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), ks)
    for rho in rhos:
        _linear_case(rmm, A, B, rho)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("rho", [0.2, 0.9])
def test_wide_column_pack(rmm, dtype, rho):
    """Packed A rows wider than 1024 columns: a CTA whose 2048 retained columns
    span few source columns (rho = 0.9) copies the span through shared memory;
    at rho = 0.2 the first CTA's span is too wide and it loads its columns one
    by one (bf16, d = 14336: the ragged second CTA's span is staged)."""
    n, d, m = 200, (14336 if dtype == torch.bfloat16 else 8192), 264
    k = oracle.retained_count(rho, d)
    assert k > 1024
    (A, B), _ = gap.enforce_boundary_gaps(
        lambda g: W.mlp_down(13, n=n, d=d, m=m, col_gain=g, dtype=dtype),
        lambda x: gap.scores_2d(x[0]), [k])
    _linear_case(rmm, A, B, rho)


def test_wide_column_pack_given_span(rmm):
    """A given index set whose first 2048 columns reach across the whole row
    (the direct body) and whose rest is dense (the staged body)."""
    n, d, m = 136, 14336, 264
    A, B = W.mlp_down(14, n=n, d=d, m=m)
    I = np.concatenate([np.arange(0, 1024), np.arange(d - 4096, d)]).astype(np.int32)
    Y = rmm.matmul(A.cuda(), B.cuda(), indices=torch.from_numpy(I).cuda())
    torch.cuda.synchronize()
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    assert_product_close(Y, oracle.reduced_product(A64, B64, I), np.abs(A64[:, I]), np.abs(B64[I]))


def test_select_scores_and_indices(rmm):
    A, _ = W.mlp_up(3, n=300, d=4096, m=8)
    Ag = A.cuda()
    for rho in (0.5, 0.8):
        I, s2 = rmm.select(Ag, rho=rho, return_scores=True)
        torch.cuda.synchronize()
        s2_ref = oracle.column_scores_sq(A)
        rel = np.abs(np64(s2) - s2_ref) / np.maximum(s2_ref, 1e-30)
        assert rel.max() <= 300 * 2.0 ** -24 + 1e-7
        # the index set is the TopK of the GPU's own scores (ties to the lower index)
        mine = oracle.topk_indices(np64(s2), I.numel())
        assert np.array_equal(I.cpu().numpy(), mine)


@pytest.mark.parametrize("d", [128, 4096, 32768, 40000])
def test_one_row_select_ties(rmm, d):
    """One row per head (n = 1): scores are squares of bf16 values, exact in
    fp32, so classes of equal values are exact ties; the boundary falls inside
    a class and its lowest indices are kept.  Values of both signs, zeros and
    ragged k; several heads; scores returned as a_j^2."""
    rng = np.random.default_rng(5)
    vals = np.array([0.0, 0.5, -0.5, 1.0, -1.0, 1.5, 2.0, -2.0, 3.0, 0.125], dtype=np.float32)
    A = torch.from_numpy(vals[rng.integers(0, len(vals), size=(3, 1, d))]).to(torch.bfloat16)
    A64 = oracle.as_f64(A)
    for k in sorted({1, 7, d // 3, d // 2 + 5, d - 1}):
        I, s2 = rmm.select(A.cuda(), k=k, return_scores=True)
        torch.cuda.synchronize()
        for h in range(3):
            assert np.array_equal(np64(s2[h]), oracle.column_scores_sq(A64[h]))
            assert np.array_equal(I[h].cpu().numpy(), oracle.select(A64[h], k=k)[0])


def test_few_feature_select(rmm):
    """d <= 256 columns and a few rows per head (one warp ranks a head's
    columns): 5 heads of 3 x 200, the last 32-column word ragged."""
    k = oracle.retained_count(0.6, 200)
    (A, _), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(61, n=3, heads=5, kv_heads=5, head_dim=200, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), [k])
    I, s2 = rmm.select(A.cuda(), k=k, return_scores=True)
    torch.cuda.synchronize()
    for h in range(5):
        s2_ref = oracle.column_scores_sq(A[h])
        assert np.max(np.abs(np64(s2[h]) - s2_ref) / np.maximum(s2_ref, 1e-30)) <= 3 * 2.0 ** -24 + 1e-7
        assert np.array_equal(I[h].cpu().numpy(), oracle.select(A[h], k=k)[0])


def test_given_indices(rmm):
    A, B = W.mlp_up(4, n=150, d=1024, m=264)
    rng = np.random.default_rng(0)
    I = np.sort(rng.choice(1024, size=333, replace=False)).astype(np.int32)
    Y = rmm.matmul(A.cuda(), B.cuda(), indices=torch.from_numpy(I).cuda())
    torch.cuda.synchronize()
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    assert_product_close(Y, oracle.reduced_product(A64, B64, I), np.abs(A64[:, I]), np.abs(B64[I]))


def test_dense_identity_and_indices_out(rmm):
    A, B = W.mlp_down(6, n=140, d=512, m=136)
    Y, I = rmm.matmul(A.cuda(), B.cuda(), rho=1.0, return_indices=True)
    torch.cuda.synchronize()
    assert np.array_equal(I.cpu().numpy(), np.arange(512))
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    assert_product_close(Y, A64 @ B64, np.abs(A64), np.abs(B64))


def test_single_index_and_empty(rmm):
    A, B = W.mlp_up(8, n=40, d=256, m=72)
    Y, I = rmm.matmul(A.cuda(), B.cuda(), k=1, return_indices=True)
    torch.cuda.synchronize()
    I_ref, _ = oracle.select(A, k=1)
    assert_indices_equal(I, I_ref)
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    assert_product_close(Y, oracle.reduced_product(A64, B64, I_ref), np.abs(A64[:, I_ref]),
                         np.abs(B64[I_ref]))
    Y0 = rmm.matmul(torch.empty((0, 256), dtype=torch.bfloat16, device="cuda"), B.cuda(), rho=0.5)
    assert Y0.shape == (0, 72)
    Ym = rmm.matmul(A.cuda(), torch.empty((256, 0), dtype=torch.bfloat16, device="cuda"), rho=0.5)
    assert Ym.shape == (40, 0)


def test_deterministic(rmm):
    A, B = W.mlp_up(9, n=260, d=4096, m=520)
    Ag, Bg = A.cuda(), B.cuda()
    Y1, I1 = rmm.matmul(Ag, Bg, rho=0.7, return_indices=True)
    Y2, I2 = rmm.matmul(Ag, Bg, rho=0.7, return_indices=True)
    torch.cuda.synchronize()
    assert torch.equal(I1, I2) and torch.equal(Y1, Y2)


@pytest.mark.parametrize("n,d,m,rho", [(260, 4096, 520, 0.7), (256, 1024, 512, 0.3), (1100, 8192, 2056, 0.6)])
def test_linear_back_to_back(rmm, n, d, m, rho):
    """Two different inputs run back to back on one plan and workspace with no
    host synchronisation in between (the workspace's counters are returned
    to zero by the kernels), each matching the oracle; shapes with ragged
    row / column tiles, a grid smaller than one wave, and a split tail."""
    k = oracle.retained_count(rho, d)
    dev = torch.device("cuda")
    ins = []
    for seed in (61, 62):
        (A, B), _ = gap.enforce_boundary_gaps(lambda g: W.mlp_up(seed, n=n, d=d, m=m, col_gain=g),
                                              lambda x: gap.scores_2d(x[0]), [k])
        ins.append((A, B))
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, n, d, m)
    p.rho = rho
    plan = rmm.Plan(p)
    ws = rmm.workspace_for(plan)
    outs = []
    for A, B in ins:
        Y = torch.empty((n, m), dtype=torch.bfloat16, device=dev)
        I = torch.empty(plan.k, dtype=torch.int32, device=dev)
        rmm.rmm_matmul(plan, A.to(dev), B.to(dev), Y, I, ws)
        outs.append((Y, I))
    torch.cuda.synchronize()
    rmm.check_workspaces()
    rows = list(range(0, n, 7))
    for (A, B), (Y, I) in zip(ins, outs):
        I_ref, _ = oracle.select(A, rho=rho)
        assert_indices_equal(I, I_ref)
        A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
        assert_product_close(Y[rows], oracle.reduced_product(A64, B64, I_ref, rows),
                             np.abs(A64[rows][:, I_ref]), np.abs(B64[I_ref]))


def _split_parts(tiles, num_kb):
    """Parts per tile of the CTA-pair kernel's split tail on this GPU (1 = none):
    the last wave's tiles are cut into f <= 4 K-parts that still fit one wave,
    each at least 8 k-blocks long."""
    clusters = torch.cuda.get_device_properties(0).multi_processor_count // 2
    rem = tiles % clusters
    if rem == 0:
        return 1
    f = min(clusters // rem, 4, num_kb // 8)
    return f if f >= 2 else 1


# (n, d, m, rho): tiles of 256 x 256 and k-blocks of 64 that give split tails
# of 4, 3 and 2 parts, one after a full wave of whole tiles
SPLIT_SHAPES = [(300, 4096, 704, 0.6), (1024, 4096, 1280, 0.8), (1280, 4096, 1536, 0.5),
                (2048, 2048, 2560, 0.7)]


@pytest.mark.parametrize("n,d,m,rho", SPLIT_SHAPES)
def test_split_tail_linear(rmm, n, d, m, rho):
    """Tiles of the last wave computed as K-parts and added in part order."""
    k = oracle.retained_count(rho, d)
    tiles = -(-n // 256) * -(-m // 256)
    assert _split_parts(tiles, -(-k // 64)) > 1
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: W.mlp_up(41, n=n, d=d, m=m, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), [k])
    Y1, _ = _linear_case(rmm, A, B, rho)
    Y2 = rmm.matmul(A.cuda(), B.cuda(), rho=rho)  # counters were reset by the first call
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    rmm.check_workspaces()


def test_split_tail_fp32(rmm):
    n, d, m, rho = 300, 1024, 600, 0.5
    k = oracle.retained_count(rho, d)
    assert _split_parts(-(-n // 256) * -(-m // 256), -(-k // 32)) > 1
    (A, B), _ = gap.enforce_boundary_gaps(
        lambda g: W.mlp_up(42, n=n, d=d, m=m, col_gain=g, dtype=torch.float32),
        lambda x: gap.scores_2d(x[0]), [k])
    _linear_case(rmm, A, B, rho)
    rmm.check_workspaces()


def test_split_tail_pv(rmm):
    H, Hkv, n, dv, rho = 2, 1, 2048, 128, 0.8
    k = oracle.retained_count(rho, n)
    assert _split_parts(H * (n // 256), -(-k // 64)) > 1
    (P, V), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_pv(43, n=n, heads=H, kv_heads=Hkv, v_dim=dv, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), [k])
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=rho, return_indices=True)
    torch.cuda.synchronize()
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=rho)
    assert_indices_equal(T, T_ref)
    P64, V64 = oracle.as_f64(P), oracle.as_f64(V)
    for h in range(H):
        assert_product_close(O[h], O_ref[h], np.abs(P64[h][:, T_ref[h]]), np.abs(V64[0][T_ref[h]]))
    rmm.check_workspaces()


@pytest.mark.parametrize("rho", [0.5, 0.9])
def test_attention_pv_wide_values(rmm, rho):
    """PV with value heads wider than 256 (no masked-V path): P's kept columns
    are packed and V's kept rows copied per query head (grouped-query V heads);
    at rho = 0.9 (k = 1080 > 1024) both in one launch, at 0.5 the narrow pack."""
    H, Hkv, n, dv = 4, 2, 1200, 320
    ks = [oracle.retained_count(r, n) for r in (0.5, 0.9)]
    (P, V), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_pv(44, n=n, heads=H, kv_heads=Hkv, v_dim=dv, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), ks)
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=rho, return_indices=True)
    torch.cuda.synchronize()
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=rho)
    assert_indices_equal(T, T_ref)
    P64, V64 = oracle.as_f64(P), oracle.as_f64(V)
    for h in range(H):
        g = oracle.kv_head_of(h, H, Hkv)
        assert_product_close(O[h], O_ref[h], np.abs(P64[h][:, T_ref[h]]), np.abs(V64[g][T_ref[h]]))
    rmm.check_workspaces()


def test_cuda_graph_capture(rmm):
    """Every kernel is launched with programmatic serialisation and the ops never
    synchronise with the host: a CUDA graph of linear (CTA-pair product with a
    split tail, and the small-n product), QK and PV calls replays to the same bits
    as the eager calls."""
    dev = torch.device("cuda")
    s = torch.cuda.Stream()
    cases = []
    A, B = W.mlp_up(51, n=300, d=4096, m=704)
    cases.append((rmm.RMM_LINEAR, A.to(dev), B.to(dev), 300, 4096, 704, 1, 1, 0.6))
    A, B = W.mlp_down(52, n=16, d=4096, m=264)
    cases.append((rmm.RMM_LINEAR, A.to(dev), B.to(dev), 16, 4096, 264, 1, 1, 0.7))
    Q, K = W.attn_qk(53, n=200, heads=4, kv_heads=2, head_dim=128)
    cases.append((rmm.RMM_QK, Q.to(dev), K.to(dev), 200, 128, 200, 4, 2, 0.5))
    P, V = W.attn_pv(54, n=264, heads=4, kv_heads=2)
    cases.append((rmm.RMM_PV, P.to(dev), V.to(dev), 264, 264, 128, 4, 2, 0.8))
    runs = []
    for mode, X, Z, n, d, m, H, Hkv, rho in cases:
        p = rmm.rmm_problem_init(mode, rmm.RMM_BF16, n, d, m)
        p.rho = rho
        if H > 1:
            p.heads, p.kv_heads = H, Hkv
            p.stride_a, p.stride_b = X.stride(0), Z.stride(0)
            p.ldy, p.stride_y = m, n * m
        if mode == rmm.RMM_QK:
            p.alpha = 1.0 / math.sqrt(d)
            p.flags = rmm.RMM_FLAG_CAUSAL
        plan = rmm.Plan(p)
        ws = rmm.workspace_for(plan, dev, s)
        Y = torch.empty((H, n, m) if H > 1 else (n, m), dtype=torch.bfloat16, device=dev)
        I = torch.empty((H, plan.k) if H > 1 else (plan.k,), dtype=torch.int32, device=dev)
        runs.append((plan, X, Z, Y, I, ws))
    call = lambda r: rmm.rmm_matmul_batched(r[0], r[1], r[2], r[3], r[4], r[5], s)
    with torch.cuda.stream(s):
        for r in runs:
            call(r)
    torch.cuda.synchronize()
    eager = [(r[3].clone(), r[4].clone()) for r in runs]
    for r in runs:
        r[3].zero_()
        r[4].zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for r in runs:
            call(r)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for (Ye, Ie), r in zip(eager, runs):
        assert torch.equal(r[4], Ie)
        assert torch.equal(r[3], Ye)
    rmm.check_workspaces()
    del g


def _qk_check(rmm, Q, K, rho, causal):
    H, n, dh = Q.shape
    alpha = 1.0 / math.sqrt(dh)
    S, I = rmm.qk(Q.cuda(), K.cuda(), rho=rho, alpha=alpha, causal=causal, return_indices=True)
    torch.cuda.synchronize()
    S_ref, I_ref = oracle.rmm_qk(Q, K, rho=rho, alpha=alpha, causal=causal)
    assert_indices_equal(I, I_ref)
    Q64, K64 = oracle.as_f64(Q), oracle.as_f64(K)
    mask = np.triu(np.ones((n, K.shape[1]), dtype=bool), 1) if causal else None
    for h in range(H):
        g = oracle.kv_head_of(h, H, K.shape[0])
        assert_product_close(S[h], S_ref[h], np.abs(Q64[h][:, I_ref[h]]), np.abs(K64[g][:, I_ref[h]]).T,
                             alpha=alpha, mask=mask)


@pytest.mark.parametrize("dh,n,H,Hkv,causal", [
    (64, 1000, 8, 2, True),    # eight CTAs per head in the selection's cluster, 125 rows each
    (96, 80, 4, 4, False),     # four CTAs; 12 column groups: 21 row groups, 4 idle threads
    (256, 520, 2, 1, True),    # eight CTAs per head, eight 32-feature words
    (128, 40, 64, 8, True),    # many heads, few rows: two CTAs per head
    (128, 24, 8, 2, False),    # one CTA per head
])
def test_qk_cluster_selection(rmm, dh, n, H, Hkv, causal):
    """The QK op's selection and masked copy of Q in one cluster launch (bf16,
    d_h <= 256): I bit-exact and S against the oracle across head dims,
    cluster sizes and ragged row ranges."""
    rhos = (0.5, 0.8)
    ks = [oracle.retained_count(r, dh) for r in rhos]
    (Q, K), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(26, n=n, heads=H, kv_heads=Hkv, head_dim=dh, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), ks)
    for rho in rhos:
        _qk_check(rmm, Q, K, rho, causal)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
def test_attention_qk(rmm, rho, causal):
    H, Hkv, n, dh = 4, 2, 200, 128
    ks = [oracle.retained_count(r, dh) for r in (0.5, 0.8)]
    (Q, K), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(21, n=n, heads=H, kv_heads=Hkv, head_dim=dh, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), ks)
    _qk_check(rmm, Q, K, rho, causal)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
def test_attention_pv(rmm, rho, causal):
    """P is a causal softmax; causal=True lets the op skip the blocks above the
    diagonal (here the second column block of the scores skips its first 256
    rows, and the first 256-row tile drops its last k-block)."""
    H, Hkv, n, dv = 4, 2, 264, 128
    ks = [oracle.retained_count(r, n) for r in (0.5, 0.8)]
    (P, V), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_pv(31, n=n, heads=H, kv_heads=Hkv, v_dim=dv, col_gain=g),
        lambda x: gap.scores_per_head(x[0]), ks)
    assert not bool(torch.triu(P.float(), 1).any())
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=rho, return_indices=True, causal=causal)
    torch.cuda.synchronize()
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=rho)
    assert_indices_equal(T, T_ref)
    P64, V64 = oracle.as_f64(P), oracle.as_f64(V)
    for h in range(H):
        g = oracle.kv_head_of(h, H, Hkv)
        assert_product_close(O[h], O_ref[h], np.abs(P64[h][:, T_ref[h]]), np.abs(V64[g][T_ref[h]]))


def test_attention_fp32(rmm):
    """fp32 attention (tf32 tensor cores): causal QK with GQA and PV."""
    H, Hkv, n, dh = 4, 2, 200, 128
    ks = [oracle.retained_count(0.5, dh)]
    (Q, K), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_qk(71, n=n, heads=H, kv_heads=Hkv, head_dim=dh, col_gain=g, dtype=torch.float32),
        lambda x: gap.scores_per_head(x[0]), ks)
    _qk_check(rmm, Q, K, 0.5, True)
    n = 264
    ks = [oracle.retained_count(0.8, n)]
    (P, V), _ = gap.enforce_boundary_gaps(
        lambda g: W.attn_pv(72, n=n, heads=H, kv_heads=Hkv, col_gain=g, dtype=torch.float32),
        lambda x: gap.scores_per_head(x[0]), ks)
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=0.8, return_indices=True)
    torch.cuda.synchronize()
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=0.8)
    assert_indices_equal(T, T_ref)
    P64, V64 = oracle.as_f64(P), oracle.as_f64(V)
    for h in range(H):
        g = oracle.kv_head_of(h, H, Hkv)
        assert_product_close(O[h], O_ref[h], np.abs(P64[h][:, T_ref[h]]), np.abs(V64[g][T_ref[h]]))


def test_bounded_wait_reports_timeout(rmm):
    """A wait that nothing completes runs out after the limit, the status word
    says so once, and the context stays usable: the next op matches the oracle."""
    import time
    n, d, m, rho = 200, 1024, 264, 0.5
    k = oracle.retained_count(rho, d)
    (A, B), _ = gap.enforce_boundary_gaps(lambda g: W.mlp_up(61, n=n, d=d, m=m, col_gain=g),
                                          lambda x: gap.scores_2d(x[0]), [k])
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, n, d, m)
    p.rho = rho
    plan = rmm.Plan(p)
    ws = rmm.workspace_for(plan)
    assert rmm.rmm_workspace_status(plan, ws) == rmm.RMM_OK
    t0 = time.monotonic()
    rmm.rmm_selftest_wait_timeout(plan, ws)
    assert rmm.rmm_workspace_status(plan, ws) == rmm.RMM_ERR_TIMEOUT
    assert time.monotonic() - t0 >= 1.5  # the wait gave up at its limit, not at once
    assert rmm.rmm_workspace_status(plan, ws) == rmm.RMM_OK  # read once, then cleared
    Ag, Bg = A.cuda(), B.cuda()
    Y = torch.empty((n, m), dtype=torch.bfloat16, device="cuda")
    I = torch.empty(plan.k, dtype=torch.int32, device="cuda")
    rmm.rmm_matmul(plan, Ag, Bg, Y, I, ws)
    assert rmm.rmm_workspace_status(plan, ws) == rmm.RMM_OK
    I_ref, _ = oracle.select(A, rho=rho)
    assert_indices_equal(I, I_ref)
    A64, B64 = oracle.as_f64(A), oracle.as_f64(B)
    assert_product_close(Y, oracle.reduced_product(A64, B64, I_ref), np.abs(A64[:, I_ref]), np.abs(B64[I_ref]))


def test_workspace_status_clean(rmm):
    A, B = W.mlp_up(12, n=64, d=512, m=64)
    Ag, Bg = A.cuda(), B.cuda()
    p = rmm.rmm_problem_init(rmm.RMM_LINEAR, rmm.RMM_BF16, 64, 512, 64)
    p.rho = 0.5
    plan = rmm.Plan(p)
    ws = rmm.workspace_for(plan)
    Y = torch.empty((64, 64), dtype=torch.bfloat16, device="cuda")
    rmm.rmm_matmul(plan, Ag, Bg, Y, None, ws)
    assert rmm.rmm_workspace_status(plan, ws) == rmm.RMM_OK
    with pytest.raises(rmm.RmmError) as e:
        rmm.rmm_matmul(plan, Ag, Bg, Y, None, ws[: plan.workspace_bytes - 1])
    assert e.value.status == rmm.RMM_ERR_WORKSPACE
    with pytest.raises(rmm.RmmError) as e:
        rmm.rmm_matmul(plan, Ag[:, 1:], Bg, Y, None, ws)  # 2-byte offset: misaligned
    assert e.value.status == rmm.RMM_ERR_INVALID_ARG


# Decode step: (batch, n, heads, kv_heads, head_dim = d_v, t).  n = 1 scores
# are squares of bf16 values, exact in fp32 and fp64 alike, so equal scores
# are ties on both sides and the lower index wins on both; n = 2 inputs get
# the usual boundary gap.
DECODE_CASES = [
    (2, 1, 32, 8, 128, 1000),  # Llama-3.1-8B grouping, t not a multiple of the tiles
    (1, 2, 32, 8, 128, 520),   # two query rows: 8 query vectors per KV head
    (1, 1, 64, 8, 128, 264),   # groups of 8 query heads
    (1, 1, 8, 4, 64, 96),      # d_h = d_v = 64, a single token range
]


def _decode_inputs(case, seed, which):
    batch, n, H, Hkv, dh, t = case
    make = lambda g: W.attn_decode(seed, t=t, batch=batch, n=n, heads=H, kv_heads=Hkv, head_dim=dh, v_dim=dh,
                                   **({which: g} if g is not None else {}))
    if n == 1:
        return make(None)
    d = dh if which == "q_gain" else t
    ks = [oracle.retained_count(r, d) for r in (0.5, 0.8)]
    idx = 0 if which == "q_gain" else 3
    out, _ = gap.enforce_boundary_gaps(make, lambda x: gap.scores_per_head(x[idx]), ks)
    return out


def _decode_qk_close(S, S_ref, I_ref, q, K, alpha):
    q64, K64 = oracle.as_f64(q), oracle.as_f64(K)
    H, Hkv = q.shape[0], K.shape[0]
    absA = [np.abs(q64[h][:, I_ref[h]]) for h in range(H)]
    absB = [np.abs(K64[oracle.kv_head_of(h, H, Hkv)][:, I_ref[h]]).T for h in range(H)]
    assert_heads_close(S, S_ref, absA, absB, alpha=alpha)


def _decode_pv_close(O, O_ref, T_ref, P, V):
    P64, V64 = oracle.as_f64(P), oracle.as_f64(V)
    H, Hkv = P.shape[0], V.shape[0]
    absA = [np.abs(P64[h][:, T_ref[h]]) for h in range(H)]
    absB = [np.abs(V64[oracle.kv_head_of(h, H, Hkv)][T_ref[h]]) for h in range(H)]
    assert_heads_close(O, O_ref, absA, absB)


def _launches(rmm, mode, X, Z, m, rho):
    H, n, d = X.shape
    p = rmm.rmm_problem_init(mode, rmm.RMM_BF16, n, d, m)
    p.rho = rho
    p.heads, p.kv_heads = H, Z.shape[0]
    p.lda, p.ldb = d, Z.shape[2]
    p.stride_a, p.stride_b = X.stride(0), Z.stride(0)
    p.ldy, p.stride_y = m, n * m
    return rmm.Plan(p).kernel_launches


@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_qk(rmm, case, rho):
    """Scores of a decode step: the group's query vectors against each K row once,
    the features selected inside the same kernel (one launch)."""
    q, K, _, _ = _decode_inputs(case, 81, "q_gain")
    H, n, dh = q.shape
    assert _launches(rmm, rmm.RMM_QK, q, K, K.shape[1], rho) == 1
    alpha = 1.0 / math.sqrt(dh)
    S, I = rmm.qk(q.cuda(), K.cuda(), rho=rho, alpha=alpha, causal=False, return_indices=True)
    torch.cuda.synchronize()
    S_ref, I_ref = oracle.rmm_qk(q, K, rho=rho, alpha=alpha, causal=False)
    assert_indices_equal(I, I_ref)
    _decode_qk_close(S, S_ref, I_ref, q, K, alpha)


def test_decode_qk_head_dim_256(rmm):
    q, K, _, _ = W.attn_decode(82, t=200, batch=1, n=1, heads=8, kv_heads=2, head_dim=256)
    S, I = rmm.qk(q.cuda(), K.cuda(), rho=0.7, alpha=0.0625, causal=False, return_indices=True)
    torch.cuda.synchronize()
    S_ref, I_ref = oracle.rmm_qk(q, K, rho=0.7, alpha=0.0625, causal=False)
    assert_indices_equal(I, I_ref)
    _decode_qk_close(S, S_ref, I_ref, q, K, 0.0625)


@pytest.mark.parametrize("rho", [0.5, 0.8, 1.0])
@pytest.mark.parametrize("case", DECODE_CASES)
def test_decode_pv(rmm, case, rho):
    """Value product of a decode step: the union of the group's kept tokens is
    read once per KV head, each weighed only for the heads that kept it."""
    _, _, V, P = _decode_inputs(case, 91, "p_gain")
    H, n, t = P.shape
    Hkv = V.shape[0]
    assert _launches(rmm, rmm.RMM_PV, P, V, V.shape[2], rho) == (1 if rho < 1 else 0) + 1
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=rho, return_indices=True)
    torch.cuda.synchronize()
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=rho)
    assert_indices_equal(T, T_ref)
    _decode_pv_close(O, O_ref, T_ref, P, V)
    O2 = rmm.pv(P.cuda(), V.cuda(), rho=rho)  # the token ranges' counters were reset
    torch.cuda.synchronize()
    assert torch.equal(O, O2)
    rmm.check_workspaces()


def test_decode_rows_past_the_group_take_the_general_path(rmm):
    """group * n > 8 query vectors per KV head: the general kernels (the
    selection with the masked copy of Q, then the product; the decode kernel
    is one launch)."""
    case = (1, 4, 8, 2, 128, 264)
    q, K, _, _ = _decode_inputs(case, 83, "q_gain")
    _, _, V, P = _decode_inputs(case, 84, "p_gain")
    assert _launches(rmm, rmm.RMM_QK, q, K, K.shape[1], 0.5) == 2
    S, I = rmm.qk(q.cuda(), K.cuda(), rho=0.5, alpha=0.1, causal=False, return_indices=True)
    O, T = rmm.pv(P.cuda(), V.cuda(), rho=0.5, return_indices=True)
    torch.cuda.synchronize()
    S_ref, I_ref = oracle.rmm_qk(q, K, rho=0.5, alpha=0.1, causal=False)
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=0.5)
    assert_indices_equal(I, I_ref)
    assert_indices_equal(T, T_ref)
    _decode_qk_close(S, S_ref, I_ref, q, K, 0.1)
    _decode_pv_close(O, O_ref, T_ref, P, V)


def test_decode_strided_views(rmm):
    """Decode ops on views with padded rows and head strides (q and the K / V
    caches 136 wide holding d_h = 128, P 8 tokens longer than t): the kernels
    use the leading dimensions and head strides they are given."""
    t, H, Hkv = 1000, 32, 8
    q, K, V, P = W.attn_decode(85, t=t, batch=1)
    dev = torch.device("cuda")
    def padded(x, extra):
        big = torch.zeros(x.shape[:-1] + (x.shape[-1] + extra,), dtype=x.dtype, device=dev)
        big[..., : x.shape[-1]] = x.to(dev)
        return big[..., : x.shape[-1]]
    qv, Kv, Vv, Pv = padded(q, 8), padded(K, 8), padded(V, 8), padded(P, 8)
    assert Kv.stride(1) == 136 and Pv.stride(0) == t + 8
    alpha = 1.0 / math.sqrt(128)
    S, I = rmm.qk(qv, Kv, rho=0.5, alpha=alpha, causal=False, return_indices=True)
    O, T = rmm.pv(Pv, Vv, rho=0.5, return_indices=True)
    torch.cuda.synchronize()
    S_ref, I_ref = oracle.rmm_qk(q, K, rho=0.5, alpha=alpha, causal=False)
    O_ref, T_ref = oracle.rmm_pv(P, V, rho=0.5)
    assert_indices_equal(I, I_ref)
    assert_indices_equal(T, T_ref)
    _decode_qk_close(S, S_ref, I_ref, q, K, alpha)
    _decode_pv_close(O, O_ref, T_ref, P, V)


def test_workspace_belongs_to_its_plan(rmm):
    """A plan's workspace is zero-initialised for that plan's layout and dies
    with it: a new plan, even one that takes a dead plan's Python id, gets its
    own workspace, and the decode PV op (whose range counters sit in the
    workspace header) still matches the oracle."""
    import gc
    q, K, V, P = W.attn_decode(86, t=1000, batch=1)
    Pg, Vg = P.cuda(), V.cuda()
    seen = []
    for rho in (0.5, 0.8, 0.5, 0.7):
        p = rmm.rmm_problem_init(rmm.RMM_PV, rmm.RMM_BF16, 1, 1000, 128)
        p.rho = rho
        p.heads, p.kv_heads = 32, 8
        p.lda, p.ldb = 1000, 128
        p.stride_a, p.stride_b = Pg.stride(0), Vg.stride(0)
        p.ldy, p.stride_y = 128, 128
        plan = rmm.Plan(p)
        ws = rmm.workspace_for(plan)
        assert all(ws is not w for w in seen)
        seen.append(ws)
        O = torch.empty((32, 1, 128), dtype=torch.bfloat16, device="cuda")
        T = torch.empty((32, plan.k), dtype=torch.int32, device="cuda")
        rmm.rmm_matmul_batched(plan, Pg, Vg, O, T, ws)
        torch.cuda.synchronize()
        O_ref, T_ref = oracle.rmm_pv(P, V, rho=rho)
        assert_indices_equal(T, T_ref)
        _decode_pv_close(O, O_ref, T_ref, P, V)
        del plan, ws
        gc.collect()
    rmm.check_workspaces()
