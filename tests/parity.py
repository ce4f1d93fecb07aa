"""Comparison helpers for GPU-vs-oracle parity (test infrastructure).

Acceptance: the index set is bit-exact; the product on that index set has a
relative Frobenius error <= 2e-3 and per element
|err| <= 1e-2 * alpha * (|A[:, I]| |B[I, :]|)_ij (bf16 inputs, fp32
accumulation; the tf32 path meets the same bounds).
"""
import numpy as np

REL_FRO = 2e-3
ELEM = 1e-2


def np64(t) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def assert_indices_equal(I_gpu, I_ref):
    g = np.asarray(I_gpu.detach().cpu().numpy() if hasattr(I_gpu, "detach") else I_gpu)
    r = np.asarray(I_ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    if not np.array_equal(g, r):
        bad = np.argwhere(g != r)
        raise AssertionError(f"index sets differ at {len(bad)} positions, first {bad[:5].tolist()}: "
                             f"gpu {g[tuple(bad[0])]} oracle {r[tuple(bad[0])]}")


def assert_product_close(Y_gpu, Y_ref, absA_I, absB_I, alpha=1.0, mask=None, rel_fro=REL_FRO):
    """Y_gpu: torch tensor; Y_ref fp64 array; absA_I (rows x k), absB_I (k x m).
    mask: boolean array of entries that must be -inf on both sides.
    rel_fro: the relative Frobenius bound (REL_FRO unless the op rounds an
    operand it computes itself, see the fused attention's tests)."""
    Yg = np64(Y_gpu)
    Yr = np.asarray(Y_ref, dtype=np.float64)
    assert Yg.shape == Yr.shape, (Yg.shape, Yr.shape)
    if mask is not None:
        assert np.all(np.isneginf(Yg[mask])), "masked entries must be -inf"
        assert np.all(np.isneginf(Yr[mask]))
        keep = ~mask
    else:
        keep = np.ones(Yr.shape, dtype=bool)
    assert np.all(np.isfinite(Yg[keep])), "non-finite values where finite ones are expected"
    err = np.where(keep, Yg - np.where(keep, Yr, 0.0), 0.0)
    ref = np.where(keep, Yr, 0.0)
    denom = max(np.linalg.norm(ref), 1e-300)
    fro = np.linalg.norm(err) / denom
    assert fro <= rel_fro, f"relative Frobenius error {fro:.3e} > {rel_fro}"
    bound = ELEM * abs(alpha) * (absA_I @ absB_I)
    over = np.abs(err) > bound + 1e-30
    if np.any(over):
        i = np.argwhere(over)[0]
        raise AssertionError(f"{int(over.sum())} elements exceed 1e-2*(|A_I||B_I|); first at "
                             f"{i.tolist()}: err {err[tuple(i)]:.3e} bound {bound[tuple(i)]:.3e}")
    return fro


def assert_heads_close(Y_gpu, Y_ref, absA_I, absB_I, alpha=1.0):
    """Batched output Y [H, n, m] against the oracle's: the relative Frobenius
    bound on the op's whole output, the element bound per head with that head's
    absA_I[h] (n x k) and absB_I[h] (k x m).  Rounding the output to bf16 alone
    costs ~1.6e-3 of relative Frobenius error on average, so a head with a few
    dozen outputs (one decode row) can exceed 2e-3 by rounding luck alone; the
    bound is therefore taken over all heads together."""
    Yg = np64(Y_gpu)
    Yr = np.asarray(Y_ref, dtype=np.float64)
    assert Yg.shape == Yr.shape, (Yg.shape, Yr.shape)
    assert np.all(np.isfinite(Yg)), "non-finite values where finite ones are expected"
    err = Yg - Yr
    fro = np.linalg.norm(err) / max(np.linalg.norm(Yr), 1e-300)
    assert fro <= REL_FRO, f"relative Frobenius error {fro:.3e} > {REL_FRO}"
    for h in range(Yr.shape[0]):
        bound = ELEM * abs(alpha) * (absA_I[h] @ absB_I[h])
        over = np.abs(err[h]) > bound + 1e-30
        if np.any(over):
            i = np.argwhere(over)[0]
            raise AssertionError(f"head {h}: {int(over.sum())} elements exceed 1e-2*(|A_I||B_I|); first at "
                                 f"{i.tolist()}: err {err[h][tuple(i)]:.3e} bound {bound[tuple(i)]:.3e}")
    return fro


def sample_rows(n: int, seed: int = 0, per_tile: int = 2, tile: int = 128):
    """Two seeded rows from every 128-row tile (all rows when n is small)."""
    rng = np.random.default_rng(seed)
    rows = []
    for t0 in range(0, n, tile):
        t1 = min(n, t0 + tile)
        c = min(per_tile, t1 - t0)
        rows.extend(sorted(rng.choice(np.arange(t0, t1), size=c, replace=False).tolist()))
    return rows
