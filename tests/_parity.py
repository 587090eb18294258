"""Shared helpers for the GPU parity tests (GPU result vs the fp64 oracle)."""
import numpy as np

# Tolerances (fixed by the target: bf16 O vs fp64 O, fp32 LSE)
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 1e-3
CUT_BAND = 1e-4


def to_device_bf16(a_u16):
    import torch
    t = torch.from_numpy(a_u16.view(np.int16)).view(torch.bfloat16)
    return t.cuda().contiguous()


def csr_to_mask(row_ptr, col_idx, nrows, nb):
    m = np.zeros((nrows, nb), dtype=np.uint8)
    for g in range(nrows):
        m[g, col_idx[row_ptr[g]:row_ptr[g + 1]]] = 1
    return m


def check_csr(row_ptr, col_idx, nrows, nb):
    """Monotone row_ptr, ascending in-range column indices, no duplicates."""
    assert row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    nnz = row_ptr[nrows]
    cols = col_idx[:nnz]
    assert np.all((cols >= 0) & (cols < nb))
    seg = np.repeat(np.arange(nrows), np.diff(row_ptr[:nrows + 1]))
    same_row = seg[1:] == seg[:-1]
    assert np.all(cols[1:][same_row] > cols[:-1][same_row]), "columns not strictly ascending"


def compare_masks(gpu_mask, ora_mask, diag, thr):
    """Mask parity: bit-exact except rows whose cut sits within CUT_BAND of
    1 - thr (or whose cut probabilities tie to 1e-6); those rows must differ
    by at most two blocks.  Returns a dict of counts: rows, rows that differ,
    near-cut rows, near-tie rows, exempt rows (either) and exempt rows that
    differ."""
    import oracle
    g = gpu_mask.reshape(-1, gpu_mask.shape[-1])
    o = ora_mask.reshape(-1, ora_mask.shape[-1])
    dg = diag.reshape(-1, 4)
    diff = (g != o).sum(axis=1)
    near_cut = oracle.near_cut_rows(dg, thr, CUT_BAND)
    near_tie = oracle.near_tie_rows(dg)
    exempt = near_cut | near_tie
    bad = (diff > 0) & ~exempt
    assert not bad.any(), (f"{bad.sum()} non-exempt rows differ; first {np.nonzero(bad)[0][:5]}, "
                           f"diff counts {diff[bad][:5]}")
    assert diff[exempt].max(initial=0) <= 2
    return {"rows": int(g.shape[0]), "rows_differing": int((diff > 0).sum()),
            "near_cut": int(near_cut.sum()), "near_tie": int(near_tie.sum()),
            "exempt": int(exempt.sum()), "exempt_differing": int(((diff > 0) & exempt).sum())}


def compare_attention(o_gpu, lse_gpu, o_ref, lse_ref):
    """o_gpu: [n, d] float; o_ref: [n, d] fp64; LSE may contain -inf (empty rows)."""
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    assert np.isfinite(o_gpu).all()
    assert err.max() <= O_MAX_ABS, f"max-abs {err.max():.3g}"
    assert err.mean() <= O_MEAN_ABS, f"mean-abs {err.mean():.3g}"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin)
    if fin.any():
        lerr = np.abs(lse_gpu[fin].astype(np.float64) - lse_ref[fin])
        assert lerr.max() <= LSE_ABS, f"LSE max-abs {lerr.max():.3g}"
    return float(err.max()), float(err.mean())


def sample_rows(B, H, S, nblocks_per_head, rows_per_block, seed=0):
    """Global row ids: every head x a seeded sample of query blocks (always
    including the first and last block) x a sample of rows inside each."""
    rng = np.random.default_rng(seed)
    nb = S // 64
    out = []
    for bh in range(B * H):
        blocks = set(rng.choice(nb, size=min(nblocks_per_head, nb), replace=False).tolist())
        blocks |= {0, nb - 1}
        for r in sorted(blocks):
            rows = rng.choice(64, size=min(rows_per_block, 64), replace=False)
            out.extend((bh * S + r * 64 + rows).tolist())
    return np.array(sorted(out), dtype=np.int64)


def rows_with_same_mask(rows, gpu_mask, ora_mask, S, min_frac=0.95):
    """The oracle computes attention with its own mask only; the GPU layer ran
    with the GPU's mask.  Keep the sampled rows whose query block has the same
    mask row on both sides (the rest differ only at near-cut rows, which the
    mask tests check) and require that most of them do."""
    nb = S // 64
    g = gpu_mask.reshape(-1, nb)
    o = ora_mask.reshape(-1, nb)
    same = (g == o).all(axis=1)
    blk = (rows // S) * nb + (rows % S) // 64
    keep = same[blk]
    assert keep.mean() >= min_frac, f"only {keep.mean():.3f} of sampled rows share a mask row"
    return rows[keep]
