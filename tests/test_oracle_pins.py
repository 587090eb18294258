"""Pins for the fp64 oracle against facts fixed outside the oracle itself.

Each test checks the oracle against something other than its own formulas:
closed forms (the geometric-decay row model of the NABLA paper's Appendix C),
hand-computed two-block reduced maps (tests/golden/two_block_cases.txt),
library routines (numpy means, scipy softmax, torch fp64 attention), and
invariants the selection rule must satisfy.  A dropped term, wrong sign,
wrong index or transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x):
    """float array -> bf16 bit patterns, exact for bf16-representable values."""
    x = np.asarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def _rand_bits(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    u = x.view(np.uint32)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- pooling, logits, softmax

def test_pool_matches_numpy_mean(oracle_mod):
    rng = np.random.default_rng(1)
    x = _rand_bits(rng, (2, 3, 256, 16))
    got = oracle_mod.pool(x)
    want = _f(x).reshape(2, 3, 4, 64, 16).mean(axis=3)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)


def test_pool_constant_blocks_exact(oracle_mod):
    vals = np.array([0.5, -3.0, 1.25, 7.0], dtype=np.float32)
    x = np.repeat(vals, 64)[:, None] * np.ones((1, 8), dtype=np.float32)
    got = oracle_mod.pool(_bf16_bits(x))
    assert got.shape == (4, 8)
    assert np.array_equal(got, np.repeat(vals.astype(np.float64)[:, None], 8, axis=1))


def test_pool_block_boundaries(oracle_mod):
    # a single nonzero token at position 64*b + t only moves block b's mean
    x = np.zeros((256, 4), dtype=np.float32)
    x[64 * 2 + 63, 1] = 64.0
    got = oracle_mod.pool(_bf16_bits(x))
    want = np.zeros((4, 4))
    want[2, 1] = 1.0
    assert np.array_equal(got, want)


def test_logits_hand_computed(oracle_mod):
    qbar = np.array([[1.0, 2.0], [0.0, 1.0]])
    kbar = np.array([[3.0, 0.0], [1.0, 1.0]])
    got = oracle_mod.logits(qbar, kbar)
    # rows: q0.k0 = 3, q0.k1 = 3, q1.k0 = 0, q1.k1 = 1; scaled by 1/sqrt(2)
    want = np.array([[3.0, 3.0], [0.0, 1.0]]) / math.sqrt(2.0)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # asymmetric operands: transposing them changes the answer
    assert not np.allclose(oracle_mod.logits(kbar, qbar), got)


def test_softmax_matches_scipy(oracle_mod):
    from scipy.special import softmax
    rng = np.random.default_rng(2)
    for n in (1, 2, 17, 1200):
        L = rng.standard_normal(n) * 5 + 300.0   # large offset: max subtraction needed
        np.testing.assert_allclose(oracle_mod.softmax_row(L), softmax(L), rtol=1e-12, atol=0)


# ---------------------------------------------------------------- selection rule

def _geometric_count(rho, n, thr):
    """Closed form for the geometric-decay row p_j = (1-rho) rho^(j-1) / (1-rho^n):
    mass of the top r is (1-rho^r)/(1-rho^n); the smallest r with mass >= 1-thr
    is ceil(log(1 - (1-thr)(1-rho^n)) / log(rho))."""
    if thr <= 0:
        return n
    x = math.log(1.0 - (1.0 - thr) * (1.0 - rho ** n)) / math.log(rho)
    return max(1, min(n, math.ceil(x - 1e-12)))


@pytest.mark.parametrize("rho", [0.5, 0.8, 0.9, 0.97, 0.995])
@pytest.mark.parametrize("n", [16, 128, 1200])
@pytest.mark.parametrize("thr", [0.2, 0.4, 0.7])
def test_row_select_geometric_closed_form(oracle_mod, rho, n, thr):
    j = np.arange(n, dtype=np.float64)
    p = (1 - rho) * rho ** j / (1 - rho ** n)
    x = math.log(1.0 - (1.0 - thr) * (1.0 - rho ** n)) / math.log(rho)
    if abs(x - round(x)) < 1e-6:
        pytest.skip("cut falls on an exact boundary")
    want = _geometric_count(rho, n, thr)
    rng = np.random.default_rng(n)
    perm = rng.permutation(n)
    pp = np.empty(n)
    pp[perm] = p          # block perm[j] holds the j-th largest probability
    keep, cnt, _ = oracle_mod.row_select(pp, thr)
    assert cnt == want
    assert keep.sum() == want
    assert set(np.nonzero(keep)[0]) == set(perm[:want])


def test_row_select_two_block_golden(oracle_mod):
    path = os.path.join(GOLDEN, "two_block_cases.txt")
    n_cases = 0
    for line in open(path):
        if not line.strip() or line.startswith("#"):
            continue
        a, e0, e1, probs = [s.split() for s in line.split("|")]
        q0, q1, k0, k1, thr = map(float, a)
        x = np.zeros((128, 64), dtype=np.float32)
        x[:64, 0], x[64:, 0] = q0, q1
        y = np.zeros((128, 64), dtype=np.float32)
        y[:64, 0], y[64:, 0] = k0, k1
        q = _bf16_bits(x)[None, None]
        k = _bf16_bits(y)[None, None]
        mask = oracle_mod.build_mask(q, k, (1, 1, 2), thr, None)
        assert mask[0, 0, 0].tolist() == [int(t) for t in e0], line
        assert mask[0, 0, 1].tolist() == [int(t) for t in e1], line
        # the pooled map itself: p[0][0] and p[1][1]
        qb, kb = oracle_mod.pool(q[0, 0]), oracle_mod.pool(k[0, 0])
        L = oracle_mod.logits(qb, kb)
        p0, p1 = oracle_mod.softmax_row(L[0]), oracle_mod.softmax_row(L[1])
        assert abs(p0[0] - float(probs[0])) < 1e-12 and abs(p1[1] - float(probs[1])) < 1e-12
        n_cases += 1
    assert n_cases >= 10


def test_row_select_ties_go_to_lower_index(oracle_mod):
    p = np.full(8, 1.0 / 8)           # exact in binary: E_k = k/8
    keep, cnt, _ = oracle_mod.row_select(p, 0.5)
    assert cnt == 4 and keep.tolist() == [1, 1, 1, 1, 0, 0, 0, 0]
    keep, cnt, _ = oracle_mod.row_select(p, 0.3)   # k/8 < 0.7 -> k <= 5
    assert cnt == 6 and keep.tolist() == [1, 1, 1, 1, 1, 1, 0, 0]


def test_row_select_invariants_random(oracle_mod):
    rng = np.random.default_rng(3)
    for trial in range(300):
        n = int(rng.integers(1, 300))
        alpha = float(rng.choice([0.05, 0.3, 1.0, 5.0]))
        p = rng.dirichlet(np.full(n, alpha))
        thr = float(rng.choice([0.0, 0.05, 0.2, 0.4, 0.7, 0.95, 1.0]))
        keep, cnt, diag = oracle_mod.row_select(p, thr)
        kept = np.nonzero(keep)[0]
        assert cnt == kept.size >= 1
        assert keep[np.argmax(p)] == 1                          # argmax always kept
        mass = p[kept].sum()
        if thr <= 0:
            assert cnt == n
            continue
        assert mass >= (1 - thr) - 1e-12 or cnt == n            # enough mass kept
        smallest = kept[np.argmin(p[kept])]
        if cnt > 1:                                              # minimal prefix
            assert mass - p[smallest] < (1 - thr) + 1e-12
        # kept blocks dominate dropped ones
        dropped = np.nonzero(keep == 0)[0]
        if dropped.size:
            assert p[kept].min() >= p[dropped].max()
        # diagnostics are consistent with the kept set
        assert abs(diag[1] - mass) < 1e-9 and abs(diag[0] - (mass - diag[2])) < 1e-9


def test_row_select_monotone_in_thr(oracle_mod):
    rng = np.random.default_rng(4)
    for _ in range(50):
        p = rng.dirichlet(np.full(64, 0.5))
        counts = [oracle_mod.row_select(p, t)[1] for t in (0.0, 0.1, 0.2, 0.4, 0.7, 0.9, 1.0)]
        assert all(a >= b for a, b in zip(counts, counts[1:]))
        assert counts[0] == 64 and counts[-1] == 1



# ---------------------------------------------------------------- diagnostics and exemptions
# The GPU/oracle mask comparison forgives a differing row only when the
# oracle's own diagnostics put its cut inside the rounding band: E_{k*} or
# E_{k*+1} within 1e-4 of 1 - thr ("near-cut"), or the probabilities at sorted
# positions k* and k*+1 equal to 1e-6 relative ("near-tie").  These pins fix
# what diag holds and what both predicates accept, on hand-built values.

def test_row_select_diag_four_blocks(oracle_mod):
    # p = (1, 8, 4, 3)/16, all exact in binary; sorted: 8/16 (block 1),
    # 4/16 (block 2), 3/16 (block 3), 1/16 (block 0)
    p = np.array([1.0, 8.0, 4.0, 3.0]) / 16.0
    # thr 0.4: E_0 = 0 and E_1 = 1/2 lie below 0.6, E_2 = 3/4 does not -> k* = 1
    keep, cnt, diag = oracle_mod.row_select(p, 0.4)
    assert keep.tolist() == [0, 1, 1, 0] and cnt == 2
    assert diag.tolist() == [0.5, 0.75, 0.25, 0.1875]
    # thr 1: only the first sorted block (k = 0 rule) -> k* = 0
    keep, cnt, diag = oracle_mod.row_select(p, 1.0)
    assert keep.tolist() == [0, 1, 0, 0] and diag.tolist() == [0.0, 0.5, 0.5, 0.25]
    # thr 0.01: every exclusive prefix (at most 15/16) stays below 0.99 -> all
    # kept, k* = 3 is the last position and diag[3] = -1 (no k*+1)
    keep, cnt, diag = oracle_mod.row_select(p, 0.01)
    assert cnt == 4 and diag.tolist() == [0.9375, 1.0, 0.0625, -1.0]
    # thr 0 keeps all by rule
    keep, cnt, diag = oracle_mod.row_select(p, 0.0)
    assert cnt == 4 and diag[3] == -1.0


def _diag(e0, e1, a=0.3, b=0.1):
    return np.array([e0, e1, a, b], dtype=np.float64)


def test_near_cut_band_edges(oracle_mod):
    nc = oracle_mod.near_cut_rows
    t = 0.8                                               # thr 0.2
    # E_{k*} just inside / just outside the band below the target
    assert nc(_diag(t - 0.99e-4, 0.95), 0.2)
    assert not nc(_diag(t - 1.01e-4, 0.95), 0.2)
    # E_{k*+1} just inside / just outside above it
    assert nc(_diag(0.5, t + 0.99e-4), 0.2)
    assert not nc(_diag(0.5, t + 1.01e-4), 0.2)
    # both far: no exemption
    assert not nc(_diag(0.5, 0.95), 0.2)
    # the target is 1 - thr, not thr
    assert not nc(_diag(0.3, 0.9), 0.3) and nc(_diag(0.7 - 5e-5, 0.9), 0.3)
    # the band is absolute mass: 0.9e-4 from the target is inside at target
    # 0.8 and at 0.5 (a relative band would put it outside at both)
    assert nc(_diag(0.8 - 0.9e-4, 0.95), 0.2) and nc(_diag(0.5 - 0.9e-4, 0.95), 0.5)
    # a wider band is honoured
    assert nc(_diag(t - 1.01e-4, 0.95), 0.2, band=1e-3)
    # thr = 0 keeps every block: nothing is near a cut
    assert not nc(_diag(1.0, 1.0), 0.0) and not nc(_diag(1.0 - 1e-9, 1.0), 0.0)
    # shape: one flag per row, batched over leading axes
    d = np.stack([_diag(t - 1e-5, 0.95), _diag(0.1, 0.95)] * 3).reshape(2, 3, 4)
    got = nc(d, 0.2)
    assert got.shape == (2, 3) and got.tolist() == [[True, False, True], [False, True, False]]


def test_near_tie_band_edges(oracle_mod):
    nt = oracle_mod.near_tie_rows
    a = 0.25
    assert nt(_diag(0, 0, a, a * (1 - 0.99e-6)))
    assert not nt(_diag(0, 0, a, a * (1 - 1.01e-6)))
    # relative, not absolute: 1e-8 vs 0.5e-8 differ by 5e-9 (under 1e-6
    # absolute) but by half of themselves
    assert not nt(_diag(0, 0, 1e-8, 0.5e-8))
    assert nt(_diag(0, 0, 1e-8, 1e-8 * (1 - 0.5e-6)))
    # no position k*+1 (every block kept): b = -1 never ties
    assert not nt(_diag(0, 0, 0.5, -1.0)) and not nt(_diag(0, 0, 1e-300, -1.0))
    # exact ties, including two zero probabilities
    assert nt(_diag(0, 0, 0.125, 0.125)) and nt(_diag(0, 0, 0.0, 0.0))
    got = nt(np.stack([_diag(0, 0, a, a), _diag(0, 0, a, 0.5 * a)]).reshape(1, 2, 4))
    assert got.shape == (1, 2) and got.tolist() == [[True, False]]


def test_exemptions_from_row_select_diagnostics(oracle_mod):
    """The predicates applied to the oracle's own diagnostics of crafted rows."""
    nc, nt = oracle_mod.near_cut_rows, oracle_mod.near_tie_rows
    # thr 0.2 (target 0.8): sorted masses 0.5, 0.29995, 0.20005 -> E_2 = 0.79995
    # stays below the target, k* = 2, E_{k*} 5e-5 from the target
    keep, cnt, diag = oracle_mod.row_select(np.array([0.20005, 0.5, 0.29995]), 0.2)
    assert cnt == 3 and nc(diag, 0.2) and not nt(diag)
    # 0.29985: E_2 = 0.79985 is 1.5e-4 away and E_3 = 1 far: not near the cut
    keep, cnt, diag = oracle_mod.row_select(np.array([0.20015, 0.5, 0.29985]), 0.2)
    assert cnt == 3 and not nc(diag, 0.2)
    # thr 0.4 (target 0.6): 0.4, 0.3 + e, 0.3 - e -> k* = 1; the cut separates
    # 0.3 + e from 0.3 - e, a relative gap of 2e/0.3
    for e, tie in [(1e-7, True), (2e-7, False)]:
        keep, cnt, diag = oracle_mod.row_select(np.array([0.3 - e, 0.4, 0.3 + e]), 0.4)
        assert keep.tolist() == [0, 1, 1] and not nc(diag, 0.4)
        assert bool(nt(diag)) == tie


# ---------------------------------------------------------------- STA window

def _clipped(c, w, T):
    return min(c + w, T - 1) - max(c - w, 0) + 1


@pytest.mark.parametrize("grid,window", [((2, 8, 8), (1, 1, 1)), ((5, 12, 20), (1, 2, 2)),
                                         ((3, 4, 5), (0, 0, 0)), ((4, 4, 4), (5, 5, 5))])
def test_sta_window_counts(oracle_mod, grid, window):
    Tt, Th, Tw = grid
    for r in range(Tt * Th * Tw):
        row = oracle_mod.sta_row(r, grid, window)
        rt, rh, rw = r // (Th * Tw), (r // Tw) % Th, r % Tw
        want = (_clipped(rt, window[0], Tt) * _clipped(rh, window[1], Th) *
                _clipped(rw, window[2], Tw))
        assert row.sum() == want
        assert row[r] == 1
    if grid == (5, 12, 20):
        interior = (2 * 12 + 6) * 20 + 10
        assert oracle_mod.sta_row(interior, grid, window).sum() == 3 * 5 * 5


def test_sta_window_membership_brute_force(oracle_mod):
    grid, window = (3, 5, 4), (1, 2, 1)
    Tt, Th, Tw = grid
    coords = [(t, h, w) for t in range(Tt) for h in range(Th) for w in range(Tw)]
    for r, (a, b, c) in enumerate(coords):
        row = oracle_mod.sta_row(r, grid, window)
        for j, (x, y, z) in enumerate(coords):
            inside = abs(x - a) <= 1 and abs(y - b) <= 2 and abs(z - c) <= 1
            assert row[j] == inside


# ---------------------------------------------------------------- full mask builder

def test_build_mask_geometric_pipeline(oracle_mod):
    """Pooled logits L[r][c] = -(c) * delta for every query block: each row is
    exactly the geometric model with rho = exp(-delta)."""
    nb, d, delta = 32, 64, 0.125
    x = np.zeros((nb * 64, d), dtype=np.float32)
    x[:, 0] = 8.0                                  # qbar = 8 e0, sqrt(d) = 8
    y = np.zeros((nb * 64, d), dtype=np.float32)
    y[:, 0] = np.repeat(-delta * np.arange(nb), 64)
    q, k = _bf16_bits(x)[None, None], _bf16_bits(y)[None, None]
    rho = math.exp(-delta)
    for thr in (0.2, 0.4, 0.7):
        mask = oracle_mod.build_mask(q, k, (2, 4, 4), thr, None)
        want = _geometric_count(rho, nb, thr)
        assert (mask[0, 0].sum(axis=1) == want).all()
        assert (mask[0, 0][:, :want] == 1).all() and (mask[0, 0][:, want:] == 0).all()


def test_build_mask_invariants_tiny(oracle_mod, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, _ = synth_mod.make_qkv(w)
    # thr = 0 keeps every block
    assert oracle_mod.build_mask(q, k, w.tile_grid, 0.0, None).min() == 1
    # STA OR gives a superset, and contains the window
    m0 = oracle_mod.build_mask(q, k, w.tile_grid, 0.7, None)
    m1 = oracle_mod.build_mask(q, k, w.tile_grid, 0.7, (1, 1, 1))
    assert (m1 >= m0).all() and (m1.sum() > m0.sum())
    for r in range(w.nb):
        assert (m1[0, 0, r] >= oracle_mod.sta_row(r, w.tile_grid, (1, 1, 1))).all()
    # monotone in thr
    m2 = oracle_mod.build_mask(q, k, w.tile_grid, 0.4, None)
    m3 = oracle_mod.build_mask(q, k, w.tile_grid, 0.2, None)
    assert (m3 >= m2).all() and (m2 >= m0).all()
    # argmax and kept mass, from an independent numpy reduced map
    qb = _f(q).reshape(1, 2, w.nb, 64, 64).mean(axis=3)
    kb = _f(k).reshape(1, 2, w.nb, 64, 64).mean(axis=3)
    L = qb @ np.swapaxes(kb, -1, -2) / 8.0
    P = np.exp(L - L.max(-1, keepdims=True))
    P /= P.sum(-1, keepdims=True)
    mask, diag, counts = oracle_mod.build_mask(q, k, w.tile_grid, 0.2, None, with_diag=True)
    assert (np.take_along_axis(mask, P.argmax(-1)[..., None], -1) == 1).all()
    assert ((P * mask).sum(-1) >= 0.8 - 1e-12).all()


def test_build_mask_key_permutation_invariance(oracle_mod):
    """Permuting key blocks permutes mask columns (no STA, no ties)."""
    rng = np.random.default_rng(5)
    nb, d = 16, 32
    q = _rand_bits(rng, (1, 1, nb * 64, d), 2.0)
    k = _rand_bits(rng, (1, 1, nb * 64, d), 2.0)
    perm = rng.permutation(nb)
    kp = k.reshape(1, 1, nb, 64, d)[:, :, perm].reshape(1, 1, nb * 64, d)
    m = oracle_mod.build_mask(q, k, (1, 4, 4), 0.3, None)
    mp = oracle_mod.build_mask(q, kp, (1, 4, 4), 0.3, None)
    assert np.array_equal(mp[0, 0], m[0, 0][:, perm])


# ---------------------------------------------------------------- attention

def _torch_ref(q, k, v, mask_tok, scale):
    import torch
    Q = torch.from_numpy(_f(q))
    K = torch.from_numpy(_f(k))
    V = torch.from_numpy(_f(v))
    s = (Q @ K.transpose(-1, -2)) * scale
    s = s.masked_fill(~torch.from_numpy(mask_tok), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    o = torch.softmax(s, dim=-1) @ V
    return o.numpy(), lse.numpy()


def test_dense_attention_matches_torch_sdpa(oracle_mod):
    import torch
    rng = np.random.default_rng(6)
    q = _rand_bits(rng, (1, 2, 192, 32))
    k = _rand_bits(rng, (1, 2, 192, 32))
    v = _rand_bits(rng, (1, 2, 192, 32))
    O, lse = oracle_mod.dense_attention(q, k, v)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(_f(q)), torch.from_numpy(_f(k)), torch.from_numpy(_f(v)))
    np.testing.assert_allclose(O, ref.numpy().reshape(-1, 32), rtol=0, atol=1e-12)
    # all-ones block mask reproduces dense attention
    ones = np.ones((1, 2, 3, 3), dtype=np.uint8)
    O2, lse2 = oracle_mod.masked_attention(q, k, v, ones)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


def test_masked_attention_matches_torch_masked(oracle_mod):
    rng = np.random.default_rng(7)
    B, H, S, d, nb = 1, 3, 256, 64, 4
    q, k, v = (_rand_bits(rng, (B, H, S, d)) for _ in range(3))
    mask = (rng.random((B, H, nb, nb)) < 0.5).astype(np.uint8)
    mask[..., np.arange(nb), np.arange(nb)] = 1
    scale = 0.17
    O, lse = oracle_mod.masked_attention(q, k, v, mask, scale=scale)
    tok = np.repeat(np.repeat(mask.astype(bool), 64, axis=2), 64, axis=3)
    ro, rl = _torch_ref(q, k, v, tok, scale)
    np.testing.assert_allclose(O, ro.reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl.reshape(-1), rtol=0, atol=1e-12)


def test_single_block_rows_and_empty_rows(oracle_mod):
    import torch
    rng = np.random.default_rng(8)
    S, d, nb = 192, 16, 3
    q, k, v = (_rand_bits(rng, (1, 1, S, d)) for _ in range(3))
    mask = np.zeros((1, 1, nb, nb), dtype=np.uint8)
    mask[0, 0, 0, 2] = 1        # query block 0 sees only key block 2
    mask[0, 0, 1, 1] = 1        # query block 1 sees only itself
    # query block 2 sees nothing
    O, lse = oracle_mod.masked_attention(q, k, v, mask)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(_f(q[0, 0, :64])), torch.from_numpy(_f(k[0, 0, 128:])),
        torch.from_numpy(_f(v[0, 0, 128:])))
    np.testing.assert_allclose(O[:64], ref.numpy(), atol=1e-12, rtol=0)
    assert np.all(O[128:] == 0.0) and np.all(np.isneginf(lse[128:]))


def test_thr0_mask_reproduces_full_attention(oracle_mod, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, v = synth_mod.make_qkv(w)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, 0.0, None)
    rows = np.arange(0, w.H * w.S, 37, dtype=np.int64)
    O1, l1 = oracle_mod.masked_attention(q, k, v, mask, rows)
    O2, l2 = oracle_mod.dense_attention(q, k, v, rows)
    np.testing.assert_allclose(O1, O2, atol=1e-13, rtol=0)
    np.testing.assert_allclose(l1, l2, atol=1e-13, rtol=0)


# ---------------------------------------------------------------- fixed top-k rule

def test_topk_keeps_k_largest_with_lower_index_ties(oracle_mod):
    rng = np.random.default_rng(11)
    for trial in range(200):
        n = int(rng.integers(1, 200))
        k = int(rng.integers(1, n + 5))
        p = rng.dirichlet(np.full(n, 0.5))
        if trial % 5 == 0:                      # force ties
            p = np.round(p * 8) / 8
        keep, cnt = oracle_mod.row_select_topk(p, k)
        assert cnt == min(k, n) == keep.sum()
        order = sorted(range(n), key=lambda c: (-p[c], c))   # independent ordering
        assert set(np.nonzero(keep)[0]) == set(order[:min(k, n)])


def test_topk_matches_mass_rule_at_its_own_count(oracle_mod):
    """At k = the mass rule's kept count both rules keep the same blocks."""
    rng = np.random.default_rng(12)
    for _ in range(100):
        p = rng.dirichlet(np.full(int(rng.integers(2, 120)), 0.3))
        keep_m, cnt, _ = oracle_mod.row_select(p, 0.3)
        keep_t, cnt_t = oracle_mod.row_select_topk(p, cnt)
        assert cnt_t == cnt and np.array_equal(keep_m, keep_t)


def test_topk_geometric_pipeline(oracle_mod):
    nb, d, delta = 32, 64, 0.125
    x = np.zeros((nb * 64, d), dtype=np.float32)
    x[:, 0] = 8.0
    y = np.zeros((nb * 64, d), dtype=np.float32)
    y[:, 0] = np.repeat(-delta * np.arange(nb), 64)
    q, k = _bf16_bits(x)[None, None], _bf16_bits(y)[None, None]
    for topk in (1, 5, 32, 40):
        mask = oracle_mod.build_mask(q, k, (2, 4, 4), 0.2, None, topk=topk)
        kk = min(topk, nb)
        assert (mask[0, 0][:, :kk] == 1).all() and (mask[0, 0][:, kk:] == 0).all()


# ---------------------------------------------------------------------------
# Token reordering (NABLA review, Figure 4: each attention block becomes one
# 4x4x4 spatial-temporal patch of the token grid).


def _coord_rows(T, H, W, d):
    """Raster-ordered rows whose first three channels hold (t, h, w) exactly."""
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    rows = np.zeros((T * H * W, d), dtype=np.float32)
    rows[:, 0], rows[:, 1], rows[:, 2] = t.ravel(), h.ravel(), w.ravel()
    rows[:, 3:] = np.arange(d - 3, dtype=np.float32)  # integers < 256: exact in bf16
    return (rows.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("grid", [(1, 1, 1), (2, 3, 1), (3, 2, 5)])
def test_reorder_matches_numpy_axis_permutation(oracle_mod, grid):
    # Tile-major order is the raster grid reshaped to (Tt,4,Th,4,Tw,4) with the
    # tile axes moved in front of the in-tile axes: a numpy transpose.
    Tt, Th, Tw = grid
    d = 8
    x = _coord_rows(4 * Tt, 4 * Th, 4 * Tw, d)
    y = oracle_mod.reorder(x, grid, to_tile_major=True)
    ref = x.reshape(Tt, 4, Th, 4, Tw, 4, d).transpose(0, 2, 4, 1, 3, 5, 6).reshape(-1, d)
    assert np.array_equal(y, ref)
    back = oracle_mod.reorder(y, grid, to_tile_major=False)
    assert np.array_equal(back, x)


def test_reorder_tiles_are_local_patches(oracle_mod):
    # Every 64-row block after the reorder spans exactly a 4x4x4 patch whose
    # corner is a multiple of 4 along each axis.
    grid = (2, 3, 2)
    x = _coord_rows(8, 12, 8, 8)
    y = oracle_mod.reorder(x, grid, to_tile_major=True)
    c = (y[:, :3].astype(np.uint32) << 16).view(np.float32).astype(np.int64)
    for b in range(y.shape[0] // 64):
        blk = c[b * 64:(b + 1) * 64]
        lo = blk.min(axis=0)
        assert np.all(lo % 4 == 0)
        assert np.all(blk.max(axis=0) - lo == 3)
        assert len({tuple(r) for r in blk}) == 64


def test_reorder_agrees_with_synth_tile_major_positions(oracle_mod, synth_mod):
    # The seeded generator lays tokens out tile-major; its noise-free tensor
    # must equal the raster-ordered embedding moved by the oracle's reorder.
    grid = (2, 2, 3)
    Tt, Th, Tw = grid
    d = 24
    S = 64 * Tt * Th * Tw
    tm = synth_mod.make_tensor(0, 5, 1, 1, S, d, grid=grid, pos_weight=1.0, noise_weight=0.0)
    T, H, W = 4 * Tt, 4 * Th, 4 * Tw
    raster = np.empty((S, d), dtype=np.float64)
    for t in range(T):
        for h in range(H):
            for w in range(W):
                raster[(t * H + h) * W + w] = synth_mod.embedding(d, t, h, w)
    to_bf16 = np.vectorize(lambda v: int(synth_mod.lib().synth_f64_to_bf16(float(v))))
    raster_bits = to_bf16(raster).astype(np.uint16)
    moved = oracle_mod.reorder(raster_bits.reshape(1, 1, S, d), grid, to_tile_major=True)
    assert np.array_equal(moved.reshape(S, d), tm.reshape(S, d))


def test_reorder_batched_heads_independent(oracle_mod):
    rng = np.random.default_rng(3)
    grid = (1, 2, 2)
    x = rng.integers(0, 1 << 16, size=(2, 3, 64 * 4, 16), dtype=np.uint16)
    y = oracle_mod.reorder(x, grid)
    for b in range(2):
        for h in range(3):
            assert np.array_equal(y[b, h], oracle_mod.reorder(x[b, h], grid))


# ---------------------------------------------------------------------------
# Block energy (CalibAtt's per-block energy; the NABLA review's true block mass)


def _torch_block_energy(q, k, scale=None):
    """fp64 torch: dense softmax of the score matrix, summed over 64 x 64 blocks
    and divided by 64 (mean over the block's queries)."""
    import torch
    B, H, S, d = q.shape
    nb = S // 64
    qf = torch.from_numpy(_f(q))
    kf = torch.from_numpy(_f(k))
    s = torch.einsum("bhid,bhjd->bhij", qf, kf) * (scale if scale else 1.0 / math.sqrt(d))
    p = torch.softmax(s, dim=-1)
    e = p.reshape(B, H, nb, 64, nb, 64).sum(dim=(3, 5)) / 64.0
    lse = torch.logsumexp(s, dim=-1)
    return e.numpy(), lse.numpy()


def test_block_energy_matches_torch_dense_softmax(oracle_mod):
    rng = np.random.default_rng(21)
    B, H, S, d = 1, 2, 256, 64
    q = _rand_bits(rng, (B, H, S, d), 0.6)
    k = _rand_bits(rng, (B, H, S, d), 0.6)
    want, lse = _torch_block_energy(q, k)
    full = np.ones((B, H, S // 64, S // 64), dtype=np.uint8)
    got, mass = oracle_mod.block_energy(q, k, lse, full)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(mass, 1.0, rtol=0, atol=1e-12)
    # the block map is not symmetric in (r, c): a transposed index would show
    assert np.abs(want - np.swapaxes(want, -1, -2)).max() > 1e-3
    # a row subset returns the same rows
    rows = np.array([3, 0, 6], dtype=np.int64)
    sub, smass = oracle_mod.block_energy(q, k, lse, full, rows=rows)
    np.testing.assert_array_equal(sub, got.reshape(-1, S // 64)[rows])
    np.testing.assert_array_equal(smass, mass.reshape(-1)[rows])


def test_block_energy_rows_sum_to_one_with_dense_lse(oracle_mod, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, v = synth_mod.make_qkv(w)
    _, lse = oracle_mod.dense_attention(q, k, v)
    full = np.ones((w.B, w.H, w.nb, w.nb), dtype=np.uint8)
    E, mass = oracle_mod.block_energy(q, k, lse.reshape(w.B, w.H, w.S), full)
    np.testing.assert_allclose(E.sum(axis=-1), 1.0, atol=1e-12)
    np.testing.assert_allclose(mass, 1.0, atol=1e-12)
    assert (E > 0).all()


def test_block_energy_uniform_attention_closed_form(oracle_mod):
    # q = 0: every score is 0, LSE = ln S, and each block holds 64*64/S of the
    # mass of its 64 queries: E = 64/S = 1/nb at listed blocks, 0 elsewhere.
    rng = np.random.default_rng(4)
    B, H, S, d = 1, 1, 512, 64
    nb = S // 64
    q = np.zeros((B, H, S, d), dtype=np.uint16)
    k = _rand_bits(rng, (B, H, S, d))
    lse = np.full((B, H, S), math.log(S))
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    E, mass = oracle_mod.block_energy(q, k, lse, mask)
    np.testing.assert_allclose(E, mask / nb, rtol=1e-14, atol=0)
    np.testing.assert_allclose(mass, mask.sum(-1) / nb, rtol=1e-14)


def test_block_energy_nonfinite_lse_rows_contribute_nothing(oracle_mod):
    rng = np.random.default_rng(5)
    B, H, S, d = 1, 1, 256, 64
    q = _rand_bits(rng, (B, H, S, d))
    k = _rand_bits(rng, (B, H, S, d))
    want, lse = _torch_block_energy(q, k)
    lse = lse.copy()
    lse[0, 0, 64:128] = -np.inf          # query block 1 has no kept key
    lse[0, 0, 130] = np.nan              # and one row of block 2 is undefined
    full = np.ones((B, H, 4, 4), dtype=np.uint8)
    E, _ = oracle_mod.block_energy(q, k, lse, full)
    assert (E[0, 0, 1] == 0).all()
    np.testing.assert_allclose(E[0, 0, [0, 3]], want[0, 0, [0, 3]], rtol=1e-10)
    assert (E[0, 0, 2] < want[0, 0, 2]).all()


# ---------------------------------------------------------------------------
# Calibration (CalibAtt, Methodology A: threshold per row, aggregate over runs)


@pytest.mark.parametrize("rho,eps", [(0.8, 0.2), (0.9, 0.4), (0.97, 0.1)])
def test_calib_geometric_energy_closed_form(oracle_mod, rho, eps):
    # an energy row proportional to rho^c (any positive scale) keeps the
    # closed-form count of the geometric model, at the largest blocks
    n = 96
    x = math.log(1.0 - (1.0 - eps) * (1.0 - rho ** n)) / math.log(rho)
    assert abs(x - round(x)) > 1e-6
    want = _geometric_count(rho, n, eps)
    rng = np.random.default_rng(9)
    perm = rng.permutation(n)
    row = np.empty(n)
    row[perm] = 3.7e-3 * rho ** np.arange(n)     # unnormalised energies
    votes = np.zeros((1, 1, 1, n), dtype=np.int32)
    oracle_mod.calib_accumulate(row.reshape(1, 1, 1, n), eps, votes)
    assert votes.sum() == want
    assert set(np.nonzero(votes[0, 0, 0])[0]) == set(perm[:want])


def test_calib_votes_union_and_intersection(oracle_mod):
    rng = np.random.default_rng(12)
    nb = 24
    runs = [rng.gamma(0.5, size=(1, 2, nb, nb)) for _ in range(3)]
    votes = np.zeros((1, 2, nb, nb), dtype=np.int32)
    sel = []
    for e in runs:
        one = np.zeros_like(votes)
        oracle_mod.calib_accumulate(e, 0.3, one)
        sel.append(one.astype(bool))
        oracle_mod.calib_accumulate(e, 0.3, votes)
    assert votes.max() <= 3
    np.testing.assert_array_equal(votes, sum(s.astype(np.int32) for s in sel))
    union = oracle_mod.calib_finalize(votes, 1).astype(bool)
    inter = oracle_mod.calib_finalize(votes, 3).astype(bool)
    np.testing.assert_array_equal(union, sel[0] | sel[1] | sel[2])
    np.testing.assert_array_equal(inter, sel[0] & sel[1] & sel[2])
    # each run keeps at least the row's largest block
    for e, s in zip(runs, sel):
        am = e.argmax(-1)
        assert np.take_along_axis(s, am[..., None], -1).all()


def test_calib_scale_invariance_and_zero_rows(oracle_mod):
    rng = np.random.default_rng(13)
    nb = 40
    e = rng.gamma(0.7, size=(1, 1, nb, nb))
    e[0, 0, 5] = 0.0                  # an all-zero row keeps nothing
    e[0, 0, 6, :3] = -1.0             # negative energies count as zero
    a = np.zeros(e.shape, dtype=np.int32)
    b = np.zeros(e.shape, dtype=np.int32)
    oracle_mod.calib_accumulate(e, 0.25, a)
    oracle_mod.calib_accumulate(e * 1024.0, 0.25, b)
    np.testing.assert_array_equal(a, b)
    assert a[0, 0, 5].sum() == 0
    assert (a[0, 0, 6, :3] == 0).all()
    full = np.zeros(e.shape, dtype=np.int32)
    oracle_mod.calib_accumulate(e, 0.0, full)      # eps = 0 keeps every block of a live row
    assert full[0, 0, 5].sum() == 0 and (np.delete(full[0, 0], 5, axis=0) == 1).all()


# ---------------------------------------------------------------------------
# Backward of block-masked attention


def _torch_masked_attention_grads(q, k, v, dO, mask, scale=None):
    """fp64 torch autograd of O = softmax(scale QK^T, kept blocks) V; rows with
    no kept block give O = 0 and carry no gradient."""
    import torch
    B, H, S, d = q.shape
    nb = S // 64
    tq, tk, tv = (torch.from_numpy(_f(a)).requires_grad_(True) for a in (q, k, v))
    tdo = torch.from_numpy(_f(dO))
    keep = torch.from_numpy(np.repeat(np.repeat(mask.astype(bool), 64, axis=2), 64, axis=3))
    live = keep.any(dim=-1, keepdim=True)
    s = torch.einsum("bhid,bhjd->bhij", tq, tk) * (scale if scale else 1.0 / math.sqrt(d))
    s = torch.where(keep, s, torch.full_like(s, -math.inf))
    s = torch.where(live, s, torch.zeros_like(s))          # empty rows: finite, then zeroed
    p = torch.softmax(s, dim=-1) * live
    o = torch.einsum("bhij,bhjd->bhid", p, tv)
    (o * tdo).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def test_attention_bwd_matches_torch_autograd(oracle_mod):
    rng = np.random.default_rng(31)
    B, H, S, d = 1, 2, 320, 64
    nb = S // 64
    q, k, v, dO = (_rand_bits(rng, (B, H, S, d), sc) for sc in (0.7, 0.7, 1.0, 1.0))
    mask = (rng.random((B, H, nb, nb)) < 0.5).astype(np.uint8)
    mask[..., np.arange(nb), np.arange(nb)] = 1
    mask[0, 1, 3, :] = 0                                   # one empty query block
    gq, gk, gv = _torch_masked_attention_grads(q, k, v, dO, mask)
    dQ, dK, dV = oracle_mod.attention_bwd(q, k, v, dO, mask)
    for got, want in ((dQ, gq), (dK, gk), (dV, gv)):
        np.testing.assert_allclose(got, want.reshape(-1, d), rtol=1e-9, atol=1e-12)
    assert np.all(dQ.reshape(B, H, S, d)[0, 1, 192:256] == 0)


def test_attention_bwd_invariants(oracle_mod):
    # sum_j dS_ij = 0 for every row, so dK summed over a head's keys vanishes;
    # sum_j p_ij = 1, so dV summed over keys equals dO summed over live rows
    rng = np.random.default_rng(32)
    B, H, S, d = 1, 1, 256, 64
    nb = S // 64
    q, k, v, dO = (_rand_bits(rng, (B, H, S, d)) for _ in range(4))
    mask = (rng.random((B, H, nb, nb)) < 0.6).astype(np.uint8)
    mask[0, 0, 2, :] = 0
    mask[0, 0, 0, 0] = 1
    dQ, dK, dV = oracle_mod.attention_bwd(q, k, v, dO, mask)
    live_rows = np.repeat(mask[0, 0].any(axis=1), 64)
    np.testing.assert_allclose(dK.sum(axis=0), 0.0, atol=1e-10)
    np.testing.assert_allclose(dV.sum(axis=0), _f(dO)[0, 0][live_rows].sum(axis=0), atol=1e-10)
    # uniform attention (q = 0): p = 1/n over the n kept keys of a row
    q0 = np.zeros_like(q)
    _, _, dV0 = oracle_mod.attention_bwd(q0, k, v, dO, mask)
    n_kept = 64 * mask[0, 0].sum(axis=1)                    # keys per query block
    want = np.zeros((S, d))
    for r in range(nb):
        if n_kept[r] == 0:
            continue
        g = _f(dO)[0, 0, 64 * r:64 * (r + 1)].sum(axis=0) / n_kept[r]
        for c in np.nonzero(mask[0, 0, r])[0]:
            want[64 * c:64 * (c + 1)] += g
    np.testing.assert_allclose(dV0, want, atol=1e-12)


def test_attention_bwd_row_subsets(oracle_mod):
    rng = np.random.default_rng(33)
    B, H, S, d = 2, 1, 192, 64
    q, k, v, dO = (_rand_bits(rng, (B, H, S, d)) for _ in range(4))
    mask = (rng.random((B, H, 3, 3)) < 0.7).astype(np.uint8)
    dQ, dK, dV = oracle_mod.attention_bwd(q, k, v, dO, mask)
    qr = np.array([5, 300, 191], dtype=np.int64)
    kr = np.array([0, 250], dtype=np.int64)
    sq, sk, sv = oracle_mod.attention_bwd(q, k, v, dO, mask, qrows=qr, krows=kr)
    np.testing.assert_array_equal(sq, dQ[qr])
    np.testing.assert_array_equal(sk, dK[kr])
    np.testing.assert_array_equal(sv, dV[kr])
    eq, ek, ev = oracle_mod.attention_bwd(q, k, v, dO, mask, qrows=qr, krows=np.empty(0, np.int64))
    assert ek.shape == (0, d) and np.array_equal(eq, dQ[qr])


# ---------------------------------------------------------------------------
# XAttention antidiagonal scoring


def _brute_xattn(q, k, St):
    """Explicit antidiagonal sums of the full fp64 score matrix, scipy softmax,
    block means; independent of the oracle's strided loops."""
    from scipy.special import softmax
    B, H, S, d = q.shape
    nb, L, per = S // 64, S // St, 64 // St
    out = np.zeros((B, H, nb, nb))
    for b in range(B):
        for h in range(H):
            M = _f(q[b, h]) @ _f(k[b, h]).T / math.sqrt(d)
            A = np.zeros((L, L))
            for s in range(St):
                A += M[np.arange(L)[:, None] * St + St - 1 - s, np.arange(L)[None, :] * St + s]
            P = softmax(A / St, axis=1)
            out[b, h] = P.reshape(nb, per, nb, per).sum(axis=(1, 3)) / per
    return out


@pytest.mark.parametrize("St", [1, 4, 8, 16])
def test_xattn_matches_brute_force_antidiagonals(oracle_mod, St):
    rng = np.random.default_rng(40 + St)
    q = _rand_bits(rng, (1, 2, 256, 64), 0.7)
    k = _rand_bits(rng, (1, 2, 256, 64), 0.7)
    got = oracle_mod.xattn_scores(q, k, St)
    np.testing.assert_allclose(got, _brute_xattn(q, k, St), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(got.sum(axis=-1), 1.0, atol=1e-12)
    # an antidiagonal is not a diagonal: reversing the query order inside each
    # stride group changes the scores (St > 1)
    if St > 1:
        qf = q.reshape(1, 2, 256 // St, St, 64)[:, :, :, ::-1].reshape(q.shape)
        assert np.abs(oracle_mod.xattn_scores(np.ascontiguousarray(qf), k, St) - got).max() > 1e-4


def test_xattn_stride1_is_block_energy(oracle_mod):
    # stride 1: every strided row is a token and a_ij the attention logit, so
    # the scores are the true block energies with the dense LSE
    rng = np.random.default_rng(50)
    q = _rand_bits(rng, (1, 1, 192, 64))
    k = _rand_bits(rng, (1, 1, 192, 64))
    v = _rand_bits(rng, (1, 1, 192, 64))
    _, lse = oracle_mod.dense_attention(q, k, v)
    E, _ = oracle_mod.block_energy(q, k, lse.reshape(1, 1, 192), np.ones((1, 1, 3, 3), np.uint8))
    np.testing.assert_allclose(oracle_mod.xattn_scores(q, k, 1), E, rtol=1e-10)


def test_xattn_uniform_and_rows(oracle_mod):
    rng = np.random.default_rng(51)
    q = np.zeros((1, 1, 320, 64), dtype=np.uint16)
    k = _rand_bits(rng, (1, 1, 320, 64))
    np.testing.assert_allclose(oracle_mod.xattn_scores(q, k, 8), 1.0 / 5, rtol=1e-13)
    q = _rand_bits(rng, (2, 1, 320, 64))
    k = _rand_bits(rng, (2, 1, 320, 64))
    full = oracle_mod.xattn_scores(q, k, 8).reshape(-1, 5)
    rows = np.array([7, 0, 4], dtype=np.int64)
    np.testing.assert_array_equal(oracle_mod.xattn_scores(q, k, 8, rows=rows), full[rows])


def test_select_rows_matches_builder_on_its_own_map(oracle_mod):
    # the builder's selection applied to the softmax of its own reduced map
    # gives the builder's mask
    rng = np.random.default_rng(52)
    grid = (1, 2, 2)
    q = _rand_bits(rng, (1, 2, 256, 64))
    k = _rand_bits(rng, (1, 2, 256, 64))
    want = oracle_mod.build_mask(q, k, grid, 0.3, (0, 1, 0))
    qb, kb = oracle_mod.pool(q), oracle_mod.pool(k)
    P = np.stack([[np.stack([oracle_mod.softmax_row(r) for r in oracle_mod.logits(qb[0, h], kb[0, h])])
                   for h in range(2)]])
    np.testing.assert_array_equal(oracle_mod.select_rows(P * 3.0, grid, 0.3, (0, 1, 0)), want)
