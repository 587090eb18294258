"""Block-sparse attention backward on the GPU vs the fp64 oracle.

The GPU path is the product one: bsa_fwd over a block CSR, then bsa_bwd from
its O and LSE.  The oracle gets only Q, K, V, dO and the mask (its own NABLA
mask or a host-made one) and computes the exact gradients in fp64.

Tolerance, from the arithmetic: P and dS enter the tensor-core products as
bf16 (relative rounding 2^-9), D = rowsum(dO o O) uses the bf16 O, S and dP
are fp32-accumulated bf16 products, and the outputs are rounded to bf16.
Each gradient element is a sum of many such terms with independent rounding,
so its error is a small multiple of 2^-9 of the magnitude of the terms.  The
bar per tensor G: max |G - G_ref| <= 2e-2 * max |G_ref| and
mean |G - G_ref| <= 1e-2 * mean |G_ref|."""
import numpy as np
import pytest

from _parity import to_device_bf16

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 1e-2


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _csr(mask):
    import torch
    nb = mask.shape[-1]
    flat = mask.reshape(-1, nb)
    row_ptr = np.concatenate([[0], np.cumsum(flat.sum(axis=1))]).astype(np.int32)
    col_idx = np.nonzero(flat)[1].astype(np.int32)
    if col_idx.size == 0:
        col_idx = np.zeros(1, dtype=np.int32)
    return torch.from_numpy(row_ptr).cuda(), torch.from_numpy(col_idx).cuda()


def _fwd_bwd(nl, q, k, v, dO, mask, scale=None):
    B, H, S, d = q.shape
    qd, kd, vd, dod = (to_device_bf16(a) for a in (q, k, v, dO))
    rp, ci = _csr(mask)
    shape = nl.make_shape(B, H, S, d)
    wsf = nl.Workspace.create(shape, nl.OP_FWD)
    o, lse = nl.bsa_fwd(qd, kd, vd, rp, ci, scale=scale, workspace=wsf)
    assert wsf.query_status() == 0
    wsb = nl.Workspace.create(shape, nl.OP_BWD)
    dq, dk, dv = nl.bsa_bwd(qd, kd, vd, o, dod, lse, rp, ci, scale=scale, workspace=wsb)
    assert wsb.query_status() == 0
    return dq, dk, dv, (qd, kd, vd, dod, o, lse, rp, ci)


def _host(t):
    return t.float().cpu().numpy().reshape(-1, t.shape[-1]).astype(np.float64)


def _compare(name, got, ref):
    err = np.abs(got - ref)
    scale_max = max(np.abs(ref).max(), 1e-30)
    scale_mean = max(np.abs(ref).mean(), 1e-30)
    print(f"{name}: max-abs {err.max():.3g} (rel {err.max() / scale_max:.3g}), "
          f"mean-abs {err.mean():.3g} (rel {err.mean() / scale_mean:.3g})")
    assert np.isfinite(got).all()
    assert err.max() <= MAX_REL * scale_max, name
    assert err.mean() <= MEAN_REL * scale_mean, name
    return float(err.max() / scale_max)


def _dout(synth_mod, B, H, S, d, seed):
    return synth_mod.make_tensor(3, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_bwd_parity_nabla_mask(nl, oracle_mod, synth_mod, name):
    w = synth_mod.WORKLOADS[name]
    q, k, v = synth_mod.make_qkv(w)
    if name == "small":            # keep the oracle to seconds: 2 heads
        q, k, v = q[:, :2].copy(), k[:, :2].copy(), v[:, :2].copy()
    B, H, S, d = q.shape
    dO = _dout(synth_mod, B, H, S, d, seed=1)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    dq, dk, dv, _ = _fwd_bwd(nl, q, k, v, dO, mask)
    rq, rk, rv = oracle_mod.attention_bwd(q, k, v, dO, mask)
    _compare("dQ", _host(dq), rq)
    _compare("dK", _host(dk), rk)
    _compare("dV", _host(dv), rv)


@pytest.mark.parametrize("B,H,nb,d", [(1, 1, 1, 64), (1, 2, 3, 128), (2, 3, 5, 64),
                                      (1, 1, 7, 128), (2, 1, 33, 64)])
def test_bwd_edge_cases(nl, oracle_mod, synth_mod, B, H, nb, d):
    """Odd block counts (a stationary pair with one block), empty query rows,
    key blocks no query lists, single-block and dense rows, both head dims."""
    S = 64 * nb
    q, k, v = (synth_mod.make_tensor(i, 50 + nb, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
               for i in range(3))
    dO = _dout(synth_mod, B, H, S, d, seed=60 + nb)
    rng = np.random.default_rng(nb + 100)
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    mask[..., 0, :] = 0                      # an empty query block
    if nb > 1:
        mask[..., 1, :] = 0
        mask[..., 1, nb - 1] = 1             # a single far block
    if nb > 2:
        mask[..., 2, :] = 1                  # a dense row
    if nb > 3:
        mask[..., :, 3] = 0                  # a key block no query lists
    dq, dk, dv, _ = _fwd_bwd(nl, q, k, v, dO, mask)
    rq, rk, rv = oracle_mod.attention_bwd(q, k, v, dO, mask)
    _compare("dQ", _host(dq), rq)
    _compare("dK", _host(dk), rk)
    _compare("dV", _host(dv), rv)
    g = _host(dq).reshape(B * H, nb, 64, d)
    assert np.all(g[:, 0] == 0.0)            # empty rows get no gradient
    if nb > 3:
        assert np.all(_host(dk).reshape(B * H, nb, 64, d)[:, 3] == 0.0)
        assert np.all(_host(dv).reshape(B * H, nb, 64, d)[:, 3] == 0.0)


def test_bwd_explicit_scale_and_determinism(nl, oracle_mod, synth_mod):
    B, H, nb, d = 1, 2, 4, 128
    S = 64 * nb
    q, k, v = (synth_mod.make_tensor(i, 9, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
               for i in range(3))
    dO = _dout(synth_mod, B, H, S, d, seed=10)
    mask = np.ones((B, H, nb, nb), dtype=np.uint8)
    mask[0, 1, 2, 1] = 0
    dq, dk, dv, st = _fwd_bwd(nl, q, k, v, dO, mask, scale=0.3)
    rq, rk, rv = oracle_mod.attention_bwd(q, k, v, dO, mask, scale=0.3)
    _compare("dQ", _host(dq), rq)
    _compare("dK", _host(dk), rk)
    _compare("dV", _host(dv), rv)
    qd, kd, vd, dod, o, lse, rp, ci = st
    dq2, dk2, dv2 = nl.bsa_bwd(qd, kd, vd, o, dod, lse, rp, ci, scale=0.3)
    import torch
    for a, b in ((dq, dq2), (dk, dk2), (dv, dv2)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_bwd_full_size_wan(nl, oracle_mod, synth_mod):
    """Wan 720p layer with its NABLA mask: sampled dQ rows against the oracle;
    over every head, sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (identities of
    the exact gradient that hold at any size)."""
    import torch
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = synth_mod.make_qkv(w)
    dO = _dout(synth_mod, w.B, w.H, w.S, w.d, seed=1)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    dq, dk, dv, _ = _fwd_bwd(nl, q, k, v, dO, mask)
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(w.B * w.H * w.S, 96, replace=False)).astype(np.int64)
    rq, _, _ = oracle_mod.attention_bwd(q, k, v, dO, mask, qrows=rows,
                                        krows=np.empty(0, np.int64))
    got = dq.reshape(-1, w.d)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
    _compare("dQ sampled", got.astype(np.float64), rq)
    BH = w.B * w.H
    dk_sum = dk.float().reshape(BH, w.S, w.d).sum(dim=1)
    dk_abs = dk.float().abs().reshape(BH, w.S, w.d).sum(dim=1)
    assert (dk_sum.abs() <= 2e-3 * dk_abs + 1e-3).all()
    dv_sum = dv.float().reshape(BH, w.S, w.d).sum(dim=1).cpu().numpy()
    do_sum = (torch.from_numpy(dO.view(np.int16)).view(torch.bfloat16).float()
              .reshape(BH, w.S, w.d).sum(dim=1).numpy())
    dv_abs = dv.float().abs().reshape(BH, w.S, w.d).sum(dim=1).cpu().numpy()
    assert (np.abs(dv_sum - do_sum) <= 2e-3 * dv_abs + 1e-2).all()


def test_bwd_wan_sliced_heads_dk_dv_rows(nl, oracle_mod, synth_mod, parity_record):
    """Two heads of the Wan 720p layer (full 76,800-token length, their NABLA
    mask): dK and dV on 192 seeded key rows per head (three whole key blocks,
    the first, the last and one seeded between them), element by element
    against the oracle, plus 64 dQ rows per head.  A misplaced or swapped key
    row, which the dK / dV sum identities cannot see, fails here."""
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = synth_mod.make_qkv(w)
    heads = [0, w.H - 1]
    qs, ks, vs = (np.ascontiguousarray(a[:, heads]) for a in (q, k, v))
    B, H, S, d = qs.shape
    nb = S // 64
    dO = _dout(synth_mod, B, H, S, d, seed=7)
    mask = oracle_mod.build_mask(qs, ks, w.tile_grid, w.thr, w.sta)
    dq, dk, dv, _ = _fwd_bwd(nl, qs, ks, vs, dO, mask)
    rng = np.random.default_rng(11)
    krows, qrows = [], []
    for h in range(H):
        for blk in (0, int(rng.integers(1, nb - 1)), nb - 1):
            krows.extend(h * S + 64 * blk + np.arange(64))
        qrows.extend(h * S + np.sort(rng.choice(S, 64, replace=False)))
    krows = np.array(krows, dtype=np.int64)
    qrows = np.array(qrows, dtype=np.int64)
    rq, rk, rv = oracle_mod.attention_bwd(qs, ks, vs, dO, mask, qrows=qrows, krows=krows)
    _compare("dQ rows", _host(dq)[qrows], rq)
    ek = _compare("dK rows", _host(dk)[krows], rk)
    ev = _compare("dV rows", _host(dv)[krows], rv)
    parity_record("backward wan720p heads 0 and 39", key_rows=int(krows.size),
                  query_rows=int(qrows.size), dk_max_rel=ek, dv_max_rel=ev)
