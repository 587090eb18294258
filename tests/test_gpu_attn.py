"""Block-sparse attention forward on the GPU vs the fp64 oracle: bf16 O within
max-abs 2e-2 / mean-abs 2e-3, fp32 LSE within 1e-3.  The oracle always uses
its own mask (or a host-made static mask) and never takes a GPU result as
input.  For the composed NABLA layer (GPU mask -> GPU attention), the sampled
rows whose mask row the GPU and the oracle agree on are compared directly;
the rows of query blocks whose mask rows differ (near-cut rows) are compared
after a second GPU forward over the oracle's own mask, so the attention on
exactly those rows is checked as well."""
import numpy as np
import pytest

from _parity import compare_attention, rows_with_same_mask, sample_rows, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _gather(o, lse, rows, S):
    o = o.float().cpu().numpy().reshape(-1, o.shape[-1])
    lse = lse.cpu().numpy().reshape(-1)
    return o[rows], lse[rows]


def _nabla_layer(nl, w, q, k, v, thr=None, sta="cfg", exact=False, passes=None):
    """Mask + forward.  exact: run only the exact-reference kernel; passes: the
    number of exact-reference recomputations the call must report."""
    thr = w.thr if thr is None else thr
    sta = w.sta if sta == "cfg" else sta
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    row_ptr, col_idx, nnz, mask = nl.nabla_build_mask(qd, kd, w.tile_grid, thr, sta,
                                                      want_mask=True)
    ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d), nl.OP_FWD)
    nl.set_exact_reference(exact)
    try:
        o, lse = nl.bsa_fwd(qd, kd, vd, row_ptr, col_idx, workspace=ws)
        assert ws.query_status() == 0
    finally:
        nl.set_exact_reference(False)
    if passes is not None:
        assert ws.exact_passes() == passes
    return o, lse, mask.cpu().numpy()


@pytest.mark.parametrize("exact", [False, True], ids=["fixed-ref", "exact-ref"])
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_attention_parity_all_rows(nl, oracle_mod, synth_mod, name, exact):
    """Both forward kernels on the same inputs: the fixed-reference one (no
    recomputation needed here) and the exact-reference one alone."""
    w = synth_mod.WORKLOADS[name]
    q, k, v = synth_mod.make_qkv(w)
    o, lse, gmask = _nabla_layer(nl, w, q, k, v, exact=exact, passes=1 if exact else 0)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    rows = rows_with_same_mask(np.arange(w.B * w.H * w.S, dtype=np.int64), gmask, mask, w.S)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go, gl = _gather(o, lse, rows, w.S)
    mx, mean = compare_attention(go, gl, ro, rl)
    print(f"{name}: max-abs {mx:.3g} mean-abs {mean:.3g}")


@pytest.mark.parametrize("name", ["hunyuan720p", "wan720p"])
def test_attention_parity_full_size(nl, oracle_mod, synth_mod, parity_record, name):
    """Every head x 64 seeded query blocks (plus the first and last) x all 64
    rows of each block."""
    import torch
    w = synth_mod.WORKLOADS[name]
    q, k, v = synth_mod.make_qkv(w)
    # the Wan-shaped layer runs on the fixed-reference kernel alone
    o, lse, gmask = _nabla_layer(nl, w, q, k, v, passes=0 if name == "wan720p" else None)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    rows = sample_rows(w.B, w.H, w.S, 64, 64, seed=1)
    same_rows = rows_with_same_mask(rows, gmask, mask, w.S)
    diff_rows = np.setdiff1d(rows, same_rows)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    sel = np.isin(rows, same_rows)
    go, gl = _gather(o, lse, same_rows, w.S)
    mx, mean = compare_attention(go, gl, ro[sel], rl[sel])
    if diff_rows.size:
        # the same forward over the oracle's mask, on the rows whose masks differ
        qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
        o2, lse2 = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda())
        go2, gl2 = _gather(o2, lse2, diff_rows, w.S)
        compare_attention(go2, gl2, ro[~sel], rl[~sel])
    parity_record(f"attention {name}", sampled_rows=int(rows.size),
                  rows_compared_on_gpu_mask=int(same_rows.size),
                  rows_compared_on_oracle_mask=int(diff_rows.size), o_max_abs=mx, o_mean_abs=mean)


@pytest.mark.parametrize("p", [0.05, 0.1, 0.2, 0.4, 0.7, 1.0])
def test_static_mask_sweep_parity(nl, oracle_mod, synth_mod, parity_record, p):
    w = synth_mod.WORKLOADS["sweep"]
    q, k, v = synth_mod.make_qkv(w)
    mask = synth_mod.make_bernoulli_mask(0, w.B * w.H, w.nb, p).reshape(w.B, w.H, w.nb, w.nb)
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    import torch
    ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d), nl.OP_FWD_WITH_MASK)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda(), workspace=ws)
    assert ws.query_status() == 0
    rows = sample_rows(w.B, w.H, w.S, 64, 64, seed=2)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go, gl = _gather(o, lse, rows, w.S)
    mx, mean = compare_attention(go, gl, ro, rl)
    parity_record(f"attention sweep p={p}", sampled_rows=int(rows.size), o_max_abs=mx,
                  o_mean_abs=mean)


def _random_qkv(synth_mod, B, H, S, d, seed):
    q = synth_mod.make_tensor(0, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    k = synth_mod.make_tensor(1, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    v = synth_mod.make_tensor(2, seed, B, H, S, d, pos_weight=0.0, noise_weight=1.0)
    return q, k, v


@pytest.mark.parametrize("B,H,nb,d", [(1, 1, 1, 64), (1, 2, 3, 128), (2, 3, 5, 64),
                                      (1, 1, 7, 128), (2, 1, 33, 64)])
def test_static_mask_edge_cases(nl, oracle_mod, synth_mod, B, H, nb, d):
    """Odd block counts (a query pair with one block), empty rows, single-block
    rows, dense rows, on both head dims."""
    import torch
    S = 64 * nb
    q, k, v = _random_qkv(synth_mod, B, H, S, d, seed=nb)
    rng = np.random.default_rng(nb)
    mask = (rng.random((B, H, nb, nb)) < 0.4).astype(np.uint8)
    mask[..., 0, :] = 0                      # an empty row
    if nb > 1:
        mask[..., 1, :] = 0
        mask[..., 1, nb - 1] = 1             # a single far block
    if nb > 2:
        mask[..., 2, :] = 1                  # a dense row
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD_WITH_MASK)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda(), workspace=ws)
    assert ws.query_status() == 0
    rows = np.arange(B * H * S, dtype=np.int64)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go, gl = _gather(o, lse, rows, S)
    compare_attention(go, gl, ro, rl)
    assert np.all(go.reshape(B * H, nb, 64, d)[:, 0] == 0.0)
    assert np.all(np.isneginf(gl.reshape(B * H, nb, 64)[:, 0]))


def test_thr0_is_dense_attention(nl, oracle_mod, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, v = synth_mod.make_qkv(w)
    o, lse, mask = _nabla_layer(nl, w, q, k, v, thr=0.0, sta=None)
    assert mask.min() == 1
    rows = np.arange(0, w.B * w.H * w.S, 3, dtype=np.int64)
    ro, rl = oracle_mod.dense_attention(q, k, v, rows)
    go, gl = _gather(o, lse, rows, w.S)
    compare_attention(go, gl, ro, rl)


def test_explicit_scale(nl, oracle_mod, synth_mod):
    import torch
    B, H, nb, d = 1, 2, 4, 128
    S = 64 * nb
    q, k, v = _random_qkv(synth_mod, B, H, S, d, seed=11)
    mask = np.ones((B, H, nb, nb), dtype=np.uint8)
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda(), scale=0.3)
    rows = np.arange(B * H * S, dtype=np.int64)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows, scale=0.3)
    go, gl = _gather(o, lse, rows, S)
    compare_attention(go, gl, ro, rl)


def test_bad_csr_index_reported(nl, oracle_mod, synth_mod):
    import torch
    B, H, nb, d = 1, 1, 4, 64
    S = 64 * nb
    q, k, v = _random_qkv(synth_mod, B, H, S, d, seed=5)
    row_ptr = torch.tensor([0, 2, 4, 5, 7], dtype=torch.int32).cuda()
    col_idx = torch.tensor([0, 1, 1, 99, 2, 3, -1], dtype=torch.int32).cuda()
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD)
    o, lse = nl.bsa_fwd(qd, kd, vd, row_ptr, col_idx, workspace=ws)
    assert ws.query_status() == 6          # NABLA_ERR_BAD_INDEX
    mask = np.zeros((1, 1, nb, nb), dtype=np.uint8)
    mask[0, 0, 0, [0, 1]] = 1
    mask[0, 0, 1, 1] = 1
    mask[0, 0, 2, 2] = 1
    mask[0, 0, 3, 3] = 1
    rows = np.arange(S, dtype=np.int64)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go, gl = _gather(o, lse, rows, S)
    compare_attention(go, gl, ro, rl)


@pytest.mark.parametrize("d", [64, 128])
def test_union_shapes_of_query_pairs(nl, oracle_mod, synth_mod, d):
    """Pairs of query blocks whose union of key blocks has every size modulo
    four (the last 256-key tile padded with 1, 2 or 3 masked entries), is
    empty, or holds entries only one of the two blocks lists."""
    import torch
    B, H, nb = 1, 3, 12
    S = 64 * nb
    q, k, v = _random_qkv(synth_mod, B, H, S, d, seed=77 + d)
    mask = np.zeros((B, H, nb, nb), dtype=np.uint8)
    for h in range(H):
        m = mask[0, h]
        # pair 0 (rows 0, 1): both empty
        m[2, (h + 5) % nb] = 1                           # pair 1: union of 1, row 3 empty
        m[4, [1, 2]] = 1
        m[5, 3 + h] = 1                                  # pair 2: union of 3, disjoint lists
        m[6, 0:5] = 1
        m[7, 5:9] = 1                                    # pair 3: union of 9
        m[8, :] = 1
        m[9, ::2] = 1                                    # pair 4: union of 12, row 9 half of it
        m[10, [h, nb - 1 - h]] = 1
        m[11, [h, (h + 6) % nb]] = 1                     # pair 5: union of 3 with one shared
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    ws = nl.Workspace.create(nl.make_shape(B, H, S, d), nl.OP_FWD_WITH_MASK)
    o, lse = nl.bsa_fwd_with_mask(qd, kd, vd, torch.from_numpy(mask).cuda(), workspace=ws)
    assert ws.query_status() == 0
    rows = np.arange(B * H * S, dtype=np.int64)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go, gl = _gather(o, lse, rows, S)
    compare_attention(go, gl, ro, rl)
    empty = mask.reshape(B * H, nb, nb).sum(-1) == 0
    assert np.all(go.reshape(B * H, nb, 64, d)[empty] == 0.0)
    assert np.all(np.isneginf(gl.reshape(B * H, nb, 64)[empty]))
