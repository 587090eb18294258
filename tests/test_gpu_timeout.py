"""Failure path of the attention kernel without faulting the GPU: a 1 ns limit
on every pipeline wait makes the kernel give up, drain its own copies and MMAs,
free tensor memory and report NABLA_ERR_TIMEOUT; with the default limit back,
the same context computes correct results."""
import numpy as np
import pytest

from _parity import compare_attention, rows_with_same_mask, sample_rows, to_device_bf16

pytestmark = pytest.mark.gpu


def test_wait_limit_reports_timeout_and_context_survives(oracle_mod, synth_mod):
    import torch
    import block_sparse_attention_23_b200 as nl
    w = synth_mod.WORKLOADS["small"]
    q, k, v = synth_mod.make_qkv(w)
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    row_ptr, col_idx, nnz, mask = nl.nabla_build_mask(qd, kd, w.tile_grid, w.thr, w.sta,
                                                      want_mask=True)
    ws = nl.Workspace.create(nl.make_shape(w.B, w.H, w.S, w.d), nl.OP_FWD)
    try:
        nl.set_wait_limit_ns(1)
        nl.bsa_fwd(qd, kd, vd, row_ptr, col_idx, workspace=ws)
        assert ws.query_status() == 5          # NABLA_ERR_TIMEOUT
    finally:
        nl.set_wait_limit_ns(0)
    o, lse = nl.bsa_fwd(qd, kd, vd, row_ptr, col_idx, workspace=ws)
    assert ws.query_status() == 0
    ora_mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    rows = rows_with_same_mask(sample_rows(w.B, w.H, w.S, 4, 16, seed=9), mask.cpu().numpy(),
                               ora_mask, w.S)
    ro, rl = oracle_mod.masked_attention(q, k, v, ora_mask, rows)
    go = o.float().cpu().numpy().reshape(-1, w.d)[rows]
    gl = lse.cpu().numpy().reshape(-1)[rows]
    compare_attention(go, gl, ro, rl)
    torch.cuda.synchronize()
