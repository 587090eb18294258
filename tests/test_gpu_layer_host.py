"""nabla_layer_host (mask + forward on host tensors, heads streamed through the
device in chunks) on the GPU: against the fp64 oracle on the rows whose mask
the GPU and the oracle agree on, and bit for bit against the same layer run
on device tensors, with ragged last chunks and chunks that span batches."""
import numpy as np
import pytest

from _parity import compare_attention, rows_with_same_mask, sample_rows, to_device_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nl():
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    return nl


def _host_bf16(a_u16, pin=True):
    import torch
    t = torch.from_numpy(a_u16.view(np.int16)).view(torch.bfloat16).contiguous()
    return t.pin_memory() if pin else t


def _device_layer(nl, tile_grid, thr, sta, q, k, v):
    qd, kd, vd = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    row_ptr, col_idx, _, mask = nl.nabla_build_mask(qd, kd, tile_grid, thr, sta, want_mask=True)
    o, lse = nl.bsa_fwd(qd, kd, vd, row_ptr, col_idx)
    return o.cpu(), lse.cpu(), mask.cpu().numpy()


def _host_layer(nl, tile_grid, thr, sta, q, k, v, hpc, pin=True, expect_status=0):
    import torch
    qh, kh, vh = _host_bf16(q, pin), _host_bf16(k, pin), _host_bf16(v, pin)
    B, H, S, d = qh.shape
    ws = nl.layer_host_workspace(nl.make_shape(B, H, S, d, tile_grid), hpc)
    o, lse = nl.nabla_layer_host(qh, kh, vh, tile_grid, thr, sta, heads_per_chunk=hpc,
                                 workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert ws.query_status() == expect_status
    return o, lse


def _same_bits(a, b):
    import torch
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


@pytest.mark.parametrize("hpc", [5, 1, 12, 64])
def test_layer_host_matches_device_layer_bitwise(nl, synth_mod, hpc):
    w = synth_mod.WORKLOADS["small"]
    q, k, v = synth_mod.make_qkv(w)
    od, ld, _ = _device_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v)
    oh, lh = _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, hpc)
    assert _same_bits(oh, od)
    assert _same_bits(lh, ld)


def test_layer_host_pageable_buffers(nl, synth_mod):
    w = synth_mod.WORKLOADS["tiny"]
    q, k, v = synth_mod.make_qkv(w)
    od, ld, _ = _device_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v)
    oh, lh = _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, 1, pin=False)
    assert _same_bits(oh, od) and _same_bits(lh, ld)


def test_layer_host_chunks_span_batches(nl, synth_mod):
    # B = 2, H = 3, chunks of 2 heads: chunk 1 holds (b0, h2) and (b1, h0)
    w = synth_mod.WORKLOADS["small"]
    B, H, S, d = 2, 3, w.S, w.d
    x = [synth_mod.make_tensor(t, 7, B, H, S, d, grid=w.tile_grid)
         for t in (synth_mod.TENSOR_Q, synth_mod.TENSOR_K, synth_mod.TENSOR_V)]
    od, ld, _ = _device_layer(nl, w.tile_grid, 0.3, (1, 1, 1), *x)
    oh, lh = _host_layer(nl, w.tile_grid, 0.3, (1, 1, 1), *x, 2)
    assert _same_bits(oh, od) and _same_bits(lh, ld)


def test_layer_host_parity_vs_oracle(nl, oracle_mod, synth_mod):
    w = synth_mod.WORKLOADS["small"]
    q, k, v = synth_mod.make_qkv(w)
    oh, lh = _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, 5)
    _, _, gmask = _device_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v)
    mask = oracle_mod.build_mask(q, k, w.tile_grid, w.thr, w.sta)
    rows = rows_with_same_mask(sample_rows(w.B, w.H, w.S, 4, 16, seed=3), gmask, mask, w.S)
    ro, rl = oracle_mod.masked_attention(q, k, v, mask, rows)
    go = oh.float().numpy().reshape(-1, w.d)[rows]
    gl = lh.numpy().reshape(-1)[rows]
    compare_attention(go, gl, ro, rl)


def test_layer_host_full_size_bitwise(nl, synth_mod):
    # the Wan 720p-shaped layer in the chunking the benchmark uses
    w = synth_mod.WORKLOADS["wan720p"]
    q, k, v = synth_mod.make_qkv(w)
    od, ld, _ = _device_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v)
    oh, lh = _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, 4)
    assert _same_bits(oh, od) and _same_bits(lh, ld)


def test_layer_host_back_to_back_calls(nl, synth_mod):
    # two calls queued without a host synchronisation between them share the
    # workspace, the copy streams and the second compute stream
    import torch
    w = synth_mod.WORKLOADS["small"]
    xa = synth_mod.make_qkv(w, seed=0)
    xb = synth_mod.make_qkv(w, seed=5)
    ref = [_device_layer(nl, w.tile_grid, w.thr, w.sta, *x)[:2] for x in (xa, xb)]
    ws = nl.layer_host_workspace(nl.make_shape(w.B, w.H, w.S, w.d, w.tile_grid), 3)
    outs = []
    for x in (xa, xb):
        h = [_host_bf16(a) for a in x]
        outs.append(nl.nabla_layer_host(*h, w.tile_grid, w.thr, w.sta, heads_per_chunk=3,
                                        workspace=ws))
    torch.cuda.current_stream().synchronize()
    assert ws.query_status() == 0
    for (oh, lh), (od, ld) in zip(outs, ref):
        assert _same_bits(oh, od) and _same_bits(lh, ld)


def test_layer_host_reports_timeout_from_both_streams(nl, synth_mod):
    # a 1 ns limit on every pipeline wait: the attention kernels of every chunk
    # give up and report NABLA_ERR_TIMEOUT into the one status header; with the
    # default limit back the same workspace computes the exact layer
    w = synth_mod.WORKLOADS["small"]
    q, k, v = synth_mod.make_qkv(w)
    try:
        nl.set_wait_limit_ns(1)
        _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, 2, expect_status=5)
    finally:
        nl.set_wait_limit_ns(0)
    od, ld, _ = _device_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v)
    oh, lh = _host_layer(nl, w.tile_grid, w.thr, w.sta, q, k, v, 2)
    assert _same_bits(oh, od) and _same_bits(lh, ld)
