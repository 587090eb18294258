#!/usr/bin/env python
"""Benchmark: one NABLA attention layer (mask build + block-sparse forward).

A step is one pass of the whole hot path over one synthetic layer: pool Q/K,
reduced map, row softmax + prefix selection + STA union, CSR compaction
(nabla_build_mask), then the block-sparse attention forward (bsa_fwd).  The
workload is the Wan-2.1-14B-720p-shaped layer: B=1, 40 heads, d=128, token grid
20x48x80 (76,800 tokens, 1,200 blocks), thr=0.2, STA window (1,2,2) tiles.

Metric: kept-block TFLOP/s (4*d*64^2 per kept block pair, summed over heads)
over the step time, plus ms per layer and the fraction of dense-BF16 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs the full layer on its own replica inputs
(weak scaling; the path shards by head with no data exchange); the time is the
max over ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "wan720p"
METRIC = "kept-block attn TFLOP/s & ms/layer at 76.8k tokens; % of dense BF16 peak"
ATTN_SRC = os.path.join(ROOT, "block_sparse_attention_23_b200", "csrc", "attn_kernel.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "bsa_fwd_wan720p_traffic.json")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _attn_src_sha():
    return hashlib.sha256(open(ATTN_SRC, "rb").read()).hexdigest()[:16]


def _traffic_per_launch():
    """DRAM bytes per bsa_fwd launch from a committed ncu capture, or None if the
    kernel source changed since the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    if d.get("attn_src_sha") != _attn_src_sha():
        return None
    return d.get("bytes_per_launch")


def _workload_desc(w):
    T, Hh, W = w.grid
    sta = f"STA half-window {w.sta} tiles" if w.sta else "no STA"
    return (f"{w.name}: B={w.B} H={w.H} d={w.d} grid {T}x{Hh}x{W} ({w.S} tokens, {w.nb} blocks), "
            f"thr={w.thr}, {sta}, Q,K = {w.pos_weight}*e(t,h,w) + {w.noise_weight}*z, V ~ N(0,1)")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, log_dir=None):
        self.index = index
        self.proc = None
        base = log_dir or tempfile.gettempdir()
        self.path = os.path.join(base, f"nabla_clocks_rank{index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}",
                                          f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                                          "-lms", "200"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                mx = float(parts[2].split()[0])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _init_pg(ws, backend):
    import torch.distributed as dist
    from datetime import timedelta
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def _max_over_ranks(x: float, ws: int, device) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _mask_kernel_rooflines(stage_ms, BH, nb, d, S, kept, peaks, fp64_peak, exp_peak):
    """Per-kernel rooflines of the mask build from its stage times (ms):
    pooling against HBM (Q, K read; fp64 block means written), the reduced map
    against the measured fp64 FMA rate (2*nb^2*d per head), the selection
    against the measured fp64 exp rate (one exp(L - max) per map entry, its one
    transcendental step per entry; its HBM traffic, the fp64 map read once, is
    reported beside it), the compaction against HBM (bitmap and counts read;
    row_ptr and col_idx written)."""
    nw = (nb + 31) // 32
    hbm = peaks["hbm_gbs"]
    parts = {
        "pool": ("hbm", 2.0 * BH * S * d * 2 + 2.0 * BH * nb * d * 8),
        "reduced_map": ("fp64", 2.0 * BH * nb * nb * d),
        "select": ("alu", float(BH) * nb * nb),
        "compact": ("hbm", 4.0 * BH * nb * nw + 8.0 * BH * nb + 4.0 * kept),
    }
    out = {}
    for (name, (bound, work)), ms in zip(parts.items(), stage_ms):
        if bound == "hbm":
            ach = work / (ms * 1e-3) / 1e9
            out[name] = {"bound": "hbm", "ms": float(ms), "bytes": work, "achieved": ach,
                         "peak": hbm, "unit": "GB/s", "frac": ach / hbm}
        elif bound == "alu":
            ach = work / (ms * 1e-3) / 1e9
            hbm_bytes = 8.0 * BH * nb * nb + 4.0 * BH * nb * nw + 4.0 * BH * nb
            out[name] = {"bound": "alu", "ms": float(ms), "entries": work, "achieved": ach,
                         "peak": exp_peak, "unit": "Gentry/s", "frac": ach / exp_peak,
                         "peak_source": "measured fp64 exp chains (nabla_selftest_fp64_exp_rate), "
                                        "one exp per entry",
                         "hbm_frac": hbm_bytes / (ms * 1e-3) / 1e9 / hbm}
        else:
            ach = work / (ms * 1e-3) / 1e12
            out[name] = {"bound": "fp64", "ms": float(ms), "flops": work, "achieved": ach,
                         "peak": fp64_peak, "unit": "TFLOP/s", "frac": ach / fp64_peak,
                         "peak_source": "measured fp64 FMA chains (nabla_selftest_fp64_tflops)"}
    out["what"] = ("the mask build's kernels timed one by one with events between them, "
                   "outside the timed step")
    return out


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(w, q, k, v, nrows: int, head: int = 0, seed: int = 0):
    """Time the fp64 oracle on one head's full mask plus `nrows` sampled query
    rows of that head; return (TFLOP/s of kept-block work, seconds, description)."""
    import oracle
    S, nb = w.S, w.nb
    qh, kh, vh = q[:, head:head + 1], k[:, head:head + 1], v[:, head:head + 1]
    t0 = time.perf_counter()
    mask = oracle.build_mask(qh, kh, w.tile_grid, w.thr, w.sta)
    t_mask = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(S, size=nrows, replace=False)).astype(np.int64)
    t1 = time.perf_counter()
    ro, rl = oracle.masked_attention(qh, kh, vh, mask, rows)
    t_attn = time.perf_counter() - t1
    kept_blocks = mask[0, 0].sum(axis=1)[rows // 64]
    flops = float((4.0 * w.d * 64 * kept_blocks).sum())
    t = t_attn + t_mask * nrows / S      # the mask cost of the sampled rows' share
    desc = (f"head {head}: full oracle mask ({t_mask:.2f} s, charged pro rata) + oracle "
            f"attention on {nrows} seeded query rows ({t_attn:.2f} s)")
    return flops / t / 1e12, t, desc, (mask[0, 0], rows, ro, rl)


def executed_tile_products(row_ptr, col_idx, BH, nb):
    """128 x 128 tile products the attention kernel executes for a block CSR:
    pairs of query blocks, their union of key blocks in ascending order taken
    four at a time into 256-key tiles, each computed in full (S and PV over two
    128 x 128 products per tile)."""
    rp = row_ptr[:BH * nb + 1].cpu().numpy()
    ci = col_idx[:int(rp[-1])].cpu().numpy()
    total = 0
    for bh in range(BH):
        for g0 in range(0, nb, 2):
            nq = min(2, nb - g0)
            mem = np.zeros(nb, dtype=bool)
            for i in range(nq):
                r = bh * nb + g0 + i
                mem[ci[rp[r]:rp[r + 1]]] = True
            n_u = int(mem.sum())
            total += 2 * ((n_u + 3) // 4)
    return total


def mask_parity_all_heads(w, q16, k16, gpu_row_ptr, gpu_col_idx):
    """The timed layer's mask over every head against the oracle's: rows that
    differ, and the oracle's near-cut rows (E_{k*} or E_{k*+1} within 1e-4 of
    1 - thr) and near-tie rows (cut probabilities equal to 1e-6 relative), the
    only rows allowed to differ."""
    import oracle
    t0 = time.perf_counter()
    omask, diag, _ = oracle.build_mask(q16, k16, w.tile_grid, w.thr, w.sta, with_diag=True)
    t_or = time.perf_counter() - t0
    nb = w.nb
    nrows = w.B * w.H * nb
    rp = gpu_row_ptr[:nrows + 1].cpu().numpy()
    ci = gpu_col_idx[:int(rp[-1])].cpu().numpy()
    gmask = np.zeros((nrows, nb), dtype=np.uint8)
    gmask[np.repeat(np.arange(nrows), np.diff(rp)), ci] = 1
    o = omask.reshape(nrows, nb)
    diff = (gmask != o).any(axis=1)
    dg = diag.reshape(nrows, 4)
    near_cut = oracle.near_cut_rows(dg, w.thr, 1e-4)
    near_tie = oracle.near_tie_rows(dg)
    exempt = near_cut | near_tie
    return {"rows": nrows, "rows_differing": int(diff.sum()),
            "rows_differing_not_exempt": int((diff & ~exempt).sum()),
            "near_cut_rows": int(near_cut.sum()), "near_tie_rows": int(near_tie.sum()),
            "oracle_mask_s": t_or,
            "rule": "bit-exact except near-cut / near-tie rows of the oracle"}


def bwd_executed_flops(row_ptr, col_idx, BH, nb, d):
    """FLOPs the two backward kernels execute for a block CSR: the dK/dV kernel
    pairs key blocks and visits the union of the query blocks that list either,
    two per 128-query tile, with four products per tile (S^T, dP^T, dV, dK);
    the dQ kernel pairs query blocks and visits the union of their key blocks,
    two per 128-key tile, with three (S, dP, dQ).  Each product is 128 x 128 x d."""
    rp = row_ptr[:BH * nb + 1].cpu().numpy()
    ci = col_idx[:int(rp[-1])].cpu().numpy()
    m = np.zeros((BH * nb, nb), dtype=bool)
    m[np.repeat(np.arange(BH * nb), np.diff(rp)), ci] = True
    m = m.reshape(BH, nb, nb)

    def tiles(a):   # blocks paired along axis 1, the union along axis 2, two per tile
        if a.shape[1] % 2:
            a = np.concatenate([a, np.zeros((a.shape[0], 1, a.shape[2]), dtype=bool)], axis=1)
        return int(((((a[:, 0::2] | a[:, 1::2]).sum(-1)) + 1) // 2).sum())

    tiles_q = tiles(m)
    tiles_k = tiles(np.ascontiguousarray(m.transpose(0, 2, 1)))
    return (3.0 * tiles_q + 4.0 * tiles_k) * 2.0 * 128 * 128 * d


def sweep_executed_over_kept(mask):
    """Executed / kept attention FLOPs of a static mask [B,H,nb,nb]: query
    blocks in pairs, the union of their lists in 256-key tiles."""
    BH, nb = int(np.prod(mask.shape[:-2])), mask.shape[-1]
    m = mask.reshape(BH, nb, nb).astype(bool)
    if nb % 2:
        m = np.concatenate([m, np.zeros((BH, 1, nb), dtype=bool)], axis=1)
    n_u = (m[:, 0::2] | m[:, 1::2]).sum(-1)
    tiles = int(((n_u + 3) // 4).sum())
    return 8.0 * tiles / max(int(mask.sum()), 1)


def parity_sample(gpu_row_ptr, gpu_col_idx, gpu_o, gpu_lse, nb, d, sample):
    """The bench layer's head 0 against the oracle's run above: mask rows that
    differ, and O / LSE errors on the sampled rows whose mask row agrees."""
    omask, rows, ro, rl = sample
    rp = gpu_row_ptr[:nb + 1].cpu().numpy()
    ci = gpu_col_idx[:int(rp[-1])].cpu().numpy()
    gmask = np.zeros((nb, nb), dtype=np.uint8)
    gmask[np.repeat(np.arange(nb), np.diff(rp)), ci] = 1
    same = (gmask == omask).all(axis=1)
    keep = same[rows // 64]
    go = gpu_o[0, 0].float().cpu().numpy()[rows[keep]]
    gl = gpu_lse[0, 0].cpu().numpy()[rows[keep]]
    err = np.abs(go - ro[keep])
    some = bool(keep.any())
    return {"head": 0, "mask_rows_differing": int((~same).sum()), "mask_rows": nb,
            "rows_compared": int(keep.sum()),
            "o_max_abs": float(err.max()) if some else None,
            "o_mean_abs": float(err.mean()) if some else None,
            "lse_max_abs": float(np.abs(gl - rl[keep]).max()) if some else None,
            "bars": {"o_max_abs": 2e-2, "o_mean_abs": 2e-3, "lse_max_abs": 1e-3}}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    import synth
    oracle.build()
    w = synth.WORKLOADS[args.workload]
    q, k, v = synth.make_qkv(w)
    cores = oracle.max_threads()
    nrows = args.ref_rows
    for i in range(args.warmup):
        oracle_sample(w, q, k, v, nrows, head=i % w.H, seed=i)
    vals, times, desc = [], [], ""
    for i in range(args.steps):
        val, t, desc, _ = oracle_sample(w, q, k, v, nrows, head=(args.warmup + i) % w.H,
                                     seed=1000 + i)
        vals.append(val)
        times.append(t)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": float(np.mean(times)) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": _workload_desc(w), "global_batch": w.B, "seq_len": w.S,
                   "parallelism": "cpu oracle (fp64, OpenMP)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = _init_pg(ws, "nccl")
    import synth
    import block_sparse_attention_23_b200 as nl
    nl.lib()
    w = synth.WORKLOADS[args.workload]
    if args.profile_heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.profile_heads)   # profiling subset, not a bench line
    peaks = _peaks()

    # inputs: generated on the host (pinned, for the end-to-end leg), resident copies in HBM
    q16, k16, v16 = synth.make_qkv(w, seed=args.seed + rank)
    pinned = []
    for a in (q16, k16, v16):
        t = torch.empty(a.shape, dtype=torch.bfloat16, pin_memory=True)
        t.view(torch.int16).numpy()[...] = a.view(np.int16)
        pinned.append(t)
    q, k, v = (t.to(dev) for t in pinned)
    B, H, S, d = q.shape
    nb = S // 64
    shape = nl.make_shape(B, H, S, d, w.tile_grid)
    ws_mask = nl.Workspace.create(shape, nl.OP_BUILD_MASK, dev)
    ws_fwd = nl.Workspace.create(shape, nl.OP_FWD, dev)
    cap = B * H * nb * nb
    mask_out = (torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev),
                torch.empty(cap, dtype=torch.int32, device=dev),
                torch.empty(1, dtype=torch.int32, device=dev), None)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        row_ptr, col_idx, nnz, _ = nl.nabla_build_mask(q, k, w.tile_grid, w.thr, w.sta,
                                                       workspace=ws_mask, out=mask_out)
        nl.bsa_fwd(q, k, v, row_ptr, col_idx, workspace=ws_fwd, out=(o, lse))

    step()
    torch.cuda.synchronize()
    ws_mask.check()
    ws_fwd.check()
    kept = int(mask_out[2].item())
    kept_flops = 4.0 * d * 64 * 64 * kept
    mask_bytes = 2.0 * B * H * S * d * 2 + 4.0 * kept + 4.0 * (B * H * nb + 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clocks = ClockSampler(local, args.clock_log_dir)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        e0, e1, e2 = ev[i]
        e0.record(stream)
        row_ptr, col_idx, nnz, _ = nl.nabla_build_mask(q, k, w.tile_grid, w.thr, w.sta,
                                                       workspace=ws_mask, out=mask_out)
        e1.record(stream)
        nl.bsa_fwd(q, k, v, row_ptr, col_idx, workspace=ws_fwd, out=(o, lse))
        e2.record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ws > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    mask_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in ev]))
    attn_ms = float(np.mean([b.elapsed_time(c) for _, b, c in ev]))
    total_ms_max = _max_over_ranks(total_ms, ws, dev)
    ms_per_step = total_ms_max / args.steps
    value = kept_flops * ws / (ms_per_step * 1e-3) / 1e12
    ws_mask.check()
    ws_fwd.check()
    # forwards (check, warm-up, timed) that needed the exact-reference kernel
    fwd_exact_passes = ws_fwd.exact_passes()

    # the mask build's four kernels timed one by one (events between them),
    # outside the timed region, and the device's measured fp64 FMA and exp rates
    stage = np.zeros(4)
    nl.nabla_build_mask_stage_ms(q, k, w.tile_grid, w.thr, w.sta, workspace=ws_mask, out=mask_out)
    n_stage = 5
    for _ in range(n_stage):
        stage += np.array(nl.nabla_build_mask_stage_ms(q, k, w.tile_grid, w.thr, w.sta,
                                                       workspace=ws_mask, out=mask_out))
    stage /= n_stage
    ws_mask.check()
    fp64_peak = nl.selftest_fp64_tflops()
    exp_peak = nl.selftest_fp64_exp_rate()

    # end to end through the public API with host buffers: nabla_layer_host
    # reads Q, K, V from pinned memory and writes O and LSE back to it every
    # step, streaming heads through the device in chunks so that the PCIe
    # copies overlap the mask and attention kernels of neighbouring chunks
    o_host = torch.empty(o.shape, dtype=torch.bfloat16, pin_memory=True)
    lse_host = torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
    hpc = max(1, min(args.e2e_heads_per_chunk, w.B * w.H))
    ws_host = nl.layer_host_workspace(nl.make_shape(w.B, w.H, w.S, w.d, w.tile_grid), hpc,
                                      device=dev)

    def e2e_step():
        nl.nabla_layer_host(pinned[0], pinned[1], pinned[2], w.tile_grid, w.thr, w.sta,
                            heads_per_chunk=hpc, workspace=ws_host, out=(o_host, lse_host))

    e2e_steps = max(1, min(args.steps, 5))
    e2e_step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    ws_host.check()
    e2e_ms = _max_over_ranks(a.elapsed_time(b), ws, dev) / e2e_steps
    e2e_val = kept_flops * ws / (e2e_ms * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    d2h = o_host.numel() * 2 + lse_host.numel() * 4
    e2e_chunks = (w.B * w.H + hpc - 1) // hpc
    del ws_host

    # token reordering (raster -> tile-major of one [B,H,S,d] tensor), timed on
    # its own after the layer: algorithmic bytes = read + write of the tensor
    qr = torch.empty_like(q)
    for _ in range(3):
        nl.nabla_reorder_tokens(q, w.tile_grid, nl.TO_TILE_MAJOR, out=qr)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_re = 20
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n_re):
        nl.nabla_reorder_tokens(q, w.tile_grid, nl.TO_TILE_MAJOR, out=qr)
    b.record(stream)
    torch.cuda.synchronize()
    re_ms = a.elapsed_time(b) / n_re
    re_bytes = 2.0 * q.numel() * q.element_size()
    re_gbs = re_bytes / (re_ms * 1e-3) / 1e9
    del qr

    # the same layer on raster-ordered tokens, read in place (reorder fused into
    # the pooling loads and the attention's TMA boxes and O / LSE stores)
    qr, kr, vr = (nl.nabla_reorder_tokens(t, w.tile_grid, nl.TO_RASTER) for t in (q, k, v))
    shape_r = nl.make_shape(B, H, S, d, w.tile_grid, nl.LAYOUT_RASTER)
    ws_mask_r = nl.Workspace.create(shape_r, nl.OP_BUILD_MASK, dev)
    ws_fwd_r = nl.Workspace.create(shape_r, nl.OP_FWD, dev)
    o_r, lse_r = torch.empty_like(q), torch.empty_like(lse)

    # separate CSR buffers: the step's own CSR stays intact for the parity sample
    mask_out_x = tuple(t.clone() if t is not None else None for t in mask_out)

    def raster_step():
        rp, ci, _, _ = nl.nabla_build_mask(qr, kr, w.tile_grid, w.thr, w.sta, workspace=ws_mask_r,
                                           out=mask_out_x, layout=nl.LAYOUT_RASTER)
        nl.bsa_fwd(qr, kr, vr, rp, ci, workspace=ws_fwd_r, out=(o_r, lse_r), tile_grid=w.tile_grid,
                   layout=nl.LAYOUT_RASTER)

    for _ in range(2):
        raster_step()
    torch.cuda.synchronize()
    n_ra = 3
    a.record(stream)
    for _ in range(n_ra):
        raster_step()
    b.record(stream)
    torch.cuda.synchronize()
    ws_mask_r.check()
    ws_fwd_r.check()
    raster_ms = a.elapsed_time(b) / n_ra
    del qr, kr, vr, o_r, lse_r

    # block energy over the step's own block list (the retained-mass check of
    # the NABLA mask) and one calibration vote pass over the energy map
    energy = torch.empty((B, H, nb, nb), dtype=torch.float32, device=dev)
    bmass = torch.empty((B, H, nb), dtype=torch.float32, device=dev)
    votes = torch.zeros((B, H, nb, nb), dtype=torch.int32, device=dev)
    row_ptr, col_idx = mask_out[0], mask_out[1]
    # dense LSE (every block listed) so that E is the true block attention map
    # and the retained mass of the NABLA list is its fidelity
    full_rp = torch.arange(0, B * H * nb + 1, dtype=torch.int64, device=dev).mul_(nb).to(torch.int32)
    full_ci = torch.arange(nb, dtype=torch.int32, device=dev).repeat(B * H * nb)
    o_dense = torch.empty_like(q)
    lse_dense = torch.empty_like(lse)
    nl.bsa_fwd(q, k, v, full_rp, full_ci, workspace=ws_fwd, out=(o_dense, lse_dense))
    del full_rp, full_ci, o_dense

    def energy_call():
        nl.nabla_block_energy(q, k, lse_dense, row_ptr, col_idx, workspace=ws_fwd,
                              out=(energy, bmass))

    for _ in range(2):
        energy_call()
    n_en = 3
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n_en):
        energy_call()
    b.record(stream)
    torch.cuda.synchronize()
    en_ms = a.elapsed_time(b) / n_en
    ws_fwd.check()
    en_flops = 2.0 * d * 64 * 64 * kept
    en_tflops = en_flops / (en_ms * 1e-3) / 1e12
    # its floor is the exponential unit: 4,096 exponentials per kept block
    en_gexp = 4096.0 * kept / (en_ms * 1e-3) / 1e9
    ex2_peak = nl.selftest_ex2_rate()
    retained = float(bmass.mean().item())
    retained_min = float(bmass.min().item())
    nl.nabla_calib_accumulate(energy, 0.2, votes)
    a.record(stream)
    nl.nabla_calib_accumulate(energy, 0.2, votes)
    b.record(stream)
    torch.cuda.synchronize()
    cal_ms = a.elapsed_time(b)
    del energy, votes

    # backward over the step's block list (dO ~ N(0,1)), outside the step;
    # algorithmic FLOPs = the five 64x64xd products per kept block pair
    g = torch.Generator(device=dev).manual_seed(args.seed + 17)
    dout = torch.randn(q.shape, device=dev, generator=g).to(torch.bfloat16)
    ws_bwd = nl.Workspace.create(shape, nl.OP_BWD, dev)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))

    def bwd_call():
        nl.bsa_bwd(q, k, v, o, dout, lse, row_ptr, col_idx, workspace=ws_bwd, out=grads)

    bwd_call()
    torch.cuda.synchronize()
    ws_bwd.check()
    n_bw = 3
    a.record(stream)
    for _ in range(n_bw):
        bwd_call()
    b.record(stream)
    torch.cuda.synchronize()
    ws_bwd.check()
    bwd_ms = a.elapsed_time(b) / n_bw
    bwd_flops = 2.5 * kept_flops
    bwd_tflops = bwd_flops / (bwd_ms * 1e-3) / 1e12
    bwd_exec = bwd_executed_flops(mask_out[0], mask_out[1], B * H, nb, d)
    del dout, grads

    # XAttention scorer (stride 8) + the same selection, outside the step;
    # algorithmic FLOPs = two passes over the strided score matrix
    ws_x = nl.Workspace.create(shape, nl.OP_BUILD_XATTN, dev)

    def xattn_call():
        nl.nabla_build_mask_xattn(q, k, w.thr, 8, tile_grid=w.tile_grid, sta=w.sta,
                                  workspace=ws_x, out=mask_out_x)

    xattn_call()
    torch.cuda.synchronize()
    ws_x.check()
    x_kept = int(mask_out_x[2].item())
    n_x = 3
    a.record(stream)
    for _ in range(n_x):
        xattn_call()
    b.record(stream)
    torch.cuda.synchronize()
    ws_x.check()
    x_ms = a.elapsed_time(b) / n_x
    x_flops = 4.0 * S * S * d * B * H / 8
    x_tflops = x_flops / (x_ms * 1e-3) / 1e12

    # static-mask attention over a density sweep (i.i.d. N(0,1) Q, K, V on the
    # 32,768-token sweep shape, Bernoulli block masks, diagonal forced), outside the step
    sweep = []
    if not args.profile_heads:
        ws_ = synth.WORKLOADS["sweep"]
        qs16, ks16, vs16 = synth.make_qkv(ws_, seed=args.seed)
        qs, ks, vs = (torch.from_numpy(t.view(np.int16)).view(torch.bfloat16).to(dev)
                      for t in (qs16, ks16, vs16))
        shape_s = nl.make_shape(ws_.B, ws_.H, ws_.S, ws_.d)
        wsw = nl.Workspace.create(shape_s, nl.OP_FWD_WITH_MASK, dev)
        os_, ls_ = torch.empty_like(qs), torch.empty((ws_.B, ws_.H, ws_.S), dtype=torch.float32,
                                                     device=dev)
        for pden in ws_.densities:
            mk = torch.from_numpy(synth.make_bernoulli_mask(0, ws_.B * ws_.H, ws_.nb, pden)).to(dev)
            for _ in range(2):
                nl.bsa_fwd_with_mask(qs, ks, vs, mk, workspace=wsw, out=(os_, ls_))
            a.record(stream)
            for _ in range(3):
                nl.bsa_fwd_with_mask(qs, ks, vs, mk, workspace=wsw, out=(os_, ls_))
            b.record(stream)
            torch.cuda.synchronize()
            wsw.check()
            ms_ = a.elapsed_time(b) / 3
            kept_s = int(mk.sum().item())
            eok = sweep_executed_over_kept(mk.cpu().numpy())
            kt = 4.0 * ws_.d * 64 * 64 * kept_s / (ms_ * 1e-3) / 1e12
            sweep.append({"density": pden, "kept_fraction": kept_s / mk.numel(), "ms": ms_,
                          "kept_tflops": kt, "kept_frac_of_sustained": kt / peaks["bf16_tflops_sustained"],
                          "executed_over_kept": eok, "executed_tflops": kt * eok})
        del qs, ks, vs, os_, ls_

    attn_tflops = kept_flops / (attn_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    exec_tiles = executed_tile_products(mask_out[0], mask_out[1], B * H, nb)
    exec_flops = 4.0 * d * 128 * 128 * exec_tiles
    traffic = _traffic_per_launch() if (args.workload == WORKLOAD and not args.profile_heads) else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": _workload_desc(w), "global_batch": B * ws, "seq_len": S,
                   "heads": H, "head_dim": d,
                   "parallelism": "replicas" if ws > 1 else "single GPU",
                   "l2": f"inputs (Q,K,V {3 * q.numel() * 2 / 1e9:.2f} GB per rank) larger than L2; no flush",
                   "kept_blocks": kept, "density": kept / (B * H * nb * nb),
                   "mask_arith": "fp64 pooling, reduced map and row probabilities; exact "
                                 "fixed-point prefix masses",
                   "attn_arith": "bf16 MMA, fp32 accumulate"},
        "ms_per_layer": ms_per_step, "mask_ms": mask_ms, "attn_ms": attn_ms,
        "attn_kept_tflops": attn_tflops,
        "attn_executed": {"tile_products": exec_tiles, "flops": exec_flops,
                          "tflops": exec_flops / (attn_ms * 1e-3) / 1e12,
                          "over_kept": exec_flops / kept_flops,
                          "what": "128x128 S and PV products the kernel runs (union of two "
                                  "query blocks in 256-key tiles), counted on the host"},
        "attn_exact_passes": {"count": fwd_exact_passes, "forwards": 1 + args.warmup + args.steps,
                              "what": "forwards in which some query tile outgrew its fixed "
                                      "softmax reference and ran the exact-reference pass"},
        "pct_of_dense_bf16_peak": {"attn_vs_sustained": attn_tflops / peak,
                                   "attn_vs_burst": attn_tflops / peaks["bf16_tflops"],
                                   "layer_vs_sustained": value / ws / peak},
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "traffic": traffic, "kernel": "bsa_fwd_kernel",
                     "peak_source": f"{peaks['source']} bf16 sustained (cuBLAS, power-capped)"},
        "mask_roofline": {"bound": "hbm", "achieved": mask_bytes / (mask_ms * 1e-3) / 1e9,
                          "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": mask_bytes / (mask_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                          "bytes": mask_bytes},
        "mask_kernels": _mask_kernel_rooflines(stage, B * H, nb, d, S, kept, peaks, fp64_peak,
                                               exp_peak),
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "call": "nabla_layer_host", "heads_per_chunk": hpc, "chunks": e2e_chunks},
        "reorder": {"bound": "hbm", "ms": re_ms, "achieved": re_gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": re_gbs / peaks["hbm_gbs"], "bytes": re_bytes,
                    "what": "raster -> tile-major of one [B,H,S,d] bf16 tensor, outside the step"},
        "block_energy": {"bound": "alu", "ms": en_ms, "achieved": en_gexp, "peak": ex2_peak,
                         "unit": "Gexp/s", "frac": en_gexp / ex2_peak,
                         "peak_source": "measured ex2.approx chains (nabla_selftest_ex2_rate), "
                                        "4,096 exponentials per kept block",
                         "tensor": {"achieved": en_tflops, "peak": peak, "unit": "TFLOP/s",
                                    "frac": en_tflops / peak},
                         "flops": en_flops, "blocks": kept,
                         "mean_true_mass_retained_by_mask": retained,
                         "min_true_mass_retained_by_mask": retained_min,
                         "what": "E over the step's kept blocks (QK^T + exp + block sums), "
                                 "outside the step; FLOPs = 2*d*64*64 per block"},
        "calib_accumulate_ms": cal_ms,
        "static_mask_sweep": {"workload": "32,768 tokens, 24 heads, d 128, Q,K,V ~ N(0,1), "
                                          "Bernoulli(p) block masks with the diagonal forced; "
                                          "mask compaction + attention per call",
                              "points": sweep},
        "xattn_mask": {"bound": "tensor", "ms": x_ms, "achieved": x_tflops, "peak": peak,
                       "unit": "TFLOP/s", "frac": x_tflops / peak, "flops": x_flops,
                       "kept_blocks": x_kept, "density": x_kept / (B * H * nb * nb),
                       "what": "XAttention antidiagonal scores (stride 8, two passes) + selection "
                               "at the layer's thr and STA, outside the step"},
        "bwd": {"bound": "tensor", "ms": bwd_ms, "achieved": bwd_tflops, "peak": peak,
                "unit": "TFLOP/s", "frac": bwd_tflops / peak, "flops": bwd_flops,
                "executed": {"flops": bwd_exec, "over_algorithmic": bwd_exec / bwd_flops,
                             "tflops": bwd_exec / (bwd_ms * 1e-3) / 1e12,
                             "frac_of_sustained": bwd_exec / (bwd_ms * 1e-3) / 1e12 / peak,
                             "what": "products the two kernels run: 4 per 128-query tile of the "
                                     "dK/dV kernel, 3 per 128-key tile of the dQ kernel, tiles "
                                     "over unions of paired blocks, counted on the host"},
                "what": "bsa_bwd (D, column bitmaps, dK/dV and dQ kernels) over the step's "
                        "block list, outside the step; FLOPs = 10*d*64*64 per kept block"},
        "raster_layer": {"ms_per_layer": raster_ms, "vs_tile_major": raster_ms / ms_per_step,
                         "what": "mask + attention on raster-ordered Q, K, V (O, LSE raster), "
                                 "Q read by 5D boxes, K and V reordered to tile-major copies in the "
                                 "workspace first; outside the step"},
        "gpu_launches": 6 * args.steps,
        "clocks": clk,
    }
    if args.profile_heads:
        line["config"]["profiling_subset_heads"] = args.profile_heads
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        val, t, desc, sample = oracle_sample(w, q16, k16, v16, args.ref_rows, head=0, seed=0)
        line["cpu_baseline"] = {"value": val, "unit": "TFLOP/s", "cores": oracle.max_threads(),
                                "kind": "oracle", "sample": desc}
        line["parity_sample"] = parity_sample(mask_out[0], mask_out[1], o, lse, nb, d, sample)
        line["parity_sample"]["mask_all_heads"] = mask_parity_all_heads(w, q16, k16, mask_out[0],
                                                                        mask_out[1])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-rows", type=int, default=2048,
                    help="oracle attention rows per CPU sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-heads-per-chunk", type=int, default=4,
                    help="heads per pipeline chunk of the host-buffer (e2e) leg")
    ap.add_argument("--clock-log-dir", default=None,
                    help="directory for the raw nvidia-smi clock samples (default: the temp dir)")
    ap.add_argument("--profile-heads", type=int, default=0,
                    help="profiling only: run the layer with this many heads")
    ap.add_argument("--workload", default=WORKLOAD, choices=["wan720p", "hunyuan720p", "small"],
                    help="layer to time (default: the Wan 2.1 720p-shaped layer)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
