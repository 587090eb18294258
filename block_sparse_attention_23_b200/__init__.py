"""Python binding for libnabla (NABLA block-sparse attention on B200, sm_100a).

Argument marshalling only: every step of the mask builder and the attention
forward runs in the CUDA kernels of ``libnabla.so`` (built from ``csrc/`` by
``buildlib.py``).  PyTorch is used for device memory and the current stream.
There is no CPU fallback: if the library is missing or no CUDA device is
present, the calls raise.

The names mirror the C ABI in ``include/nabla.h``:

* ``nabla_build_mask(q, k, tile_grid, thr, sta=None, ...)`` -> block CSR
* ``bsa_fwd(q, k, v, row_ptr, col_idx, scale=None)`` -> (O, LSE)
* ``bsa_fwd_with_mask(q, k, v, mask_u8, scale=None)`` -> (O, LSE)
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnabla.so")

NABLA_OK = 0
STATUS_NAMES = {0: "NABLA_OK", 1: "NABLA_ERR_INVALID_ARG", 2: "NABLA_ERR_UNSUPPORTED",
                3: "NABLA_ERR_CAPACITY", 4: "NABLA_ERR_CUDA", 5: "NABLA_ERR_TIMEOUT",
                6: "NABLA_ERR_BAD_INDEX"}
OP_BUILD_MASK, OP_FWD, OP_FWD_WITH_MASK, OP_BWD, OP_BUILD_XATTN = 0, 1, 2, 3, 4
LAYOUT_TILE_MAJOR, LAYOUT_RASTER = 0, 1
EXPORTED = ["nabla_workspace_size", "nabla_workspace_init", "nabla_query_status",
            "nabla_build_mask", "bsa_fwd", "bsa_fwd_with_mask", "nabla_last_error",
            "nabla_version", "nabla_set_wait_limit_ns", "nabla_selftest_mma",
            "bsa_fwd_with_mask_static", "nabla_reorder_tokens", "nabla_block_energy",
            "nabla_calib_accumulate", "nabla_calib_finalize", "bsa_bwd",
            "nabla_build_mask_xattn", "nabla_layer_host_workspace_size", "nabla_layer_host",
            "nabla_layer_host_chunks", "nabla_set_exact_reference", "nabla_query_exact_passes",
            "nabla_build_mask_stage_ms", "nabla_selftest_fp64_tflops",
            "nabla_selftest_fp64_exp_rate", "nabla_selftest_ex2_rate", "nabla_selftest_mma_pair",
            "nabla_set_pair_mode"]
TO_TILE_MAJOR, TO_RASTER = 0, 1


class NablaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("S", ctypes.c_int32),
                ("d", ctypes.c_int32), ("Tt", ctypes.c_int32), ("Th", ctypes.c_int32),
                ("Tw", ctypes.c_int32), ("layout", ctypes.c_int32)]


class _MaskParams(ctypes.Structure):
    _fields_ = [("thr", ctypes.c_float), ("use_sta", ctypes.c_int32), ("wt", ctypes.c_int32),
                ("wh", ctypes.c_int32), ("ww", ctypes.c_int32), ("topk", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    from .buildlib import build as _build
    return _build(force=force)


def lib() -> ctypes.CDLL:
    """Load libnabla.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m block_sparse_attention_23_b200.buildlib`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                     ctypes.c_float, ctypes.c_size_t)
            sp = ctypes.POINTER(_Shape)
            L.nabla_workspace_size.restype = sz
            L.nabla_workspace_size.argtypes = [sp, i32]
            L.nabla_workspace_init.restype = i32
            L.nabla_workspace_init.argtypes = [vp, vp]
            L.nabla_query_status.restype = i32
            L.nabla_query_status.argtypes = [vp, vp]
            L.nabla_build_mask.restype = i32
            L.nabla_build_mask.argtypes = [sp, ctypes.POINTER(_MaskParams), vp, vp, vp, vp, vp,
                                           i64, vp, vp, vp]
            L.bsa_fwd.restype = i32
            L.bsa_fwd.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
            L.bsa_fwd_with_mask.restype = i32
            L.bsa_fwd_with_mask.argtypes = [sp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
            L.nabla_last_error.restype = ctypes.c_char_p
            L.nabla_last_error.argtypes = []
            L.nabla_version.restype = i32
            L.nabla_version.argtypes = []
            L.nabla_set_wait_limit_ns.restype = None
            L.nabla_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
            L.nabla_set_exact_reference.restype = None
            L.nabla_set_exact_reference.argtypes = [i32]
            L.nabla_query_exact_passes.restype = i32
            L.nabla_query_exact_passes.argtypes = [vp, vp]
            L.nabla_selftest_mma.restype = i32
            L.nabla_selftest_mma.argtypes = [i32, vp, vp, vp, vp, vp]
            L.nabla_reorder_tokens.restype = i32
            L.nabla_reorder_tokens.argtypes = [sp, i32, vp, vp, vp]
            L.nabla_block_energy.restype = i32
            L.nabla_block_energy.argtypes = [sp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
            L.nabla_calib_accumulate.restype = i32
            L.nabla_calib_accumulate.argtypes = [sp, vp, f32, vp, vp]
            L.nabla_calib_finalize.restype = i32
            L.nabla_calib_finalize.argtypes = [sp, vp, i32, vp, vp]
            L.nabla_build_mask_xattn.restype = i32
            L.nabla_build_mask_xattn.argtypes = [sp, ctypes.POINTER(_MaskParams), i32, vp, vp, vp,
                                                 vp, vp, vp, i64, vp, vp, vp]
            L.bsa_bwd.restype = i32
            L.bsa_bwd.argtypes = [sp, vp, vp, vp, vp, vp, vp, vp, vp, f32, vp, vp, vp, vp, vp]
            L.bsa_fwd_with_mask_static.restype = i32
            L.bsa_fwd_with_mask_static.argtypes = [sp, vp, vp, vp, vp, f32, vp, vp, vp, vp]
            L.nabla_layer_host_workspace_size.restype = sz
            L.nabla_layer_host_workspace_size.argtypes = [sp, i32]
            L.nabla_layer_host_chunks.restype = ctypes.c_int64
            L.nabla_layer_host_chunks.argtypes = [ctypes.c_int64, i32, vp, ctypes.c_int64]
            L.nabla_build_mask_stage_ms.restype = i32
            L.nabla_build_mask_stage_ms.argtypes = [sp, ctypes.POINTER(_MaskParams), vp, vp, vp,
                                                    vp, ctypes.c_int64, vp, vp, vp, vp]
            L.nabla_set_pair_mode.restype = None
            L.nabla_set_pair_mode.argtypes = [i32]
            L.nabla_selftest_mma_pair.restype = i32
            L.nabla_selftest_mma_pair.argtypes = [i32, vp, vp, vp, vp, vp]
            L.nabla_selftest_fp64_tflops.restype = i32
            L.nabla_selftest_fp64_tflops.argtypes = [vp, vp]
            L.nabla_selftest_fp64_exp_rate.restype = i32
            L.nabla_selftest_fp64_exp_rate.argtypes = [vp, vp]
            L.nabla_selftest_ex2_rate.restype = i32
            L.nabla_selftest_ex2_rate.argtypes = [vp, vp]
            L.nabla_layer_host.restype = i32
            L.nabla_layer_host.argtypes = [sp, ctypes.POINTER(_MaskParams), vp, vp, vp, vp, vp,
                                           i32, vp, vp]
            _lib = L
    return _lib


def _check(status: int) -> None:
    if status != NABLA_OK:
        raise NablaError(status, lib().nabla_last_error().decode())


def _torch():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("libnabla needs a CUDA device; there is no CPU path")
    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def make_shape(B: int, H: int, S: int, d: int, tile_grid=(0, 0, 0),
               layout: int = LAYOUT_TILE_MAJOR) -> _Shape:
    Tt, Th, Tw = tile_grid if tile_grid is not None else (0, 0, 0)
    return _Shape(B, H, S, d, Tt, Th, Tw, int(layout))


def workspace_size(shape: _Shape, op: int) -> int:
    n = lib().nabla_workspace_size(ctypes.byref(shape), op)
    if n == 0:
        raise NablaError(1, lib().nabla_last_error().decode())
    return int(n)


@dataclass
class Workspace:
    """Caller-owned device workspace with a zeroed status header."""
    buf: "object"
    op: int

    @classmethod
    def create(cls, shape: _Shape, op: int, device=None, stream=None, nbytes=None) -> "Workspace":
        torch = _torch()
        n = workspace_size(shape, op) if nbytes is None else int(nbytes)
        if n == 0:
            raise NablaError(1, lib().nabla_last_error().decode())
        buf = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
        _check(lib().nabla_workspace_init(_ptr(buf), _stream(stream)))
        return cls(buf, op)

    def query_status(self, stream=None) -> int:
        """Synchronise, read and clear the device status word (0 = OK)."""
        return int(lib().nabla_query_status(_ptr(self.buf), _stream(stream)))

    def check(self, stream=None) -> None:
        _check(self.query_status(stream))

    def exact_passes(self, stream=None) -> int:
        """Synchronise and return how many forwards on this workspace needed the
        exact-reference kernel."""
        n = int(lib().nabla_query_exact_passes(_ptr(self.buf), _stream(stream)))
        if n < 0:
            raise NablaError(4, lib().nabla_last_error().decode())
        return n


def _check_workspace(workspace: Workspace, shape: _Shape, op: int) -> None:
    """The library writes up to workspace_size(shape, op) bytes (raster token
    order needs room for K/V copies): refuse a smaller buffer."""
    need = workspace_size(shape, op)
    if workspace.buf.numel() < need:
        raise ValueError(f"workspace holds {workspace.buf.numel()} bytes; this call needs {need}")


def _shape_of(q, tile_grid=(0, 0, 0), layout: int = LAYOUT_TILE_MAJOR) -> _Shape:
    if q.dim() != 4:
        raise ValueError("q must be [B, H, S, d]")
    B, H, S, d = q.shape
    return make_shape(B, H, S, d, tile_grid, layout)


def _bf16_contig(*ts):
    torch = _torch()
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous bf16 CUDA tensors [B, H, S, d]")


def nabla_build_mask(q, k, tile_grid, thr: float, sta: Optional[Tuple[int, int, int]] = None,
                     want_mask: bool = False, col_capacity: Optional[int] = None,
                     workspace: Optional[Workspace] = None, out=None, stream=None,
                     topk: int = 0, layout: int = LAYOUT_TILE_MAJOR):
    """NABLA block mask of (q, k) as block CSR (``topk`` > 0: fixed top-k rule;
    ``layout`` = LAYOUT_RASTER reads raster-ordered tokens in place).

    Returns (row_ptr int32 [B*H*nb+1], col_idx int32 [capacity], nnz int32 [1],
    mask uint8 [B,H,nb,nb] or None).  Only the first nnz entries of col_idx
    are meaningful.  ``out`` may pass preallocated (row_ptr, col_idx, nnz, mask)."""
    torch = _torch()
    _bf16_contig(q, k)
    shape = _shape_of(q, tile_grid, layout)
    B, H, S, d = q.shape
    nb = S // 64
    if workspace is None:
        workspace = Workspace.create(shape, OP_BUILD_MASK, q.device, stream)
    if out is None:
        cap = col_capacity if col_capacity is not None else B * H * nb * nb
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=q.device)
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=q.device)
        nnz = torch.empty(1, dtype=torch.int32, device=q.device)
        mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=q.device) if want_mask else None
    else:
        row_ptr, col_idx, nnz, mask = out
        cap = col_idx.numel() if col_capacity is None else col_capacity
    prm = _MaskParams(float(thr), 1 if sta is not None else 0,
                      *(sta if sta is not None else (0, 0, 0)), int(topk))
    _check(lib().nabla_build_mask(ctypes.byref(shape), ctypes.byref(prm), _ptr(q), _ptr(k),
                                  _ptr(mask), _ptr(row_ptr), _ptr(col_idx), int(cap), _ptr(nnz),
                                  _ptr(workspace.buf), _stream(stream)))
    return row_ptr, col_idx, nnz, mask


def nabla_build_mask_stage_ms(q, k, tile_grid, thr: float, sta=None, workspace=None, out=None,
                              stream=None, topk: int = 0):
    """Diagnostic: one mask build with events between its kernels.  Returns the
    milliseconds of (pooling, reduced map, selection, compaction); synchronises."""
    torch = _torch()
    _bf16_contig(q, k)
    shape = _shape_of(q, tile_grid, LAYOUT_TILE_MAJOR)
    B, H, S, d = q.shape
    nb = S // 64
    if workspace is None:
        workspace = Workspace.create(shape, OP_BUILD_MASK, q.device, stream)
    if out is None:
        out = (torch.empty(B * H * nb + 1, dtype=torch.int32, device=q.device),
               torch.empty(B * H * nb * nb, dtype=torch.int32, device=q.device),
               torch.empty(1, dtype=torch.int32, device=q.device), None)
    row_ptr, col_idx, nnz = out[0], out[1], out[2]
    prm = _MaskParams(float(thr), 1 if sta is not None else 0,
                      *(sta if sta is not None else (0, 0, 0)), int(topk))
    ms = (ctypes.c_float * 4)()
    _check(lib().nabla_build_mask_stage_ms(ctypes.byref(shape), ctypes.byref(prm), _ptr(q),
                                           _ptr(k), _ptr(row_ptr), _ptr(col_idx),
                                           int(col_idx.numel()), _ptr(nnz), _ptr(workspace.buf),
                                           _stream(stream), ms))
    return tuple(float(x) for x in ms)


def selftest_fp64_tflops(stream=None) -> float:
    """Diagnostic: the device's measured fp64 FMA rate in TFLOP/s (synchronises)."""
    out = ctypes.c_double(0.0)
    _check(lib().nabla_selftest_fp64_tflops(_stream(stream), ctypes.byref(out)))
    return float(out.value)


def selftest_fp64_exp_rate(stream=None) -> float:
    """Diagnostic: the device's measured fp64 exp throughput in Gexp/s (synchronises)."""
    out = ctypes.c_double(0.0)
    _check(lib().nabla_selftest_fp64_exp_rate(_stream(stream), ctypes.byref(out)))
    return float(out.value)


def selftest_ex2_rate(stream=None) -> float:
    """Diagnostic: the device's measured fp32 ex2.approx throughput in Gexp/s (synchronises)."""
    out = ctypes.c_double(0.0)
    _check(lib().nabla_selftest_ex2_rate(_stream(stream), ctypes.byref(out)))
    return float(out.value)


def bsa_fwd(q, k, v, row_ptr, col_idx, scale: Optional[float] = None,
            workspace: Optional[Workspace] = None, out=None, stream=None, tile_grid=None,
            layout: int = LAYOUT_TILE_MAJOR):
    """Block-sparse attention forward over a block CSR.  Returns (O bf16, LSE fp32).
    ``layout`` = LAYOUT_RASTER (with ``tile_grid``) takes and returns raster-ordered tokens."""
    torch = _torch()
    _bf16_contig(q, k, v)
    shape = _shape_of(q, tile_grid, layout)
    if workspace is None:
        workspace = Workspace.create(shape, OP_FWD, q.device, stream)
    _check_workspace(workspace, shape, OP_FWD)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(lib().bsa_fwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(row_ptr),
                         _ptr(col_idx), float(scale or 0.0), _ptr(o), _ptr(lse),
                         _ptr(workspace.buf), _stream(stream)))
    return o, lse


def bsa_fwd_with_mask(q, k, v, mask_u8, scale: Optional[float] = None,
                      workspace: Optional[Workspace] = None, out=None, stream=None,
                      tile_grid=None, layout: int = LAYOUT_TILE_MAJOR):
    """Block-sparse attention forward with a static uint8 block mask [B,H,nb,nb]."""
    torch = _torch()
    _bf16_contig(q, k, v)
    shape = _shape_of(q, tile_grid, layout)
    if mask_u8.dtype != torch.uint8 or not mask_u8.is_cuda or not mask_u8.is_contiguous():
        raise ValueError("mask must be a contiguous uint8 CUDA tensor [B, H, nb, nb]")
    if workspace is None:
        workspace = Workspace.create(shape, OP_FWD_WITH_MASK, q.device, stream)
    _check_workspace(workspace, shape, OP_FWD_WITH_MASK)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(lib().bsa_fwd_with_mask(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(mask_u8), float(scale or 0.0), _ptr(o), _ptr(lse),
                                   _ptr(workspace.buf), _stream(stream)))
    return o, lse


def set_wait_limit_ns(ns: int) -> None:
    lib().nabla_set_wait_limit_ns(int(ns))


def set_exact_reference(on: bool) -> None:
    """Process-wide: run every forward's exact-reference kernel alone."""
    lib().nabla_set_exact_reference(1 if on else 0)


def selftest_mma(variant: int, a, b, workspace: Optional[Workspace] = None, stream=None):
    """One 128x128x128 tcgen05 product (layout check); returns C fp32 [128,128]."""
    torch = _torch()
    if workspace is None:
        workspace = Workspace.create(make_shape(1, 1, 64, 64), OP_FWD, a.device, stream)
    c = torch.empty((128, 128), dtype=torch.float32, device=a.device)
    _check(lib().nabla_selftest_mma(int(variant), _ptr(a), _ptr(b), _ptr(c), _ptr(workspace.buf),
                                    _stream(stream)))
    workspace.check(stream)
    return c


PAIR_NEVER, PAIR_BUILDER_LISTS, PAIR_ALWAYS = 0, 1, 2


def set_pair_mode(mode: int) -> None:
    """Kernel for the forward's fixed-reference pass (d = 128, tile-major):
    PAIR_NEVER (the default: one CTA per two query blocks), PAIR_BUILDER_LISTS
    (CTA pairs for mask-builder block lists) or PAIR_ALWAYS.  Process-wide."""
    lib().nabla_set_pair_mode(int(mode))


def selftest_mma_pair(variant: int, a, b, workspace: Optional[Workspace] = None, stream=None):
    """One product over a pair of CTAs (layout check); returns C fp32
    [256,256] (variant 0: A B^T) or [256,128] (variant 1: P V)."""
    torch = _torch()
    if workspace is None:
        workspace = Workspace.create(make_shape(1, 1, 64, 64), OP_FWD, a.device, stream)
    c = torch.empty((256, 256 if variant == 0 else 128), dtype=torch.float32, device=a.device)
    _check(lib().nabla_selftest_mma_pair(int(variant), _ptr(a), _ptr(b), _ptr(c),
                                         _ptr(workspace.buf), _stream(stream)))
    workspace.check(stream)
    return c


def bsa_fwd_with_mask_static(q, k, v, mask_u8, scale: Optional[float] = None, out=None,
                             status_out=None, stream=None, tile_grid=None,
                             layout: int = LAYOUT_TILE_MAJOR):
    """Static-mask attention forward that allocates no device memory inside the
    library and takes no workspace: for callers (memory-pool runtimes, code
    inside another framework's graph capture, fixed-budget hosts) that cannot
    allocate.  Its scratch is a fixed 32 MiB array owned by the library and
    shared by all calls, so calls that overlap on the GPU must not be issued.
    Returns (O, LSE); ``out`` may pass preallocated (O, LSE)."""
    torch = _torch()
    _bf16_contig(q, k, v)
    shape = _shape_of(q, tile_grid, layout)
    if out is None:
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    _check(lib().bsa_fwd_with_mask_static(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                          _ptr(mask_u8), float(scale or 0.0), _ptr(o), _ptr(lse),
                                          _ptr(status_out), _stream(stream)))
    return o, lse


def layer_host_workspace(shape: _Shape, heads_per_chunk: int, device=None,
                         stream=None) -> Workspace:
    """Device workspace for nabla_layer_host with this shape and chunking."""
    n = lib().nabla_layer_host_workspace_size(ctypes.byref(shape), int(heads_per_chunk))
    return Workspace.create(shape, OP_BUILD_MASK, device, stream, nbytes=n)


def layer_host_chunks(heads: int, heads_per_chunk: int):
    """Chunk sizes (heads) nabla_layer_host streams B*H = ``heads`` heads in."""
    n = int(lib().nabla_layer_host_chunks(int(heads), int(heads_per_chunk), None, 0))
    buf = (ctypes.c_int32 * max(n, 1))()
    lib().nabla_layer_host_chunks(int(heads), int(heads_per_chunk), buf, n)
    return [int(buf[i]) for i in range(n)]


def nabla_layer_host(q, k, v, tile_grid, thr: float, sta: Optional[Tuple[int, int, int]] = None,
                     topk: int = 0, heads_per_chunk: int = 4,
                     workspace: Optional[Workspace] = None, out=None, stream=None):
    """One NABLA layer (mask + block-sparse forward, scale 1/sqrt(d)) on host
    tensors: q, k, v contiguous bf16 CPU tensors [B,H,S,d] (pinned for
    copy/compute overlap).  Heads stream through the device in chunks of at
    most ``heads_per_chunk`` (``layer_host_chunks`` gives the schedule).  Returns host (O bf16, LSE fp32); ``out`` may pass
    preallocated host (O, LSE).  The call only queues the work: synchronise
    ``stream`` (the current stream by default) before reading the outputs."""
    torch = _torch()
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("q, k, v must be contiguous bf16 host tensors [B, H, S, d]")
    B, H, S, d = q.shape
    shape = make_shape(B, H, S, d, tile_grid)
    if workspace is None:
        workspace = layer_host_workspace(shape, heads_per_chunk, stream=stream)
    if out is None:
        pin = q.is_pinned()
        o = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=pin)
        lse = torch.empty((B, H, S), dtype=torch.float32, pin_memory=pin)
    else:
        o, lse = out
        if o.is_cuda or lse.is_cuda or not (o.is_contiguous() and lse.is_contiguous()):
            raise ValueError("out must be contiguous host tensors")
    prm = _MaskParams(float(thr), 1 if sta is not None else 0,
                      *(sta if sta is not None else (0, 0, 0)), int(topk))
    _check(lib().nabla_layer_host(ctypes.byref(shape), ctypes.byref(prm), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(o), _ptr(lse), int(heads_per_chunk),
                                  _ptr(workspace.buf), _stream(stream)))
    return o, lse


def nabla_reorder_tokens(x, tile_grid, direction: int = TO_TILE_MAJOR, out=None, stream=None):
    """Permute the token axis of a [B,H,S,d] bf16 tensor between raster (t,h,w)
    order and tile-major order (4x4x4 tiles, one per 64-token block)."""
    torch = _torch()
    _bf16_contig(x)
    shape = _shape_of(x, tile_grid)
    y = torch.empty_like(x) if out is None else out
    _check(lib().nabla_reorder_tokens(ctypes.byref(shape), int(direction), _ptr(x), _ptr(y),
                                      _stream(stream)))
    return y


def nabla_block_energy(q, k, lse, row_ptr, col_idx, scale: Optional[float] = None,
                       workspace: Optional[Workspace] = None, out=None, want_block_mass=True,
                       stream=None):
    """Per-block attention energy E [B,H,nb,nb] fp32 over the blocks of a CSR
    (zeros elsewhere), and the row sums of the listed E [B,H,nb] (or None)."""
    torch = _torch()
    _bf16_contig(q, k)
    shape = _shape_of(q)
    B, H, S, _ = q.shape
    nb = S // 64
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, S):
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, S]")
    if workspace is None:
        workspace = Workspace.create(shape, OP_FWD, q.device, stream)
    if out is None:
        energy = torch.empty((B, H, nb, nb), dtype=torch.float32, device=q.device)
        mass = (torch.empty((B, H, nb), dtype=torch.float32, device=q.device)
                if want_block_mass else None)
    else:
        energy, mass = out
    _check(lib().nabla_block_energy(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(lse),
                                    _ptr(row_ptr), _ptr(col_idx), float(scale or 0.0),
                                    _ptr(energy), _ptr(mass) if mass is not None else None,
                                    _ptr(workspace.buf), _stream(stream)))
    return energy, mass


def nabla_calib_accumulate(energy, eps: float, votes, stream=None):
    """votes[b,h,r,c] += 1 for each block the minimal-prefix rule keeps at eps."""
    torch = _torch()
    for t, dt in ((energy, torch.float32), (votes, torch.int32)):
        if t.dtype != dt or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("energy fp32 and votes int32 must be contiguous CUDA [B,H,nb,nb]")
    B, H, nb, _ = energy.shape
    shape = make_shape(B, H, nb * 64, 64)
    _check(lib().nabla_calib_accumulate(ctypes.byref(shape), _ptr(energy), float(eps), _ptr(votes),
                                        _stream(stream)))
    return votes


def nabla_calib_finalize(votes, min_votes: int = 1, out=None, stream=None):
    """uint8 static mask [B,H,nb,nb] = votes >= min_votes."""
    torch = _torch()
    if votes.dtype != torch.int32 or not votes.is_cuda or not votes.is_contiguous() or votes.dim() != 4:
        raise ValueError("votes must be a contiguous int32 CUDA tensor [B,H,nb,nb]")
    B, H, nb, _ = votes.shape
    mask = torch.empty(votes.shape, dtype=torch.uint8, device=votes.device) if out is None else out
    shape = make_shape(B, H, nb * 64, 64)
    _check(lib().nabla_calib_finalize(ctypes.byref(shape), _ptr(votes), int(min_votes), _ptr(mask),
                                      _stream(stream)))
    return mask


def bsa_bwd(q, k, v, o, dout, lse, row_ptr, col_idx, scale: Optional[float] = None,
            workspace: Optional[Workspace] = None, out=None, stream=None):
    """Gradients (dQ, dK, dV), bf16 [B,H,S,d], of the block-sparse forward over
    the same CSR, from its O and LSE and the output gradient dO."""
    torch = _torch()
    _bf16_contig(q, k, v, o, dout)
    shape = _shape_of(q)
    B, H, S, _ = q.shape
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, S):
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, S]")
    if workspace is None:
        workspace = Workspace.create(shape, OP_BWD, q.device, stream)
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = out
    _check(lib().bsa_bwd(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout),
                         _ptr(lse), _ptr(row_ptr), _ptr(col_idx), float(scale or 0.0), _ptr(dq),
                         _ptr(dk), _ptr(dv), _ptr(workspace.buf), _stream(stream)))
    return dq, dk, dv


def nabla_build_mask_xattn(q, k, thr: float, stride: int = 8, tile_grid=None,
                           sta: Optional[Tuple[int, int, int]] = None, topk: int = 0,
                           want_mask: bool = False, want_scores: bool = False,
                           col_capacity: Optional[int] = None,
                           workspace: Optional[Workspace] = None, out=None, stream=None):
    """Block CSR selected from XAttention antidiagonal scores (stride 4, 8, 16).

    Returns (row_ptr, col_idx, nnz, mask or None, scores fp32 [B,H,nb,nb] or None)."""
    torch = _torch()
    _bf16_contig(q, k)
    shape = _shape_of(q, tile_grid)
    B, H, S, d = q.shape
    nb = S // 64
    if workspace is None:
        workspace = Workspace.create(shape, OP_BUILD_XATTN, q.device, stream)
    if out is None:
        cap = col_capacity if col_capacity is not None else B * H * nb * nb
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=q.device)
        col_idx = torch.empty(max(cap, 1), dtype=torch.int32, device=q.device)
        nnz = torch.empty(1, dtype=torch.int32, device=q.device)
        mask = torch.empty((B, H, nb, nb), dtype=torch.uint8, device=q.device) if want_mask else None
    else:
        row_ptr, col_idx, nnz, mask = out
        cap = col_idx.numel() if col_capacity is None else col_capacity
    scores = (torch.empty((B, H, nb, nb), dtype=torch.float32, device=q.device)
              if want_scores else None)
    prm = _MaskParams(float(thr), 1 if sta is not None else 0,
                      *(sta if sta is not None else (0, 0, 0)), int(topk))
    _check(lib().nabla_build_mask_xattn(ctypes.byref(shape), ctypes.byref(prm), int(stride),
                                        _ptr(q), _ptr(k), _ptr(scores), _ptr(mask), _ptr(row_ptr),
                                        _ptr(col_idx), int(cap), _ptr(nnz), _ptr(workspace.buf),
                                        _stream(stream)))
    return row_ptr, col_idx, nnz, mask, scores
