"""Seeded synthetic inputs (shared by the fp64 oracle, the CUDA path's tests and the bench).

This package only generates input data: counter-based SplitMix64 streams,
Box-Muller normals, a fixed 3D sinusoidal embedding and bf16 rounding.  It
holds none of the method's arithmetic.  The C source (``synth.c``) is
compiled with gcc on first use (or by ``build()``) into ``libsynth.so``
beside it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .workloads import WORKLOADS, Workload  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_MASK = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile libsynth.so with gcc (OpenMP, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            u64, i32, i64, f64 = ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            vp = ctypes.c_void_p
            lib.synth_splitmix64_at.restype = u64
            lib.synth_splitmix64_at.argtypes = [u64, u64]
            lib.synth_tensor_key.restype = u64
            lib.synth_tensor_key.argtypes = [u64, i32]
            lib.synth_uniform_at.restype = f64
            lib.synth_uniform_at.argtypes = [u64, u64]
            lib.synth_normal_at.restype = f64
            lib.synth_normal_at.argtypes = [u64, u64]
            lib.synth_f64_to_bf16.restype = ctypes.c_uint16
            lib.synth_f64_to_bf16.argtypes = [f64]
            lib.synth_embedding.restype = None
            lib.synth_embedding.argtypes = [i32, i32, i32, i32, vp]
            lib.synth_fill_tensor.restype = i32
            lib.synth_fill_tensor.argtypes = [vp, i32, u64, i32, i32, i64, i32, i32, i32, i32, f64, f64]
            lib.synth_fill_bernoulli_mask.restype = i32
            lib.synth_fill_bernoulli_mask.argtypes = [vp, i32, u64, i64, i32, f64, i32]
            _lib = lib
    return _lib


def lib():
    return _load()


def fill_tensor_ptr(ptr: int, tensor_id: int, seed: int, B: int, H: int, S: int, d: int,
                    grid=(0, 0, 0), pos_weight: float = 1.0, noise_weight: float = 0.5) -> None:
    """Write a [B,H,S,d] bf16 tensor (as uint16 bits) to host memory at ``ptr``."""
    Tt, Th, Tw = grid
    rc = _load().synth_fill_tensor(ctypes.c_void_p(ptr), tensor_id, seed, B, H, S, d, Tt, Th, Tw,
                                   float(pos_weight), float(noise_weight))
    if rc != 0:
        raise ValueError(f"synth_fill_tensor failed with code {rc}")


def make_tensor(tensor_id: int, seed: int, B: int, H: int, S: int, d: int, grid=(0, 0, 0),
                pos_weight: float = 1.0, noise_weight: float = 0.5) -> np.ndarray:
    """Return a [B,H,S,d] uint16 array holding bf16 bit patterns."""
    out = np.empty((B, H, S, d), dtype=np.uint16)
    fill_tensor_ptr(out.ctypes.data, tensor_id, seed, B, H, S, d, grid, pos_weight, noise_weight)
    return out


def make_qkv(w: "Workload", seed: int = 0):
    """Q, K, V (uint16 bf16 bits, [B,H,S,d]) for a workload recipe."""
    if w.iid_normal:
        args = dict(grid=(0, 0, 0), pos_weight=0.0, noise_weight=1.0)
        q = make_tensor(TENSOR_Q, seed, w.B, w.H, w.S, w.d, **args)
        k = make_tensor(TENSOR_K, seed, w.B, w.H, w.S, w.d, **args)
    else:
        args = dict(grid=w.tile_grid, pos_weight=w.pos_weight, noise_weight=w.noise_weight)
        q = make_tensor(TENSOR_Q, seed, w.B, w.H, w.S, w.d, **args)
        k = make_tensor(TENSOR_K, seed, w.B, w.H, w.S, w.d, **args)
    v = make_tensor(TENSOR_V, seed, w.B, w.H, w.S, w.d, grid=(0, 0, 0), pos_weight=0.0,
                    noise_weight=1.0)
    return q, k, v


def fill_bernoulli_mask_ptr(ptr: int, seed: int, BH: int, nb: int, p: float,
                            force_diag: bool = True, tensor_id: int = TENSOR_MASK) -> None:
    rc = _load().synth_fill_bernoulli_mask(ctypes.c_void_p(ptr), tensor_id, seed, BH, nb, float(p),
                                           1 if force_diag else 0)
    if rc != 0:
        raise ValueError(f"synth_fill_bernoulli_mask failed with code {rc}")


def make_bernoulli_mask(seed: int, BH: int, nb: int, p: float, force_diag: bool = True) -> np.ndarray:
    """[BH, nb, nb] uint8 block mask, i.i.d. Bernoulli(p), diagonal forced on."""
    out = np.empty((BH, nb, nb), dtype=np.uint8)
    fill_bernoulli_mask_ptr(out.ctypes.data, seed, BH, nb, p, force_diag)
    return out


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen uint16 bf16 bit patterns to float32 (exact)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def embedding(d: int, t: int, h: int, w: int) -> np.ndarray:
    e = np.empty(d, dtype=np.float64)
    _load().synth_embedding(d, t, h, w, e.ctypes.data)
    return e
