"""Seeded synthetic inputs for the deformable-convolution core.

This package holds no arithmetic of the operator.  It turns a workload
description (shapes, value distributions) and a seed into host arrays, and
both the CPU oracle and the CUDA path are fed from it.  Random numbers come
from the counter-based generator in ``dcn_gen.c`` (SplitMix64 + Box-Muller),
so a value depends only on (seed, tensor id, flat index).

Tensor ids: input x = 1, offset = 2, mask = 3, grad_out = 4, far-offset
selector = 5, far-offset value = 6.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .workloads import WORKLOADS, Workload, output_hw

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dcn_gen.c")
_LIB_PATH = os.path.join(_HERE, "libdcngen.so")

TID_X, TID_OFFSET, TID_MASK, TID_GRAD_OUT, TID_FAR_SELECT, TID_FAR_VALUE = 1, 2, 3, 4, 5, 6
# inputs of the offset / mask projection: query features, weight, bias
TID_QUERY, TID_WEIGHT, TID_BIAS = 7, 8, 9
TID_OUT_WEIGHT = 10  # output_proj weight of the block's core path
# parameters of the guide branch: depthwise weight and bias, LayerNorm gamma and beta
TID_DW_WEIGHT, TID_DW_BIAS, TID_LN_GAMMA, TID_LN_BETA = 11, 12, 13, 14

_lib = None


def build(force: bool = False) -> str:
    """Compile dcn_gen.c into libdcngen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = ctypes.POINTER(ctypes.c_float)
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        lib.gen_uniform_f32.argtypes = [u64, u64, i64, dbl, dbl, f32p]
        lib.gen_uniform_f32.restype = None
        lib.gen_normal_f32.argtypes = [u64, u64, i64, dbl, dbl, f32p]
        lib.gen_normal_f32.restype = None
        lib.gen_redraw_pairs_f32.argtypes = [u64, u64, u64, i64, dbl, dbl, dbl, f32p]
        lib.gen_redraw_pairs_f32.restype = i64
        lib.gen_hash.argtypes = [u64, u64, u64]
        lib.gen_hash.restype = u64
        _lib = lib
    return _lib


def _fptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def uniform(seed: int, tensor_id: int, shape, lo: float, hi: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().gen_uniform_f32(seed, tensor_id, out.size, lo, hi, _fptr(out))
    return out


def normal(seed: int, tensor_id: int, shape, mean: float, sd: float) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().gen_normal_f32(seed, tensor_id, out.size, mean, sd, _fptr(out))
    return out


def redraw_pairs(seed: int, pairs: np.ndarray, frac: float, lo: float, hi: float) -> int:
    """Redraw a fraction ``frac`` of the (dx, dy) pairs of ``pairs`` (float32,
    C-contiguous, even length) from U(lo, hi), in place."""
    assert pairs.dtype == np.float32 and pairs.flags.c_contiguous and pairs.size % 2 == 0
    return int(_load().gen_redraw_pairs_f32(seed, TID_FAR_SELECT, TID_FAR_VALUE,
                                            pairs.size // 2, frac, lo, hi, _fptr(pairs)))


def raw_hash(seed: int, tensor_id: int, i: int) -> int:
    return int(_load().gen_hash(seed, tensor_id, i))


def draw(seed: int, tensor_id: int, shape, dist) -> np.ndarray:
    kind, a, b = dist
    if kind == "normal":
        return normal(seed, tensor_id, shape, a, b)
    if kind == "uniform":
        return uniform(seed, tensor_id, shape, a, b)
    if kind == "zeros":
        return np.zeros(shape, dtype=np.float32)
    raise ValueError(kind)


def make_inputs(wl: Workload | str, seed: int | None = None, n_images: int | None = None,
                with_grad_out: bool | None = None) -> dict:
    """Host float32 arrays for one workload: x (N,H,W,G*Cg), offset
    (N,Ho,Wo,G*T*2) as (dx, dy) pairs, mask (N,Ho,Wo,G*T) with T = wl.KK taps
    per (pixel, group), and, for backward workloads, grad_out (N,Ho,Wo,G*Cg).

    ``n_images`` generates only the first n images of the batch; because the
    generator is counter-based these are bit-identical to the leading images
    of the full batch.
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    seed = wl.seed if seed is None else seed
    N = wl.N if n_images is None else n_images
    Ho, Wo = output_hw(wl)
    C, KK = wl.G * wl.Cg, wl.KK

    def gen_prefix(tid, full_shape, dist):
        # Draw the full tensor's first N images only: same values as the full draw.
        full = full_shape[1:]
        per = int(np.prod(full))
        arr = np.empty((N,) + tuple(full), dtype=np.float32)
        kind, a, b = dist
        if kind == "zeros":
            arr[...] = 0
            return arr
        fn = _load().gen_normal_f32 if kind == "normal" else _load().gen_uniform_f32
        fn(seed, tid, N * per, a, b, _fptr(arr))
        return arr

    x = gen_prefix(TID_X, (wl.N, wl.H, wl.W, C), wl.x_dist)
    off = gen_prefix(TID_OFFSET, (wl.N, Ho, Wo, wl.G * KK * 2), wl.offset_dist)
    if wl.far is not None:
        frac, lo, hi = wl.far
        redraw_pairs(seed, off.reshape(-1), frac, lo, hi)
    mask = gen_prefix(TID_MASK, (wl.N, Ho, Wo, wl.G * KK), wl.mask_dist)
    out = {"x": x, "offset": off, "mask": mask}
    if with_grad_out if with_grad_out is not None else wl.backward:
        out["grad_out"] = gen_prefix(TID_GRAD_OUT, (wl.N, Ho, Wo, C), ("normal", 0.0, 1.0))
    return out


def make_projection_inputs(wl, Cq: int, seed=None) -> dict:
    """Host float32 arrays for the offset / mask projection of a workload:
    query (N, Ho, Wo, Cq) ~ N(0, 1), weight (G*KK*3, Cq) ~ N(0, 1/Cq) (unit
    output variance) and bias (G*KK*3) ~ N(0, 1)."""
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    seed = wl.seed if seed is None else seed
    Ho, Wo = output_hw(wl)
    nout = wl.G * wl.KK * 3
    return {"query": normal(seed, TID_QUERY, (wl.N, Ho, Wo, Cq), 0.0, 1.0),
            "weight": normal(seed, TID_WEIGHT, (nout, Cq), 0.0, float(Cq) ** -0.5),
            "bias": normal(seed, TID_BIAS, (nout,), 0.0, 1.0)}


__all__ = ["WORKLOADS", "Workload", "output_hw", "make_inputs", "make_projection_inputs", "uniform", "normal",
           "redraw_pairs", "raw_hash", "draw", "build"]


def make_guide_params(wl, seed=None) -> dict:
    """Host float32 parameters of the guide branch for a workload's C channels:
    depthwise weight (3, 3, C) ~ N(0, 1/9), bias ~ N(0, 0.1^2), LayerNorm
    gamma ~ N(1, 0.1^2) and beta ~ N(0, 0.1^2)."""
    seed = wl.seed if seed is None else seed
    C = wl.C
    return {"dw_weight": normal(seed, TID_DW_WEIGHT, (3, 3, C), 0.0, 1.0 / 3.0),
            "dw_bias": normal(seed, TID_DW_BIAS, (C,), 0.0, 0.1),
            "ln_gamma": normal(seed, TID_LN_GAMMA, (C,), 1.0, 0.1),
            "ln_beta": normal(seed, TID_LN_BETA, (C,), 0.0, 0.1)}
