"""Helpers shared by the GPU tests: device copies of the generator's arrays,
exact widening back to float64, and the parity measures with their
tolerances (forward fp32: 1e-5 * max|x|; bf16 storage: 1e-2 * max|ref|;
fp16 storage: 1e-3 * max|ref|; backward fp32: 1e-4 * max|ref| per gradient)."""
from __future__ import annotations

import numpy as np
import torch

import deformable_convolution_core_b200 as dcn

FWD_F32_TOL = 1e-5     # max |gpu - ref| <= FWD_F32_TOL * max|x|
FWD_BF16_TOL = 1e-2    # max |gpu - ref| <= FWD_BF16_TOL * max|ref|
BWD_F32_TOL = 1e-4     # max |gpu - ref| <= BWD_F32_TOL * max|ref|, per gradient
BWD_BF16_TOL = 1e-2    # bf16 storage: each gradient rounded to bf16 once; same gate as the forward
# fp16 storage: one rounding to fp16 is at most 2^-11 relative; the gate allows
# twice that, normalised by max|ref| like the bf16 gate (forward and backward).
FWD_F16_TOL = 1e-3
BWD_F16_TOL = 1e-3

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def to_dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Round a float32 host array to the storage type (bf16: nearest even) on the device."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(device).to(TORCH_DTYPE[dtype]).contiguous()


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a tensor of fp32 or bf16 values."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def gpu_forward(problem, x, off, mask, stream=None) -> torch.Tensor:
    Ho, Wo = dcn.dcn_core_output_hw(problem)
    out = torch.empty((problem.N, Ho, Wo, problem.G * problem.Cg), dtype=x.dtype, device=x.device)
    dcn.dcn_core_forward(problem, x, off, mask, out, stream)
    return out


def gpu_backward(problem, x, off, mask, gout, stream=None):
    gx = torch.empty_like(x)
    goff = torch.empty_like(off)
    gm = torch.empty_like(mask)
    ws = dcn.dcn_core_backward_workspace(problem)
    wbuf = torch.empty(max(ws, 1), dtype=torch.uint8, device=x.device) if ws else None
    dcn.dcn_core_backward(problem, x, off, mask, gout, gx, goff, gm, wbuf, ws, stream)
    return gx, goff, gm


def fwd_error(got: np.ndarray, ref: np.ndarray, x: np.ndarray, dtype: str):
    """(error, bound) of the forward parity gate."""
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    if dtype == "f32":
        return err, FWD_F32_TOL * max(float(np.abs(x).max()), 1e-30)
    tol = FWD_F16_TOL if dtype == "f16" else FWD_BF16_TOL
    return err, tol * max(float(np.abs(ref).max()), 1e-30)


def assert_fwd(got, ref, x, dtype, what=""):
    err, bound = fwd_error(got, ref, x, dtype)
    assert err <= bound, f"{what}: forward max error {err:.3e} > {bound:.3e}"


def assert_bwd(got, ref, what="", dtype="f32"):
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    tol = {"f32": BWD_F32_TOL, "f16": BWD_F16_TOL}.get(dtype, BWD_BF16_TOL)
    bound = tol * max(float(np.abs(ref).max()), 1e-30)
    assert err <= bound, f"{what}: backward max error {err:.3e} > {bound:.3e}"


def problem_kwargs(problem) -> dict:
    return dict(G=problem.G, K=problem.K, stride=problem.stride, pad=problem.pad,
                dil=problem.dilation, offset_scale=problem.offset_scale, softmax=problem.softmax,
                remove_center=problem.remove_center,
                stride_w=problem.stride_w if problem.separate_axes else None,
                pad_w=problem.pad_w if problem.separate_axes else None,
                dil_w=problem.dilation_w if problem.separate_axes else None)
