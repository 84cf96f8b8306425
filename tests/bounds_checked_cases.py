"""Adversarial cases for the bounds-checked build (libdcncore_checked.so).

Run as a script in its own process with DCN_CORE_LIBRARY pointing at the
checked library (the binding loads one library per process).  Every call must
finish with DCN_OK from dcn_core_sync_status -- no access outside a tensor was
skipped -- and match the oracle.  Prints one line per case and exits non-zero
on the first failure.
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import deformable_convolution_core_b200 as dcn  # noqa: E402
import oracle  # noqa: E402
from tests.dcn_testutil import (assert_bwd, assert_fwd, f64, gpu_backward, gpu_forward,  # noqa: E402
                                problem_kwargs, to_dev)

RNG = np.random.default_rng(8)


def env(**kv):
    for k, v in kv.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


def case(name, p, off_fn=None, dtype="f32"):
    Ho, Wo = dcn.dcn_core_output_hw(p)
    T = dcn.taps(p)
    x = RNG.standard_normal((p.N, p.H, p.W, p.G * p.Cg)).astype(np.float32)
    off = (2.0 * RNG.standard_normal((p.N, Ho, Wo, p.G, T, 2))).astype(np.float32)
    if off_fn is not None:
        off_fn(off)
    off = off.reshape(p.N, Ho, Wo, -1)
    mask = RNG.standard_normal((p.N, Ho, Wo, p.G * T)).astype(np.float32)
    gout = RNG.standard_normal((p.N, Ho, Wo, p.G * p.Cg)).astype(np.float32)
    xd, od, md, gd = (to_dev(a, dtype) for a in (x, off, mask, gout))
    kw = problem_kwargs(p)
    ref = oracle.forward(f64(xd), f64(od), f64(md), **kw)
    rx, roff, rm = oracle.backward(f64(xd), f64(od), f64(md), f64(gd), **kw)
    for fpath in ("auto", "direct"):
        env(DCN_CORE_FORWARD="direct" if fpath == "direct" else None)
        out = gpu_forward(p, xd, od, md)
        dcn.dcn_core_sync_status()
        assert_fwd(f64(out), ref, f64(xd), dtype, f"{name} forward {fpath}")
    for bpath in ("auto", "direct"):
        env(DCN_CORE_BACKWARD="direct" if bpath == "direct" else None)
        gx, goff, gm = gpu_backward(p, xd, od, md, gd)
        dcn.dcn_core_sync_status()
        for got, r, what in ((gx, rx, "grad_input"), (goff, roff, "grad_offset"), (gm, rm, "grad_mask")):
            assert_bwd(f64(got), r, f"{name} {what} {bpath}", dtype)
        nbytes = dcn.dcn_core_backward_deterministic_workspace(p)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        dgx, dgoff, dgm = torch.empty_like(xd), torch.empty_like(od), torch.empty_like(md)
        dcn.dcn_core_backward_deterministic(p, xd, od, md, gd, dgx, dgoff, dgm, ws, nbytes)
        dcn.dcn_core_sync_status()
        assert_bwd(f64(dgx), rx, f"{name} deterministic grad_input {bpath}", dtype)
    env(DCN_CORE_FORWARD=None, DCN_CORE_BACKWARD=None)
    print(f"ok {name}", flush=True)


def borders(W):
    def f(off):  # dx of tap 4 puts samples exactly at X = -1, 0, W-1, W (offset_scale 2)
        n, Ho, Wo = off.shape[:3]
        wo = np.arange(Wo)
        target = np.array([-1, 0, W - 1, W] * ((Wo + 3) // 4))[:Wo]
        off[:, :, :, :, 4, 0] = ((target - wo) / 2.0)[None, None, :, None]
    return f


def far(off):
    off[..., :] = RNG.uniform(-1e4, 1e4, off.shape)


def main():
    torch.cuda.set_device(0)
    mk = dcn.make_problem
    case("tiny fp32", mk(1, 14, 14, 4, 16, offset_scale=1.0))
    case("offsets +-1e4", mk(2, 9, 11, 2, 16, offset_scale=2.0), far)
    case("exact borders", mk(1, 7, 10, 2, 16, offset_scale=2.0), borders(10))
    case("one pixel", mk(1, 1, 1, 2, 16, offset_scale=2.0))
    case("stride above the image", mk(2, 3, 3, 2, 16, stride=5, offset_scale=2.0))
    case("bf16 remove_center", mk(2, 13, 12, 3, 16, offset_scale=2.0, dtype="bf16",
                                  remove_center=1), dtype="bf16")
    case("separate axes K=5", mk(1, 12, 15, 2, 8, K=5, pad=2, stride_w=2, pad_w=1,
                                 offset_scale=2.0))
    case("Cg 32 raw mask", mk(1, 10, 9, 3, 32, softmax=0, offset_scale=2.0))
    # the 3x3 tiled forward with 8 channels of a 2-byte type (16-byte groups)
    case("Cg 8 bf16 offsets +-1e4", mk(2, 11, 13, 3, 8, offset_scale=2.0, dtype="bf16"), far,
         dtype="bf16")
    case("Cg 8 fp16 borders remove_center", mk(1, 9, 10, 2, 8, offset_scale=2.0, dtype="f16",
                                               remove_center=1), borders(10), dtype="f16")
    # the wide-window tiled forward (5x5 and 7x7 windows, chunked taps)
    case("K=5 wide", mk(2, 13, 17, 3, 16, K=5, pad=2, offset_scale=2.0))
    case("K=7 bf16 dilation 2 remove_center raw mask",
         mk(1, 15, 14, 2, 16, K=7, pad=6, dilation=2, softmax=0, offset_scale=2.0,
            dtype="bf16", remove_center=1), dtype="bf16")
    case("K=7 fp16 offsets +-1e4", mk(1, 9, 12, 2, 16, K=7, pad=3, offset_scale=2.0,
                                      dtype="f16"), far, dtype="f16")
    # the tensor-core projection, ragged in pixels and columns
    p = mk(1, 7, 9, 5, 16, offset_scale=2.0)
    q = torch.randn(1, 7, 9, 64).to(torch.bfloat16).cuda()
    w = torch.randn(5 * 27, 64).to(torch.bfloat16).cuda()
    off = torch.empty(1, 7, 9, 90, device="cuda")
    msk = torch.empty(1, 7, 9, 45, device="cuda")
    dcn.dcn_core_offset_mask_projection(p, q, 64, w, None, off, msk)
    dcn.dcn_core_sync_status()
    ro, rm = oracle.projection(q.cpu(), w.cpu(), None, G=5)
    assert np.abs(f64(off) - ro).max() <= 1e-4 * np.abs(ro).max()
    assert np.abs(f64(msk) - rm).max() <= 1e-4 * np.abs(rm).max()
    print("ok projection", flush=True)
    # the guide features: ragged column and row tiles, a one-pixel image, bf16
    # input, and C = 196 (lanes left idle in the last quad group)
    for (N, H, W, G, Cg, dtype) in ((2, 11, 37, 4, 16, "f32"), (1, 1, 1, 2, 16, "bf16"),
                                    (1, 9, 5, 49, 4, "f32")):
        C = G * Cg
        pg = mk(N, H, W, G, Cg, dtype=dtype)
        xg = to_dev(RNG.standard_normal((N, H, W, C)).astype(np.float32), dtype)
        prm = [RNG.uniform(-0.5, 0.5, size=s_).astype(np.float32) for s_ in ((3, 3, C), (C,))]
        prm += [RNG.uniform(0.5, 1.5, size=C).astype(np.float32),
                RNG.uniform(-0.3, 0.3, size=C).astype(np.float32)]
        qg = torch.empty(xg.shape, dtype=torch.bfloat16, device="cuda")
        dcn.dcn_core_offset_mask_guide(pg, xg, *(torch.from_numpy(a).cuda() for a in prm), 1e-6, qg)
        dcn.dcn_core_sync_status()
        rg = oracle.guide(f64(xg), *prm, 1e-6)
        assert (np.abs(f64(qg) - rg) <= 2.0 ** -8 * np.abs(rg) + 2e-5).all(), f"guide {N}x{H}x{W}x{C}"
    print("ok guide", flush=True)
    print("all cases passed")


if __name__ == "__main__":
    main()
