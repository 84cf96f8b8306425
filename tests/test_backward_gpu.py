"""Backward parity: grad_input, grad_offset and grad_mask (w.r.t. the logits
when softmax is on) of the CUDA path against the CPU oracle, plus the
adjoint identity and the softmax-Jacobian row sums at the full backward size.
"""
import contextlib
import os

import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from gen.workloads import WORKLOADS
from tests.dcn_testutil import assert_bwd, f64, gpu_backward, gpu_forward, problem_kwargs, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(77)


@contextlib.contextmanager
def env(**kv):
    """Set (value) or clear (None) environment variables for the block."""
    old = {k: os.environ.get(k) for k in kv}
    for k, v in kv.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v
    try:
        yield
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def backward_path(path):
    """"auto": the library's choice (the TMA-tiled kernel where it applies);
    "direct": the direct-gather kernel."""
    return env(DCN_CORE_BACKWARD="direct" if path == "direct" else None)


def near_kink_taps(p, off):
    """Count taps whose sample coordinate lies within 1e-6 of an integer, where
    the offset gradient switches between one-sided derivatives."""
    N, Ho, Wo = off.shape[:3]
    K = p.K
    T = dcn.taps(p)
    o = off.reshape(N, Ho, Wo, p.G, T, 2).astype(np.float32)
    ho = np.arange(Ho).reshape(1, Ho, 1, 1, 1)
    wo = np.arange(Wo).reshape(1, 1, Wo, 1, 1)
    k = np.array([q for q in range(K * K) if not (p.remove_center and q == (K * K) // 2)])
    a, b = (k // K).reshape(1, 1, 1, 1, -1), (k % K).reshape(1, 1, 1, 1, -1)
    s = np.float32(p.offset_scale)
    Y = (ho * p.stride - p.pad + a * p.dilation).astype(np.float32) + s * o[..., 1]
    sw, pw, dw = ((p.stride_w, p.pad_w, p.dilation_w) if p.separate_axes
                  else (p.stride, p.pad, p.dilation))
    X = (wo * sw - pw + b * dw).astype(np.float32) + s * o[..., 0]
    fy, fx = Y - np.floor(Y), X - np.floor(X)
    near = (np.minimum(fy, 1 - fy) < 1e-6) | (np.minimum(fx, 1 - fx) < 1e-6)
    return int(near.sum())


def check(oracle_mod, p, x, off, mask, gout, dtype="f32"):
    xd, od, md, gd = (to_dev(a, dtype) for a in (x, off, mask, gout))
    gx, goff, gm = gpu_backward(p, xd, od, md, gd)
    torch.cuda.synchronize()
    # the oracle sees exactly the values the GPU saw (bf16-rounded for bf16)
    rx, roff, rm = oracle_mod.backward(f64(xd), f64(od), f64(md), f64(gd), **problem_kwargs(p))
    assert_bwd(f64(gx), rx, f"grad_input {p}", dtype)
    assert_bwd(f64(goff), roff, f"grad_offset {p} (near-kink taps: {near_kink_taps(p, f64(od))})",
               dtype)
    assert_bwd(f64(gm), rm, f"grad_mask {p}", dtype)
    return gx, goff, gm


CASES = [
    (2, 23, 29, 3, 16, dict()),
    (2, 19, 17, 5, 16, dict(softmax=0)),
    (2, 15, 21, 4, 4, dict()),
    (2, 15, 21, 4, 8, dict()),
    (2, 13, 14, 3, 32, dict()),
    (2, 17, 19, 3, 16, dict(K=5, pad=2)),
    (2, 17, 19, 3, 16, dict(K=1, pad=0)),
    (2, 24, 26, 3, 16, dict(stride=2)),
    (2, 21, 22, 3, 16, dict(dilation=2, pad=2)),
    (1, 1, 1, 2, 16, dict()),
    (1, 30, 3, 40, 16, dict()),
    (2, 23, 29, 3, 16, dict(remove_center=1)),
    (2, 19, 17, 5, 16, dict(softmax=0, remove_center=1)),
    (2, 15, 21, 4, 8, dict(remove_center=1, stride=2)),
    (2, 17, 19, 3, 16, dict(K=5, pad=2, remove_center=1)),
    (1, 17, 19, 2, 16, dict(K=7, pad=3, remove_center=1, softmax=0)),
    (2, 25, 23, 3, 16, dict(stride=2, dilation=2, pad=2)),
    (2, 13, 14, 3, 32, dict(softmax=0)),
    (1, 2, 40, 2, 16, dict()),
    (2, 23, 29, 3, 16, dict(stride_w=2, pad_w=0)),
    (2, 26, 21, 4, 16, dict(stride=2, dilation_w=2, pad_w=2, softmax=0)),
    (2, 11, 13, 2, 64, dict()),                  # 16 lanes per unit
    (1, 9, 10, 3, 64, dict(softmax=0, stride=2)),
]


@pytest.mark.parametrize("path", ["auto", "direct"])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}_G{c[3]}_Cg{c[4]}_" +
                                             "_".join(f"{k}{v}" for k, v in c[5].items())
                                             for c in CASES])
def test_backward_matches_oracle(oracle_mod, case, dtype, path):
    N, H, W, G, Cg, kw = case
    if dtype == "bf16" and Cg * 2 < 16:
        pytest.skip("bf16 needs Cg >= 8")
    kw = {"K": 3, "stride": 1, "pad": 1, "dilation": 1, "softmax": 1, "remove_center": 0,
          "stride_w": None, "pad_w": None, "dilation_w": None, **kw}
    p = dcn.make_problem(N, H, W, G, Cg, kw["K"], kw["stride"], kw["pad"], kw["dilation"],
                         2.0, kw["softmax"], dtype, kw["remove_center"], kw["stride_w"],
                         kw["pad_w"], kw["dilation_w"])
    Ho, Wo = dcn.dcn_core_output_hw(p)
    KK = dcn.taps(p)
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    off = (1.5 * RNG.standard_normal((N, Ho, Wo, G * KK * 2))).astype(np.float32)
    mask = RNG.standard_normal((N, Ho, Wo, G * KK)).astype(np.float32)
    gout = RNG.standard_normal((N, Ho, Wo, G * Cg)).astype(np.float32)
    with backward_path(path):
        check(oracle_mod, p, x, off, mask, gout, dtype)


@pytest.mark.parametrize("halo,tile", [("0", "1x1"), ("2", "3x5"), ("9", "32x32"), ("5", "7x64")])
def test_tiled_backward_tile_and_halo_settings(oracle_mod, halo, tile):
    """Every tile shape and halo width of the tiled backward gives the same
    gradients (only the split between box reads and global reads changes)."""
    with env(DCN_CORE_HALO=halo, DCN_CORE_BWD_TILED_TILE=tile):
        for dtype in ("f32", "bf16"):
            for kw in (dict(), dict(stride=2, softmax=0), dict(remove_center=1)):
                kw = {"stride": 1, "softmax": 1, "remove_center": 0, **kw}
                N, H, W, G, Cg = 2, 29, 31, 3, 16
                p = dcn.make_problem(N, H, W, G, Cg, 3, kw["stride"], 1, 1, 2.0, kw["softmax"],
                                     dtype, kw["remove_center"])
                Ho, Wo = dcn.dcn_core_output_hw(p)
                T = dcn.taps(p)
                x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
                off = (3.0 * RNG.standard_normal((N, Ho, Wo, G * T * 2))).astype(np.float32)
                mask = RNG.standard_normal((N, Ho, Wo, G * T)).astype(np.float32)
                gout = RNG.standard_normal((N, Ho, Wo, G * Cg)).astype(np.float32)
                check(oracle_mod, p, x, off, mask, gout, dtype)


def test_backward_paths_agree_on_nonfinite_and_border_offsets(oracle_mod):
    """NaN, infinite, huge and exact-border offsets: both backward kernels
    match the oracle."""
    N, H, W, G, Cg = 1, 9, 11, 2, 16
    p = dcn.make_problem(N, H, W, G, Cg, offset_scale=2.0)
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    off = (1.5 * RNG.standard_normal((N, H, W, G, 9, 2))).astype(np.float32)
    off[0, 0, 0, 0, :, 0] = np.nan
    off[0, 1, 1, 0, :, 1] = np.inf
    off[0, 2, 2, 1, :, 0] = -np.inf
    off[0, 3, 3, 0, :, :] = 1e30
    off[0, 4, :, 1, 4, 0] = (np.array([-1, 0, W - 1, W] * 3)[:W] - np.arange(W)) / 2.0
    off = off.reshape(N, H, W, -1)
    mask = RNG.standard_normal((N, H, W, G * 9)).astype(np.float32)
    gout = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    for path in ("auto", "direct"):
        with backward_path(path):
            xd, od, md, gd = (to_dev(a, "f32") for a in (x, off, mask, gout))
            gx, goff, gm = gpu_backward(p, xd, od, md, gd)
            torch.cuda.synchronize()
        rx, roff, rm = oracle_mod.backward(x, off, mask, gout, **problem_kwargs(p))
        # NaN / inf offsets give NaN-free zeros on both sides
        assert_bwd(f64(gx), rx, f"grad_input {path}")
        assert_bwd(f64(goff), roff, f"grad_offset {path}")
        assert_bwd(f64(gm), rm, f"grad_mask {path}")


def test_full_size_backward(gen_mod, oracle_mod):
    wl = WORKLOADS["internimage_l_stage2_bwd_fp32_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl)
    p = dcn.problem_for(wl)
    gx, goff, gm = check(oracle_mod, p, d["x"], d["offset"], d["mask"], d["grad_out"])
    # adjoint identity: <gout, F(v)> = <grad_input(gout), v>, v random
    v = RNG.standard_normal(d["x"].shape).astype(np.float32)
    xd, od, md = (to_dev(d[k], "f32") for k in ("x", "offset", "mask"))
    gxv, _, _ = gpu_backward(p, to_dev(v, "f32"), od, md, to_dev(d["grad_out"], "f32"))
    fv = gpu_forward(p, to_dev(v, "f32"), od, md)
    torch.cuda.synchronize()
    lt = f64(fv) * d["grad_out"].astype(np.float64)
    rt = f64(gxv) * v.astype(np.float64)
    lhs, rhs = float(lt.sum()), float(rt.sum())
    # Each of the 23.6 M products carries the fp32 rounding of its output or
    # gradient element (relative ~1e-7); the signed errors add like a random
    # walk, so the difference is gated on the 2-norm of the terms, not on the
    # (heavily cancelled) sums themselves.  A wrong or missing scatter term
    # would move it by orders of magnitude more.
    scale = float(np.sqrt((lt ** 2).sum() + (rt ** 2).sum()))
    assert abs(lhs - rhs) <= 1e-5 * scale, (lhs, rhs, scale)
    # softmax Jacobian rows: the logit gradients of every (pixel, group) sum to zero
    rows = f64(gm).reshape(-1, 9)
    assert np.abs(rows.sum(1)).max() <= 1e-5 * np.abs(rows).max()


def test_backward_rerun_differs_only_by_rounding(gen_mod):
    wl = WORKLOADS["internimage_l_stage2_bwd_fp32_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl, n_images=4)
    p = dcn.make_problem(4, wl.H, wl.W, wl.G, wl.Cg, offset_scale=wl.offset_scale)
    args = [to_dev(d[k], "f32") for k in ("x", "offset", "mask", "grad_out")]
    a = gpu_backward(p, *args)
    b = gpu_backward(p, *args)
    torch.cuda.synchronize()
    # offset and mask gradients are computed without atomics: bitwise equal
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # the input gradient sums atomically: equal up to the order of additions
    assert torch.allclose(a[0], b[0], rtol=0, atol=1e-5 * float(a[0].abs().max()))


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_full_size_backward_half(gen_mod, oracle_mod, dtype):
    """The stage-2 backward with 2-byte storage, every element against the
    oracle fed the same rounded inputs."""
    wl = WORKLOADS[f"internimage_l_stage2_bwd_{'bf16' if dtype == 'bf16' else 'fp16'}_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl)
    p = dcn.problem_for(wl)
    check(oracle_mod, p, d["x"], d["offset"], d["mask"], d["grad_out"], dtype)


@pytest.mark.parametrize("N,H,W,G,dtype", [(5, 21, 23, 4, "f32"), (11, 12, 13, 3, "f32"),
                                           (9, 16, 16, 2, "bf16"), (3, 7, 5, 2, "bf16"),
                                           (1, 14, 15, 3, "f32"), (6, 10, 9, 2, "f16")])
def test_backward_host_entry_point(oracle_mod, N, H, W, G, dtype):
    """The chunked host backward: grad_offset and grad_mask have the bits of
    the device backward on the whole batch (they do not depend on the order of
    additions), grad_input agrees within the usual gate, and all three match
    the oracle."""
    Cg = 16
    p = dcn.make_problem(N, H, W, G, Cg, offset_scale=2.0, dtype=dtype)
    Ho, Wo = dcn.dcn_core_output_hw(p)
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    off = (1.5 * RNG.standard_normal((N, Ho, Wo, G * 18))).astype(np.float32)
    mask = RNG.standard_normal((N, Ho, Wo, G * 9)).astype(np.float32)
    gout = RNG.standard_normal((N, Ho, Wo, G * Cg)).astype(np.float32)
    xd, od, md, gd = (to_dev(a, dtype) for a in (x, off, mask, gout))
    hg = gd.cpu().pin_memory()
    hgx, hgo, hgm = (torch.full(t.shape, float("nan"), dtype=t.dtype).pin_memory()
                     for t in (xd, od, md))
    dg, dgx, dgo, dgm = (torch.full_like(t, 3.0) for t in (gd, xd, od, md))
    ws = dcn.dcn_core_backward_workspace(p)
    wbuf = torch.empty(ws, dtype=torch.uint8, device="cuda") if ws else None
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    dcn.dcn_core_backward_host(p, xd, od, md, hg, hgx, hgo, hgm, dg, dgx, dgo, dgm, wbuf, ws,
                               stream=s)
    dcn.dcn_core_sync_status(s)
    rgx, rgo, rgm = gpu_backward(p, xd, od, md, gd)
    torch.cuda.synchronize()
    assert torch.equal(hgo, rgo.cpu()) and torch.equal(hgm, rgm.cpu())
    assert_bwd(f64(hgx), f64(rgx), "host vs device grad_input", dtype)
    rx, roff, rm = oracle_mod.backward(f64(xd), f64(od), f64(md), f64(gd), **problem_kwargs(p))
    assert_bwd(f64(hgx), rx, "grad_input", dtype)
    assert_bwd(f64(hgo), roff, "grad_offset", dtype)
    assert_bwd(f64(hgm), rm, "grad_mask", dtype)
