"""The deterministic backward, dcn_core_backward_deterministic.

grad_input is accumulated exactly in 64-bit fixed point, so its bits must not
depend on the order of the additions: these tests check parity with the oracle
(same gates as the other backward tests), bitwise agreement across reruns,
streams, tile shapes and both backward kernels, bitwise agreement of
grad_offset / grad_mask with dcn_core_backward, and the documented NaN result
for a non-finite grad_out.
"""
import contextlib
import os

import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from gen.workloads import WORKLOADS
from tests.dcn_testutil import assert_bwd, f64, gpu_backward, problem_kwargs, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(99)


@contextlib.contextmanager
def env(**kv):
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


def det_backward(p, x, off, mask, gout, stream=None):
    gx, goff, gm = torch.empty_like(x), torch.empty_like(off), torch.empty_like(mask)
    nbytes = dcn.dcn_core_backward_deterministic_workspace(p)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    dcn.dcn_core_backward_deterministic(p, x, off, mask, gout, gx, goff, gm, ws, nbytes, stream)
    return gx, goff, gm


def random_inputs(p, off_sd=1.5):
    Ho, Wo = dcn.dcn_core_output_hw(p)
    T = dcn.taps(p)
    x = RNG.standard_normal((p.N, p.H, p.W, p.G * p.Cg)).astype(np.float32)
    off = (off_sd * RNG.standard_normal((p.N, Ho, Wo, p.G * T * 2))).astype(np.float32)
    mask = RNG.standard_normal((p.N, Ho, Wo, p.G * T)).astype(np.float32)
    gout = RNG.standard_normal((p.N, Ho, Wo, p.G * p.Cg)).astype(np.float32)
    return x, off, mask, gout


CASES = [
    dict(N=2, H=23, W=29, G=3, Cg=16),
    dict(N=2, H=19, W=17, G=5, Cg=16, softmax=0),
    dict(N=2, H=23, W=29, G=3, Cg=16, remove_center=1),
    dict(N=2, H=24, W=26, G=3, Cg=16, stride=2),
    dict(N=2, H=17, W=19, G=3, Cg=16, K=5, pad=2),
    dict(N=2, H=15, W=21, G=4, Cg=8),
    dict(N=2, H=13, W=14, G=3, Cg=32, softmax=0),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("case", CASES, ids=["_".join(f"{k}{v}" for k, v in c.items())
                                             for c in CASES])
def test_deterministic_backward_matches_oracle(oracle_mod, case, dtype):
    kw = {"K": 3, "stride": 1, "pad": 1, "softmax": 1, "remove_center": 0, **case}
    p = dcn.make_problem(kw["N"], kw["H"], kw["W"], kw["G"], kw["Cg"], kw["K"], kw["stride"],
                         kw["pad"], 1, 2.0, kw["softmax"], dtype, kw["remove_center"])
    xd, od, md, gd = (to_dev(a, dtype) for a in random_inputs(p))
    gx, goff, gm = det_backward(p, xd, od, md, gd)
    ref = gpu_backward(p, xd, od, md, gd)
    torch.cuda.synchronize()
    rx, roff, rm = oracle_mod.backward(f64(xd), f64(od), f64(md), f64(gd), **problem_kwargs(p))
    assert_bwd(f64(gx), rx, f"grad_input {p}", dtype)
    assert_bwd(f64(goff), roff, f"grad_offset {p}", dtype)
    assert_bwd(f64(gm), rm, f"grad_mask {p}", dtype)
    # offset and mask gradients do not use the accumulator: the same bits as dcn_core_backward
    assert torch.equal(goff, ref[1]) and torch.equal(gm, ref[2])


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_offset_and_mask_gradients_have_the_same_raw_bits_in_both_kernels(gen_mod, dtype):
    """With 2-byte storage the tiled backward forms the corner dot products
    with the mixed-precision FMA on the raw 16-bit words; the direct kernel
    widens both operands first.  The products are exact either way, so
    grad_offset and grad_mask carry the same bits, the sign of zero included
    (compared as integers).  The batch includes zero grad_out rows."""
    wl = WORKLOADS[f"internimage_l_stage2_bwd_{ {'bf16': 'bf16', 'f16': 'fp16'}[dtype]}_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl, n_images=4)
    d["grad_out"][1, 5:9] = 0.0    # whole rows of zero gradient
    d["grad_out"][2, :, 7] = -0.0
    p = dcn.make_problem(4, wl.H, wl.W, wl.G, wl.Cg, offset_scale=wl.offset_scale, dtype=dtype)
    args = [to_dev(d[k], dtype) for k in ("x", "offset", "mask", "grad_out")]
    tiled = gpu_backward(p, *args)
    with env(DCN_CORE_BACKWARD="direct"):
        direct = gpu_backward(p, *args)
    torch.cuda.synchronize()
    for a, b in ((tiled[1], direct[1]), (tiled[2], direct[2])):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_deterministic_backward_is_bitwise_reproducible(gen_mod, dtype):
    """Reruns, another stream, other tile shapes and the direct kernel all
    give the same grad_input bits: the fixed-point sum does not depend on the
    order of the additions."""
    wl = WORKLOADS[f"internimage_l_stage2_bwd_{ {'f32': 'fp32', 'bf16': 'bf16', 'f16': 'fp16'}[dtype]}_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl, n_images=6)
    p = dcn.make_problem(6, wl.H, wl.W, wl.G, wl.Cg, offset_scale=wl.offset_scale, dtype=dtype)
    args = [to_dev(d[k], dtype) for k in ("x", "offset", "mask", "grad_out")]
    base = det_backward(p, *args)
    runs = [det_backward(p, *args)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        runs.append(det_backward(p, *args, stream=s))
    s.synchronize()
    for tile in ("3x5", "16x16", "48x8"):
        with env(DCN_CORE_BWD_TILED_TILE=tile):
            runs.append(det_backward(p, *args))
    with env(DCN_CORE_BACKWARD="direct"):
        runs.append(det_backward(p, *args))
    torch.cuda.synchronize()
    for i, r in enumerate(runs):
        assert torch.equal(r[0], base[0]), f"grad_input differs in run {i}"
        assert torch.equal(r[1], base[1]) and torch.equal(r[2], base[2]), f"run {i}"
    # and it agrees with the atomic backward within the usual gate
    ref = gpu_backward(p, *args)
    torch.cuda.synchronize()
    assert_bwd(f64(base[0]), f64(ref[0]), "deterministic vs atomic grad_input", dtype)


def test_deterministic_backward_full_size(gen_mod, oracle_mod):
    wl = WORKLOADS["internimage_l_stage2_bwd_fp32_n32_48x48_c320"]
    d = gen_mod.make_inputs(wl)
    p = dcn.problem_for(wl)
    args = [to_dev(d[k], "f32") for k in ("x", "offset", "mask", "grad_out")]
    gx, goff, gm = det_backward(p, *args)
    torch.cuda.synchronize()
    rx, roff, rm = oracle_mod.backward(d["x"], d["offset"], d["mask"], d["grad_out"],
                                       **problem_kwargs(p))
    assert_bwd(f64(gx), rx, "grad_input")
    assert_bwd(f64(goff), roff, "grad_offset")
    assert_bwd(f64(gm), rm, "grad_mask")


def test_deterministic_backward_nonfinite_grad_out_gives_nan():
    p = dcn.make_problem(1, 9, 10, 2, 16, offset_scale=2.0)
    x, off, mask, gout = random_inputs(p)
    gout[0, 3, 4, 5] = np.inf
    gx, goff, gm = det_backward(p, *(to_dev(a, "f32") for a in (x, off, mask, gout)))
    torch.cuda.synchronize()
    assert torch.isnan(gx).all()
    dcn.dcn_core_sync_status()
