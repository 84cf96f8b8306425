"""The allocation-free backward, dcn_core_backward_noalloc.

It serves callers that cannot allocate device memory where they run the
backward (runtimes that hand an operator only its input and output buffers,
latency-critical code that may not call cudaMalloc).  For bf16 storage its
fp32 grad_input accumulator lives in a fixed array inside the library, so
these tests check that two calls in a row -- with different inputs, so a
second call that did not start from a cleared array would show -- agree with
dcn_core_backward given a caller-allocated workspace, within the tolerances
the other backward tests use.  This file is collected last on purpose.
"""
import os

import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from tests.dcn_testutil import assert_bwd, f64, problem_kwargs, to_dev

RNG = np.random.default_rng(4242)


def inputs(p):
    Ho, Wo = dcn.dcn_core_output_hw(p)
    KK = dcn.taps(p)
    C = p.G * p.Cg
    x = RNG.standard_normal((p.N, p.H, p.W, C)).astype(np.float32)
    off = (1.5 * RNG.standard_normal((p.N, Ho, Wo, p.G * KK * 2))).astype(np.float32)
    mask = RNG.standard_normal((p.N, Ho, Wo, p.G * KK)).astype(np.float32)
    gout = RNG.standard_normal((p.N, Ho, Wo, C)).astype(np.float32)
    return x, off, mask, gout


def with_workspace(p, args):
    gx, goff, gm = (torch.empty_like(args[i]) for i in (0, 1, 2))
    ws_bytes = dcn.dcn_core_backward_workspace(p)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda") if ws_bytes else None
    dcn.dcn_core_backward(p, *args, gx, goff, gm, ws, ws_bytes)
    return gx, goff, gm


def without_alloc(p, args):
    gx, goff, gm = (torch.empty_like(args[i]) for i in (0, 1, 2))
    dcn.dcn_core_backward_noalloc(p, *args, gx, goff, gm)
    return gx, goff, gm


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_backward_matches_workspace_backward(dtype):
    # InternImage-L stage-2 shape with 4 images: the bf16 accumulator
    # (4*48*48*320*4 bytes = 11.8 MB) fits the library's 16 MiB array.
    p = dcn.make_problem(4, 48, 48, 20, 16, offset_scale=2.0, softmax=1, dtype=dtype)
    for call in range(2):
        args = [to_dev(a, dtype) for a in inputs(p)]
        ref = with_workspace(p, args)
        got = without_alloc(p, args)
        torch.cuda.synchronize()
        for name, g, r in zip(("grad_input", "grad_offset", "grad_mask"), got, ref):
            assert_bwd(f64(g), f64(r), f"call {call}: {name}", dtype)
    dcn.dcn_core_sync_status()


@pytest.mark.gpu
@pytest.mark.parametrize("case", [dict(K=5, Cg=16), dict(K=3, Cg=8), dict(K=3, Cg=32, softmax=0)],
                         ids=["K5", "Cg8", "Cg32_raw_mask"])
def test_noalloc_backward_matches_oracle_on_the_direct_kernels(oracle_mod, case):
    """bf16 through the shared array on shapes the tiled kernel does not serve
    (K = 5, 8 or 32 channels per group), and with the tiled kernel switched
    off, against the float64 oracle fed the same bf16-rounded inputs; two calls
    in a row with different inputs."""
    kw = {"softmax": 1, **case}
    old = os.environ.get("DCN_CORE_BACKWARD")
    os.environ["DCN_CORE_BACKWARD"] = "direct"
    try:
        p = dcn.make_problem(2, 13, 11, 3, kw.pop("Cg"), K=kw.pop("K"), offset_scale=2.0,
                             dtype="bf16", **kw)
        for call in range(2):
            args = [to_dev(a, "bf16") for a in inputs(p)]
            got = without_alloc(p, args)
            torch.cuda.synchronize()
            ref = oracle_mod.backward(*(f64(a) for a in args), **problem_kwargs(p))
            for name, g, r in zip(("grad_input", "grad_offset", "grad_mask"), got, ref):
                assert_bwd(f64(g), r, f"call {call}: {name}", "bf16")
        dcn.dcn_core_sync_status()
    finally:
        if old is None:
            os.environ.pop("DCN_CORE_BACKWARD", None)
        else:
            os.environ["DCN_CORE_BACKWARD"] = old


@pytest.mark.gpu
def test_noalloc_backward_at_the_exact_scratch_size():
    """A bf16 problem whose fp32 accumulator fills the array exactly
    (1 x 128 x 128 x 256 channels x 4 bytes = 16 MiB) is accepted and matches
    the workspace backward."""
    p = dcn.make_problem(1, 128, 128, 16, 16, offset_scale=2.0, softmax=1, dtype="bf16")
    assert p.N * p.H * p.W * p.G * p.Cg * 4 == dcn.DCN_CORE_NOALLOC_SCRATCH_BYTES
    args = [to_dev(a, "bf16") for a in inputs(p)]
    ref = with_workspace(p, args)
    got = without_alloc(p, args)
    torch.cuda.synchronize()
    for name, g, r in zip(("grad_input", "grad_offset", "grad_mask"), got, ref):
        assert_bwd(f64(g), f64(r), name, "bf16")
    dcn.dcn_core_sync_status()


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_backward_allocates_nothing(dtype):
    """After one warm call (which may load the kernels), a further call leaves
    the device's free memory and torch's reserved pool unchanged."""
    p = dcn.make_problem(2, 48, 48, 20, 16, offset_scale=2.0, softmax=1, dtype=dtype)
    args = [to_dev(a, dtype) for a in inputs(p)]
    outs = [torch.empty_like(args[i]) for i in (0, 1, 2)]
    dcn.dcn_core_backward_noalloc(p, *args, *outs)
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    dcn.dcn_core_backward_noalloc(p, *args, *outs)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0
    dcn.dcn_core_sync_status()


def test_noalloc_backward_rejects_problems_beyond_its_scratch():
    """A bf16 problem whose fp32 accumulator exceeds the fixed array is
    refused on the host, before anything is enqueued (no GPU needed)."""
    fake = 1 << 20  # 16-byte aligned, never dereferenced: the call fails before any launch
    p = dcn.make_problem(8, 96, 96, 10, 16, dtype="bf16")  # 8*96*96*160*4 = 47 MB
    assert p.N * p.H * p.W * p.G * p.Cg * 4 > dcn.DCN_CORE_NOALLOC_SCRATCH_BYTES
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_noalloc(p, *([fake] * 7), stream=0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    assert "scratch" in str(e.value)
