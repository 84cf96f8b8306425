"""The operator inside a CUDA graph: forward + backward (and the deterministic
backward) captured once on a side stream and replayed.  The library allocates
nothing and never synchronises, so every launch and the grad_input zero-fill
are captured as graph nodes; replays must match eager calls."""
import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from tests.dcn_testutil import to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(5)


def inputs(p):
    Ho, Wo = dcn.dcn_core_output_hw(p)
    T = dcn.taps(p)
    x = RNG.standard_normal((p.N, p.H, p.W, p.G * p.Cg)).astype(np.float32)
    off = (1.5 * RNG.standard_normal((p.N, Ho, Wo, p.G * T * 2))).astype(np.float32)
    mask = RNG.standard_normal((p.N, Ho, Wo, p.G * T)).astype(np.float32)
    gout = RNG.standard_normal((p.N, Ho, Wo, p.G * p.Cg)).astype(np.float32)
    return x, off, mask, gout


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_backward_replay_in_a_cuda_graph(dtype):
    p = dcn.make_problem(4, 48, 48, 20, 16, offset_scale=2.0, dtype=dtype)
    x, off, mask, gout = (to_dev(a, dtype) for a in inputs(p))
    Ho, Wo = dcn.dcn_core_output_hw(p)
    out = torch.empty((p.N, Ho, Wo, p.G * p.Cg), dtype=x.dtype, device="cuda")
    gx, goff, gm = torch.empty_like(x), torch.empty_like(off), torch.empty_like(mask)
    ws_bytes = dcn.dcn_core_backward_workspace(p)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    dws_bytes = dcn.dcn_core_backward_deterministic_workspace(p)
    dws = torch.empty(dws_bytes, dtype=torch.uint8, device="cuda")
    dgx, dgoff, dgm = torch.empty_like(x), torch.empty_like(off), torch.empty_like(mask)

    s = torch.cuda.Stream()

    def step(stream):
        dcn.dcn_core_forward(p, x, off, mask, out, stream)
        dcn.dcn_core_backward(p, x, off, mask, gout, gx, goff, gm, ws if ws_bytes else None,
                              ws_bytes, stream)
        dcn.dcn_core_backward_deterministic(p, x, off, mask, gout, dgx, dgoff, dgm, dws,
                                            dws_bytes, stream)

    with torch.cuda.stream(s):
        step(s)  # eager, also the first-call lookups before capture
    s.synchronize()
    eager = [t.clone() for t in (out, gx, goff, gm, dgx, dgoff, dgm)]
    for t in (out, gx, goff, gm, dgx, dgoff, dgm):
        t.fill_(float("nan"))
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(torch.cuda.current_stream())
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status()
    got = (out, gx, goff, gm, dgx, dgoff, dgm)
    names = ("out", "grad_input", "grad_offset", "grad_mask", "det grad_input",
             "det grad_offset", "det grad_mask")
    for name, a, b in zip(names, got, eager):
        if name == "grad_input":  # atomic accumulation: equal up to the order of additions
            tol = 1e-5 if dtype == "f32" else 1e-2
            assert torch.allclose(a.float(), b.float(), rtol=0,
                                  atol=tol * float(b.float().abs().max())), name
        else:
            assert torch.equal(a, b), name
    del g
