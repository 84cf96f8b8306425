"""Guide features of the offset / mask branch (dcn_core_offset_mask_guide:
depthwise 3x3, LayerNorm, GELU, bf16 out) against the oracle, element by
element.

Gate: the output is rounded once to bf16 (relative error at most 2^-9 of the
value); the fp32 convolution, LayerNorm and erf before it add errors of order
1e-6 on values of order one.  So |got - ref| <= 2^-8 |ref| + 2e-5.
"""
import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from tests.dcn_testutil import f64, gpu_forward, problem_kwargs, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(53)


def gate(got, ref):
    return np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-5


def params(C, affine=True):
    w = RNG.uniform(-0.5, 0.5, size=(3, 3, C)).astype(np.float32)
    if not affine:
        return w, None, None, None
    b = RNG.uniform(-0.2, 0.2, size=C).astype(np.float32)
    g = RNG.uniform(0.5, 1.5, size=C).astype(np.float32)
    be = RNG.uniform(-0.3, 0.3, size=C).astype(np.float32)
    return w, b, g, be


def run_guide(p, x_dev, w, b, g, be, eps, stream=None):
    dev = lambda a: None if a is None else torch.from_numpy(a).cuda()
    q = torch.empty(x_dev.shape, dtype=torch.bfloat16, device="cuda")
    dcn.dcn_core_offset_mask_guide(p, x_dev, dev(w), dev(b), dev(g), dev(be), eps, q, stream)
    return q


# (N, H, W, G, Cg, dtype): the lanes-per-pixel choices 8 x 5 quads (C=160), 16 x 1
# (C=64), 16 x 5 (320), 32 x 10 (1280), 4 x 1 with three live quads (C=12),
# 4 x 13 (C=196, ragged), 32 x 16 with 64 KB of shared memory (C=2048); ragged
# column and row tiles; a one-pixel image
CASES = [(2, 13, 11, 10, 16, "f32"), (1, 9, 37, 4, 16, "bf16"), (2, 5, 70, 20, 16, "bf16"),
         (1, 3, 3, 80, 16, "f32"), (1, 1, 1, 2, 4, "f32"), (2, 17, 9, 3, 4, "f32"),
         (1, 4, 5, 49, 4, "f32"), (1, 6, 7, 128, 16, "bf16"), (3, 10, 33, 12, 16, "bf16"),
         (2, 7, 19, 20, 16, "f32")]  # fp32 at C = 320: two rows per pass, an odd row count


@pytest.mark.parametrize("case", CASES, ids=[f"N{c[0]}_{c[1]}x{c[2]}_C{c[3] * c[4]}_{c[5]}"
                                             for c in CASES])
def test_guide_matches_oracle(oracle_mod, case):
    N, H, W, G, Cg, dtype = case
    C = G * Cg
    p = dcn.make_problem(N, H, W, G, Cg, dtype=dtype)
    x = RNG.standard_normal((N, H, W, C)).astype(np.float32)
    xd = to_dev(x, dtype)
    w, b, g, be = params(C)
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    dcn.dcn_core_sync_status()
    ref = oracle_mod.guide(f64(xd), w, b, g, be, 1e-6)
    ok = gate(f64(q), ref)
    assert ok.all(), f"{int((~ok).sum())} of {ok.size} outside the gate, max err {np.abs(f64(q) - ref).max():.3e}"


def test_guide_without_affine_parameters(oracle_mod):
    """NULL bias, gamma and beta read as 0, 1 and 0."""
    N, H, W, G, Cg = 2, 8, 12, 4, 16
    C = G * Cg
    p = dcn.make_problem(N, H, W, G, Cg)
    x = RNG.standard_normal((N, H, W, C)).astype(np.float32)
    w = params(C, affine=False)[0]
    q = run_guide(p, to_dev(x, "f32"), w, None, None, None, 1e-5)
    dcn.dcn_core_sync_status()
    ref = oracle_mod.guide(x, w, np.zeros(C), np.ones(C), np.zeros(C), 1e-5)
    assert gate(f64(q), ref).all()


def test_guide_at_stage1_size(oracle_mod):
    """InternImage-L stage 1 in bf16 (N=64, 96x96, C=160): sampled pixels plus
    every pixel of the image border of two images."""
    N, H, W, G, Cg = 64, 96, 96, 10, 16
    C = G * Cg
    p = dcn.make_problem(N, H, W, G, Cg, dtype="bf16")
    xd = torch.randn((N, H, W, C), device="cuda").to(torch.bfloat16)
    w, b, g, be = params(C)
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    dcn.dcn_core_sync_status()
    border = [n * H * W + y * W + xx for n in (0, N - 1) for y in range(H) for xx in range(W)
              if y in (0, H - 1) or xx in (0, W - 1)]
    pix = np.unique(np.concatenate([RNG.integers(0, N * H * W, size=3000), np.array(border)]))
    ref = oracle_mod.guide(f64(xd), w, b, g, be, 1e-6, pixels=pix)
    got = f64(q).reshape(-1, C)[pix]
    ok = gate(got, ref)
    assert ok.all(), f"{int((~ok).sum())} outside the gate, max err {np.abs(got - ref).max():.3e}"


def test_guide_projection_forward_chain(oracle_mod):
    """The offset / mask branch end to end, bf16: guide -> projection (tensor
    cores) -> core forward.  Each GPU stage is checked against the oracle fed
    that stage's GPU inputs."""
    N, H, W, G, Cg = 2, 20, 18, 4, 16
    C = G * Cg
    p = dcn.make_problem(N, H, W, G, Cg, offset_scale=2.0, dtype="bf16")
    xd = to_dev(RNG.standard_normal((N, H, W, C)).astype(np.float32), "bf16")
    w, b, g, be = params(C)
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    pw = torch.from_numpy((RNG.standard_normal((G * 27, C)) / np.sqrt(C)).astype(np.float32))
    pw = pw.to(torch.bfloat16).cuda()
    pb = torch.from_numpy((0.1 * RNG.standard_normal(G * 27)).astype(np.float32)).cuda()
    off = torch.empty((N, H, W, G * 18), dtype=torch.bfloat16, device="cuda")
    msk = torch.empty((N, H, W, G * 9), dtype=torch.bfloat16, device="cuda")
    dcn.dcn_core_offset_mask_projection(p, q, C, pw, pb, off, msk)
    out = gpu_forward(p, xd, off, msk)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status()
    ref_q = oracle_mod.guide(f64(xd), w, b, g, be, 1e-6)
    assert gate(f64(q), ref_q).all()
    ro, rm = oracle_mod.projection(f64(q), f64(pw), f64(pb), G=G)
    tol = 4 * C * 2.0 ** -24 * 8 + 2.0 ** -8
    assert np.abs(f64(off) - ro).max() <= tol * max(1.0, np.abs(ro).max())
    assert np.abs(f64(msk) - rm).max() <= tol * max(1.0, np.abs(rm).max())
    ref = oracle_mod.forward(f64(xd), f64(off), f64(msk), **problem_kwargs(p))
    assert np.abs(f64(out) - ref).max() <= 1e-2 * np.abs(ref).max()


def fused_inputs(N, H, W, G, dtype, affine=True):
    C = G * 16
    p = dcn.make_problem(N, H, W, G, 16, offset_scale=2.0, dtype=dtype)
    xd = to_dev(RNG.standard_normal((N, H, W, C)).astype(np.float32), dtype)
    w, b, g, be = params(C, affine)
    pw = torch.from_numpy((RNG.standard_normal((G * 27, C)) / np.sqrt(C)).astype(np.float32))
    pw = pw.to(torch.bfloat16).cuda()
    pb = torch.from_numpy((0.1 * RNG.standard_normal(G * 27)).astype(np.float32)).cuda()
    return p, xd, (w, b, g, be), pw, pb


def projection_outputs(p, dtype):
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    off = torch.empty((p.N, p.H, p.W, p.G * 18), dtype=tdt, device="cuda")
    msk = torch.empty((p.N, p.H, p.W, p.G * 9), dtype=tdt, device="cuda")
    return off, msk


# (N, H, W, G, dtype): C = 160 (8 lanes x 5 quads, two A tiles in flight) and
# 320 (16 lanes, one A tile); a last 128-pixel tile that is partly outside the
# batch; a batch smaller than one tile; fp32, bf16 and fp16 inputs and outputs
FUSED = [(2, 12, 13, 10, "bf16"), (3, 9, 11, 10, "f32"), (1, 20, 17, 20, "bf16"),
         (2, 7, 9, 20, "f32"), (2, 11, 10, 10, "f16"), (1, 1, 3, 10, "bf16")]


@pytest.mark.parametrize("case", FUSED, ids=[f"N{c[0]}_{c[1]}x{c[2]}_C{c[3] * 16}_{c[4]}"
                                             for c in FUSED])
def test_fused_guide_projection_equals_the_two_calls(oracle_mod, case):
    """dcn_core_offset_mask_guide_projection gives, bit for bit, the offsets
    and mask of the guide followed by the projection (the same arithmetic, the
    same bf16 query, the same tensor-core products), and both match the oracle."""
    N, H, W, G, dtype = case
    C = G * 16
    p, xd, (w, b, g, be), pw, pb = fused_inputs(N, H, W, G, dtype)
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    off1, msk1 = projection_outputs(p, dtype)
    dcn.dcn_core_offset_mask_projection(p, q, C, pw, pb, off1, msk1)
    off2, msk2 = projection_outputs(p, dtype)
    dev = lambda a: torch.from_numpy(a).cuda()
    dcn.dcn_core_offset_mask_guide_projection(p, xd, dev(w), dev(b), dev(g), dev(be), 1e-6, pw,
                                              pb, off2, msk2)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status()
    assert torch.equal(off1, off2) and torch.equal(msk1, msk2)
    ref_q = oracle_mod.guide(f64(xd), w, b, g, be, 1e-6)
    assert gate(f64(q), ref_q).all()
    ro, rm = oracle_mod.projection(f64(q), f64(pw), f64(pb.cpu()), G=G)
    tol = 4 * C * 2.0 ** -24 * 8 + (2.0 ** -8 if dtype != "f32" else 0.0)
    assert np.abs(f64(off2) - ro).max() <= tol * max(1.0, np.abs(ro).max())
    assert np.abs(f64(msk2) - rm).max() <= tol * max(1.0, np.abs(rm).max())


def test_fused_guide_projection_at_stage1_size():
    """InternImage-L stage 1, bf16 (N=64, 96x96, C=160): the fused branch equals
    the two calls bit for bit over the whole batch."""
    N, H, W, G = 64, 96, 96, 10
    p, xd, (w, b, g, be), pw, pb = fused_inputs(N, H, W, G, "bf16")
    dev = lambda a: torch.from_numpy(a).cuda()
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    off1, msk1 = projection_outputs(p, "bf16")
    dcn.dcn_core_offset_mask_projection(p, q, G * 16, pw, pb, off1, msk1)
    off2, msk2 = projection_outputs(p, "bf16")
    dcn.dcn_core_offset_mask_guide_projection(p, xd, dev(w), dev(b), dev(g), dev(be), 1e-6, pw,
                                              pb, off2, msk2)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status()
    assert torch.equal(off1, off2) and torch.equal(msk1, msk2)


def test_fused_block_path_chain(oracle_mod):
    """The block's forward around the core operator with the fused branch,
    bf16, C = 160: guide + projection in one kernel -> core forward ->
    output_proj.  Each GPU stage is checked against the oracle fed that stage's
    GPU inputs (the query the branch keeps on chip is the standalone guide's,
    bit for bit)."""
    N, H, W, G = 2, 20, 18, 10
    C = G * 16
    p, xd, (w, b, g, be), pw, pb = fused_inputs(N, H, W, G, "bf16")
    dev = lambda a: torch.from_numpy(a).cuda()
    off, msk = projection_outputs(p, "bf16")
    dcn.dcn_core_offset_mask_guide_projection(p, xd, dev(w), dev(b), dev(g), dev(be), 1e-6, pw,
                                              pb, off, msk)
    core = gpu_forward(p, xd, off, msk)
    w_out = torch.from_numpy((RNG.standard_normal((C, C)) / np.sqrt(C)).astype(np.float32))
    w_out = w_out.to(torch.bfloat16)
    b_out = torch.from_numpy((0.1 * RNG.standard_normal(C)).astype(np.float32))
    y = torch.empty((N * H * W, C), dtype=torch.bfloat16, device="cuda")
    dcn.dcn_core_linear_bf16(core, N * H * W, C, w_out.cuda(), C, b_out.cuda(), y, "bf16")
    q = run_guide(p, xd, w, b, g, be, 1e-6)
    torch.cuda.synchronize()
    dcn.dcn_core_sync_status()
    assert gate(f64(q), oracle_mod.guide(f64(xd), w, b, g, be, 1e-6)).all()
    ro, rm = oracle_mod.projection(f64(q), f64(pw), f64(pb.cpu()), G=G)
    tol = 4 * C * 2.0 ** -24 * 8 + 2.0 ** -8
    assert np.abs(f64(off) - ro).max() <= tol * max(1.0, np.abs(ro).max())
    assert np.abs(f64(msk) - rm).max() <= tol * max(1.0, np.abs(rm).max())
    ref_core = oracle_mod.forward(f64(xd), f64(off), f64(msk), **problem_kwargs(p))
    assert np.abs(f64(core) - ref_core).max() <= 1e-2 * np.abs(ref_core).max()
    ref_y = oracle_mod.linear(f64(core).reshape(-1, C), f64(w_out), b_out.numpy())
    assert np.abs(f64(y) - ref_y).max() <= 1e-2 * np.abs(ref_y).max()


def test_fused_guide_projection_rejects_before_launch():
    """Shapes the fused kernel does not serve are refused on the host."""
    fake = 1 << 20
    for p in (dcn.make_problem(1, 8, 8, 4, 16, dtype="bf16"),           # C = 64
              dcn.make_problem(1, 8, 8, 40, 16, dtype="bf16"),          # C = 640
              dcn.make_problem(1, 8, 8, 10, 16, stride=2, dtype="bf16")):  # output 4 x 4
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_offset_mask_guide_projection(p, fake, fake, None, None, None, 1e-6,
                                                      fake, None, fake, fake, stream=0)
        assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
