"""Offset / mask projection on the tensor cores (dcn_core_offset_mask_projection)
against the oracle's float64 matrix product, element by element.

bf16 x bf16 products are exact in fp32, so the only error of the fp32 output
is the rounding of the K-term sum: the gate is 4 * Cq * 2^-24 times the sum of
the absolute terms (plus |bias|), per element; bf16 outputs add one rounding,
2^-8 of the value.
"""
import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from tests.dcn_testutil import f64, gpu_forward, problem_kwargs, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(31)


def bf16_round(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def run_case(oracle_mod, N, Ho, Wo, G, Cq, dtype="f32", K=3, remove_center=0, bias=True,
             scale=1.0):
    pad = K // 2
    p = dcn.make_problem(N, Ho, Wo, G, 16, K, 1, pad, 1, 2.0, 1, dtype, remove_center)
    assert dcn.dcn_core_output_hw(p) == (Ho, Wo)
    T = dcn.taps(p)
    q = bf16_round(scale * RNG.standard_normal((N, Ho, Wo, Cq)))
    w = bf16_round(RNG.standard_normal((G * T * 3, Cq)) / np.sqrt(Cq))
    b = torch.from_numpy(RNG.standard_normal(G * T * 3).astype(np.float32)) if bias else None
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    off = torch.empty((N, Ho, Wo, G * T * 2), dtype=tdt, device="cuda")
    msk = torch.empty((N, Ho, Wo, G * T), dtype=tdt, device="cuda")
    qd, wd = q.cuda(), w.cuda()
    bd = b.cuda() if bias else None
    dcn.dcn_core_offset_mask_projection(p, qd, Cq, wd, bd, off, msk)
    torch.cuda.synchronize()
    qf, wf = f64(q), f64(w)
    bf = None if b is None else b.numpy().astype(np.float64)
    ro, rm = oracle_mod.projection(qf, wf, bf, G=G, K=K, remove_center=remove_center)
    # per-element bound from the absolute terms of each sum
    absP = np.abs(qf).reshape(-1, Cq) @ np.abs(wf).T
    if bf is not None:
        absP = absP + np.abs(bf)[None, :]
    absP = absP.reshape(N, Ho, Wo, -1)
    bound = 4 * Cq * 2.0 ** -24 * absP + 1e-30
    for got, ref, bnd, name in ((off, ro, bound[..., :G * T * 2], "offset"),
                                (msk, rm, bound[..., G * T * 2:], "mask")):
        g = f64(got)
        tol = bnd + (2.0 ** -8 * np.abs(ref) if dtype == "bf16" else 0.0)
        bad = np.abs(g - ref) > tol
        assert not bad.any(), (f"{name}: {int(bad.sum())} of {bad.size} outside the bound, "
                               f"max err {np.abs(g - ref).max():.3e}")
    return p, off, msk


CASES = [
    dict(N=2, Ho=13, Wo=11, G=10, Cq=160),               # stage-1 channels, ragged pixel count
    dict(N=1, Ho=7, Wo=9, G=5, Cq=64),                   # 135 columns: two ragged column tiles
    dict(N=1, Ho=16, Wo=16, G=4, Cq=72),                 # a partial K block
    dict(N=2, Ho=5, Wo=7, G=2, Cq=8),                    # the smallest K
    dict(N=1, Ho=9, Wo=9, G=3, Cq=96, remove_center=1),  # 8-tap set: 72 columns
    dict(N=1, Ho=12, Wo=10, G=10, Cq=160, bias=False),
    dict(N=1, Ho=8, Wo=8, G=20, Cq=320),                 # 540 columns, five K blocks
    dict(N=1, Ho=6, Wo=6, G=2, Cq=64, K=5),              # 25 taps
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=["_".join(f"{k}{v}" for k, v in c.items())
                                             for c in CASES])
def test_projection_matches_oracle(oracle_mod, case, dtype):
    run_case(oracle_mod, dtype=dtype, **case)
    dcn.dcn_core_sync_status()


def test_projection_at_stage1_size(oracle_mod):
    """InternImage-L stage 1 (N=32, 96x96, Cq=160, G=10): 294 912 pixels, 2304 x 3
    tiles over the persistent grid; checked on sampled pixels."""
    N, Ho, Wo, G, Cq = 32, 96, 96, 10, 160
    p = dcn.make_problem(N, Ho, Wo, G, 16, offset_scale=2.0)
    q = bf16_round(RNG.standard_normal((N, Ho, Wo, Cq)))
    w = bf16_round(RNG.standard_normal((G * 27, Cq)) / np.sqrt(Cq))
    b = torch.from_numpy(RNG.standard_normal(G * 27).astype(np.float32))
    off = torch.empty((N, Ho, Wo, G * 18), device="cuda")
    msk = torch.empty((N, Ho, Wo, G * 9), device="cuda")
    dcn.dcn_core_offset_mask_projection(p, q.cuda(), Cq, w.cuda(), b.cuda(), off, msk)
    torch.cuda.synchronize()
    pix = RNG.integers(0, N * Ho * Wo, size=4000)
    qs = f64(q).reshape(-1, Cq)[pix]
    ro, rm = oracle_mod.projection(qs, f64(w), b.numpy().astype(np.float64), G=G)
    bound = 4 * Cq * 2.0 ** -24 * (np.abs(qs) @ np.abs(f64(w)).T + np.abs(b.numpy())[None, :])
    go = f64(off).reshape(-1, G * 18)[pix]
    gm = f64(msk).reshape(-1, G * 9)[pix]
    assert (np.abs(go - ro) <= bound[:, :G * 18]).all()
    assert (np.abs(gm - rm) <= bound[:, G * 18:]).all()
    dcn.dcn_core_sync_status()


def test_projection_feeds_the_forward(oracle_mod):
    """The DCNv3 block's path: projection on the tensor cores, then the core
    forward on its offsets and mask, equals the oracle forward on the same
    offsets and mask."""
    N, H, W, G, Cq = 2, 20, 18, 4, 64
    p, off, msk = run_case(oracle_mod, N, H, W, G, Cq, scale=0.5)
    x = RNG.standard_normal((N, H, W, G * 16)).astype(np.float32)
    xd = to_dev(x, "f32")
    out = gpu_forward(p, xd, off, msk)
    torch.cuda.synchronize()
    ref = oracle_mod.forward(x, f64(off), f64(msk), **problem_kwargs(p))
    assert np.abs(f64(out) - ref).max() <= 1e-5 * np.abs(x).max()


@pytest.mark.parametrize("M,K,Nout,out_dtype", [(300, 160, 160, "f32"), (1000, 320, 320, "bf16"),
                                                (129, 64, 40, "f32"), (77, 8, 130, "bf16"),
                                                (50, 16, 33, "bf16"), (70, 24, 33, "f32")])
def test_linear_matches_oracle(oracle_mod, M, K, Nout, out_dtype):
    x = bf16_round(RNG.standard_normal((M, K)))
    w = bf16_round(RNG.standard_normal((Nout, K)) / np.sqrt(K))
    b = torch.from_numpy(RNG.standard_normal(Nout).astype(np.float32))
    y = torch.empty((M, Nout), dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16,
                    device="cuda")
    dcn.dcn_core_linear_bf16(x.cuda(), M, K, w.cuda(), Nout, b.cuda(), y, out_dtype)
    torch.cuda.synchronize()
    xf, wf, bf = f64(x), f64(w), b.numpy().astype(np.float64)
    ref = oracle_mod.linear(xf, wf, bf)
    bound = 4 * K * 2.0 ** -24 * (np.abs(xf) @ np.abs(wf).T + np.abs(bf)[None, :])
    if out_dtype == "bf16":
        bound = bound + 2.0 ** -8 * np.abs(ref)
    assert (np.abs(f64(y) - ref) <= bound).all()


def test_dcnv3_block_core_path_bf16(oracle_mod):
    """The block around the core operator, bf16 activations: offset / mask
    projection (tensor cores) -> core forward -> output_proj (tensor cores).
    Each GPU stage is checked against the oracle fed that stage's GPU inputs."""
    N, H, W, G, Cg = 2, 24, 20, 4, 16
    C = G * Cg
    p, off, msk = run_case(oracle_mod, N, H, W, G, C, dtype="bf16", scale=0.5)
    x = bf16_round(RNG.standard_normal((N, H, W, C))).cuda()
    core = gpu_forward(p, x, off, msk)
    w_out = bf16_round(RNG.standard_normal((C, C)) / np.sqrt(C))
    b_out = torch.from_numpy(RNG.standard_normal(C).astype(np.float32))
    y = torch.empty((N * H * W, C), dtype=torch.bfloat16, device="cuda")
    dcn.dcn_core_linear_bf16(core, N * H * W, C, w_out.cuda(), C, b_out.cuda(), y, "bf16")
    torch.cuda.synchronize()
    ref_core = oracle_mod.forward(f64(x), f64(off), f64(msk), **problem_kwargs(p))
    assert np.abs(f64(core) - ref_core).max() <= 1e-2 * np.abs(ref_core).max()
    ref_y = oracle_mod.linear(f64(core).reshape(-1, C), f64(w_out), b_out.numpy())
    assert np.abs(f64(y) - ref_y).max() <= 1e-2 * np.abs(ref_y).max()
