"""Forward parity: the CUDA path against the CPU oracle on the same seeded
inputs, element by element, through the C ABI.

Small and medium problems are compared in full (they span several tiles and
ragged tile edges); the full-size workloads, in the launch configuration the
benchmark times, are compared on sampled units the oracle computes one by one.
"""
import contextlib
import os

import numpy as np
import pytest
import torch

import deformable_convolution_core_b200 as dcn
from gen.workloads import WORKLOADS
from tests.dcn_testutil import assert_bwd, assert_fwd, f64, gpu_backward, gpu_forward, problem_kwargs, to_dev

pytestmark = pytest.mark.gpu

RNG = np.random.default_rng(2024)


def random_case(N, H, W, G, Cg, K=3, stride=1, pad=None, dil=1, sigma=2.0, softmax=1,
                dtype="f32", off_sd=1.5, off_lo=None, remove_center=0, stride_w=None,
                pad_w=None, dil_w=None):
    pad = (K // 2) * dil if pad is None else pad
    p = dcn.make_problem(N, H, W, G, Cg, K, stride, pad, dil, sigma, softmax, dtype,
                         remove_center, stride_w, pad_w, dil_w)
    Ho, Wo = dcn.dcn_core_output_hw(p)
    T = dcn.taps(p)
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    if off_lo is None:
        off = (off_sd * RNG.standard_normal((N, Ho, Wo, G * T * 2))).astype(np.float32)
    else:
        off = RNG.uniform(off_lo, -off_lo, (N, Ho, Wo, G * T * 2)).astype(np.float32)
    if softmax:
        mask = RNG.standard_normal((N, Ho, Wo, G * T)).astype(np.float32)
    else:
        mask = RNG.uniform(-1, 1, (N, Ho, Wo, G * T)).astype(np.float32)
    return p, x, off, mask


@contextlib.contextmanager
def forward_path(path):
    """Select the forward kernel: "auto" (the library's choice: the TMA-tiled
    kernel where it applies) or "direct" (the direct-gather kernel)."""
    old = os.environ.get("DCN_CORE_FORWARD")
    if path == "direct":
        os.environ["DCN_CORE_FORWARD"] = "direct"
    else:
        os.environ.pop("DCN_CORE_FORWARD", None)
    try:
        yield
    finally:
        if old is None:
            os.environ.pop("DCN_CORE_FORWARD", None)
        else:
            os.environ["DCN_CORE_FORWARD"] = old


def check_full(oracle_mod, p, x, off, mask, dtype):
    xd, od, md = to_dev(x, dtype), to_dev(off, dtype), to_dev(mask, dtype)
    out = gpu_forward(p, xd, od, md)
    torch.cuda.synchronize()
    ref = oracle_mod.forward(f64(xd), f64(od), f64(md), **problem_kwargs(p))
    assert_fwd(f64(out), ref, f64(xd), dtype, repr(p))
    return out


CASES = [
    # (N, H, W, G, Cg, dict)  -- ragged sizes, several tiles per image
    (2, 23, 29, 3, 16, dict(dtype="f32")),
    (2, 19, 27, 5, 16, dict(dtype="bf16")),
    (1, 33, 17, 10, 16, dict(dtype="bf16", softmax=0)),
    (3, 12, 12, 8, 16, dict(dtype="f32", softmax=0, sigma=1.0)),
    (2, 15, 21, 4, 4, dict(dtype="f32")),        # 16-byte units, fp32
    (2, 15, 21, 4, 8, dict(dtype="f32")),        # 32-byte units, fp32
    (2, 13, 14, 3, 32, dict(dtype="f32")),       # 128-byte units, fp32 (4 lanes)
    (2, 15, 21, 4, 8, dict(dtype="bf16")),       # 16-byte units, bf16
    (2, 13, 14, 3, 32, dict(dtype="bf16")),      # 64-byte units, bf16 (2 lanes)
    (1, 11, 10, 2, 64, dict(dtype="bf16")),      # 128-byte units, bf16 (4 lanes)
    (2, 17, 19, 3, 16, dict(dtype="f32", K=1, pad=0)),
    (2, 17, 19, 3, 16, dict(dtype="f32", K=5)),
    (1, 17, 19, 2, 16, dict(dtype="bf16", K=7, softmax=0)),
    (2, 24, 26, 3, 16, dict(dtype="f32", stride=2)),
    (2, 25, 27, 3, 16, dict(dtype="bf16", stride=2, softmax=0)),
    (2, 21, 22, 3, 16, dict(dtype="f32", dil=2)),
    (2, 21, 22, 3, 16, dict(dtype="f32", pad=0)),
    (1, 1, 1, 2, 16, dict(dtype="f32")),         # single pixel
    (1, 1, 7, 2, 16, dict(dtype="bf16")),        # single row
    (2, 3, 3, 2, 16, dict(dtype="f32", stride=5)),   # stride larger than the image
    (1, 40, 3, 80, 16, dict(dtype="bf16")),      # many groups
    (2, 20, 20, 2, 16, dict(dtype="f32", off_lo=-40.0)),   # most samples far outside
    # remove_center: the window without its centre (8 taps at K = 3, 24 at K = 5, 48 at K = 7)
    (2, 23, 29, 3, 16, dict(dtype="f32", remove_center=1)),
    (1, 33, 17, 10, 16, dict(dtype="bf16", softmax=0, remove_center=1)),
    (2, 25, 27, 4, 8, dict(dtype="bf16", stride=2, remove_center=1)),
    (2, 13, 14, 3, 32, dict(dtype="f32", softmax=0, remove_center=1)),
    (2, 17, 19, 3, 16, dict(dtype="f32", K=5, remove_center=1)),
    (1, 17, 19, 2, 16, dict(dtype="bf16", K=7, softmax=0, dil=2, remove_center=1)),
    # fp16 storage: the tiled kernel (3x3, 16 channels) and the direct one
    (2, 23, 29, 3, 16, dict(dtype="f16")),
    (1, 33, 17, 10, 16, dict(dtype="f16", softmax=0)),
    (2, 15, 21, 4, 8, dict(dtype="f16")),        # 16-byte units, fp16
    (2, 13, 14, 3, 32, dict(dtype="f16")),       # 64-byte units, fp16
    (2, 25, 27, 3, 16, dict(dtype="f16", stride=2, softmax=0)),
    (2, 23, 29, 3, 16, dict(dtype="f16", remove_center=1)),
    (1, 17, 19, 2, 16, dict(dtype="f16", K=5)),
    # separate height / width stride, padding and dilation
    (2, 23, 29, 3, 16, dict(dtype="f32", stride=1, stride_w=2, pad=1, pad_w=0)),
    (2, 26, 21, 4, 16, dict(dtype="bf16", stride=2, stride_w=1, dil=1, dil_w=2, pad_w=2)),
    (1, 19, 33, 3, 8, dict(dtype="f32", K=5, pad=2, pad_w=0, dil_w=2, remove_center=1)),
]


@pytest.mark.parametrize("path", ["auto", "direct"])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}x{c[1]}x{c[2]}_G{c[3]}_Cg{c[4]}_" +
                                             "_".join(f"{k}{v}" for k, v in c[5].items())
                                             for c in CASES])
def test_forward_matches_oracle(oracle_mod, case, path):
    N, H, W, G, Cg, kw = case
    dtype = kw.get("dtype", "f32")
    p, x, off, mask = random_case(N, H, W, G, Cg, **kw)
    with forward_path(path):
        check_full(oracle_mod, p, x, off, mask, dtype)


@pytest.mark.parametrize("halo,tile", [("0", "1x1"), ("2", "3x5"), ("9", "32x32"), ("5", "7x64")])
def test_tiled_kernel_tile_and_halo_settings(oracle_mod, halo, tile):
    """Every tile shape and halo width of the tiled kernel gives the same
    operator (only the split between box reads and global reads changes)."""
    old = {k: os.environ.get(k) for k in ("DCN_CORE_HALO", "DCN_CORE_TILED_TILE")}
    os.environ["DCN_CORE_HALO"], os.environ["DCN_CORE_TILED_TILE"] = halo, tile
    try:
        for dtype in ("f32", "bf16", "f16"):
            p, x, off, mask = random_case(2, 37, 41, 3, 16, dtype=dtype, off_sd=3.0)
            check_full(oracle_mod, p, x, off, mask, dtype)
            p, x, off, mask = random_case(1, 40, 36, 2, 16, dtype=dtype, stride=2, softmax=0)
            check_full(oracle_mod, p, x, off, mask, dtype)
            p, x, off, mask = random_case(2, 29, 31, 3, 16, dtype=dtype, off_sd=3.0,
                                          remove_center=1)
            check_full(oracle_mod, p, x, off, mask, dtype)
            if dtype != "f32":  # 8 channels of a 2-byte type: 16-byte groups
                p, x, off, mask = random_case(2, 37, 41, 3, 8, dtype=dtype, off_sd=3.0)
                check_full(oracle_mod, p, x, off, mask, dtype)
                p, x, off, mask = random_case(1, 40, 36, 4, 8, dtype=dtype, stride=2, softmax=0,
                                              remove_center=1)
                check_full(oracle_mod, p, x, off, mask, dtype)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def test_identity_and_box_filter_on_gpu(oracle_mod):
    # Zero offsets with a one-hot centre mask give the input back exactly; zero
    # logits give the 3x3 box filter (the "plain 3x3 convolution" start state).
    N, H, W, G, Cg = 2, 13, 17, 3, 16
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    off = np.zeros((N, H, W, G * 18), np.float32)
    onehot = np.zeros((N, H, W, G, 9), np.float32)
    onehot[..., 4] = 1.0
    p = dcn.make_problem(N, H, W, G, Cg, softmax=0)
    out = gpu_forward(p, to_dev(x, "f32"), to_dev(off, "f32"), to_dev(onehot.reshape(N, H, W, -1), "f32"))
    assert np.array_equal(f64(out), x.astype(np.float64))
    p1 = dcn.make_problem(N, H, W, G, Cg, softmax=1)
    logits = np.zeros((N, H, W, G * 9), np.float32)
    out = gpu_forward(p1, to_dev(x, "f32"), to_dev(off, "f32"), to_dev(logits, "f32"))
    xp = np.pad(x.astype(np.float64), ((0, 0), (1, 1), (1, 1), (0, 0)))
    box = sum(xp[:, i:i + H, j:j + W, :] for i in range(3) for j in range(3)) / 9.0
    np.testing.assert_allclose(f64(out), box, rtol=0, atol=1e-5 * np.abs(x).max())


@pytest.mark.parametrize("K", [3, 5])
def test_remove_center_ring_mean_on_gpu(K):
    # Zero offsets and equal logits without the centre tap: the zero-padded
    # mean of the other K*K - 1 window positions.
    N, H, W, G, Cg = 2, 14, 11, 3, 16
    r, T = K // 2, K * K - 1
    x = RNG.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    p = dcn.make_problem(N, H, W, G, Cg, K, pad=r, softmax=1, remove_center=1)
    off = np.zeros((N, H, W, G * T * 2), np.float32)
    logits = np.full((N, H, W, G * T), 0.25, np.float32)
    out = gpu_forward(p, to_dev(x, "f32"), to_dev(off, "f32"), to_dev(logits, "f32"))
    xp = np.pad(x.astype(np.float64), ((0, 0), (r, r), (r, r), (0, 0)))
    ring = sum(xp[:, i:i + H, j:j + W, :] for i in range(K) for j in range(K)
               if (i, j) != (r, r)) / T
    np.testing.assert_allclose(f64(out), ring, rtol=0, atol=1e-5 * np.abs(x).max())


def test_nonfinite_and_border_offsets(oracle_mod):
    N, H, W, G, Cg = 1, 9, 11, 2, 16
    p, x, off, mask = random_case(N, H, W, G, Cg)
    o = off.reshape(N, H, W, G, 9, 2)
    o[0, 0, 0, 0, :, 0] = np.nan
    o[0, 1, 1, 0, :, 1] = np.inf
    o[0, 2, 2, 1, :, 0] = -np.inf
    o[0, 3, 3, 0, :, :] = 1e30
    # samples exactly on the borders -1, 0, W-1 and W (sigma = 2)
    o[0, 4, :, 1, 4, 0] = (np.array([-1, 0, W - 1, W] * 3)[:W] - np.arange(W)) / 2.0
    check_full(oracle_mod, p, x, off, mask, "f32")


@pytest.mark.parametrize("halo,tile", [("0", "1x1"), ("2", "3x5"), ("4", "24x24"), ("5", "9x40")])
def test_wide_window_tiled_kernel_tile_and_halo_settings(oracle_mod, halo, tile):
    """The wide-window tiled kernel (5x5 and 7x7 windows: batches of 8 units,
    taps in chunks) at every tile shape and halo width, in all three storage
    types: small tiles and no halo send most taps to the far path."""
    old = {k: os.environ.get(k) for k in ("DCN_CORE_HALO", "DCN_CORE_TILED_TILE")}
    os.environ["DCN_CORE_HALO"], os.environ["DCN_CORE_TILED_TILE"] = halo, tile
    try:
        for dtype in ("f32", "bf16", "f16"):
            p, x, off, mask = random_case(2, 23, 29, 3, 16, K=5, dtype=dtype, off_sd=2.0)
            check_full(oracle_mod, p, x, off, mask, dtype)
            p, x, off, mask = random_case(1, 26, 21, 2, 16, K=7, dtype=dtype, softmax=0,
                                          remove_center=1)
            check_full(oracle_mod, p, x, off, mask, dtype)
            p, x, off, mask = random_case(1, 30, 27, 2, 16, K=5, dtype=dtype, stride=2, dil=2,
                                          remove_center=1)
            check_full(oracle_mod, p, x, off, mask, dtype)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def test_tiled_kernels_alternate_shared_memory_sizes(oracle_mod):
    """The same tiled kernels launched with a large, a small and again the
    large shared-memory size (big image, tiny image, big image): the
    library's once-per-kernel shared-memory limit must only ever grow."""
    shapes = [(2, 96, 96), (1, 6, 7), (2, 96, 96)]
    for N, H, W in shapes:
        p, x, off, mask = random_case(N, H, W, 2, 16, dtype="bf16", off_sd=3.0)
        check_full(oracle_mod, p, x, off, mask, "bf16")
        xd, od, md = to_dev(x, "bf16"), to_dev(off, "bf16"), to_dev(mask, "bf16")
        gd = to_dev(RNG.standard_normal((N, H, W, 32)).astype(np.float32), "bf16")
        gx, goff, gm = gpu_backward(p, xd, od, md, gd)
        torch.cuda.synchronize()
        dcn.dcn_core_sync_status()
        rx, roff, rm = oracle_mod.backward(f64(xd), f64(od), f64(md), f64(gd), **problem_kwargs(p))
        assert_bwd(f64(gx), rx, f"grad_input {N}x{H}x{W}", "bf16")
        assert_bwd(f64(goff), roff, f"grad_offset {N}x{H}x{W}", "bf16")


def test_forward_is_deterministic_and_stream_safe(oracle_mod):
    p, x, off, mask = random_case(2, 31, 29, 6, 16, dtype="bf16")
    xd, od, md = to_dev(x, "bf16"), to_dev(off, "bf16"), to_dev(mask, "bf16")
    a = gpu_forward(p, xd, od, md)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = gpu_forward(p, xd, od, md, stream=s)
    s.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    dcn.dcn_core_sync_status(s)


# (N, H, W, G, Cg, dtype): image counts that cut into ragged chunks (5 -> 2+2+1,
# 11 -> five of 2 and 1, 17 -> four of 4 and 1, 9 -> four of 2 and 1) and sizes
# whose 32-byte chunk alignment forces one chunk (N=3 at 7x5 bf16: 1260-byte mask
# images; N=6 at 11x9, Cg 8)
HOST_CASES = [(2, 21, 23, 4, 16, "f32"), (5, 21, 23, 4, 16, "f32"), (11, 12, 13, 3, 16, "f32"),
              (17, 9, 10, 2, 16, "bf16"), (9, 16, 16, 2, 16, "bf16"), (3, 7, 5, 2, 16, "bf16"),
              (6, 11, 9, 3, 8, "f32"), (1, 30, 30, 2, 16, "f32")]


@pytest.mark.parametrize("case", HOST_CASES, ids=[f"N{c[0]}_{c[1]}x{c[2]}_G{c[3]}_Cg{c[4]}_{c[5]}"
                                                  for c in HOST_CASES])
def test_forward_host_entry_point(case):
    """The chunked, overlapped host path writes the same bits as the device
    forward on the whole batch, and orders itself after earlier work on the
    stream (the device buffers are first filled with garbage there)."""
    N, H, W, G, Cg, dtype = case
    p, x, off, mask = random_case(N, H, W, G, Cg, dtype=dtype)
    Ho, Wo = dcn.dcn_core_output_hw(p)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    hx, ho, hm = (torch.from_numpy(a).to(tdt).pin_memory() for a in (x, off, mask))
    hout = torch.full((N, Ho, Wo, G * Cg), float("nan"), dtype=tdt).pin_memory()
    dx, do, dm = (torch.empty_like(t, device="cuda") for t in (hx, ho, hm))
    dout = torch.empty(hout.shape, dtype=tdt, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for t in (dx, do, dm, dout):
            t.fill_(7.0)
    dcn.dcn_core_forward_host(p, hx, ho, hm, hout, dx, do, dm, dout, stream=s)
    dcn.dcn_core_sync_status(s)
    ref = gpu_forward(p, hx.cuda(), ho.cuda(), hm.cuda())
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())
    assert torch.equal(dx.cpu(), hx) and torch.equal(dm.cpu(), hm)


def test_forward_host_in_a_cuda_graph():
    """The host path's library streams join the caller's stream, so the call
    can be captured and replayed."""
    p, x, off, mask = random_case(5, 21, 23, 4, 16, dtype="f32")
    Ho, Wo = dcn.dcn_core_output_hw(p)
    hx, ho, hm = (torch.from_numpy(a).pin_memory() for a in (x, off, mask))
    hout = torch.zeros((5, Ho, Wo, 64), dtype=torch.float32).pin_memory()
    dx, do, dm = (torch.empty_like(t, device="cuda") for t in (hx, ho, hm))
    dout = torch.empty(hout.shape, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    dcn.dcn_core_forward_host(p, hx, ho, hm, hout, dx, do, dm, dout, stream=s)  # warm-up
    s.synchronize()
    hout.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dcn.dcn_core_forward_host(p, hx, ho, hm, hout, dx, do, dm, dout,
                                  stream=torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    ref = gpu_forward(p, hx.cuda(), ho.cuda(), hm.cuda())
    torch.cuda.synchronize()
    assert torch.equal(hout, ref.cpu())
    del g


# --- full-size workloads, sampled ----------------------------------------------------

def sampled_units(wl, imgs, per_img=3000):
    """Units u = ((n*Ho+ho)*Wo+wo)*G+g of a few images: random ones plus every
    unit of the first and last output rows and columns (the image border)."""
    Ho, Wo, G = wl.Ho, wl.Wo, wl.G
    units = []
    for j, _ in enumerate(imgs):
        base = j * Ho * Wo * G
        r = RNG.integers(0, Ho * Wo * G, size=per_img)
        border = [((ho * Wo + wo) * G + g) for ho in (0, Ho - 1) for wo in range(Wo) for g in range(G)]
        border += [((ho * Wo + wo) * G + g) for ho in range(Ho) for wo in (0, Wo - 1) for g in range(G)]
        units.append(base + np.unique(np.concatenate([r, np.array(border)])))
    return np.concatenate(units)


FULL = [n for n, w in WORKLOADS.items() if not w.backward]


@pytest.mark.parametrize("path", ["auto", "direct"])
@pytest.mark.parametrize("name", FULL)
def test_full_size_workload_sampled(gen_mod, oracle_mod, name, path):
    wl = WORKLOADS[name]
    d = gen_mod.make_inputs(wl)
    p = dcn.problem_for(wl)
    xd, od, md = to_dev(d["x"], wl.dtype), to_dev(d["offset"], wl.dtype), to_dev(d["mask"], wl.dtype)
    with forward_path(path):
        out = gpu_forward(p, xd, od, md)
    torch.cuda.synchronize()
    imgs = sorted({0, wl.N // 2, wl.N - 1})
    units = sampled_units(wl, imgs)
    xs, os_, ms = (f64(t[imgs]) for t in (xd, od, md))
    ref = oracle_mod.forward_units(xs, os_, ms, units, **problem_kwargs(p))
    got = f64(out[imgs]).reshape(-1, wl.Cg)[units]
    assert_fwd(got, ref, xs, wl.dtype, name)
    # the whole output is finite and, for bf16, every value is a rounded fp32
    assert torch.isfinite(out).all()


@pytest.mark.parametrize("K,Cg,dtype", [(3, 16, "f32"), (5, 16, "f32"), (3, 8, "bf16")])
def test_bounded_wait_expiry_is_reported_and_recoverable(K, Cg, dtype):
    """Failure detection without a GPU fault: with the test knob the first TMA
    box of every CTA never arrives, the bounded mbarrier waits give up (about a
    second), the kernel sets the device error word and returns;
    dcn_core_sync_status reports DCN_ERR_TIMEOUT and clears the word, and the
    next call works normally.  K = 5 runs the wide-window kernel, whose
    consumers also have staging copies in flight when they give up; 8 bf16
    channels run the 3x3 tiled kernel's 16-byte-group form (the timeout also
    shows that such a problem takes the tiled path)."""
    p, x, off, mask = random_case(2, 23, 29, 3, Cg, K=K, dtype=dtype)
    xd, od, md = to_dev(x, dtype), to_dev(off, dtype), to_dev(mask, dtype)
    with forward_path("auto"):
        ref = gpu_forward(p, xd, od, md)
        dcn.dcn_core_sync_status()
        old = os.environ.get("DCN_CORE_TEST_STALL")
        os.environ["DCN_CORE_TEST_STALL"] = "1"
        try:
            gpu_forward(p, xd, od, md)
            with pytest.raises(dcn.DcnError) as e:
                dcn.dcn_core_sync_status()
            assert e.value.status == dcn.DCN_ERR_TIMEOUT
        finally:
            if old is None:
                os.environ.pop("DCN_CORE_TEST_STALL", None)
            else:
                os.environ["DCN_CORE_TEST_STALL"] = old
        out = gpu_forward(p, xd, od, md)
        dcn.dcn_core_sync_status()
    assert torch.equal(out, ref)
