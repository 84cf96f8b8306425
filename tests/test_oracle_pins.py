"""Pins of the CPU oracle to facts the pages and the mathematics fix.

No page prints a worked numeric example, so every pin is a closed form, an
invariant or a brute-force recomputation through an independent library
routine (torch.nn.functional.grid_sample, which the pure-PyTorch path of the
InternImage-L DCNv3 explainer (wmrh.cn, sections 二 and 五) names as the
sampling step).  They are chosen so that a dropped term, a swapped (dx, dy),
a transposed tap index, a wrong sign or a wrong stride/dilation in the oracle
fails at least one of them.
"""
import numpy as np
import pytest
import torch

from gen.workloads import WORKLOADS

RNG = np.random.default_rng(12345)


def rand(*shape, lo=-1.0, hi=1.0):
    return RNG.uniform(lo, hi, size=shape).astype(np.float32).astype(np.float64)


def one_hot_mask(N, Ho, Wo, G, K, tap, softmax):
    KK = K * K
    if softmax:
        m = np.full((N, Ho, Wo, G, KK), -40.0)
        m[..., tap] = 40.0
    else:
        m = np.zeros((N, Ho, Wo, G, KK))
        m[..., tap] = 1.0
    return m.reshape(N, Ho, Wo, G * KK)


# --- output extent ---------------------------------------------------------------

def test_output_extent_same_size_and_stride2(oracle_mod):
    # Same spatial size at kernel 3 / stride 1 / pad 1 (DCNv3 extension build
    # guide (trdm.cn), section 2.3); 256 -> 128 at stride 2.
    assert oracle_mod.output_extent(14, 3, 1, 1, 1) == 14
    assert oracle_mod.output_extent(96, 3, 1, 1, 1) == 96
    assert oracle_mod.output_extent(256, 3, 2, 1, 1) == 128
    assert oracle_mod.output_extent(5, 5, 1, 2, 1) == 5
    assert oracle_mod.output_extent(7, 3, 1, 0, 2) == 3
    assert oracle_mod.output_extent(2, 5, 1, 0, 1) == 0
    for wl in WORKLOADS.values():
        assert oracle_mod.output_hw(wl.H, wl.W, wl.K, wl.stride, wl.pad, wl.dilation) == \
            (wl.Ho, wl.Wo), wl.name


# --- P1 identity -----------------------------------------------------------------

@pytest.mark.parametrize("K", [1, 3, 5])
@pytest.mark.parametrize("softmax", [0, 1])
def test_identity(oracle_mod, K, softmax):
    N, H, W, G, Cg = 2, 6, 7, 3, 5
    x = rand(N, H, W, G * Cg)
    off = np.zeros((N, H, W, G * K * K * 2))
    centre = (K // 2) * K + K // 2
    mask = one_hot_mask(N, H, W, G, K, centre, softmax)
    out = oracle_mod.forward(x, off, mask, G=G, K=K, pad=K // 2, softmax=softmax,
                             offset_scale=2.0)
    if softmax:
        np.testing.assert_allclose(out, x, rtol=0, atol=1e-15)
    else:
        assert np.array_equal(out, x)


# --- P2 zero offsets + uniform mask = zero-padded box filter ----------------------

def test_zero_init_is_box_filter(oracle_mod):
    # The explainer (wmrh.cn, section 二, "details") notes that with zero-initialised
    # offset and mask projections the block starts out as a plain 3x3 convolution:
    # zero offsets and zero logits give m = 1/9, i.e. a zero-padded 3x3 mean.
    N, H, W, G, Cg = 2, 5, 6, 2, 3
    x = rand(N, H, W, G * Cg)
    off = np.zeros((N, H, W, G * 18))
    logits = np.zeros((N, H, W, G * 9))
    out = oracle_mod.forward(x, off, logits, G=G, softmax=1, offset_scale=2.0)
    xp = np.pad(x, ((0, 0), (1, 1), (1, 1), (0, 0)))
    box = sum(xp[:, i:i + H, j:j + W, :] for i in range(3) for j in range(3)) / 9.0
    np.testing.assert_allclose(out, box, rtol=0, atol=1e-14)


@pytest.mark.parametrize("K", [3, 5])
def test_zero_init_without_centre_is_ring_mean(oracle_mod, K):
    # With remove_center (DCNv4 speed-up write-up (pnsm.cn), section 3.3) the
    # centre point is not sampled: zero offsets and equal logits average the
    # K*K - 1 other window positions, zero-padded.
    N, H, W, G, Cg = 2, 6, 5, 2, 3
    r = K // 2
    x = rand(N, H, W, G * Cg)
    T = K * K - 1
    off = np.zeros((N, H, W, G * T * 2))
    logits = np.full((N, H, W, G * T), 0.3)
    out = oracle_mod.forward(x, off, logits, G=G, K=K, pad=r, softmax=1, offset_scale=2.0,
                             remove_center=1)
    xp = np.pad(x, ((0, 0), (r, r), (r, r), (0, 0)))
    ring = sum(xp[:, i:i + H, j:j + W, :] for i in range(K) for j in range(K)
               if (i, j) != (r, r)) / T
    np.testing.assert_allclose(out, ring, rtol=0, atol=1e-14)
    # the raw-mask variant with weight 1 per tap: the ring sum
    out4 = oracle_mod.forward(x, off, np.ones_like(logits), G=G, K=K, pad=r, softmax=0,
                              offset_scale=2.0, remove_center=1)
    np.testing.assert_allclose(out4, ring * T, rtol=0, atol=1e-13)


@pytest.mark.parametrize("softmax", [0, 1])
def test_remove_center_is_full_window_with_centre_weight_zero(oracle_mod, softmax):
    # Dropping the centre tap equals keeping it with a zero weight: a raw
    # mask of 0 (DCNv4) or a logit of -inf (DCNv3 softmax), whatever its offset.
    N, H, W, G, Cg, K = 2, 7, 6, 3, 4, 3
    c = (K * K) // 2
    x = rand(N, H, W, G * Cg)
    off8 = rand(N, H, W, G, K * K - 1, 2, lo=-2.5, hi=2.5)
    m8 = rand(N, H, W, G, K * K - 1, lo=-2, hi=2)
    gout = rand(N, H, W, G * Cg)
    off9 = np.insert(off8, c, rand(N, H, W, G, 2, lo=-3, hi=3), axis=4)
    m9 = np.insert(m8, c, -np.inf if softmax else 0.0, axis=4)
    kw = dict(G=G, K=K, offset_scale=2.0, softmax=softmax)
    a8 = (off8.reshape(N, H, W, -1), m8.reshape(N, H, W, -1))
    a9 = (off9.reshape(N, H, W, -1), m9.reshape(N, H, W, -1))
    f8 = oracle_mod.forward(x, *a8, remove_center=1, **kw)
    f9 = oracle_mod.forward(x, *a9, **kw)
    assert np.array_equal(f8, f9)
    gx8, go8, gm8 = oracle_mod.backward(x, *a8, gout, remove_center=1, **kw)
    gx9, go9, gm9 = oracle_mod.backward(x, *a9, gout, **kw)
    assert np.array_equal(gx8, gx9)
    keep = [k for k in range(K * K) if k != c]
    assert np.array_equal(go8.reshape(N, H, W, G, -1, 2), go9.reshape(N, H, W, G, -1, 2)[..., keep, :])
    assert np.array_equal(gm8.reshape(N, H, W, G, -1), gm9.reshape(N, H, W, G, -1)[..., keep])


def test_remove_center_needs_a_tap(oracle_mod):
    # K = 1 without its centre has no tap left: the oracle refuses it.
    x = np.zeros((1, 3, 3, 2))
    with pytest.raises(AssertionError):
        oracle_mod.forward(x, np.zeros((1, 3, 3, 0)), np.zeros((1, 3, 3, 0)), G=1, K=1, pad=0,
                           remove_center=1)


# --- P3 integer offsets = exact shifts ---------------------------------------------

@pytest.mark.parametrize("stride,dil,sigma", [(1, 1, 2.0), (2, 1, 1.0), (1, 2, 1.0), (2, 2, 2.0)])
@pytest.mark.parametrize("tap", [0, 2, 5, 7])
def test_integer_shift(oracle_mod, stride, dil, sigma, tap):
    N, H, W, G, Cg, K = 1, 9, 11, 2, 3, 3
    pad = dil
    Ho, Wo = oracle_mod.output_hw(H, W, K, stride, pad, dil)
    x = rand(N, H, W, G * Cg)
    u, v = 1, -2          # dx, dy: different so that swapping them is caught
    off = np.zeros((N, Ho, Wo, G, K * K, 2))
    off[..., 0] = u
    off[..., 1] = v
    off = off.reshape(N, Ho, Wo, -1)
    mask = one_hot_mask(N, Ho, Wo, G, K, tap, 0)
    out = oracle_mod.forward(x, off, mask, G=G, K=K, stride=stride, pad=pad, dil=dil,
                             offset_scale=sigma, softmax=0)
    a, b = tap // K, tap % K
    exp = np.zeros_like(out)
    for ho in range(Ho):
        for wo in range(Wo):
            y = ho * stride - pad + a * dil + int(sigma * v)
            xx = wo * stride - pad + b * dil + int(sigma * u)
            if 0 <= y < H and 0 <= xx < W:
                exp[:, ho, wo, :] = x[:, y, xx, :]
    assert np.array_equal(out, exp)


# --- P4 linearity in x -------------------------------------------------------------

def test_linearity_in_input(oracle_mod):
    N, H, W, G, Cg = 2, 7, 6, 2, 4
    x1, x2 = rand(N, H, W, G * Cg), rand(N, H, W, G * Cg)
    off = rand(N, H, W, G * 18, lo=-3, hi=3)
    mask = rand(N, H, W, G * 9, lo=-2, hi=2)
    al, be = 0.37, -1.9
    kw = dict(G=G, softmax=1, offset_scale=2.0)
    lhs = oracle_mod.forward(al * x1 + be * x2, off, mask, **kw)
    rhs = al * oracle_mod.forward(x1, off, mask, **kw) + be * oracle_mod.forward(x2, off, mask, **kw)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12 * np.abs(rhs).max())


# --- P5 half-pixel ------------------------------------------------------------------

def test_half_pixel_is_mean_of_neighbours(oracle_mod):
    N, H, W, G, Cg = 1, 5, 6, 1, 2
    x = rand(N, H, W, Cg)
    off = np.zeros((N, H, W, 9, 2))
    off[..., 4, 0] = 0.5           # centre tap, dx = +1/2
    off = off.reshape(N, H, W, 18)
    mask = one_hot_mask(N, H, W, 1, 3, 4, 0)
    out = oracle_mod.forward(x, off, mask, G=1, softmax=0, offset_scale=1.0)
    for ho in range(H):
        for wo in range(W - 1):
            np.testing.assert_allclose(out[0, ho, wo], 0.5 * (x[0, ho, wo] + x[0, ho, wo + 1]),
                                       rtol=0, atol=1e-15)
        # last column: the right neighbour is outside, so only half of x remains
        np.testing.assert_allclose(out[0, ho, W - 1], 0.5 * x[0, ho, W - 1], rtol=0, atol=1e-15)


# --- P6 brute force through torch grid_sample -------------------------------------

@pytest.mark.parametrize("softmax,stride,K,remove_center",
                         [(1, 1, 3, 0), (0, 1, 3, 0), (1, 2, 3, 0), (1, 1, 3, 1), (0, 2, 3, 1),
                          (1, 1, 5, 1)])
def test_grid_sample_brute_force(oracle_mod, softmax, stride, K, remove_center):
    N, H, W, G, Cg = 2, 7, 8, 2, 3
    pad, dil, sigma = K // 2, 1, 2.0
    # The window positions, row-major; remove_center (DCNv4 speed-up write-up
    # (pnsm.cn), section 3.3) leaves the centre out of the list.
    window = [(a, b) for a in range(K) for b in range(K)
              if not (remove_center and a == K // 2 and b == K // 2)]
    T = len(window)
    Ho, Wo = oracle_mod.output_hw(H, W, K, stride, pad, dil)
    x = rand(N, H, W, G * Cg)
    off = rand(N, Ho, Wo, G * T * 2, lo=-2.5, hi=2.5)   # many samples cross the border
    mask = rand(N, Ho, Wo, G * T, lo=-2, hi=2)
    got = oracle_mod.forward(x, off, mask, G=G, K=K, stride=stride, pad=pad, dil=dil,
                             offset_scale=sigma, softmax=softmax, fd=True,
                             remove_center=remove_center)
    xt = torch.from_numpy(x).reshape(N, H, W, G, Cg)
    o = torch.from_numpy(off).reshape(N, Ho, Wo, G, T, 2)
    m = torch.from_numpy(mask).reshape(N, Ho, Wo, G, T)
    if softmax:
        m = torch.softmax(m, dim=-1)
    ref = torch.zeros(N, Ho, Wo, G, Cg, dtype=torch.float64)
    hh = torch.arange(Ho, dtype=torch.float64).view(Ho, 1)
    ww = torch.arange(Wo, dtype=torch.float64).view(1, Wo)
    for g in range(G):
        img = xt[:, :, :, g, :].permute(0, 3, 1, 2)          # (N, Cg, H, W)
        for k, (a, b) in enumerate(window):
            Y = hh * stride - pad + a * dil + sigma * o[:, :, :, g, k, 1]
            X = ww * stride - pad + b * dil + sigma * o[:, :, :, g, k, 0]
            grid = torch.stack([(2 * X + 1) / W - 1, (2 * Y + 1) / H - 1], dim=-1)
            s = torch.nn.functional.grid_sample(img, grid, mode="bilinear",
                                                padding_mode="zeros", align_corners=False)
            ref[:, :, :, g, :] += m[:, :, :, g, k, None] * s.permute(0, 2, 3, 1)
    np.testing.assert_allclose(got, ref.reshape(N, Ho, Wo, G * Cg).numpy(), rtol=0, atol=1e-12)


# --- P7 softmax weights sum to one ------------------------------------------------

def test_softmax_mask_preserves_constants(oracle_mod):
    N, H, W, G, Cg = 1, 8, 9, 3, 2
    c = 1.7
    x = np.full((N, H, W, G * Cg), c)
    off = rand(N, H, W, G * 18, lo=-0.45, hi=0.45)
    mask = rand(N, H, W, G * 9, lo=-3, hi=3)
    out = oracle_mod.forward(x, off, mask, G=G, softmax=1, offset_scale=1.0)
    np.testing.assert_allclose(out[:, 2:H - 2, 2:W - 2, :], c, rtol=0, atol=1e-14)
    # DCNv4 (no softmax): the same constant image gives c * sum_k m_k
    out4 = oracle_mod.forward(x, off, mask, G=G, softmax=0, offset_scale=1.0)
    msum = mask.reshape(N, H, W, G, 9).sum(-1)
    got4 = out4.reshape(N, H, W, G, Cg)[:, 2:H - 2, 2:W - 2]
    np.testing.assert_allclose(got4, np.broadcast_to(c * msum[:, 2:H - 2, 2:W - 2, :, None],
                                                     got4.shape), rtol=0, atol=1e-13)


# --- P8 stride consistency ---------------------------------------------------------

def test_stride2_is_subsampled_stride1(oracle_mod):
    N, H, W, G, Cg = 2, 10, 12, 2, 4
    x = rand(N, H, W, G * Cg)
    off1 = rand(N, H, W, G * 18, lo=-2, hi=2)
    m1 = rand(N, H, W, G * 9, lo=-2, hi=2)
    for softmax in (0, 1):
        o1 = oracle_mod.forward(x, off1, m1, G=G, stride=1, softmax=softmax, offset_scale=2.0)
        o2 = oracle_mod.forward(x, off1[:, ::2, ::2], m1[:, ::2, ::2], G=G, stride=2,
                                softmax=softmax, offset_scale=2.0)
        assert o2.shape == (N, 5, 6, G * Cg)
        assert np.array_equal(o2, o1[:, ::2, ::2])


# --- P9 group independence ----------------------------------------------------------

def test_groups_are_independent(oracle_mod):
    N, H, W, G, Cg = 1, 6, 6, 3, 4
    x = rand(N, H, W, G * Cg)
    off = rand(N, H, W, G * 18, lo=-2, hi=2)
    m = rand(N, H, W, G * 9)
    base = oracle_mod.forward(x, off, m, G=G)
    x2, off2, m2 = x.copy(), off.copy(), m.copy()
    x2[..., Cg:2 * Cg] += 1.0
    off2[..., 18:36] += 0.7
    m2[..., 9:18] -= 0.3
    for args in [(x2, off, m), (x, off2, m), (x, off, m2)]:
        out = oracle_mod.forward(*args, G=G)
        assert np.array_equal(out[..., :Cg], base[..., :Cg])
        assert np.array_equal(out[..., 2 * Cg:], base[..., 2 * Cg:])
        assert not np.array_equal(out[..., Cg:2 * Cg], base[..., Cg:2 * Cg])


# --- P10 finite differences ---------------------------------------------------------

def kink_free_offsets(N, Ho, Wo, G, T, sigma):
    """Offsets of T taps whose sample coordinates have fractional parts in
    [0.05, 0.95] (grid points are integers, so the offset alone sets the
    fraction), so that no finite-difference stencil crosses a floor()
    boundary."""
    shift = RNG.integers(-2, 3, size=(N, Ho, Wo, G, T, 2)) + \
        RNG.uniform(0.05, 0.95, size=(N, Ho, Wo, G, T, 2))
    return (shift / sigma).reshape(N, Ho, Wo, -1)


@pytest.mark.parametrize("softmax,stride,remove_center",
                         [(1, 1, 0), (0, 1, 0), (1, 2, 0), (1, 1, 1), (0, 2, 1)])
def test_backward_matches_finite_differences(oracle_mod, softmax, stride, remove_center):
    N, H, W, G, Cg, K, pad, dil, sigma = 1, 5, 5, 2, 4, 3, 1, 1, 2.0
    T = K * K - remove_center
    Ho, Wo = oracle_mod.output_hw(H, W, K, stride, pad, dil)
    x = rand(N, H, W, G * Cg)
    off = kink_free_offsets(N, Ho, Wo, G, T, sigma)
    m = rand(N, Ho, Wo, G * T, lo=-1.5, hi=1.5)
    gout = rand(N, Ho, Wo, G * Cg)
    kw = dict(G=G, K=K, stride=stride, pad=pad, dil=dil, offset_scale=sigma,
              softmax=softmax, fd=True, remove_center=remove_center)
    gx, goff, gm = oracle_mod.backward(x, off, m, gout, **kw)

    def L(xx, oo, mm):
        return float((oracle_mod.forward(xx, oo, mm, **kw) * gout).sum())

    h = 1e-4
    for arr, grad, which in ((x, gx, 0), (off, goff, 1), (m, gm, 2)):
        flat = arr.reshape(-1)
        idxs = RNG.choice(flat.size, size=min(flat.size, 60), replace=False)
        fd = np.zeros(idxs.size)
        for j, i in enumerate(idxs):
            p, q = flat.copy(), flat.copy()
            p[i] += h
            q[i] -= h
            args_p = [x, off, m]
            args_q = [x, off, m]
            args_p[which] = p.reshape(arr.shape)
            args_q[which] = q.reshape(arr.shape)
            fd[j] = (L(*args_p) - L(*args_q)) / (2 * h)
        an = grad.reshape(-1)[idxs]
        np.testing.assert_allclose(an, fd, rtol=0, atol=1e-7 * max(1.0, np.abs(fd).max()))


# --- P11 adjoint identity ---------------------------------------------------------

def test_adjoint_identity(oracle_mod):
    N, H, W, G, Cg = 2, 9, 8, 3, 4
    v = rand(N, H, W, G * Cg)
    off = rand(N, H, W, G * 18, lo=-3, hi=3)
    m = rand(N, H, W, G * 9, lo=-2, hi=2)
    gout = rand(N, H, W, G * Cg)
    kw = dict(G=G, softmax=1, offset_scale=2.0)
    lhs = float((gout * oracle_mod.forward(v, off, m, **kw)).sum())
    gx, _, _ = oracle_mod.backward(v, off, m, gout, **kw)
    rhs = float((gx * v).sum())
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)


# --- P12 softmax Jacobian rows sum to zero ------------------------------------------

def test_softmax_logit_gradients_sum_to_zero(oracle_mod):
    N, H, W, G, Cg = 1, 6, 7, 4, 2
    x = rand(N, H, W, G * Cg)
    off = rand(N, H, W, G * 18, lo=-3, hi=3)
    m = rand(N, H, W, G * 9, lo=-2, hi=2)
    gout = rand(N, H, W, G * Cg)
    _, _, gl = oracle_mod.backward(x, off, m, gout, G=G, softmax=1, offset_scale=2.0)
    s = gl.reshape(N, H, W, G, 9).sum(-1)
    assert np.abs(s).max() <= 1e-12 * np.abs(gl).max()


# --- sampled entry points agree with the full ones -----------------------------------

def test_unit_entry_points_match_full(oracle_mod):
    N, H, W, G, Cg = 2, 6, 5, 3, 4
    x = rand(N, H, W, G * Cg)
    off = rand(N, H, W, G * 18, lo=-3, hi=3)
    m = rand(N, H, W, G * 9, lo=-2, hi=2)
    gout = rand(N, H, W, G * Cg)
    kw = dict(G=G, softmax=1, offset_scale=2.0)
    full = oracle_mod.forward(x, off, m, **kw).reshape(-1, Cg)
    units = np.array([0, 7, 31, N * H * W * G - 1])
    assert np.array_equal(oracle_mod.forward_units(x, off, m, units, **kw), full[units])
    _, goff, gm = oracle_mod.backward(x, off, m, gout, **kw)
    bo, bm = oracle_mod.backward_units(x, off, m, gout, units, **kw)
    assert np.array_equal(bo, goff.reshape(-1, 18)[units])
    assert np.array_equal(bm, gm.reshape(-1, 9)[units])


# --- non-finite and far samples -------------------------------------------------------

def test_far_and_nonfinite_samples_contribute_zero(oracle_mod):
    N, H, W, G, Cg = 1, 4, 4, 1, 2
    x = rand(N, H, W, Cg)
    off = np.zeros((N, H, W, 18))
    off[..., 0::2] = 1e6
    mask = one_hot_mask(N, H, W, 1, 3, 4, 0)
    assert np.array_equal(oracle_mod.forward(x, off, mask, G=1, softmax=0), np.zeros_like(x))
    off[..., 0::2] = np.nan
    assert np.array_equal(oracle_mod.forward(x, off, mask, G=1, softmax=0), np.zeros_like(x))
    off[..., 0::2] = -np.inf
    assert np.array_equal(oracle_mod.forward(x, off, mask, G=1, softmax=0), np.zeros_like(x))


# --- offset / mask projection -------------------------------------------------------

def test_projection_matches_explicit_sums(oracle_mod):
    # the stacked linear layers written out as loops, on a tiny case
    G, K, Cq = 2, 3, 5
    q = rand(2, 3, Cq)
    w = rand(G * 9 * 3, Cq)
    b = rand(G * 9 * 3)
    off, msk = oracle_mod.projection(q, w, b, G=G, K=K)
    for i in range(2):
        for j in range(3):
            for col in range(G * 27):
                v = b[col] + sum(q[i, j, c] * w[col, c] for c in range(Cq))
                got = off[i, j, col] if col < G * 18 else msk[i, j, col - G * 18]
                assert abs(got - v) <= 1e-14


def test_projection_identity_and_bias(oracle_mod):
    # identity weight: the offsets and mask are the query's columns, split at G*T*2;
    # zero weight: the bias everywhere
    G, K, rc = 1, 3, 1
    T = 8
    q = rand(4, T * 3)
    off, msk = oracle_mod.projection(q, np.eye(T * 3), None, G=G, K=K, remove_center=rc)
    assert np.array_equal(off, q[:, :T * 2]) and np.array_equal(msk, q[:, T * 2:])
    b = rand(T * 3)
    off, msk = oracle_mod.projection(q, np.zeros((T * 3, T * 3)), b, G=G, K=K, remove_center=rc)
    assert np.array_equal(off, np.broadcast_to(b[:T * 2], off.shape))
    assert np.array_equal(msk, np.broadcast_to(b[T * 2:], msk.shape))


def test_linear_matches_explicit_sums(oracle_mod):
    x = rand(3, 2, 4)
    w = rand(5, 4)
    b = rand(5)
    y = oracle_mod.linear(x, w, b)
    for idx in np.ndindex(3, 2):
        for j in range(5):
            assert abs(y[idx + (j,)] - (b[j] + sum(x[idx + (c,)] * w[j, c] for c in range(4)))) <= 1e-14
    assert np.array_equal(oracle_mod.linear(x, np.eye(4)), x)


# --- guide features: depthwise 3x3 + LayerNorm + GELU --------------------------------

def guide_inputs(N, H, W, C):
    return (rand(N, H, W, C), rand(3, 3, C), rand(C), rand(C, lo=0.5, hi=1.5), rand(C))


@pytest.mark.parametrize("shape", [(2, 5, 7, 8), (1, 1, 1, 4), (1, 3, 9, 12), (2, 4, 4, 1)])
def test_guide_matches_torch_library_ops(oracle_mod, shape):
    """The oracle's loops against torch's own depthwise conv2d (groups = C),
    layer_norm and exact GELU, all in float64 on the CPU."""
    import torch.nn.functional as F
    N, H, W, C = shape
    x, w, b, g, be = guide_inputs(N, H, W, C)
    eps = 1e-6
    got = oracle_mod.guide(x, w, b, g, be, eps)
    t = torch.from_numpy(x).permute(0, 3, 1, 2)                       # NCHW
    wt = torch.from_numpy(w).permute(2, 0, 1).unsqueeze(1).contiguous()  # (C, 1, 3, 3)
    conv = F.conv2d(t, wt, torch.from_numpy(b), stride=1, padding=1, groups=C)
    z = F.layer_norm(conv.permute(0, 2, 3, 1), (C,), torch.from_numpy(g), torch.from_numpy(be), eps)
    ref = F.gelu(z, approximate="none").numpy()
    assert np.abs(got - ref).max() <= 1e-12
    # the sampled form returns the same rows
    pix = RNG.integers(0, N * H * W, size=5)
    assert np.array_equal(oracle_mod.guide(x, w, b, g, be, eps, pixels=pix),
                          got.reshape(-1, C)[pix])


def test_guide_two_channel_closed_form(oracle_mod):
    """Two channels with different values normalise to -1 and +1 (exactly, up
    to eps), so with gamma = 1, beta = 0 the outputs are GELU(-1) = -Phi(-1)
    and GELU(1) = Phi(1), Phi the standard normal CDF.  A centre-only kernel
    passes the input through the convolution; the bias adds per channel."""
    x = np.zeros((1, 3, 3, 2))
    x[0, 1, 1] = [0.25, 2.0]
    w = np.zeros((3, 3, 2))
    w[1, 1] = 1.0
    out = oracle_mod.guide(x, w, np.array([0.5, -0.5]), np.ones(2), np.zeros(2), 0.0)
    # centre pixel: conv = (0.75, 1.5) -> z = (-1, 1)
    assert abs(out[0, 1, 1, 0] - (-0.15865525393145707)) <= 1e-15
    assert abs(out[0, 1, 1, 1] - 0.8413447460685429) <= 1e-15
    # a corner pixel sees only the bias (0.5, -0.5) -> z = (1, -1)
    assert abs(out[0, 0, 0, 0] - 0.8413447460685429) <= 1e-15
    assert abs(out[0, 0, 0, 1] - (-0.15865525393145707)) <= 1e-15


def test_guide_window_orientation(oracle_mod):
    """Weight [a, b] multiplies input pixel (y + a - 1, x + b - 1): a one-hot
    kernel shifts the image, and a shifted pixel beyond the border reads zero.
    gamma = 0 would hide the convolution, so the check goes through a
    constant-plus-channel-ramp input whose normalisation is known."""
    N, H, W, C = 1, 4, 5, 2
    base = RNG.uniform(1.0, 2.0, size=(N, H, W))
    x = np.stack([base, base + 1.0], axis=-1)          # channel 1 = channel 0 + 1
    for a in range(3):
        for b in range(3):
            w = np.zeros((3, 3, C))
            w[a, b] = 1.0
            # eps = 1e-30: the +-1 normalisation stays exact in float64, and a
            # constant (all-zero) pixel normalises to 0 instead of 0/0
            out = oracle_mod.guide(x, w, np.zeros(C), np.ones(C), np.zeros(C), 1e-30)
            for y in range(H):
                for xx in range(W):
                    yy, xs = y + a - 1, xx + b - 1
                    inside = 0 <= yy < H and 0 <= xs < W
                    # inside: conv = (v, v + 1) -> z = (-1, 1); outside: conv = (0, 0) -> z = 0,
                    # GELU(0) = 0
                    exp = (-0.15865525393145707, 0.8413447460685429) if inside else (0.0, 0.0)
                    assert np.allclose(out[0, y, xx], exp, atol=1e-15), (a, b, y, xx)


# --- separate height / width stride, padding and dilation ---------------------------

AXES = [dict(stride=1, stride_w=2, pad=1, pad_w=0, dil=1, dil_w=1),
        dict(stride=2, stride_w=1, pad=2, pad_w=1, dil=2, dil_w=1),
        dict(stride=1, stride_w=1, pad=0, pad_w=3, dil=1, dil_w=3)]


@pytest.mark.parametrize("ax", AXES)
def test_grid_sample_brute_force_separate_axes(oracle_mod, ax):
    N, H, W, G, Cg, K = 2, 9, 10, 2, 3, 3
    sigma = 2.0
    Ho, Wo = oracle_mod.output_hw(H, W, K, ax["stride"], ax["pad"], ax["dil"],
                                  ax["stride_w"], ax["pad_w"], ax["dil_w"])
    # the size rule per axis
    assert Ho == (H + 2 * ax["pad"] - ax["dil"] * (K - 1) - 1) // ax["stride"] + 1
    assert Wo == (W + 2 * ax["pad_w"] - ax["dil_w"] * (K - 1) - 1) // ax["stride_w"] + 1
    x = rand(N, H, W, G * Cg)
    off = rand(N, Ho, Wo, G * K * K * 2, lo=-2.5, hi=2.5)
    mask = rand(N, Ho, Wo, G * K * K, lo=-2, hi=2)
    got = oracle_mod.forward(x, off, mask, G=G, K=K, offset_scale=sigma, softmax=1, fd=True, **ax)
    xt = torch.from_numpy(x).reshape(N, H, W, G, Cg)
    o = torch.from_numpy(off).reshape(N, Ho, Wo, G, K * K, 2)
    m = torch.softmax(torch.from_numpy(mask).reshape(N, Ho, Wo, G, K * K), dim=-1)
    ref = torch.zeros(N, Ho, Wo, G, Cg, dtype=torch.float64)
    hh = torch.arange(Ho, dtype=torch.float64).view(Ho, 1)
    ww = torch.arange(Wo, dtype=torch.float64).view(1, Wo)
    for g in range(G):
        img = xt[:, :, :, g, :].permute(0, 3, 1, 2)
        for k in range(K * K):
            a, b = divmod(k, K)
            Y = hh * ax["stride"] - ax["pad"] + a * ax["dil"] + sigma * o[:, :, :, g, k, 1]
            X = ww * ax["stride_w"] - ax["pad_w"] + b * ax["dil_w"] + sigma * o[:, :, :, g, k, 0]
            grid = torch.stack([(2 * X + 1) / W - 1, (2 * Y + 1) / H - 1], dim=-1)
            s = torch.nn.functional.grid_sample(img, grid, mode="bilinear", padding_mode="zeros",
                                                align_corners=False)
            ref[:, :, :, g, :] += m[:, :, :, g, k, None] * s.permute(0, 2, 3, 1)
    np.testing.assert_allclose(got, ref.reshape(N, Ho, Wo, G * Cg).numpy(), rtol=0, atol=1e-12)


def test_backward_finite_differences_separate_axes(oracle_mod):
    ax = dict(stride=2, stride_w=1, pad=1, pad_w=2, dil=1, dil_w=2)
    N, H, W, G, Cg, K, sigma = 1, 6, 5, 2, 3, 3, 2.0
    Ho, Wo = oracle_mod.output_hw(H, W, K, ax["stride"], ax["pad"], ax["dil"],
                                  ax["stride_w"], ax["pad_w"], ax["dil_w"])
    x = rand(N, H, W, G * Cg)
    off = kink_free_offsets(N, Ho, Wo, G, K * K, sigma)
    m = rand(N, Ho, Wo, G * K * K, lo=-1.5, hi=1.5)
    gout = rand(N, Ho, Wo, G * Cg)
    kw = dict(G=G, K=K, offset_scale=sigma, softmax=1, fd=True, **ax)
    gx, goff, gm = oracle_mod.backward(x, off, m, gout, **kw)

    def L(xx, oo, mm):
        return float((oracle_mod.forward(xx, oo, mm, **kw) * gout).sum())

    h = 1e-4
    for arr, grad, which in ((x, gx, 0), (off, goff, 1), (m, gm, 2)):
        flat = arr.reshape(-1)
        for i in RNG.choice(flat.size, size=min(flat.size, 40), replace=False):
            args_p, args_q = [x, off, m], [x, off, m]
            pp, qq = flat.copy(), flat.copy()
            pp[i] += h
            qq[i] -= h
            args_p[which], args_q[which] = pp.reshape(arr.shape), qq.reshape(arr.shape)
            fd = (L(*args_p) - L(*args_q)) / (2 * h)
            assert abs(grad.reshape(-1)[i] - fd) <= 1e-7 * max(1.0, abs(fd))
