"""CPU oracle for the DCNv3 / DCNv4 core operator (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and it
shares no code with ``dcn_oracle.c``.

Every function here is argument marshalling around the plain, single-threaded
C loops of ``dcn_oracle.c`` (double accumulation); see that file for what is
computed and for the page passages each step follows.  Inputs are converted
to float64 exactly (fp32 and bf16 values are exactly representable).

Parity status: every function is pinned by the closed forms, invariants and
brute-force checks in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dcn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdcnoracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc.  -ffp-contract=off keeps every fp32
    multiply and add of the sampling location separately rounded."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        ci, cd, i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        shape = [ci] * 9 + [cd, ci, ci, ci, ci, ci, ci]
        lib.oracle_output_extent.argtypes = [ci] * 5
        lib.oracle_output_extent.restype = ci
        lib.oracle_forward.argtypes = [dp] * 4 + shape
        lib.oracle_forward.restype = ci
        lib.oracle_forward_units.argtypes = [dp] * 3 + [i64p, i64, dp] + shape
        lib.oracle_forward_units.restype = ci
        lib.oracle_backward.argtypes = [dp] * 7 + shape
        lib.oracle_backward.restype = ci
        lib.oracle_backward_units.argtypes = [dp] * 4 + [i64p, i64, dp, dp] + shape
        lib.oracle_backward_units.restype = ci
        _lib = lib
    return _lib


def _d(a) -> np.ndarray:
    """Exact float64 copy of a host array (numpy or CPU torch tensor)."""
    if hasattr(a, "detach"):  # torch tensor: bf16 has no numpy dtype, widen via fp32
        import torch
        a = a.detach().to("cpu", torch.float32).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def output_extent(n_in: int, K: int, stride: int, pad: int, dil: int) -> int:
    return int(_load().oracle_output_extent(n_in, K, stride, pad, dil))


def output_hw(H, W, K, stride, pad, dil, stride_w=None, pad_w=None, dil_w=None):
    return (output_extent(H, K, stride, pad, dil),
            output_extent(W, K, stride if stride_w is None else stride_w,
                          pad if pad_w is None else pad_w, dil if dil_w is None else dil_w))


def taps(K: int, remove_center=0) -> int:
    """Taps per (pixel, group): the K x K window, less its centre with
    remove_center (DCNv4 speed-up write-up (pnsm.cn), section 3.3)."""
    return K * K - (1 if remove_center else 0)


def _shape_args(N, H, W, G, Cg, K, stride, pad, dil, offset_scale, softmax, fd, remove_center,
                stride_w=None, pad_w=None, dil_w=None):
    """Arguments of the C entry points: stride, pad and dil are the height
    axis's; the width axis takes the *_w values, or the same ones when None."""
    return (int(N), int(H), int(W), int(G), int(Cg), int(K), int(stride), int(pad),
            int(dil), float(offset_scale), int(softmax), int(bool(fd)),
            int(bool(remove_center)), int(stride if stride_w is None else stride_w),
            int(pad if pad_w is None else pad_w), int(dil if dil_w is None else dil_w))


def forward(x, offset, mask, *, G, K=3, stride=1, pad=1, dil=1, offset_scale=1.0,
            softmax=1, fd=False, remove_center=0, stride_w=None, pad_w=None,
            dil_w=None) -> np.ndarray:
    """Forward of the whole problem.  x: (N,H,W,G*Cg), offset: (N,Ho,Wo,G*T*2),
    mask: (N,Ho,Wo,G*T) with T = taps(K, remove_center).  Returns float64
    (N,Ho,Wo,G*Cg)."""
    x, offset, mask = _d(x), _d(offset), _d(mask)
    N, H, W, C = x.shape
    Cg = C // G
    Ho, Wo = output_hw(H, W, K, stride, pad, dil, stride_w, pad_w, dil_w)
    out = np.zeros((N, Ho, Wo, C), dtype=np.float64)
    if out.size == 0:
        return out
    T = taps(K, remove_center)
    assert offset.shape == (N, Ho, Wo, G * T * 2), offset.shape
    assert mask.shape == (N, Ho, Wo, G * T), mask.shape
    rc = _load().oracle_forward(_p(x), _p(offset), _p(mask), _p(out),
                                *_shape_args(N, H, W, G, Cg, K, stride, pad, dil,
                                             offset_scale, softmax, fd, remove_center,
                                             stride_w, pad_w, dil_w))
    assert rc == 0, rc
    return out


def forward_units(x, offset, mask, units, *, G, K=3, stride=1, pad=1, dil=1,
                  offset_scale=1.0, softmax=1, fd=False, remove_center=0, stride_w=None,
                  pad_w=None, dil_w=None) -> np.ndarray:
    """Forward outputs of selected units u = ((n*Ho+ho)*Wo+wo)*G+g only.
    Returns float64 (len(units), Cg)."""
    x, offset, mask = _d(x), _d(offset), _d(mask)
    N, H, W, C = x.shape
    Cg = C // G
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int64))
    out = np.zeros((units.size, Cg), dtype=np.float64)
    rc = _load().oracle_forward_units(
        _p(x), _p(offset), _p(mask), units.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        units.size, _p(out),
        *_shape_args(N, H, W, G, Cg, K, stride, pad, dil, offset_scale, softmax, fd,
                     remove_center, stride_w, pad_w, dil_w))
    assert rc == 0, rc
    return out


def backward(x, offset, mask, grad_out, *, G, K=3, stride=1, pad=1, dil=1,
             offset_scale=1.0, softmax=1, fd=False, remove_center=0, stride_w=None, pad_w=None,
             dil_w=None):
    """Returns float64 (grad_input, grad_offset, grad_mask); grad_mask is the
    gradient with respect to the logits when softmax=1."""
    x, offset, mask, grad_out = _d(x), _d(offset), _d(mask), _d(grad_out)
    N, H, W, C = x.shape
    Cg = C // G
    gx = np.zeros_like(x)
    goff = np.zeros_like(offset)
    gm = np.zeros_like(mask)
    rc = _load().oracle_backward(_p(x), _p(offset), _p(mask), _p(grad_out), _p(gx), _p(goff),
                                 _p(gm), *_shape_args(N, H, W, G, Cg, K, stride, pad, dil,
                                                      offset_scale, softmax, fd, remove_center,
                                                      stride_w, pad_w, dil_w))
    assert rc == 0, rc
    return gx, goff, gm


def backward_units(x, offset, mask, grad_out, units, *, G, K=3, stride=1, pad=1, dil=1,
                   offset_scale=1.0, softmax=1, fd=False, remove_center=0, stride_w=None,
                   pad_w=None, dil_w=None):
    """Offset and mask gradients of selected units.  Returns float64
    (goff (len, T*2), gmask (len, T)), T = taps(K, remove_center)."""
    x, offset, mask, grad_out = _d(x), _d(offset), _d(mask), _d(grad_out)
    N, H, W, C = x.shape
    Cg = C // G
    KK = taps(K, remove_center)
    units = np.ascontiguousarray(np.asarray(units, dtype=np.int64))
    goff = np.zeros((units.size, KK * 2), dtype=np.float64)
    gm = np.zeros((units.size, KK), dtype=np.float64)
    rc = _load().oracle_backward_units(
        _p(x), _p(offset), _p(mask), _p(grad_out),
        units.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), units.size, _p(goff), _p(gm),
        *_shape_args(N, H, W, G, Cg, K, stride, pad, dil, offset_scale, softmax, fd,
                     remove_center, stride_w, pad_w, dil_w))
    assert rc == 0, rc
    return goff, gm


def projection(query, weight, bias=None, *, G, K=3, remove_center=0):
    """Offset and mask projection of the DCNv3 block (InternImage-L DCNv3
    explainer (wmrh.cn), section 二 steps 1-3: linear layers on the query
    features predict each group's and tap's offset pair and mask logit).  With
    the two layers' weights stacked row-wise:
        P[pixel, j] = sum_c query[pixel, c] * weight[j, c] + bias[j]
    in float64 (a matrix product).  query (..., Cq), weight (G*T*3, Cq), bias
    (G*T*3) or None.  Returns (offset (..., G*T*2), mask (..., G*T)): the first
    G*T*2 columns in the order (g, k, {dx, dy}), then the G*T mask logits."""
    T = taps(K, remove_center)
    q = _d(query)
    w = _d(weight)
    assert w.shape == (G * T * 3, q.shape[-1]), (w.shape, q.shape)
    P = q.reshape(-1, q.shape[-1]) @ w.T
    if bias is not None:
        P = P + _d(bias)[None, :]
    P = P.reshape(q.shape[:-1] + (G * T * 3,))
    return P[..., :G * T * 2], P[..., G * T * 2:]


def linear(x, weight, bias=None):
    """A linear layer in float64: x (..., K) @ weight (Nout, K)^T + bias (Nout).
    The DCNv3 block's input_proj and output_proj around the core operator
    (InternImage-L DCNv3 explainer (wmrh.cn), section 二)."""
    a = _d(x)
    w = _d(weight)
    assert w.shape[1] == a.shape[-1], (w.shape, a.shape)
    y = a.reshape(-1, a.shape[-1]) @ w.T
    if bias is not None:
        y = y + _d(bias)[None, :]
    return y.reshape(a.shape[:-1] + (w.shape[0],))


def guide(x, dw_weight, dw_bias, ln_gamma, ln_beta, ln_eps, pixels=None):
    """Guide features of the DCNv3 block's offset / mask branch (InternImage-L
    DCNv3 explainer (wmrh.cn), section 二 step 1: the input passes a depthwise
    convolution, LayerNorm and GELU before the linear layers of steps 2-3), in
    float64:
        conv[n, y, x, c] = dw_bias[c] + sum_{a, b < 3} dw_weight[a, b, c] * x[n, y+a-1, x+b-1, c]
                           (zero outside the image: a 3x3 window, stride 1, padding 1)
        z = (conv - mean_c conv) / sqrt(var_c conv + ln_eps) * ln_gamma + ln_beta
            (mean and biased variance over the C channels of one pixel)
        out = z * (1 + erf(z / sqrt(2))) / 2       (GELU, exact form)
    x (N, H, W, C); dw_weight (3, 3, C); dw_bias, ln_gamma, ln_beta (C,).
    Returns (N, H, W, C), or, with `pixels` (flat indices n*H*W + y*W + x),
    the rows of those pixels only, (len(pixels), C)."""
    import math
    a = _d(x)
    N, H, W, C = a.shape
    w = _d(dw_weight).reshape(3, 3, C)
    xp = np.zeros((N, H + 2, W + 2, C))
    xp[:, 1:H + 1, 1:W + 1, :] = a
    if pixels is None:
        pix = np.arange(N * H * W)
    else:
        pix = np.asarray(pixels, dtype=np.int64)
    n, rem = pix // (H * W), pix % (H * W)
    y, xx = rem // W, rem % W
    conv = np.tile(_d(dw_bias).reshape(1, C), (len(pix), 1))
    for ta in range(3):
        for tb in range(3):
            # padded row y + ta is input row y + ta - 1
            conv = conv + w[ta, tb][None, :] * xp[n, y + ta, xx + tb, :]
    mean = conv.mean(axis=1, keepdims=True)
    var = ((conv - mean) ** 2).mean(axis=1, keepdims=True)
    z = (conv - mean) / np.sqrt(var + float(ln_eps)) * _d(ln_gamma)[None, :] + _d(ln_beta)[None, :]
    erf = np.vectorize(math.erf, otypes=[np.float64])
    out = z * (1.0 + erf(z / math.sqrt(2.0))) / 2.0
    return out.reshape(N, H, W, C) if pixels is None else out


def workload_kwargs(wl) -> dict:
    """Keyword arguments of forward()/backward() for a gen.Workload."""
    return dict(G=wl.G, K=wl.K, stride=wl.stride, pad=wl.pad, dil=wl.dilation,
                offset_scale=wl.offset_scale, softmax=wl.softmax,
                remove_center=getattr(wl, "remove_center", 0))
