"""Python binding of the B200 deformable-convolution core (DCNv3 / DCNv4).

Argument marshalling only: every step of the operator runs in the CUDA
kernels of ``libdcncore.so`` behind the C ABI declared in
``include/dcn_core.h``.  The functions below carry the same names as the C
entry points.  Tensors may be given as torch tensors (their device pointer is
passed) or as raw integer addresses; streams as ``torch.cuda.Stream``, a raw
handle or None (the current torch stream).

There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DCN_CORE_LIBRARY selects another build of the library, e.g. the
# bounds-checked libdcncore_checked.so.
LIB_PATH = os.environ.get("DCN_CORE_LIBRARY") or os.path.join(_HERE, "libdcncore.so")

# DCN_CORE_ABI_VERSION of include/dcn_core.h that DcnProblem mirrors.
ABI_VERSION = 5
DCN_OK, DCN_ERR_INVALID_ARG, DCN_ERR_UNSUPPORTED, DCN_ERR_CUDA, DCN_ERR_TIMEOUT = 0, 1, 2, 3, 4
DCN_ERR_OUT_OF_BOUNDS = 5  # only from the bounds-checked build
# Scratch the allocation-free backward owns per GPU (DCN_CORE_NOALLOC_SCRATCH_BYTES).
DCN_CORE_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024
DCN_F32, DCN_BF16, DCN_F16 = 0, 1, 2
# storage-type names accepted wherever a dtype is given as a string
DTYPES = {"f32": DCN_F32, "float32": DCN_F32, "bf16": DCN_BF16, "bfloat16": DCN_BF16,
          "f16": DCN_F16, "float16": DCN_F16}

# Every entry point of include/dcn_core.h.
EXPORTED_SYMBOLS = (
    "dcn_core_output_hw",
    "dcn_core_forward",
    "dcn_core_forward_host",
    "dcn_core_backward_workspace",
    "dcn_core_backward",
    "dcn_core_backward_host",
    "dcn_core_backward_noalloc",
    "dcn_core_backward_deterministic_workspace",
    "dcn_core_backward_deterministic",
    "dcn_core_offset_mask_guide",
    "dcn_core_offset_mask_projection",
    "dcn_core_linear_bf16",
    "dcn_core_offset_mask_guide_projection",
    "dcn_core_sync_status",
    "dcn_status_string",
    "dcn_core_abi_version",
)


class DcnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dcn_status_string(status)} (status {status})")


class DcnProblem(ctypes.Structure):
    """Mirror of ``dcn_problem`` in include/dcn_core.h."""
    _fields_ = [("N", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("G", ctypes.c_int), ("Cg", ctypes.c_int), ("K", ctypes.c_int),
                ("stride", ctypes.c_int), ("pad", ctypes.c_int), ("dilation", ctypes.c_int),
                ("offset_scale", ctypes.c_float), ("softmax", ctypes.c_int),
                ("dtype", ctypes.c_int), ("remove_center", ctypes.c_int),
                ("separate_axes", ctypes.c_int), ("stride_w", ctypes.c_int),
                ("pad_w", ctypes.c_int), ("dilation_w", ctypes.c_int)]

    def __repr__(self):
        return "DcnProblem(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_problem(N, H, W, G, Cg, K=3, stride=1, pad=1, dilation=1, offset_scale=1.0,
                 softmax=1, dtype="f32", remove_center=0, stride_w=None, pad_w=None,
                 dilation_w=None) -> DcnProblem:
    """stride, pad and dilation apply to both axes unless a width value
    (stride_w, pad_w, dilation_w) is given; then they are the height axis's."""
    if isinstance(dtype, str):
        dtype = DTYPES[dtype]
    separate = stride_w is not None or pad_w is not None or dilation_w is not None
    sw = stride if stride_w is None else stride_w
    pw = pad if pad_w is None else pad_w
    dw = dilation if dilation_w is None else dilation_w
    return DcnProblem(int(N), int(H), int(W), int(G), int(Cg), int(K), int(stride), int(pad),
                      int(dilation), float(offset_scale), int(softmax), int(dtype),
                      int(remove_center), int(separate), int(sw), int(pw), int(dw))


def problem_for(wl) -> DcnProblem:
    """DcnProblem of a workload description (any object with the fields of
    gen.workloads.Workload)."""
    return make_problem(wl.N, wl.H, wl.W, wl.G, wl.Cg, wl.K, wl.stride, wl.pad, wl.dilation,
                        wl.offset_scale, wl.softmax, wl.dtype,
                        getattr(wl, "remove_center", 0))


def taps(problem: DcnProblem) -> int:
    """Taps per (pixel, group): K*K, or K*K - 1 with remove_center."""
    return problem.K * problem.K - (1 if problem.remove_center else 0)


_lib = None


def library_path() -> str:
    return LIB_PATH


def load_library():
    """Load libdcncore.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m deformable_convolution_core_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, pp = ctypes.c_void_p, ctypes.POINTER(DcnProblem)
    ip = ctypes.POINTER(ctypes.c_int)
    st = ctypes.c_int
    lib.dcn_core_output_hw.argtypes = [pp, ip, ip]
    lib.dcn_core_output_hw.restype = st
    lib.dcn_core_forward.argtypes = [pp, vp, vp, vp, vp, vp]
    lib.dcn_core_forward.restype = st
    lib.dcn_core_forward_host.argtypes = [pp] + [vp] * 9
    lib.dcn_core_forward_host.restype = st
    lib.dcn_core_backward_workspace.argtypes = [pp]
    lib.dcn_core_backward_workspace.restype = ctypes.c_size_t
    lib.dcn_core_backward.argtypes = [pp] + [vp] * 8 + [ctypes.c_size_t, vp]
    lib.dcn_core_backward.restype = st
    lib.dcn_core_backward_host.argtypes = [pp] + [vp] * 12 + [ctypes.c_size_t, vp]
    lib.dcn_core_backward_host.restype = st
    lib.dcn_core_backward_noalloc.argtypes = [pp] + [vp] * 8
    lib.dcn_core_backward_noalloc.restype = st
    lib.dcn_core_backward_deterministic_workspace.argtypes = [pp]
    lib.dcn_core_backward_deterministic_workspace.restype = ctypes.c_size_t
    lib.dcn_core_backward_deterministic.argtypes = [pp] + [vp] * 8 + [ctypes.c_size_t, vp]
    lib.dcn_core_backward_deterministic.restype = st
    lib.dcn_core_offset_mask_guide.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_float, vp, vp]
    lib.dcn_core_offset_mask_guide.restype = st
    lib.dcn_core_offset_mask_projection.argtypes = [pp, vp, ctypes.c_int, vp, vp, vp, vp, vp]
    lib.dcn_core_offset_mask_projection.restype = st
    lib.dcn_core_offset_mask_guide_projection.argtypes = [pp, vp, vp, vp, vp, vp, ctypes.c_float,
                                                          vp, vp, vp, vp, vp]
    lib.dcn_core_offset_mask_guide_projection.restype = st
    lib.dcn_core_linear_bf16.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, ctypes.c_int, vp, vp,
                                         ctypes.c_int, vp]
    lib.dcn_core_linear_bf16.restype = st
    lib.dcn_core_sync_status.argtypes = [vp]
    lib.dcn_core_sync_status.restype = st
    lib.dcn_status_string.argtypes = [st]
    lib.dcn_status_string.restype = ctypes.c_char_p
    lib.dcn_core_abi_version.argtypes = []
    lib.dcn_core_abi_version.restype = ctypes.c_int
    if lib.dcn_core_abi_version() != ABI_VERSION:
        raise ImportError(f"{LIB_PATH} has ABI version {lib.dcn_core_abi_version()}, this binding "
                          f"expects {ABI_VERSION}: rebuild it")
    _lib = lib
    return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        if not t.is_contiguous():
            raise ValueError("tensors passed to the C ABI must be contiguous")
        return t.data_ptr()
    raise TypeError(f"cannot pass {type(t)} as a pointer")


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != DCN_OK:
        raise DcnError(status, where)


def dcn_status_string(status: int) -> str:
    return load_library().dcn_status_string(int(status)).decode()


def dcn_core_abi_version() -> int:
    return int(load_library().dcn_core_abi_version())


def dcn_core_output_hw(problem: DcnProblem) -> tuple[int, int]:
    ho, wo = ctypes.c_int(0), ctypes.c_int(0)
    _check(load_library().dcn_core_output_hw(ctypes.byref(problem), ctypes.byref(ho),
                                             ctypes.byref(wo)), "dcn_core_output_hw")
    return ho.value, wo.value


def dcn_core_forward(problem: DcnProblem, input, offset, mask, output, stream=None) -> None:
    _check(load_library().dcn_core_forward(ctypes.byref(problem), _ptr(input), _ptr(offset),
                                           _ptr(mask), _ptr(output), _stream(stream)),
           "dcn_core_forward")


def dcn_core_forward_host(problem: DcnProblem, h_input, h_offset, h_mask, h_output, d_input,
                          d_offset, d_mask, d_output, stream=None) -> None:
    _check(load_library().dcn_core_forward_host(
        ctypes.byref(problem), _ptr(h_input), _ptr(h_offset), _ptr(h_mask), _ptr(h_output),
        _ptr(d_input), _ptr(d_offset), _ptr(d_mask), _ptr(d_output), _stream(stream)),
        "dcn_core_forward_host")


def dcn_core_backward_workspace(problem: DcnProblem) -> int:
    return int(load_library().dcn_core_backward_workspace(ctypes.byref(problem)))


def dcn_core_backward(problem: DcnProblem, input, offset, mask, grad_out, grad_input,
                      grad_offset, grad_mask, workspace=None, workspace_bytes=0,
                      stream=None) -> None:
    _check(load_library().dcn_core_backward(
        ctypes.byref(problem), _ptr(input), _ptr(offset), _ptr(mask), _ptr(grad_out),
        _ptr(grad_input), _ptr(grad_offset), _ptr(grad_mask), _ptr(workspace),
        int(workspace_bytes), _stream(stream)), "dcn_core_backward")


def dcn_core_backward_host(problem: DcnProblem, input, offset, mask, h_grad_out, h_grad_input,
                           h_grad_offset, h_grad_mask, d_grad_out, d_grad_input, d_grad_offset,
                           d_grad_mask, workspace=None, workspace_bytes=0, stream=None) -> None:
    """Backward with grad_out and the three gradients on (pinned) host
    buffers; input, offset and mask are the device tensors of the forward."""
    _check(load_library().dcn_core_backward_host(
        ctypes.byref(problem), _ptr(input), _ptr(offset), _ptr(mask), _ptr(h_grad_out),
        _ptr(h_grad_input), _ptr(h_grad_offset), _ptr(h_grad_mask), _ptr(d_grad_out),
        _ptr(d_grad_input), _ptr(d_grad_offset), _ptr(d_grad_mask), _ptr(workspace),
        int(workspace_bytes), _stream(stream)), "dcn_core_backward_host")


def dcn_core_backward_noalloc(problem: DcnProblem, input, offset, mask, grad_out, grad_input,
                              grad_offset, grad_mask, stream=None) -> None:
    """Backward without a workspace, for callers that cannot allocate device
    memory (see include/dcn_core.h).  For bf16 or fp16 storage the fp32 grad_input
    accumulator must fit the library's fixed DCN_CORE_NOALLOC_SCRATCH_BYTES
    array; calls that may overlap on the GPU must be serialised."""
    status = load_library().dcn_core_backward_noalloc(
        ctypes.byref(problem), _ptr(input), _ptr(offset), _ptr(mask), _ptr(grad_out),
        _ptr(grad_input), _ptr(grad_offset), _ptr(grad_mask), _stream(stream))
    if status == DCN_ERR_UNSUPPORTED and problem.dtype != DCN_F32:
        need = problem.N * problem.H * problem.W * problem.G * problem.Cg * 4
        if need > DCN_CORE_NOALLOC_SCRATCH_BYTES:
            raise DcnError(status, f"dcn_core_backward_noalloc: the fp32 accumulator of 2-byte storage needs {need} "
                                   f"bytes, more than the {DCN_CORE_NOALLOC_SCRATCH_BYTES} bytes "
                                   "of scratch this entry point owns")
    _check(status, "dcn_core_backward_noalloc")


def dcn_core_backward_deterministic_workspace(problem: DcnProblem) -> int:
    return int(load_library().dcn_core_backward_deterministic_workspace(ctypes.byref(problem)))


def dcn_core_backward_deterministic(problem: DcnProblem, input, offset, mask, grad_out,
                                    grad_input, grad_offset, grad_mask, workspace,
                                    workspace_bytes, stream=None) -> None:
    """Bitwise-reproducible backward (see include/dcn_core.h): grad_input is
    accumulated exactly in 64-bit fixed point inside `workspace`."""
    _check(load_library().dcn_core_backward_deterministic(
        ctypes.byref(problem), _ptr(input), _ptr(offset), _ptr(mask), _ptr(grad_out),
        _ptr(grad_input), _ptr(grad_offset), _ptr(grad_mask), _ptr(workspace),
        int(workspace_bytes), _stream(stream)), "dcn_core_backward_deterministic")


def dcn_core_offset_mask_guide(problem: DcnProblem, input, dw_weight, dw_bias, ln_gamma,
                               ln_beta, ln_eps: float, query, stream=None) -> None:
    """Depthwise 3x3 + LayerNorm + GELU of the block's input into the bf16
    query of the offset / mask projection (see include/dcn_core.h)."""
    _check(load_library().dcn_core_offset_mask_guide(
        ctypes.byref(problem), _ptr(input), _ptr(dw_weight), _ptr(dw_bias), _ptr(ln_gamma),
        _ptr(ln_beta), float(ln_eps), _ptr(query), _stream(stream)), "dcn_core_offset_mask_guide")


def dcn_core_offset_mask_projection(problem: DcnProblem, query, Cq: int, weight, bias, offset,
                                    mask, stream=None) -> None:
    """offset / mask = query @ weight.T + bias on the tensor cores (see
    include/dcn_core.h).  query (N, Ho, Wo, Cq) and weight (G*KK*3, Cq) are
    bf16; bias (G*KK*3) fp32 or None; offset and mask are written in the
    problem's storage type and the layouts dcn_core_forward reads."""
    _check(load_library().dcn_core_offset_mask_projection(
        ctypes.byref(problem), _ptr(query), int(Cq), _ptr(weight), _ptr(bias), _ptr(offset),
        _ptr(mask), _stream(stream)), "dcn_core_offset_mask_projection")


def dcn_core_offset_mask_guide_projection(problem: DcnProblem, input, dw_weight, dw_bias,
                                          ln_gamma, ln_beta, ln_eps: float, weight, bias, offset,
                                          mask, stream=None) -> None:
    """Guide features and offset / mask projection in one kernel (the query
    stays on chip; see include/dcn_core.h): the result of
    dcn_core_offset_mask_guide followed by dcn_core_offset_mask_projection."""
    _check(load_library().dcn_core_offset_mask_guide_projection(
        ctypes.byref(problem), _ptr(input), _ptr(dw_weight), _ptr(dw_bias), _ptr(ln_gamma),
        _ptr(ln_beta), float(ln_eps), _ptr(weight), _ptr(bias), _ptr(offset), _ptr(mask),
        _stream(stream)), "dcn_core_offset_mask_guide_projection")


def dcn_core_linear_bf16(input, M: int, K: int, weight, Nout: int, bias, output,
                         out_dtype="f32", stream=None) -> None:
    """output (M, Nout) = input (M, K) @ weight (Nout, K).T + bias on the tensor
    cores; bf16 operands, fp32 accumulation, output in out_dtype."""
    if isinstance(out_dtype, str):
        out_dtype = DTYPES[out_dtype]
    _check(load_library().dcn_core_linear_bf16(
        _ptr(input), int(M), int(K), _ptr(weight), int(Nout), _ptr(bias), _ptr(output),
        int(out_dtype), _stream(stream)), "dcn_core_linear_bf16")


def dcn_core_sync_status(stream=None) -> None:
    _check(load_library().dcn_core_sync_status(_stream(stream)), "dcn_core_sync_status")


__all__ = ["DcnProblem", "DcnError", "make_problem", "problem_for", "taps", "load_library",
           "library_path", "EXPORTED_SYMBOLS", *EXPORTED_SYMBOLS, "ABI_VERSION",
           "DCN_CORE_NOALLOC_SCRATCH_BYTES",
           "DCN_OK", "DCN_ERR_INVALID_ARG", "DCN_ERR_UNSUPPORTED", "DCN_ERR_CUDA",
           "DCN_ERR_TIMEOUT", "DCN_ERR_OUT_OF_BOUNDS", "DCN_F32", "DCN_BF16", "DCN_F16",
           "DTYPES"]
