"""The C-ABI library builds, loads and exports every entry point its header
declares; host-side validation rejects bad arguments before any launch.
Runs without a GPU: no call here reaches a kernel."""
import os
import re

import pytest

import deformable_convolution_core_b200 as dcn
from deformable_convolution_core_b200 import build as dcn_build
from tests.conftest import ROOT


@pytest.fixture(scope="module")
def lib():
    dcn_build.build()
    return dcn.load_library()


def declared_symbols():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names += re.findall(r"DCN_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert set(dcn.EXPORTED_SYMBOLS) <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert dcn.dcn_core_abi_version() == dcn.ABI_VERSION == 5
    for st in range(6):
        assert dcn.dcn_status_string(st)
    assert "unknown" in dcn.dcn_status_string(99)


def test_output_hw(lib):
    assert dcn.dcn_core_output_hw(dcn.make_problem(1, 96, 96, 10, 16)) == (96, 96)
    assert dcn.dcn_core_output_hw(dcn.make_problem(2, 256, 256, 12, 16, stride=2)) == (128, 128)
    assert dcn.dcn_core_output_hw(dcn.make_problem(1, 7, 9, 1, 8, K=5, pad=0, dilation=1)) == (3, 5)
    with pytest.raises(dcn.DcnError):
        dcn.dcn_core_output_hw(dcn.make_problem(1, 2, 2, 1, 8, K=5, pad=0))
    # separate axes: Ho from the height values, Wo from the width ones
    assert dcn.dcn_core_output_hw(dcn.make_problem(1, 20, 21, 1, 8, stride=2, pad=1,
                                                   stride_w=1, pad_w=0, dilation_w=2)) == (10, 17)
    # removing the centre tap leaves the output grid unchanged
    assert dcn.dcn_core_output_hw(dcn.make_problem(1, 7, 9, 1, 8, K=3, remove_center=1)) == (7, 9)


def test_problem_mirrors_header_struct():
    """DcnProblem has the fields of dcn_problem, in order."""
    text = open(os.path.join(ROOT, "include", "dcn_core.h")).read()
    body = re.search(r"typedef struct \{(.*?)\} dcn_problem;", text, re.S).group(1)
    names = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            names += [n.strip().lstrip("*") for n in decl.split(None, 1)[1].split(",")]
    assert names == [n for n, _ in dcn.DcnProblem._fields_]


GOOD = dict(N=1, H=8, W=8, G=2, Cg=16, K=3, stride=1, pad=1, dilation=1, offset_scale=1.0,
            softmax=1, dtype="f32")
FAKE = 1 << 20  # an address that is 16- and 32-byte aligned; never dereferenced here


@pytest.mark.parametrize("change,status", [
    (dict(N=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(H=-1), dcn.DCN_ERR_INVALID_ARG),
    (dict(G=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(Cg=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(K=2), dcn.DCN_ERR_INVALID_ARG),
    (dict(K=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(stride=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(pad=-1), dcn.DCN_ERR_INVALID_ARG),
    (dict(dilation=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(softmax=2), dcn.DCN_ERR_INVALID_ARG),
    (dict(remove_center=2), dcn.DCN_ERR_INVALID_ARG),
    (dict(remove_center=1, K=1, pad=0), dcn.DCN_ERR_INVALID_ARG),  # no tap left
    (dict(stride_w=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(pad_w=-1), dcn.DCN_ERR_INVALID_ARG),
    (dict(dilation_w=0), dcn.DCN_ERR_INVALID_ARG),
    (dict(W=2, pad_w=0, dilation_w=2), dcn.DCN_ERR_INVALID_ARG),   # empty output along W
    (dict(dtype=7), dcn.DCN_ERR_INVALID_ARG),
    (dict(dtype=3), dcn.DCN_ERR_INVALID_ARG),
    (dict(offset_scale=float("nan")), dcn.DCN_ERR_INVALID_ARG),
    (dict(H=2, W=2, K=5, pad=0), dcn.DCN_ERR_INVALID_ARG),     # empty output
    (dict(N=1 << 16, H=1 << 8, W=1 << 8, G=16, Cg=16), dcn.DCN_ERR_INVALID_ARG),  # >= 2^31 elements
    (dict(Cg=5), dcn.DCN_ERR_UNSUPPORTED),                      # 20 bytes: no kernel
    (dict(Cg=48), dcn.DCN_ERR_UNSUPPORTED),                     # 192 bytes
])
def test_forward_rejects_before_launch(lib, change, status):
    p = dcn.make_problem(**{**GOOD, **change})
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_forward(p, FAKE, FAKE, FAKE, FAKE, 0)
    assert e.value.status == status


def test_forward_rejects_null_and_misaligned(lib):
    p = dcn.make_problem(**GOOD)
    for args in [(0, FAKE, FAKE, FAKE), (FAKE, 0, FAKE, FAKE), (FAKE, FAKE, 0, FAKE),
                 (FAKE, FAKE, FAKE, 0)]:
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_forward(p, *args, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    for args in [(FAKE + 4, FAKE, FAKE, FAKE), (FAKE, FAKE + 8, FAKE, FAKE),
                 (FAKE, FAKE, FAKE + 2, FAKE), (FAKE, FAKE, FAKE, FAKE + 16)]:
        with pytest.raises(dcn.DcnError) as e:   # Cg=16 fp32: 32-byte vectors on x and out
            dcn.dcn_core_forward(p, *args, 0)
        assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_backward_rejects_before_launch(lib):
    p = dcn.make_problem(**GOOD)
    ptrs = [FAKE] * 7
    for i in range(7):
        bad = list(ptrs)
        bad[i] = 0
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward(p, *bad, None, 0, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    pb = dcn.make_problem(**{**GOOD, "dtype": "bf16"})
    need = dcn.dcn_core_backward_workspace(pb)
    assert need == 1 * 8 * 8 * 2 * 16 * 4          # fp32 accumulator for grad_input
    for ws, nbytes in [(None, 0), (FAKE, need - 16)]:  # bf16 needs the full workspace
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward(pb, *ptrs, ws, nbytes, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    assert dcn.dcn_core_backward_workspace(p) == 0
    pc = dcn.make_problem(**{**GOOD, "Cg": 12})
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward(pc, *ptrs, None, 0, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_noalloc_backward_rejects_before_launch(lib):
    p = dcn.make_problem(**GOOD)
    ptrs = [FAKE] * 7
    for i in range(7):
        bad = list(ptrs)
        bad[i] = 0
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward_noalloc(p, *bad, stream=0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
        bad[i] = FAKE + 8          # every pointer must be 16-byte aligned
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward_noalloc(p, *bad, stream=0)
        assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    pc = dcn.make_problem(**{**GOOD, "Cg": 12})
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_noalloc(pc, *ptrs, stream=0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_noalloc_scratch_size_matches_header():
    """The binding's DCN_CORE_NOALLOC_SCRATCH_BYTES is the header's #define."""
    text = open(os.path.join(ROOT, "include", "dcn_core.h")).read()
    expr = re.search(r"#define\s+DCN_CORE_NOALLOC_SCRATCH_BYTES\s+\((.*?)\)\s*$", text, re.M).group(1)
    assert re.fullmatch(r"[0-9u*\s]+", expr), expr
    assert eval(expr.replace("u", "")) == dcn.DCN_CORE_NOALLOC_SCRATCH_BYTES


def test_deterministic_backward_rejects_before_launch(lib):
    p = dcn.make_problem(**GOOD)
    need = dcn.dcn_core_backward_deterministic_workspace(p)
    assert need == 256 + 1 * 8 * 8 * 2 * 16 * 8   # header + 64-bit accumulator
    ptrs = [FAKE] * 7
    for i in range(7):
        bad = list(ptrs)
        bad[i] = 0
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward_deterministic(p, *bad, FAKE, need, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    for ws, nbytes in [(None, need), (FAKE, need - 8)]:
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_backward_deterministic(p, *ptrs, ws, nbytes, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    with pytest.raises(dcn.DcnError) as e:   # the workspace must be 256-byte aligned
        dcn.dcn_core_backward_deterministic(p, *ptrs, FAKE + 16, need, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    pc = dcn.make_problem(**{**GOOD, "Cg": 12})
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_deterministic(pc, *ptrs, FAKE, 1 << 20, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    assert dcn.dcn_core_backward_deterministic_workspace(dcn.make_problem(**{**GOOD, "N": 0})) == 0


def test_forward_host_rejects_before_copy(lib):
    p = dcn.make_problem(**GOOD)
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_forward_host(p, 0, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0)
    assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_forward_host(p, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_backward_host_rejects_before_copy(lib):
    """Every argument error of the chunked host backward is found before the
    first copy is enqueued (no CUDA call is reached here)."""
    p = dcn.make_problem(**GOOD)
    dev3 = [FAKE] * 3          # input, offset, mask (device)
    host4 = [FAKE] * 4         # grad_out, grad_input, grad_offset, grad_mask (host)
    dgrads = [FAKE] * 4        # the device staging buffers
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_host(p, *dev3, 0, *host4[1:], *dgrads, None, 0, 0)
    assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_host(p, *dev3, *host4, FAKE + 4, *dgrads[1:], None, 0, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    pb = dcn.make_problem(**{**GOOD, "dtype": "bf16"})
    with pytest.raises(dcn.DcnError) as e:  # bf16 needs the fp32 accumulator workspace
        dcn.dcn_core_backward_host(pb, *dev3, *host4, *dgrads, None, 0, 0)
    assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    pc = dcn.make_problem(**{**GOOD, "Cg": 12})
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_backward_host(pc, *dev3, *host4, *dgrads, None, 0, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_guide_rejects_before_launch(lib):
    p = dcn.make_problem(**GOOD)
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_offset_mask_guide(p, 0, FAKE, FAKE, FAKE, FAKE, 1e-6, FAKE, 0)
    assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    for eps in (-1.0, float("nan"), float("inf")):
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_offset_mask_guide(p, FAKE, FAKE, None, None, None, eps, FAKE, 0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    for bad in (dict(G=1, Cg=6), dict(G=3, Cg=688)):  # C not a multiple of 4; C above 2048
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_offset_mask_guide(dcn.make_problem(**{**GOOD, **bad}), FAKE, FAKE, None,
                                           None, None, 1e-6, FAKE, 0)
        assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    with pytest.raises(dcn.DcnError) as e:  # an unaligned weight
        dcn.dcn_core_offset_mask_guide(p, FAKE, FAKE + 4, None, None, None, 1e-6, FAKE, 0)
    assert e.value.status == dcn.DCN_ERR_UNSUPPORTED


def test_library_has_no_oracle_dependency():
    """The CUDA library and binding never reference the oracle."""
    pkg = os.path.join(ROOT, "deformable_convolution_core_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), os.path.join(dirpath, f)


def test_projection_and_linear_reject_before_launch(lib):
    p = dcn.make_problem(**GOOD)
    for args in [(0, 64, FAKE, None, FAKE, FAKE), (FAKE, 64, 0, None, FAKE, FAKE),
                 (FAKE, 64, FAKE, None, 0, FAKE), (FAKE, 64, FAKE, None, FAKE, 0),
                 (FAKE, 0, FAKE, None, FAKE, FAKE)]:
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_offset_mask_projection(p, *args, stream=0)
        assert e.value.status == dcn.DCN_ERR_INVALID_ARG
    for args in [(FAKE, 60, FAKE, None, FAKE, FAKE),        # Cq not a multiple of 8
                 (FAKE + 8, 64, FAKE, None, FAKE, FAKE),    # unaligned query
                 (FAKE, 64, FAKE, FAKE + 2, FAKE, FAKE)]:   # unaligned bias
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_offset_mask_projection(p, *args, stream=0)
        assert e.value.status == dcn.DCN_ERR_UNSUPPORTED
    for args, status in [((0, 16, 64, FAKE, 32, None, FAKE), dcn.DCN_ERR_INVALID_ARG),
                         ((FAKE, 0, 64, FAKE, 32, None, FAKE), dcn.DCN_ERR_INVALID_ARG),
                         ((FAKE, 16, 60, FAKE, 32, None, FAKE), dcn.DCN_ERR_UNSUPPORTED),
                         ((FAKE, 16, 64, FAKE, 32, None, FAKE + 4), dcn.DCN_ERR_UNSUPPORTED)]:
        with pytest.raises(dcn.DcnError) as e:
            dcn.dcn_core_linear_bf16(*args, stream=0)
        assert e.value.status == status
    with pytest.raises(dcn.DcnError) as e:
        dcn.dcn_core_linear_bf16(FAKE, 16, 64, FAKE, 32, None, FAKE, out_dtype=7, stream=0)
    assert e.value.status == dcn.DCN_ERR_INVALID_ARG
