"""The synthetic workloads, as data.

Shapes stand in for InternImage-L at 384x384 input (four stages with
groups [10, 20, 40, 80], channels 160 -> 1280, offset_scale 2.0, as the
InternImage-L DCNv3 explainer (wmrh.cn) gives in its sections 三 and 四), plus
a tiny case, a high-resolution DCNv4-style case with an un-normalised mask,
and a backward case.  No dataset or trained weight is involved: every tensor
is drawn from the seeded generator with the distribution listed here.

Output sizes (Ho, Wo) are stored as data, not computed, so that this module
holds none of the operator's arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    cfg: int                 # workload family: 1 tiny, 2 stage-1 fp32, 3 bf16 sweep, 4 hi-res, 5 backward
    N: int
    H: int
    W: int
    G: int
    Cg: int
    K: int
    stride: int
    pad: int
    dilation: int
    offset_scale: float
    softmax: int             # 1: mask holds logits (DCNv3); 0: mask used as-is (DCNv4)
    dtype: str               # "f32", "bf16" or "f16" storage; arithmetic is fp32 always
    Ho: int
    Wo: int
    x_dist: tuple = ("normal", 0.0, 1.0)
    offset_dist: tuple = ("normal", 0.0, 1.5)
    mask_dist: tuple = ("normal", 0.0, 1.0)
    far: tuple | None = None  # (fraction of (dx,dy) pairs, lo, hi) redrawn from U(lo, hi)
    backward: bool = False
    remove_center: int = 0    # 1: the window's centre is not sampled (DCNv4), K*K - 1 taps
    seed_base: int = 1000
    tags: tuple = field(default_factory=tuple)

    @property
    def seed(self) -> int:
        return self.seed_base + self.cfg

    @property
    def C(self) -> int:
        return self.G * self.Cg

    @property
    def KK(self) -> int:
        """Taps per (pixel, group): the K x K window, less its centre with remove_center."""
        return self.K * self.K - self.remove_center

    @property
    def units(self) -> int:
        """(pixel, group) pairs of the output."""
        return self.N * self.Ho * self.Wo * self.G

    @property
    def samples(self) -> int:
        """(pixel, group, tap) bilinear samples of Cg channels."""
        return self.units * self.KK

    @property
    def esize(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def forward_bytes(self) -> int:
        """Compulsory forward traffic: x, offset and mask read once, output written once."""
        e = self.esize
        x = self.N * self.H * self.W * self.C
        off = self.units * self.KK * 2
        msk = self.units * self.KK
        out = self.N * self.Ho * self.Wo * self.C
        return e * (x + off + msk + out)

    def backward_bytes(self) -> int:
        """Compulsory backward traffic: x, offset, mask, grad_out read once;
        grad_input, grad_offset, grad_mask written once (the zero-fill of
        grad_input that the scatter needs is not counted)."""
        e = self.esize
        x = self.N * self.H * self.W * self.C
        off = self.units * self.KK * 2
        msk = self.units * self.KK
        gout = self.N * self.Ho * self.Wo * self.C
        return e * (2 * x + 2 * off + 2 * msk + gout)


def _wl(**kw) -> Workload:
    return Workload(**kw)


_STAGE = dict(K=3, stride=1, pad=1, dilation=1, offset_scale=2.0, softmax=1, Cg=16)

WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    # Tiny forward, fp32: a few seconds on CPU.
    _wl(name="tiny_fp32_n1_14x14_c64", cfg=1, N=1, H=14, W=14, G=4, Cg=16, K=3, stride=1,
        pad=1, dilation=1, offset_scale=1.0, softmax=1, dtype="f32", Ho=14, Wo=14,
        offset_dist=("uniform", -2.0, 2.0)),
    # InternImage-L stage 1 at 384x384 input, fp32.
    _wl(name="internimage_l_stage1_fp32_n32_96x96_c160", cfg=2, N=32, H=96, W=96, G=10,
        dtype="f32", Ho=96, Wo=96, **_STAGE),
    # Four-stage InternImage-L sweep, bf16 storage, 10% far offsets.
    _wl(name="internimage_l_stage1_bf16_n64_96x96_c160", cfg=3, N=64, H=96, W=96, G=10,
        dtype="bf16", Ho=96, Wo=96, far=(0.1, -8.0, 8.0), tags=("sweep",), **_STAGE),
    _wl(name="internimage_l_stage2_bf16_n64_48x48_c320", cfg=3, N=64, H=48, W=48, G=20,
        dtype="bf16", Ho=48, Wo=48, far=(0.1, -8.0, 8.0), tags=("sweep",), **_STAGE),
    _wl(name="internimage_l_stage3_bf16_n64_24x24_c640", cfg=3, N=64, H=24, W=24, G=40,
        dtype="bf16", Ho=24, Wo=24, far=(0.1, -8.0, 8.0), tags=("sweep",), **_STAGE),
    _wl(name="internimage_l_stage4_bf16_n64_12x12_c1280", cfg=3, N=64, H=12, W=12, G=80,
        dtype="bf16", Ho=12, Wo=12, far=(0.1, -8.0, 8.0), tags=("sweep",), **_STAGE),
    # High-resolution DCNv4-style forward: un-normalised mask ~U(-1,1), offsets ~N(0,2).
    _wl(name="dcnv4_hires_bf16_n2_256x256_c192_s1", cfg=4, N=2, H=256, W=256, G=12, Cg=16,
        K=3, stride=1, pad=1, dilation=1, offset_scale=1.0, softmax=0, dtype="bf16",
        Ho=256, Wo=256, offset_dist=("normal", 0.0, 2.0), mask_dist=("uniform", -1.0, 1.0)),
    _wl(name="dcnv4_hires_bf16_n2_256x256_c192_s2", cfg=4, N=2, H=256, W=256, G=12, Cg=16,
        K=3, stride=2, pad=1, dilation=1, offset_scale=1.0, softmax=0, dtype="bf16",
        Ho=128, Wo=128, offset_dist=("normal", 0.0, 2.0), mask_dist=("uniform", -1.0, 1.0)),
    # The same forward without the centre tap (DCNv4's remove_center: 8 taps).
    _wl(name="dcnv4_hires_bf16_n2_256x256_c192_s1_remove_center", cfg=4, N=2, H=256, W=256,
        G=12, Cg=16, K=3, stride=1, pad=1, dilation=1, offset_scale=1.0, softmax=0,
        dtype="bf16", Ho=256, Wo=256, offset_dist=("normal", 0.0, 2.0),
        mask_dist=("uniform", -1.0, 1.0), remove_center=1),
    # Backward at InternImage-L stage-2 shape, fp32.
    _wl(name="internimage_l_stage2_bwd_fp32_n32_48x48_c320", cfg=5, N=32, H=48, W=48, G=20,
        dtype="f32", Ho=48, Wo=48, backward=True, **_STAGE),
    # The same backward with bf16 storage (fp32 arithmetic, grad_input accumulated in fp32).
    _wl(name="internimage_l_stage2_bwd_bf16_n32_48x48_c320", cfg=5, N=32, H=48, W=48, G=20,
        dtype="bf16", Ho=48, Wo=48, backward=True, **_STAGE),
    # Other tap sets and channel widths on the stage-1 bf16 shape (the direct
    # kernels): 5x5 and 7x7 windows, 8 and 32 channels per group.
    _wl(name="internimage_l_stage1_k5_bf16_n16_96x96_c160", cfg=6, N=16, H=96, W=96, G=10,
        Cg=16, K=5, stride=1, pad=2, dilation=1, offset_scale=2.0, softmax=1, dtype="bf16",
        Ho=96, Wo=96),
    _wl(name="internimage_l_stage1_k7_bf16_n16_96x96_c160", cfg=6, N=16, H=96, W=96, G=10,
        Cg=16, K=7, stride=1, pad=3, dilation=1, offset_scale=2.0, softmax=1, dtype="bf16",
        Ho=96, Wo=96),
    _wl(name="internimage_l_stage1_cg8_bf16_n64_96x96_c160", cfg=6, N=64, H=96, W=96, G=20,
        Cg=8, K=3, stride=1, pad=1, dilation=1, offset_scale=2.0, softmax=1, dtype="bf16",
        Ho=96, Wo=96),
    _wl(name="internimage_l_stage1_cg32_bf16_n64_96x96_c160", cfg=6, N=64, H=96, W=96, G=5,
        Cg=32, K=3, stride=1, pad=1, dilation=1, offset_scale=2.0, softmax=1, dtype="bf16",
        Ho=96, Wo=96),
    # fp16 storage (the autocast type the pages train and serve with), fp32
    # arithmetic: the tiny case, the four stage shapes and the stage-2 backward.
    _wl(name="tiny_fp16_n1_14x14_c64", cfg=1, N=1, H=14, W=14, G=4, Cg=16, K=3, stride=1,
        pad=1, dilation=1, offset_scale=1.0, softmax=1, dtype="f16", Ho=14, Wo=14,
        offset_dist=("uniform", -2.0, 2.0)),
    _wl(name="internimage_l_stage1_fp16_n64_96x96_c160", cfg=3, N=64, H=96, W=96, G=10,
        dtype="f16", Ho=96, Wo=96, far=(0.1, -8.0, 8.0), tags=("sweep",), **_STAGE),
    _wl(name="internimage_l_stage2_fp16_n64_48x48_c320", cfg=3, N=64, H=48, W=48, G=20,
        dtype="f16", Ho=48, Wo=48, far=(0.1, -8.0, 8.0), **_STAGE),
    _wl(name="internimage_l_stage3_fp16_n64_24x24_c640", cfg=3, N=64, H=24, W=24, G=40,
        dtype="f16", Ho=24, Wo=24, far=(0.1, -8.0, 8.0), **_STAGE),
    _wl(name="internimage_l_stage4_fp16_n64_12x12_c1280", cfg=3, N=64, H=12, W=12, G=80,
        dtype="f16", Ho=12, Wo=12, far=(0.1, -8.0, 8.0), **_STAGE),
    _wl(name="internimage_l_stage2_bwd_fp16_n32_48x48_c320", cfg=5, N=32, H=48, W=48, G=20,
        dtype="f16", Ho=48, Wo=48, backward=True, **_STAGE),
]}


def output_hw(wl: Workload) -> tuple[int, int]:
    return wl.Ho, wl.Wo


# The step that the benchmark times at one GPU: forward + backward of the
# InternImage-L stage-1 fp32 shape.
BENCH_WORKLOAD = "internimage_l_stage1_fp32_n32_96x96_c160"
