// Forward gather-reduce kernel of the deformable-convolution core (sm_100a).
//
// What it computes (InternImage-L DCNv3 explainer (wmrh.cn), section 二 steps
// 2-4, section 三): out[n,ho,wo,g,:] = sum_k m_k * bilinear(x[n,:,:,g,:],
// Y_k, X_k), with (Y_k, X_k) the tap's grid point plus offset_scale * (dy, dx)
// and m the softmax of the group's mask logits (DCNv3) or the raw mask
// (DCNv4).
//
// Mapping: LANES lanes own one (pixel, group) unit and CPL channels each
// (CPL * sizeof(T) = 16 or 32 bytes), so every corner of a sample is one
// 16/32-byte vector per lane, and a warp-level gather of one corner reads
// 32 / LANES full 32-byte sectors.  Arithmetic is fp32; bf16 is widened on
// load and rounded once on store.  No tensor cores: the operator is a
// gather-reduce, not a dense contraction.
#pragma once

#include "dcn_tile.cuh"

namespace dcn {

struct FwdArgs {
  const void* x;
  const void* off;
  const void* mask;
  void* out;
  TileParams t;
};

template <typename T, int CPL, int LANES, int KKS, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads) dcn_forward_kernel(const FwdArgs a) {
  using S = Storage<T>;
  using St = Staged<T>;
  constexpr int VB = CPL * S::kSize;  // bytes per lane per corner
  static_assert(VB == 16 || VB == 32, "a lane gathers 16 or 32 bytes per corner");
  constexpr int NW = VB / 4;
  using V = Vec<VB>;
  constexpr int UPW = 32 / LANES;  // units per warp pass

  const TileParams& t = a.t;
  const int KK = KKS ? KKS : t.KK;
  const int GKK = t.G * KK;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto* s_off = reinterpret_cast<typename St::Pair*>(smem_raw);
  auto* s_msk = reinterpret_cast<typename St::One*>(smem_raw + size_t(GKK) * t.P1 *
                                                                   sizeof(typename St::Pair));

  const TileCoord tc = tile_coord(t, blockIdx.x);
  stage_tile<T>(t, tc, KK, a.off, a.mask, s_off, s_msk);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const int units = t.G * t.tile_px;
  const size_t pixB = size_t(t.C) * S::kSize;
  const size_t rowB = size_t(t.W) * pixB;
  const char* xbase = reinterpret_cast<const char*>(a.x) +
                      size_t(tc.n) * t.H * rowB + size_t(sub) * CPL * S::kSize;
  const size_t x_bytes = size_t(t.N) * t.H * rowB;                     // bounds-checked build
  const size_t out_bytes = size_t(t.N) * t.Ho * t.Wo * t.C * S::kSize;  // bounds-checked build

  for (int v0 = warp * UPW; v0 < units; v0 += kWarps * UPW) {
    const UnitCoord u = unit_coord(t, tc, v0 + lane / LANES);
    if (!u.valid) continue;
    const int row0 = u.g * KK;
    const char* xg = xbase + size_t(u.g) * t.Cg * S::kSize;
    const int by = u.ho * t.stride - t.pad, bx = u.wo * t.stride_w - t.pad_w;

    float acc[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) acc[j] = 0.f;

    // One tap: location, footprint, four predicated corner gathers, FMAs.
    auto tap = [&](int k, int ka, int kb, float mk) {
      const float2 d = St::pair(s_off[(row0 + k) * t.P1 + u.pix]);
      const float Y = tap_coord(by + ka * t.dil, t.sigma, d.y);
      const float X = tap_coord(bx + kb * t.dil_w, t.sigma, d.x);
      const Footprint f = footprint(Y, X, t.H, t.W);
      if (!f.in_support) return;
      const float hy = 1.f - f.ly, hx = 1.f - f.lx;
      const float w00 = hy * hx * mk, w01 = hy * f.lx * mk;
      const float w10 = f.ly * hx * mk, w11 = f.ly * f.lx * mk;
      const char* p = xg + ptrdiff_t(f.y0) * ptrdiff_t(rowB) + ptrdiff_t(f.x0) * ptrdiff_t(pixB);
      V c00, c01, c10, c11;
#pragma unroll
      for (int i = 0; i < NW; ++i) c00.w[i] = c01.w[i] = c10.w[i] = c11.w[i] = 0u;
      if (f.v00 && in_tensor(p, VB, a.x, x_bytes)) ldg_nc(c00, p);
      if (f.v01 && in_tensor(p + pixB, VB, a.x, x_bytes)) ldg_nc(c01, p + pixB);
      if (f.v10 && in_tensor(p + rowB, VB, a.x, x_bytes)) ldg_nc(c10, p + rowB);
      if (f.v11 && in_tensor(p + rowB + pixB, VB, a.x, x_bytes)) ldg_nc(c11, p + rowB + pixB);
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        float s = acc[j];
        s = fmaf(w00, S::chan(c00.w, j), s);
        s = fmaf(w01, S::chan(c01.w, j), s);
        s = fmaf(w10, S::chan(c10.w, j), s);
        s = fmaf(w11, S::chan(c11.w, j), s);
        acc[j] = s;
      }
    };

    if constexpr (KKS > 0) {
      float m[KKS];
      mask_weights<T, KKS, SOFTMAX>(s_msk, row0, t.P1, u.pix, m);
      constexpr int K = tap_side(KKS);
#pragma unroll
      for (int k = 0; k < KKS; ++k) tap(k, tap_pos(KKS, k) / K, tap_pos(KKS, k) % K, m[k]);
    } else {
      float mx, inv;
      mask_stats<T, SOFTMAX>(s_msk, row0, t.P1, u.pix, KK, mx, inv);
      for (int k = 0, ka = 0, kb = 0; k < KK; ++k) {
        skip_removed_tap(t, ka, kb);
        tap(k, ka, kb, mask_weight_at<T, SOFTMAX>(s_msk, row0 + k, t.P1, u.pix, mx, inv));
        if (++kb == t.K) { kb = 0; ++ka; }
      }
    }

    V o;
    S::pack(o.w, acc);
    char* op = reinterpret_cast<char*>(a.out) +
               ((size_t(tc.n * t.Ho + u.ho) * t.Wo + u.wo) * t.C + size_t(u.g) * t.Cg +
                size_t(sub) * CPL) * S::kSize;
    if (in_tensor(op, VB, a.out, out_bytes)) stg(op, o);
  }
}

}  // namespace dcn
