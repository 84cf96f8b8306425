// Backward kernel of the deformable-convolution core (sm_100a, fp32).
//
// Gradients of the forward (InternImage-L DCNv3 explainer (wmrh.cn), section
// 二 steps 2-4; the DCNv3 extension build guide (trdm.cn), section 2.1, names
// the forward and backward device code that this replaces).  Per unit
// (pixel, group) and tap k, with v_k the unweighted bilinear sample and g the
// upstream gradient of the unit's Cg outputs:
//   s_k      = <g, v_k>
//   grad dx  = offset_scale * m_k * <g, dv/dX>,  grad dy likewise with dv/dY
//   grad logit_k = m_k (s_k - sum_j m_j s_j)   (softmax; raw mask: s_k)
//   grad x[corner] += m_k * w_corner * g       (vectorised float4 atomics)
// With the four corner dot products d_c = <g, x[corner c]>,
//   s_k = sum_c w_c d_c,  <g, dv/dX> = hy (d01 - d00) + ly (d11 - d10),
//   <g, dv/dY> = hx (d10 - d00) + lx (d11 - d01),
// so each corner is loaded once and reduced immediately.
#pragma once

#include "dcn_tile.cuh"

namespace dcn {

struct BwdArgs {
  const float* x;
  const void* off;
  const void* mask;
  const float* gout;
  float* gx;
  float* goff;
  float* gmask;
  TileParams t;
};

template <int LANES>
__device__ __forceinline__ float unit_sum(float v, unsigned mask) {
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o);
  return v;
}

template <int CPL, int LANES, int KKS, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads) dcn_backward_kernel(const BwdArgs a) {
  using St = Staged<float>;
  constexpr int VB = CPL * 4;
  static_assert(VB == 16 || VB == 32, "a lane gathers 16 or 32 bytes per corner");
  using V = Vec<VB>;
  constexpr int UPW = 32 / LANES;

  const TileParams& t = a.t;
  const int KK = KKS ? KKS : t.KK;
  const int GKK = t.G * KK;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  auto* s_off = reinterpret_cast<float2*>(smem_raw);
  auto* s_msk = reinterpret_cast<float*>(smem_raw + size_t(GKK) * t.P1 * sizeof(float2));

  const TileCoord tc = tile_coord(t, blockIdx.x);
  stage_tile<float>(t, tc, KK, a.off, a.mask, s_off, s_msk);
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LANES;
  const unsigned umask = LANES == 32 ? 0xFFFFFFFFu
                                     : (((1u << LANES) - 1u) << (lane & ~(LANES - 1)));
  const int units = t.G * t.tile_px;
  const size_t pixE = size_t(t.C);
  const size_t rowE = size_t(t.W) * pixE;
  const size_t img_off = size_t(tc.n) * t.H * rowE + size_t(sub) * CPL;

  for (int v0 = warp * UPW; v0 < units; v0 += kWarps * UPW) {
    const UnitCoord u = unit_coord(t, tc, v0 + lane / LANES);
    if (!u.valid) continue;
    const int row0 = u.g * KK;
    const size_t g_off = img_off + size_t(u.g) * t.Cg;
    const float* xg = a.x + g_off;
    float* gxg = a.gx + g_off;
    const size_t upix = size_t(tc.n * t.Ho + u.ho) * t.Wo + u.wo;
    const size_t unit = upix * t.G + u.g;
    const int by = u.ho * t.stride - t.pad, bx = u.wo * t.stride - t.pad;

    float go[CPL];
    {
      V gv;
      ldg_nc(gv, a.gout + upix * t.C + size_t(u.g) * t.Cg + size_t(sub) * CPL);
#pragma unroll
      for (int j = 0; j < CPL; ++j) go[j] = __uint_as_float(gv.w[j]);
    }

    // One tap: returns s_k (reduced over the unit's lanes) and writes the
    // offset gradient of the tap.
    auto tap = [&](int k, int ka, int kb, float mk) -> float {
      const float2 d = St::pair(s_off[(row0 + k) * t.P1 + u.pix]);
      const float Y = tap_coord(by + ka * t.dil, t.sigma, d.y);
      const float X = tap_coord(bx + kb * t.dil, t.sigma, d.x);
      const Footprint f = footprint(Y, X, t.H, t.W);
      float s = 0.f, gX = 0.f, gY = 0.f;
      if (f.in_support) {
        const float hy = 1.f - f.ly, hx = 1.f - f.lx;
        const ptrdiff_t base = ptrdiff_t(f.y0) * ptrdiff_t(rowE) + ptrdiff_t(f.x0) * ptrdiff_t(pixE);
        const ptrdiff_t cofs[4] = {base, base + ptrdiff_t(pixE), base + ptrdiff_t(rowE),
                                   base + ptrdiff_t(rowE + pixE)};
        const bool cval[4] = {f.v00, f.v01, f.v10, f.v11};
        const float cw[4] = {hy * hx, hy * f.lx, f.ly * hx, f.ly * f.lx};
        float dc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          V cv;
#pragma unroll
          for (int i = 0; i < CPL; ++i) cv.w[i] = 0u;
          if (cval[c]) ldg_nc(cv, xg + cofs[c]);
          float dsum = 0.f;
#pragma unroll
          for (int j = 0; j < CPL; ++j) dsum = fmaf(go[j], __uint_as_float(cv.w[j]), dsum);
          dc[c] = dsum;
          if (cval[c]) {
            const float wv = mk * cw[c];
            float* gp = gxg + cofs[c];
#pragma unroll
            for (int q = 0; q < CPL / 4; ++q)
              atomicAdd(reinterpret_cast<float4*>(gp) + q,
                        make_float4(wv * go[4 * q], wv * go[4 * q + 1], wv * go[4 * q + 2],
                                    wv * go[4 * q + 3]));
          }
        }
        s = cw[0] * dc[0] + cw[1] * dc[1] + cw[2] * dc[2] + cw[3] * dc[3];
        gX = hy * (dc[1] - dc[0]) + f.ly * (dc[3] - dc[2]);
        gY = hx * (dc[2] - dc[0]) + f.lx * (dc[3] - dc[1]);
      }
      if (LANES > 1) {
        s = unit_sum<LANES>(s, umask);
        gX = unit_sum<LANES>(gX, umask);
        gY = unit_sum<LANES>(gY, umask);
      }
      if (sub == 0) {
        const float sc = t.sigma * mk;
        reinterpret_cast<float2*>(a.goff)[unit * KK + k] = make_float2(sc * gX, sc * gY);
      }
      return s;
    };

    if constexpr (KKS > 0) {
      constexpr int K = KKS == 1 ? 1 : (KKS == 9 ? 3 : (KKS == 25 ? 5 : 7));
      static_assert(K * K == KKS, "compile-time tap counts are odd squares");
      float m[KKS], s[KKS];
      mask_weights<float, KKS, SOFTMAX>(s_msk, row0, t.P1, u.pix, m);
#pragma unroll
      for (int k = 0; k < KKS; ++k) s[k] = tap(k, k / K, k % K, m[k]);
      if (sub == 0) {
        float ms = 0.f;
        if (SOFTMAX) {
#pragma unroll
          for (int k = 0; k < KKS; ++k) ms = fmaf(m[k], s[k], ms);
        }
#pragma unroll
        for (int k = 0; k < KKS; ++k)
          a.gmask[unit * KK + k] = SOFTMAX ? m[k] * (s[k] - ms) : s[k];
      }
    } else {
      // Runtime tap count: keep (s_k, m_k) in the tap's staged offset slot,
      // which no other unit reads and this unit no longer needs.
      float mx, inv;
      mask_stats<float, SOFTMAX>(s_msk, row0, t.P1, u.pix, KK, mx, inv);
      for (int k = 0, ka = 0, kb = 0; k < KK; ++k) {
        const float mk = mask_weight_at<float, SOFTMAX>(s_msk, row0 + k, t.P1, u.pix, mx, inv);
        const float sk = tap(k, ka, kb, mk);
        if (LANES > 1) __syncwarp(umask);
        if (sub == 0) s_off[(row0 + k) * t.P1 + u.pix] = make_float2(sk, mk);
        if (++kb == t.K) { kb = 0; ++ka; }
      }
      if (sub == 0) {
        float ms = 0.f;
        if (SOFTMAX)
          for (int k = 0; k < KK; ++k) {
            const float2 sm = s_off[(row0 + k) * t.P1 + u.pix];
            ms = fmaf(sm.y, sm.x, ms);
          }
        for (int k = 0; k < KK; ++k) {
          const float2 sm = s_off[(row0 + k) * t.P1 + u.pix];
          a.gmask[unit * KK + k] = SOFTMAX ? sm.y * (sm.x - ms) : sm.x;
        }
      }
    }
  }
}

}  // namespace dcn
