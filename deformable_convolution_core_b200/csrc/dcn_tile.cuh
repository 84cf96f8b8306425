// Tile decomposition shared by the forward and backward kernels.
//
// One CTA owns a tile of TH x TW output pixels of one image and ALL G groups
// of those pixels.  It first copies the tile's offsets and mask into shared
// memory, then walks the tile's (group, pixel) units group by group, so that
// the warps working at any moment all gather from one group's Cg channels of
// one small neighbourhood of the input: that keeps the L1 working set at about
// (TH + halo) x (TW + halo) x Cg elements.
#pragma once

#include "dcn_common.cuh"

namespace dcn {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct TileParams {
  int N, H, W, G, Cg, C, K, KK, stride, pad, dil, Ho, Wo;  // stride/pad/dil: height axis
  int stride_w, pad_w, dil_w;                              // width axis
  int kc;       // window position (a*K + b) left out by remove_center, else -1
  float sigma;
  int TH, TW, nTY, nTX;
  int tile_px;  // TH * TW
  int P1;       // pixel stride of the shared-memory tables (odd, >= tile_px)
  FastDiv fd_tile_px, fd_TW, fd_GKK, fd_tiles_per_img, fd_nTX;
};

// Shared-memory element types of the staged offset pairs and mask values:
// the raw storage bits, widened when read.
template <typename T>
struct Staged;
template <>
struct Staged<float> {
  using Pair = float2;
  using One = float;
  __device__ __forceinline__ static float2 pair(const Pair& p) { return p; }
  __device__ __forceinline__ static float one(const One& v) { return v; }
  __device__ __forceinline__ static Pair load_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const float2*>(base) + i);
  }
  __device__ __forceinline__ static One load_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const float*>(base) + i);
  }
};
template <>
struct Staged<__nv_bfloat16> {
  using Pair = uint32_t;
  using One = unsigned short;
  __device__ __forceinline__ static float2 pair(const Pair& p) {
    return make_float2(bf16lo_to_f32(p), bf16hi_to_f32(p));
  }
  __device__ __forceinline__ static float one(const One& v) {
    return __uint_as_float(uint32_t(v) << 16);
  }
  __device__ __forceinline__ static Pair load_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned int*>(base) + i);
  }
  __device__ __forceinline__ static One load_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned short*>(base) + i);
  }
};

template <>
struct Staged<__half> {
  using Pair = uint32_t;
  using One = unsigned short;
  __device__ __forceinline__ static float2 pair(const Pair& p) { return f16x2_to_f32x2(p); }
  __device__ __forceinline__ static float one(const One& v) {
    return __half2float(__ushort_as_half(v));
  }
  __device__ __forceinline__ static Pair load_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned int*>(base) + i);
  }
  __device__ __forceinline__ static One load_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned short*>(base) + i);
  }
};

template <typename T>
__host__ __device__ constexpr int staged_bytes_per_entry() {
  return int(sizeof(typename Staged<T>::Pair) + sizeof(typename Staged<T>::One));
}

// Compile-time tap sets: KKS = K*K taps of a K x K window, or 8 for the 3 x 3
// window without its centre (DCNv4's remove_center, DCNv4 speed-up write-up
// (pnsm.cn), section 3.3).  Tap k sits at window position tap_pos(KKS, k).
__host__ __device__ constexpr int tap_side(int kks) {
  return kks == 8 || kks == 9 ? 3 : (kks == 25 ? 5 : (kks == 49 ? 7 : 1));
}
__host__ __device__ constexpr int tap_pos(int kks, int k) {
  return (tap_side(kks) * tap_side(kks) != kks && k >= kks / 2) ? k + 1 : k;
}
static_assert(tap_pos(8, 3) == 3 && tap_pos(8, 4) == 5 && tap_pos(8, 7) == 8 &&
                  tap_pos(9, 4) == 4,
              "the 8-tap set skips window position 4");

// Runtime tap sets: step (ka, kb) over the window row by row, skipping the
// position kc (remove_center; kc = -1 skips nothing).
__device__ __forceinline__ void skip_removed_tap(const TileParams& t, int& ka, int& kb) {
  if (ka * t.K + kb == t.kc && ++kb == t.K) {
    kb = 0;
    ++ka;
  }
}

struct TileCoord {
  int n, ho0, wo0;
};

__device__ __forceinline__ TileCoord tile_coord(const TileParams& t, uint32_t tile) {
  TileCoord c;
  const uint32_t n = fdiv(tile, t.fd_tiles_per_img);
  const uint32_t rem = tile - n * uint32_t(t.nTY * t.nTX);
  const uint32_t ty = fdiv(rem, t.fd_nTX);
  const uint32_t tx = rem - ty * uint32_t(t.nTX);
  c.n = int(n);
  c.ho0 = int(ty) * t.TH;
  c.wo0 = int(tx) * t.TW;
  return c;
}

// Copy the tile's offset pairs and mask values into shared memory, transposed
// to [g*KK + k][pixel] so that a warp reading one tap of 32 consecutive pixels
// hits 32 consecutive entries.  Global reads are coalesced: consecutive
// threads read consecutive (g, k) entries of one pixel.
template <typename T>
__device__ __forceinline__ void stage_tile(const TileParams& t, const TileCoord& tc, int KK,
                                           const void* __restrict__ off,
                                           const void* __restrict__ mask,
                                           typename Staged<T>::Pair* s_off,
                                           typename Staged<T>::One* s_msk) {
  const int GKK = t.G * KK;
  const int n_elem = t.tile_px * GKK;
  for (int e = threadIdx.x; e < n_elem; e += kThreads) {
    const int pix = int(fdiv(uint32_t(e), t.fd_GKK));
    const int j = e - pix * GKK;
    const int r = int(fdiv(uint32_t(pix), t.fd_TW));
    const int c = pix - r * t.TW;
    const int ho = tc.ho0 + r, wo = tc.wo0 + c;
    const size_t q = (size_t(tc.n * t.Ho + ho) * t.Wo + wo) * GKK + j;
    if (ho < t.Ho && wo < t.Wo && in_range(q, size_t(t.N) * t.Ho * t.Wo * GKK)) {
      s_off[j * t.P1 + pix] = Staged<T>::load_pair(off, q);
      s_msk[j * t.P1 + pix] = Staged<T>::load_one(mask, q);
    }
  }
}

// Unit v of a tile (v = g * tile_px + pixel) -> group, pixel and output pixel.
struct UnitCoord {
  int g, pix, ho, wo;
  bool valid;
};

__device__ __forceinline__ UnitCoord unit_coord(const TileParams& t, const TileCoord& tc, int v) {
  UnitCoord u;
  u.g = int(fdiv(uint32_t(v), t.fd_tile_px));
  u.pix = v - u.g * t.tile_px;
  const int r = int(fdiv(uint32_t(u.pix), t.fd_TW));
  u.ho = tc.ho0 + r;
  u.wo = tc.wo0 + (u.pix - r * t.TW);
  u.valid = (u.g < t.G) && (u.ho < t.Ho) && (u.wo < t.Wo);
  return u;
}

// Mask weights of one (pixel, group) for a compile-time tap count: softmax
// over the taps (DCNv3) or the raw values (DCNv4).
template <typename T, int KKS, bool SOFTMAX>
__device__ __forceinline__ void mask_weights(const typename Staged<T>::One* s_msk, int row0,
                                             int P1, int pix, float (&m)[KKS]) {
#pragma unroll
  for (int k = 0; k < KKS; ++k) m[k] = Staged<T>::one(s_msk[(row0 + k) * P1 + pix]);
  if (SOFTMAX) {
    float mx = m[0];
#pragma unroll
    for (int k = 1; k < KKS; ++k) mx = fmaxf(mx, m[k]);
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < KKS; ++k) {
      m[k] = expf(m[k] - mx);
      sum += m[k];
    }
    const float inv = 1.0f / sum;
#pragma unroll
    for (int k = 0; k < KKS; ++k) m[k] *= inv;
  }
}

// Runtime tap count: max and normaliser of the softmax, evaluated per tap later.
template <typename T, bool SOFTMAX>
__device__ __forceinline__ void mask_stats(const typename Staged<T>::One* s_msk, int row0,
                                           int P1, int pix, int KK, float& mx, float& inv) {
  mx = 0.f;
  inv = 1.f;
  if (!SOFTMAX) return;
  mx = Staged<T>::one(s_msk[row0 * P1 + pix]);
  for (int k = 1; k < KK; ++k) mx = fmaxf(mx, Staged<T>::one(s_msk[(row0 + k) * P1 + pix]));
  float sum = 0.f;
  for (int k = 0; k < KK; ++k) sum += expf(Staged<T>::one(s_msk[(row0 + k) * P1 + pix]) - mx);
  inv = 1.0f / sum;
}

template <typename T, bool SOFTMAX>
__device__ __forceinline__ float mask_weight_at(const typename Staged<T>::One* s_msk, int row,
                                                int P1, int pix, float mx, float inv) {
  const float l = Staged<T>::one(s_msk[row * P1 + pix]);
  return SOFTMAX ? expf(l - mx) * inv : l;
}

}  // namespace dcn
