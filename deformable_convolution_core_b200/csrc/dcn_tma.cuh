// Shared pieces of the kernels that stage the input in shared memory by TMA
// (sm_100a): the work-item decomposition, the box geometry, and the mbarrier
// and bulk-tensor-copy primitives.
//
// A persistent CTA walks work items (image n, output tile, group g).  For
// each item one TMA tensor copy brings the group's Cg channels of the input
// box the tile can reach into shared memory, zero filled outside the image,
// which is exactly the operator's zero padding.  Every mbarrier wait is
// bounded; on expiry the kernel sets the device error word, waits (bounded)
// for its own copies in flight and returns.
#pragma once

#include <cuda.h>

#include "dcn_common.cuh"
#include "dcn_tile.cuh"

namespace dcn {

constexpr int kTiledWarps = 15;  // consumer warps: with the producer, 4 warps per SM sub-partition
constexpr int kTiledThreads = (kTiledWarps + 1) * 32;  // + one TMA producer warp
constexpr int kTiledBatch = 32;                       // units per warp batch
constexpr int kTiledMaxTaps = 9;  // the tiled kernels serve 3x3 windows (9 or 8 taps)
constexpr int kTiledMaxBufs = 8;  // input boxes in flight, at most

struct TiledParams {
  int N, H, W, G, Cg, C, stride, pad, dil, Ho, Wo;  // stride/pad/dil: height axis
  int stride_w, pad_w, dil_w;                       // width axis
  float sigma;
  int TH, TW, nTY, nTX, halo, BH, BW;  // BW: the box row pitch in pixels (all of it is loaded)
  int clamp_box;       // 1: box origins are clamped to the image and its one-pixel zero ring
  int nbuf;            // input boxes in flight (2 .. kTiledMaxBufs)
  int items;           // N * nTY * nTX * G
  int inject_stall;    // test knob: 1 = never load the first item's box, so the
                       // bounded waits expire and the error path runs
  int batches;         // warp batches per item: ceil(TH * TW / kTiledBatch)
  uint32_t box_bytes;  // BH * BW * Cg * sizeof(T)
  uint32_t box_stride; // box_bytes rounded up to 1024
  FastDiv fd_G, fd_nTX, fd_tiles, fd_TW;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// try_wait with a suspend-time hint: the thread may sleep up to `ns`
// nanoseconds inside the instruction instead of spinning on issue slots; it
// returns as soon as the phase completes.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase with the given parity: gives up after 2^22
// polls or one second, whichever comes first.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < (1u << 22); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && global_ns() - t0 > 1000000000ull) return false;
  }
  return false;
}

// The same bound (one second) for waits that may be long (a consumer waiting
// for its box, a producer waiting for a free buffer): each poll sleeps up to 2
// microseconds inside try_wait, so waiting warps leave the issue slots to the
// working ones.
__device__ __forceinline__ bool mbar_wait_bounded_sleep(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < (1u << 20); ++i) {
    if (mbar_try_wait_sleep(bar, parity, 2000u)) return true;
    if ((i & 15u) == 15u && global_ns() - t0 > 1000000000ull) return false;
  }
  return false;
}

__device__ __forceinline__ void tma_load_box(void* dst, const CUtensorMap* map, uint64_t* bar,
                                             int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}

// The same from a 32-bit shared-window address.
__device__ __forceinline__ uint4 lds128_a(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

__device__ __forceinline__ uint4 ldg128(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// 16 bytes from global memory, zeros unless pred (a false predicate issues no access).
__device__ __forceinline__ uint4 ldg128_pred(const void* p, bool pred) {
  uint4 v;
  asm("{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
      " mov.b32 %0, 0;\n mov.b32 %1, 0;\n mov.b32 %2, 0;\n mov.b32 %3, 0;\n"
      " @q ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];\n}"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p), "r"(int(pred)));
  return v;
}

// Item -> (n, ho0, wo0, g); g is the fastest index, so consecutive items of a
// CTA reuse one input neighbourhood (different channels) and one run of
// offset/mask rows.
struct ItemCoord {
  int n, ho0, wo0, g;
};

__device__ __forceinline__ ItemCoord item_coord(const TiledParams& t, int item) {
  ItemCoord c;
  const uint32_t tile = fdiv(uint32_t(item), t.fd_G);
  c.g = item - int(tile) * t.G;
  const uint32_t n = fdiv(tile, t.fd_tiles);
  const uint32_t rem = tile - n * uint32_t(t.nTY * t.nTX);
  const uint32_t ty = fdiv(rem, t.fd_nTX);
  c.n = int(n);
  c.ho0 = int(ty) * t.TH;
  c.wo0 = int(rem - ty * uint32_t(t.nTX)) * t.TW;
  return c;
}

// First input row (or column) of an item's box.  Unclamped it is the tile's
// first sampling row less the halo.  With clamp_box the box is slid to stay
// within the rows that can matter, [-1, extent]: a footprint has rows y0 and
// y0 + 1 with -1 <= y0 < extent for any sample that contributes, and the
// image's zero ring (row -1 or row `extent`) is read as TMA zero fill.  A box
// taller than extent + 2 starts at -1 and covers every such row.
__host__ __device__ __forceinline__ int box_origin(int first, int box, int extent, bool clamp) {
  if (!clamp) return first;
  const int hi = extent + 1 - box;  // last origin whose box still ends at row `extent`
  return first < -1 ? -1 : (first > hi ? (hi < -1 ? -1 : hi) : first);
}

template <typename T>
struct TiledIO;
template <>
struct TiledIO<float> {
  static constexpr int kEpc = 4;  // channels per 16-byte piece
  using Pair = float2;
  using One = float;
  __device__ __forceinline__ static Pair ld_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const float2*>(base) + i);
  }
  __device__ __forceinline__ static One ld_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const float*>(base) + i);
  }
  __device__ __forceinline__ static float2 pair(Pair p) { return p; }
  __device__ __forceinline__ static float one(One v) { return v; }
  // acc += w * (the piece's 4 channels), as two packed fp32x2 FMAs.
  __device__ __forceinline__ static void fma16(float2* acc, float2 w, const uint4& v) {
    acc[0] = __ffma2_rn(make_float2(__uint_as_float(v.x), __uint_as_float(v.y)), w, acc[0]);
    acc[1] = __ffma2_rn(make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), w, acc[1]);
  }
};
template <>
struct TiledIO<__nv_bfloat16> {
  static constexpr int kEpc = 8;
  using Pair = uint32_t;
  using One = unsigned short;
  __device__ __forceinline__ static Pair ld_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned int*>(base) + i);
  }
  __device__ __forceinline__ static One ld_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned short*>(base) + i);
  }
  __device__ __forceinline__ static float2 pair(Pair p) {
    return make_float2(bf16lo_to_f32(p), bf16hi_to_f32(p));
  }
  __device__ __forceinline__ static float one(One v) { return __uint_as_float(uint32_t(v) << 16); }
  // acc += w * (the piece's 8 channels, widened), as four packed fp32x2 FMAs.
  __device__ __forceinline__ static void fma16(float2* acc, float2 w, const uint4& v) {
    acc[0] = __ffma2_rn(make_float2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x)), w, acc[0]);
    acc[1] = __ffma2_rn(make_float2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y)), w, acc[1]);
    acc[2] = __ffma2_rn(make_float2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z)), w, acc[2]);
    acc[3] = __ffma2_rn(make_float2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w)), w, acc[3]);
  }
};

template <>
struct TiledIO<__half> {
  static constexpr int kEpc = 8;
  using Pair = uint32_t;
  using One = unsigned short;
  __device__ __forceinline__ static Pair ld_pair(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned int*>(base) + i);
  }
  __device__ __forceinline__ static One ld_one(const void* base, size_t i) {
    return __ldg(reinterpret_cast<const unsigned short*>(base) + i);
  }
  __device__ __forceinline__ static float2 pair(Pair p) { return f16x2_to_f32x2(p); }
  __device__ __forceinline__ static float one(One v) { return __half2float(__ushort_as_half(v)); }
  __device__ __forceinline__ static void fma16(float2* acc, float2 w, const uint4& v) {
    acc[0] = __ffma2_rn(f16x2_to_f32x2(v.x), w, acc[0]);
    acc[1] = __ffma2_rn(f16x2_to_f32x2(v.y), w, acc[1]);
    acc[2] = __ffma2_rn(f16x2_to_f32x2(v.z), w, acc[2]);
    acc[3] = __ffma2_rn(f16x2_to_f32x2(v.w), w, acc[3]);
  }
};

// Output of four fp32 values in storage type T: 16 bytes (fp32) or 8 bytes.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  return pack_bf16x2(lo, hi);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  return pack_f16x2(lo, hi);
}

}  // namespace dcn
