// Forward kernel with the input staged in shared memory by TMA (sm_100a).
//
// Same operator as dcn_forward_kernel (InternImage-L DCNv3 explainer
// (wmrh.cn), section 二 steps 2-4, section 三).  The difference is where the
// bilinear corners are read from.  A global gather costs the L1 one
// wavefront per distinct 128-byte line touched, i.e. one per corner whatever
// its size, so a direct-gather kernel is capped near four L1 cycles per
// sample.  Here a persistent CTA walks work items (image n, output tile,
// group g); for each item one TMA tensor copy brings the group's Cg channels
// of the input box the tile can reach (tile + kernel extent + halo, zero
// filled outside the image) into shared memory, double-buffered on two
// mbarriers.  The four corners of one sample are then two 2-pixel row chunks
// of the box; 4*Cg*sizeof(T)/16 lanes each read one 16-byte piece, and with
// the box row pitch chosen so that the two rows fall into complementary bank
// halves the whole footprint is one conflict-free shared-memory wavefront
// per 128 bytes.  Samples whose corners lie outside the box (large offsets)
// read those corners from global memory instead; the result is the same.
//
// Every mbarrier wait is bounded; on expiry the kernel sets the device error
// word, waits (bounded) for its own copies in flight and returns.
#pragma once

#include <cuda.h>

#include "dcn_common.cuh"

namespace dcn {

constexpr int kTiledWarps = 15;  // consumer warps: with the producer, 4 warps per SM sub-partition
constexpr int kTiledThreads = (kTiledWarps + 1) * 32;  // + one TMA producer warp
constexpr int kTiledBatch = 32;                       // units per warp batch
constexpr int kTiledMaxTaps = 9;  // the tiled kernel serves 3x3 windows (9 or 8 taps)
// Shared memory after the unit slots: the full/empty mbarriers and the abort
// flag (bytes 0-35), then at kTiledZeroAt a 128-byte area of zeros that the
// forward's box reads of far or dead taps are pointed at.
constexpr int kTiledZeroAt = 64;
constexpr int kTiledZeroBytes = 128;
constexpr int kTiledTailBytes = kTiledZeroAt + kTiledZeroBytes;

struct TiledParams {
  int N, H, W, G, Cg, C, stride, pad, dil, Ho, Wo;  // stride/pad/dil: height axis
  int stride_w, pad_w, dil_w;                       // width axis
  float sigma;
  int TH, TW, nTY, nTX, halo, BH, BW;
  int items;           // N * nTY * nTX * G
  int inject_stall;    // test knob: 1 = never load the first item's box, so the
                       // bounded waits expire and the error path runs
  int batches;         // warp batches per item: ceil(TH * TW / kTiledBatch)
  uint32_t box_bytes;  // BH * BW * Cg * sizeof(T)
  uint32_t box_stride; // box_bytes rounded up to 1024
  FastDiv fd_G, fd_nTX, fd_tiles, fd_TW;
};

struct TiledArgs {
  const void* x;
  const void* off;
  const void* mask;
  void* out;
  unsigned int* error_word;
  TiledParams t;
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

__device__ __forceinline__ uint4 ldg128(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
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
  __device__ __forceinline__ static uint4 pack(const float (&acc)[4]) {
    return make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                      __float_as_uint(acc[3]));
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
  __device__ __forceinline__ static uint4 pack(const float (&acc)[8]) {
    return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                      pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
};

// Tap records, written by the unit's owner lane in phase A and read by the
// unit's eight lanes in phase B.  A unit slot holds w[9][4] (the tap's four
// corner weights, mask weight folded in) followed by code[9], of which the
// 8-tap set (remove_center) uses the first eight.  code >= 0 is
// the byte offset in the box of corner (y0, x0) when the whole 2x2 footprint
// lies in the box; otherwise code = INT_MIN | (y0 + 1) << 15 | (x0 + 1), and
// the corners are read from global memory ((y0, x0) = (32766, 32766) marks a
// sample that contributes nothing).
constexpr int kFarCell = 32766;
__device__ __forceinline__ int far_code(int y0, int x0) {
  return int(0x80000000u | (uint32_t(y0 + 1) << 15) | uint32_t(x0 + 1));
}
// 184 bytes: w[9][4] (144) then code[9] (36), padded to a multiple of 8 so
// that staged fp32 offset pairs (8-byte float2) stay aligned in every slot;
// 46 words per slot also keeps both the 32-lane phase-A reads and the
// four-unit phase-B reads free of bank conflicts.
constexpr int kSlotBytes = 184;
constexpr int kCodeAt = kTiledMaxTaps * 16;
constexpr int kLogitAt = 80;               // staged mask values (before the records)
constexpr int kFarMaskAt = kCodeAt + kTiledMaxTaps * 4;  // 180: bit k = tap k is read from global
static_assert(kSlotBytes % 8 == 0 && kFarMaskAt + 4 <= kSlotBytes, "slot layout");

// Phase-B lane roles: 8 lanes per unit, lane li = (corner r = li >> 1, q = li & 1).
// A 32-byte group (bf16 x 16) is one 16-byte piece per lane: piece q.  A
// 64-byte group (fp32 x 16) is two pieces per lane; in read j a lane takes
// piece (2j + q + 2*dy) & 3, so the eight lanes of a unit touch eight
// different bank quads when the box row pitch is even.
template <int CS>
struct LaneRole {
  static constexpr int kPieces = CS / 32;  // pieces per lane: 1 or 2
  __device__ __forceinline__ static int piece(int j, int q, int dyc) {
    return CS == 32 ? q : ((2 * j + q + 2 * dyc) & 3);
  }
};

// KKS: 9 (the 3x3 window) or 8 (the window without its centre).
template <typename T, int CS, int KKS, bool SOFTMAX>
__global__ void __launch_bounds__(kTiledThreads, 1)
    dcn_forward_tiled_kernel(const __grid_constant__ CUtensorMap xmap, const TiledArgs a) {
  using IO = TiledIO<T>;
  using Pair = typename IO::Pair;
  using One = typename IO::One;
  using Role = LaneRole<CS>;
  constexpr int KK = KKS, K = tap_side(KKS);
  static_assert(K == 3 && KK <= kTiledMaxTaps, "the tiled kernel serves 3x3 tap sets");
  constexpr int LU = 8;            // phase-B lanes per unit
  constexpr int UPW = 32 / LU;     // units per phase-B step
  constexpr int NP = Role::kPieces;
  constexpr int EPC = IO::kEpc;    // channels per piece
  static_assert(CS == 32 || CS == 64, "the tiled kernel serves 32- or 64-byte groups");
  static_assert(KK * sizeof(Pair) <= kLogitAt && kLogitAt + KK * sizeof(One) <= kSlotBytes,
                "staged inputs fit in a slot");

  const TiledParams& t = a.t;
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* bufs = smem;
  unsigned char* slots = smem + 2 * size_t(t.box_stride);
  uint64_t* full =
      reinterpret_cast<uint64_t*>(slots + size_t(kTiledWarps) * kTiledBatch * kSlotBytes);
  uint64_t* empty = full + 2;
  int* s_abort = reinterpret_cast<int*>(empty + 2);
  unsigned char* zero = reinterpret_cast<unsigned char*>(full) + kTiledZeroAt;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&empty[0], kTiledWarps);
    mbar_init(&empty[1], kTiledWarps);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < kTiledZeroBytes / 4) reinterpret_cast<uint32_t*>(zero)[tid] = 0u;
  __syncthreads();
  volatile int* abort_flag = s_abort;

  // ---- producer warp: one TMA box per item, two buffers in flight ----
  if (warp == kTiledWarps) {
    if (lane != 0) return;
    int i = 0;
    for (;; ++i) {
      const int item = int(blockIdx.x) + i * int(gridDim.x);
      if (item >= t.items || *abort_flag) break;
      const int b = i & 1;
      if (i >= 2 && !mbar_wait_bounded(&empty[b], ((i >> 1) - 1) & 1)) {
        atomicOr(a.error_word, 1u);
        *abort_flag = 1;
        break;
      }
      const ItemCoord c = item_coord(t, item);
      if (t.inject_stall && i == 0) continue;  // the first box never arrives
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&full[b], t.box_bytes);
      tma_load_box(bufs + size_t(b) * t.box_stride, &xmap, &full[b], c.g * t.Cg,
                   c.wo0 * t.stride_w - t.pad_w - t.halo, c.ho0 * t.stride - t.pad - t.halo, c.n);
    }
    // Copies issued for items i-2 and i-1 may still be landing: wait for them
    // (bounded) before this thread, possibly the CTA's last, exits.
    for (int j = i - 2; j < i; ++j)
      if (j >= 0) (void)mbar_wait_bounded(&full[j & 1], (j >> 1) & 1);
    return;
  }

  // ---- consumer warps ----
  unsigned char* myslots = slots + size_t(warp) * kTiledBatch * kSlotBytes;
  const int ul = lane / LU;         // phase B: unit of this lane within a step
  const int li = lane - ul * LU;
  const int r = li >> 1, q = li & 1;
  const int dyc = r >> 1, dxc = r & 1;
  const unsigned umask = 0xFFu << (ul * LU);
  int cdelta[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j)
    cdelta[j] = (dyc * t.BW + dxc) * CS + Role::piece(j, q, dyc) * 16;
  const size_t pixB = size_t(t.C) * sizeof(T);
  const int npx = t.TH * t.TW;
  const int nb = t.batches;
  // the staging element e = lane + 32 k (k < KK) belongs to unit e / KK, tap e % KK
  int st_unit[KK], st_tap[KK];
#pragma unroll
  for (int k = 0; k < KK; ++k) {
    st_unit[k] = (lane + 32 * k) / KK;
    st_tap[k] = (lane + 32 * k) - st_unit[k] * KK;
  }

  // Batch beta of this CTA (over all its items) -> this lane's unit.
  auto batch_unit = [&](int beta, bool& valid, int& ho, int& wo, size_t& qbase) {
    const int il = beta / nb;
    const int v = (beta - il * nb) * kTiledBatch + lane;
    const int item = int(blockIdx.x) + il * int(gridDim.x);
    valid = false;
    ho = wo = 0;
    qbase = 0;
    if (item >= t.items) return;
    const ItemCoord c = item_coord(t, item);
    const int rr = int(fdiv(uint32_t(v), t.fd_TW));
    ho = c.ho0 + rr;
    wo = c.wo0 + (v - rr * t.TW);
    valid = (v < npx) && (ho < t.Ho) && (wo < t.Wo);
    qbase = ((size_t(c.n * t.Ho + ho) * t.Wo + wo) * t.G + c.g) * KK;
  };

  // Raw inputs of the next batch, prefetched in the staging layout.
  const size_t n_entries = size_t(t.N) * t.Ho * t.Wo * t.G * KK;  // offset pairs, mask values
  const size_t x_bytes = size_t(t.N) * t.H * t.W * pixB;            // bounds-checked build
  const size_t out_bytes = size_t(t.N) * t.Ho * t.Wo * pixB;
  Pair pf_pair[KK];
  One pf_one[KK];
  auto prefetch = [&](int beta) {
    bool valid;
    int ho, wo;
    size_t qbase;
    batch_unit(beta, valid, ho, wo, qbase);
    const unsigned long long qv = valid ? (unsigned long long)qbase : ~0ull;
#pragma unroll
    for (int k = 0; k < KK; ++k) {
      const unsigned long long src = __shfl_sync(0xFFFFFFFFu, qv, st_unit[k]);
      if (src != ~0ull && in_range(size_t(src) + st_tap[k], n_entries)) {
        pf_pair[k] = IO::ld_pair(a.off, size_t(src) + st_tap[k]);
        pf_one[k] = IO::ld_one(a.mask, size_t(src) + st_tap[k]);
      } else {
        pf_pair[k] = Pair();
        pf_one[k] = One();
      }
    }
  };

  const int n_items_cta =
      int(blockIdx.x) < t.items ? (t.items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int total_batches = n_items_cta * nb;
  int beta = warp;
  if (beta < total_batches) prefetch(beta);

  for (int il = 0; il < n_items_cta; ++il) {
    const int b = il & 1;
    const int item = int(blockIdx.x) + il * int(gridDim.x);
    // Every consumer warp observes every item's box, even one in which it has
    // no batch: that keeps each warp within one item of the producer, so the
    // parity it waits for is never ambiguous and it arrives on `empty` exactly
    // once per phase.
    if (!mbar_wait_bounded(&full[b], (il >> 1) & 1)) {
      atomicOr(a.error_word, 1u);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const ItemCoord c = item_coord(t, item);
    const unsigned char* box = bufs + size_t(b) * t.box_stride;
    // Phase B reads piece j of a tap at box + min(code, zlim) + cdelta[j]: a
    // box tap's code (>= 0, below the box size) is kept, a far or dead tap's
    // (negative, so above 2^31 unsigned) becomes zlim, which puts this lane's
    // pieces at zero + 48 + (cdelta[j] - cdelta[0]), inside the zero area
    // (pieces of one lane lie at most 32 bytes apart).  zlim exceeds every box
    // offset because the zero area lies after both buffers and the slots.
    const uint32_t zlim = uint32_t((zero + 48 - cdelta[0]) - box);
    const int Y0 = c.ho0 * t.stride - t.pad - t.halo;
    const int X0 = c.wo0 * t.stride_w - t.pad_w - t.halo;
    const char* ximg = reinterpret_cast<const char*>(a.x) + size_t(c.n) * t.H * t.W * pixB +
                       size_t(c.g) * CS;

    for (; beta < (il + 1) * nb; beta += kTiledWarps) {
      // Staging: the prefetched inputs go to the unit slots.
#pragma unroll
      for (int k = 0; k < KK; ++k) {
        unsigned char* sl = myslots + st_unit[k] * kSlotBytes;
        reinterpret_cast<Pair*>(sl)[st_tap[k]] = pf_pair[k];
        reinterpret_cast<One*>(sl + kLogitAt)[st_tap[k]] = pf_one[k];
      }
      bool valid;
      int ho, wo;
      size_t qbase;
      batch_unit(beta, valid, ho, wo, qbase);
      __syncwarp();

      // Phase A: this lane's unit -> softmax, then per tap the footprint code
      // and the four corner weights.
      {
        unsigned char* sl = myslots + lane * kSlotBytes;
        float2 d[KK];
        float m[KK];
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          d[k] = IO::pair(reinterpret_cast<const Pair*>(sl)[k]);
          m[k] = IO::one(reinterpret_cast<const One*>(sl + kLogitAt)[k]);
        }
        if (SOFTMAX) {
          float mx = m[0];
#pragma unroll
          for (int k = 1; k < KK; ++k) mx = fmaxf(mx, m[k]);
          float sum = 0.f;
#pragma unroll
          for (int k = 0; k < KK; ++k) {
            m[k] = expf(m[k] - mx);
            sum += m[k];
          }
          const float inv = 1.0f / sum;
#pragma unroll
          for (int k = 0; k < KK; ++k) m[k] *= inv;
        }
        __syncwarp();  // every lane has read its staged inputs
        float* wsl = reinterpret_cast<float*>(sl);
        int* csl = reinterpret_cast<int*>(sl + kCodeAt);
        unsigned farmask = 0u;
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const int ka = tap_pos(KK, k) / K, kb = tap_pos(KK, k) % K;
          const float Y = tap_coord(ho * t.stride - t.pad + ka * t.dil, t.sigma, d[k].y);
          const float X = tap_coord(wo * t.stride_w - t.pad_w + kb * t.dil_w, t.sigma, d[k].x);
          const Footprint f = footprint(Y, X, t.H, t.W);
          const bool live = valid && f.in_support;
          const int by = f.y0 - Y0, bx = f.x0 - X0;
          int code;
          if (!live) code = far_code(kFarCell, kFarCell);
          else if (by >= 0 && by + 1 < t.BH && bx >= 0 && bx + 1 < t.BW)
            code = (by * t.BW + bx) * CS;
          else {
            code = far_code(f.y0, f.x0);
            farmask |= 1u << k;
          }
          const float mk = live ? m[k] : 0.f;
          const float hy = 1.f - f.ly, hx = 1.f - f.lx;
          wsl[4 * k + 0] = hy * hx * mk;
          wsl[4 * k + 1] = hy * f.lx * mk;
          wsl[4 * k + 2] = f.ly * hx * mk;
          wsl[4 * k + 3] = f.ly * f.lx * mk;
          csl[k] = code;
        }
        *reinterpret_cast<unsigned*>(sl + kFarMaskAt) = farmask;
      }
      __syncwarp();
      // The next batch's inputs are loaded while this one is gathered.
      if (beta + kTiledWarps < total_batches) prefetch(beta + kTiledWarps);

      // Phase B: UPW units per step, eight lanes each.  Box taps are
      // branch-free (predicated shared-memory reads); a unit's taps whose
      // footprint leaves the box ("far" taps) read global memory: the first
      // one of each unit is fetched a step ahead, any further ones in a
      // warp-uniform loop.
      const int v0 = (beta - il * nb) * kTiledBatch;
      // Global read of this lane's corner piece(s) for tap k of the unit in slot sl.
      auto far_fetch = [&](const unsigned char* sl, int k, uint4 (&fv)[NP], float& fw) {
        const int code = reinterpret_cast<const int*>(sl + kCodeAt)[k];
        fw = reinterpret_cast<const float*>(sl)[4 * k + r];
        const int yc = ((code >> 15) & 0x7FFF) - 1 + dyc;
        const int xc = (code & 0x7FFF) - 1 + dxc;
        const bool in = unsigned(yc) < unsigned(t.H) && unsigned(xc) < unsigned(t.W);
        const char* gp = ximg + (size_t(in ? yc : 0) * t.W + (in ? xc : 0)) * pixB;
#pragma unroll
        for (int j = 0; j < NP; ++j)
          fv[j] = (in && in_tensor(gp + Role::piece(j, q, dyc) * 16, 16, a.x, x_bytes))
                      ? ldg128(gp + Role::piece(j, q, dyc) * 16)
                      : make_uint4(0u, 0u, 0u, 0u);
        if (!in) fw = 0.f;
      };
      auto far_first = [&](int u, uint4 (&fv)[NP], float& fw) {
        const unsigned char* sl = myslots + u * kSlotBytes;
        const unsigned fm = *reinterpret_cast<const unsigned*>(sl + kFarMaskAt);
        fw = 0.f;
#pragma unroll
        for (int j = 0; j < NP; ++j) fv[j] = make_uint4(0u, 0u, 0u, 0u);
        if (fm) far_fetch(sl, __ffs(fm) - 1, fv, fw);
      };
      uint4 fv_cur[NP], fv_nxt[NP];
      float fw_cur, fw_nxt;
      far_first(ul, fv_cur, fw_cur);
#pragma unroll 1
      for (int s = 0; s < kTiledBatch / UPW; ++s) {
        const int u = s * UPW + ul;
        const unsigned char* sl = myslots + u * kSlotBytes;
        const float* wsl = reinterpret_cast<const float*>(sl) + r;
        const int* csl = reinterpret_cast<const int*>(sl + kCodeAt);
        if (s + 1 < kTiledBatch / UPW) far_first(u + UPW, fv_nxt, fw_nxt);
        constexpr int NV = NP * EPC;  // 8 values per lane, as 4 packed pairs
        static_assert(NV == 8, "eight accumulated values per lane");
        float2 acc[NV / 2];
#pragma unroll
        for (int e = 0; e < NV / 2; ++e) acc[e] = make_float2(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const uint32_t off = min(uint32_t(csl[k]), zlim);  // far or dead: the zero area
          const float w = wsl[4 * k];
          const float2 w2 = make_float2(w, w);
#pragma unroll
          for (int j = 0; j < NP; ++j) IO::fma16(acc + j * (EPC / 2), w2, lds128(box + off + cdelta[j]));
        }
        // First far tap (fetched during the previous step), then any others.
#pragma unroll
        for (int j = 0; j < NP; ++j)
          IO::fma16(acc + j * (EPC / 2), make_float2(fw_cur, fw_cur), fv_cur[j]);
        unsigned more = *reinterpret_cast<const unsigned*>(sl + kFarMaskAt);
        more &= more - 1u;
        while (__any_sync(0xFFFFFFFFu, more != 0u)) {
          if (more) {
            uint4 fv[NP];
            float fw;
            far_fetch(sl, __ffs(more) - 1, fv, fw);
#pragma unroll
            for (int j = 0; j < NP; ++j) IO::fma16(acc + j * (EPC / 2), make_float2(fw, fw), fv[j]);
            more &= more - 1u;
          }
        }
        // Lanes with dy = 1 hold their pieces in the other order (fp32 only).
        if (NP == 2 && dyc) {
#pragma unroll
          for (int e = 0; e < EPC / 2; ++e) {
            const float2 tmp = acc[e];
            acc[e] = acc[EPC / 2 + e];
            acc[EPC / 2 + e] = tmp;
          }
        }
        // Reduce-scatter over the four corner lanes of each piece: the dx pair
        // splits the 8 values in halves, the dy pair splits those again, so each
        // lane ends with 2 summed values: value index 4*dxc + 2*dyc + {0, 1}.
        float h4[4], h2[2];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = (i & 1) ? acc[i >> 1].y : acc[i >> 1].x;           // value i
          const float hi = (i & 1) ? acc[2 + (i >> 1)].y : acc[2 + (i >> 1)].x;  // value 4 + i
          const float keep = dxc ? hi : lo;
          const float send = dxc ? lo : hi;
          h4[i] = keep + __shfl_xor_sync(umask, send, 2);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float keep = dyc ? h4[2 + i] : h4[i];
          const float send = dyc ? h4[i] : h4[2 + i];
          h2[i] = keep + __shfl_xor_sync(umask, send, 4);
        }
        const int v = v0 + u;
        const int rr = int(fdiv(uint32_t(v), t.fd_TW));
        const int uho = c.ho0 + rr, uwo = c.wo0 + (v - rr * t.TW);
        if (v < npx && uho < t.Ho && uwo < t.Wo) {
          const size_t pix = size_t(c.n * t.Ho + uho) * t.Wo + uwo;
          char* op = reinterpret_cast<char*>(a.out) + (pix * t.C + size_t(c.g) * t.Cg) * sizeof(T);
          // channel of h2[0]: piece p, element 2*dyc (+ 4*dxc for bf16's 8-wide pieces)
          if (CS == 32) {
            const int ch = 8 * q + 4 * dxc + 2 * dyc;
            const uint32_t w = pack_bf16x2(h2[0], h2[1]);
            if (in_tensor(op + ch * 2, 4, a.out, out_bytes))
              asm volatile("st.global.b32 [%0], %1;" ::"l"(op + ch * 2), "r"(w) : "memory");
          } else {
            const int ch = 4 * (q + 2 * dxc) + 2 * dyc;
            if (in_tensor(op + ch * 4, 8, a.out, out_bytes))
              asm volatile("st.global.v2.f32 [%0], {%1, %2};" ::"l"(op + ch * 4), "f"(h2[0]),
                         "f"(h2[1])
                         : "memory");
          }
        }
#pragma unroll
        for (int j = 0; j < NP; ++j) fv_cur[j] = fv_nxt[j];
        fw_cur = fw_nxt;
      }
      __syncwarp();  // slots are rewritten by the next batch
    }
    __syncwarp();
    if (lane == 0) {
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&empty[b]))
                   : "memory");
    }
  }
}

}  // namespace dcn
