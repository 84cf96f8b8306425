// Forward kernel for the wider windows (K = 5 or 7) with the input staged in
// shared memory by TMA (sm_100a).
//
// Same operator (InternImage-L DCNv3 explainer (wmrh.cn), section 二 steps
// 2-4, section 三; DCNv4 speed-up write-up, section 3.3 for the raw mask and
// remove_center) and the same machinery as dcn_forward_tiled_kernel: a
// persistent CTA walks items (image, output tile, group), a producer warp
// brings each item's input box into shared memory with one TMA tensor copy,
// and each bilinear footprint is read by four lanes, one per corner, in
// conflict-free 16-byte pieces.  What changes is the batch.  With 25 to 49
// taps the records of 32 units do not fit in a warp's region, so a warp takes
// 8 units at a time, one phase-B step:
//   staging  the 8 units' offset pairs and mask values (each unit's taps are
//            contiguous in memory) are copied into the region with cp.async,
//            issued during the previous batch once its records are built;
//   softmax  each unit's four lanes take every fourth tap; two shuffle rounds
//            combine their maxima and their sums;
//   chunks   the taps are processed CH at a time: phase A (lane r of a unit
//            builds the records of the chunk's taps r, r + 4, ...), phase B
//            (lane = bilinear corner, records read back as in the 3x3
//            kernel), then the chunk's far taps from global memory;
//   store    after the last chunk, the reduce-scatter over the four corner
//            lanes and one 8- or 16-byte store per lane, as in the 3x3 kernel.
#pragma once

#include "dcn_forward_tiled.cuh"

namespace dcn {

constexpr int kWideUnits = 8;      // units per warp batch (one phase-B step)
constexpr int kWideMaxTaps = 49;   // a 7x7 window

struct WideArgs {
  const void* x;
  const void* off;
  const void* mask;
  void* out;
  unsigned int* error_word;
  TiledParams t;
  int K, KK;
  int kc;      // window position a*K + b left out by remove_center, else -1
  int CH;      // taps per chunk
  int rec;     // byte offset of the chunk records in a warp region
  FastDiv fd_K;
};

// Region bytes of the staged offsets and mask of one batch, and the size of a
// chunk's records (W[CH][8] float4, OFF[CH][8]).
__host__ __device__ constexpr int wide_stage_bytes(int KK, int pair_bytes) {
  return (kWideUnits * KK * pair_bytes + 15) / 16 * 16 + kWideUnits * KK * 4;
}
__host__ __device__ constexpr int wide_rec_bytes(int CH) { return CH * kWideUnits * 20; }

// Asynchronous 4- or 8-byte global -> shared copy; zero fill when !ok (no
// bytes are read then).
template <int BYTES>
__device__ __forceinline__ void cp_async_pred(uint32_t dst, const void* src, bool ok) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src), "n"(BYTES),
               "r"(ok ? BYTES : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

template <typename T, bool SOFTMAX, bool FAR>
__global__ void __launch_bounds__(kTiledThreads, 1)
    dcn_forward_tiled_wide_kernel(const __grid_constant__ CUtensorMap xmap, const WideArgs a) {
  using IO = TiledIO<T>;
  using Pair = typename IO::Pair;
  constexpr int CS = 16 * int(sizeof(T));  // bytes of one pixel of the group
  constexpr int NP = CS / 16;              // 16-byte pieces per corner

  const TiledParams& t = a.t;
  const int KK = a.KK;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int nbuf = t.nbuf;
  unsigned char* const bufs = smem;
  unsigned char* const zero = smem + size_t(nbuf) * t.box_stride;
  unsigned char* const regions = zero + zero_band_bytes(t.BW, CS);
  uint64_t* const full = reinterpret_cast<uint64_t*>(regions + size_t(kTiledWarps) * kFwdRegion);
  uint64_t* const empty = full + kTiledMaxBufs;
  int* const s_abort = reinterpret_cast<int*>(empty + kTiledMaxBufs);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < nbuf; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kTiledWarps);
    }
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < zero_band_bytes(t.BW, CS) / 16; i += kTiledThreads)
    reinterpret_cast<uint4*>(zero)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  volatile int* abort_flag = s_abort;

  // ---- producer warp: one TMA box per item, nbuf buffers in flight ----
  if (warp == kTiledWarps) {
    if (lane != 0) return;
    int i = 0, b = 0;
    uint32_t ph = 0;
    for (;; ++i) {
      const int item = int(blockIdx.x) + i * int(gridDim.x);
      if (item >= t.items || *abort_flag) break;
      if (i >= nbuf && !mbar_wait_bounded_sleep(&empty[b], ph ^ 1u)) {
        atomicOr(a.error_word, kErrTimeout);
        *abort_flag = 1;
        break;
      }
      const ItemCoord c = item_coord(t, item);
      if (!(t.inject_stall && i == 0)) {
        const int Y0 = box_origin(c.ho0 * t.stride - t.pad - t.halo, t.BH, t.H, t.clamp_box);
        const int X0 = box_origin(c.wo0 * t.stride_w - t.pad_w - t.halo, t.BW, t.W, t.clamp_box);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[b], t.box_bytes);
        tma_load_box(bufs + size_t(b) * t.box_stride, &xmap, &full[b], c.g * t.Cg, X0, Y0, c.n);
      }
      if (++b == nbuf) {
        b = 0;
        ph ^= 1u;
      }
    }
    for (int j = i - nbuf < 0 ? 0 : i - nbuf; j < i; ++j)
      if (!(t.inject_stall && j == 0))
        (void)mbar_wait_bounded(&full[j % nbuf], uint32_t(j / nbuf) & 1u);
    return;
  }

  // ---- consumer warps ----
  unsigned char* const reg = regions + size_t(warp) * kFwdRegion;
  const uint32_t reg_a = smem_addr(reg);
  const uint32_t zero_a = smem_addr(zero);
  Pair* const st_off = reinterpret_cast<Pair*>(reg);  // [unit][tap]
  float* const st_msk =
      reinterpret_cast<float*>(reg + (kWideUnits * KK * int(sizeof(Pair)) + 15) / 16 * 16);
  const uint32_t rec_w = reg_a + uint32_t(a.rec);                         // W[c][u] float4
  const uint32_t rec_off = rec_w + uint32_t(a.CH * kWideUnits * 16);     // OFF[c][u]
  // lanes: unit u8 of the batch; r = bilinear corner (dy, dx) in phase B and
  // the tap residue in phase A
  const int u8 = lane >> 2, r = lane & 3, dy = r >> 1, dx = r & 1, rho = u8 & 1;
  const int rot = NP == 2 ? rho : 2 * dy + rho;
  const uint32_t corner_b = uint32_t((dy * t.BW + dx) * CS + 16 * rot);
  const int npx = t.TH * t.TW;
  const int nb = t.batches;
  const float Hf = float(t.H), Wf = float(t.W);
  const size_t pixB = size_t(t.C) * sizeof(T);
  const size_t x_bytes = size_t(t.N) * t.H * t.W * pixB;  // bounds-checked build
  const size_t out_bytes = size_t(t.N) * t.Ho * t.Wo * pixB;
  const size_t n_entries = size_t(t.N) * t.Ho * t.Wo * t.G * KK;

  const int n_items_cta =
      int(blockIdx.x) < t.items ? (t.items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int total_batches = n_items_cta * nb;

  // Unit of this lane in batch bb (over all the CTA's items): its pixel and,
  // if it lies in the output, the element index of its first offset pair.
  struct BatchUnit {
    int ho, wo;
    bool valid;
    uint32_t q;
  };
  auto batch_unit = [&](int bb) {
    const int il = bb / nb;
    const ItemCoord ic = item_coord(t, int(blockIdx.x) + il * int(gridDim.x));
    const int v = (bb - il * nb) * kWideUnits + u8;
    const int rr = int(fdiv(uint32_t(v), t.fd_TW));
    BatchUnit bu;
    bu.ho = ic.ho0 + rr;
    bu.wo = ic.wo0 + (v - rr * t.TW);
    bu.valid = (v < npx) && (bu.ho < t.Ho) && (bu.wo < t.Wo);
    bu.q = bu.valid ? (uint32_t((ic.n * t.Ho + bu.ho) * t.Wo + bu.wo) * uint32_t(t.G) +
                       uint32_t(ic.g)) * uint32_t(KK)
                    : ~0u;
    return bu;
  };
  // Staging of batch bb into the region, issued early: the offset pairs (and
  // fp32 mask values) by cp.async; 2-byte mask values through registers,
  // written when the batch starts (cp.async copies 4 bytes at least).
  constexpr bool kMaskRegs = sizeof(T) == 2;
  uint32_t pm[kWideUnits][2];
  auto stage_issue = [&](int bb) {
    const uint32_t qq = batch_unit(bb).q;
#pragma unroll
    for (int uu = 0; uu < kWideUnits; ++uu) {
      const uint32_t src = __shfl_sync(0xFFFFFFFFu, qq, uu * 4);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int e = lane + 32 * i;
        if (e < KK) {
          const bool ok = src != ~0u && in_range(size_t(src) + e, n_entries);
          const size_t idx = ok ? size_t(src) + e : 0;
          cp_async_pred<int(sizeof(Pair))>(smem_addr(st_off + uu * KK + e),
                                          static_cast<const Pair*>(a.off) + idx, ok);
          if constexpr (kMaskRegs)
            pm[uu][i] = ok ? uint32_t(IO::ld_one(a.mask, idx)) : 0u;
          else
            cp_async_pred<4>(smem_addr(st_msk + uu * KK + e), static_cast<const float*>(a.mask) + idx,
                             ok);
        }
      }
    }
    cp_async_commit();
  };
  auto stage_finish = [&]() {
    cp_async_wait_all();
    if constexpr (kMaskRegs) {
#pragma unroll
      for (int uu = 0; uu < kWideUnits; ++uu)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int e = lane + 32 * i;
          if (e < KK) st_msk[uu * KK + e] = IO::one(typename IO::One(pm[uu][i]));
        }
    }
    __syncwarp();
  };

  int beta = warp;
  if (beta < total_batches) stage_issue(beta);
  int b = 0;
  uint32_t ph = 0;
  for (int il = 0; il < n_items_cta; ++il) {
    // Every consumer warp observes every item's box (see the 3x3 kernel).
    if (!mbar_wait_bounded_sleep(&full[b], ph)) {
      atomicOr(a.error_word, kErrTimeout);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const ItemCoord c = item_coord(t, int(blockIdx.x) + il * int(gridDim.x));
    const unsigned char* const box = bufs + size_t(b) * t.box_stride;
    const uint32_t box_a = smem_addr(box);
    const uint32_t lane_base = box_a + corner_b;
    const uint32_t zoff = zero_a - box_a;
    const int Y0 = box_origin(c.ho0 * t.stride - t.pad - t.halo, t.BH, t.H, t.clamp_box);
    const int X0 = box_origin(c.wo0 * t.stride_w - t.pad_w - t.halo, t.BW, t.W, t.clamp_box);
    const char* const ximg = reinterpret_cast<const char*>(a.x) +
                             size_t(c.n) * t.H * t.W * pixB + size_t(c.g) * CS;

    for (; beta < (il + 1) * nb; beta += kTiledWarps) {
      const BatchUnit bu = batch_unit(beta);
      const int ho = bu.ho, wo = bu.wo;
      const bool valid = bu.valid;
      stage_finish();  // this batch's offsets and mask are in the region

      // Softmax over this lane's unit: its four lanes take every fourth tap;
      // exp(l - max) replaces the staged logit.
      float inv = 1.f;
      if (SOFTMAX) {
        float mx = -INFINITY;
        for (int k = r; k < KK; k += 4) mx = fmaxf(mx, st_msk[u8 * KK + k]);
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
        float sum = 0.f;
        for (int k = r; k < KK; k += 4) {
          const float ex = expf(st_msk[u8 * KK + k] - mx);
          st_msk[u8 * KK + k] = ex;
          sum += ex;
        }
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
        inv = 1.0f / sum;
        __syncwarp();  // phase A reads taps another lane of the unit wrote
      }
      const int yb = ho * t.stride - t.pad, xb = wo * t.stride_w - t.pad_w;

      float2 acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = make_float2(0.f, 0.f);

#pragma unroll 1
      for (int k0 = 0; k0 < KK; k0 += a.CH) {
        const int ch = min(a.CH, KK - k0);
        // Phase A: lane r builds the records of the chunk's taps r, r + 4, ...
        uint32_t fm = 0u;
#pragma unroll 1
        for (int cc = r; cc < ch; cc += 4) {
          const int k = k0 + cc;
          const int pos = (a.kc >= 0 && k >= a.kc) ? k + 1 : k;
          const int ka = int(fdiv(uint32_t(pos), a.fd_K)), kb = pos - ka * a.K;
          const float2 d = IO::pair(st_off[u8 * KK + k]);
          const float m = SOFTMAX ? st_msk[u8 * KK + k] * inv : st_msk[u8 * KK + k];
          const float Y = tap_coord(yb + ka * t.dil, t.sigma, d.y);
          const float X = tap_coord(xb + kb * t.dil_w, t.sigma, d.x);
          const float fy = floorf(Y), fx = floorf(X);
          const int y0 = __float2int_rd(Y), x0 = __float2int_rd(X);
          const float ly = Y - fy, lx = X - fx;
          const int by = y0 - Y0, bx = x0 - X0;
          const bool inbox = unsigned(by) < unsigned(t.BH - 1) && unsigned(bx) < unsigned(t.BW - 1);
          const bool box_tap = valid && inbox && (Y == Y) && (X == X);
          const bool far = FAR && !box_tap && valid && (Y >= -1.0f) && (Y < Hf) &&
                           (X >= -1.0f) && (X < Wf);
          const float hy = 1.f - ly, hx = 1.f - lx;
          const float wy0 = hy * m, wy1 = ly * m;
          float4 w;
          if (box_tap)
            w = make_float4(wy0 * hx, wy0 * lx, wy1 * hx, wy1 * lx);
          else if (far)
            w = make_float4(wy0, wy1, lx,
                            __uint_as_float((uint32_t(y0 + 1) << kFarShift) | uint32_t(x0 + 1)));
          else
            w = make_float4(0.f, 0.f, 0.f, 0.f);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(
                           rec_w + uint32_t(cc * kWideUnits + u8) * 16u),
                       "f"(w.x), "f"(w.y), "f"(w.z), "f"(w.w)
                       : "memory");
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(rec_off + uint32_t(cc * kWideUnits + u8) * 4u),
                       "r"(box_tap ? uint32_t((by * t.BW + bx) * CS) : zoff)
                       : "memory");
          fm |= far ? (1u << cc) : 0u;
        }
        // the unit's far taps of this chunk, on all four of its lanes
        fm |= __shfl_xor_sync(0xFFFFFFFFu, fm, 1);
        fm |= __shfl_xor_sync(0xFFFFFFFFu, fm, 2);
        __syncwarp();
        // After the last chunk's phase A the staging area is free: the next
        // batch's copies overlap this chunk's phase B, far taps and stores.
        if (k0 + a.CH >= KK && beta + kTiledWarps < total_batches) stage_issue(beta + kTiledWarps);

        // Phase B: lane = corner, the chunk's taps from the box.
        const uint32_t wa = rec_w + uint32_t(u8) * 16u + uint32_t(r) * 4u;
        const uint32_t oa = rec_off + uint32_t(u8) * 4u;
#pragma unroll 4
        for (int cc = 0; cc < ch; ++cc) {
          float w;
          uint32_t off;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(w) : "r"(wa + uint32_t(cc * kWideUnits) * 16u));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(off) : "r"(oa + uint32_t(cc * kWideUnits) * 4u));
          const float2 w2 = make_float2(w, w);
          const uint32_t a0 = lane_base + off;
#pragma unroll
          for (int j = 0; j < NP; ++j)
            IO::fma16(acc + j * (8 / NP), w2, lds128_a(a0 ^ uint32_t(16 * j)));
        }
        // The chunk's far taps: this lane's corner from global memory.
        if (FAR) {
          while (__any_sync(0xFFFFFFFFu, fm != 0u)) {
            if (fm != 0u) {
              const int cc = __ffs(fm) - 1;
              const uint4 rw = lds128_a(rec_w + uint32_t(cc * kWideUnits + u8) * 16u);
              const uint32_t pk = rw.w;
              const int yc = int(pk >> kFarShift) - 1 + dy;
              const int xc = int(pk & ((1u << kFarShift) - 1u)) - 1 + dx;
              const bool in = unsigned(yc) < unsigned(t.H) && unsigned(xc) < unsigned(t.W);
              const float flx = __uint_as_float(rw.z);
              const float fw = in ? __uint_as_float(dy ? rw.y : rw.x) * (dx ? flx : 1.f - flx) : 0.f;
              const char* gp = ximg + (size_t(in ? yc : 0) * t.W + (in ? xc : 0)) * pixB;
#pragma unroll
              for (int j = 0; j < NP; ++j) {
                const char* pp = gp + 16 * (j ^ rot);
                IO::fma16(acc + j * (8 / NP), make_float2(fw, fw),
                          ldg128_pred(pp, in && in_tensor(pp, 16, a.x, x_bytes)));
              }
              fm &= fm - 1u;
            }
          }
        }
        __syncwarp();  // the next chunk rewrites the records
      }

      // Reduce-scatter over the unit's four corner lanes, then store.
      const uint32_t ob =
          valid ? uint32_t(((c.n * t.Ho + ho) * t.Wo + wo) * t.C + c.g * t.Cg) : ~0u;
      if constexpr (NP == 2) {
        float2 k4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 keep = dx ? acc[4 + i] : acc[i];
          const float2 send = dx ? acc[i] : acc[4 + i];
          k4[i].x = keep.x + __shfl_xor_sync(0xFFFFFFFFu, send.x, 1);
          k4[i].y = keep.y + __shfl_xor_sync(0xFFFFFFFFu, send.y, 1);
        }
        float2 k2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float2 keep = dy ? k4[2 + i] : k4[i];
          const float2 send = dy ? k4[i] : k4[2 + i];
          k2[i].x = keep.x + __shfl_xor_sync(0xFFFFFFFFu, send.x, 2);
          k2[i].y = keep.y + __shfl_xor_sync(0xFFFFFFFFu, send.y, 2);
        }
        if (ob != ~0u) {
          char* op = reinterpret_cast<char*>(a.out) +
                     (size_t(ob) + size_t(8 * (rho ^ dx) + 4 * dy)) * sizeof(T);
          if (in_tensor(op, 8, a.out, out_bytes))
            asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(op),
                         "r"(pack2<T>(k2[0].x, k2[0].y)), "r"(pack2<T>(k2[1].x, k2[1].y))
                         : "memory");
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i].x += __shfl_xor_sync(0xFFFFFFFFu, acc[4 + i].x, 2);
          acc[i].y += __shfl_xor_sync(0xFFFFFFFFu, acc[4 + i].y, 2);
        }
        float2 k2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float2 keep = dx ? acc[2 + i] : acc[i];
          const float2 send = dx ? acc[i] : acc[2 + i];
          k2[i].x = keep.x + __shfl_xor_sync(0xFFFFFFFFu, send.x, 1);
          k2[i].y = keep.y + __shfl_xor_sync(0xFFFFFFFFu, send.y, 1);
        }
        if (ob != ~0u) {
          char* op = reinterpret_cast<char*>(a.out) + (size_t(ob) + size_t(4 * (dx ^ rot))) * sizeof(T);
          if (in_tensor(op, 16, a.out, out_bytes))
            asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(op), "f"(k2[0].x),
                         "f"(k2[0].y), "f"(k2[1].x), "f"(k2[1].y)
                         : "memory");
        }
      }
      __syncwarp();  // the next batch rewrites the staging area
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);
    if (++b == nbuf) {
      b = 0;
      ph ^= 1u;
    }
  }
  cp_async_wait_all();  // (after an abort a batch's copies may still be landing)
}

}  // namespace dcn
