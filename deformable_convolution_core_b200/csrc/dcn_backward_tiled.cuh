// Backward kernel with the input staged in shared memory by TMA (sm_100a).
//
// Same gradients as dcn_backward_kernel (InternImage-L DCNv3 explainer
// (wmrh.cn), section 二 steps 2-4, differentiated; the DCNv3 extension build
// guide (trdm.cn), section 2.1, names the backward device code this
// replaces): per unit (pixel, group) and tap k, with d_c = <g, x[corner c]>
// over the group's channels and g the unit's upstream gradient,
//   s_k = sum_c w_c d_c,  grad (dx, dy)_k = offset_scale * m_k * (<g, dv/dX>, <g, dv/dY>),
//   grad logit_k = m_k (s_k - sum_j m_j s_j)  (raw mask: s_k),
//   grad x[corner c] += m_k w_c g            (float4 reductions).
//
// What changes is where the corners come from.  The direct kernel gathers
// them through L1 and L2 next to its grad_input reductions; both compete for
// the same L1 wavefronts and L2 bandwidth.  Here the work items, the TMA box,
// the producer warp and the bounded mbarrier protocol are those of
// dcn_forward_tiled_kernel: a persistent CTA walks (image, output tile,
// group) items and reads the footprints from the group's input box in shared
// memory.  Phase A (one lane per unit) computes the softmax and, per tap, a
// record: where corner (y0, x0) sits in the box (or that the corners must be
// read from global memory), its element offset in the image for the
// reductions, which corners lie in the image, and the fractional parts.
// Phase B gives each unit four lanes of four channels: a lane loads its piece
// of each corner, forms its partial dot products and issues its float4
// reduction, so one warp instruction still covers a unit's whole 64-byte
// corner chunk of grad_input.
#pragma once

#include "dcn_backward.cuh"
#include "dcn_forward_tiled.cuh"

namespace dcn {

struct TiledBwdArgs {
  const void* x;
  const void* off;
  const void* mask;
  const void* gout;
  void* gx;  // grad_input accumulator (fp32, or 64-bit fixed point), zero-filled first
  void* goff;
  void* gmask;
  const unsigned int* det_hdr;  // deterministic backward: the pre-pass bounds
  int det_cbits;
  unsigned int* error_word;
  TiledParams t;
};

// Unit slot of the backward (kSlotBytes, 8-byte aligned): tap k's record at 16*k holds
// {code, element offset of corner (y0, x0) in the image, lx, ly}; the mask
// weights m_k follow at kBwdMaskAt.  code bit 31: the corners are read from
// global memory; bits 24-27: corners (0,0), (0,1), (1,0), (1,1) lie in the
// image (all clear for a sample that contributes nothing); bits 0-23: byte
// offset of corner (y0, x0) in the box.
constexpr int kBwdMaskAt = kTiledMaxTaps * 16;
static_assert(kBwdMaskAt + kTiledMaxTaps * 4 <= kSlotBytes, "backward slot layout");
constexpr uint32_t kBwdFar = 0x80000000u;

// A lane's four channels of one corner through a generic address (the box in
// shared memory or the input in global memory); zeros unless `pred`, and a
// false predicate issues no access.
template <typename T>
struct BwdPiece;
template <>
struct BwdPiece<float> {
  __device__ __forceinline__ static void load(const void* p, bool pred, float (&v)[4]) {
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
        " mov.b32 %0, 0;\n mov.b32 %1, 0;\n mov.b32 %2, 0;\n mov.b32 %3, 0;\n"
        " @q ld.v4.f32 {%0, %1, %2, %3}, [%4];\n}"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
        : "l"(p), "r"(int(pred))
        : "memory");
  }
};
// The same four channels from the box in shared memory (always in bounds).
template <typename T>
struct BoxPiece;
template <>
struct BoxPiece<float> {
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
                 : "r"(smem_addr(p)));
  }
};
template <>
struct BoxPiece<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    uint32_t w0, w1;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w0), "=r"(w1) : "r"(smem_addr(p)));
    v[0] = bf16lo_to_f32(w0);
    v[1] = bf16hi_to_f32(w0);
    v[2] = bf16lo_to_f32(w1);
    v[3] = bf16hi_to_f32(w1);
  }
};
template <>
struct BwdPiece<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const void* p, bool pred, float (&v)[4]) {
    uint32_t w0, w1;
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %3, 0;\n mov.b32 %0, 0;\n mov.b32 %1, 0;\n"
        " @q ld.v2.b32 {%0, %1}, [%2];\n}"
        : "=r"(w0), "=r"(w1)
        : "l"(p), "r"(int(pred))
        : "memory");
    v[0] = bf16lo_to_f32(w0);
    v[1] = bf16hi_to_f32(w0);
    v[2] = bf16lo_to_f32(w1);
    v[3] = bf16hi_to_f32(w1);
  }
};

// KKS: 9 (the 3x3 window) or 8 (the window without its centre).  CS = the
// group's bytes per pixel = 16 channels.  DET: exact fixed-point accumulation
// of grad_input (GxScatter).
template <typename T, int CS, int KKS, bool SOFTMAX, bool DET>
__global__ void __launch_bounds__(kTiledThreads, 1)
    dcn_backward_tiled_kernel(const __grid_constant__ CUtensorMap xmap, const TiledBwdArgs a) {
  using IO = TiledIO<T>;
  using Pair = typename IO::Pair;
  using One = typename IO::One;
  constexpr int KK = KKS, K = tap_side(KKS);
  static_assert(K == 3 && KK <= kTiledMaxTaps, "the tiled kernel serves 3x3 tap sets");
  static_assert(CS == 16 * int(sizeof(T)), "16 channels per group");
  constexpr int LU = 4;          // phase-B lanes per unit, four channels each
  constexpr int UPW = 32 / LU;   // units per phase-B step
  constexpr int PB = 4 * int(sizeof(T));  // bytes of a lane's piece of one corner
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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&empty[0], kTiledWarps);
    mbar_init(&empty[1], kTiledWarps);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
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
  const int ul = lane / LU;  // phase B: unit of this lane within a step
  const int sub = lane - ul * LU;
  const unsigned umask = 0xFu << (ul * LU);
  const int pixE = t.C;            // elements between horizontally adjacent pixels
  const int rowE = t.W * t.C;      // ... vertically adjacent pixels
  const int cofs[4] = {0, pixE, rowE, rowE + pixE};  // corner (dy, dx) from corner (0, 0)
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
  const size_t n_taps = size_t(t.N) * t.Ho * t.Wo * t.G * KK;  // offset pairs, mask values
  const size_t n_img = size_t(t.N) * t.H * t.W * t.C;           // input, accumulator elements
  const size_t n_out = size_t(t.N) * t.Ho * t.Wo * t.C;
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
      if (src != ~0ull && in_range(size_t(src) + st_tap[k], n_taps)) {
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
    // Every consumer warp observes every item's box (see the forward kernel).
    if (!mbar_wait_bounded(&full[b], (il >> 1) & 1)) {
      atomicOr(a.error_word, 1u);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const ItemCoord c = item_coord(t, item);
    const unsigned char* box_lane = bufs + size_t(b) * t.box_stride + sub * PB;
    const int Y0 = c.ho0 * t.stride - t.pad - t.halo;
    const int X0 = c.wo0 * t.stride_w - t.pad_w - t.halo;
    const size_t img = size_t(c.n) * t.H * t.W * t.C + size_t(c.g) * t.Cg + size_t(sub) * 4;
    const char* xg = reinterpret_cast<const char*>(a.x) + img * sizeof(T);
    const GxScatter<DET> gxs(a.gx, a.det_hdr, SOFTMAX, a.det_cbits, n_img);
    typename GxScatter<DET>::Acc* const gx_item = gxs.p + img;

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

      // Phase A: this lane's unit -> mask weights and the tap records.
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
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const int q = tap_pos(KK, k);
          const float Y = tap_coord(ho * t.stride - t.pad + (q / K) * t.dil, t.sigma, d[k].y);
          const float X =
              tap_coord(wo * t.stride_w - t.pad_w + (q % K) * t.dil_w, t.sigma, d[k].x);
          const Footprint f = footprint(Y, X, t.H, t.W);
          const bool live = valid && f.in_support;
          // a sample that contributes nothing keeps code 0: box offset 0, no corner
          uint32_t code = 0;
          int ce = 0;
          if (live) {
            code = (uint32_t(f.v00) | uint32_t(f.v01) << 1 | uint32_t(f.v10) << 2 |
                    uint32_t(f.v11) << 3)
                   << 24;
            const int by = f.y0 - Y0, bx = f.x0 - X0;
            if (by >= 0 && by + 1 < t.BH && bx >= 0 && bx + 1 < t.BW)
              code |= uint32_t((by * t.BW + bx) * CS);
            else
              code |= kBwdFar;
            ce = f.y0 * rowE + f.x0 * pixE;
          }
          // slots are 8-byte aligned (184-byte stride): two 8-byte stores
          reinterpret_cast<uint2*>(sl + 16 * k)[0] = make_uint2(code, uint32_t(ce));
          reinterpret_cast<uint2*>(sl + 16 * k)[1] =
              make_uint2(__float_as_uint(f.lx), __float_as_uint(f.ly));
          reinterpret_cast<float*>(sl + kBwdMaskAt)[k] = m[k];
        }
      }
      __syncwarp();
      // The next batch's inputs are loaded while this one is processed.
      if (beta + kTiledWarps < total_batches) prefetch(beta + kTiledWarps);

      // Phase B: UPW units per step, LU lanes of four channels each.
      const int v0 = (beta - il * nb) * kTiledBatch;
#pragma unroll 1
      for (int s = 0; s < kTiledBatch / UPW; ++s) {
        const int u = s * UPW + ul;
        const unsigned char* sl = myslots + u * kSlotBytes;
        const int v = v0 + u;
        const int rr = int(fdiv(uint32_t(v), t.fd_TW));
        const int uho = c.ho0 + rr, uwo = c.wo0 + (v - rr * t.TW);
        const bool uvalid = v < npx && uho < t.Ho && uwo < t.Wo;
        const size_t pix = size_t(c.n * t.Ho + uho) * t.Wo + uwo;
        const size_t unit = pix * t.G + c.g;
        // grad_offset pairs of this unit, written by its first lane without a branch
        char* const goff_u = reinterpret_cast<char*>(a.goff) + unit * KK * sizeof(Pair);
        const uint32_t st_ok = (sub == 0 && uvalid) ? 1u : 0u;
        float go[4];
        Quad<T>::load_pred(reinterpret_cast<const char*>(a.gout) +
                               (pix * t.C + size_t(c.g) * t.Cg + size_t(sub) * 4) * sizeof(T),
                           uvalid && in_range(pix * t.C + size_t(c.g) * t.Cg + size_t(sub) * 4 + 3,
                                              n_out),
                           go);
        const float2 g01 = make_float2(go[0], go[1]), g23 = make_float2(go[2], go[3]);
        float sk[KK];
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const uint2 r0 = reinterpret_cast<const uint2*>(sl + 16 * k)[0];
          const uint2 r1 = reinterpret_cast<const uint2*>(sl + 16 * k)[1];
          const float mk = reinterpret_cast<const float*>(sl + kBwdMaskAt)[k];
          const uint32_t code = r0.x;
          const int ce = int(r0.y);
          const float lx = __uint_as_float(r1.x), ly = __uint_as_float(r1.y);
          const bool far = (code & kBwdFar) != 0u;
          const unsigned char* bp = box_lane + (code & 0xFFFFFFu);
          const float hy = 1.f - ly, hx = 1.f - lx;
          const float cw[4] = {hy * hx, hy * lx, ly * hx, ly * lx};
          float cv[4][4];
          if (__any_sync(0xFFFFFFFFu, far)) {
            // some footprint of this step lies outside the box: box or global
            // memory per lane through a generic address, predicated per corner
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int dy = cc >> 1, dx = cc & 1;
              const bool in = ((code >> (24 + cc)) & 1u) != 0u;
              const int e = ce + dy * rowE + dx * pixE;
              const void* src =
                  far ? static_cast<const void*>(xg + ptrdiff_t(e) * ptrdiff_t(sizeof(T)))
                      : static_cast<const void*>(bp + (dy * t.BW + dx) * CS);
              BwdPiece<T>::load(src,
                                in && (!far || in_range(img + size_t(e) + 3, n_img)), cv[cc]);
            }
          } else {
            // every footprint is in the box: plain shared loads (corners outside
            // the image read the box's zero fill, and dc is masked below anyway)
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              BoxPiece<T>::load(bp + ((cc >> 1) * t.BW + (cc & 1)) * CS, cv[cc]);
          }
          float dc[4];
          auto* const p00 = gx_item + ce;  // accumulator at corner (y0, x0)
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint32_t inb = code & (1u << (24 + cc));  // corner in the image
            float2 pd = __fmul2_rn(make_float2(cv[cc][0], cv[cc][1]), g01);
            pd = __ffma2_rn(make_float2(cv[cc][2], cv[cc][3]), g23, pd);
            dc[cc] = inb ? pd.x + pd.y : 0.f;
            const float wv = mk * cw[cc];
            const float2 w2 = make_float2(wv, wv);
            gxs.add_at(p00 + cofs[cc], kCheckBounds ? img + size_t(ce + cofs[cc]) : 0,
                       __fmul2_rn(w2, g01), __fmul2_rn(w2, g23), inb);
          }
          // a sample that contributes nothing has no corner in the image: every dc is 0
          float sv = cw[0] * dc[0] + cw[1] * dc[1] + cw[2] * dc[2] + cw[3] * dc[3];
          float gX = hy * (dc[1] - dc[0]) + ly * (dc[3] - dc[2]);
          float gY = hx * (dc[2] - dc[0]) + lx * (dc[3] - dc[1]);
          sv = unit_sum<LU>(sv, umask);
          gX = unit_sum<LU>(gX, umask);
          gY = unit_sum<LU>(gY, umask);
          sk[k] = sv;
          const float sc = t.sigma * mk;
          Quad<T>::store_pair_pred(goff_u + k * sizeof(Pair), sc * gX, sc * gY,
                                   (st_ok != 0u && in_range(unit * KK + k, n_taps)) ? 1u : 0u);
        }
        if (sub == 0 && uvalid) {
          const float* ms_ = reinterpret_cast<const float*>(sl + kBwdMaskAt);
          float msum = 0.f;
          if (SOFTMAX) {
#pragma unroll
            for (int k = 0; k < KK; ++k) msum = fmaf(ms_[k], sk[k], msum);
          }
#pragma unroll
          for (int k = 0; k < KK; ++k)
            if (in_range(unit * KK + k, n_taps)) Quad<T>::store_one(a.gmask, unit * KK + k,
                               SOFTMAX ? ms_[k] * (sk[k] - msum) : sk[k]);
        }
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
