// Backward kernel with the input staged in shared memory by TMA (sm_100a).
//
// Same gradients as dcn_backward_kernel (InternImage-L DCNv3 explainer
// (wmrh.cn), section 二 steps 2-4, differentiated; the DCNv3 extension build
// guide (trdm.cn), section 2.1, names the backward device code this
// replaces): per unit (pixel, group) and tap k, with d_c = <g, x[corner c]>
// over the group's 16 channels and g the unit's upstream gradient,
//   s_k = sum_c b_c d_c,  grad (dx, dy)_k = offset_scale * m_k * (<g, dv/dX>, <g, dv/dY>),
//   <g, dv/dX> = hy (d01 - d00) + ly (d11 - d10),  <g, dv/dY> = hx (d10 - d00) + lx (d11 - d01),
//   grad logit_k = m_k (s_k - sum_j m_j s_j)  (raw mask: s_k),
//   grad x[corner c] += m_k b_c g            (16-byte vector reductions),
// b_c the bilinear weights.
//
// The work items, boxes, zero band, staging and phase A follow
// dcn_forward_tiled_kernel (clamped boxes, nbuf in flight, structures of
// arrays).  Phase A stores per tap {ly, lx, m_k, box offset | in-image bits}
// and the image offset of corner (y0, x0).  Phase B gives each unit four
// lanes, one per bilinear corner: a lane reads its corner's 16 channels from
// the box (conflict-free, as in the forward) with the unit's upstream gradient
// loaded in the same piece order, so d_c is one in-lane dot product; three
// shuffles bring the four d_c to the unit's first lane, which forms s_k and the
// offset gradient.  Every lane then scatters its four channels of m_k b_c g
// into each corner, so one warp instruction covers a corner's whole 64-byte
// chunk of eight units.  A far tap (footprint outside the box) reads its
// corner from global memory instead.
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

// Per-warp region of the backward: R[9][32] float4 {ly, lx, m, box offset |
// in-image bits << 24} (bit 24 + c: corner c = (dy, dx) = (c >> 1, c & 1) lies
// in the image; all clear for a tap that contributes nothing), CE[9][32] (element offset of corner (y0, x0) from the
// image's group base), FM[32] (far taps), PIX[32] (output pixel, ~0 outside).
// The same size as the forward's region; the staged inputs alias it.
constexpr int kBwdRegR = 0;
constexpr int kBwdRegCe = kTiledMaxTaps * kTiledBatch * 16;
constexpr int kBwdRegFm = kBwdRegCe + kTiledMaxTaps * kTiledBatch * 4;
constexpr int kBwdRegPix = kBwdRegFm + kTiledBatch * 4;
static_assert(kBwdRegPix + kTiledBatch * 4 == kFwdRegion, "backward region = forward region");
constexpr uint32_t kBwdOffMask = 0xFFFFFFu;  // box offset bits of R.w (in-image bits above)

// Four channels of the upstream gradient (fp32) from storage type T.
template <typename T>
struct BwdIO;
template <>
struct BwdIO<float> {
  // 16 bytes = 4 channels; zeros unless pred
  __device__ __forceinline__ static void quad(const char* p, bool pred, float2& lo, float2& hi) {
    float v[4];
    Quad<float>::load_pred(p, pred, v);
    lo = make_float2(v[0], v[1]);
    hi = make_float2(v[2], v[3]);
  }
};
template <>
struct BwdIO<__nv_bfloat16> {
  __device__ __forceinline__ static void quad(const char* p, bool pred, float2& lo, float2& hi) {
    float v[4];
    Quad<__nv_bfloat16>::load_pred(p, pred, v);
    lo = make_float2(v[0], v[1]);
    hi = make_float2(v[2], v[3]);
  }
};

template <>
struct BwdIO<__half> {
  __device__ __forceinline__ static void quad(const char* p, bool pred, float2& lo, float2& hi) {
    float v[4];
    Quad<__half>::load_pred(p, pred, v);
    lo = make_float2(v[0], v[1]);
    hi = make_float2(v[2], v[3]);
  }
};

// Dot product of a 16-byte piece (storage type T) with the matching gradient
// channels, in the canonical order of quarter_dot: the sum of the piece's
// quarters (one for fp32, two for 2-byte types, added pairwise).
template <typename T>
__device__ __forceinline__ float piece_dot(const uint4& v, const float2* g);
template <>
__device__ __forceinline__ float piece_dot<float>(const uint4& v, const float2* g) {
  return quarter_dot(make_float2(__uint_as_float(v.x), __uint_as_float(v.y)),
                     make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), g[0], g[1]);
}
template <>
__device__ __forceinline__ float piece_dot<__nv_bfloat16>(const uint4& v, const float2* g) {
  const float q0 = quarter_dot(make_float2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x)),
                               make_float2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y)), g[0], g[1]);
  const float q1 = quarter_dot(make_float2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z)),
                               make_float2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w)), g[2], g[3]);
  return __fadd_rn(q0, q1);
}

template <>
__device__ __forceinline__ float piece_dot<__half>(const uint4& v, const float2* g) {
  const float q0 = quarter_dot(f16x2_to_f32x2(v.x), f16x2_to_f32x2(v.y), g[0], g[1]);
  const float q1 = quarter_dot(f16x2_to_f32x2(v.z), f16x2_to_f32x2(v.w), g[2], g[3]);
  return __fadd_rn(q0, q1);
}

// 2-byte storage: a corner channel and its upstream-gradient channel are both
// 16-bit values, so their product is exact in fp32.  sm_100a's mixed-precision
// FMA (16-bit multiplicands, fp32 addend and result, one rounding) therefore
// gives quarter_dot's bits on the raw words, without widening either operand.
// The first product of each pair is formed with a -0 addend, which leaves
// every product unchanged, including the sign of a zero.
template <typename T>
__device__ __forceinline__ float quarter_dot16(uint32_t x01, uint32_t x23, uint32_t g01,
                                               uint32_t g23);
#define DCN_QUARTER_DOT16(TYPE, SUFFIX)                                                       \
  template <>                                                                                 \
  __device__ __forceinline__ float quarter_dot16<TYPE>(uint32_t x01, uint32_t x23,           \
                                                       uint32_t g01, uint32_t g23) {         \
    float p0, p1;                                                                             \
    asm("{\n .reg .b16 a0, a1, a2, a3, b0, b1, b2, b3;\n .reg .f32 t0, t1;\n"                  \
        " mov.b32 {a0, a1}, %2;\n mov.b32 {a2, a3}, %3;\n"                                     \
        " mov.b32 {b0, b1}, %4;\n mov.b32 {b2, b3}, %5;\n"                                     \
        " fma.rn.f32." SUFFIX " t0, a0, b0, 0f80000000;\n"                                      \
        " fma.rn.f32." SUFFIX " t1, a1, b1, 0f80000000;\n"                                      \
        " fma.rn.f32." SUFFIX " %0, a2, b2, t0;\n"                                              \
        " fma.rn.f32." SUFFIX " %1, a3, b3, t1;\n}"                                             \
        : "=f"(p0), "=f"(p1)                                                                  \
        : "r"(x01), "r"(x23), "r"(g01), "r"(g23));                                            \
    return __fadd_rn(p0, p1);                                                                 \
  }
DCN_QUARTER_DOT16(__nv_bfloat16, "bf16")
DCN_QUARTER_DOT16(__half, "f16")
#undef DCN_QUARTER_DOT16

// piece_dot of a 2-byte piece with the raw gradient piece g (same channels).
template <typename T>
__device__ __forceinline__ float piece_dot16(const uint4& v, const uint4& g) {
  return __fadd_rn(quarter_dot16<T>(v.x, v.y, g.x, g.y), quarter_dot16<T>(v.z, v.w, g.z, g.w));
}

// Sum of a lane's pieces in the canonical order: (p0 + p1) for two pieces,
// (p0 + p1) + (p2 + p3) for four; the lane's slot order (piece j ^ rot) only
// swaps the operands of these pairwise sums.
template <int NP>
__device__ __forceinline__ float pieces_sum(const float (&p)[NP]) {
  if constexpr (NP == 2) return __fadd_rn(p[0], p[1]);
  else return __fadd_rn(__fadd_rn(p[0], p[1]), __fadd_rn(p[2], p[3]));
}

// 16 bytes of storage type T (a piece of the upstream gradient) -> fp32 pairs.
template <typename T>
__device__ __forceinline__ void piece_widen(const uint4& v, float2* g);
template <>
__device__ __forceinline__ void piece_widen<float>(const uint4& v, float2* g) {
  g[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
  g[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}
template <>
__device__ __forceinline__ void piece_widen<__nv_bfloat16>(const uint4& v, float2* g) {
  g[0] = make_float2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x));
  g[1] = make_float2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y));
  g[2] = make_float2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z));
  g[3] = make_float2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w));
}

template <>
__device__ __forceinline__ void piece_widen<__half>(const uint4& v, float2* g) {
  g[0] = f16x2_to_f32x2(v.x);
  g[1] = f16x2_to_f32x2(v.y);
  g[2] = f16x2_to_f32x2(v.z);
  g[3] = f16x2_to_f32x2(v.w);
}

// Deterministic backward: after the warp regions and the barriers, each warp
// has a staging slot of [8 units][CPR corners][16 channels] 64-bit fixed-point
// values.  A tap's contributions go there, CPR corners per round, and lane r
// of a unit sends its corner r to the accumulator as one 128-byte bulk
// reduction (cp.reduce.async.bulk .add.u64): 16 channel adds per request
// instead of 16 scalar red.global.add.u64 (measured on B200: 798 G adds/s
// against 466 G/s for the scalar reductions on random corners of an
// L2-resident accumulator).  fp32 takes two corners per round, so that the
// slots leave its twice larger boxes room for the tiles the fp32 pass needs.
__host__ __device__ constexpr int det_corners_per_round(int esize) { return esize == 4 ? 2 : 4; }
__host__ __device__ constexpr int det_stage_bytes(int esize) {  // per warp
  return 8 * det_corners_per_round(esize) * 16 * 8;
}
__host__ __device__ constexpr size_t det_stage_total(int esize) {
  return size_t(kTiledWarps) * det_stage_bytes(esize);
}

// KKS: 9 (the 3x3 window) or 8 (the window without its centre).  DET: exact
// fixed-point accumulation of grad_input (GxScatter), through the staging slots
// above (the launch adds det_stage_total(sizeof(T)) bytes of shared memory).  FAR: some
// footprint can leave the box.
template <typename T, int KKS, bool SOFTMAX, bool DET, bool FAR>
__global__ void __launch_bounds__(kTiledThreads, 1)
    dcn_backward_tiled_kernel(const __grid_constant__ CUtensorMap xmap, const TiledBwdArgs a) {
  using IO = TiledIO<T>;
  using Pair = typename IO::Pair;
  using One = typename IO::One;
  constexpr int KK = KKS, K = tap_side(KKS);
  static_assert(K == 3 && KK <= kTiledMaxTaps, "the tiled kernel serves 3x3 tap sets");
  constexpr int CS = 16 * int(sizeof(T));  // bytes of one pixel of the group
  constexpr int NP = CS / 16;              // 16-byte pieces per corner
  constexpr int GP = 8 / NP;               // gradient pairs per piece

  const TiledParams& t = a.t;
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
      if (!(t.inject_stall && i == 0)) {  // test knob: the first box never arrives
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
  // this warp's staging slot (deterministic backward), 128-byte aligned: the
  // regions and the barrier tail are multiples of 128 bytes
  constexpr int CPR = det_corners_per_round(int(sizeof(T)));
  const uint32_t stage_a = smem_addr(regions + size_t(kTiledWarps) * kFwdRegion + kFwdTailBytes) +
                           uint32_t(warp) * det_stage_bytes(int(sizeof(T)));
  const uint32_t zero_a = smem_addr(zero);
  const int u8 = lane >> 2, r = lane & 3, dy = r >> 1, dx = r & 1, rho = u8 & 1;
  const int rot = NP == 2 ? rho : 2 * dy + rho;  // piece j ^ rot in read j (as the forward)
  const uint32_t corner_b = uint32_t((dy * t.BW + dx) * CS + 16 * rot);
  const int ulead = lane & ~3;  // the unit's first lane
  const int npx = t.TH * t.TW;
  const int nb = t.batches;
  const float Hf = float(t.H), Wf = float(t.W);
  const int pixE = t.C, rowE = t.W * t.C;  // element steps to the next pixel / row
  const int cofs_r = dy * rowE + dx * pixE;  // this lane's corner from corner (y0, x0)
  const size_t n_img = size_t(t.N) * t.H * t.W * t.C;  // accumulator elements
  const size_t x_bytes = n_img * sizeof(T);
  const size_t n_out = size_t(t.N) * t.Ho * t.Wo * t.C;
  const size_t n_taps = size_t(t.N) * t.Ho * t.Wo * t.G * KK;
  int st_unit[KK], st_tap[KK];
#pragma unroll
  for (int k = 0; k < KK; ++k) {
    st_unit[k] = (lane + 32 * k) / KK;
    st_tap[k] = (lane + 32 * k) - st_unit[k] * KK;
  }

  auto batch_unit = [&](int beta, int& ho, int& wo, uint32_t& q) {
    const int il = beta / nb;
    const int v = (beta - il * nb) * kTiledBatch + lane;
    const ItemCoord c = item_coord(t, int(blockIdx.x) + il * int(gridDim.x));
    const int rr = int(fdiv(uint32_t(v), t.fd_TW));
    ho = c.ho0 + rr;
    wo = c.wo0 + (v - rr * t.TW);
    const bool valid = (v < npx) && (ho < t.Ho) && (wo < t.Wo);
    q = valid ? (uint32_t((c.n * t.Ho + ho) * t.Wo + wo) * uint32_t(t.G) + uint32_t(c.g)) *
                    uint32_t(KK)
              : ~0u;
    return c;
  };

  Pair pf_pair[KK];
  One pf_one[KK];
  auto prefetch = [&](int beta) {
    int ho, wo;
    uint32_t q;
    batch_unit(beta, ho, wo, q);
#pragma unroll
    for (int k = 0; k < KK; ++k) {
      const uint32_t src = __shfl_sync(0xFFFFFFFFu, q, st_unit[k]);
      const bool ok = src != ~0u && in_range(size_t(src) + st_tap[k], n_taps);
      pf_pair[k] = ok ? IO::ld_pair(a.off, size_t(src) + st_tap[k]) : Pair();
      pf_one[k] = ok ? IO::ld_one(a.mask, size_t(src) + st_tap[k]) : One();
    }
  };

  const int n_items_cta =
      int(blockIdx.x) < t.items ? (t.items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int total_batches = n_items_cta * nb;
  int beta = warp;
  if (beta < total_batches) prefetch(beta);

  int b = 0;
  uint32_t ph = 0;
  for (int il = 0; il < n_items_cta; ++il) {
    if (!mbar_wait_bounded_sleep(&full[b], ph)) {
      atomicOr(a.error_word, kErrTimeout);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const ItemCoord c = item_coord(t, int(blockIdx.x) + il * int(gridDim.x));
    const uint32_t box_a = smem_addr(bufs + size_t(b) * t.box_stride);
    const uint32_t lane_base = box_a + corner_b;
    const uint32_t zoff = zero_a - box_a;
    const int Y0 = box_origin(c.ho0 * t.stride - t.pad - t.halo, t.BH, t.H, t.clamp_box);
    const int X0 = box_origin(c.wo0 * t.stride_w - t.pad_w - t.halo, t.BW, t.W, t.clamp_box);
    // element offset of the item's image and group: the base of CE
    const size_t img = size_t(c.n) * t.H * t.W * t.C + size_t(c.g) * t.Cg;
    const char* const ximg = reinterpret_cast<const char*>(a.x) + img * sizeof(T);
    const GxScatter<DET> gxs(a.gx, a.det_hdr, SOFTMAX, a.det_cbits, n_img);
    // this lane's first accumulator channel of corner (y0, x0) at CE = 0
    typename GxScatter<DET>::Acc* const gx_lane = gxs.p + img + 4 * r;

    for (; beta < (il + 1) * nb; beta += kTiledWarps) {
#pragma unroll
      for (int k = 0; k < KK; ++k) {
        const int e = lane + 32 * k;
        if (sizeof(T) == 4)
          reinterpret_cast<Pair*>(reg)[e] = pf_pair[k];
        else
          reinterpret_cast<uint32_t*>(reg)[e] = *reinterpret_cast<const uint32_t*>(&pf_pair[k]);
        reinterpret_cast<float*>(reg + kFwdStageMask)[e] = IO::one(pf_one[k]);
      }
      int ho, wo;
      uint32_t q;
      batch_unit(beta, ho, wo, q);
      const bool valid = q != ~0u;
      __syncwarp();

      // Phase A: this lane's unit -> mask weights and the tap records.
      {
        float2 d[KK];
        float m[KK];
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const int e = lane * KK + k;
          d[k] = sizeof(T) == 4
                     ? IO::pair(reinterpret_cast<const Pair*>(reg)[e])
                     : IO::pair(*reinterpret_cast<const Pair*>(reg + 4 * e));
          m[k] = reinterpret_cast<const float*>(reg + kFwdStageMask)[e];
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
        __syncwarp();
        const int yb = ho * t.stride - t.pad, xb = wo * t.stride_w - t.pad_w;
        uint32_t fm = 0u;
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const int ka = tap_pos(KK, k) / K, kb = tap_pos(KK, k) % K;
          const float Y = tap_coord(yb + ka * t.dil, t.sigma, d[k].y);
          const float X = tap_coord(xb + kb * t.dil_w, t.sigma, d[k].x);
          const float fy = floorf(Y), fx = floorf(X);
          const int y0 = __float2int_rd(Y), x0 = __float2int_rd(X);
          const int by = y0 - Y0, bx = x0 - X0;
          const bool inbox = unsigned(by) < unsigned(t.BH - 1) && unsigned(bx) < unsigned(t.BW - 1);
          // -1 <= Y < H and -1 <= X < W (NaN fails): the sample has a corner in the image
          const bool live = valid && (Y >= -1.0f) && (Y < Hf) && (X >= -1.0f) && (X < Wf);
          const bool box_tap = live && inbox;
          const bool far = FAR && live && !inbox;
          const uint32_t inb = live ? (uint32_t(y0 >= 0 && x0 >= 0) |
                                       uint32_t(y0 >= 0 && x0 + 1 < t.W) << 1 |
                                       uint32_t(y0 + 1 < t.H && x0 >= 0) << 2 |
                                       uint32_t(y0 + 1 < t.H && x0 + 1 < t.W) << 3)
                                    : 0u;
          const uint32_t off = box_tap ? uint32_t((by * t.BW + bx) * CS) : zoff;
          reinterpret_cast<float4*>(reg + kBwdRegR)[k * kTiledBatch + lane] =
              make_float4(live ? Y - fy : 0.f, live ? X - fx : 0.f, m[k],
                          __uint_as_float(off | (inb << 24)));
          reinterpret_cast<int*>(reg + kBwdRegCe)[k * kTiledBatch + lane] =
              live ? y0 * rowE + x0 * pixE : 0;
          fm |= far ? (1u << k) : 0u;
        }
        reinterpret_cast<uint32_t*>(reg + kBwdRegFm)[lane] = fm;
        reinterpret_cast<uint32_t*>(reg + kBwdRegPix)[lane] =
            valid ? uint32_t((c.n * t.Ho + ho) * t.Wo + wo) : ~0u;
      }
      __syncwarp();
      if (beta + kTiledWarps < total_batches) prefetch(beta + kTiledWarps);

      // Phase B: 8 units per step, one lane per corner.
#pragma unroll 1
      for (int s = 0; s < kTiledBatch / 8; ++s) {
        const int u = s * 8 + u8;
        uint32_t pix, fm;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(pix) : "r"(reg_a + kBwdRegPix + 4u * u));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(fm) : "r"(reg_a + kBwdRegFm + 4u * u));
        const bool uvalid = pix != ~0u;
        const size_t ob = size_t(uvalid ? pix : 0u) * t.C + size_t(c.g) * t.Cg;  // output element
        // upstream gradient: all 16 channels in this lane's piece order, and this
        // lane's four scatter channels
        const char* const gp = reinterpret_cast<const char*>(a.gout) + ob * sizeof(T);
        const bool gok = uvalid && in_range(ob + 15, n_out);
        // (fp32: as pairs; 2-byte types: the raw words, see quarter_dot16)
        float2 gs[NP == 4 ? 8 : 1];
        uint4 gw[NP == 2 ? 2 : 1];
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          const uint4 gv = ldg128_pred(gp + 16 * (j ^ rot), gok);
          if constexpr (NP == 4) piece_widen<T>(gv, gs + j * GP);
          else gw[j] = gv;
        }
        auto pdot = [&](const uint4& v, int j) {
          if constexpr (NP == 4) return piece_dot<T>(v, gs + j * GP);
          else return piece_dot16<T>(v, gw[j]);
        };
        // scatter channels of this lane: 4r .. 4r+3
        float2 gr_lo, gr_hi;
        BwdIO<T>::quad(gp + 4 * r * sizeof(T), gok, gr_lo, gr_hi);
        char* const goff_u = reinterpret_cast<char*>(a.goff) +
                             (size_t(uvalid ? pix : 0u) * t.G + c.g) * KK * sizeof(Pair);
        const uint32_t lead_ok = (r == 0 && uvalid) ? 1u : 0u;
        const uint32_t ra = reg_a + kBwdRegR + uint32_t(u) * 16u;
        const uint32_t ca = reg_a + kBwdRegCe + uint32_t(u) * 4u;
        float sk[KK];
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const uint4 rw = lds128_a(ra + k * kTiledBatch * 16);
          int ce;
          asm volatile("ld.shared.s32 %0, [%1];" : "=r"(ce) : "r"(ca + k * kTiledBatch * 4));
          const float lx = __uint_as_float(rw.y), ly = __uint_as_float(rw.x);
          const float m = __uint_as_float(rw.z);
          const uint32_t inb = rw.w >> 24;
          const uint32_t a0 = lane_base + (rw.w & kBwdOffMask);
          float pp[NP];
#pragma unroll
          for (int j = 0; j < NP; ++j) pp[j] = pdot(lds128_a(a0 ^ uint32_t(16 * j)), j);
          if (FAR && __any_sync(0xFFFFFFFFu, (fm >> k) & 1u)) {
            if ((fm >> k) & 1u) {
              // this corner from global memory (zero outside the image)
              const bool in = (inb >> r) & 1u;
              const char* xp = ximg + ptrdiff_t(ce + cofs_r) * ptrdiff_t(sizeof(T));
#pragma unroll
              for (int j = 0; j < NP; ++j) {
                const char* q = xp + 16 * (j ^ rot);
                pp[j] = pdot(ldg128_pred(q, in && in_tensor(q, 16, a.x, x_bytes)), j);
              }
            }
          }
          const float dc = pieces_sum<NP>(pp);
          // corner products d00, d01, d10, d11 at the unit's first lane
          const float d0 = __shfl_sync(0xFFFFFFFFu, dc, ulead);
          const float d1 = __shfl_sync(0xFFFFFFFFu, dc, ulead + 1);
          const float d2 = __shfl_sync(0xFFFFFFFFu, dc, ulead + 2);
          const float d3 = __shfl_sync(0xFFFFFFFFu, dc, ulead + 3);
          const float dd[4] = {d0, d1, d2, d3};
          const TapGrads tg = tap_grads(dd, ly, lx);
          sk[k] = tg.s;
          const float sm = __fmul_rn(t.sigma, m);
          Quad<T>::store_pair_pred(goff_u + k * sizeof(Pair), __fmul_rn(sm, tg.gx),
                                   __fmul_rn(sm, tg.gy),
                                   (lead_ok != 0u && in_range((size_t(pix) * t.G + c.g) * KK + k,
                                                              n_taps))
                                       ? 1u
                                       : 0u);
          // grad_input: this lane's four channels of m b_c g into each corner
          float bw[4];
          bilinear_weights(ly, lx, bw);
          const float wc[4] = {__fmul_rn(m, bw[0]), __fmul_rn(m, bw[1]), __fmul_rn(m, bw[2]),
                               __fmul_rn(m, bw[3])};
          if constexpr (DET) {
#pragma unroll
           for (int c0 = 0; c0 < 4; c0 += CPR) {
            // The previous round's bulk reductions have read the slot (each lane
            // waits for its own, then the warp), so it can be rewritten.
            asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            __syncwarp();
            // slot (u8, cc - c0) holds corner cc's 16 channels; this lane's four
            // at 4r, as two 16-byte stores (odd units store the halves in the
            // other order: the two units of a quarter-warp hit other banks)
#pragma unroll
            for (int cc = c0; cc < c0 + CPR; ++cc) {
              const float2 w2 = make_float2(wc[cc], wc[cc]);
              const float2 lo = __fmul2_rn(w2, gr_lo), hi = __fmul2_rn(w2, gr_hi);
              const uint32_t sa = stage_a + uint32_t(((u8 * CPR + cc - c0) * 16 + 4 * r) * 8);
              const long long f0 = gxs.fixed(lo.x), f1 = gxs.fixed(lo.y);
              const long long f2 = gxs.fixed(hi.x), f3 = gxs.fixed(hi.y);
              if (rho) {
                asm volatile("st.shared.v2.u64 [%0], {%1, %2};" ::"r"(sa + 16u), "l"(f2), "l"(f3) : "memory");
                asm volatile("st.shared.v2.u64 [%0], {%1, %2};" ::"r"(sa), "l"(f0), "l"(f1) : "memory");
              } else {
                asm volatile("st.shared.v2.u64 [%0], {%1, %2};" ::"r"(sa), "l"(f0), "l"(f1) : "memory");
                asm volatile("st.shared.v2.u64 [%0], {%1, %2};" ::"r"(sa + 16u), "l"(f2), "l"(f3) : "memory");
              }
            }
            // the slot, written through the generic proxy, is read by the bulk copies
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            // lane r: corner r of its unit (in this round), if it lies in the image
            const int e = ce + (r >> 1) * rowE + (r & 1) * pixE;
            const size_t ge = img + size_t(ptrdiff_t(e));  // its channel 0
            if (r >= c0 && r < c0 + CPR && ((inb >> r) & 1u) != 0u && in_range(ge + 15, n_img)) {
              unsigned long long* const gq = gxs.p + ge;
              asm volatile(
                  "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.u64 [%0], [%1], 128;" ::"l"(gq),
                  "r"(stage_a + uint32_t((u8 * CPR + r - c0) * 128))
                  : "memory");
            }
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
           }
          } else {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int e = ce + (cc >> 1) * rowE + (cc & 1) * pixE;
              const float2 w2 = make_float2(wc[cc], wc[cc]);
              gxs.add_at(gx_lane + e,
                         kCheckBounds ? img + size_t(4 * r) + size_t(ptrdiff_t(e)) : 0,
                         __fmul2_rn(w2, gr_lo), __fmul2_rn(w2, gr_hi), (inb >> cc) & 1u);
            }
          }
        }
        if (lead_ok) {
          const size_t q0 = (size_t(pix) * t.G + c.g) * KK;
          float mk[KK];  // the mask weights, read back from the records
#pragma unroll
          for (int k = 0; k < KK; ++k)
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(mk[k]) : "r"(ra + k * kTiledBatch * 16 + 8));
          const float msum = mask_grad_sum<SOFTMAX>(mk, sk);
#pragma unroll
          for (int k = 0; k < KK; ++k)
            if (in_range(q0 + k, n_taps))
              Quad<T>::store_one(a.gmask, q0 + k, mask_grad<SOFTMAX>(mk[k], sk[k], msum));
        }
      }
      __syncwarp();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);
    if (++b == nbuf) {
      b = 0;
      ph ^= 1u;
    }
  }
  // the bulk reductions of this thread are complete before it exits
  if constexpr (DET) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace dcn
