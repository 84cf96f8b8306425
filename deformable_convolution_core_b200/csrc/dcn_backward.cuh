// Backward kernel of the deformable-convolution core (sm_100a; fp32 or bf16
// storage, fp32 arithmetic).
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

#include <type_traits>

#include "dcn_tile.cuh"

namespace dcn {

struct BwdArgs {
  const void* x;
  const void* off;
  const void* mask;
  const void* gout;
  void* gx;      // input-gradient accumulator: fp32 (grad_input itself for fp32
                 // storage, the caller's workspace for bf16 storage) or, for the
                 // deterministic backward, 64-bit fixed point
  void* goff;
  void* gmask;
  const unsigned int* det_hdr;  // deterministic backward: the pre-pass bounds
  int det_cbits;                // ... and ceil(log2(contributions per element))
  TileParams t;
};

// Four channels of storage type T <-> four floats.
template <typename T>
struct Quad;
template <>
struct Quad<float> {
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    Vec<16> w;
    ldg_nc(w, p);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(w.w[i]);
  }
  // Zeros unless `pred`; a false predicate issues no memory access (p may then
  // point anywhere).
  __device__ __forceinline__ static void load_pred(const void* p, bool pred, float (&v)[4]) {
    asm("{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
        " mov.b32 %0, 0;\n mov.b32 %1, 0;\n mov.b32 %2, 0;\n mov.b32 %3, 0;\n"
        " @q ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];\n}"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3])
        : "l"(p), "r"(int(pred)));
  }
  __device__ __forceinline__ static void store_pair(void* base, size_t i, float a, float b) {
    reinterpret_cast<float2*>(base)[i] = make_float2(a, b);
  }
  // (a, b) to the pair at p if pred != 0, without a branch
  __device__ __forceinline__ static void store_pair_pred(void* p, float a, float b, uint32_t pred) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %3, 0;\n @q st.global.v2.f32 [%0], {%1, %2};\n}"
                 ::"l"(p), "f"(a), "f"(b), "r"(pred)
                 : "memory");
  }
  __device__ __forceinline__ static void store_one(void* base, size_t i, float a) {
    reinterpret_cast<float*>(base)[i] = a;
  }
};
template <>
struct Quad<__nv_bfloat16> {
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    uint32_t w0, w1;
    asm("ld.global.nc.v2.b32 {%0,%1}, [%2];" : "=r"(w0), "=r"(w1) : "l"(p));
    v[0] = bf16lo_to_f32(w0);
    v[1] = bf16hi_to_f32(w0);
    v[2] = bf16lo_to_f32(w1);
    v[3] = bf16hi_to_f32(w1);
  }
  __device__ __forceinline__ static void load_pred(const void* p, bool pred, float (&v)[4]) {
    uint32_t w0, w1;
    asm("{\n .reg .pred q;\n setp.ne.b32 q, %3, 0;\n mov.b32 %0, 0;\n mov.b32 %1, 0;\n"
        " @q ld.global.nc.v2.b32 {%0, %1}, [%2];\n}"
        : "=r"(w0), "=r"(w1)
        : "l"(p), "r"(int(pred)));
    v[0] = bf16lo_to_f32(w0);
    v[1] = bf16hi_to_f32(w0);
    v[2] = bf16lo_to_f32(w1);
    v[3] = bf16hi_to_f32(w1);
  }
  __device__ __forceinline__ static void store_pair(void* base, size_t i, float a, float b) {
    reinterpret_cast<uint32_t*>(base)[i] = pack_bf16x2(a, b);
  }
  __device__ __forceinline__ static void store_pair_pred(void* p, float a, float b, uint32_t pred) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %2, 0;\n @q st.global.b32 [%0], %1;\n}"
                 ::"l"(p), "r"(pack_bf16x2(a, b)), "r"(pred)
                 : "memory");
  }
  __device__ __forceinline__ static void store_one(void* base, size_t i, float a) {
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(a);
  }
};
template <>
struct Quad<__half> {
  __device__ __forceinline__ static void load(const void* p, float (&v)[4]) {
    uint32_t w0, w1;
    asm("ld.global.nc.v2.b32 {%0,%1}, [%2];" : "=r"(w0), "=r"(w1) : "l"(p));
    v[0] = f16lo_to_f32(w0);
    v[1] = f16hi_to_f32(w0);
    v[2] = f16lo_to_f32(w1);
    v[3] = f16hi_to_f32(w1);
  }
  __device__ __forceinline__ static void load_pred(const void* p, bool pred, float (&v)[4]) {
    uint32_t w0, w1;
    asm("{\n .reg .pred q;\n setp.ne.b32 q, %3, 0;\n mov.b32 %0, 0;\n mov.b32 %1, 0;\n"
        " @q ld.global.nc.v2.b32 {%0, %1}, [%2];\n}"
        : "=r"(w0), "=r"(w1)
        : "l"(p), "r"(int(pred)));
    v[0] = f16lo_to_f32(w0);
    v[1] = f16hi_to_f32(w0);
    v[2] = f16lo_to_f32(w1);
    v[3] = f16hi_to_f32(w1);
  }
  __device__ __forceinline__ static void store_pair(void* base, size_t i, float a, float b) {
    reinterpret_cast<uint32_t*>(base)[i] = pack_f16x2(a, b);
  }
  __device__ __forceinline__ static void store_pair_pred(void* p, float a, float b, uint32_t pred) {
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %2, 0;\n @q st.global.b32 [%0], %1;\n}"
                 ::"l"(p), "r"(pack_f16x2(a, b)), "r"(pred)
                 : "memory");
  }
  __device__ __forceinline__ static void store_one(void* base, size_t i, float a) {
    reinterpret_cast<__half*>(base)[i] = __float2half_rn(a);
  }
};

// fp32 accumulator -> grad_input of a 2-byte storage type (bf16 or fp16),
// rounded to nearest even once.
template <typename T>
__global__ void dcn_round_to_half_kernel(const float4* __restrict__ in, uint2* __restrict__ out,
                                         size_t n4) {
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += size_t(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(in + i);
    if constexpr (sizeof(T) == 2 && std::is_same<T, __half>::value)
      out[i] = make_uint2(pack_f16x2(v.x, v.y), pack_f16x2(v.z, v.w));
    else
      out[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// grad_input[p .. p+3] += v, as one 16-byte vector reduction, only if `pred`
// (a false predicate issues no memory access).
__device__ __forceinline__ void red_add_v4_pred(float* p, float2 lo, float2 hi, bool pred) {
  asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
               " @q red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n}" ::"l"(p),
               "f"(lo.x), "f"(lo.y), "f"(hi.x), "f"(hi.y), "r"(int(pred))
               : "memory");
}

// ---------------------------------------------------------------------------
// grad_input accumulation.
//
// GxScatter<false>: fp32 vector reductions; the order of the additions, hence
// the last bits of the sum, may differ between runs.
// GxScatter<true> (deterministic backward): each fp32 contribution v is turned
// into the 64-bit integer round(v * 2^S) and added exactly, so the sum does not
// depend on the order.  S is chosen so that no partial sum can overflow: a
// pre-pass stores max|grad_out| (and, for a raw mask, max|mask|) in the
// header; every contribution is at most their product P in magnitude (bilinear
// weights and softmax weights are <= 1), an element receives at most
// 2^cbits contributions, hence |sum| * 2^S < 2^(cbits + e + S) <= 2^62 with
// P < 2^e and S = 62 - cbits - e (clamped to [-120, 120]).
// ---------------------------------------------------------------------------
constexpr int kDetHeaderBytes = 256;  // header in front of the 64-bit accumulator

// The fixed-point exponent S; false when the bounds are not finite (then the
// result is NaN: the conversion writes NaN into every element).
__device__ __forceinline__ bool det_exponent(const unsigned int* hdr, bool softmax, int cbits,
                                             int* S) {
  const unsigned gb = __ldg(hdr), mb = softmax ? 0x3f800000u : __ldg(hdr + 1);
  if (gb >= 0x7f800000u || mb >= 0x7f800000u) return false;  // inf or NaN met
  const double P = double(__uint_as_float(gb)) * double(__uint_as_float(mb));
  int e = 0;
  if (P > 0.0) (void)frexp(P, &e);  // P = f * 2^e, 0.5 <= f < 1
  int s = 62 - cbits - e;
  s = s > 120 ? 120 : s;
  if (s < -120) return false;
  *S = s;
  return true;
}

template <bool DET>
struct GxScatter;
template <>
struct GxScatter<false> {
  using Acc = float;
  float* p;
  size_t n;  // accumulator elements (checked in the bounds-checked build)
  __device__ __forceinline__ GxScatter(void* base, const unsigned int*, bool, int, size_t n_)
      : p(static_cast<float*>(base)), n(n_) {}
  // accumulator[e .. e+3] += (lo, hi) if pred
  __device__ __forceinline__ void add(size_t e, float2 lo, float2 hi, bool pred) const {
    if (pred && !in_range(e + 3, n)) pred = false;
    red_add_v4_pred(p + e, lo, hi, pred);
  }
  // the same at q = p + e, the address computed by the caller, if pred != 0
  // (e is only read by the bounds-checked build)
  __device__ __forceinline__ void add_at(float* q, size_t e, float2 lo, float2 hi,
                                         uint32_t pred) const {
    if (pred != 0u && !in_range(e + 3, n)) pred = 0u;
    asm volatile("{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
                 " @q red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n}" ::"l"(q),
                 "f"(lo.x), "f"(lo.y), "f"(hi.x), "f"(hi.y), "r"(pred)
                 : "memory");
  }
};
template <>
struct GxScatter<true> {
  using Acc = unsigned long long;
  unsigned long long* p;
  size_t n;     // accumulator elements (checked in the bounds-checked build)
  float scale;  // 2^S, or 0 when the bounds are not finite
  __device__ __forceinline__ GxScatter(void* base, const unsigned int* hdr, bool softmax,
                                       int cbits, size_t n_)
      : p(static_cast<unsigned long long*>(base)), n(n_) {
    int S = 0;
    scale = det_exponent(hdr, softmax, cbits, &S) ? __int_as_float((S + 127) << 23) : 0.f;
  }
  // v * 2^S is exact (a power-of-two scaling below 2^62); the conversion rounds
  // it to the nearest integer.
  __device__ __forceinline__ long long fixed(float v) const { return __float2ll_rn(v * scale); }
  __device__ __forceinline__ void add(size_t e, float2 lo, float2 hi, bool pred) const {
    if (pred && !in_range(e + 3, n)) pred = false;
    // v * 2^S is exact (a power-of-two scaling below 2^62); the conversion rounds
    // it to the nearest integer.
    const long long a = __float2ll_rn(lo.x * scale), b = __float2ll_rn(lo.y * scale);
    const long long c = __float2ll_rn(hi.x * scale), d = __float2ll_rn(hi.y * scale);
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
        " @q red.global.add.u64 [%0], %1;\n @q red.global.add.u64 [%0+8], %2;\n"
        " @q red.global.add.u64 [%0+16], %3;\n @q red.global.add.u64 [%0+24], %4;\n}" ::"l"(p + e),
        "l"(a), "l"(b), "l"(c), "l"(d), "r"(int(pred))
        : "memory");
  }
  __device__ __forceinline__ void add_at(unsigned long long* q, size_t e, float2 lo, float2 hi,
                                         uint32_t pred) const {
    add(size_t(q - p), lo, hi, pred != 0u && in_range(e + 3, n));
  }
  // accumulator[q + 4i] += v[i], i < 4, if pred: the channels c, c+4, c+8,
  // c+12 of a 16-channel group, so that the four lanes c = 0..3 of a unit
  // write one 32-byte sector per instruction (e: q's element, checked build)
  __device__ __forceinline__ void add4_strided(unsigned long long* q, size_t e, float2 lo,
                                               float2 hi, uint32_t pred) const {
    if (pred != 0u && !in_range(e + 12, n)) pred = 0u;
    const long long a = __float2ll_rn(lo.x * scale), b = __float2ll_rn(lo.y * scale);
    const long long c = __float2ll_rn(hi.x * scale), d = __float2ll_rn(hi.y * scale);
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %5, 0;\n"
        " @q red.global.add.u64 [%0], %1;\n @q red.global.add.u64 [%0+32], %2;\n"
        " @q red.global.add.u64 [%0+64], %3;\n @q red.global.add.u64 [%0+96], %4;\n}" ::"l"(q),
        "l"(a), "l"(b), "l"(c), "l"(d), "r"(pred)
        : "memory");
  }
};

// max |v| over n values, as float bits, into *out (atomicMax; *out starts at 0).
// NaN compares above +inf, so a non-finite input shows as bits >= 0x7f800000.
template <typename T>
__global__ void dcn_absmax_kernel(const T* __restrict__ v, size_t n, unsigned int* out) {
  unsigned m = 0;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    const float f = Storage<T>::to_float(v[i]);
    m = max(m, __float_as_uint(f) & 0x7fffffffu);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(out, m);
}

// 64-bit fixed-point accumulator -> grad_input: sum * 2^-S, rounded once to
// fp32 (then to nearest-even bf16 for bf16 storage); NaN everywhere when the
// bounds were not finite.
template <typename T>
__global__ void dcn_fixed_to_grad_kernel(const long long* __restrict__ acc, T* __restrict__ out,
                                         size_t n, const unsigned int* hdr, int softmax,
                                         int cbits) {
  int S = 0;
  const bool ok = det_exponent(hdr, softmax != 0, cbits, &S);
  const double inv = ok ? ldexp(1.0, -S) : 0.0;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += size_t(gridDim.x) * blockDim.x) {
    const float f = ok ? float(double(acc[i]) * inv) : __int_as_float(0x7fc00000);
    Storage<T>::store_float(out + i, f);
  }
}

// ---------------------------------------------------------------------------
// The per-tap arithmetic of the backward, shared by both kernels so that
// grad_offset and grad_mask have the same bits whatever the kernel, tile or
// lane mapping (every operation is an explicitly rounded intrinsic: no
// contraction choice is left to the compiler).  With 16 channels per group the
// corner dot product d_c = <g, x_c> is summed in one canonical order: four
// channel quarters q, each (x0 g0 + x2 g2) + (x1 g1 + x3 g3) as two packed
// pairs, then (d_q0 + d_q1) + (d_q2 + d_q3).  Pairwise sums are exact under
// swapping their operands, so a lane that meets the quarters in the order
// q ^ r (any r) gets the same bits.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float quarter_dot(float2 x01, float2 x23, float2 g01, float2 g23) {
  const float2 pd = __ffma2_rn(x23, g23, __fmul2_rn(x01, g01));
  return __fadd_rn(pd.x, pd.y);
}

struct TapGrads {
  float s;   // <g, v_k> = sum_c b_c d_c
  float gx;  // <g, dv/dX>
  float gy;  // <g, dv/dY>
};

// Bilinear weights b00, b01, b10, b11 of fractional parts (ly, lx).
__device__ __forceinline__ void bilinear_weights(float ly, float lx, float (&b)[4]) {
  const float hy = __fsub_rn(1.f, ly), hx = __fsub_rn(1.f, lx);
  b[0] = __fmul_rn(hy, hx);
  b[1] = __fmul_rn(hy, lx);
  b[2] = __fmul_rn(ly, hx);
  b[3] = __fmul_rn(ly, lx);
}

__device__ __forceinline__ TapGrads tap_grads(const float (&d)[4], float ly, float lx) {
  const float hy = __fsub_rn(1.f, ly), hx = __fsub_rn(1.f, lx);
  float b[4];
  bilinear_weights(ly, lx, b);
  TapGrads r;
  r.s = __fmaf_rn(b[3], d[3], __fmaf_rn(b[2], d[2], __fmaf_rn(b[1], d[1], __fmul_rn(b[0], d[0]))));
  r.gx = __fmaf_rn(ly, __fsub_rn(d[3], d[2]), __fmul_rn(hy, __fsub_rn(d[1], d[0])));
  r.gy = __fmaf_rn(lx, __fsub_rn(d[3], d[1]), __fmul_rn(hx, __fsub_rn(d[2], d[0])));
  return r;
}

// grad logit_k (softmax: m_k (s_k - sum_j m_j s_j)) or grad mask_k (raw: s_k).
template <bool SOFTMAX, int KK>
__device__ __forceinline__ float mask_grad_sum(const float (&m)[KK], const float (&s)[KK]) {
  float ms = 0.f;
  if (SOFTMAX) {
#pragma unroll
    for (int k = 0; k < KK; ++k) ms = __fmaf_rn(m[k], s[k], ms);
  }
  return ms;
}
template <bool SOFTMAX>
__device__ __forceinline__ float mask_grad(float m, float s, float ms) {
  return SOFTMAX ? __fmul_rn(m, __fsub_rn(s, ms)) : s;
}

// Sum of a corner dot product over the unit's lanes (one channel quarter per
// lane), lowest lane bit first: (d_q0 + d_q1) + (d_q2 + d_q3) for four lanes,
// the canonical order above.
template <int LANES>
__device__ __forceinline__ float quarters_sum(float v, unsigned mask) {
#pragma unroll
  for (int o = 1; o < LANES; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(mask, v, o));
  return v;
}

template <int LANES>
__device__ __forceinline__ float unit_sum(float v, unsigned mask) {
#pragma unroll
  for (int o = LANES / 2; o > 0; o >>= 1) v += __shfl_xor_sync(mask, v, o);
  return v;
}

// A lane owns 4 channels of its unit: LANES = Cg / 4 lanes per unit.
template <typename T, int LANES, int KKS, bool SOFTMAX, bool DET>
__global__ void __launch_bounds__(kThreads, 2) dcn_backward_kernel(const BwdArgs a) {
  using St = Staged<T>;
  constexpr int CPL = 4;
  constexpr int UPW = 32 / LANES;

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
  const unsigned umask = LANES == 32 ? 0xFFFFFFFFu
                                     : (((1u << LANES) - 1u) << (lane & ~(LANES - 1)));
  const int units = t.G * t.tile_px;
  const size_t pixE = size_t(t.C);
  const size_t rowE = size_t(t.W) * pixE;
  const size_t img_off = size_t(tc.n) * t.H * rowE + size_t(sub) * CPL;
  const char* xbytes = reinterpret_cast<const char*>(a.x);
  const char* gobytes = reinterpret_cast<const char*>(a.gout);
  const size_t n_img = size_t(t.N) * t.H * rowE;  // input (and accumulator) elements
  const size_t n_out = size_t(t.N) * t.Ho * t.Wo * pixE;
  const size_t n_taps = size_t(t.N) * t.Ho * t.Wo * t.G * KK;
  const GxScatter<DET> gxs(a.gx, a.det_hdr, SOFTMAX, a.det_cbits, n_img);

  for (int v0 = warp * UPW; v0 < units; v0 += kWarps * UPW) {
    const UnitCoord u = unit_coord(t, tc, v0 + lane / LANES);
    if (!u.valid) continue;
    const int row0 = u.g * KK;
    const size_t g_off = img_off + size_t(u.g) * t.Cg;
    const char* xg = xbytes + g_off * sizeof(T);
    const size_t upix = size_t(tc.n * t.Ho + u.ho) * t.Wo + u.wo;
    const size_t unit = upix * t.G + u.g;
    const int by = u.ho * t.stride - t.pad, bx = u.wo * t.stride_w - t.pad_w;

    float go[CPL];
    const size_t gi = upix * t.C + size_t(u.g) * t.Cg + size_t(sub) * CPL;
    Quad<T>::load_pred(gobytes + gi * sizeof(T), in_range(gi + CPL - 1, n_out), go);

    // One tap: returns s_k (reduced over the unit's lanes) and writes the
    // offset gradient of the tap.
    auto tap = [&](int k, int ka, int kb, float mk) -> float {
      const float2 d = St::pair(s_off[(row0 + k) * t.P1 + u.pix]);
      const float Y = tap_coord(by + ka * t.dil, t.sigma, d.y);
      const float X = tap_coord(bx + kb * t.dil_w, t.sigma, d.x);
      const Footprint f = footprint(Y, X, t.H, t.W);
      // (lanes of one unit share the footprint, so the branch is unit-uniform)
      float dc[4] = {0.f, 0.f, 0.f, 0.f};
      float ly = 0.f, lx = 0.f;
      if (f.in_support) {
        ly = f.ly;
        lx = f.lx;
        const ptrdiff_t base = ptrdiff_t(f.y0) * ptrdiff_t(rowE) + ptrdiff_t(f.x0) * ptrdiff_t(pixE);
        const ptrdiff_t cofs[4] = {base, base + ptrdiff_t(pixE), base + ptrdiff_t(rowE),
                                   base + ptrdiff_t(rowE + pixE)};
        const bool cval[4] = {f.v00, f.v01, f.v10, f.v11};
        float cw[4];
        bilinear_weights(ly, lx, cw);
        const float2 g01 = make_float2(go[0], go[1]), g23 = make_float2(go[2], go[3]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float cv[CPL] = {0.f, 0.f, 0.f, 0.f};
          if (cval[c] && in_range(size_t(ptrdiff_t(g_off) + cofs[c]) + CPL - 1, n_img))
            Quad<T>::load(xg + cofs[c] * ptrdiff_t(sizeof(T)), cv);
          dc[c] = quarter_dot(make_float2(cv[0], cv[1]), make_float2(cv[2], cv[3]), g01, g23);
          const float wv = __fmul_rn(mk, cw[c]);
          const float2 w2 = make_float2(wv, wv);
          gxs.add(size_t(ptrdiff_t(g_off) + cofs[c]), __fmul2_rn(w2, g01), __fmul2_rn(w2, g23),
                  cval[c]);
        }
      }
      if (LANES > 1) {
#pragma unroll
        for (int c = 0; c < 4; ++c) dc[c] = quarters_sum<LANES>(dc[c], umask);
      }
      const TapGrads tg = tap_grads(dc, ly, lx);
      if (sub == 0) {
        const float sc = __fmul_rn(t.sigma, mk);
        if (in_range(unit * KK + k, n_taps))
          Quad<T>::store_pair(a.goff, unit * KK + k, __fmul_rn(sc, tg.gx), __fmul_rn(sc, tg.gy));
      }
      return tg.s;
    };

    if constexpr (KKS > 0) {
      constexpr int K = tap_side(KKS);
      float m[KKS], s[KKS];
      mask_weights<T, KKS, SOFTMAX>(s_msk, row0, t.P1, u.pix, m);
      const float2 g01 = make_float2(go[0], go[1]), g23 = make_float2(go[2], go[3]);
      // Taps in groups of three (two for the 8-tap set), without branches:
      // the group's corner gathers are issued together, then reduced and
      // scattered; loads and reductions are predicated on the corner lying in
      // the image, and the products run as packed fp32 pairs.
      constexpr int GRP = KKS % 3 == 0 ? 3 : 2;
      static_assert(KKS % GRP == 0, "the tap set splits into whole groups");
#pragma unroll
      for (int k0 = 0; k0 < KKS; k0 += GRP) {
        Footprint f[GRP];
        float cv[GRP][4][CPL];
        int cofs[GRP][4];  // element offsets within the image (< 2^31)
        bool cval[GRP][4];
#pragma unroll
        for (int j = 0; j < GRP; ++j) {
          const int k = k0 + j;
          const float2 d = St::pair(s_off[(row0 + k) * t.P1 + u.pix]);
          const int q = tap_pos(KKS, k);  // window position of tap k
          const float Y = tap_coord(by + (q / K) * t.dil, t.sigma, d.y);
          const float X = tap_coord(bx + (q % K) * t.dil_w, t.sigma, d.x);
          f[j] = footprint(Y, X, t.H, t.W);
          const int base = f[j].y0 * int(rowE) + f[j].x0 * int(pixE);
          cofs[j][0] = base;
          cofs[j][1] = base + int(pixE);
          cofs[j][2] = base + int(rowE);
          cofs[j][3] = base + int(rowE + pixE);
          cval[j][0] = f[j].v00;
          cval[j][1] = f[j].v01;
          cval[j][2] = f[j].v10;
          cval[j][3] = f[j].v11;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            Quad<T>::load_pred(xg + ptrdiff_t(cofs[j][c]) * ptrdiff_t(sizeof(T)),
                               cval[j][c] && in_range(size_t(ptrdiff_t(g_off) + cofs[j][c]) +
                                                          CPL - 1, n_img),
                               cv[j][c]);
        }
#pragma unroll
        for (int j = 0; j < GRP; ++j) {
          const int k = k0 + j;
          float cw[4];
          bilinear_weights(f[j].ly, f[j].lx, cw);
          float dc[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            // <g, x[corner]>: the lane's quarter, then the sum over the unit's
            // quarters in the canonical order (butterfly xor 1, then xor 2)
            dc[c] = quarter_dot(make_float2(cv[j][c][0], cv[j][c][1]),
                                make_float2(cv[j][c][2], cv[j][c][3]), g01, g23);
            if (LANES > 1) dc[c] = quarters_sum<LANES>(dc[c], umask);
            const float wv = __fmul_rn(m[k], cw[c]);
            const float2 w2 = make_float2(wv, wv);
            gxs.add(size_t(ptrdiff_t(g_off) + cofs[j][c]), __fmul2_rn(w2, g01),
                    __fmul2_rn(w2, g23), cval[j][c]);
          }
          // out-of-support samples have no valid corner: every dc is 0
          const TapGrads tg = tap_grads(dc, f[j].ly, f[j].lx);
          s[k] = tg.s;
          if (sub == 0) {
            const float sc = __fmul_rn(t.sigma, m[k]);
            if (in_range(unit * KK + k, n_taps))
              Quad<T>::store_pair(a.goff, unit * KK + k, __fmul_rn(sc, tg.gx),
                                  __fmul_rn(sc, tg.gy));
          }
        }
      }
      if (sub == 0) {
        const float ms = mask_grad_sum<SOFTMAX>(m, s);
#pragma unroll
        for (int k = 0; k < KKS; ++k)
          if (in_range(unit * KK + k, n_taps))
            Quad<T>::store_one(a.gmask, unit * KK + k, mask_grad<SOFTMAX>(m[k], s[k], ms));
      }
    } else {
      // Runtime tap count: keep s_k in the tap's staged offset slot, which no
      // other unit reads and this unit no longer needs (its mask weight m_k is
      // recomputed from the staged logit).
      float mx, inv;
      mask_stats<T, SOFTMAX>(s_msk, row0, t.P1, u.pix, KK, mx, inv);
      for (int k = 0, ka = 0, kb = 0; k < KK; ++k) {
        skip_removed_tap(t, ka, kb);
        const float mk = mask_weight_at<T, SOFTMAX>(s_msk, row0 + k, t.P1, u.pix, mx, inv);
        const float sk = tap(k, ka, kb, mk);
        if (LANES > 1) __syncwarp(umask);
        if (sub == 0)  // first 4 bytes of the tap's staged pair
          *reinterpret_cast<float*>(s_off + (row0 + k) * t.P1 + u.pix) = sk;
        if (++kb == t.K) { kb = 0; ++ka; }
      }
      if (sub == 0) {
        auto s_at = [&](int k) {
          return *reinterpret_cast<const float*>(s_off + (row0 + k) * t.P1 + u.pix);
        };
        float ms = 0.f;
        if (SOFTMAX)
          for (int k = 0; k < KK; ++k)
            ms = __fmaf_rn(mask_weight_at<T, SOFTMAX>(s_msk, row0 + k, t.P1, u.pix, mx, inv),
                           s_at(k), ms);
        for (int k = 0; k < KK; ++k) {
          const float sk = s_at(k);
          const float mk = mask_weight_at<T, SOFTMAX>(s_msk, row0 + k, t.P1, u.pix, mx, inv);
          if (in_range(unit * KK + k, n_taps))
            Quad<T>::store_one(a.gmask, unit * KK + k, mask_grad<SOFTMAX>(mk, sk, ms));
        }
      }
    }
  }
}

}  // namespace dcn
