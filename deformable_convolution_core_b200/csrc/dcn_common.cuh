// Shared device helpers of the B200 deformable-convolution core.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dcn {

// Device error word, read and cleared by dcn_core_sync_status: bit 0 = a
// bounded wait gave up, bit 1 = the bounds-checked build skipped an access
// that would have left its tensor.
constexpr unsigned int kErrTimeout = 1u, kErrOutOfBounds = 2u;
__device__ unsigned int g_dcn_error_word = 0;

// ---------------------------------------------------------------------------
// Bounds-checked build (compiled with -DDCN_CHECK_BOUNDS), the substitute for
// a memory checker: every global load, store and reduction of the kernels is
// first tested against its tensor's extent, and an access that would leave it
// is skipped and recorded in the error word.  Without the macro the tests
// compile away.
// ---------------------------------------------------------------------------
#ifdef DCN_CHECK_BOUNDS
constexpr bool kCheckBounds = true;
#else
constexpr bool kCheckBounds = false;
#endif

// Element i of a tensor of n elements?
__device__ __forceinline__ bool in_range(size_t i, size_t n) {
  if (!kCheckBounds) return true;
  const bool ok = i < n;
  if (!ok) atomicOr(&g_dcn_error_word, kErrOutOfBounds);
  return ok;
}

// [p, p + nbytes) inside the tensor [base, base + bytes)?
__device__ __forceinline__ bool in_tensor(const void* p, size_t nbytes, const void* base,
                                          size_t bytes) {
  if (!kCheckBounds) return true;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
  const bool ok = a >= b && a + nbytes <= b + bytes;
  if (!ok) atomicOr(&g_dcn_error_word, kErrOutOfBounds);
  return ok;
}

// ---------------------------------------------------------------------------
// Division by a runtime-invariant divisor with one multiply-high and a shift
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, section 4): for d >= 1 let l = ceil(log2 d) and
// m = floor(2^32 * (2^l - d) / d) + 1; then for every 32-bit n,
// floor(n / d) = (mulhi(m, n) + n) >> l, evaluated without overflow in 64 bits.
// ---------------------------------------------------------------------------
struct FastDiv {
  uint32_t d;
  uint32_t m;
  uint32_t l;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t l = 0;
  while (l < 32 && (uint64_t(1) << l) < d) ++l;
  f.l = l;
  f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  return f;
}

__host__ __device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
#ifdef __CUDA_ARCH__
  uint32_t hi = __umulhi(f.m, n);
#else
  uint32_t hi = uint32_t((uint64_t(f.m) * n) >> 32);
#endif
  return uint32_t((uint64_t(hi) + n) >> f.l);
}

// ---------------------------------------------------------------------------
// Storage types.  bf16 is widened to fp32 exactly by placing its 16 bits in
// the high half of an fp32 word; fp32 -> bf16 rounds to nearest even.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

// fp16 storage: widened to fp32 exactly (every fp16 value is an fp32 value);
// fp32 -> fp16 rounds to nearest even (overflow to +-inf, as the conversion
// defines).
__device__ __forceinline__ float f16lo_to_f32(uint32_t w) {
  return __low2float(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ float f16hi_to_f32(uint32_t w) {
  return __high2float(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

// Read-only gathers of 16 or 32 bytes through the non-coherent path.
template <int BYTES>
struct Vec;
template <>
struct Vec<16> {
  uint32_t w[4];
};
template <>
struct Vec<32> {
  uint32_t w[8];
};

__device__ __forceinline__ void ldg_nc(Vec<16>& v, const void* p) {
  asm("ld.global.nc.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3])
               : "l"(p));
}
__device__ __forceinline__ void ldg_nc(Vec<32>& v, const void* p) {
  asm("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]),
                 "=r"(v.w[4]), "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
               : "l"(p));
}
__device__ __forceinline__ void stg(void* p, const Vec<16>& v) {
  asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.w[0]), "r"(v.w[1]),
               "r"(v.w[2]), "r"(v.w[3])
               : "memory");
}
__device__ __forceinline__ void stg(void* p, const Vec<32>& v) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v.w[0]),
               "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]), "r"(v.w[6]),
               "r"(v.w[7])
               : "memory");
}

// Storage-type traits: how a lane's CPL channels map onto 16/32-byte vectors.
template <typename T>
struct Storage;

template <>
struct Storage<float> {
  static constexpr int kSize = 4;
  __device__ __forceinline__ static float to_float(float v) { return v; }
  __device__ __forceinline__ static void store_float(float* p, float v) { *p = v; }
  // Widen the j-th channel held in a vector of words.
  template <int N>
  __device__ __forceinline__ static float chan(const uint32_t (&w)[N], int j) {
    return __uint_as_float(w[j]);
  }
  template <int N>
  __device__ __forceinline__ static void pack(uint32_t (&w)[N], const float* acc) {
#pragma unroll
    for (int j = 0; j < N; ++j) w[j] = __float_as_uint(acc[j]);
  }
};

template <>
struct Storage<__half> {
  static constexpr int kSize = 2;
  __device__ __forceinline__ static float to_float(__half v) { return __half2float(v); }
  // round to nearest even
  __device__ __forceinline__ static void store_float(__half* p, float v) {
    *p = __float2half_rn(v);
  }
  template <int N>
  __device__ __forceinline__ static float chan(const uint32_t (&w)[N], int j) {
    return (j & 1) ? f16hi_to_f32(w[j >> 1]) : f16lo_to_f32(w[j >> 1]);
  }
  template <int N>
  __device__ __forceinline__ static void pack(uint32_t (&w)[N], const float* acc) {
#pragma unroll
    for (int j = 0; j < N; ++j) w[j] = pack_f16x2(acc[2 * j], acc[2 * j + 1]);
  }
};

template <>
struct Storage<__nv_bfloat16> {
  static constexpr int kSize = 2;
  __device__ __forceinline__ static float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
  // round to nearest even
  __device__ __forceinline__ static void store_float(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
  template <int N>
  __device__ __forceinline__ static float chan(const uint32_t (&w)[N], int j) {
    return (j & 1) ? bf16hi_to_f32(w[j >> 1]) : bf16lo_to_f32(w[j >> 1]);
  }
  template <int N>
  __device__ __forceinline__ static void pack(uint32_t (&w)[N], const float* acc) {
#pragma unroll
    for (int j = 0; j < N; ++j) w[j] = pack_bf16x2(acc[2 * j], acc[2 * j + 1]);
  }
};

// ---------------------------------------------------------------------------
// Sampling location of one tap: two separately rounded fp32 operations per
// coordinate (no contraction into an FMA), so that floor() of the location is
// reproducible on any implementation that follows the same rule.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float tap_coord(int base, float scale, float delta) {
  return __fadd_rn(float(base), __fmul_rn(scale, delta));
}

// Bilinear footprint of one sample: the top-left corner cell, the fractional
// parts and which of the four corners lie inside the image.  in_support ==
// false means the sample contributes nothing (and has no derivative).
struct Footprint {
  bool in_support;
  bool v00, v01, v10, v11;
  int y0, x0;
  float ly, lx;  // fractional parts
};

__device__ __forceinline__ Footprint footprint(float Y, float X, int H, int W) {
  Footprint f;
  // -1 <= Y < H and -1 <= X < W: some corner may be inside.  NaN and inf fail.
  f.in_support = (Y >= -1.0f) && (Y < float(H)) && (X >= -1.0f) && (X < float(W));
  if (!f.in_support) {
    f.v00 = f.v01 = f.v10 = f.v11 = false;
    f.y0 = f.x0 = 0;
    f.ly = f.lx = 0.f;
    return f;
  }
  const float yf = floorf(Y), xf = floorf(X);
  f.y0 = int(yf);
  f.x0 = int(xf);
  f.ly = Y - yf;  // exact for Y >= 0; within one rounding for Y in [-1, 0)
  f.lx = X - xf;
  const bool y0in = f.y0 >= 0, y1in = f.y0 + 1 < H;
  const bool x0in = f.x0 >= 0, x1in = f.x0 + 1 < W;
  f.v00 = y0in && x0in;
  f.v01 = y0in && x1in;
  f.v10 = y1in && x0in;
  f.v11 = y1in && x1in;
  return f;
}

}  // namespace dcn
