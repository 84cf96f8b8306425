// Guide features of the offset / mask branch (sm_100a).
//
// Before its linear layers predict the offsets and the mask, the DCNv3 block
// passes its input through a depthwise convolution, LayerNorm and GELU
// (InternImage-L DCNv3 explainer (wmrh.cn), section 二 step 1: a light 3x3
// look at the neighbourhood that guides where to sample).  One kernel does
// all three per pixel and writes the bf16 query the projection GEMM reads:
//   conv[c] = bias[c] + sum_{a, b < 3} w[a][b][c] * x[y + a - 1][x + b - 1][c]
//             (zero outside the image; stride 1)
//   z[c]    = (conv[c] - mean) / sqrt(var + eps) * gamma[c] + beta[c]
//             (mean and biased variance over the pixel's C channels)
//   out[c]  = z[c] * (1 + erf(z[c] / sqrt(2))) / 2, rounded to bf16 once.
// Arithmetic is fp32 (two-pass variance).
//
// Layout of the work: a pixel's C channels are Q = C/4 quads, spread over a
// group of LP lanes (quad sub + LP*j for lane sub, j < NJ), so a warp holds
// 32/LP pixels of one row; LP is picked on the host so that the quads fill
// the lanes (C = 160: 8 lanes x 5 quads, four pixels per warp).  A lane
// convolves up to kGuideChunk of its quads at once in registers (one address
// per tap) and parks the results in shared memory for the two LayerNorm
// passes, so registers do not grow with C.  The weights and the affine
// parameters are staged in shared memory once per CTA.  A CTA of
// kGuideWarps warps covers adjacent columns and walks up to kGuideRows rows
// down (the image's rows split evenly over the row tiles):
// consecutive windows of a lane group share six of their nine input pixels
// and neighbouring groups share columns, so the input is read from DRAM
// about once and re-read from L1.
#pragma once

#include <cuda_bf16.h>

#include "dcn_common.cuh"

namespace dcn {

constexpr int kGuideWarps = 8;
constexpr int kGuideRows = 8;
constexpr int kGuideMaxQuads = 16;  // quads per lane (NJ), at most
constexpr int kGuideChunk = 5;      // quads per lane convolved together in registers

struct GuideArgs {
  const void* x;       // (N, H, W, C) of T
  const float* w;      // (3, 3, C): w[(a * 3 + b) * C + c]
  const float* bias;   // (C) or null
  const float* gamma;  // (C) or null (1)
  const float* beta;   // (C) or null (0)
  float eps;
  __nv_bfloat16* out;  // (N, H, W, C)
  int N, H, W, C, Q, NJ;
  int tiles_x, tiles_y;
  int rows;  // rows a CTA walks: ceil(H / tiles_y), at most kGuideRows
  size_t x_bytes, out_bytes;  // bounds-checked build
};

// Four consecutive channels of storage type T as floats (read-only path).
template <typename T>
__device__ __forceinline__ float4 guide_ld4(const T* p);
template <>
__device__ __forceinline__ float4 guide_ld4<float>(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
template <>
__device__ __forceinline__ float4 guide_ld4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(bf16lo_to_f32(u.x), bf16hi_to_f32(u.x), bf16lo_to_f32(u.y),
                     bf16hi_to_f32(u.y));
}
template <>
__device__ __forceinline__ float4 guide_ld4<__half>(const __half* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = f16x2_to_f32x2(u.x), b = f16x2_to_f32x2(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float4 ld4_or(const float* p, bool ok, float dflt) {
  return ok && p != nullptr ? __ldg(reinterpret_cast<const float4*>(p))
                            : make_float4(dflt, dflt, dflt, dflt);
}

// Sum over the LP lanes of this lane's group (xor offsets below LP stay inside it).
template <int LP>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = LP / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

// Output rows a CTA computes per pass (see the kernel).
template <typename T, int LP, int NJS>
__host__ __device__ constexpr int guide_rows_per_pass() {
  return (NJS > 0 && LP <= 16 && sizeof(T) == 4) ? 2 : 1;
}

// Three CTAs per SM for groups of 8 or 16 lanes (more warps to cover the
// load latency; measured 10% faster at C = 160), two for the two-row fp32
// passes (their second accumulator set would spill at three); 32-lane groups
// are left to the compiler (their spills at three cost more than the warps
// gain).
// NJS > 0: the quads fill the lane groups exactly (Q = LP * NJS, the channel
// widths of the InternImage stages), so the quad count is a compile-time
// constant and no quad needs a bounds predicate; NJS = 0: any C.
template <typename T, int LP, int NJS>
__global__ void __launch_bounds__(kGuideWarps * 32,
                                  LP <= 16 ? (guide_rows_per_pass<T, LP, NJS>() == 2 ? 2 : 3) : 1)
    dcn_guide_kernel(const GuideArgs a) {
  constexpr int PPW = 32 / LP;  // pixels per warp
  constexpr int kThreads = kGuideWarps * 32;
  constexpr int CH = kGuideChunk;
  constexpr bool FULL = NJS > 0;
  const int NJ = FULL ? NJS : a.NJ;
  // Shared memory: the 9 weight quads and the bias, gamma and beta quads of
  // every channel (12 * Q float4, staged once per CTA), then the conv results
  // of this thread's quads, [quad j][thread]: consecutive lanes touch
  // consecutive 16-byte words, and each thread reads back only its own.
  extern __shared__ float4 guide_smem[];
  float4* const w_s = guide_smem;            // [(a * 3 + b) * Q + q]
  float4* const bias_s = w_s + 9 * a.Q;      // [q]
  float4* const gamma_s = bias_s + a.Q;
  float4* const beta_s = gamma_s + a.Q;
  float4* const conv_buf = beta_s + a.Q;     // [j * kThreads + tid]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Several loads in flight per thread (at C = 1280 a thread stages 15 quads;
  // at the narrow widths, under the 3-CTA register cap, two at a time).
  constexpr int IF = LP <= 16 ? 2 : 4;
  for (int i0 = tid; i0 < 12 * a.Q; i0 += IF * kThreads) {
    float4 v[IF];
#pragma unroll
    for (int u = 0; u < IF; ++u) {
      const int i = i0 + u * kThreads;
      if (i >= 12 * a.Q) break;
      if (i < 9 * a.Q) v[u] = __ldg(reinterpret_cast<const float4*>(a.w) + i);
      else {
        const int r = (i - 9 * a.Q) / a.Q, q = i - 9 * a.Q - r * a.Q;
        const float* src = r == 0 ? a.bias : (r == 1 ? a.gamma : a.beta);
        v[u] = ld4_or(src != nullptr ? src + 4 * q : nullptr, true, r == 1 ? 1.f : 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < IF; ++u) {
      const int i = i0 + u * kThreads;
      if (i >= 12 * a.Q) break;
      w_s[i] = v[u];
    }
  }
  __syncthreads();

  const int gi = lane / LP, sub = lane - gi * LP;
  int t = blockIdx.x;
  const int tx = t % a.tiles_x;
  t /= a.tiles_x;
  const int ty = t % a.tiles_y;
  const int n = t / a.tiles_y;
  const int col = (tx * kGuideWarps + warp) * PPW + gi;
  const bool col_ok = col < a.W;
  const T* xs = static_cast<const T*>(a.x);
  const size_t rowE = size_t(a.W) * a.C;  // elements per image row
  const float inv_c = 1.0f / float(a.C);

  // (the narrow widths, under the 3-CTA register cap, keep the row count a
  // compile-time constant: one register less)
  // fp32 input at the stage widths: two output rows per pass, which share each
  // weight read from shared memory (a 16-byte weight load serves 8 pixels
  // instead of 4); measured 23% faster at stage 1 (two CTAs per SM), while the
  // 2-byte types lose 5% and keep one row per pass
  constexpr int R = guide_rows_per_pass<T, LP, NJS>();
  if constexpr (R == 2) {
    const int rows = LP == 32 ? a.rows : kGuideRows;
    for (int i = 0; i < rows; i += R) {
      const int y = ty * rows + i;
      if (y >= a.H) break;  // the same for the whole CTA
      float s[R];
#pragma unroll
      for (int r = 0; r < R; ++r) s[r] = 0.f;
#pragma unroll(FULL ? 4 : 1)
      for (int j0 = 0; j0 < NJ; j0 += CH) {
        float2 acc[R][2 * CH];
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          const int q = sub + LP * (j0 + u);
          const float4 b = ((FULL || (j0 + u < NJ && q < a.Q)) && col_ok)
                               ? bias_s[FULL && CH > NJS ? (u < NJS ? q : sub) : q]
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            acc[r][2 * u] = make_float2(b.x, b.y);
            acc[r][2 * u + 1] = make_float2(b.z, b.w);
          }
        }
#pragma unroll
        for (int ta = 0; ta < 3; ++ta) {
          bool ok[R];
          const T* rowp[R];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const int yy = y + r + ta - 1;
            ok[r] = y + r < a.H && yy >= 0 && yy < a.H;  // the same for the whole CTA
            rowp[r] = xs + size_t(n * a.H + (ok[r] ? yy : 0)) * rowE;
          }
          bool any = false;
#pragma unroll
          for (int r = 0; r < R; ++r) any = any || ok[r];
          if (!any) continue;
#pragma unroll
          for (int tb = 0; tb < 3; ++tb) {
            const int xx = col + tb - 1;
            if (!(col_ok && xx >= 0 && xx < a.W)) continue;
            const float4* wq = w_s + (ta * 3 + tb) * a.Q + sub;
#pragma unroll
            for (int u = 0; u < CH; ++u) {
              const int j = j0 + u;
              if (!(FULL ? j < NJS : (j < NJ && sub + LP * j < a.Q))) continue;
              const float4 wv = wq[LP * j];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                const T* pq = rowp[r] + xx * a.C + 4 * sub + 4 * LP * j;
                if (ok[r] && in_tensor(pq, 4 * sizeof(T), a.x, a.x_bytes)) {
                  const float4 v = guide_ld4<T>(pq);
                  acc[r][2 * u] =
                      __ffma2_rn(make_float2(wv.x, wv.y), make_float2(v.x, v.y), acc[r][2 * u]);
                  acc[r][2 * u + 1] =
                      __ffma2_rn(make_float2(wv.z, wv.w), make_float2(v.z, v.w), acc[r][2 * u + 1]);
                }
              }
            }
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int u = 0; u < CH; ++u) {
            if (j0 + u < NJ) {
              const float2 lo = acc[r][2 * u], hi = acc[r][2 * u + 1];
              s[r] += (lo.x + lo.y) + (hi.x + hi.y);  // quads outside C hold 0
              conv_buf[(r * NJ + j0 + u) * kThreads + tid] = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
          }
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (y + r >= a.H) break;  // the same for the whole CTA
        // LayerNorm over the pixel's channels: the mean, then the mean squared deviation
        const float mean = group_sum<LP>(s[r]) * inv_c;
        float ss = 0.f;
#pragma unroll(FULL ? 16 : 1)
        for (int j = 0; j < NJ; ++j) {
          if (!FULL && sub + LP * j >= a.Q) break;
          const float4 v = conv_buf[(r * NJ + j) * kThreads + tid];
          const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
          ss = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, ss))));
        }
        const float rstd = 1.0f / sqrtf(group_sum<LP>(ss) * inv_c + a.eps);
        if (!col_ok) continue;
        __nv_bfloat16* op = a.out + (size_t(n * a.H + y + r) * a.W + col) * a.C;
#pragma unroll(FULL ? 16 : 1)
        for (int j = 0; j < NJ; ++j) {
          const int q = sub + LP * j;
          if (!FULL && q >= a.Q) break;
          const float4 v = conv_buf[(r * NJ + j) * kThreads + tid];
          const float4 g = gamma_s[q], b = beta_s[q];
          const float o0 = gelu_erf((v.x - mean) * rstd * g.x + b.x);
          const float o1 = gelu_erf((v.y - mean) * rstd * g.y + b.y);
          const float o2 = gelu_erf((v.z - mean) * rstd * g.z + b.z);
          const float o3 = gelu_erf((v.w - mean) * rstd * g.w + b.w);
          if (in_tensor(op + 4 * q, 8, a.out, a.out_bytes))
            *reinterpret_cast<uint2*>(op + 4 * q) = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
        }
      }
    }
  } else {
    const int rows = LP == 32 ? a.rows : kGuideRows;
    for (int i = 0; i < rows; ++i) {
      const int y = ty * rows + i;
      if (y >= a.H) break;  // the same for the whole CTA
      // depthwise 3x3 convolution, CH quads of this lane at a time in registers
      float s = 0.f;
#pragma unroll(FULL ? 4 : 1)
      for (int j0 = 0; j0 < NJ; j0 += CH) {
        float2 acc[2 * CH];  // quad u: channels (x, y) in acc[2u], (z, w) in acc[2u + 1]
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          const int q = sub + LP * (j0 + u);
          const float4 b = ((FULL || (j0 + u < NJ && q < a.Q)) && col_ok)
                               ? bias_s[FULL && CH > NJS ? (u < NJS ? q : sub) : q]
                               : make_float4(0.f, 0.f, 0.f, 0.f);
          acc[2 * u] = make_float2(b.x, b.y);
          acc[2 * u + 1] = make_float2(b.z, b.w);
        }
#pragma unroll
        for (int ta = 0; ta < 3; ++ta) {
          const int yy = y + ta - 1;
          if (yy < 0 || yy >= a.H) continue;  // the same for the whole CTA
          const T* row = xs + size_t(n * a.H + yy) * rowE;
#pragma unroll
          for (int tb = 0; tb < 3; ++tb) {
            const int xx = col + tb - 1;
            if (!(col_ok && xx >= 0 && xx < a.W)) continue;
            const T* px = row + xx * a.C + 4 * sub;
            const float4* wq = w_s + (ta * 3 + tb) * a.Q + sub;
#pragma unroll
            for (int u = 0; u < CH; ++u) {
              const int j = j0 + u;
              if ((FULL ? j < NJS : (j < NJ && sub + LP * j < a.Q)) &&
                  in_tensor(px + 4 * LP * j, 4 * sizeof(T), a.x, a.x_bytes)) {
                const float4 v = guide_ld4<T>(px + 4 * LP * j);
                const float4 wv = wq[LP * j];
                acc[2 * u] = __ffma2_rn(make_float2(wv.x, wv.y), make_float2(v.x, v.y), acc[2 * u]);
                acc[2 * u + 1] =
                    __ffma2_rn(make_float2(wv.z, wv.w), make_float2(v.z, v.w), acc[2 * u + 1]);
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < CH; ++u) {
          if (j0 + u < NJ) {
            const float2 lo = acc[2 * u], hi = acc[2 * u + 1];
            s += (lo.x + lo.y) + (hi.x + hi.y);  // quads outside C hold 0
            conv_buf[(j0 + u) * kThreads + tid] = make_float4(lo.x, lo.y, hi.x, hi.y);
          }
        }
      }
      // LayerNorm over the pixel's channels: the mean, then the mean squared deviation
      const float mean = group_sum<LP>(s) * inv_c;
      float ss = 0.f;
#pragma unroll(FULL ? 16 : 1)
      for (int j = 0; j < NJ; ++j) {
        if (!FULL && sub + LP * j >= a.Q) break;
        const float4 v = conv_buf[j * kThreads + tid];
        const float d0 = v.x - mean, d1 = v.y - mean, d2 = v.z - mean, d3 = v.w - mean;
        ss = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, ss))));
      }
      const float rstd = 1.0f / sqrtf(group_sum<LP>(ss) * inv_c + a.eps);
      if (!col_ok) continue;
      __nv_bfloat16* op = a.out + (size_t(n * a.H + y) * a.W + col) * a.C;
#pragma unroll(FULL ? 16 : 1)
      for (int j = 0; j < NJ; ++j) {
        const int q = sub + LP * j;
        if (!FULL && q >= a.Q) break;
        const float4 v = conv_buf[j * kThreads + tid];
        const float4 g = gamma_s[q], b = beta_s[q];
        const float o0 = gelu_erf((v.x - mean) * rstd * g.x + b.x);
        const float o1 = gelu_erf((v.y - mean) * rstd * g.y + b.y);
        const float o2 = gelu_erf((v.z - mean) * rstd * g.z + b.z);
        const float o3 = gelu_erf((v.w - mean) * rstd * g.w + b.w);
        if (in_tensor(op + 4 * q, 8, a.out, a.out_bytes))
          *reinterpret_cast<uint2*>(op + 4 * q) = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
      }
    }
  }
}

}  // namespace dcn
