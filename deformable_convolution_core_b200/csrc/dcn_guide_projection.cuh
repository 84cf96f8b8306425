// The offset / mask branch of the DCNv3 block in one kernel (sm_100a): guide
// features (depthwise 3x3 convolution, LayerNorm, GELU; InternImage-L DCNv3
// explainer (wmrh.cn), section 二 step 1) computed straight into the A operand
// of the offset / mask projection GEMM (the same section, steps 1-3) on the
// 5th-generation tensor cores.  The bf16 query never leaves the SM.
//
// A persistent CTA walks 128-pixel row tiles of the GEMM (M = N*H*W pixels):
//   guide warps (16)   compute the guide features of the tile's pixels, with
//                      the arithmetic of dcn_guide_kernel (lane groups of LP
//                      lanes, NJ channel quads per lane), round them to bf16 and
//                      write them into the A tile in the 128-byte-swizzled
//                      K-major layout tcgen05.mma reads, one 64-channel K block
//                      per 16 KB; then fence to the async proxy and arrive on
//                      the tile's mbarrier.  Up to two A tiles are in flight, so
//                      the guide of the next tile overlaps the GEMM of this one;
//   TMA warp           streams the weight tiles (128 columns x 64 channels) into
//                      a four-stage ring;
//   MMA warp           for every 128-column block of outputs, M128 N128 K16
//                      MMAs over the tile's K blocks into one of two TMEM
//                      accumulators; frees the A tile when its last MMA is done;
//   epilogue warps (8) drain an accumulator, add the bias and store the offset
//                      and mask columns, as dcn_projection_kernel does.
// The A tile's channels past C (up to the next multiple of 64) are zero.  Every
// mbarrier wait is bounded; on expiry the kernel sets the device error word,
// stops issuing work, waits (bounded) for what is in flight and frees its
// tensor memory.
#pragma once

#include "dcn_guide.cuh"
#include "dcn_projection.cuh"

namespace dcn {

constexpr int kGpGuideWarps = 16;
constexpr int kGpEpiWarps = 8;  // two per TMEM lane quarter, each draining 64 columns
constexpr int kGpFirstGuideWarp = 2 + kGpEpiWarps;
constexpr int kGpThreads = (kGpFirstGuideWarp + kGpGuideWarps) * 32;
constexpr uint32_t kGpABlockBytes = kPjBM * kPjBK * 2;  // 128 rows x 64 bf16
constexpr uint32_t kGpBStageBytes = kPjBN * kPjBK * 2;

struct GuideProjArgs {
  const void* x;        // (N, H, W, C) of the input storage type
  const float* w;       // (3, 3, C) depthwise weight
  const float* bias;    // (C) or null
  const float* gamma;   // (C) or null (1)
  const float* beta;    // (C) or null (0)
  float eps;
  const float* pbias;   // (Nout) projection bias, or null
  void* offset;         // (M, n_off) of the output type
  void* mask;           // (M, Nout - n_off)
  unsigned int* error_word;
  int N, H, W, C, Q;
  int M, Nout, n_off, KB;  // KB: 64-channel K blocks, ceil(C / 64)
  int m_tiles, n_tiles;
  int nA;               // A tiles in flight (1 or 2)
  size_t x_bytes;       // bounds-checked build
  FastDiv fd_W, fd_H;
};

__host__ __device__ constexpr size_t guide_proj_smem(int nA, int KB, int Q) {
  return 1024 /* alignment slack */ + size_t(nA) * KB * kGpABlockBytes +
         size_t(kPjStages) * kGpBStageBytes + size_t(12) * Q * 16 +
         size_t(kGpEpiWarps) * 32 * kPjEpiPitch * 4 + 256 /* barriers, TMEM address */;
}

// T: input storage type; TO: offset / mask storage type; LP lanes per pixel and
// NJ channel quads per lane, with C = 4 * LP * NJ.
template <typename T, typename TO, int LP, int NJ>
__global__ void __launch_bounds__(kGpThreads, 1)
    dcn_guide_projection_kernel(const __grid_constant__ CUtensorMap wmap,
                                const GuideProjArgs a) {
  extern __shared__ __align__(1024) unsigned char gp_smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(gp_smem_raw) & 1023u)) & 1023u;
  unsigned char* smem = gp_smem_raw + pad;
  const size_t a_tile = size_t(a.KB) * kGpABlockBytes;
  unsigned char* const a_buf = smem;                                   // [nA][KB][16 KB]
  unsigned char* const b_buf = a_buf + size_t(a.nA) * a_tile;          // [4][16 KB]
  float4* const prm = reinterpret_cast<float4*>(b_buf + size_t(kPjStages) * kGpBStageBytes);
  float4* const w_s = prm;                // [(ta * 3 + tb) * Q + q]
  float4* const bias_s = w_s + 9 * a.Q;
  float4* const gamma_s = bias_s + a.Q;
  float4* const beta_s = gamma_s + a.Q;
  float* const epi = reinterpret_cast<float*>(beta_s + a.Q);
  uint64_t* const bfull = reinterpret_cast<uint64_t*>(epi + kGpEpiWarps * 32 * kPjEpiPitch);
  uint64_t* const bempty = bfull + kPjStages;
  uint64_t* const tfull = bempty + kPjStages;  // accumulator ready (2)
  uint64_t* const tempty = tfull + 2;          // accumulator drained (2)
  uint64_t* const afull = tempty + 2;          // A tile written (2)
  uint64_t* const aempty = afull + 2;          // A tile read by its last MMA (2)
  uint64_t* const mma_done = aempty + 2;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* const s_abort = reinterpret_cast<int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kGpEpiWarps);
      mbar_init(&afull[b], kGpGuideWarps);
      mbar_init(&aempty[b], 1);
    }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // A tiles start at zero (the K padding past C is never written), then the
  // guide parameters: 9 weight quads and the bias, gamma and beta quads.
  for (size_t i = tid; i < size_t(a.nA) * a_tile / 16; i += kGpThreads)
    reinterpret_cast<uint4*>(a_buf)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < 12 * a.Q; i += kGpThreads) {
    float4 v;
    if (i < 9 * a.Q) {
      v = __ldg(reinterpret_cast<const float4*>(a.w) + i);
    } else {
      const int r = (i - 9 * a.Q) / a.Q, q = i - 9 * a.Q - r * a.Q;
      const float* src = r == 0 ? a.bias : (r == 1 ? a.gamma : a.beta);
      v = ld4_or(src != nullptr ? src + 4 * q : nullptr, true, r == 1 ? 1.f : 0.f);
    }
    w_s[i] = v;
  }
  fence_proxy_async_smem();  // the zeroed A tiles are read by the tensor cores
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kPjTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_flag = s_abort;
  auto give_up = [&]() {
    atomicOr(a.error_word, kErrTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---- TMA producer of the weight tiles ----
    if (lane == 0) {
      uint32_t it = 0;
      bool stop = false;
      for (int mt = blockIdx.x; mt < a.m_tiles && !stop; mt += gridDim.x) {
        for (int nt = 0; nt < a.n_tiles && !stop; ++nt) {
          for (int kb = 0; kb < a.KB; ++kb) {
            if (*abort_flag) { stop = true; break; }
            const int s = int(it % kPjStages);
            const uint32_t u = it / kPjStages;
            if (u > 0 && !mbar_wait_bounded(&bempty[s], (u - 1) & 1)) {
              give_up();
              stop = true;
              break;
            }
            mbar_arrive_expect_tx(&bfull[s], kGpBStageBytes);
            tma_load_2d(b_buf + size_t(s) * kGpBStageBytes, &wmap, &bfull[s], kb * kPjBK,
                        nt * kPjBN);
            ++it;
          }
        }
      }
      for (uint32_t j = it > uint32_t(kPjStages) ? it - kPjStages : 0; j < it; ++j)
        (void)mbar_wait_bounded(&bfull[j % kPjStages], (j / kPjStages) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(kPjBM, kPjBN);
      uint32_t it = 0, li = 0, lm = 0;
      bool stop = false;
      for (int mt = blockIdx.x; mt < a.m_tiles && !stop; mt += gridDim.x, ++lm) {
        const int ab = int(lm % uint32_t(a.nA));
        if (!mbar_wait_bounded(&afull[ab], (lm / uint32_t(a.nA)) & 1)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t a_addr0 = smem_addr(a_buf + size_t(ab) * a_tile);
        for (int nt = 0; nt < a.n_tiles && !stop; ++nt, ++li) {
          const int acc = int(li & 1);
          const uint32_t ua = li >> 1;
          if (ua > 0 && !mbar_wait_bounded(&tempty[acc], (ua - 1) & 1)) {
            give_up();
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + uint32_t(acc * kPjBN);
          for (int kb = 0; kb < a.KB; ++kb) {
            const int s = int(it % kPjStages);
            if (*abort_flag || !mbar_wait_bounded(&bfull[s], (it / kPjStages) & 1)) {
              give_up();
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = a_addr0 + uint32_t(kb) * kGpABlockBytes;
            const uint32_t b_addr = smem_addr(b_buf + size_t(s) * kGpBStageBytes);
#pragma unroll
            for (int k = 0; k < kPjBK / 16; ++k)
              umma_bf16(d_tmem, umma_desc_sw128(a_addr + 32 * k),
                        umma_desc_sw128(b_addr + 32 * k), idesc, uint32_t((kb | k) != 0));
            umma_commit(&bempty[s]);
            ++it;
          }
          if (!stop) umma_commit(&tfull[acc]);
        }
        if (!stop) umma_commit(&aempty[ab]);  // the guide warps may rewrite this A tile
      }
      umma_commit(mma_done);
      (void)mbar_wait_bounded(mma_done, 0);
    }
  } else if (warp < kGpFirstGuideWarp) {
    // ---- epilogue: warps 2-9, TMEM lane quarter warp % 4, column half ----
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    float* st = epi + (warp - 2) * 32 * kPjEpiPitch;
    const int n_mask = a.Nout - a.n_off;
    uint32_t li = 0;
    bool stop = false;
    for (int mt = blockIdx.x; mt < a.m_tiles && !stop; mt += gridDim.x) {
      for (int nt = 0; nt < a.n_tiles; ++nt, ++li) {
        const int acc = int(li & 1);
        if (*abort_flag || !mbar_wait_bounded(&tfull[acc], (li >> 1) & 1)) {
          give_up();
          stop = true;
          break;
        }
        tc_fence_after();
        const int row0 = mt * kPjBM + q * 32;
        const int rows = min(a.M - row0, 32);
#pragma unroll 1
        for (int c = 2 * h; c < 2 * h + 2; ++c) {
          if (nt * kPjBN + c * 32 >= a.Nout || rows <= 0) continue;
          float v[32];
          tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kPjBN + c * 32), v);
#pragma unroll
          for (int i = 0; i < 32; ++i) st[lane * kPjEpiPitch + i] = v[i];
          __syncwarp();
          const int col = nt * kPjBN + c * 32 + lane;
          const bool cin = col < a.Nout;
          const float b = (a.pbias != nullptr && cin) ? a.pbias[col] : 0.f;
          TO* dst;
          size_t pitch;
          const TO* tensor;
          if (col < a.n_off) {
            dst = static_cast<TO*>(a.offset) + col;
            pitch = size_t(a.n_off);
            tensor = static_cast<const TO*>(a.offset);
          } else {
            dst = static_cast<TO*>(a.mask) + (col - a.n_off);
            pitch = size_t(n_mask);
            tensor = static_cast<const TO*>(a.mask);
          }
          const size_t tensor_bytes = size_t(a.M) * pitch * sizeof(TO);
          dst += size_t(row0) * pitch;
#pragma unroll 8
          for (int r = 0; r < rows; ++r) {
            if (cin && in_tensor(dst, sizeof(TO), tensor, tensor_bytes))
              Storage<TO>::store_float(dst, st[r * kPjEpiPitch + lane] + b);
            dst += pitch;
          }
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      }
    }
  } else {
    // ---- guide warps: the tile's pixels, 32 / LP per warp at a time ----
    constexpr int PPW = 32 / LP;
    const int gw = warp - kGpFirstGuideWarp;
    const int gi = lane / LP, sub = lane - gi * LP;
    const T* xs = static_cast<const T*>(a.x);
    const float inv_c = 1.0f / float(a.C);
    uint32_t lm = 0;
    for (int mt = blockIdx.x; mt < a.m_tiles; mt += gridDim.x, ++lm) {
      const int ab = int(lm % uint32_t(a.nA));
      const uint32_t use = lm / uint32_t(a.nA);
      if (use > 0 && !mbar_wait_bounded(&aempty[ab], (use - 1) & 1)) give_up();
      if (*abort_flag) break;
      unsigned char* const at = a_buf + size_t(ab) * a_tile;
      for (int i0 = 0; i0 < kPjBM; i0 += kGpGuideWarps * PPW) {
        const int i = i0 + gw * PPW + gi;  // row of the A tile
        const int m = mt * kPjBM + i;      // pixel (n*H + y)*W + x
        const bool ok = i < kPjBM && m < a.M;
        const int mm = ok ? m : 0;
        const int ny = int(fdiv(uint32_t(mm), a.fd_W));
        const int xcol = mm - ny * a.W;
        const int n = int(fdiv(uint32_t(ny), a.fd_H));
        const int y = ny - n * a.H;
        // depthwise 3x3 convolution of this lane's quads (bias first, taps in order)
        float2 acc[2 * NJ];
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float4 b = ok ? bias_s[sub + LP * j] : make_float4(0.f, 0.f, 0.f, 0.f);
          acc[2 * j] = make_float2(b.x, b.y);
          acc[2 * j + 1] = make_float2(b.z, b.w);
        }
#pragma unroll
        for (int ta = 0; ta < 3; ++ta) {
          const int yy = y + ta - 1;
          if (!ok || yy < 0 || yy >= a.H) continue;
          const T* row = xs + size_t(n * a.H + yy) * a.W * a.C;
#pragma unroll
          for (int tb = 0; tb < 3; ++tb) {
            const int xx = xcol + tb - 1;
            if (xx < 0 || xx >= a.W) continue;
            const T* px = row + size_t(xx) * a.C + 4 * sub;
            const float4* wq = w_s + (ta * 3 + tb) * a.Q + sub;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
              if (in_tensor(px + 4 * LP * j, 4 * sizeof(T), a.x, a.x_bytes)) {
                const float4 v = guide_ld4<T>(px + 4 * LP * j);
                const float4 wv = wq[LP * j];
                acc[2 * j] = __ffma2_rn(make_float2(wv.x, wv.y), make_float2(v.x, v.y), acc[2 * j]);
                acc[2 * j + 1] =
                    __ffma2_rn(make_float2(wv.z, wv.w), make_float2(v.z, v.w), acc[2 * j + 1]);
              }
            }
          }
        }
        // LayerNorm over the pixel's channels: the mean, then the mean squared deviation
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float2 lo = acc[2 * j], hi = acc[2 * j + 1];
          s += (lo.x + lo.y) + (hi.x + hi.y);
        }
        const float mean = group_sum<LP>(s) * inv_c;
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const float d0 = acc[2 * j].x - mean, d1 = acc[2 * j].y - mean;
          const float d2 = acc[2 * j + 1].x - mean, d3 = acc[2 * j + 1].y - mean;
          ss = fmaf(d0, d0, fmaf(d1, d1, fmaf(d2, d2, fmaf(d3, d3, ss))));
        }
        const float rstd = 1.0f / sqrtf(group_sum<LP>(ss) * inv_c + a.eps);
        if (ok) {
          // GELU, rounded to bf16, into row i of the A tile: channel quad qd sits
          // in K block qd / 16, 16-byte chunk (qd % 16) / 2 (128-byte swizzle:
          // XOR with the row's position in its 8-row atom), half qd % 2
          unsigned char* const rowp = at + size_t(i) * 128;
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const int qd = sub + LP * j;
            const float4 g = gamma_s[qd], b = beta_s[qd];
            const float2 lo = acc[2 * j], hi = acc[2 * j + 1];
            const float o0 = gelu_erf((lo.x - mean) * rstd * g.x + b.x);
            const float o1 = gelu_erf((lo.y - mean) * rstd * g.y + b.y);
            const float o2 = gelu_erf((hi.x - mean) * rstd * g.z + b.z);
            const float o3 = gelu_erf((hi.y - mean) * rstd * g.w + b.w);
            const int kb = qd >> 4, chunk = (qd & 15) >> 1;
            *reinterpret_cast<uint2*>(rowp + size_t(kb) * kGpABlockBytes +
                                      ((chunk ^ (i & 7)) << 4) + ((qd & 1) << 3)) =
                make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
          }
        }
      }
      fence_proxy_async_smem();  // the tensor cores read the tile through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kPjTmemCols)
                 : "memory");
  }
}

}  // namespace dcn
