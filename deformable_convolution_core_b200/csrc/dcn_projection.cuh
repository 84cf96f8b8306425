// Offset / mask projection on the 5th-generation tensor cores (sm_100a).
//
// The DCNv3 block computes the sampling offsets and the mask of the core
// operator with linear layers on the block's query features (InternImage-L
// DCNv3 explainer (wmrh.cn), section 二 steps 1-3: per group and tap an offset
// pair and a mask logit predicted from the features).  Stacking the two
// layers' weights row-wise makes one GEMM,
//     P[pixel, j] = sum_c query[pixel, c] * weight[j, c] + bias[j],
// j < G*KK*2 giving offset element j and the remaining G*KK columns the mask
// logits, exactly in the layouts dcn_core_forward reads.  bf16 operands,
// fp32 accumulation in tensor memory.
//
// Kernel: persistent CTAs over (128-pixel, 128-column) output tiles.  Warp 0
// streams 64-wide K blocks of the query and weight tiles into a 4-stage
// shared-memory ring with TMA (128-byte swizzle); warp 1 allocates 256 TMEM
// columns (two 128-column accumulators) and one of its threads issues
// tcgen05.mma (M = 128, N = 128, K = 16) and tcgen05.commit; warps 2-17 drain
// an accumulator with tcgen05.ld (four warps per 32-lane quarter of TMEM, each
// taking 32 of the 128 columns), add the bias and store, staging each 32x32
// block through shared memory so that every store instruction writes one
// pixel's contiguous columns.  The epilogue is latency-bound (a dependent
// load / add / store chain per row), so it runs in as many warps as the
// column blocks allow.  The epilogue of one tile overlaps the MMAs of
// the next.  Every mbarrier wait is bounded; on expiry the kernel sets the
// device error word, stops issuing work, waits (bounded) for what is in
// flight and frees its tensor memory.
#pragma once

#include <cuda.h>

#include "dcn_tma.cuh"

namespace dcn {

constexpr int kPjBM = 128;      // pixels per tile (MMA M, TMEM lanes)
constexpr int kPjBN = 128;      // columns per tile (MMA N)
constexpr int kPjBK = 64;       // K block: one 128-byte swizzle atom of bf16
constexpr int kPjStages = 4;
constexpr int kPjEpiWarps = 16;  // four per TMEM lane quarter, each draining 32 of the columns
constexpr int kPjEpiChunks = 16 / kPjEpiWarps;  // 32-column blocks per epilogue warp and tile
constexpr int kPjThreads = (2 + kPjEpiWarps) * 32;  // TMA warp, MMA warp, epilogue warps
constexpr uint32_t kPjTmemCols = 256;
constexpr uint32_t kPjStageBytes = (kPjBM + kPjBN) * kPjBK * 2;  // A + B, 32 KB
constexpr int kPjEpiPitch = 33;  // floats per staged row (conflict-free transpose)
constexpr size_t kPjSmemBytes = 1024 /* alignment slack */ + size_t(kPjStages) * kPjStageBytes +
                                size_t(kPjEpiWarps) * 32 * kPjEpiPitch * 4 +
                                256 /* barriers, TMEM address */;

struct ProjArgs {
  int M;         // pixels N*Ho*Wo
  int Nout;      // G*KK*3 projection columns
  int n_off;     // G*KK*2: columns [0, n_off) are offsets, the rest mask logits
  int k_blocks;  // ceil(Cq / kPjBK)
  int m_tiles, n_tiles, tiles;
  const float* bias;  // Nout values, or null
  void* offset;       // (M, n_off) of the output type
  void* mask;         // (M, Nout - n_off)
  unsigned int* error_word;
};

// ---- tcgen05 helpers (inline PTX) ----

// Shared-memory matrix descriptor: K-major operand tile in the 128-byte
// swizzle layout TMA writes (8-row x 128-byte atoms, 1024 bytes apart).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_byte_addr) {
  return uint64_t((smem_byte_addr >> 4) & 0x3FFFu)  // start address
         | (uint64_t(1) << 16)                       // leading byte offset (unused with swizzle)
         | (uint64_t(1024 >> 4) << 32)               // stride byte offset: next 8-row atom
         | (uint64_t(1) << 46)                       // descriptor version (sm_100)
         | (uint64_t(2) << 61);                      // layout: 128-byte swizzle
}

// Instruction descriptor of kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
  return (1u << 4)                     // D format: fp32
         | (1u << 7)                   // A format: bf16
         | (1u << 10)                  // B format: bf16
         | (uint32_t(N >> 3) << 17)    // N / 8
         | (uint32_t(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes: lane i gets row i.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// T: storage type of the offset and mask outputs (fp32 or bf16).
template <typename T>
__global__ void __launch_bounds__(kPjThreads, 1)
    dcn_projection_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap wmap, const ProjArgs a) {
  extern __shared__ __align__(1024) unsigned char pj_smem_raw[];
  // the swizzled operand tiles need 1024-byte aligned shared addresses
  const uint32_t pad = (1024u - (smem_addr(pj_smem_raw) & 1023u)) & 1023u;
  unsigned char* smem = pj_smem_raw + pad;
  unsigned char* stage_a = smem;
  unsigned char* stage_b = smem + size_t(kPjStages) * kPjBM * kPjBK * 2;
  float* epi = reinterpret_cast<float*>(smem + size_t(kPjStages) * kPjStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kPjEpiWarps * 32 * kPjEpiPitch);
  uint64_t* empty = full + kPjStages;
  uint64_t* tfull = empty + kPjStages;  // accumulator ready (2)
  uint64_t* tempty = tfull + 2;         // accumulator drained (2)
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* s_abort = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPjStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kPjEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {  // the whole warp allocates the two accumulators
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
    atomicOr(a.error_word, 1u);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      uint32_t it = 0;  // stages issued so far
      bool stop = false;
      for (int tile = blockIdx.x; tile < a.tiles && !stop; tile += gridDim.x) {
        const int mt = tile / a.n_tiles, nt = tile - mt * a.n_tiles;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (*abort_flag) { stop = true; break; }
          const int s = int(it % kPjStages);
          const uint32_t u = it / kPjStages;
          if (u > 0 && !mbar_wait_bounded(&empty[s], (u - 1) & 1)) {
            give_up();
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kPjStageBytes);
          tma_load_2d(stage_a + size_t(s) * kPjBM * kPjBK * 2, &qmap, &full[s], kb * kPjBK,
                      mt * kPjBM);
          tma_load_2d(stage_b + size_t(s) * kPjBN * kPjBK * 2, &wmap, &full[s], kb * kPjBK,
                      nt * kPjBN);
          ++it;
        }
      }
      // the copies of the last issued stages may still be landing
      for (uint32_t j = it > uint32_t(kPjStages) ? it - kPjStages : 0; j < it; ++j)
        (void)mbar_wait_bounded(&full[j % kPjStages], (j / kPjStages) & 1);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16_f32(kPjBM, kPjBN);
      uint32_t it = 0, li = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < a.tiles && !stop; tile += gridDim.x, ++li) {
        const int acc = int(li & 1);
        const uint32_t ua = li >> 1;
        if (ua > 0 && !mbar_wait_bounded(&tempty[acc], (ua - 1) & 1)) {
          give_up();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * kPjBN);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          const int s = int(it % kPjStages);
          if (*abort_flag || !mbar_wait_bounded(&full[s], (it / kPjStages) & 1)) {
            give_up();
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(stage_a + size_t(s) * kPjBM * kPjBK * 2);
          const uint32_t b_addr = smem_addr(stage_b + size_t(s) * kPjBN * kPjBK * 2);
#pragma unroll
          for (int k = 0; k < kPjBK / 16; ++k)  // 32 bytes of K per MMA inside the swizzle atom
            umma_bf16(d_tmem, umma_desc_sw128(a_addr + 32 * k), umma_desc_sw128(b_addr + 32 * k),
                      idesc, uint32_t((kb | k) != 0));
          umma_commit(&empty[s]);  // the stage is free once these MMAs are done
          ++it;
        }
        if (!stop) umma_commit(&tfull[acc]);
      }
      // every MMA issued has retired before the accumulators are freed
      umma_commit(mma_done);
      (void)mbar_wait_bounded(mma_done, 0);
    }
  } else {
    // ---- epilogue: warps 2-17; TMEM lanes 32 * (warp % 4) ... + 31, column block(s) h ----
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    float* st = epi + (warp - 2) * 32 * kPjEpiPitch;
    const int n_mask = a.Nout - a.n_off;
    uint32_t li = 0;
    for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++li) {
      const int acc = int(li & 1);
      if (*abort_flag || !mbar_wait_bounded(&tfull[acc], (li >> 1) & 1)) {
        give_up();
        break;
      }
      tc_fence_after();
      const int mt = tile / a.n_tiles, nt = tile - mt * a.n_tiles;
      const int row0 = mt * kPjBM + q * 32;
      const int rows = min(a.M - row0, 32);  // rows of this quarter inside the image batch
#pragma unroll 1
      for (int c = kPjEpiChunks * h; c < kPjEpiChunks * (h + 1); ++c) {
        // a block with no column below Nout (the padding of the last column
        // tile) or no row inside the batch has nothing to store
        if (nt * kPjBN + c * 32 >= a.Nout || rows <= 0) continue;
        float v[32];
        tmem_ld32(tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kPjBN + c * 32), v);
#pragma unroll
        for (int i = 0; i < 32; ++i) st[lane * kPjEpiPitch + i] = v[i];  // row = lane
        __syncwarp();
        // this lane's column, its tensor and that tensor's row pitch
        const int col = nt * kPjBN + c * 32 + lane;
        const bool cin = col < a.Nout;
        const float b = (a.bias != nullptr && cin) ? a.bias[col] : 0.f;
        T* dst;
        size_t pitch;
        const T* tensor;  // the output tensor of this column (bounds-checked build)
        if (col < a.n_off) {
          dst = static_cast<T*>(a.offset) + col;
          pitch = size_t(a.n_off);
          tensor = static_cast<const T*>(a.offset);
        } else {
          dst = static_cast<T*>(a.mask) + (col - a.n_off);
          pitch = size_t(n_mask);
          tensor = static_cast<const T*>(a.mask);
        }
        const size_t tensor_bytes = size_t(a.M) * pitch * sizeof(T);
        dst += size_t(row0) * pitch;
#pragma unroll 8
        for (int r = 0; r < rows; ++r) {
          if (cin && in_tensor(dst, sizeof(T), tensor, tensor_bytes))
            Storage<T>::store_float(dst, st[r * kPjEpiPitch + lane] + b);
          dst += pitch;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
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
