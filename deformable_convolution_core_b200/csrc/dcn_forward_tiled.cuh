// Forward kernel with the input staged in shared memory by TMA (sm_100a).
//
// Same operator as dcn_forward_kernel (InternImage-L DCNv3 explainer
// (wmrh.cn), section 二 steps 2-4, section 三).  The difference is where the
// bilinear corners are read from.  A global gather costs the L1 one
// wavefront per distinct 128-byte line touched, i.e. one per corner whatever
// its size, so a direct-gather kernel is capped near four L1 cycles per
// sample.  Here a persistent CTA walks work items (image n, output tile,
// group g); for each item one TMA tensor copy brings the group's 16 channels
// of the input box the tile can reach into shared memory, with up to eight
// boxes in flight on full/empty mbarriers.
//
// Per warp batch of 32 units (pixel, group):
//   staging  the batch's offsets and mask, loaded coalesced one batch ahead,
//            are written to the warp's region in their global order (element
//            e = 9u + k at word e: conflict-free both ways, 9 being odd);
//   phase A  one lane per unit: softmax over the taps, then per tap its four
//            corner weights and the byte offset of corner (y0, x0) in the box,
//            stored as structures of arrays W[k][u], OFF[k][u];
//   phase B  four lanes per unit, one per bilinear corner, each holding all
//            16 channels of its corner, 8 units per step.  A lane reads its
//            corner as two (bf16) or four (fp32) 16-byte pieces; the units of
//            a quarter-warp read complementary pieces (unit parity rho), so
//            every footprint read is one conflict-free wavefront per 128
//            bytes whatever the offsets.  A reduce-scatter over the four
//            corner lanes ends with four channels per lane, stored directly.
// A tap whose footprint lies in the box reads it there.  A tap that
// contributes nothing gets weight 0 and reads a band of zeros (exact even for
// non-finite inputs).  A tap whose footprint leaves the box ("far") also reads
// the zeros in the box pass; its record then carries the weights' factors and
// the corner's coordinates, and a second pass reads its corners from global
// memory.  With the box covering the whole image and its zero ring (small
// images) there are no far taps.
#pragma once

#include "dcn_tma.cuh"

namespace dcn {

struct TiledArgs {
  const void* x;
  const void* off;
  const void* mask;
  void* out;
  unsigned int* error_word;
  TiledParams t;
};

// Per-warp region of the forward: W[9][32] float4, OFF[9][32], FM[32] (far
// taps of each unit, bit k = tap k), OUT[32] (element offset of the unit's
// output channels, or ~0 for a unit outside the output).  The staged inputs
// of a batch alias it: they are read into registers before the records are
// written.
constexpr int kFwdRegW = 0;
constexpr int kFwdRegOff = kTiledMaxTaps * kTiledBatch * 16;
constexpr int kFwdRegFm = kFwdRegOff + kTiledMaxTaps * kTiledBatch * 4;
constexpr int kFwdRegOut = kFwdRegFm + kTiledBatch * 4;
constexpr int kFwdRegion = kFwdRegOut + kTiledBatch * 4;  // 6016 bytes
static_assert(kFwdRegion % 128 == 0, "warp regions stay 128-byte aligned");
// Staged offsets and mask: element e of the batch (unit e / KK, tap e % KK):
// the offset pair at 4e (bf16) or 8e (fp32), the mask value (as fp32) after them.
constexpr int kFwdStageMask = kTiledMaxTaps * kTiledBatch * 8;
static_assert(kFwdStageMask + kTiledMaxTaps * kTiledBatch * 4 <= kFwdRegion, "staging fits");
// After the regions: full[8], empty[8] mbarriers and the abort flag.
constexpr int kFwdTailBytes = 256;
// Far-tap record: y0 + 1 and x0 + 1 packed into 14 bits each; as fp32 bits the
// word is a finite number (below 2^28, sign clear), so the box pass may
// multiply it by the zero band.
constexpr int kFarShift = 14;

// Zero band: (BW + 2) pixels of zeros; a dead or far tap's offset points at
// it, so that every corner lane (row pitch BW) lands on zeros.
__host__ __device__ constexpr int zero_band_bytes(int BW, int cs) {
  return ((BW + 2) * cs + 127) / 128 * 128;
}

// Shared-memory bytes of the forward kernel.
__host__ __device__ constexpr size_t fwd_tiled_smem(int nbuf, uint32_t box_stride, int BW, int cs) {
  return size_t(nbuf) * box_stride + size_t(zero_band_bytes(BW, cs)) +
         size_t(kTiledWarps) * kFwdRegion + kFwdTailBytes;
}

// KKS: 9 (the 3x3 window) or 8 (the window without its centre).  FAR: some
// footprint can leave the box (the box does not cover the whole image).  CG:
// channels per group, 16, or 8 with 2-byte storage (a 16-byte pixel: one
// piece per corner lane, and the reduce-scatter ends with two channels a lane).
template <typename T, int KKS, bool SOFTMAX, bool FAR, int CG = 16>
__global__ void __launch_bounds__(kTiledThreads, 1)
    dcn_forward_tiled_kernel(const __grid_constant__ CUtensorMap xmap, const TiledArgs a) {
  using IO = TiledIO<T>;
  using Pair = typename IO::Pair;
  using One = typename IO::One;
  constexpr int KK = KKS, K = tap_side(KKS);
  static_assert(K == 3 && KK <= kTiledMaxTaps, "the tiled kernel serves 3x3 tap sets");
  static_assert(CG == 16 || (CG == 8 && sizeof(T) == 2), "16 channels, or 8 of a 2-byte type");
  constexpr int CS = CG * int(sizeof(T));  // bytes of one pixel of the group
  constexpr int NP = CS / 16;              // 16-byte pieces per corner: 1, 2 (bf16) or 4 (fp32)
  constexpr int PA = CG / 2 / NP;          // accumulator pairs per piece

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
    uint32_t ph = 0;  // parity of this round over the buffers
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
    // Copies issued for the last items may still be landing: wait for them
    // (bounded) before this thread, possibly the CTA's last, exits.
    for (int j = i - nbuf < 0 ? 0 : i - nbuf; j < i; ++j)
      if (!(t.inject_stall && j == 0))
        (void)mbar_wait_bounded(&full[j % nbuf], uint32_t(j / nbuf) & 1u);
    return;
  }

  // ---- consumer warps ----
  unsigned char* const reg = regions + size_t(warp) * kFwdRegion;
  const uint32_t reg_a = smem_addr(reg);
  const uint32_t zero_a = smem_addr(zero);
  // phase-B roles: unit u8 of the step, corner r = (dy, dx), unit parity rho
  const int u8 = lane >> 2, r = lane & 3, dy = r >> 1, dx = r & 1, rho = u8 & 1;
  // piece rotation: bf16 lanes read pieces rho, 1 - rho; fp32 lanes read piece
  // j ^ rot in their j-th read, rot = 2 dy + rho; a one-piece pixel has none
  const int rot = NP == 1 ? 0 : (NP == 2 ? rho : 2 * dy + rho);
  const uint32_t corner_b = uint32_t((dy * t.BW + dx) * CS + 16 * rot);
  const int npx = t.TH * t.TW;
  const int nb = t.batches;
  const float Hf = float(t.H), Wf = float(t.W);
  const size_t pixB = size_t(t.C) * sizeof(T);
  const size_t x_bytes = size_t(t.N) * t.H * t.W * pixB;  // bounds-checked build
  const size_t out_bytes = size_t(t.N) * t.Ho * t.Wo * pixB;
  // the staging element e = lane + 32 k (k < KK) belongs to unit e / KK, tap e % KK
  int st_unit[KK], st_tap[KK];
#pragma unroll
  for (int k = 0; k < KK; ++k) {
    st_unit[k] = (lane + 32 * k) / KK;
    st_tap[k] = (lane + 32 * k) - st_unit[k] * KK;
  }

  // Unit of this lane in batch beta (over all the CTA's items): element offset
  // of its first offset pair / mask value, or ~0 outside the output.
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

  const size_t n_entries = size_t(t.N) * t.Ho * t.Wo * t.G * KK;  // offset pairs, mask values
  Pair pf_pair[KK];
  One pf_one[KK];
  auto prefetch = [&](int beta) {
    int ho, wo;
    uint32_t q;
    batch_unit(beta, ho, wo, q);
#pragma unroll
    for (int k = 0; k < KK; ++k) {
      const uint32_t src = __shfl_sync(0xFFFFFFFFu, q, st_unit[k]);
      const bool ok = src != ~0u && in_range(size_t(src) + st_tap[k], n_entries);
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
    // Every consumer warp observes every item's box, even one in which it has
    // no batch: that keeps each warp within nbuf - 1 items of the slowest, so
    // the parity it waits for is never ambiguous and it arrives on `empty`
    // exactly once per phase.
    if (!mbar_wait_bounded_sleep(&full[b], ph)) {
      atomicOr(a.error_word, kErrTimeout);
      *abort_flag = 1;
    }
    if (*abort_flag) break;
    const int item = int(blockIdx.x) + il * int(gridDim.x);
    const ItemCoord c = item_coord(t, item);
    const unsigned char* const box = bufs + size_t(b) * t.box_stride;
    const uint32_t box_a = smem_addr(box);
    const uint32_t lane_base = box_a + corner_b;
    const uint32_t zoff = zero_a - box_a;  // box-relative offset of the zero band
    const int Y0 = box_origin(c.ho0 * t.stride - t.pad - t.halo, t.BH, t.H, t.clamp_box);
    const int X0 = box_origin(c.wo0 * t.stride_w - t.pad_w - t.halo, t.BW, t.W, t.clamp_box);
    const char* const ximg = reinterpret_cast<const char*>(a.x) +
                             size_t(c.n) * t.H * t.W * pixB + size_t(c.g) * CS;

    for (; beta < (il + 1) * nb; beta += kTiledWarps) {
      // Staging: the prefetched inputs go to the region in their global order.
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
      // Phase-B steps that hold pixels of the tile: the last batch of a tile
      // whose pixel count is not a multiple of 32 is partly empty.  Only the
      // whole-image boxes (no far taps) get such tiles from the host's choice;
      // the far-tap kernel keeps a compile-time step count (a runtime one made
      // the stage-1 bf16 forward 3.5% slower).
      const int nsteps = FAR ? kTiledBatch / 8
                             : min(kTiledBatch / 8, (npx - (beta - il * nb) * kTiledBatch + 7) / 8);
      __syncwarp();

      // Phase A: this lane's unit -> softmax, then per tap the corner weights
      // and the box offset of corner (y0, x0).
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
        __syncwarp();  // every lane has read its staged inputs: the records overwrite them
        const int yb = ho * t.stride - t.pad, xb = wo * t.stride_w - t.pad_w;
        uint32_t fm = 0u;
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          const int ka = tap_pos(KK, k) / K, kb = tap_pos(KK, k) % K;
          const float Y = tap_coord(yb + ka * t.dil, t.sigma, d[k].y);
          const float X = tap_coord(xb + kb * t.dil_w, t.sigma, d[k].x);
          const float fy = floorf(Y), fx = floorf(X);
          const int y0 = __float2int_rd(Y), x0 = __float2int_rd(X);  // NaN -> 0, inf saturates
          const float ly = Y - fy, lx = X - fx;
          const int by = y0 - Y0, bx = x0 - X0;
          const bool inbox = unsigned(by) < unsigned(t.BH - 1) && unsigned(bx) < unsigned(t.BW - 1);
          const bool box_tap = valid && inbox && (Y == Y) && (X == X);
          const bool far = FAR && !box_tap && valid && (Y >= -1.0f) && (Y < Hf) &&
                           (X >= -1.0f) && (X < Wf);
          const float hy = 1.f - ly, hx = 1.f - lx;
          const float wy0 = hy * m[k], wy1 = ly * m[k];
          float4 w;
          if (box_tap)
            w = make_float4(wy0 * hx, wy0 * lx, wy1 * hx, wy1 * lx);
          else if (far)
            w = make_float4(wy0, wy1, lx,
                            __uint_as_float((uint32_t(y0 + 1) << kFarShift) | uint32_t(x0 + 1)));
          else
            w = make_float4(0.f, 0.f, 0.f, 0.f);
          reinterpret_cast<float4*>(reg + kFwdRegW)[k * kTiledBatch + lane] = w;
          reinterpret_cast<uint32_t*>(reg + kFwdRegOff)[k * kTiledBatch + lane] =
              box_tap ? uint32_t((by * t.BW + bx) * CS) : zoff;
          fm |= far ? (1u << k) : 0u;
        }
        reinterpret_cast<uint32_t*>(reg + kFwdRegFm)[lane] = fm;
        reinterpret_cast<uint32_t*>(reg + kFwdRegOut)[lane] =
            valid ? uint32_t(((c.n * t.Ho + ho) * t.Wo + wo) * t.C + c.g * t.Cg) : ~0u;
      }
      __syncwarp();
      // The next batch's inputs are loaded while this one is gathered.
      if (beta + kTiledWarps < total_batches) prefetch(beta + kTiledWarps);

      // Far taps: this lane's corner of tap k of unit u from global memory
      // (zeros outside the image) and its weight.
      auto far_fetch = [&](int u, int k, uint4 (&fv)[NP], float& fw) {
        const uint4 rw = lds128_a(reg_a + kFwdRegW + uint32_t(k * kTiledBatch + u) * 16u);
        const uint32_t pk = rw.w;
        const int yc = int(pk >> kFarShift) - 1 + dy;
        const int xc = int(pk & ((1u << kFarShift) - 1u)) - 1 + dx;
        const bool in = unsigned(yc) < unsigned(t.H) && unsigned(xc) < unsigned(t.W);
        const float lx = __uint_as_float(rw.z);
        fw = in ? __uint_as_float(dy ? rw.y : rw.x) * (dx ? lx : 1.f - lx) : 0.f;
        const char* gp = ximg + (size_t(in ? yc : 0) * t.W + (in ? xc : 0)) * pixB;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          const char* pp = gp + 16 * (j ^ rot);
          fv[j] = ldg128_pred(pp, in && in_tensor(pp, 16, a.x, x_bytes));
        }
      };
      // Phase B: 8 units per step, one lane per corner.
#pragma unroll 1
      for (int s = 0; s < nsteps; ++s) {
        const int u = s * 8 + u8;
        float2 acc[CG / 2];
#pragma unroll
        for (int i = 0; i < CG / 2; ++i) acc[i] = make_float2(0.f, 0.f);
        const uint32_t wa = reg_a + kFwdRegW + uint32_t(u) * 16u + uint32_t(r) * 4u;
        const uint32_t oa = reg_a + kFwdRegOff + uint32_t(u) * 4u;
#pragma unroll
        for (int k = 0; k < KK; ++k) {
          float w;
          uint32_t off;
          asm volatile("ld.shared.f32 %0, [%1];" : "=f"(w) : "r"(wa + k * kTiledBatch * 16));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(off) : "r"(oa + k * kTiledBatch * 4));
          const float2 w2 = make_float2(w, w);
          const uint32_t a0 = lane_base + off;
#pragma unroll
          for (int j = 0; j < NP; ++j)
            IO::fma16(acc + j * PA, w2, lds128_a(a0 ^ uint32_t(16 * j)));
        }
        if (FAR) {
          // The unit's far taps, in a warp-uniform loop.  (Fetching the first
          // one a step ahead cost more in registers and per-step work than it
          // saved: 4-6% slower at the stage shapes.)
          uint32_t fm;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(fm) : "r"(reg_a + kFwdRegFm + 4u * u));
          while (__any_sync(0xFFFFFFFFu, fm != 0u)) {
            if (fm != 0u) {
              uint4 fv[NP];
              float fw;
              far_fetch(u, __ffs(fm) - 1, fv, fw);
#pragma unroll
              for (int j = 0; j < NP; ++j)
                IO::fma16(acc + j * PA, make_float2(fw, fw), fv[j]);
              fm &= fm - 1u;
            }
          }
        }
        // Reduce-scatter over the unit's four corner lanes, then store.
        uint32_t ob;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(ob) : "r"(reg_a + kFwdRegOut + 4u * u));
        if constexpr (NP == 1) {
          // acc[0..3]: the 8 channels.  dx partner: keep channels 4 dx ..
          // 4 dx + 3, then dy partner: keep the pair 4 dx + 2 dy.
          float2 k2[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float2 keep = dx ? acc[2 + i] : acc[i];
            const float2 send = dx ? acc[i] : acc[2 + i];
            k2[i].x = keep.x + __shfl_xor_sync(0xFFFFFFFFu, send.x, 1);
            k2[i].y = keep.y + __shfl_xor_sync(0xFFFFFFFFu, send.y, 1);
          }
          const float2 keep = dy ? k2[1] : k2[0];
          const float2 send = dy ? k2[0] : k2[1];
          const float o0 = keep.x + __shfl_xor_sync(0xFFFFFFFFu, send.x, 2);
          const float o1 = keep.y + __shfl_xor_sync(0xFFFFFFFFu, send.y, 2);
          if (ob != ~0u) {
            char* op = reinterpret_cast<char*>(a.out) +
                       (size_t(ob) + size_t(4 * dx + 2 * dy)) * sizeof(T);
            if (in_tensor(op, 4, a.out, out_bytes))
              asm volatile("st.global.b32 [%0], %1;" ::"l"(op), "r"(pack2<T>(o0, o1)) : "memory");
          }
        } else if constexpr (NP == 2) {
          // acc[0..3]: piece rho (channels 8 rho ..), acc[4..7]: piece 1 - rho.
          // dx partner: keep piece rho ^ dx, then dy partner: keep half dy of it.
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
          // slot j = acc[2j, 2j+1] holds piece j ^ rot, rot = 2 dy + rho.  The dy
          // partner's rot differs in bit 1: both keep slots 0, 1 and add the
          // partner's slots 2, 3 (the same pieces).  Then the dx partner (same
          // rot) splits slots 0 and 1.
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
            char* op = reinterpret_cast<char*>(a.out) +
                       (size_t(ob) + size_t(4 * (dx ^ rot))) * sizeof(T);
            if (in_tensor(op, 16, a.out, out_bytes))
              asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(op), "f"(k2[0].x),
                           "f"(k2[0].y), "f"(k2[1].x), "f"(k2[1].y)
                           : "memory");
          }
        }
      }
      __syncwarp();  // the region is rewritten by the next batch
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);
    if (++b == nbuf) {
      b = 0;
      ph ^= 1u;
    }
  }
}

}  // namespace dcn
