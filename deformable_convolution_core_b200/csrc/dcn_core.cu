// C ABI of the B200 deformable-convolution core: argument validation, tile
// choice, kernel dispatch.  Declarations and the full contract are in
// include/dcn_core.h.
#include "dcn_core.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <numeric>

#include "dcn_backward.cuh"
#include "dcn_backward_tiled.cuh"
#include "dcn_forward.cuh"
#include "dcn_forward_tiled.cuh"
#include "dcn_forward_tiled_wide.cuh"
#include "dcn_guide.cuh"
#include "dcn_guide_projection.cuh"
#include "dcn_projection.cuh"

namespace dcn {
namespace {

// Shared memory a CTA may use for its staged offsets and mask, by default.
constexpr int kDefaultSmemBudget = 40 * 1024;

int64_t out_extent(int in, int K, int stride, int pad, int dil) {
  const int64_t span = int64_t(in) + 2 * int64_t(pad) - int64_t(dil) * (K - 1) - 1;
  if (span < 0 || stride < 1) return 0;
  return span / stride + 1;
}

int esize(dcn_dtype d) { return d == DCN_F32 ? 4 : 2; }

// Calls f with a value of the storage type of d (fp32, bf16 or fp16).
template <typename F>
auto with_storage(dcn_dtype d, F&& f) {
  switch (d) {
    case DCN_BF16: return f(__nv_bfloat16());
    case DCN_F16: return f(__half());
    default: return f(float());
  }
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Width-axis stride, padding and dilation: the height ones unless separate_axes.
int stride_w(const dcn_problem* p) { return p->separate_axes ? p->stride_w : p->stride; }
int pad_w(const dcn_problem* p) { return p->separate_axes ? p->pad_w : p->pad; }
int dil_w(const dcn_problem* p) { return p->separate_axes ? p->dilation_w : p->dilation; }

// Taps per (pixel, group): the K x K window, less its centre with remove_center.
int taps(const dcn_problem* p) { return p->K * p->K - (p->remove_center ? 1 : 0); }

// Compile-time tap set of a problem: 9 (3 x 3 window), 8 (3 x 3 without its
// centre), or 0 (any other window, counted at run time).
int compile_time_taps(const dcn_problem* p) {
  if (p->K != 3) return 0;
  return p->remove_center ? 8 : 9;
}

// Basic validity of the problem description.
dcn_status check_problem(const dcn_problem* p, int64_t* Ho, int64_t* Wo) {
  if (!p) return DCN_ERR_INVALID_ARG;
  if (p->N < 1 || p->H < 1 || p->W < 1 || p->G < 1 || p->Cg < 1) return DCN_ERR_INVALID_ARG;
  if (p->K < 1 || (p->K % 2) == 0) return DCN_ERR_INVALID_ARG;
  if (p->stride < 1 || p->pad < 0 || p->dilation < 1) return DCN_ERR_INVALID_ARG;
  if (p->separate_axes != 0 && p->separate_axes != 1) return DCN_ERR_INVALID_ARG;
  if (stride_w(p) < 1 || pad_w(p) < 0 || dil_w(p) < 1) return DCN_ERR_INVALID_ARG;
  if (p->softmax != 0 && p->softmax != 1) return DCN_ERR_INVALID_ARG;
  if (p->remove_center != 0 && p->remove_center != 1) return DCN_ERR_INVALID_ARG;
  if (p->remove_center && p->K < 3) return DCN_ERR_INVALID_ARG;  // no tap would be left
  if (p->dtype != DCN_F32 && p->dtype != DCN_BF16 && p->dtype != DCN_F16)
    return DCN_ERR_INVALID_ARG;
  if (!(p->offset_scale == p->offset_scale)) return DCN_ERR_INVALID_ARG;  // NaN
  const int64_t ho = out_extent(p->H, p->K, p->stride, p->pad, p->dilation);
  const int64_t wo = out_extent(p->W, p->K, stride_w(p), pad_w(p), dil_w(p));
  if (ho < 1 || wo < 1) return DCN_ERR_INVALID_ARG;
  const int64_t C = int64_t(p->G) * p->Cg;
  const int64_t KK = taps(p);
  const int64_t n_in = int64_t(p->N) * p->H * p->W * C;
  const int64_t n_out = int64_t(p->N) * ho * wo * C;
  const int64_t n_off = int64_t(p->N) * ho * wo * p->G * KK * 2;
  const int64_t lim = int64_t(INT_MAX);
  if (C > lim || n_in > lim || n_out > lim || n_off > lim) return DCN_ERR_INVALID_ARG;
  // Sampling coordinates are integers up to about H*stride + K*dilation in fp32.
  if (int64_t(p->H) * p->stride + int64_t(p->K) * p->dilation > (int64_t(1) << 22) ||
      int64_t(p->W) * stride_w(p) + int64_t(p->K) * dil_w(p) > (int64_t(1) << 22))
    return DCN_ERR_UNSUPPORTED;
  *Ho = ho;
  *Wo = wo;
  return DCN_OK;
}

// Lane mapping for a channel width: bytes of one unit's channels UB =
// Cg*sizeof(T) in {16, 32, 64, 128}; a lane gathers 16 (UB = 16) or 32 bytes.
struct LaneMap {
  int cpl, lanes;
};

bool lane_map(const dcn_problem* p, LaneMap* lm) {
  const int ub = p->Cg * esize(p->dtype);
  const int e = esize(p->dtype);
  switch (ub) {
    case 16: *lm = {16 / e, 1}; return true;
    case 32: *lm = {32 / e, 1}; return true;
    case 64: *lm = {32 / e, 2}; return true;
    case 128: *lm = {32 / e, 4}; return true;
    default: return false;
  }
}

bool backward_lane_map(const dcn_problem* p, LaneMap* lm);

struct Plan {
  TileParams t;
  size_t smem;
  unsigned grid;
  LaneMap lm;
};

// Pick the tile (TH x TW output pixels, all groups).  The cost model counts
// warp passes including those wasted on the ragged border, weighted by how
// much of the gathered neighbourhood of a tile is halo (which costs L1 misses).
void choose_tile(int Ho, int Wo, int G, int lanes, size_t entry_bytes, int KK, size_t budget,
                 int* TH_out, int* TW_out) {
  const int upw = 32 / lanes;
  const size_t per_px = size_t(G) * KK * entry_bytes;
  int max_px = int(std::max<size_t>(1, budget / per_px));
  max_px = std::min(max_px, 1024);
  const double halo = 3.0;
  double best = 1e300;
  int bth = 1, btw = 1;
  for (int th = 1; th <= std::min(Ho, max_px); ++th) {
    for (int tw = 1; tw <= std::min(Wo, max_px / th); ++tw) {
      const int px = th * tw;
      const int64_t tiles = int64_t((Ho + th - 1) / th) * ((Wo + tw - 1) / tw);
      const int64_t passes = tiles * ((int64_t(G) * px + upw - 1) / upw);
      const double reach = (th + 2 * halo) * (tw + 2 * halo) / double(px);
      const double cost = double(passes) * (1.0 + 0.25 * reach) + 4.0 * double(tiles);
      if (cost < best) {
        best = cost;
        bth = th;
        btw = tw;
      }
    }
  }
  *TH_out = bth;
  *TW_out = btw;
}

dcn_status make_plan(const dcn_problem* p, int64_t Ho, int64_t Wo, size_t entry_bytes,
                     Plan* plan, bool backward = false) {
  if (!(backward ? backward_lane_map(p, &plan->lm) : lane_map(p, &plan->lm)))
    return DCN_ERR_UNSUPPORTED;
  TileParams& t = plan->t;
  t.N = p->N; t.H = p->H; t.W = p->W; t.G = p->G; t.Cg = p->Cg; t.C = p->G * p->Cg;
  t.K = p->K; t.KK = taps(p); t.stride = p->stride; t.pad = p->pad; t.dil = p->dilation;
  t.stride_w = stride_w(p); t.pad_w = pad_w(p); t.dil_w = dil_w(p);
  t.kc = p->remove_center ? (p->K * p->K) / 2 : -1;
  t.Ho = int(Ho); t.Wo = int(Wo); t.sigma = p->offset_scale;
  size_t budget = kDefaultSmemBudget;
  if (const char* s = std::getenv("DCN_CORE_SMEM_BUDGET")) budget = size_t(std::atol(s));
  int TH = 0, TW = 0;
  if (const char* s = std::getenv("DCN_CORE_TILE")) {  // "THxTW", for tuning sweeps
    if (std::sscanf(s, "%dx%d", &TH, &TW) != 2 || TH < 1 || TW < 1) TH = TW = 0;
    TH = std::min(TH, t.Ho);
    TW = std::min(TW, t.Wo);
  }
  if (TH == 0) choose_tile(t.Ho, t.Wo, t.G, plan->lm.lanes, entry_bytes, t.KK, budget, &TH, &TW);
  t.TH = TH; t.TW = TW;
  t.nTY = (t.Ho + TH - 1) / TH;
  t.nTX = (t.Wo + TW - 1) / TW;
  t.tile_px = TH * TW;
  t.P1 = t.tile_px | 1;
  t.fd_tile_px = make_fastdiv(uint32_t(t.tile_px));
  t.fd_TW = make_fastdiv(uint32_t(TW));
  t.fd_GKK = make_fastdiv(uint32_t(t.G * t.KK));
  t.fd_tiles_per_img = make_fastdiv(uint32_t(t.nTY * t.nTX));
  t.fd_nTX = make_fastdiv(uint32_t(t.nTX));
  plan->smem = size_t(t.G) * t.KK * t.P1 * entry_bytes;
  const int64_t tiles = int64_t(t.N) * t.nTY * t.nTX;
  if (tiles > INT_MAX) return DCN_ERR_UNSUPPORTED;
  plan->grid = unsigned(tiles);
  return DCN_OK;
}

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}

// Dynamic shared memory above 48 KB needs an opt-in per kernel and device.
template <typename Kernel>
dcn_status prepare_smem(Kernel k, size_t smem) {
  if (smem <= 48 * 1024) return DCN_OK;
  int dev = current_device();
  int max_optin = 0;
  if (cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
      cudaSuccess)
    return DCN_ERR_CUDA;
  if (smem > size_t(max_optin)) return DCN_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return DCN_ERR_CUDA;
  return DCN_OK;
}

template <typename Kernel, typename Args>
dcn_status launch(Kernel k, const Plan& plan, const Args& args, cudaStream_t stream) {
  dcn_status st = prepare_smem(k, plan.smem);
  if (st != DCN_OK) return st;
  k<<<plan.grid, kThreads, plan.smem, stream>>>(args);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

template <typename T, int CPL, int LANES, bool SOFTMAX>
dcn_status forward_dispatch_sm(const dcn_problem* p, const Plan& plan, const FwdArgs& args,
                               cudaStream_t stream) {
  switch (compile_time_taps(p)) {
    case 9: return launch(dcn_forward_kernel<T, CPL, LANES, 9, SOFTMAX>, plan, args, stream);
    case 8: return launch(dcn_forward_kernel<T, CPL, LANES, 8, SOFTMAX>, plan, args, stream);
    default: return launch(dcn_forward_kernel<T, CPL, LANES, 0, SOFTMAX>, plan, args, stream);
  }
}

template <typename T, int CPL, int LANES>
dcn_status forward_dispatch_kk(const dcn_problem* p, const Plan& plan, const FwdArgs& args,
                               cudaStream_t stream) {
  return p->softmax ? forward_dispatch_sm<T, CPL, LANES, true>(p, plan, args, stream)
                    : forward_dispatch_sm<T, CPL, LANES, false>(p, plan, args, stream);
}

template <typename T>
dcn_status forward_dispatch(const dcn_problem* p, const Plan& plan, const FwdArgs& args,
                            cudaStream_t stream) {
  constexpr int e = sizeof(T);
  const int cpl = plan.lm.cpl, lanes = plan.lm.lanes;
  if (cpl == 16 / e && lanes == 1) return forward_dispatch_kk<T, 16 / e, 1>(p, plan, args, stream);
  if (cpl == 32 / e && lanes == 1) return forward_dispatch_kk<T, 32 / e, 1>(p, plan, args, stream);
  if (cpl == 32 / e && lanes == 2) return forward_dispatch_kk<T, 32 / e, 2>(p, plan, args, stream);
  if (cpl == 32 / e && lanes == 4) return forward_dispatch_kk<T, 32 / e, 4>(p, plan, args, stream);
  return DCN_ERR_UNSUPPORTED;
}

template <typename T, int LANES, bool SOFTMAX, bool DET>
dcn_status backward_dispatch_sm(const dcn_problem* p, const Plan& plan, const BwdArgs& args,
                                cudaStream_t stream) {
  switch (compile_time_taps(p)) {
    case 9: return launch(dcn_backward_kernel<T, LANES, 9, SOFTMAX, DET>, plan, args, stream);
    case 8: return launch(dcn_backward_kernel<T, LANES, 8, SOFTMAX, DET>, plan, args, stream);
    default: return launch(dcn_backward_kernel<T, LANES, 0, SOFTMAX, DET>, plan, args, stream);
  }
}

template <typename T, int LANES, bool DET>
dcn_status backward_dispatch_kk(const dcn_problem* p, const Plan& plan, const BwdArgs& args,
                                cudaStream_t stream) {
  return p->softmax ? backward_dispatch_sm<T, LANES, true, DET>(p, plan, args, stream)
                    : backward_dispatch_sm<T, LANES, false, DET>(p, plan, args, stream);
}

// The backward always gives a lane 4 channels (16 bytes), so that one warp
// instruction covers a unit's whole corner chunk: a gather or a float4 atomic
// touches one cache line per (unit, corner) instead of one per lane.
bool backward_lane_map(const dcn_problem* p, LaneMap* lm) {
  switch (p->Cg) {
    case 4: *lm = {4, 1}; return true;
    case 8: *lm = {4, 2}; return true;
    case 16: *lm = {4, 4}; return true;
    case 32: *lm = {4, 8}; return true;
    case 64: *lm = {4, 16}; return true;
    default: return false;
  }
}

template <typename T, bool DET>
dcn_status backward_dispatch_t(const dcn_problem* p, const Plan& plan, const BwdArgs& args,
                               cudaStream_t stream) {
  switch (plan.lm.lanes) {
    case 1: return backward_dispatch_kk<T, 1, DET>(p, plan, args, stream);
    case 2: return backward_dispatch_kk<T, 2, DET>(p, plan, args, stream);
    case 4: return backward_dispatch_kk<T, 4, DET>(p, plan, args, stream);
    case 8: return backward_dispatch_kk<T, 8, DET>(p, plan, args, stream);
    case 16: return backward_dispatch_kk<T, 16, DET>(p, plan, args, stream);
    default: return DCN_ERR_UNSUPPORTED;
  }
}

// det: the accumulator is 64-bit fixed point (the deterministic backward).
dcn_status backward_dispatch(const dcn_problem* p, const Plan& plan, const BwdArgs& args,
                             bool det, cudaStream_t stream) {
  return with_storage(p->dtype, [&](auto tag) {
    using T = decltype(tag);
    return det ? backward_dispatch_t<T, true>(p, plan, args, stream)
               : backward_dispatch_t<T, false>(p, plan, args, stream);
  });
}

// Bytes of the fp32 grad_input accumulator that 2-byte storage (bf16, fp16) needs.
size_t bf16_accumulator_bytes(const dcn_problem* p) {
  return size_t(p->N) * p->H * p->W * p->G * p->Cg * sizeof(float);
}

dcn_status check_forward_pointers(const dcn_problem* p, const void* x, const void* off,
                                  const void* mask, const void* out) {
  if (!x || !off || !mask || !out) return DCN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(off, 16) || !aligned(mask, 16) || !aligned(out, 16))
    return DCN_ERR_UNSUPPORTED;
  LaneMap lm;
  if (!lane_map(p, &lm)) return DCN_ERR_UNSUPPORTED;
  const size_t vb = size_t(lm.cpl) * esize(p->dtype);  // per-lane vector: 16 or 32 bytes
  if (!aligned(x, vb) || !aligned(out, vb)) return DCN_ERR_UNSUPPORTED;
  return DCN_OK;
}


// ---------------------------------------------------------------------------
// Tiled forward (input box staged by TMA).
// ---------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// Unique id of the current CUDA context (cuCtxGetId; 0 if it cannot be
// read).  The per-device state the library keeps (the error word's address,
// the host entry points' streams and events, the allocation-free backward's
// array address) is tagged with it: after cudaDeviceReset the device has a
// new context and the state is created again instead of being reused.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_cur = []() -> PFN_cuCtxGetCurrent_v4000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  }();
  static PFN_cuCtxGetId_v12000 get_id = []() -> PFN_cuCtxGetId_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  }();
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&c) != CUDA_SUCCESS || c == nullptr ||
      get_id(c, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;
  unsigned int* error_word = nullptr;
};

// Per-device constants, looked up once per device (under a lock: calls may
// come from several host threads).
dcn_status device_info(DeviceInfo* out) {
  constexpr int kMaxDev = 64;
  static DeviceInfo cache[kMaxDev];
  static bool ready[kMaxDev] = {};
  static unsigned long long ctx[kMaxDev] = {};  // context the entry was made in
  static std::mutex lock;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return DCN_ERR_CUDA;
  std::lock_guard<std::mutex> guard(lock);
  const unsigned long long id = current_context_id();
  if (!ready[dev] || ctx[dev] != id) {
    DeviceInfo d;
    void* ew = nullptr;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaGetSymbolAddress(&ew, g_dcn_error_word) != cudaSuccess)
      return DCN_ERR_CUDA;
    d.error_word = static_cast<unsigned int*>(ew);
    cache[dev] = d;
    ctx[dev] = id;
    ready[dev] = true;
  }
  *out = cache[dev];
  return DCN_OK;
}

int env_int(const char* name, int dflt) {
  const char* s = std::getenv(name);
  return s ? std::atoi(s) : dflt;
}

bool tiled_eligible(const dcn_problem* p, int64_t Ho, int64_t Wo) {
  const char* mode = std::getenv("DCN_CORE_FORWARD");
  if (mode && std::strcmp(mode, "direct") == 0) return false;
  // 16 channels per group in any storage type: 32-byte 2-byte-type groups or
  // 64-byte fp32 groups (eight accumulated values per phase-B lane); 3x3
  // windows, and 5x5 and 7x7 ones in the wide-window kernel.  The 3x3 kernel
  // also takes 8 channels of a 2-byte type (16-byte groups).
  const bool cg8 = p->K == 3 && p->Cg == 8 && esize(p->dtype) == 2;
  if (!cg8 && ((p->K != 3 && p->K != 5 && p->K != 7) || p->Cg != 16)) return false;
  if (p->H > 16000 || p->W > 16000 || Ho > 16000 || Wo > 16000) return false;
  return tensor_map_encoder() != nullptr;
}

// Box row pitch (pixels) that makes the footprint reads conflict-free: for
// 32-byte groups the two rows of a footprint must fall into complementary
// halves of the 32 banks (pitch = 2 mod 4); for 64-byte groups the pitch
// must be even (the lanes' piece rotation does the rest).  16-byte groups
// take pitch = 4 mod 8: a unit's four corners then sit in four distinct
// 16-byte bank groups, and the two units of a quarter-warp meet at most two
// to a bank group (no pitch keeps every random pair apart).
int box_pitch(int bw, int cs) {
  if (cs == 32) return bw + (2 - bw % 4 + 4) % 4;
  if (cs == 16) return bw + (4 - bw % 8 + 8) % 8;
  return bw + (bw & 1);
}

// Units per warp batch of the tiled kernels: 32 for 3x3 windows, 8 in the
// wide-window kernel (5x5, 7x7).
int tiled_batch(const dcn_problem* p) { return p->K == 3 ? kTiledBatch : kWideUnits; }

// Box extent along one axis for a tile of `tile` outputs.
int box_extent(int tile, int stride, int dil, int halo, int K) {
  return (tile - 1) * stride + (K - 1) * dil + 2 + 2 * halo;
}

// Launch a persistent tiled kernel: as many CTAs as fit on the GPU at once,
// never more than there are items.
template <typename Kernel, typename Args>
dcn_status launch_persistent(Kernel k, const CUtensorMap& map, const Args& args, size_t smem,
                             int sms, cudaStream_t stream) {
  // Driver calls made once, not per launch: the kernel's dynamic shared-memory
  // limit (per context and kernel; only ever raised, since a lower limit would
  // refuse an earlier, larger configuration) and its occupancy (per context,
  // kernel and byte count).
  using KernelKey = std::pair<unsigned long long, const void*>;
  using OccKey = std::tuple<unsigned long long, const void*, size_t>;
  static std::map<KernelKey, size_t> smem_limit;
  static std::map<OccKey, int> blocks_per_sm;
  static std::mutex lock;
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> guard(lock);
    const unsigned long long ctx = current_context_id();
    const void* kp = reinterpret_cast<const void*>(k);
    auto lim = smem_limit.find(KernelKey{ctx, kp});
    if (lim == smem_limit.end() || lim->second < smem) {
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
          cudaSuccess)
        return DCN_ERR_CUDA;
      smem_limit[KernelKey{ctx, kp}] = smem;
    }
    const OccKey key{ctx, kp, smem};
    auto it = blocks_per_sm.find(key);
    if (it == blocks_per_sm.end()) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kTiledThreads, smem) !=
          cudaSuccess)
        return DCN_ERR_UNSUPPORTED;
      if (blocks_per_sm.size() > 4096) blocks_per_sm.clear();
      it = blocks_per_sm.emplace(key, per_sm).first;
    }
    per_sm = it->second;
  }
  if (per_sm < 1) return DCN_ERR_UNSUPPORTED;
  const int64_t grid = std::min<int64_t>(args.t.items, int64_t(sms) * per_sm);
  k<<<unsigned(grid), kTiledThreads, smem, stream>>>(map, args);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

template <typename T, bool FAR, int CG>
dcn_status forward_tiled_dispatch_cg(const dcn_problem* p, const CUtensorMap& map,
                                     const TiledArgs& args, size_t smem, int sms,
                                     cudaStream_t stream) {
  if (p->remove_center)
    return p->softmax
               ? launch_persistent(dcn_forward_tiled_kernel<T, 8, true, FAR, CG>, map, args, smem, sms, stream)
               : launch_persistent(dcn_forward_tiled_kernel<T, 8, false, FAR, CG>, map, args, smem, sms, stream);
  return p->softmax
             ? launch_persistent(dcn_forward_tiled_kernel<T, 9, true, FAR, CG>, map, args, smem, sms, stream)
             : launch_persistent(dcn_forward_tiled_kernel<T, 9, false, FAR, CG>, map, args, smem, sms, stream);
}

template <typename T, bool FAR>
dcn_status forward_tiled_dispatch_far(const dcn_problem* p, const CUtensorMap& map,
                                      const TiledArgs& args, size_t smem, int sms,
                                      cudaStream_t stream) {
  if constexpr (sizeof(T) == 2)
    if (p->Cg == 8) return forward_tiled_dispatch_cg<T, FAR, 8>(p, map, args, smem, sms, stream);
  return forward_tiled_dispatch_cg<T, FAR, 16>(p, map, args, smem, sms, stream);
}

template <typename T>
dcn_status forward_tiled_dispatch(const dcn_problem* p, const CUtensorMap& map,
                                  const TiledArgs& args, bool far, size_t smem, int sms,
                                  cudaStream_t stream) {
  return far ? forward_tiled_dispatch_far<T, true>(p, map, args, smem, sms, stream)
             : forward_tiled_dispatch_far<T, false>(p, map, args, smem, sms, stream);
}

template <typename T, bool DET, bool FAR>
dcn_status backward_tiled_dispatch_far(const dcn_problem* p, const CUtensorMap& map,
                                       const TiledBwdArgs& args, size_t smem, int sms,
                                       cudaStream_t stream) {
  if (p->remove_center)
    return p->softmax
               ? launch_persistent(dcn_backward_tiled_kernel<T, 8, true, DET, FAR>, map, args, smem, sms, stream)
               : launch_persistent(dcn_backward_tiled_kernel<T, 8, false, DET, FAR>, map, args, smem, sms, stream);
  return p->softmax
             ? launch_persistent(dcn_backward_tiled_kernel<T, 9, true, DET, FAR>, map, args, smem, sms, stream)
             : launch_persistent(dcn_backward_tiled_kernel<T, 9, false, DET, FAR>, map, args, smem, sms, stream);
}

template <typename T, bool DET>
dcn_status backward_tiled_dispatch(const dcn_problem* p, const CUtensorMap& map,
                                   const TiledBwdArgs& args, bool far, size_t smem, int sms,
                                   cudaStream_t stream) {
  return far ? backward_tiled_dispatch_far<T, DET, true>(p, map, args, smem, sms, stream)
             : backward_tiled_dispatch_far<T, DET, false>(p, map, args, smem, sms, stream);
}

// Input tensor map viewed as (C, W, H, N), innermost first; one box is
// (Cg, BW, BH, 1) starting at (g*Cg, X0, Y0, n).  Outside the tensor the box
// is zero filled, which is exactly the operator's zero padding.
dcn_status encode_input_map(const dcn_problem* p, const TiledParams& t, const void* x,
                            CUtensorMap* map) {
  const int e = esize(p->dtype);
  const cuuint64_t dims[4] = {cuuint64_t(t.C), cuuint64_t(t.W), cuuint64_t(t.H),
                              cuuint64_t(t.N)};
  const cuuint64_t strides[3] = {cuuint64_t(t.C) * e, cuuint64_t(t.W) * t.C * e,
                                 cuuint64_t(t.H) * t.W * t.C * e};
  const cuuint32_t box[4] = {cuuint32_t(t.Cg), cuuint32_t(t.BW), cuuint32_t(t.BH), 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUresult cr = tensor_map_encoder()(
      map,
      p->dtype == DCN_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
      : p->dtype == DCN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
      4, const_cast<void*>(x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cr == CUDA_SUCCESS ? DCN_OK : DCN_ERR_UNSUPPORTED;
}

// Forward tile choice.  The box of a tile is clamped to the image and its
// zero ring, so a tile near the border gets more halo inside and a small
// image's box covers it all (no far taps).  Cost, in lane-samples: every
// batch of 32 units costs its taps whether its lanes are used or not; an item
// costs a fixed overhead and its box fill; where footprints can leave the
// box, taps near the tile's edges go to global memory at several times the
// cost.  Boxes must leave room for at least two in flight.
struct FwdTile {
  int TH = 0, TW = 0, BH = 0, BW = 0, nbuf = 0;
  uint32_t box_bytes = 0, box_stride = 0;
  bool far = true;
};

int clamp_extent(int box, int extent) { return std::min(box, extent + 2); }

bool fwd_tile_geometry(const dcn_problem* p, int TH, int TW, int cs, int halo, size_t optin,
                       FwdTile* f) {
  f->TH = TH;
  f->TW = TW;
  f->BH = clamp_extent(box_extent(TH, p->stride, p->dilation, halo, p->K), p->H);
  f->BW = box_pitch(clamp_extent(box_extent(TW, stride_w(p), dil_w(p), halo, p->K), p->W), cs);
  if (f->BH > 256 || f->BW > 256) return false;
  f->box_bytes = uint32_t(size_t(f->BH) * f->BW * cs);
  f->box_stride = (f->box_bytes + 1023u) / 1024u * 1024u;
  const size_t fixed = fwd_tiled_smem(0, 0, f->BW, cs);
  if (optin <= fixed) return false;
  f->nbuf = int(std::min<size_t>(kTiledMaxBufs, (optin - fixed) / f->box_stride));
  if (f->nbuf < 2) return false;
  f->far = !(f->BH >= p->H + 2 && f->BW >= p->W + 2);
  return true;
}

// Tile choice: the shape that minimises a per-item cost times the rounds of
// items each persistent CTA runs.  Per item: the lane-samples of its batches,
// the far taps (about 0.3 (1/TH + 1/TW) of them leave the box), the box pixels
// the producer loads, and a penalty for fewer than three boxes in flight.  The
// rounds are counted for a reference batch of 64 images, not the problem's N:
// the choice, and with it which taps the box serves (the last bits of the
// forward), then does not depend on how a batch is split.  The weights were
// fitted to measured times of tile shapes on the InternImage-L stage shapes
// and the 256 x 256 DCNv4 shape.
void choose_fwd_tile(const dcn_problem* p, int Ho, int Wo, int cs, int halo, size_t optin,
                     int ctas, FwdTile* out) {
  double best = 1e300;
  for (int th = 1; th <= std::min(Ho, 64); ++th) {
    for (int tw = 1; tw <= std::min(Wo, 64); ++tw) {
      FwdTile f;
      if (!fwd_tile_geometry(p, th, tw, cs, halo, optin, &f)) continue;
      constexpr int64_t kRefImages = 64;
      const int64_t items = int64_t((Ho + th - 1) / th) * ((Wo + tw - 1) / tw) * kRefImages * p->G;
      const int64_t rounds = (items + ctas - 1) / std::max(ctas, 1);
      const int px = th * tw;
      const int bu = tiled_batch(p);
      const double lane_samples = double((px + bu - 1) / bu) * bu * taps(p);
      const double far_frac = f.far ? 0.3 * (1.0 / th + 1.0 / tw) : 0.0;
      const double per_item = lane_samples * (1.0 + far_frac) + 0.5 * double(f.box_bytes) / cs +
                              (f.nbuf < 3 ? 200.0 : 0.0);
      const double cost = double(rounds) * per_item;
      if (cost < best) {
        best = cost;
        *out = f;
      }
    }
  }
}

struct BoxLaunch {
  TiledParams t;
  CUtensorMap map;
  size_t smem;
  DeviceInfo dev;
  bool far;
};

// reserve: shared memory the kernel needs beyond the forward's layout (the
// deterministic backward's staging slots); the boxes get what is left.
dcn_status box_tiled_prepare(const dcn_problem* p, int64_t Ho, int64_t Wo, const void* x,
                             const char* tile_env, BoxLaunch* L, size_t reserve = 0) {
  dcn_status st = device_info(&L->dev);
  if (st != DCN_OK) return st;
  const int cs = p->Cg * esize(p->dtype);
  // Default halo (pixels of box around the tile's sampling window): 4 for
  // 64-byte groups, 5 for 32-byte ones, 3 for 16-byte ones.  A wider halo
  // turns more far taps into box reads but shrinks the tile the shared memory
  // allows; measured on the InternImage-L stage-1 shapes, 4 is the fastest for
  // fp32 (forward 0.437 ms against 0.459 at 5), 5 for bf16 and fp16, and 3 for
  // 8 bf16 channels (1.039 ms against 1.092 at 4 and 1.208 at 5).
  const int halo = std::max(0, env_int("DCN_CORE_HALO", cs == 64 ? 4 : (cs == 16 ? 3 : 5)));
  if (size_t(L->dev.smem_optin) <= reserve) return DCN_ERR_UNSUPPORTED;
  const size_t optin = size_t(L->dev.smem_optin) - reserve;
  FwdTile f;
  int TH = 0, TW = 0;
  if (const char* s = std::getenv(tile_env)) {  // "THxTW", for tuning sweeps
    if (std::sscanf(s, "%dx%d", &TH, &TW) != 2 || TH < 1 || TW < 1) TH = TW = 0;
  }
  if (TH > 0) {
    if (!fwd_tile_geometry(p, std::min<int>(TH, int(Ho)), std::min<int>(TW, int(Wo)), cs, halo,
                           optin, &f))
      return DCN_ERR_UNSUPPORTED;
  } else {
    // The search costs tens of microseconds of host time: remember its answer
    // for each problem shape (everything the choice depends on is in the key).
    using Key = std::tuple<int, int, int, int, int, int, int, int, int, int, int, int, int, int,
                           int, size_t, int>;
    static std::map<Key, FwdTile> memo;
    static std::mutex memo_lock;
    const Key key{0, p->H, p->W, int(Ho), int(Wo), p->G, p->K, p->stride, stride_w(p),
                  p->dilation, dil_w(p), p->remove_center, cs, halo, tiled_batch(p), optin,
                  L->dev.sms};
    std::lock_guard<std::mutex> guard(memo_lock);
    auto it = memo.find(key);
    if (it == memo.end()) {
      f = FwdTile{};
      choose_fwd_tile(p, int(Ho), int(Wo), cs, halo, optin, L->dev.sms, &f);
      if (memo.size() > 4096) memo.clear();  // bound the host memory a long run can use
      it = memo.emplace(key, f).first;
    }
    f = it->second;
    if (f.nbuf == 0) return DCN_ERR_UNSUPPORTED;
  }
  if (const int nb = env_int("DCN_CORE_TILED_BUFS", 0); nb >= 2 && nb < f.nbuf) f.nbuf = nb;

  TiledParams& t = L->t;
  t.N = p->N; t.H = p->H; t.W = p->W; t.G = p->G; t.Cg = p->Cg; t.C = p->G * p->Cg;
  t.stride = p->stride; t.pad = p->pad; t.dil = p->dilation; t.Ho = int(Ho); t.Wo = int(Wo);
  t.stride_w = stride_w(p); t.pad_w = pad_w(p); t.dil_w = dil_w(p);
  t.sigma = p->offset_scale; t.halo = halo; t.TH = f.TH; t.TW = f.TW;
  t.inject_stall = env_int("DCN_CORE_TEST_STALL", 0) == 1 ? 1 : 0;
  t.nTY = (t.Ho + t.TH - 1) / t.TH;
  t.nTX = (t.Wo + t.TW - 1) / t.TW;
  t.BH = f.BH;
  t.BW = f.BW;
  t.clamp_box = 1;
  t.nbuf = f.nbuf;
  t.box_bytes = f.box_bytes;
  t.box_stride = f.box_stride;
  const int64_t items = int64_t(t.N) * t.nTY * t.nTX * t.G;
  if (items > INT_MAX) return DCN_ERR_UNSUPPORTED;
  t.items = int(items);
  t.batches = (t.TH * t.TW + tiled_batch(p) - 1) / tiled_batch(p);
  t.fd_G = make_fastdiv(uint32_t(t.G));
  t.fd_nTX = make_fastdiv(uint32_t(t.nTX));
  t.fd_tiles = make_fastdiv(uint32_t(t.nTY * t.nTX));
  t.fd_TW = make_fastdiv(uint32_t(t.TW));
  L->far = f.far;
  L->smem = fwd_tiled_smem(t.nbuf, t.box_stride, t.BW, cs);
  if (L->smem > optin) return DCN_ERR_UNSUPPORTED;
  L->smem += reserve;
  return encode_input_map(p, t, x, &L->map);
}

// The wide-window kernel: chunk size and record offset in a warp region.
template <typename T, bool SOFTMAX>
dcn_status forward_wide_launch(const CUtensorMap& map, const WideArgs& a, bool far, size_t smem,
                               int sms, cudaStream_t stream) {
  return far ? launch_persistent(dcn_forward_tiled_wide_kernel<T, SOFTMAX, true>, map, a, smem, sms, stream)
             : launch_persistent(dcn_forward_tiled_wide_kernel<T, SOFTMAX, false>, map, a, smem, sms, stream);
}

dcn_status forward_tiled_wide(const dcn_problem* p, const BoxLaunch& L, const void* x,
                              const void* off, const void* mask, void* out, cudaStream_t stream) {
  WideArgs a;
  a.x = x; a.off = off; a.mask = mask; a.out = out;
  a.error_word = L.dev.error_word;
  a.t = L.t;
  a.K = p->K;
  a.KK = taps(p);
  a.kc = p->remove_center ? (p->K * p->K) / 2 : -1;
  a.fd_K = make_fastdiv(uint32_t(p->K));
  const int pair_bytes = 2 * esize(p->dtype);
  a.rec = (wide_stage_bytes(a.KK, pair_bytes) + 15) / 16 * 16;
  // as many taps per chunk as the region holds, then evened out over the chunks
  const int ch_max = std::min(32, (kFwdRegion - a.rec) / wide_rec_bytes(1));
  if (a.KK > kWideMaxTaps || ch_max < 1) return DCN_ERR_UNSUPPORTED;
  const int nch = (a.KK + ch_max - 1) / ch_max;
  a.CH = (a.KK + nch - 1) / nch;
  return with_storage(p->dtype, [&](auto tag) {
    using T = decltype(tag);
    return p->softmax ? forward_wide_launch<T, true>(L.map, a, L.far, L.smem, L.dev.sms, stream)
                      : forward_wide_launch<T, false>(L.map, a, L.far, L.smem, L.dev.sms, stream);
  });
}

dcn_status forward_tiled(const dcn_problem* p, int64_t Ho, int64_t Wo, const void* x,
                         const void* off, const void* mask, void* out, cudaStream_t stream) {
  BoxLaunch L;
  dcn_status st = box_tiled_prepare(p, Ho, Wo, x, "DCN_CORE_TILED_TILE", &L);
  if (st != DCN_OK) return st;
  if (p->K != 3) return forward_tiled_wide(p, L, x, off, mask, out, stream);
  TiledArgs args;
  args.t = L.t;
  args.x = x; args.off = off; args.mask = mask; args.out = out;
  args.error_word = L.dev.error_word;
  return with_storage(p->dtype, [&](auto tag) {
    return forward_tiled_dispatch<decltype(tag)>(p, L.map, args, L.far, L.smem, L.dev.sms, stream);
  });
}

// The tiled backward applies where the tiled forward does (3x3 tap sets,
// 16 channels per group); DCN_CORE_BACKWARD=direct selects the direct kernel.
bool backward_tiled_eligible(const dcn_problem* p, int64_t Ho, int64_t Wo) {
  const char* mode = std::getenv("DCN_CORE_BACKWARD");
  if (mode && std::strcmp(mode, "direct") == 0) return false;
  if (p->K != 3 || p->Cg != 16) return false;
  if (p->H > 16000 || p->W > 16000 || Ho > 16000 || Wo > 16000) return false;
  return tensor_map_encoder() != nullptr;
}

// Launch the tiled backward on the zero-filled accumulator a.gx.
dcn_status backward_tiled(const dcn_problem* p, int64_t Ho, int64_t Wo, const BwdArgs& a,
                          bool det, cudaStream_t stream) {
  BoxLaunch L;
  dcn_status st =
      box_tiled_prepare(p, Ho, Wo, a.x, "DCN_CORE_BWD_TILED_TILE", &L,
                        det ? det_stage_total(esize(p->dtype)) : 0);
  if (st != DCN_OK) return st;
  TiledBwdArgs args;
  args.t = L.t;
  args.x = a.x; args.off = a.off; args.mask = a.mask; args.gout = a.gout;
  args.gx = a.gx; args.goff = a.goff; args.gmask = a.gmask;
  args.det_hdr = a.det_hdr; args.det_cbits = a.det_cbits;
  args.error_word = L.dev.error_word;
  const int sms = L.dev.sms;
  return with_storage(p->dtype, [&](auto tag) {
    using T = decltype(tag);
    return det ? backward_tiled_dispatch<T, true>(p, L.map, args, L.far, L.smem, sms, stream)
               : backward_tiled_dispatch<T, false>(p, L.map, args, L.far, L.smem, sms, stream);
  });
}

// The backward's kernel launch on a zero-filled accumulator: the tiled kernel
// where it applies, else (or when it cannot be configured) the direct one.
dcn_status backward_launch(const dcn_problem* p, int64_t Ho, int64_t Wo, const Plan& plan,
                           const BwdArgs& a, bool det, cudaStream_t stream) {
  if (backward_tiled_eligible(p, Ho, Wo)) {
    const dcn_status st = backward_tiled(p, Ho, Wo, a, det, stream);
    if (st != DCN_ERR_UNSUPPORTED) return st;
  }
  return backward_dispatch(p, plan, a, det, stream);
}
// ---------------------------------------------------------------------------
// Host entry points.  The batch is cut into chunks of whole images; chunk i's
// host-to-device copies run on a library stream, its kernels on the caller's
// stream and its device-to-host copies on a second library stream, so that
// the two copy directions (separate copy engines) and the kernels overlap.
// Events order the three streams and join the library streams back into the
// caller's stream at the end.
// ---------------------------------------------------------------------------
constexpr int kHostChunks = 8;  // chunks per call, at most

struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  // [0] start, [1 + i] chunk i in, [1 + C + i] chunk i out, [2C + 1] and
  // [2C + 2] the joins of the device-to-host and host-to-device streams
  cudaEvent_t ev[2 * kHostChunks + 3] = {};
};

// Joins both library streams back into the caller's stream.  Runs on every
// exit after the fork, so that an error part-way leaves no copy outside the
// caller's stream order (and a stream capture no unjoined fork).
dcn_status join_host_pipe(HostPipe* hp, int chunks, cudaStream_t stream, dcn_status st) {
  cudaEvent_t* const ev = hp->ev;
  const bool ok = cudaEventRecord(ev[2 * chunks + 1], hp->d2h) == cudaSuccess &&
                  cudaStreamWaitEvent(stream, ev[2 * chunks + 1], 0) == cudaSuccess &&
                  cudaEventRecord(ev[2 * chunks + 2], hp->h2d) == cudaSuccess &&
                  cudaStreamWaitEvent(stream, ev[2 * chunks + 2], 0) == cudaSuccess;
  if (st != DCN_OK) return st;
  return ok ? DCN_OK : DCN_ERR_CUDA;
}

// The pipe of the current device, created on first use.  The returned lock is
// held while the caller enqueues: the events are re-recorded by the next call,
// which is safe because a wait already enqueued refers to the record it saw.
dcn_status host_pipe(HostPipe** out, std::unique_lock<std::mutex>* held) {
  constexpr int kMaxDev = 64;
  static HostPipe pipes[kMaxDev];
  static bool ready[kMaxDev] = {};
  static unsigned long long ctx[kMaxDev] = {};  // context the pipe was made in
  static std::mutex lock;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return DCN_ERR_CUDA;
  *held = std::unique_lock<std::mutex>(lock);
  const unsigned long long id = current_context_id();
  if (!ready[dev] || ctx[dev] != id) {
    HostPipe hp;
    if (cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) != cudaSuccess)
      return DCN_ERR_CUDA;
    for (cudaEvent_t& e : hp.ev)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return DCN_ERR_CUDA;
    pipes[dev] = hp;
    ctx[dev] = id;
    ready[dev] = true;
  }
  *out = &pipes[dev];
  return DCN_OK;
}

// Images per chunk: about N / kHostChunks, rounded up to a multiple that keeps
// every tensor's chunk start 32-byte aligned (per_image: bytes of one image of
// each tensor); one chunk when that multiple reaches N.
struct ChunkPlan {
  int64_t per = 1;
  int chunks = 1;
};
ChunkPlan chunk_plan(int64_t N, std::initializer_list<size_t> per_image) {
  int64_t q = 1;
  for (size_t bytes : per_image) q = std::lcm<int64_t>(q, int64_t(32 / std::gcd(bytes, size_t(32))));
  int64_t per = (N + kHostChunks - 1) / kHostChunks;
  per = (per + q - 1) / q * q;
  if (per >= N) per = N;
  ChunkPlan cp;
  cp.per = per;
  cp.chunks = int((N + per - 1) / per);
  return cp;
}

#define DCN_CU(call)                                   \
  do {                                                 \
    if ((call) != cudaSuccess) return DCN_ERR_CUDA;    \
  } while (0)

// Chunk offset helpers.
inline const char* at(const void* p, size_t off) { return static_cast<const char*>(p) + off; }
inline char* at(void* p, size_t off) { return static_cast<char*>(p) + off; }

// Per-image byte counts of the problem's tensors.
struct ImageBytes {
  size_t x, off, msk, out;  // input (and grad_input), offset, mask, output (and grad_out)
};
ImageBytes image_bytes(const dcn_problem* p, int64_t Ho, int64_t Wo) {
  const size_t e = size_t(esize(p->dtype));
  const size_t C = size_t(p->G) * p->Cg, KK = size_t(taps(p)), px = size_t(Ho) * Wo;
  return {size_t(p->H) * p->W * C * e, px * p->G * KK * 2 * e, px * p->G * KK * e, px * C * e};
}

}  // namespace
}  // namespace dcn

using namespace dcn;

extern "C" {

dcn_status dcn_core_output_hw(const dcn_problem* problem, int* Ho, int* Wo) {
  if (!Ho || !Wo) return DCN_ERR_INVALID_ARG;
  int64_t ho = 0, wo = 0;
  dcn_status st = check_problem(problem, &ho, &wo);
  if (st != DCN_OK && st != DCN_ERR_UNSUPPORTED) return st;
  if (ho < 1 || wo < 1) {
    ho = out_extent(problem->H, problem->K, problem->stride, problem->pad, problem->dilation);
    wo = out_extent(problem->W, problem->K, stride_w(problem), pad_w(problem), dil_w(problem));
  }
  *Ho = int(ho);
  *Wo = int(wo);
  return DCN_OK;
}

dcn_status dcn_core_forward(const dcn_problem* problem, const void* input, const void* offset,
                            const void* mask, void* output, cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  st = check_forward_pointers(problem, input, offset, mask, output);
  if (st != DCN_OK) return st;
  if (tiled_eligible(problem, Ho, Wo)) {
    st = forward_tiled(problem, Ho, Wo, input, offset, mask, output, stream);
    if (st != DCN_ERR_UNSUPPORTED) return st;
  }
  Plan plan;
  const size_t entry = with_storage(problem->dtype, [](auto tag) {
    return size_t(staged_bytes_per_entry<decltype(tag)>());
  });
  st = make_plan(problem, Ho, Wo, entry, &plan);
  if (st != DCN_OK) return st;
  FwdArgs args{input, offset, mask, output, plan.t};
  return with_storage(problem->dtype, [&](auto tag) {
    return forward_dispatch<decltype(tag)>(problem, plan, args, stream);
  });
}

dcn_status dcn_core_forward_host(const dcn_problem* problem, const void* h_input,
                                 const void* h_offset, const void* h_mask, void* h_output,
                                 void* d_input, void* d_offset, void* d_mask, void* d_output,
                                 cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!h_input || !h_offset || !h_mask || !h_output) return DCN_ERR_INVALID_ARG;
  st = check_forward_pointers(problem, d_input, d_offset, d_mask, d_output);
  if (st != DCN_OK) return st;
  const ImageBytes ib = image_bytes(problem, Ho, Wo);
  const ChunkPlan cp = chunk_plan(problem->N, {ib.x, ib.off, ib.msk, ib.out});
  HostPipe* hp = nullptr;
  std::unique_lock<std::mutex> held;
  st = host_pipe(&hp, &held);
  if (st != DCN_OK) return st;
  cudaEvent_t* const ev = hp->ev;
  DCN_CU(cudaEventRecord(ev[0], stream));
  auto chunks = [&]() -> dcn_status {
    DCN_CU(cudaStreamWaitEvent(hp->h2d, ev[0], 0));
    DCN_CU(cudaStreamWaitEvent(hp->d2h, ev[0], 0));
    for (int i = 0; i < cp.chunks; ++i) {
      const int64_t n0 = int64_t(i) * cp.per, n = std::min<int64_t>(cp.per, problem->N - n0);
      const size_t ox = size_t(n0) * ib.x, oo = size_t(n0) * ib.off, om = size_t(n0) * ib.msk,
                   oy = size_t(n0) * ib.out;
      DCN_CU(cudaMemcpyAsync(at(d_input, ox), at(h_input, ox), size_t(n) * ib.x,
                             cudaMemcpyHostToDevice, hp->h2d));
      DCN_CU(cudaMemcpyAsync(at(d_offset, oo), at(h_offset, oo), size_t(n) * ib.off,
                             cudaMemcpyHostToDevice, hp->h2d));
      DCN_CU(cudaMemcpyAsync(at(d_mask, om), at(h_mask, om), size_t(n) * ib.msk,
                             cudaMemcpyHostToDevice, hp->h2d));
      DCN_CU(cudaEventRecord(ev[1 + i], hp->h2d));
      DCN_CU(cudaStreamWaitEvent(stream, ev[1 + i], 0));
      dcn_problem q = *problem;
      q.N = int(n);
      const dcn_status cs = dcn_core_forward(&q, at(d_input, ox), at(d_offset, oo),
                                             at(d_mask, om), at(d_output, oy), stream);
      if (cs != DCN_OK) return cs;
      DCN_CU(cudaEventRecord(ev[1 + cp.chunks + i], stream));
      DCN_CU(cudaStreamWaitEvent(hp->d2h, ev[1 + cp.chunks + i], 0));
      DCN_CU(cudaMemcpyAsync(at(h_output, oy), at(d_output, oy), size_t(n) * ib.out,
                             cudaMemcpyDeviceToHost, hp->d2h));
    }
    return DCN_OK;
  };
  return join_host_pipe(hp, cp.chunks, stream, chunks());
}


size_t dcn_core_backward_workspace(const dcn_problem* problem) {
  int64_t Ho, Wo;
  if (check_problem(problem, &Ho, &Wo) != DCN_OK) return 0;
  return problem->dtype != DCN_F32 ? bf16_accumulator_bytes(problem) : 0;
}

dcn_status dcn_core_backward(const dcn_problem* problem, const void* input, const void* offset,
                             const void* mask, const void* grad_out, void* grad_input,
                             void* grad_offset, void* grad_mask, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!input || !offset || !mask || !grad_out || !grad_input || !grad_offset || !grad_mask)
    return DCN_ERR_INVALID_ARG;
  const bool bf16 = problem->dtype != DCN_F32;  // 2-byte storage: fp32 accumulator
  const size_t acc_bytes = bf16_accumulator_bytes(problem);
  if (bf16 && (!workspace || workspace_bytes < acc_bytes)) return DCN_ERR_INVALID_ARG;
  if (!aligned(input, 16) || !aligned(offset, 16) || !aligned(mask, 16) ||
      !aligned(grad_out, 16) || !aligned(grad_input, 16) || !aligned(grad_offset, 16) ||
      !aligned(grad_mask, 16) || (bf16 && !aligned(workspace, 16)))
    return DCN_ERR_UNSUPPORTED;
  Plan plan;
  st = make_plan(problem, Ho, Wo, with_storage(problem->dtype, [](auto tag) {
                   return staged_bytes_per_entry<decltype(tag)>();
                 }),
                 &plan, true);
  if (st != DCN_OK) return st;
  float* acc = bf16 ? static_cast<float*>(workspace) : static_cast<float*>(grad_input);
  if (cudaMemsetAsync(acc, 0, acc_bytes, stream) != cudaSuccess) return DCN_ERR_CUDA;
  BwdArgs args{input, offset, mask, grad_out, acc, grad_offset, grad_mask, nullptr, 0, plan.t};
  st = backward_launch(problem, Ho, Wo, plan, args, false, stream);
  if (st != DCN_OK || !bf16) return st;
  // bf16: round the fp32 accumulator once into grad_input.
  const size_t n4 = acc_bytes / 16;
  DeviceInfo dev;
  if (device_info(&dev) != DCN_OK) return DCN_ERR_CUDA;
  const unsigned grid = unsigned(std::min<size_t>((n4 + 255) / 256, size_t(dev.sms) * 8));
  if (problem->dtype == DCN_F16)
    dcn_round_to_half_kernel<__half><<<grid, 256, 0, stream>>>(
        static_cast<const float4*>(workspace), static_cast<uint2*>(grad_input), n4);
  else
    dcn_round_to_half_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const float4*>(workspace), static_cast<uint2*>(grad_input), n4);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

dcn_status dcn_core_backward_host(const dcn_problem* problem, const void* input,
                                  const void* offset, const void* mask, const void* h_grad_out,
                                  void* h_grad_input, void* h_grad_offset, void* h_grad_mask,
                                  void* d_grad_out, void* d_grad_input, void* d_grad_offset,
                                  void* d_grad_mask, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!h_grad_out || !h_grad_input || !h_grad_offset || !h_grad_mask || !input || !offset ||
      !mask || !d_grad_out || !d_grad_input || !d_grad_offset || !d_grad_mask)
    return DCN_ERR_INVALID_ARG;
  // Everything dcn_core_backward checks, on the whole problem, before the
  // first copy is enqueued (chunk starts keep the alignment).
  const bool bf16 = problem->dtype != DCN_F32;  // 2-byte storage: fp32 accumulator
  if (bf16 && (!workspace || workspace_bytes < bf16_accumulator_bytes(problem)))
    return DCN_ERR_INVALID_ARG;
  if (!aligned(input, 16) || !aligned(offset, 16) || !aligned(mask, 16) ||
      !aligned(d_grad_out, 16) || !aligned(d_grad_input, 16) || !aligned(d_grad_offset, 16) ||
      !aligned(d_grad_mask, 16) || (bf16 && !aligned(workspace, 16)))
    return DCN_ERR_UNSUPPORTED;
  {
    Plan plan;
    st = make_plan(problem, Ho, Wo, with_storage(problem->dtype, [](auto tag) {
                     return staged_bytes_per_entry<decltype(tag)>();
                   }),
                   &plan, true);
    if (st != DCN_OK) return st;
  }
  const ImageBytes ib = image_bytes(problem, Ho, Wo);
  const ChunkPlan cp = chunk_plan(problem->N, {ib.x, ib.off, ib.msk, ib.out});
  HostPipe* hp = nullptr;
  std::unique_lock<std::mutex> held;
  st = host_pipe(&hp, &held);
  if (st != DCN_OK) return st;
  cudaEvent_t* const ev = hp->ev;
  DCN_CU(cudaEventRecord(ev[0], stream));
  auto chunks = [&]() -> dcn_status {
    DCN_CU(cudaStreamWaitEvent(hp->h2d, ev[0], 0));
    DCN_CU(cudaStreamWaitEvent(hp->d2h, ev[0], 0));
    for (int i = 0; i < cp.chunks; ++i) {
      const int64_t n0 = int64_t(i) * cp.per, n = std::min<int64_t>(cp.per, problem->N - n0);
      const size_t ox = size_t(n0) * ib.x, oo = size_t(n0) * ib.off, om = size_t(n0) * ib.msk,
                   oy = size_t(n0) * ib.out;
      DCN_CU(cudaMemcpyAsync(at(d_grad_out, oy), at(h_grad_out, oy), size_t(n) * ib.out,
                             cudaMemcpyHostToDevice, hp->h2d));
      DCN_CU(cudaEventRecord(ev[1 + i], hp->h2d));
      DCN_CU(cudaStreamWaitEvent(stream, ev[1 + i], 0));
      dcn_problem q = *problem;
      q.N = int(n);
      const dcn_status cs = dcn_core_backward(
          &q, at(input, ox), at(offset, oo), at(mask, om), at(d_grad_out, oy),
          at(d_grad_input, ox), at(d_grad_offset, oo), at(d_grad_mask, om), workspace,
          workspace_bytes, stream);
      if (cs != DCN_OK) return cs;
      DCN_CU(cudaEventRecord(ev[1 + cp.chunks + i], stream));
      DCN_CU(cudaStreamWaitEvent(hp->d2h, ev[1 + cp.chunks + i], 0));
      DCN_CU(cudaMemcpyAsync(at(h_grad_input, ox), at(d_grad_input, ox), size_t(n) * ib.x,
                             cudaMemcpyDeviceToHost, hp->d2h));
      DCN_CU(cudaMemcpyAsync(at(h_grad_offset, oo), at(d_grad_offset, oo), size_t(n) * ib.off,
                             cudaMemcpyDeviceToHost, hp->d2h));
      DCN_CU(cudaMemcpyAsync(at(h_grad_mask, om), at(d_grad_mask, om), size_t(n) * ib.msk,
                             cudaMemcpyDeviceToHost, hp->d2h));
    }
    return DCN_OK;
  };
  return join_host_pipe(hp, cp.chunks, stream, chunks());
}

dcn_status dcn_core_sync_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return DCN_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return DCN_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_dcn_error_word, sizeof(word)) != cudaSuccess)
    return DCN_ERR_CUDA;
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_dcn_error_word, &zero, sizeof(zero));
    return (word & kErrOutOfBounds) ? DCN_ERR_OUT_OF_BOUNDS : DCN_ERR_TIMEOUT;
  }
  return DCN_OK;
}

const char* dcn_status_string(dcn_status status) {
  switch (status) {
    case DCN_OK: return "ok";
    case DCN_ERR_INVALID_ARG: return "invalid argument";
    case DCN_ERR_UNSUPPORTED: return "unsupported argument (alignment, channel width or dtype)";
    case DCN_ERR_CUDA: return "CUDA error";
    case DCN_ERR_TIMEOUT: return "a bounded device wait gave up";
    case DCN_ERR_OUT_OF_BOUNDS:
      return "an access outside a tensor was skipped (bounds-checked build)";
    default: return "unknown status";
  }
}

int dcn_core_abi_version(void) { return DCN_CORE_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward (dcn_core_backward_noalloc in include/dcn_core.h).
// ---------------------------------------------------------------------------
namespace dcn {
namespace {

// The bf16 backward's fp32 grad_input accumulator, owned by the library.  In
// host code this name is only a stand-in for the device array: the kernels
// get the device address that cudaGetSymbolAddress returns for the current
// device.
static __device__ __align__(256) float
    g_noalloc_scratch[DCN_CORE_NOALLOC_SCRATCH_BYTES / sizeof(float)];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kNoallocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoallocMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device and context (with that device current) and cached.
dcn_status noalloc_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices)
    return DCN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  const unsigned long long id = current_context_id();
  if (g_noalloc_addr[dev] == nullptr || g_noalloc_ctx[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return DCN_ERR_CUDA;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = id;
  }
  *out = g_noalloc_addr[dev];
  return DCN_OK;
}

}  // namespace
}  // namespace dcn

extern "C" dcn_status dcn_core_backward_noalloc(const dcn_problem* problem, const void* input,
                                                const void* offset, const void* mask,
                                                const void* grad_out, void* grad_input,
                                                void* grad_offset, void* grad_mask,
                                                cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!input || !offset || !mask || !grad_out || !grad_input || !grad_offset || !grad_mask)
    return DCN_ERR_INVALID_ARG;
  if (!aligned(input, 16) || !aligned(offset, 16) || !aligned(mask, 16) ||
      !aligned(grad_out, 16) || !aligned(grad_input, 16) || !aligned(grad_offset, 16) ||
      !aligned(grad_mask, 16))
    return DCN_ERR_UNSUPPORTED;
  const bool bf16 = problem->dtype != DCN_F32;  // 2-byte storage: fp32 accumulator
  const size_t acc_bytes = bf16_accumulator_bytes(problem);  // fp32 grad_input size
  if (bf16 && acc_bytes > size_t(DCN_CORE_NOALLOC_SCRATCH_BYTES)) return DCN_ERR_UNSUPPORTED;
  Plan plan;
  st = make_plan(problem, Ho, Wo, with_storage(problem->dtype, [](auto tag) {
                   return staged_bytes_per_entry<decltype(tag)>();
                 }),
                 &plan, true);
  if (st != DCN_OK) return st;
  float* acc = static_cast<float*>(grad_input);
  if (bf16) {
    void* scratch = nullptr;
    st = noalloc_scratch_address(&scratch);
    if (st != DCN_OK) return st;
    acc = static_cast<float*>(scratch);
  }
  // The shared array keeps the previous call's sums: clear it first.
  if (cudaMemsetAsync(acc, 0, acc_bytes, stream) != cudaSuccess) return DCN_ERR_CUDA;
  BwdArgs args{input, offset, mask, grad_out, acc, grad_offset, grad_mask, nullptr, 0, plan.t};
  st = backward_launch(problem, Ho, Wo, plan, args, false, stream);
  if (st != DCN_OK || !bf16) return st;
  const size_t n4 = acc_bytes / 16;
  DeviceInfo dev;
  if (device_info(&dev) != DCN_OK) return DCN_ERR_CUDA;
  const unsigned grid = unsigned(std::min<size_t>((n4 + 255) / 256, size_t(dev.sms) * 8));
  if (problem->dtype == DCN_F16)
    dcn_round_to_half_kernel<__half><<<grid, 256, 0, stream>>>(
        reinterpret_cast<const float4*>(acc), static_cast<uint2*>(grad_input), n4);
  else
    dcn_round_to_half_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        reinterpret_cast<const float4*>(acc), static_cast<uint2*>(grad_input), n4);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Deterministic backward (dcn_core_backward_deterministic in include/dcn_core.h).
// ---------------------------------------------------------------------------
namespace dcn {
namespace {

int ceil_log2(int64_t n) {
  int b = 0;
  while ((int64_t(1) << b) < n) ++b;
  return b;
}

size_t det_workspace_bytes(const dcn_problem* p) {
  return size_t(kDetHeaderBytes) + size_t(p->N) * p->H * p->W * p->G * p->Cg * 8;
}

unsigned grid_for(size_t n, int sms) {
  return unsigned(std::max<size_t>(1, std::min<size_t>((n + 255) / 256, size_t(sms) * 8)));
}

template <typename T>
dcn_status det_passes(const dcn_problem* p, int64_t Ho, int64_t Wo, const Plan& plan,
                      const void* input, const void* offset, const void* mask,
                      const void* grad_out, void* grad_input, void* grad_offset,
                      void* grad_mask, unsigned char* ws, int sms, cudaStream_t stream) {
  unsigned int* hdr = reinterpret_cast<unsigned int*>(ws);
  void* acc = ws + kDetHeaderBytes;
  const size_t n_out = size_t(p->N) * Ho * Wo * p->G * p->Cg;
  const size_t n_msk = size_t(p->N) * Ho * Wo * p->G * taps(p);
  const size_t n_in = size_t(p->N) * p->H * p->W * p->G * p->Cg;
  dcn_absmax_kernel<T><<<grid_for(n_out, sms), 256, 0, stream>>>(static_cast<const T*>(grad_out),
                                                                 n_out, hdr);
  if (!p->softmax)
    dcn_absmax_kernel<T><<<grid_for(n_msk, sms), 256, 0, stream>>>(static_cast<const T*>(mask),
                                                                   n_msk, hdr + 1);
  if (cudaGetLastError() != cudaSuccess) return DCN_ERR_CUDA;
  // An element of grad_input receives at most one contribution per (output
  // pixel, tap) of its image and group.
  const int cbits = ceil_log2(int64_t(Ho) * Wo * taps(p));
  BwdArgs args{input, offset, mask, grad_out, acc, grad_offset, grad_mask, hdr, cbits, plan.t};
  dcn_status st = backward_launch(p, Ho, Wo, plan, args, true, stream);
  if (st != DCN_OK) return st;
  dcn_fixed_to_grad_kernel<T><<<grid_for(n_in, sms), 256, 0, stream>>>(
      static_cast<const long long*>(acc), static_cast<T*>(grad_input), n_in, hdr, p->softmax,
      cbits);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

}  // namespace
}  // namespace dcn

extern "C" size_t dcn_core_backward_deterministic_workspace(const dcn_problem* problem) {
  int64_t Ho, Wo;
  if (check_problem(problem, &Ho, &Wo) != DCN_OK) return 0;
  return det_workspace_bytes(problem);
}

extern "C" dcn_status dcn_core_backward_deterministic(
    const dcn_problem* problem, const void* input, const void* offset, const void* mask,
    const void* grad_out, void* grad_input, void* grad_offset, void* grad_mask, void* workspace,
    size_t workspace_bytes, cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!input || !offset || !mask || !grad_out || !grad_input || !grad_offset || !grad_mask)
    return DCN_ERR_INVALID_ARG;
  const size_t ws_bytes = det_workspace_bytes(problem);
  if (!workspace || workspace_bytes < ws_bytes) return DCN_ERR_INVALID_ARG;
  if (!aligned(input, 16) || !aligned(offset, 16) || !aligned(mask, 16) ||
      !aligned(grad_out, 16) || !aligned(grad_input, 16) || !aligned(grad_offset, 16) ||
      !aligned(grad_mask, 16) || !aligned(workspace, 256))
    return DCN_ERR_UNSUPPORTED;
  Plan plan;
  st = make_plan(problem, Ho, Wo, with_storage(problem->dtype, [](auto tag) {
                   return staged_bytes_per_entry<decltype(tag)>();
                 }),
                 &plan, true);
  if (st != DCN_OK) return st;
  DeviceInfo dev;
  if (device_info(&dev) != DCN_OK) return DCN_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, ws_bytes, stream) != cudaSuccess) return DCN_ERR_CUDA;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  return with_storage(problem->dtype, [&](auto tag) {
    return det_passes<decltype(tag)>(problem, Ho, Wo, plan, input, offset, mask, grad_out,
                                     grad_input, grad_offset, grad_mask, ws, dev.sms, stream);
  });
}

// ---------------------------------------------------------------------------
// Offset / mask projection (dcn_core_offset_mask_projection in include/dcn_core.h).
// ---------------------------------------------------------------------------
namespace dcn {
namespace {

// 2-D bf16 tensor map (inner, outer) with a (64, 128) box and 128-byte swizzle.
dcn_status bf16_kmajor_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer) {
  const cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(outer)};
  const cuuint64_t strides[1] = {cuuint64_t(inner) * 2};
  const cuuint32_t box[2] = {cuuint32_t(kPjBK), cuuint32_t(kPjBM)};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult cr = tensor_map_encoder()(
      map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
      CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return cr == CUDA_SUCCESS ? DCN_OK : DCN_ERR_UNSUPPORTED;
}

template <typename T>
dcn_status launch_projection(const CUtensorMap& qmap, const CUtensorMap& wmap,
                             const ProjArgs& args, int sms, cudaStream_t stream) {
  auto k = dcn_projection_kernel<T>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(kPjSmemBytes)) != cudaSuccess)
    return DCN_ERR_CUDA;
  const int grid = std::min(args.tiles, sms);
  k<<<unsigned(grid), kPjThreads, kPjSmemBytes, stream>>>(qmap, wmap, args);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

}  // namespace
}  // namespace dcn

namespace dcn {
namespace {

// out0[m, j] (j < n_split) / out1[m, j - n_split] (j >= n_split) =
//     sum_c a[m, c] * w[j, c] + bias[j]  on the tensor cores.
dcn_status bf16_gemm(const void* a, int64_t M, int K, const void* w, int64_t nout,
                     int64_t n_split, const float* bias, void* out0, void* out1, dcn_dtype out_dtype,
                     cudaStream_t stream) {
  if (K % 8 != 0) return DCN_ERR_UNSUPPORTED;  // TMA rows must be 16-byte multiples
  if (!aligned(a, 16) || !aligned(w, 16) || !aligned(out0, 16) || !aligned(out1, 16) ||
      (bias && !aligned(bias, 4)))
    return DCN_ERR_UNSUPPORTED;
  if (M * K > INT_MAX || M * nout > INT_MAX || nout > INT_MAX) return DCN_ERR_INVALID_ARG;
  if (tensor_map_encoder() == nullptr) return DCN_ERR_UNSUPPORTED;
  DeviceInfo dev;
  if (device_info(&dev) != DCN_OK) return DCN_ERR_CUDA;
  if (size_t(dev.smem_optin) < kPjSmemBytes) return DCN_ERR_UNSUPPORTED;
  ProjArgs args;
  args.M = int(M);
  args.Nout = int(nout);
  args.n_off = int(n_split);
  args.k_blocks = (K + kPjBK - 1) / kPjBK;
  args.m_tiles = int((M + kPjBM - 1) / kPjBM);
  args.n_tiles = int((nout + kPjBN - 1) / kPjBN);
  if (int64_t(args.m_tiles) * args.n_tiles > INT_MAX) return DCN_ERR_UNSUPPORTED;
  args.tiles = args.m_tiles * args.n_tiles;
  args.bias = bias;
  args.offset = out0;
  args.mask = out1;
  args.error_word = dev.error_word;
  CUtensorMap amap, wmap;
  dcn_status st;
  if ((st = bf16_kmajor_map(&amap, a, uint64_t(K), uint64_t(M))) != DCN_OK) return st;
  if ((st = bf16_kmajor_map(&wmap, w, uint64_t(K), uint64_t(nout))) != DCN_OK) return st;
  return with_storage(out_dtype, [&](auto tag) {
    return launch_projection<decltype(tag)>(amap, wmap, args, dev.sms, stream);
  });
}

}  // namespace
}  // namespace dcn

extern "C" dcn_status dcn_core_offset_mask_projection(const dcn_problem* problem,
                                                      const void* query, int Cq,
                                                      const void* weight, const float* bias,
                                                      void* offset, void* mask,
                                                      cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!query || !weight || !offset || !mask || Cq < 1) return DCN_ERR_INVALID_ARG;
  const int64_t M = int64_t(problem->N) * Ho * Wo;
  const int64_t KK = taps(problem);
  return bf16_gemm(query, M, Cq, weight, int64_t(problem->G) * KK * 3,
                   int64_t(problem->G) * KK * 2, bias, offset, mask,
                   problem->dtype, stream);
}

namespace dcn {
namespace {

template <typename T, int LP, int NJS>
dcn_status guide_launch_nj(const GuideArgs& a, cudaStream_t stream) {
  const unsigned grid = unsigned(int64_t(a.N) * a.tiles_y * a.tiles_x);
  const unsigned block = kGuideWarps * 32;
  // parameters (12 quads per channel quad) and the conv results of R rows
  constexpr int R = guide_rows_per_pass<T, LP, NJS>();  // output rows per pass
  const size_t smem = (size_t(12) * a.Q + size_t(a.NJ) * block * R) * sizeof(float4);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(dcn_guide_kernel<T, LP, NJS>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return DCN_ERR_CUDA;
  dcn_guide_kernel<T, LP, NJS><<<grid, block, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

// The compile-time quad count where the quads fill the lane groups exactly
// (C = 160, 320, 640: 5 quads per lane; C = 1280: 10), else the general kernel.
template <typename T, int LP>
dcn_status guide_launch_lp(const GuideArgs& a, cudaStream_t stream) {
  if (a.Q == LP * a.NJ && a.NJ == 5) return guide_launch_nj<T, LP, 5>(a, stream);
  if constexpr (LP == 32)
    if (a.Q == LP * a.NJ && a.NJ == 10) return guide_launch_nj<T, LP, 10>(a, stream);
  return guide_launch_nj<T, LP, 0>(a, stream);
}

template <typename T>
dcn_status guide_launch(int LP, const GuideArgs& a, cudaStream_t stream) {
  switch (LP) {
    case 32: return guide_launch_lp<T, 32>(a, stream);
    case 16: return guide_launch_lp<T, 16>(a, stream);
    case 8: return guide_launch_lp<T, 8>(a, stream);
    default: return guide_launch_lp<T, 4>(a, stream);
  }
}

}  // namespace
}  // namespace dcn

extern "C" dcn_status dcn_core_offset_mask_guide(const dcn_problem* problem, const void* input,
                                                 const float* dw_weight, const float* dw_bias,
                                                 const float* ln_gamma, const float* ln_beta,
                                                 float ln_eps, void* query, cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!input || !dw_weight || !query) return DCN_ERR_INVALID_ARG;
  if (!std::isfinite(ln_eps) || ln_eps < 0.f) return DCN_ERR_INVALID_ARG;
  const int C = problem->G * problem->Cg;
  if (C % 4 != 0) return DCN_ERR_UNSUPPORTED;
  const int Q = C / 4;
  // lanes per pixel: the group size whose quads per lane fill the lanes best
  // (ties to the larger group), at most kGuideMaxQuads quads per lane
  int LP = 0, NJ = 0;
  double best = -1.0;
  for (int lp : {32, 16, 8, 4}) {
    const int nj = (Q + lp - 1) / lp;
    if (nj > kGuideMaxQuads) continue;
    const double eff = double(Q) / double(lp * nj);
    if (eff > best + 1e-9) {
      best = eff;
      LP = lp;
      NJ = nj;
    }
  }
  if (LP == 0) return DCN_ERR_UNSUPPORTED;
  if (!aligned(input, 16) || !aligned(dw_weight, 16) || (dw_bias && !aligned(dw_bias, 16)) ||
      (ln_gamma && !aligned(ln_gamma, 16)) || (ln_beta && !aligned(ln_beta, 16)) ||
      !aligned(query, 8))
    return DCN_ERR_UNSUPPORTED;
  GuideArgs a;
  a.x = input;
  a.w = dw_weight;
  a.bias = dw_bias;
  a.gamma = ln_gamma;
  a.beta = ln_beta;
  a.eps = ln_eps;
  a.out = static_cast<__nv_bfloat16*>(query);
  a.N = problem->N;
  a.H = problem->H;
  a.W = problem->W;
  a.C = C;
  a.Q = Q;
  a.NJ = NJ;
  a.tiles_x = (problem->W + kGuideWarps * (32 / LP) - 1) / (kGuideWarps * (32 / LP));
  a.tiles_y = (problem->H + kGuideRows - 1) / kGuideRows;
  a.rows = (problem->H + a.tiles_y - 1) / a.tiles_y;  // e.g. 6 + 6 rows at H = 12, not 8 + 4
  if (int64_t(a.N) * a.tiles_y * a.tiles_x > INT_MAX) return DCN_ERR_UNSUPPORTED;
  const size_t elems = size_t(problem->N) * problem->H * problem->W * C;
  a.x_bytes = elems * size_t(esize(problem->dtype));
  a.out_bytes = elems * 2;
  return with_storage(problem->dtype, [&](auto tag) {
    return guide_launch<decltype(tag)>(LP, a, stream);
  });
}

namespace dcn {
namespace {

template <typename T, typename TO, int LP>
dcn_status guide_projection_launch(const CUtensorMap& wmap, const GuideProjArgs& a, int sms,
                                   cudaStream_t stream) {
  auto k = dcn_guide_projection_kernel<T, TO, LP, 5>;
  const size_t smem = guide_proj_smem(a.nA, a.KB, a.Q);
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
      cudaSuccess)
    return DCN_ERR_CUDA;
  k<<<unsigned(std::min(a.m_tiles, sms)), kGpThreads, smem, stream>>>(wmap, a);
  return cudaGetLastError() == cudaSuccess ? DCN_OK : DCN_ERR_CUDA;
}

}  // namespace
}  // namespace dcn

extern "C" dcn_status dcn_core_offset_mask_guide_projection(
    const dcn_problem* problem, const void* input, const float* dw_weight, const float* dw_bias,
    const float* ln_gamma, const float* ln_beta, float ln_eps, const void* weight,
    const float* bias, void* offset, void* mask, cudaStream_t stream) {
  int64_t Ho, Wo;
  dcn_status st = check_problem(problem, &Ho, &Wo);
  if (st != DCN_OK) return st;
  if (!input || !dw_weight || !weight || !offset || !mask) return DCN_ERR_INVALID_ARG;
  if (!(ln_eps >= 0.f) || !std::isfinite(ln_eps)) return DCN_ERR_INVALID_ARG;
  // the guide features keep the input's H x W: the projection's pixel grid must be it
  if (Ho != problem->H || Wo != problem->W) return DCN_ERR_UNSUPPORTED;
  const int C = problem->G * problem->Cg;
  // five channel quads per lane in groups of 8 or 16 lanes: C = 160 or 320.  At
  // C = 640 one 128-pixel A tile is 160 KB, and with the weight ring, the
  // guide parameters and the epilogue buffer the block would need 289 KB of
  // shared memory: those widths take the two calls.
  int LP = 0;
  for (int lp : {8, 16})
    if (C == 4 * lp * 5) LP = lp;
  if (LP == 0) return DCN_ERR_UNSUPPORTED;
  if (!aligned(input, 16) || !aligned(dw_weight, 16) || (dw_bias && !aligned(dw_bias, 16)) ||
      (ln_gamma && !aligned(ln_gamma, 16)) || (ln_beta && !aligned(ln_beta, 16)) ||
      !aligned(weight, 16) || !aligned(offset, 16) || !aligned(mask, 16) ||
      (bias && !aligned(bias, 4)))
    return DCN_ERR_UNSUPPORTED;
  if (tensor_map_encoder() == nullptr) return DCN_ERR_UNSUPPORTED;
  DeviceInfo dev;
  if (device_info(&dev) != DCN_OK) return DCN_ERR_CUDA;
  const int64_t KK = taps(problem);
  GuideProjArgs a;
  a.x = input;
  a.w = dw_weight;
  a.bias = dw_bias;
  a.gamma = ln_gamma;
  a.beta = ln_beta;
  a.eps = ln_eps;
  a.pbias = bias;
  a.offset = offset;
  a.mask = mask;
  a.error_word = dev.error_word;
  a.N = problem->N;
  a.H = problem->H;
  a.W = problem->W;
  a.C = C;
  a.Q = C / 4;
  const int64_t M = int64_t(problem->N) * problem->H * problem->W;
  const int64_t nout = int64_t(problem->G) * KK * 3;
  if (M * nout > INT_MAX) return DCN_ERR_INVALID_ARG;
  a.M = int(M);
  a.Nout = int(nout);
  a.n_off = int(int64_t(problem->G) * KK * 2);
  a.KB = (C + kPjBK - 1) / kPjBK;
  a.m_tiles = int((M + kPjBM - 1) / kPjBM);
  a.n_tiles = int((nout + kPjBN - 1) / kPjBN);
  a.nA = guide_proj_smem(2, a.KB, a.Q) <= size_t(dev.smem_optin) ? 2 : 1;
  if (guide_proj_smem(a.nA, a.KB, a.Q) > size_t(dev.smem_optin)) return DCN_ERR_UNSUPPORTED;
  a.x_bytes = size_t(M) * C * size_t(esize(problem->dtype));
  a.fd_W = make_fastdiv(uint32_t(problem->W));
  a.fd_H = make_fastdiv(uint32_t(problem->H));
  CUtensorMap wmap;
  if ((st = bf16_kmajor_map(&wmap, weight, uint64_t(C), uint64_t(nout))) != DCN_OK) return st;
  // input and output storage types follow the problem's
  return with_storage(problem->dtype, [&](auto tag) {
    using T = decltype(tag);
    return LP == 8 ? guide_projection_launch<T, T, 8>(wmap, a, dev.sms, stream)
                   : guide_projection_launch<T, T, 16>(wmap, a, dev.sms, stream);
  });
}

extern "C" dcn_status dcn_core_linear_bf16(const void* input, int M, int K, const void* weight,
                                           int Nout, const float* bias, void* output,
                                           dcn_dtype out_dtype, cudaStream_t stream) {
  if (!input || !weight || !output || M < 1 || K < 1 || Nout < 1) return DCN_ERR_INVALID_ARG;
  if (out_dtype != DCN_F32 && out_dtype != DCN_BF16 && out_dtype != DCN_F16)
    return DCN_ERR_INVALID_ARG;
  return bf16_gemm(input, M, K, weight, Nout, Nout, bias, output, output, out_dtype, stream);
}
