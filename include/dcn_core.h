/*
 * dcn_core.h -- C ABI of the B200 (sm_100a) deformable-convolution core.
 *
 * The operator (InternImage-L DCNv3 explainer (wmrh.cn), section 二 steps
 * 2-4 and section 三): for every output pixel (n, ho, wo), group g and tap
 * k of a K x K window (position (a, b), k = a*K + b), take the learned
 * offset (dx, dy) of that tap, scale it by offset_scale, bilinearly sample
 * the group's Cg input channels at
 *     Y = ho*stride - pad + a*dilation + offset_scale*dy
 *     X = wo*stride - pad + b*dilation + offset_scale*dx
 * (integer coordinates are pixel centres; corners outside the image read as
 * zero), and sum the K*K samples weighted by the mask of that (pixel, group):
 * softmax-normalised over the taps for DCNv3, used as given for the DCNv4
 * variant (DCNv4 speed-up write-up (pnsm.cn), sections 1-2).  With
 * remove_center (a DCNv4 module argument, same write-up, section 3.3) the
 * window's centre position (K/2, K/2) is not sampled: the KK = K*K - 1 taps
 * are the other positions in row-major order, tap k at position k for
 * k < (K*K)/2 and at k + 1 after it.  Arithmetic is fp32 for both storage
 * types; bf16 and fp16 values are widened exactly on load and the output is
 * rounded to nearest-even once.
 *
 * Layouts (all tensors dense, row-major, element indices; C = G*Cg, KK = taps
 * = K*K, or K*K - 1 with remove_center):
 *   input   (N, H, W, C)            ((n*H + y)*W + x)*C + g*Cg + c
 *   offset  (N, Ho, Wo, G*KK*2)     ((n*Ho + ho)*Wo + wo)*G*KK*2 + (g*KK + k)*2 + {0: dx, 1: dy}
 *   mask    (N, Ho, Wo, G*KK)       ((n*Ho + ho)*Wo + wo)*G*KK + g*KK + k
 *   output  (N, Ho, Wo, C)          ((n*Ho + ho)*Wo + wo)*C + g*Cg + c
 *   Ho = floor((H + 2*pad - dilation*(K-1) - 1) / stride) + 1, Wo likewise
 *   (with the width axis's values when separate_axes = 1).
 *
 * Ownership and execution: every pointer is owned by the caller.  Device
 * pointers must stay valid until the enqueued work has finished.  All work is
 * enqueued asynchronously on the caller's stream (NULL = the legacy default
 * stream); the library never allocates device memory, never synchronises
 * (except dcn_core_sync_status) and keeps no per-call state.
 *
 * Errors: arguments are validated on the host before anything is enqueued.
 * Invalid arguments return DCN_ERR_INVALID_ARG, valid but unsupported ones
 * (alignment, channel widths without a kernel) return
 * DCN_ERR_UNSUPPORTED, and a failed launch returns DCN_ERR_CUDA.  On any
 * error nothing has been enqueued.  Device-side failures (a bounded wait
 * that gave up) are reported by dcn_core_sync_status as DCN_ERR_TIMEOUT.
 */
#ifndef DCN_CORE_H_
#define DCN_CORE_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DCN_CORE_ABI_VERSION 5

#if defined(__GNUC__)
#define DCN_API __attribute__((visibility("default")))
#else
#define DCN_API
#endif

typedef enum {
  DCN_OK = 0,
  DCN_ERR_INVALID_ARG = 1,
  DCN_ERR_UNSUPPORTED = 2,
  DCN_ERR_CUDA = 3,
  DCN_ERR_TIMEOUT = 4,
  DCN_ERR_OUT_OF_BOUNDS = 5  /* only from a library built with -DDCN_CHECK_BOUNDS */
} dcn_status;

typedef enum {
  DCN_F32 = 0,   /* fp32 storage                                    */
  DCN_BF16 = 1,  /* bf16 storage, fp32 arithmetic                   */
  DCN_F16 = 2    /* fp16 storage, fp32 arithmetic (ABI version 5)   */
} dcn_dtype;

/*
 * Problem description (the constructor arguments of the DCNv3/DCNv4 modules
 * in the DCNv4 speed-up write-up (pnsm.cn), section 3.3: channels = G*Cg,
 * kernel_size, stride, pad, dilation, group, offset_scale, remove_center).
 *   N, H, W      batch and input spatial size, >= 1
 *   G, Cg        groups and channels per group, >= 1
 *   K            kernel side, odd, >= 1 (taps = K*K)
 *   stride >= 1, pad >= 0, dilation >= 1 (same for height and width)
 *   offset_scale multiplies every offset (InternImage-L uses 2.0)
 *   softmax      1: mask holds logits, softmax over the KK taps of each
 *                   (pixel, group) (DCNv3);  0: mask used as given (DCNv4)
 *   dtype        storage type of input, offset, mask and output
 *   remove_center  0: all K*K window positions are taps;  1: the centre
 *                position is left out (KK = K*K - 1 taps; needs K >= 3)
 *   separate_axes  0: stride, pad and dilation apply to both axes (the
 *                modules' single values); 1: they apply to the height axis
 *                (ho and the tap row a) and stride_w, pad_w, dilation_w to
 *                the width axis (wo and the tap column b)
 *   stride_w >= 1, pad_w >= 0, dilation_w >= 1   (read when separate_axes = 1)
 * With separate axes the grid is Y = ho*stride - pad + a*dilation + ...,
 * X = wo*stride_w - pad_w + b*dilation_w + ..., and Wo uses the width values.
 */
typedef struct {
  int N, H, W, G, Cg;
  int K;
  int stride, pad, dilation;
  float offset_scale;
  int softmax;
  dcn_dtype dtype;
  int remove_center;
  int separate_axes;
  int stride_w, pad_w, dilation_w;
} dcn_problem;

/* Output spatial size, the convolution rule
 *     Ho = floor((H + 2*pad - dilation*(K-1) - 1) / stride) + 1   (Wo likewise),
 * which keeps the input's size at 3x3 / stride 1 / pad 1 as the DCNv3
 * extension build guide (trdm.cn), section 2.3, checks.  Ho and Wo: host
 * pointers, written on success.  DCN_ERR_INVALID_ARG if the problem is invalid
 * or the output would be empty; nothing else is touched. */
DCN_API dcn_status dcn_core_output_hw(const dcn_problem* problem, int* Ho, int* Wo);

/*
 * Forward (explainer section 二 steps 2-4).  input, offset, mask: device
 * pointers in the layouts above, of problem->dtype; output: device pointer,
 * written entirely.  All four must be 16-byte aligned and must not overlap
 * the output.  Supported channel widths: Cg*sizeof(dtype) a multiple of 16
 * bytes and at most 128 bytes: Cg in {4, 8, 16, 32} for fp32, {8, 16, 32,
 * 64} for bf16 and fp16; other widths return DCN_ERR_UNSUPPORTED.
 */
DCN_API dcn_status dcn_core_forward(const dcn_problem* problem, const void* input,
                            const void* offset, const void* mask, void* output,
                            cudaStream_t stream);

/*
 * Forward on HOST buffers: copies input, offset and mask from the host to the
 * caller's device buffers, runs dcn_core_forward and copies the output back.
 * The batch is cut into at most 8 chunks of whole images (chunk starts kept
 * 32-byte aligned in every tensor; one chunk when N is small or the sizes do
 * not allow it).  Chunk i's host-to-device copies run on a library-owned
 * stream, its forward on `stream`, its device-to-host copy on a second
 * library-owned stream, so that both copy directions and the kernels overlap.
 * Events order the three: the first copy waits for the work enqueued on
 * `stream` before the call, and `stream` waits for the last copy before any
 * work enqueued after it, so from the caller's side everything happens on
 * `stream` (CUDA graph capture included).  The two streams and a set of
 * events per device are created on first use and kept by the library (and
 * created again for a new context after cudaDeviceReset); concurrent calls
 * from several host threads are serialised while they enqueue.  Host buffers
 * should be pinned for the copies to be asynchronous; they must not be
 * touched until `stream` has reached this point.  Device buffers follow the
 * rules of dcn_core_forward.  Arguments are validated before anything is
 * enqueued; an error part-way (DCN_ERR_CUDA, or a chunk's own error) may
 * leave the chunks before it enqueued, and the library streams are joined
 * back into `stream` on that path too, so no copy runs outside its order.
 */
DCN_API dcn_status dcn_core_forward_host(const dcn_problem* problem, const void* h_input,
                                 const void* h_offset, const void* h_mask,
                                 void* h_output, void* d_input, void* d_offset,
                                 void* d_mask, void* d_output, cudaStream_t stream);

/*
 * Backward with the gradients on HOST buffers, for a forward whose input,
 * offset and mask are still on the device (as dcn_core_forward_host leaves
 * them): copies grad_out from the host into d_grad_out, runs dcn_core_backward
 * and copies grad_input, grad_offset and grad_mask back into the host
 * buffers.  Chunked and overlapped like dcn_core_forward_host (grad_out in on
 * one library stream, the backward of each chunk on `stream`, the three
 * gradients out on the other).  input, offset, mask, d_grad_out,
 * d_grad_input, d_grad_offset and d_grad_mask: device buffers with the rules
 * of dcn_core_backward; the 2-byte storage workspace is sized for the whole problem
 * (dcn_core_backward_workspace) and reused by every chunk.  Errors as for
 * dcn_core_forward_host.
 */
DCN_API dcn_status dcn_core_backward_host(const dcn_problem* problem, const void* input,
                                  const void* offset, const void* mask,
                                  const void* h_grad_out, void* h_grad_input,
                                  void* h_grad_offset, void* h_grad_mask, void* d_grad_out,
                                  void* d_grad_input, void* d_grad_offset,
                                  void* d_grad_mask, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/* Device workspace the backward needs, in bytes (the backward of the DCNv3
 * extension build guide (trdm.cn), section 2.1): 0 for fp32 storage; for
 * bf16 or fp16 storage an fp32 accumulator for grad_input, N*H*W*G*Cg*4 bytes.
 * Returns 0 for an invalid problem.  The caller allocates and owns it. */
DCN_API size_t dcn_core_backward_workspace(const dcn_problem* problem);

/*
 * Backward: the gradients of the forward above with respect to its input,
 * offsets and mask, i.e. the backward device code of the DCNv3 extension
 * build guide (trdm.cn), section 2.1, obtained by differentiating the
 * sampling and weighted sum of the InternImage-L DCNv3 explainer (wmrh.cn),
 * section 二 steps 2-4 (bilinear weights, softmax over the taps).  All
 * pointers are device pointers owned by the caller.  grad_out: (N, Ho, Wo, C).
 *   grad_input  (N, H, W, C)   OVERWRITTEN: zero-filled on the stream, then
 *               accumulated by a vectorised atomic scatter (the order of
 *               the additions, hence the last bits, may differ between runs)
 *   grad_offset (N, Ho, Wo, G*KK*2), overwritten
 *   grad_mask   (N, Ho, Wo, G*KK), overwritten; with softmax = 1 it is the
 *               gradient with respect to the logits
 * The gradient with respect to an offset at an integer sample coordinate is
 * the one-sided derivative that floor() selects.  All gradients are computed
 * in fp32.  With bf16 or fp16 storage the input gradient is accumulated in
 * the caller's workspace (dcn_core_backward_workspace bytes, 16-byte aligned,
 * contents on entry irrelevant) and rounded to the storage type once at the
 * end (nearest even); grad offset and grad mask are rounded once.  Cg must
 * be 4, 8, 16, 32 or 64; all pointers 16-byte aligned.  workspace may be NULL when the workspace size
 * is 0; a missing or short workspace returns DCN_ERR_INVALID_ARG.
 */
DCN_API dcn_status dcn_core_backward(const dcn_problem* problem, const void* input,
                             const void* offset, const void* mask,
                             const void* grad_out, void* grad_input,
                             void* grad_offset, void* grad_mask, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* Scratch bytes the allocation-free backward below owns, per GPU (16 MiB). */
#define DCN_CORE_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * Backward that allocates nothing and takes no workspace.  The paper has no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory where they run the backward -- plugin hosts and inference
 * runtimes that give a custom operator only its input and output buffers
 * (the runtime owns every other byte of device memory), and latency-critical
 * code that may not call cudaMalloc because it synchronises the device.
 *
 * Arguments and results are those of dcn_core_backward without the
 * workspace.  fp32 storage needs no scratch.  For bf16 or fp16 storage the
 * fp32 grad_input accumulator (N*H*W*G*Cg*4 bytes) lives in a fixed array
 * inside the library of DCN_CORE_NOALLOC_SCRATCH_BYTES; every GPU that loads
 * the library holds that array until the process exits, and a problem whose
 * accumulator is larger returns DCN_ERR_UNSUPPORTED without enqueuing work.
 * The first call on a device looks up the array's device address (once per
 * device and context, with that device current; after cudaDeviceReset the
 * next call looks it up again): make that first call before any stream
 * capture.  Every call shares the one array and each call clears it on its
 * stream before use; calls whose work can overlap on the GPU (other streams,
 * other host threads on the same device) race on it and must be serialised
 * by the caller.  Never calls cudaMalloc, cudaFree or any allocating routine.
 */
DCN_API dcn_status dcn_core_backward_noalloc(const dcn_problem* problem, const void* input,
                                             const void* offset, const void* mask,
                                             const void* grad_out, void* grad_input,
                                             void* grad_offset, void* grad_mask,
                                             cudaStream_t stream);

/* Device workspace dcn_core_backward_deterministic needs, in bytes:
 * 256 + N*H*W*G*Cg*8 (0 for an invalid problem). */
DCN_API size_t dcn_core_backward_deterministic_workspace(const dcn_problem* problem);

/*
 * Backward whose results are bitwise reproducible: run after run, whatever the
 * stream, the launch configuration or the scheduling, the same inputs give the
 * same grad_input, grad_offset and grad_mask bits.  (The pages' backward, DCNv3
 * extension build guide (trdm.cn), section 2.1, accumulates with atomics; this
 * entry point trades speed for reproducibility.)
 *
 * Arguments and results are those of dcn_core_backward; the workspace
 * (dcn_core_backward_deterministic_workspace bytes, 256-byte aligned, contents
 * on entry irrelevant) replaces the 2-byte storage accumulator.  grad_offset and
 * grad_mask are computed exactly as by dcn_core_backward.  grad_input is
 * accumulated exactly in 64-bit fixed point: every fp32 contribution
 * m_k * w_corner * grad_out[c] is rounded to an integer multiple of 2^-S and
 * the integers are summed, so the order of the additions does not matter; the
 * sum is then rounded once to fp32 (and to nearest-even bf16 or fp16 for 2-byte
 * storage).  S is chosen on the device from max|grad_out| (and max|mask| for
 * a raw mask) so that no sum can overflow: 2^-S is about 2^-62 times
 * (max|grad_out| * max|mask weight| * Ho*Wo*KK), far below fp32 resolution
 * for every element except those many orders of magnitude smaller than the
 * largest.  A non-finite grad_out (or raw mask) makes every grad_input
 * element NaN.  Cg must be 4, 8, 16, 32 or 64; all pointers 16-byte aligned.
 * Slower than dcn_core_backward: the 64-bit reductions are scalar.
 */
DCN_API dcn_status dcn_core_backward_deterministic(const dcn_problem* problem, const void* input,
                                                   const void* offset, const void* mask,
                                                   const void* grad_out, void* grad_input,
                                                   void* grad_offset, void* grad_mask,
                                                   void* workspace, size_t workspace_bytes,
                                                   cudaStream_t stream);

/*
 * Offset and mask projection of the DCNv3 block on the tensor cores.  The
 * block predicts each (pixel, group, tap)'s offset pair and mask logit with
 * linear layers on its query features (InternImage-L DCNv3 explainer
 * (wmrh.cn), section 二 steps 1-3); with the two layers' weights stacked
 * row-wise this is one GEMM:
 *     P[pixel, j] = sum_c query[pixel, c] * weight[j, c] + bias[j],
 *     j in [0, G*KK*3),  pixel = (n*Ho + ho)*Wo + wo.
 * Columns j < G*KK*2 are written to `offset` (element j of the pixel, i.e.
 * (g*KK + k)*2 + {dx, dy}), the others to `mask` (element j - G*KK*2), in
 * the layouts dcn_core_forward reads and in problem->dtype.
 *   query   device, bf16, (N, Ho, Wo, Cq), dense; Cq >= 8 and a multiple of 8
 *   weight  device, bf16, (G*KK*3, Cq) row-major (a linear layer's weight)
 *   bias    device, fp32, (G*KK*3), or NULL for none
 *   offset  device, (N, Ho, Wo, G*KK*2); mask device, (N, Ho, Wo, G*KK);
 *           both written entirely, must not overlap the inputs
 * bf16 products are exact in fp32 and are summed in fp32 (tensor-core
 * accumulation in tensor memory, order of the K sum unspecified); each
 * output is rounded once to the storage type.  All pointers 16-byte aligned
 * (bias 4-byte).  Cq not a multiple of 8 or unaligned pointers return
 * DCN_ERR_UNSUPPORTED; the usual problem checks apply.
 */
DCN_API dcn_status dcn_core_offset_mask_projection(const dcn_problem* problem, const void* query,
                                                   int Cq, const void* weight, const float* bias,
                                                   void* offset, void* mask,
                                                   cudaStream_t stream);

/*
 * Guide features of the offset / mask branch (InternImage-L DCNv3 explainer
 * (wmrh.cn), section 二 step 1: before the linear layers of the projection,
 * the block's input passes a depthwise convolution, LayerNorm and GELU).  One
 * pass per pixel, fp32 arithmetic:
 *   conv[c] = dw_bias[c] + sum_{a,b<3} dw_weight[(a*3 + b)*C + c] * input[n, y+a-1, x+b-1, c]
 *             (3x3 window, stride 1, zero padding 1: the output keeps H x W)
 *   z[c]    = (conv[c] - mean) / sqrt(var + ln_eps) * ln_gamma[c] + ln_beta[c]
 *             (mean and biased variance over the C = G*Cg channels of the pixel)
 *   query[n, y, x, c] = z * (1 + erf(z / sqrt(2))) / 2   (GELU), rounded once to bf16
 *   input      device, (N, H, W, C) of problem->dtype, 16-byte aligned
 *   dw_weight  device, fp32, (3, 3, C); dw_bias, ln_gamma, ln_beta device fp32 (C),
 *              each may be NULL (0, 1 and 0); all 16-byte aligned
 *   query      device, bf16, (N, H, W, C), 8-byte aligned, written entirely; it is
 *              the query of dcn_core_offset_mask_projection when Ho = H and Wo = W
 * Only N, H, W, G, Cg and dtype of the problem are used (after the usual
 * checks).  C must be a multiple of 4 and at most 2048, else
 * DCN_ERR_UNSUPPORTED; ln_eps must be finite and >= 0, else
 * DCN_ERR_INVALID_ARG.
 */
DCN_API dcn_status dcn_core_offset_mask_guide(const dcn_problem* problem, const void* input,
                                              const float* dw_weight, const float* dw_bias,
                                              const float* ln_gamma, const float* ln_beta,
                                              float ln_eps, void* query, cudaStream_t stream);

/*
 * The whole offset / mask branch of the DCNv3 block in one kernel: the guide
 * features of dcn_core_offset_mask_guide computed straight into the operand
 * of the projection of dcn_core_offset_mask_projection (InternImage-L DCNv3
 * explainer (wmrh.cn), section 二 steps 1-3), so the bf16 query never goes to
 * device memory.  The result is that of the two calls in a row (query =
 * guide features, Cq = C = G*Cg): the same arithmetic, the same bf16 rounding
 * of the query, the same tensor-core products.
 *   input, dw_weight, dw_bias, ln_gamma, ln_beta, ln_eps: as for
 *              dcn_core_offset_mask_guide (input of problem->dtype)
 *   weight     device, bf16, (G*KK*3, C) row-major; bias device fp32 (G*KK*3) or NULL
 *   offset, mask  device, (N, H, W, G*KK*2) and (N, H, W, G*KK) of problem->dtype,
 *              written entirely
 * The guide keeps the input's size, so the problem's output size must be
 * H x W (stride 1, "same" padding), else DCN_ERR_UNSUPPORTED.  C must be 160
 * or 320 (the InternImage-L stage-1 and stage-2 widths; a 128-pixel operand
 * tile of a wider query does not fit in shared memory beside the weight
 * ring), else DCN_ERR_UNSUPPORTED; alignment rules of the two calls it
 * replaces.
 */
DCN_API dcn_status dcn_core_offset_mask_guide_projection(
    const dcn_problem* problem, const void* input, const float* dw_weight, const float* dw_bias,
    const float* ln_gamma, const float* ln_beta, float ln_eps, const void* weight,
    const float* bias, void* offset, void* mask, cudaStream_t stream);

/*
 * The linear layers on either side of the core operator in the DCNv3 block
 * (InternImage-L DCNv3 explainer (wmrh.cn), section 二: input_proj before it,
 * output_proj after it), as one tensor-core GEMM with bf16 operands:
 *     output[m, j] = sum_c input[m, c] * weight[j, c] + bias[j]
 *   input   device, bf16, (M, K) row-major; K >= 8 and a multiple of 8
 *   weight  device, bf16, (Nout, K) row-major (a linear layer's weight)
 *   bias    device, fp32, (Nout), or NULL
 *   output  device, (M, Nout) in out_dtype (fp32, bf16 or fp16), written entirely
 * Same arithmetic, alignment rules and errors as
 * dcn_core_offset_mask_projection (M*K and M*Nout below 2^31).
 */
DCN_API dcn_status dcn_core_linear_bf16(const void* input, int M, int K, const void* weight,
                                        int Nout, const float* bias, void* output,
                                        dcn_dtype out_dtype, cudaStream_t stream);

/* Synchronises `stream` and reports: DCN_ERR_CUDA if CUDA reports an error,
 * DCN_ERR_OUT_OF_BOUNDS if the bounds-checked build (compiled with
 * -DDCN_CHECK_BOUNDS) skipped an access outside a tensor, DCN_ERR_TIMEOUT if a
 * kernel of this library gave up a bounded wait since the last call (the
 * device error word is then cleared), else DCN_OK. */
DCN_API dcn_status dcn_core_sync_status(cudaStream_t stream);

/* Static description of a status code. */
DCN_API const char* dcn_status_string(dcn_status status);

/* DCN_CORE_ABI_VERSION of the loaded library. */
DCN_API int dcn_core_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DCN_CORE_H_ */
