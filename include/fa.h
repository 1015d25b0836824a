/*
 * fa.h -- C ABI of libfa_sm100: exact IO-aware scaled-dot-product attention
 * (FlashAttention-2 style) for NVIDIA B200 (sm_100a).
 *
 * The operation (unite.ai, "Flash Attention: Revolutionizing Transformer
 * Efficiency", standard-attention definition; causal flag as in
 * downcodes.com "triton transformer", usage section):
 *
 *     S   = scale * Q K^T,  S_ij = -inf where causal and j > i
 *     O   = softmax_rows(S) V
 *     LSE = log(sum_j exp(S_ij))            (natural log, scaled scores)
 *
 * computed in tiles with an online softmax so that S never reaches HBM
 * (same page, "Flash Attention algorithm" and "math behind Flash
 * Attention"); the backward recomputes S from LSE instead of storing it
 * (same page, idea 2, "recomputation").
 *
 * Conventions shared by every entry point
 *   - Layout: Q, K, V, O, dO, dQ, dK, dV are contiguous [B, H, N, d] bf16
 *     (__nv_bfloat16, d fastest); LSE is contiguous [B, H, N] float32.
 *   - All pointers are DEVICE pointers on the current CUDA device, 16-byte
 *     aligned.  The caller allocates and owns every buffer; the library
 *     allocates no device memory.
 *   - d must be 64 or 128; B, H, N >= 1; B*H*N*d < 2^31; scale finite, > 0.
 *   - causal != 0 selects the square, top-left aligned mask: query i attends
 *     to keys j <= i.
 *   - Work is enqueued on `stream` (0 = legacy default stream) and returns
 *     without host synchronisation.  Outputs are fully overwritten.
 *   - Errors: arguments are checked before any launch.  Invalid arguments
 *     return FA_ERR_INVALID_ARG, unsupported shapes or devices
 *     FA_ERR_UNSUPPORTED, launch failures FA_ERR_CUDA.  Nothing is thrown,
 *     nothing exits.  Device-side waits are bounded; a wait that gives up
 *     records a code in a per-device error word read by
 *     fa_check_device_error (FA_ERR_TIMEOUT).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,
    FA_ERR_UNSUPPORTED = 2,
    FA_ERR_CUDA = 3,
    FA_ERR_TIMEOUT = 4
} fa_status;

/*
 * Forward pass.
 *   Q, K, V : [B,H,N,d] bf16 inputs (read only)
 *   O       : [B,H,N,d] bf16 output
 *   LSE     : [B,H,N]   fp32 output, natural-log logsumexp of the scaled
 *             scores per query row (needed by fa_backward)
 * Numerics: bf16 operands, fp32 accumulation and softmax statistics; P is
 * rounded to bf16 for the P.V product; O rounded to bf16 (nearest-even).
 */
fa_status fa_forward(const void *Q, const void *K, const void *V, void *O, float *LSE,
                     int B, int H, int N, int d, float scale, int causal,
                     cudaStream_t stream);

/*
 * Grouped-query / multi-query attention ("FlashAttention-2" item 3 of the
 * unite.ai page: grouped and multi-query attention).  Q and O have H heads;
 * K and V have H_kv heads ([B, H_kv, N, d]); query head h of a batch uses
 * K/V head h / (H / H_kv).  H_kv must divide H (H_kv = 1: multi-query;
 * H_kv = H: identical to fa_forward).  FA_ERR_INVALID_ARG otherwise.
 */
fa_status fa_forward_gqa(const void *Q, const void *K, const void *V, void *O, float *LSE,
                         int B, int H, int H_kv, int N, int d, float scale, int causal,
                         cudaStream_t stream);

/*
 * Padded batches (the padding mask of downcodes.com "triton transformer",
 * BERT example).  seqlens: DEVICE pointer to B int32 values, seqlens[b] in
 * 0..N real tokens of batch b (values outside are clamped), or NULL (all N
 * real, identical to fa_forward_gqa).  Tokens >= seqlens[b] are padding: as
 * keys they are masked for every query; as queries their O rows and LSE are
 * written as 0.  Key blocks entirely in the padding are not read.  Otherwise
 * as fa_forward_gqa (K/V with H_kv heads).
 */
fa_status fa_forward_varlen(const void *Q, const void *K, const void *V, void *O, float *LSE,
                            const int *seqlens, int B, int H, int H_kv, int N, int d,
                            float scale, int causal, cudaStream_t stream);

/*
 * Attention dropout (the attn_dropout option of downcodes.com "triton
 * transformer", usage section; the page gives no formula).  Inverted dropout
 * on the normalised probabilities:
 *     O_i = sum_j P_ij z_ij / q v_j,   LSE as without dropout
 * with the keep bit z_ij of query i, key j of query head bh = b * H + h taken
 * from the counter-based generator Philox-4x32 with 7 rounds (Salmon et al.,
 * "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11):
 *     W = Philox(counter = (j / 16, i, bh, offset), key = (seed & 0xffffffff, seed >> 32))
 *     u = (W[(j % 16) / 4] >> (8 * (2 * (j % 2) + (j % 4) / 2))) & 0xff   (8-bit uniform)
 *     z_ij = (u < t),  t = floor((1 - dropout_p) * 2^8 + 1/2),  q = t / 2^8
 * (i, j counted from the start of the sequence).  q, the keep probability, is
 * the multiple of 2^-8 nearest to 1 - dropout_p, and dividing by it keeps
 * the output unbiased.  The same (seed, offset) given to fa_backward_dropout
 * regenerates the mask; a caller that needs a fresh mask per call changes
 * either.
 *   dropout_p : in [0, 1 - 2^-9] (FA_ERR_INVALID_ARG otherwise, NaN
 *               included); values below 2^-9 (t = 2^8) are exactly
 *               fa_forward_varlen.
 * Other arguments as fa_forward_varlen (seqlens may be NULL; K/V with H_kv
 * heads).  The keep-bit generation costs integer work in the softmax warps.
 */
fa_status fa_forward_dropout(const void *Q, const void *K, const void *V, void *O, float *LSE,
                             const int *seqlens, int B, int H, int H_kv, int N, int d,
                             float scale, int causal, float dropout_p, unsigned long long seed,
                             unsigned int offset, cudaStream_t stream);

/*
 * FP8 forward (the FlashAttention-3 direction of the pages: FP8 compute,
 * systems-analysis.info "FlashAttention-2 (VI)", FlashAttention-3 section).
 *   Q8, K8, V8 : [B,H,N,d] / [B,H_kv,N,d] E4M3 bytes (__nv_fp8_e4m3); the
 *                real inputs are Q8 * descale_q, K8 * descale_k, V8 * descale_v
 *                (per-tensor dequantisation scales, finite and > 0)
 *   O, LSE     : as fa_forward (bf16 O, fp32 natural-log LSE of the scaled
 *                real scores)
 * The S = Q K^T and P.V products run on the tensor core in E4M3 with fp32
 * accumulation; P is rounded to E4M3 (3 mantissa bits) for the P.V product and
 * O is normalised by the sum of the same rounded weights.  d must be 128
 * (FA_ERR_UNSUPPORTED otherwise).  No backward.
 */
fa_status fa_forward_fp8(const void *Q8, const void *K8, const void *V8, void *O, float *LSE,
                         float descale_q, float descale_k, float descale_v, int B, int H,
                         int H_kv, int N, int d, float scale, int causal, cudaStream_t stream);

/*
 * Device workspace fa_backward needs, in bytes (0 on invalid shapes).  It holds
 * D_i = <dO_i, O_i>, LSE in base-2 units and the fp32 dQ accumulator, each
 * padded to a multiple of 128 rows per head, and one int32 counter per
 * 128-row query block (used by fa_backward_deterministic).
 */
size_t fa_backward_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass: the exact gradient of <O, dO> with respect to Q, K and V,
 * recomputing the scores from Q, K and the saved LSE (same page, idea 2).
 *   Q, K, V, O, dO : [B,H,N,d] bf16 (read only); O and LSE from fa_forward
 *   LSE            : [B,H,N] fp32 (read only)
 *   dQ, dK, dV     : [B,H,N,d] bf16 outputs
 *   workspace      : >= fa_backward_workspace_bytes(B,H,N,d) bytes of device
 *                    memory, 16-byte aligned, owned by the caller, contents
 *                    undefined on entry and exit; it must not be shared with
 *                    another call that may run concurrently.
 * dQ is accumulated in fp32 across key blocks with atomic reductions, so its
 * last fp32 bits (and rarely one bf16 ulp) may vary from run to run; dK and
 * dV are deterministic.
 */
fa_status fa_backward(const void *Q, const void *K, const void *V, const void *O,
                      const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                      void *workspace, size_t workspace_bytes,
                      int B, int H, int N, int d, float scale, int causal,
                      cudaStream_t stream);

/*
 * Backward of fa_forward_gqa: dQ is [B,H,N,d]; dK and dV are [B,H_kv,N,d],
 * each the sum over the H / H_kv query heads that share the K/V head (summed
 * in fp32 inside the kernel, deterministic).  Workspace as for fa_backward
 * with H query heads: fa_backward_workspace_bytes(B, H, N, d).
 */
fa_status fa_backward_gqa(const void *Q, const void *K, const void *V, const void *O,
                          const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                          void *workspace, size_t workspace_bytes,
                          int B, int H, int H_kv, int N, int d, float scale, int causal,
                          cudaStream_t stream);

/*
 * Backward of fa_forward_varlen (same seqlens): padding query rows contribute
 * nothing and every gradient row of a padding token is written as 0.
 */
fa_status fa_backward_varlen(const void *Q, const void *K, const void *V, const void *O,
                             const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                             void *workspace, size_t workspace_bytes, const int *seqlens,
                             int B, int H, int H_kv, int N, int d, float scale, int causal,
                             cudaStream_t stream);

/*
 * Backward of fa_forward_dropout: the same (dropout_p, seed, offset) and
 * seqlens as the forward call that produced O and LSE.  With
 * Pd_ij = P_ij z_ij / q:  dV_j = sum_i Pd_ij dO_i,
 * dS_ij = P_ij (z_ij <dO_i, v_j> / q - <dO_i, O_i>), dQ and dK from dS
 * as in fa_backward.  Other arguments as fa_backward_varlen.
 */
fa_status fa_backward_dropout(const void *Q, const void *K, const void *V, const void *O,
                              const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                              void *workspace, size_t workspace_bytes, const int *seqlens,
                              int B, int H, int H_kv, int N, int d, float scale, int causal,
                              float dropout_p, unsigned long long seed, unsigned int offset,
                              cudaStream_t stream);

/*
 * fa_backward_dropout with a run-to-run reproducible dQ.  The pages call the
 * method "exact and deterministic" (systems-analysis.info "FlashAttention-2
 * (VI)", performance section).  dK and dV are always bit-reproducible (each is
 * summed inside one CTA); dQ_i is a sum over key blocks, which the other entry
 * points add into an fp32 accumulator in whatever order the key-block CTAs
 * reach it, so its last bits may vary between runs.  Here the additions into
 * each 128-row dQ block are made in ascending key-block order: a CTA waits
 * (bounded) until every lower key block of the same head has added its part,
 * adds its own and publishes a per-block counter in the workspace.  Results
 * are bitwise identical across runs with the same inputs, grid and device.
 *   Arguments: as fa_backward_dropout (dropout_p = 0 and seqlens = NULL for the
 *     plain backward; H_kv = H for multi-head attention).
 *   Errors: as fa_backward_dropout; a wait that gives up is reported through
 *     fa_check_device_error as FA_ERR_TIMEOUT.
 */
fa_status fa_backward_deterministic(const void *Q, const void *K, const void *V, const void *O,
                                    const void *dO, const float *LSE, void *dQ, void *dK,
                                    void *dV, void *workspace, size_t workspace_bytes,
                                    const int *seqlens, int B, int H, int H_kv, int N, int d,
                                    float scale, int causal, float dropout_p,
                                    unsigned long long seed, unsigned int offset,
                                    cudaStream_t stream);

/*
 * Size of the device array fa_backward_noalloc uses as its workspace (64 MiB).
 * Every GPU on which this library's device code is loaded holds one such
 * array until the process exits, whether or not fa_backward_noalloc is called.
 */
#define FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * fa_backward without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code running under a framework or engine whose
 * allocator owns the whole device and forbids raw cudaMalloc, or a
 * latency-critical path that cannot take the device-wide synchronisation a
 * cudaMalloc/cudaFree may cause.  It allocates nothing: its scratch is a fixed
 * array of FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES inside the library (see the
 * macro above).  The pages describe no such variant; it has no counterpart
 * there.
 *   Arguments, layouts and results: as fa_backward, minus the workspace.
 *   Limit: returns FA_ERR_UNSUPPORTED, launching nothing, when
 *     fa_backward_workspace_bytes(B,H,N,d) > FA_BACKWARD_NOALLOC_MAX_SCRATCH_BYTES
 *     (e.g. B*H = 64 heads of N = 2048, d = 64 need 33 MiB and fit).
 *   First call on each device: looks up the array's device address and sets
 *     kernel attributes (host-side set-up only); make that first call before
 *     any stream capture.  The address is kept for the life of the process,
 *     like the device error word's, so it assumes the device's primary
 *     context lives as long: after cudaDeviceReset on a device, do not call
 *     this library on that device again.
 *   Sharing: every call on a device uses the same array.  Calls whose kernels
 *     can overlap on the GPU (other streams, other host threads) race on it
 *     and give undefined results; serialise them, e.g. on one stream.  Each
 *     call first rewrites the parts of the array it reads, so leftovers from
 *     an earlier call are harmless.
 */
fa_status fa_backward_noalloc(const void *Q, const void *K, const void *V, const void *O,
                              const void *dO, const float *LSE, void *dQ, void *dK, void *dV,
                              int B, int H, int N, int d, float scale, int causal,
                              cudaStream_t stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns FA_OK, FA_ERR_TIMEOUT if a kernel gave up at a bounded wait
 * since the last check (its outputs are then undefined), or FA_ERR_CUDA.
 * If site != NULL it receives the raw code (0 if none).
 */
fa_status fa_check_device_error(cudaStream_t stream, unsigned int *site);

/*
 * Self-test of the failure-detection path (diagnostic; not part of the
 * attention computation).  Enqueues on `stream` a one-CTA kernel whose first
 * warp waits, for at most timeout_ns (1 ns .. 1 s), on a barrier that nothing
 * ever arrives at, exactly as the attention kernels' bounded waits do; it
 * gives up, records a timeout code in the device error word and releases the
 * other waiting warp through the CTA abort flag.  A following
 * fa_check_device_error must return FA_ERR_TIMEOUT with site 0x163; the CUDA
 * context stays usable.  Returns FA_ERR_INVALID_ARG for an out-of-range
 * timeout.
 */
fa_status fa_selftest_bounded_wait(unsigned long long timeout_ns, cudaStream_t stream);

/* Static description of a status code. */
const char *fa_status_str(fa_status status);

/* Library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
