/*
 * dit_attn.h — C ABI of the B200 (sm_100a) DiT joint-attention forward.
 *
 * One call computes, for every batch entry b and head h of one DiT block,
 * full (non-causal) multi-head joint self-attention over the concatenated
 * text + image (or video) latent tokens:
 *
 *     O[b,h] = softmax(scale * Q[b,h] K[b,h]^T) V[b,h]
 *     LSE[b,h,i] = log sum_j exp(scale * Q[b,h,i] . K[b,h,j])
 *
 * This is the attention core of the repeated transformer passes that
 * dominate diffusion inference (page "How to Scale Diffusion Inference
 * Across AMD RDNA 4 GPUs", section "Understanding the Inference Pipeline"),
 * i.e. the operation behind the pages' selectable BF16 / FP8 attention
 * backends (same page, section "Select an Attention Backend and Compile the
 * Transformer"; fosswire.org summary "AMD releases xDiT configurations for
 * scaling diffusion inference on RDNA 4 GPUs", section "Technical
 * implementation of xDiT on RDNA 4").  The pages cite "Attention Is All You
 * Need" and FlashAttention-2 for it (page "xDiT: an Inference Engine for
 * Diffusion Transformers (DiTs) with Massive Parallelism", reference list);
 * they state no formula, layout or interface, so the layout below is the
 * plainest one ([B, H, L, D], D innermost, as in torch's SDPA).
 *
 * All functions are host functions, thread-safe, and never synchronise the
 * device unless stated.  The library allocates no device memory.
 *
 * Every entry point runs on the current device.  One that takes device
 * buffers checks each of them (cudaPointerGetAttributes) before anything is
 * enqueued and returns DIT_ATTN_ERR_DEVICE when one is host memory, another
 * GPU's memory, or covered by no CUDA allocation (dit_attn_fwd_ulysses takes
 * peers' memory mapped into this context for its shards).
 */
#ifndef DIT_ATTN_H
#define DIT_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Input element type. */
typedef enum {
    DIT_ATTN_BF16 = 0,      /* q, k, v bf16                                  */
    DIT_ATTN_FP8_E4M3 = 1   /* q, k, v OCP FP8 E4M3 ("fn") + fp32 scales     */
} dit_attn_dtype;

/* Return codes. */
typedef enum {
    DIT_ATTN_OK = 0,
    DIT_ATTN_ERR_NULL = 1,     /* a required pointer is NULL                 */
    DIT_ATTN_ERR_SHAPE = 2,    /* B, H, L or D outside the supported range   */
    DIT_ATTN_ERR_DTYPE = 3,    /* unknown dtype, or scales given for bf16    */
    DIT_ATTN_ERR_ALIGN = 4,    /* q/k/v/o not 16-byte, lse/scales not 4-byte aligned */
    DIT_ATTN_ERR_ARCH = 5,     /* no CUDA device, or the current device is not sm_100 */
    DIT_ATTN_ERR_LAUNCH = 6,   /* a CUDA runtime call or the kernel launch failed */
    DIT_ATTN_ERR_TIMEOUT = 7,  /* a device-side wait ran past its time limit */
    DIT_ATTN_ERR_VALUE = 8,    /* scale is negative, NaN or infinite         */
    DIT_ATTN_ERR_DEVICE = 9    /* a buffer is not device memory of the current device
                                  (host memory, another GPU's, or no allocation) */
} dit_attn_status;

/*
 * dit_attn_fwd — attention forward, asynchronous on `stream`.
 *
 * q, k, v   device pointers, contiguous [B, H, L, D] (D innermost), element
 *           type `dtype`; 16-byte aligned.  Read only.
 * o         device pointer, contiguous [B, H, L, D] bf16 (for both dtypes);
 *           16-byte aligned.  Fully overwritten.
 * lse       device pointer to [B, H, L] fp32, or NULL to skip it.  Receives
 *           the natural-log log-sum-exp of each row's scaled logits (for
 *           FP8, of the dequantised logits).
 * B, H      batch entries and heads, >= 1, B*H <= 2^31-1.
 * L         joint sequence length (text + image/video tokens), 1 <= L and
 *           B*H*L*D < 2^40.
 * D         head dimension: 64 or 128.
 * scale     softmax scale, finite and >= 0 (the DiT blocks use 1/sqrt(D)).
 * dtype     DIT_ATTN_BF16 or DIT_ATTN_FP8_E4M3.
 * q_scale, k_scale, v_scale
 *           FP8 only: device pointers to [B, H] fp32 per-head dequantisation
 *           scales (x ~= s * x_hat); logits are scale*qs*ks*(q_hat.k_hat) and
 *           O is vs * sum p v_hat / sum p.  Must be NULL for bf16.
 * stream    CUDA stream (0 = legacy default stream).
 *
 * Ownership: the caller owns every buffer; the library uses no pointer
 * after the call returns (the kernel reads them in stream order).  It keeps
 * the TMA tensor maps of the last 16 distinct (device, q, k, v, o, B*H, L, D,
 * dtype) calls, so a repeated call (every layer and denoising step) skips
 * their encoding; a map holds only an address, a shape and strides, so an
 * entry is valid for whatever buffer later sits at that address.
 * Errors: argument errors are reported before anything is enqueued.  A
 * device-side wait that exceeds its limit (default 4 s) makes the kernel
 * stop early and record an error word, reported by
 * dit_attn_check_device_error(); the output is then undefined.
 * Non-goals: causal masks, dropout, backward, variable-length batches.
 */
int dit_attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                 int B, int H, int L, int D, float scale, int dtype,
                 const float *q_scale, const float *k_scale, const float *v_scale,
                 cudaStream_t stream);

/* Static, human-readable text for a return code (never NULL). */
const char *dit_attn_status_string(int status);

/*
 * dit_attn_check_device_error — synchronises `stream`, reads the current
 * device's error word, clears it and returns DIT_ATTN_OK or
 * DIT_ATTN_ERR_TIMEOUT (DIT_ATTN_ERR_LAUNCH if a CUDA call fails).  If
 * `detail` is not NULL it receives the raw word (0 = no error; otherwise
 * bits 0..7 the code, bits 8..15 the wait site that gave up).
 */
int dit_attn_check_device_error(cudaStream_t stream, uint32_t *detail);

/*
 * dit_attn_set_wait_limit_ns — time limit of every device-side wait of
 * later launches from this process (default 4e9 ns; 0 restores it).
 */
void dit_attn_set_wait_limit_ns(uint64_t ns);

/*
 * dit_attn_selftest_wait_timeout — launches one CTA whose thread waits, with
 * the kernels' own bounded wait, on an mbarrier that nothing completes; the
 * wait gives up after `limit_ns` and records DIT_ATTN_ERR_TIMEOUT in the
 * error word.  Used by tests to check the timeout path without hanging the
 * GPU.  Asynchronous on `stream`.
 */
int dit_attn_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/*
 * dit_attn_launches_per_call — number of kernel launches one dit_attn_fwd
 * call with these arguments enqueues (for launch accounting).
 */
int dit_attn_launches_per_call(int B, int H, int L, int D, int dtype);

/* Largest number of partial results dit_attn_lse_merge combines in one call. */
#define DIT_ATTN_MERGE_MAX_PARTS 8

/*
 * dit_attn_lse_merge — combines partial attention results over disjoint key
 * chunks into the result over their union, asynchronous on `stream`.
 *
 * This is the combine step of ring attention / USP: a block of query rows
 * meets the K/V chunks one at a time and the partial results are merged.
 * The xDiT paper cites both methods in its reference list ("xDiT: an
 * Inference Engine for Diffusion Transformers (DiTs) with Massive
 * Parallelism"), and the 2-GPU script of the page "Accelerating Diffusers and
 * xDiT Image Generation with MXFP4 using AMD Quark on AMD Instinct MI350 GPUs"
 * sets its `ring degree`.  The pages give no formula; the exact log-sum-exp
 * rule is used.  Per row,
 *
 *     lse = M + log sum_c exp(lse_c - M),   M = max_c lse_c,
 *     o   = sum_c exp(lse_c - lse) o_c,
 *
 * and a row whose parts all have lse = -inf gives o = 0, lse = -inf.  The
 * (o_c, lse_c) are exactly what dit_attn_fwd returns for the same query rows
 * over key chunk c.
 *
 * o_parts   host array of n_parts device pointers, each to [rows, D] bf16
 *           (e.g. [B, H, L, D] with rows = B*H*L); 16-byte aligned.
 * lse_parts host array of n_parts device pointers, each to [rows] fp32
 *           natural-log LSE (-inf allowed: an empty chunk); 4-byte aligned.
 * n_parts   1 .. DIT_ATTN_MERGE_MAX_PARTS.
 * o         device pointer to [rows, D] bf16, 16-byte aligned; may be the
 *           same buffer as any o_parts[c] (each element is read before it is
 *           written, by the same thread).
 * lse       device pointer to [rows] fp32, or NULL to skip it; may be the
 *           same buffer as any lse_parts[c].
 * rows      >= 0; rows * D < 2^40.  With rows = 0 nothing is enqueued and
 *           the device pointers are not examined (they may be NULL).
 * D         64 or 128.
 *
 * Ownership: the caller owns every buffer; the host arrays are read during
 * the call only.  Errors: argument errors (DIT_ATTN_ERR_NULL, _SHAPE,
 * _ALIGN, _ARCH) are reported before anything is enqueued; a launch failure
 * returns DIT_ATTN_ERR_LAUNCH.  The kernel has no waits.
 */
int dit_attn_lse_merge(const void *const *o_parts, const float *const *lse_parts, int n_parts,
                       void *o, float *lse, long long rows, int D, cudaStream_t stream);

/*
 * dit_attn_residual_diff_workspace_bytes — bytes of device workspace that
 * dit_attn_residual_diff needs for n elements (0 if n < 1).  At most
 * 16 + 16 * 1184 bytes.
 */
size_t dit_attn_residual_diff_workspace_bytes(long long n);

/*
 * dit_attn_residual_diff — the step-cache reuse decision, asynchronous on
 * `stream`.
 *
 * Step caching (DBCache) reuses transformer work from the previous denoising
 * step when the residual of the first blocks has changed little, against a
 * `residual diff threshold` (0.12 in the published setting): page "How to
 * Scale Diffusion Inference Across AMD RDNA 4 GPUs", section "Skip
 * Transformer Work Only When the Model Has Enough Steps".  The page gives no
 * formula; this computes the relative L1 change
 *
 *     diff = sum_i |cur_i - prev_i| / sum_i |prev_i|    (0/0 = 0, x/0 = +inf)
 *     reuse = diff < threshold
 *
 * in one pass (fp32 per thread, fp64 across threads and blocks, summed in a
 * fixed order, so repeated calls give identical results).
 *
 * cur, prev      device pointers to n bf16 values each (the residual of the
 *                current and of the previous step), 16-byte aligned.
 * n              1 <= n < 2^40.
 * threshold      the reuse threshold; not NaN.
 * workspace      device buffer of at least
 *                dit_attn_residual_diff_workspace_bytes(n) bytes, 16-byte
 *                aligned, zero-filled before its first use; each call leaves
 *                it zeroed again.  Calls sharing a workspace must be ordered
 *                (one stream).
 * diff_out       device pointer to one fp32 (diff), or NULL.
 * reuse_out      device pointer to one int32 (1 = reuse, 0 = compute), or NULL;
 *                not both NULL.
 *
 * Ownership: the caller owns every buffer.  Errors (before anything is
 * enqueued): DIT_ATTN_ERR_NULL, _SHAPE (n out of range or workspace too
 * small), _ALIGN, _VALUE (NaN threshold), _ARCH; DIT_ATTN_ERR_LAUNCH if the
 * launch fails.  The kernel has no waits.
 */
int dit_attn_residual_diff(const void *cur, const void *prev, long long n, float threshold,
                           void *workspace, size_t workspace_bytes, float *diff_out, int *reuse_out,
                           cudaStream_t stream);

/*
 * dit_attn_mxfp4_quantize — MXFP4 (OCP Microscaling, 1x32 blocks) quantiser
 * of bf16 activations, asynchronous on `stream`.
 *
 * The page "Accelerating Diffusers and xDiT Image Generation with MXFP4 using
 * AMD Quark on AMD Instinct MI350 GPUs" (sections "MXFP4 Quantization",
 * "MXFP4 Kernel") quantises linear-layer activations on the fly to MXFP4:
 * 32 consecutive values along a row share one E8M0 scale and each is a 4-bit
 * E2M1 float.  The page does not restate the rule; the OCP MX definition it
 * cites is used: per block, s = clamp(floor(log2 max|v|) - 2, -127, 127)
 * (-127 for a zero block), q_i = E2M1(v_i / 2^s) rounded to nearest even and
 * saturated at +-6, with the sign kept (-0 included).
 *
 * x       device pointer, bf16 [rows, K] row-major, 16-byte aligned.  Finite
 *         values only (non-finite inputs give unspecified codes).
 * q       device pointer, uint8 [rows, K/2]: two codes per byte, the first
 *         element of each pair in bits 0..3; 16-byte aligned.
 * scales  device pointer, uint8 [rows, K/32]: the E8M0 byte s + 127 per block.
 * rows    >= 0 (0: nothing is enqueued, pointers unused); rows * K < 2^40.
 * K       a multiple of 32.
 *
 * Errors (before anything is enqueued): DIT_ATTN_ERR_SHAPE, _NULL, _ALIGN,
 * _ARCH; DIT_ATTN_ERR_LAUNCH if the launch fails.  The kernel has no waits.
 */
int dit_attn_mxfp4_quantize(const void *x, void *q, void *scales, long long rows, int K, cudaStream_t stream);

/*
 * Local data movement of Ulysses sequence parallelism (page "How to Scale
 * Diffusion Inference Across AMD RDNA 4 GPUs", section "Balance Transformer
 * Work and Communication": tokens are divided across GPUs and every attention
 * layer exchanges data with an all-to-all; `--use fp8 comms` sends it in
 * FP8).  The exchange itself is a collective of the caller's (NCCL); these
 * three calls are the per-GPU steps around it.  All asynchronous on
 * `stream`; argument errors are returned before anything is enqueued; no
 * waits on the device.
 *
 * dit_attn_block_transpose — out[c][r] = in[r][c] for an R x C grid of
 * contiguous blocks of block_bytes each (a multiple of 4; 16 with 16-byte
 * aligned pointers takes 16-byte copies).  in and out must not overlap.
 * R, C, block_bytes >= 0 (any 0: nothing is enqueued, pointers unused);
 * R * C * block_bytes <= 2^40.
 */
int dit_attn_block_transpose(const void *in, void *out, long long R, long long C, long long block_bytes,
                             cudaStream_t stream);

/*
 * dit_attn_absmax_rows — amax[r] = max_i |x[r][i]| (fp32) for bf16 rows of
 * row_len values (a multiple of 8), e.g. rows = B*H of a [B, H, Ls, D] shard.
 * x 16-byte aligned, amax 4-byte aligned.  Enqueues a zero fill of amax and
 * one kernel whose CTAs each take a chunk of a row and combine their maxima
 * atomically (the result does not depend on their order).  rows = 0: nothing
 * is enqueued.
 */
int dit_attn_absmax_rows(const void *x, float *amax, long long rows, long long row_len, cudaStream_t stream);

/*
 * dit_attn_quantize_e4m3_rows — per row r, with s = amax[r] / 448 (fp32,
 * correctly rounded; 1 if amax[r] == 0): q[r][i] = E4M3(x[r][i] / s), the
 * quotient correctly rounded in fp32, then rounded to nearest even and
 * saturated at +-448 (OCP FP8 E4M3).  scale_out[r] = s (the dequantisation
 * scale dit_attn_fwd takes), or NULL.  row_len a multiple of 16; x and q
 * 16-byte aligned.  rows = 0: nothing is enqueued.
 */
int dit_attn_quantize_e4m3_rows(const void *x, const float *amax, void *q, float *scale_out, long long rows,
                                long long row_len, cudaStream_t stream);

/*
 * dit_attn_fwd_ulysses — Ulysses attention with both exchanges fused into
 * the attention kernel (page "How to Scale Diffusion Inference Across AMD
 * RDNA 4 GPUs", section "Balance Transformer Work and Communication").
 *
 * n_ranks shards, shard c holding tokens [c Ls, (c + 1) Ls) of the joint
 * sequence for all H heads: q_shards[c], k_shards[c], v_shards[c] are
 * [B, H, Ls, D] (bf16, or e4m3 with dtype DIT_ATTN_FP8_E4M3), o_shards[c]
 * [B, H, Ls, D] bf16, lse_shards[c] [B, H, Ls] fp32.  The call computes
 * dit_attn_fwd's attention over all L = n_ranks Ls tokens for the head group
 * [rank H / n_ranks, (rank + 1) H / n_ranks), reading every tile from the
 * shard that holds it, and writes those heads' rows of every shard's O and
 * LSE; other heads' rows are not touched.  The n_ranks calls rank = 0 ..
 * n_ranks - 1 together produce the whole attention in the shards' layout.
 *
 * The pointer arrays are host arrays of n_ranks device pointers.  A pointer
 * may address another GPU's memory mapped into the current context (CUDA IPC
 * or peer access, set up by the caller); the kernel reads and writes it with
 * plain TMA copies (no cluster multicast).  The caller orders the call after
 * every shard's q/k/v are written and orders readers of o/lse after the calls
 * of all ranks that write them (on several GPUs: a stream synchronisation and
 * a barrier of the process group).
 *
 * FP8: q/k/v_scale are [B, H] dequantisation scales of all heads, the same in
 * every shard (per-head scales agreed across ranks).  lse_shards may be NULL
 * (no LSE); otherwise every entry is non-NULL.
 * Requirements: 1 <= n_ranks <= 8, 0 <= rank < n_ranks, H % n_ranks == 0,
 * Ls % 64 == 0, D in {64, 128}, every pointer 16-byte aligned (LSE 4-byte).
 * Errors as dit_attn_fwd (before anything is enqueued).  Device-side wait
 * timeouts (4 s) are reported by dit_attn_ulysses_check_device_error.
 */
int dit_attn_fwd_ulysses(const void *const *q_shards, const void *const *k_shards, const void *const *v_shards,
                         void *const *o_shards, float *const *lse_shards, int n_ranks, int rank, int B, int H,
                         int Ls, int D, float scale, int dtype, const float *q_scale, const float *k_scale,
                         const float *v_scale, cudaStream_t stream);

/*
 * dit_attn_ulysses_check_device_error — dit_attn_check_device_error for the
 * fused Ulysses kernel (it keeps its own device error word): synchronises
 * `stream`, returns DIT_ATTN_ERR_TIMEOUT (and clears the word) if a wait of
 * that kernel timed out, with the word in *detail if detail is non-NULL.
 */
int dit_attn_ulysses_check_device_error(cudaStream_t stream, uint32_t *detail);

/*
 * dit_attn_residual_diff_noalloc — dit_attn_residual_diff without a caller
 * workspace and without allocating anything.  The pages have no counterpart
 * of this entry point.  It is for callers that cannot allocate device memory
 * where they take the decision: a serving loop whose memory is all handed out
 * by its own pool, which must not call cudaMalloc there (cudaMalloc can
 * synchronise the device and stall every stream), or a host runtime that
 * gives its plug-ins no allocator at all.
 *
 * The scratch is a fixed array of 16 + 16 * 1184 bytes in the library's own
 * device memory, which every GPU that loads the library keeps until the
 * process exits.  It is zero at load and every call leaves it zero.  Its
 * device address is looked up (cudaGetSymbolAddress) by the first call on
 * each device and CUDA context, with that device current; make that first
 * call before any stream capture.  Later calls reuse the address.
 *
 * Same arguments, results and errors as dit_attn_residual_diff, minus the
 * workspace.  n above what the fixed scratch covers is rejected with
 * DIT_ATTN_ERR_SHAPE (the scratch covers every n < 2^40).  Because every call
 * shares the one scratch, calls on one device must be ordered (one stream, or
 * streams ordered by events): calls that overlap on the GPU race on it.
 */
int dit_attn_residual_diff_noalloc(const void *cur, const void *prev, long long n, float threshold,
                                   float *diff_out, int *reuse_out, cudaStream_t stream);

/*
 * dit_attn_gemm_fp8 — FP8 linear layer: y = a_scale * w_scale * (A W^T),
 * asynchronous on `stream`.
 *
 * The page "How to Scale Diffusion Inference Across AMD RDNA 4 GPUs" (section
 * "Make the Model Fit Before Tuning Latency") runs the DiT's linear layers
 * (QKV and output projections, MLPs) in FP8; the page prints no formula, so
 * the GEMM of the dequantised operands is taken, with one fp32
 * dequantisation scale per tensor (x ~= s * x_hat).
 *
 * a   device pointer, [M, K] e4m3 codes (OCP FP8 "fn"), row-major (K
 *     contiguous): the activations.  16-byte aligned.  Read only.
 * w   device pointer, [N, K] e4m3 codes, row-major: the weight.  16-byte
 *     aligned.  Read only.
 * y   device pointer, [M, N] bf16, row-major; fully overwritten with the
 *     fp32 result rounded to nearest.  16-byte aligned.
 * M   rows (tokens), 0 <= M < 2^31 (0: nothing is done).
 * N   output features, >= 8 and a multiple of 8.
 * K   input features, >= 16 and a multiple of 16.
 * a_scale, w_scale  finite fp32 dequantisation scales of a and w.
 *
 * Products are exact and accumulate in fp32 on the tensor cores
 * (tcgen05.mma kind::f8f6f4), in a fixed order: results are deterministic.
 * Errors (before anything is enqueued): DIT_ATTN_ERR_SHAPE, _NULL, _ALIGN,
 * _VALUE (a non-finite scale), _ARCH, _DEVICE; DIT_ATTN_ERR_LAUNCH if the
 * launch fails.  Device-side wait timeouts (4 s) are reported by
 * dit_attn_gemm_check_device_error.  NaN codes are outside the contract.
 */
int dit_attn_gemm_fp8(const void *a, const void *w, void *y, long long M, int N, int K, float a_scale,
                      float w_scale, cudaStream_t stream);

/*
 * dit_attn_mxfp4_tiled_scale_bytes — size in bytes of the tiled E8M0 scale
 * layout dit_attn_gemm_mxfp4 reads, for a matrix of `rows` rows and K columns
 * (K a multiple of 32): ceil(rows / 128) * G * 512 with G = 2 ceil(K / 256).
 * Returns 0 for rows < 1 or a bad K.  Host only; no CUDA call.
 */
long long dit_attn_mxfp4_tiled_scale_bytes(long long rows, int K);

/*
 * dit_attn_mxfp4_tile_scales — rearranges MXFP4 block scales from the plain
 * layout dit_attn_mxfp4_quantize writes ([rows, K / 32] E8M0 bytes, row-major)
 * into the tiled layout the tensor cores read in dit_attn_gemm_mxfp4:
 *
 *     tiled[((r / 128) G + b / 4) 512 + 16 (r % 32) + 4 ((r % 128) / 32) + b % 4]
 *         = plain[r][b],   G = 2 ceil(K / 256),
 *
 * zero for the padding rows and blocks.  Each 512-byte atom holds the scales
 * of 128 rows for 4 consecutive 32-element blocks.  This layout is this
 * library's choice (the pages say nothing of scale layouts); it is the one
 * from which a bulk copy and a TMEM copy put every scale where the block-scaled
 * MMA reads it.  Weights are tiled once; activations after each quantisation.
 *
 * plain  device pointer, [rows, K / 32] bytes.  Read only.
 * tiled  device pointer, dit_attn_mxfp4_tiled_scale_bytes(rows, K) bytes,
 *        16-byte aligned.  Fully overwritten.
 * Errors (before anything is enqueued): DIT_ATTN_ERR_SHAPE, _NULL, _ALIGN,
 * _ARCH, _DEVICE; DIT_ATTN_ERR_LAUNCH.  rows = 0 is a no-op.
 */
int dit_attn_mxfp4_tile_scales(const void *plain, void *tiled, long long rows, int K, cudaStream_t stream);

/*
 * dit_attn_gemm_mxfp4 — MXFP4 linear layer: Y = A W^T with A and W in MXFP4
 * (OCP Microscaling: E2M1 values sharing one E8M0 scale per 32 consecutive K
 * elements), bf16 out, asynchronous on `stream`.
 *
 * The page "Accelerating Diffusers and xDiT Image Generation with MXFP4 using
 * AMD Quark on AMD Instinct MI350 GPUs" (sections "MXFP4 Quantization" and
 * "MXFP4 Kernel") runs the DiT's linear layers as FP4 x FP4 GEMMs on MXFP4
 * activations (quantised on the fly in 1x32 blocks, dit_attn_mxfp4_quantize)
 * and MXFP4 weights.  The page prints no formula; this computes the GEMM of
 * the dequantised operands, y[m][n] = sum_k a[m][k] w[n][k].
 *
 * a         device pointer, [M, K / 2] packed E2M1 codes (two per byte, the
 *           first element of a pair in the low nibble), 16-byte aligned.
 * a_scales  device pointer, A's scales in the tiled layout
 *           (dit_attn_mxfp4_tile_scales), 16-byte aligned.
 * w         device pointer, [N, K / 2] packed codes of the weight.
 * w_scales  device pointer, W's scales, tiled.
 * y         device pointer, [M, N] bf16 row-major; fully overwritten with the
 *           fp32 result rounded to nearest.  16-byte aligned.
 * M >= 0 (0: nothing is done), N >= 8 and a multiple of 8, K >= 32 and a
 * multiple of 32.
 *
 * The scaled products are exact and accumulate in fp32 on the tensor cores
 * (tcgen05.mma kind::mxf4, block scales read from TMEM), in a fixed order.
 * Errors (before anything is enqueued): DIT_ATTN_ERR_SHAPE, _NULL, _ALIGN,
 * _ARCH, _DEVICE; DIT_ATTN_ERR_LAUNCH.  Device-side wait timeouts are
 * reported by dit_attn_gemm_check_device_error.  E8M0 0xFF (NaN) scales are
 * outside the contract.
 */
int dit_attn_gemm_mxfp4(const void *a, const void *a_scales, const void *w, const void *w_scales, void *y,
                        long long M, int N, int K, cudaStream_t stream);

/*
 * dit_attn_gemm_check_device_error — dit_attn_check_device_error for the
 * low-precision GEMM kernels (they keep their own device error word):
 * synchronises `stream`, returns DIT_ATTN_ERR_TIMEOUT (and clears the word)
 * if a wait of those kernels timed out, with the word in *detail if detail is
 * non-NULL.
 */
int dit_attn_gemm_check_device_error(cudaStream_t stream, uint32_t *detail);

#ifdef __cplusplus
}
#endif
#endif /* DIT_ATTN_H */
