/*
 * qlora.h -- C ABI of libqlora: the QLoRA frozen-base linear layer on one
 * NVIDIA B200 (sm_100a).
 *
 * The frozen base weight W [rows = N out-features, cols = K in-features] is
 * stored as blockwise NF4: 64 consecutive weights of a row share one absmax
 * scale, each weight is the 4-bit index of the nearest of 16 normal-quantile
 * levels, and the block scales are themselves quantised to 8 bits in groups
 * of 256 ("QLoRA", learning-llms.pages.dev/topics/qlora, the bullets on
 * 64-weight blocks and on NF4; "QLoRA", infra.bea.ai, §1 "How QLoRA Works",
 * subsections "Key Innovation: NF4" and "Double Quantization").  The
 * weight is dequantised to bf16 just in time for each matmul and never
 * updated; the rank-r LoRA adapters A [r, K] and B [N, r] stay in bf16 and
 * are the only tensors that receive gradients (learning-llms page, the bullet
 * on 4-bit storage with bf16 compute, and the forward equation; infra.bea.ai
 * page, section "The Backward Pass Through Quantization").
 *
 * Conventions shared by every call
 *   - All matrices are row-major.  Activations X [M, K], Y [M, N], dY [M, N],
 *     dX [M, K]; adapters A [r, K], B [N, r]; s = alpha / r.
 *   - Array arguments are DEVICE pointers owned by the caller, except where a
 *     comment says host.  bf16 arrays are passed as void*.  Every device
 *     pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Arguments are validated synchronously; the work is enqueued
 *     asynchronously on `stream`.  No call allocates memory, synchronises, or
 *     keeps state between calls.
 *   - `d_status` (nullable) is a device int the kernels OR error bits into:
 *     QLORA_DEV_NONFINITE_BIT (a non-finite weight seen by the quantiser or
 *     the merge, or a non-finite gradient seen by the Adam step) and
 *     QLORA_DEV_TIMEOUT_BIT (a pipeline wait gave up after ~2 s, or the
 *     bound set by qlora_debug_set_wait_limit; the kernel then returns
 *     early and its outputs are unspecified).  The caller zeroes
 *     it and reads it after synchronising.
 *   - Errors: a call that returns a validation error (anything but QLORA_OK
 *     and QLORA_ERR_CUDA) has enqueued nothing.  QLORA_ERR_CUDA means a
 *     launch or tensor-map call failed; launches the same call had already
 *     enqueued may still run, and its outputs are unspecified.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1, /* null pointer, bad shape, misalignment, bad enum */
  QLORA_ERR_UNSUPPORTED = 2, /* well-formed but outside what is built (e.g. block != 64) */
  QLORA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, tensor map) */
  QLORA_ERR_NONFINITE = 4,   /* reserved for callers mapping QLORA_DEV_NONFINITE_BIT */
  QLORA_ERR_TIMEOUT = 5,     /* reserved for callers mapping QLORA_DEV_TIMEOUT_BIT */
  QLORA_ERR_WORKSPACE = 6,   /* workspace null or smaller than qlora_workspace_bytes() */
  QLORA_ERR_SCRATCH_LIMIT = 7 /* problem needs more than the fixed no-allocation scratch */
} qlora_status;

#define QLORA_DEV_NONFINITE_BIT 1
#define QLORA_DEV_TIMEOUT_BIT 2

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/*
 * Optional timing hook for qlora_linear_fwd / qlora_linear_bwd: CUDA events
 * (cudaEvent_t passed as void*) that the call records on `stream` right
 * before and right after its fused NF4 GEMM launch, so that a caller can
 * time that kernel alone.  The struct and either member may be NULL; the
 * events are owned by the caller.  Under stream capture the records become
 * event nodes of the graph, so every replay records them.
 */
typedef struct {
  void* gemm_start;
  void* gemm_end;
} qlora_gemm_events;

/*
 * One NF4 weight.  Describes caller-owned device arrays; the library never
 * frees them.
 *   codes       [rows, cols/2] uint8: byte j of a row holds the code of element
 *               2j in its low nibble and of element 2j+1 in its high nibble.
 *   absmax_q8   [rows*cols/64] uint8 (double_quant = 1 or 2): block b is
 *               elements 64b .. 64b+63 of the row-major matrix.
 *   group_scale [ceil(rows*cols/64/256)] fp32 (double_quant = 1 or 2): group
 *               g covers blocks 256g .. 256g+255, so groups may cross rows.
 *   absmax_f32  [rows*cols/64] fp32 (double_quant = 0, or an optional extra
 *               output of the quantiser when non-null).
 * double_quant selects the second-level format of the block scales:
 *   0 (QLORA_DQ_NONE): fp32 absmax per block, absmax_f32[b];
 *   1 (QLORA_DQ_U8):   linear 8-bit, float(absmax_q8[b]) * group_scale[b/256],
 *                      group_scale = max absmax / 255 (the learning-llms
 *                      page's 8-bit double quantisation);
 *   2 (QLORA_DQ_E4M3): FP8 E4M3 codes, E4M3(absmax_q8[b]) * group_scale[b/256],
 *                      group_scale = max absmax / 448 ("QLoRA", infra.bea.ai,
 *                      §1 subsection "Double Quantization": scales to FP8).
 * Both 8-bit formats store 4 + 8/64 + 32/16384 = 4.127 bits per weight.
 */
#define QLORA_DQ_NONE 0
#define QLORA_DQ_U8 1
#define QLORA_DQ_E4M3 2
typedef struct {
  int64_t rows;          /* N */
  int64_t cols;          /* K, a multiple of 64 */
  int32_t blocksize;     /* must be 64 */
  int32_t group;         /* must be 256 */
  int32_t double_quant;  /* QLORA_DQ_*: 1 or 2: absmax_q8 + group_scale; 0: absmax_f32 */
  int32_t reserved;      /* must be 0 */
  uint8_t* codes;
  uint8_t* absmax_q8;
  float* group_scale;
  float* absmax_f32;
} qlora_nf4_weight;

/*
 * Byte sizes of the three arrays of an NF4 weight: codes rows*cols/2,
 * absmax rows*cols/64 (x4 without double quantisation), group scales
 * 4*ceil(rows*cols/16384) (0 without).  Storage: 4 + 8/64 + 32/16384 =
 * 4.127 bits per weight with double quantisation, 4.5 without -- the
 * overhead figures of the learning-llms page (the bullet on 64-weight blocks
 * and the paragraph after its memory table).
 * Host-only; no GPU needed.  Output pointers are host pointers.
 */
qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int double_quant,
                             size_t* codes_bytes, size_t* absmax_bytes,
                             size_t* group_bytes);

/*
 * The 16 NF4 levels (code 0..15, ascending, code 7 = 0) into host out[16].
 * Normal quantiles normalised to [-1, 1] (QLoRA paper construction).
 */
void qlora_nf4_codebook(float* out16);

/*
 * One-shot quantiser, run once when the model is loaded (katajob.com page,
 * section "The mechanism": the base is quantised a single time, at load).  W: device [rows, cols], fp32 (w_dtype = QLORA_F32) or bf16.
 * Per 64-block: absmax; x = w * fp32(1/absmax); code = nearest NF4 level
 * (ties to the lower code); a block with absmax below FLT_MIN is all code 7.
 * With double_quant = 1, per 256-block group: s = fp32(max absmax / 255),
 * q8 = min(255, rint(absmax / s)); with double_quant = 2: s = fp32(max
 * absmax / 448), q8 = the E4M3 code of fp32(absmax / s), round to nearest
 * even, saturating at 448 (in both, s = 0 and q8 = 0 when the group max is
 * below FLT_MIN); the codes use the fp32 absmax.  out->absmax_f32 is
 * written when non-null.  A non-finite weight sets QLORA_DEV_NONFINITE_BIT;
 * the outputs are then unspecified.
 */
qlora_status qlora_quantize_nf4(const void* W, qlora_dtype w_dtype,
                                const qlora_nf4_weight* out, int* d_status,
                                void* stream);

/*
 * Dequantise to bf16: W_out[e] = bf16_rne(fp32(level[code] * scale)), the
 * just-in-time bf16 reconstruction of the learning-llms page (the bullet on
 * 4-bit storage with bf16 compute).  W_out: device [rows, cols] bf16.
 */
qlora_status qlora_dequantize(const qlora_nf4_weight* Wq, void* W_out, void* stream);

/*
 * Workspace bytes that qlora_linear_fwd / qlora_linear_bwd need for this
 * shape (M tokens, weight N x K, rank r).  Host-only.  Returns 0 for an
 * invalid shape.
 */
size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Forward ("QLoRA", learning-llms page, the forward equation
 * h = W^x + (alpha/r) B(Ax), W^ = dequant(W_4bit)), row-major:
 *     T = X A^T  [M, r]          Y = X W^T + s T B^T  [M, N]
 * X bf16 [M, K]; A bf16 [r, K]; B bf16 [N, r]; Y bf16 [M, N] (written).
 * T_save (nullable) fp32 [M, r]: T for the backward.  1 <= r <= 256.
 * M > 16: W^ is dequantised tile by tile in shared memory inside the
 * GEMM; the adapter product enters the same fp32 accumulator, one bf16
 * rounding per output.  M <= 16 (decode): one weight-streaming launch
 * dequantises W^ straight into tensor memory, accumulates X W^T in fp32,
 * adds s T B^T in fp32 and rounds once; T = X A^T is computed in the same
 * launch (fp32, CUDA cores) while the weights stream.  That launch is
 * cooperative (one CTA per SM, all resident at once); if the device cannot
 * co-schedule it (e.g. under a partition with fewer SMs than the device
 * reports) the call returns QLORA_ERR_CUDA.  The workspace then also holds
 * per-CTA partial tiles, partials of T and arrival counters, which the
 * call clears on the stream before use.  Results are deterministic (fixed
 * summation order) for both paths.  Requires N % 8 == 0, K % 64 == 0.
 */
qlora_status qlora_linear_fwd(const void* X, int64_t M, const qlora_nf4_weight* Wq,
                              const void* A, const void* B, int r, float alpha,
                              void* Y, float* T_save, void* workspace,
                              size_t ws_bytes, int* d_status,
                              const qlora_gemm_events* events, void* stream);

/*
 * Backward through the frozen base ("QLoRA", infra.bea.ai, "The Backward
 * Pass Through Quantization": dequantise on the fly, only the adapters get
 * gradients, the NF4 base stays frozen):
 *     G  = dY B  [M, r]
 *     dX = dY W^ + s G A  [M, K]      (skipped when dX is NULL)
 *     dA = s G^T X        [r, K]
 *     dB = s dY^T T       [N, r]
 * dY bf16 [M, N]; X bf16 [M, K]; T_saved fp32 [M, r] from the forward, or
 * NULL to recompute T = X A^T.  dA, dB in grad_dtype (fp32 or bf16),
 * overwritten.  Wq is read only.  Same shape rules as the forward.
 */
qlora_status qlora_linear_bwd(const void* dY, const void* X, int64_t M,
                              const qlora_nf4_weight* Wq, const void* A,
                              const void* B, int r, float alpha,
                              const float* T_saved, void* dX, void* dA, void* dB,
                              qlora_dtype grad_dtype, void* workspace,
                              size_t ws_bytes, int* d_status,
                              const qlora_gemm_events* events, void* stream);

/*
 * LoRA dropout ("QLoRA", infra.bea.ai, §3 "Implementation": the adapter
 * configuration sets lora_dropout = 0.05 without defining it).  Read here as
 * inverted dropout on the adapter's input only: the frozen path sees X,
 * the adapter sees X * keep, kept elements scaled by 1 / (1 - p):
 *     T  = (X * keep) A^T / (1 - p)        Y  = X W^T + s T B^T
 *     G  = dY B                            dX = dY W^ + s ((G A) * keep) / (1 - p)
 *     dA = s G^T (X * keep) / (1 - p)      dB = s dY^T T
 * One mask per call from a counter-based generator, so the forward and the
 * backward of a step regenerate the same mask from the same (p, seed):
 * element e = m*K + k of X [M, K] is kept iff the top 32 bits of word e % 4
 * of Philox-4x64-10 (Salmon et al., SC 2011) at counter (e / 4, 0, 0, 0),
 * key (seed, 0), are >= ceil(p * 2^32).  0 <= p < 1 (p = 0 keeps every
 * element: the plain layer); a p outside that range is QLORA_ERR_INVALID_ARG.
 *
 * qlora_workspace_bytes_dropout: workspace of the two dropout entries (the
 * plain one plus X * keep [M, K] bf16, the frozen-path dX in fp32 [M, K] and
 * G in fp32 [M, r]).  Host-only; 0 for an invalid shape.
 * qlora_lora_dropout_mask: the call's keep mask into keep (device, uint8
 * [M, K], 1 = kept, 0 = dropped), for callers and tests that need it.
 * qlora_linear_fwd_dropout / qlora_linear_bwd_dropout: the forward and the
 * backward above; every other argument, layout, error and determinism rule
 * is that of qlora_linear_fwd / qlora_linear_bwd.  T_save / T_saved hold
 * T as defined above (scaled by 1 / (1 - p)).  Under dropout the adapter
 * term of dX cannot be folded into the fused GEMM (the mask is per element),
 * so the GEMM writes dY W^ in fp32 and one more pass adds the masked term
 * and rounds once to bf16.
 */
size_t qlora_workspace_bytes_dropout(int64_t M, int64_t N, int64_t K, int r);
qlora_status qlora_lora_dropout_mask(int64_t M, int64_t K, double p, uint64_t seed, uint8_t* keep,
                                     void* stream);
qlora_status qlora_linear_fwd_dropout(const void* X, int64_t M, const qlora_nf4_weight* Wq,
                                      const void* A, const void* B, int r, float alpha, double p,
                                      uint64_t seed, void* Y, float* T_save, void* workspace,
                                      size_t ws_bytes, int* d_status,
                                      const qlora_gemm_events* events, void* stream);
qlora_status qlora_linear_bwd_dropout(const void* dY, const void* X, int64_t M,
                                      const qlora_nf4_weight* Wq, const void* A, const void* B,
                                      int r, float alpha, double p, uint64_t seed,
                                      const float* T_saved, void* dX, void* dA, void* dB,
                                      qlora_dtype grad_dtype, void* workspace, size_t ws_bytes,
                                      int* d_status, const qlora_gemm_events* events,
                                      void* stream);

/*
 * The same forward and backward over a dense bf16 weight W [N, K] (plain
 * LoRA on a 16-bit base), through the same fused GEMM with the weight tile
 * loaded as is instead of dequantised.  This is the baseline the pages
 * measure QLoRA against: "QLoRA" (learning-llms page, the fine-print
 * bullet on wall-clock), "QLoRA" (scalata.ai, "What it costs, and when to
 * use it": Speed) and katajob.com ("What it costs": step time) all state
 * that dequantising every layer on every step makes QLoRA steps slower
 * than plain LoRA on the same model, without a number; timing these two
 * entries against qlora_linear_fwd / qlora_linear_bwd on the same shapes
 * gives it.  W is row-major, read only, 16-byte aligned; N % 8 == 0,
 * K % 64 == 0.  Workspace: qlora_workspace_bytes(M, N, K, r).  Every other
 * argument, the results' definitions, the error behaviour and the
 * determinism are those of qlora_linear_fwd / qlora_linear_bwd with W^
 * replaced by W (every M takes the 2-SM GEMM; T = X A^T is a separate
 * launch).
 */
qlora_status qlora_lora_linear_fwd(const void* X, int64_t M, const void* W, int64_t N,
                                   int64_t K, const void* A, const void* B, int r,
                                   float alpha, void* Y, float* T_save, void* workspace,
                                   size_t ws_bytes, int* d_status,
                                   const qlora_gemm_events* events, void* stream);
qlora_status qlora_lora_linear_bwd(const void* dY, const void* X, int64_t M, const void* W,
                                   int64_t N, int64_t K, const void* A, const void* B, int r,
                                   float alpha, const float* T_saved, void* dX, void* dA,
                                   void* dB, qlora_dtype grad_dtype, void* workspace,
                                   size_t ws_bytes, int* d_status,
                                   const qlora_gemm_events* events, void* stream);

/*
 * Merge a trained adapter into the frozen base: out = NF4(W^ + s B A),
 * s = alpha / r ("QLoRA", learning-llms page, the fine-print bullet on
 * merging: adding the bf16 update into 4-bit weights forces a
 * re-quantisation; katajob.com, "What it costs": merge friction).  Each
 * merged weight is formed in fp32, every operation rounded once, in this
 * order:  acc = 0; for j = 0..r-1: acc = acc + B[n,j] * A[j,k];
 * W'[n,k] = W^[n,k] + s * acc  (W^ the bf16 dequantised weight), and
 * quantised into `out` exactly as qlora_quantize_nf4 would quantise W'
 * held in fp32.  A bf16 [r, K], B bf16 [N, r]; 1 <= r <= 256.  `out` has
 * Wq's rows and cols and its own double_quant setting.  Two forms:
 *   W_merged non-NULL (fp32 [N, K], 16-byte aligned, caller-provided):
 *     W' is written there and left holding it, then quantised by a second
 *     launch; `out` may be Wq itself (the launches are ordered on the
 *     stream).
 *   W_merged NULL: one launch forms W' in registers and quantises it (the
 *     same codes and scales bit for bit, without the fp32 round trip);
 *     `out` must not share Wq's codes (QLORA_ERR_INVALID_ARG).
 * Non-finite merged values set QLORA_DEV_NONFINITE_BIT as in the quantiser.
 */
qlora_status qlora_merge_nf4(const qlora_nf4_weight* Wq, const void* A, const void* B, int r,
                             float alpha, float* W_merged, const qlora_nf4_weight* out,
                             int* d_status, void* stream);

/*
 * One Adam step over a flat array of n adapter parameters ("QLoRA",
 * infra.bea.ai, "How QLoRA Works", precision table: bf16 adapters and
 * gradients, Adam state in fp32 at 12 bytes per adapter parameter = an fp32
 * master copy and the two moments).  The pages print no update rule; this
 * is Adam as published, with bias correction, and optional decoupled
 * weight decay (AdamW); per element, fp32, IEEE rounding, in this order:
 *   g = grad * grad_scale;  theta = master * (1 - lr * weight_decay)
 *   m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2
 *   master = theta - lr / (1 - beta1^step) * m / (sqrt(v) / sqrt(1 - beta2^step) + eps)
 *   param_bf16 = bf16_rne(master)            (skipped when NULL)
 * (the scalar factors are computed on the host in double, then rounded to
 * fp32).  master, m, v: fp32 [n], updated in place; grad: fp32 or bf16 [n]
 * (grad_dtype), read only; param_bf16: bf16 [n] or NULL.  Any device
 * memory the kernel can address works, including managed (pageable)
 * memory for optimiser state that may be paged out to the host.  All
 * pointers 16-byte aligned; step >= 1; 0 <= beta1, beta2 < 1; eps >= 0;
 * finite scalars; n == 0 is a no-op.  A non-finite scaled gradient sets
 * QLORA_DEV_NONFINITE_BIT in *d_status (if given); results are then
 * unspecified.  Deterministic.  Use one array layout for all four buffers
 * (e.g. every projection's A then B, matching its gradient buffer).
 */
qlora_status qlora_adam_step(float* master, float* m, float* v, void* param_bf16,
                             const void* grad, qlora_dtype grad_dtype, int64_t n,
                             int64_t step, float lr, float beta1, float beta2, float eps,
                             float weight_decay, float grad_scale, int* d_status,
                             void* stream);

/*
 * Test hooks for the bounded device waits (no counterpart on the pages).
 * Every pipeline wait in the kernels gives up after a bound (2 s by default),
 * sets QLORA_DEV_TIMEOUT_BIT in the call's d_status, and lets the kernel
 * release its resources and return, so that the context stays usable.
 *   qlora_debug_set_wait_limit: the bound in ns for the current device
 *     (0 restores 2 s); a synchronous copy to device memory.
 *   qlora_debug_inject_stall(on): while on, CTA 0 of every adapter-product
 *     launch of this library (the T = X A^T, G = dY B and dA/dB products)
 *     withholds the loads of its first pipeline stage, so that its wait
 *     runs out; the launch then ends early with the timeout bit set and the
 *     call's outputs unspecified.  Calls after it is switched off are
 *     unaffected (each call clears the arrival counters it uses).
 *   qlora_debug_set_pair_mtiles(n): the fused GEMM for M > 128 runs on
 *     pairs of SMs with n = 1 (256 x 256) or n = 2 (512 x 256) output tiles
 *     per pair; 0 (the default) lets each call choose from its shape, 1 or
 *     2 forces that tile for every later call of this process (so that
 *     tests reach both); other values return QLORA_ERR_INVALID_ARG.  Both
 *     form the same products; the fp32 accumulation order differs (one
 *     tile: even and odd 64-deep stages in two accumulators added at the
 *     end; two tiles: one accumulator per tile), so the last bits of a
 *     result may differ between the two.
 * None is for production use; they apply to kernels enqueued afterwards.
 */
qlora_status qlora_debug_set_wait_limit(uint64_t ns);
qlora_status qlora_debug_inject_stall(int on);
qlora_status qlora_debug_set_pair_mtiles(int n);

/*
 * Index-range checks (no counterpart on the pages).  A library built with
 * -DQLORA_DEBUG_CHECKS (libqlora_debug.so) checks its kernels' shared-
 * memory, tensor-memory, workspace and TMA-coordinate computations; a
 * failed check records the number of its site in a device word (the first
 * failure is kept) and skips the access it guards, never traps; a launch
 * whose load was skipped then ends by a timed-out wait
 * (QLORA_DEV_TIMEOUT_BIT).  The release library compiles the checks out.
 *   qlora_debug_checks_enabled: 1 in the debug build, else 0.
 *   qlora_debug_range_check(site): *site = that word (0: no failure since
 *     the last read), then clears it; synchronous.
 *   qlora_debug_range_selftest(stream): enqueues a kernel that records a
 *     failure at site 0xFFFF without touching memory (either build), so a
 *     test can check the path from a kernel to the host.
 */
int qlora_debug_checks_enabled(void);
qlora_status qlora_debug_range_check(unsigned int* site);
qlora_status qlora_debug_range_selftest(void* stream);

/*
 * Paged optimiser state ("QLoRA", learning-llms page, the paragraph on paged
 * optimizers; "QLoRA", scalata.ai, "How it works": optimiser state kept in
 * unified memory, which the driver pages out to host RAM when a memory
 * spike would otherwise end the run, and back in when the GPU touches it).
 * qlora_adam_step takes any device-addressable pointers, so paged state
 * needs no other kernel; these three calls manage it:
 *   qlora_paged_alloc: `bytes` of CUDA managed memory into *ptr (host
 *     pointer to the handle), preferred location the current device.  This
 *     and qlora_paged_free are the library's only calls that allocate or
 *     free; bytes == 0 or ptr == NULL is QLORA_ERR_INVALID_ARG.
 *   qlora_paged_free: releases what qlora_paged_alloc returned (NULL: no-op).
 *   qlora_paged_prefetch: enqueues on `stream` a migration of
 *     [ptr, ptr + bytes) to the current device (to_device != 0) or to the
 *     host (to_device == 0: paged out; the GPU's next access faults the
 *     pages back in).  Contents are unchanged.
 * The host may read and write the memory directly between GPU work (after
 * synchronising), which is how a test fills and checks optimiser state.
 */
qlora_status qlora_paged_alloc(size_t bytes, void** ptr);
qlora_status qlora_paged_free(void* ptr);
qlora_status qlora_paged_prefetch(void* ptr, size_t bytes, int to_device, void* stream);

/*
 * Forward without a caller workspace, for callers that cannot allocate
 * device memory: a plugin host that hands a kernel only its input and
 * output buffers, a process whose device memory is held by another
 * allocator's pool, or a latency-critical loop that must not hit the
 * implicit synchronisation a device allocation can cause.  There is no
 * counterpart on the pages; it computes exactly what qlora_linear_fwd
 * computes, with the same kernels.
 *
 * Scratch: one file-scope device array of QLORA_NOALLOC_SCRATCH_BYTES
 * (16 MiB) per GPU.  CUDA materialises it when the library's device code is
 * loaded on that GPU -- with lazy module loading (CUDA's default) that is
 * the first call that runs a kernel of this library there, which therefore
 * also pays the load; make a warm-up call where that latency matters -- and
 * it stays until process exit.  A problem
 * whose forward scratch (split-K partials of T, fp32 T, the two bf16 planes
 * of s*T, a padded copy of B when r % 8 != 0) does not fit is rejected with
 * QLORA_ERR_SCRATCH_LIMIT before anything is enqueued; e.g. M = 8192,
 * r = 64 fits.  Every region is fully written before it is read, except
 * the arrival counters of the split-K and decode kernels, which each call
 * clears on its stream before its kernels run.
 *
 * All calls on a device share the one array: calls whose work overlaps on
 * the GPU (different streams, or different host threads) race and give
 * wrong results; serialise them (same stream, or events).  The first call
 * on each device looks up the array's device address with that device
 * current; make that first call before any stream capture.  The address is
 * looked up again whenever the device's current context has changed (e.g.
 * after cudaDeviceReset), so a call after a reset uses the new context's
 * array; work enqueued before the reset is lost with its context.  The call itself
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library
 * routine).  Arguments as for qlora_linear_fwd, minus the workspace.
 */
#define QLORA_NOALLOC_SCRATCH_BYTES (16u << 20)
qlora_status qlora_linear_fwd_noalloc(const void* X, int64_t M, const qlora_nf4_weight* Wq,
                                      const void* A, const void* B, int r, float alpha,
                                      void* Y, float* T_save, int* d_status, void* stream);

/* Static string for a status code. */
const char* qlora_status_string(qlora_status s);

/* Library version, "major.minor.patch". */
const char* qlora_version(void);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H */
