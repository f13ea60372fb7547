/*
 * qlora.h — C ABI of libqlora.so: the frozen-base linear layer of QLoRA on
 * one B200 (sm_100a).
 *
 * The method (QLoRA pages: intvml.com "DL0087 QLoRA: 4-bit Quantized LoRA";
 * promptingindex.com "QLoRA: Finetuning 65B Models on a Single GPU";
 * systemoverflow.com "QLoRA ... at Extreme Scale"): a frozen weight W [N, K]
 * is stored as 4-bit NF4 codes in blocks of 64 with one absmax constant per
 * block; the constants are themselves quantized to 8 bits with one fp32
 * scale per 256 constants ("double quantization"). On every forward and
 * backward pass each block is dequantized to bf16 just before the matmul and
 * discarded, and the bf16 low-rank adapters A [K, r], B [r, N] (scale
 * alpha / r) are the only tensors that receive gradients.
 *
 * Conventions for every call
 *   - Pointers named *device* live in device memory of the current device;
 *     tables (nf4, t8) are HOST pointers, read during the call.
 *   - Matrices are dense, row-major, contiguous. bf16 values travel as their
 *     16-bit patterns (qlora_bf16).
 *   - The caller owns every buffer. The library allocates no device memory;
 *     scratch space is the caller's `workspace` (size from
 *     qlora_workspace_bytes).
 *   - Calls are asynchronous on `stream` (a cudaStream_t, passed as void*;
 *     NULL = legacy default stream). Arguments are checked on the host
 *     before anything is launched: a failed check returns its status and
 *     launches nothing. A launch failure returns QLORA_ERR_CUDA. The library
 *     never exits, traps or prints.
 *   - Every device-side wait is bounded; a wait that runs out sets a bit in
 *     the device error word (qlora_device_error) and the kernel returns.
 *   - Outputs are overwritten, never accumulated into.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#define QLORA_ABI_VERSION 2
#define QLORA_BLOCK 64          /* weights per absmax constant (DL0087 component 2)        */
#define QLORA_DQ_BLOCK 256      /* constants per second-level fp32 scale (DL0087 comp. 3) */
#define QLORA_NF4_LEVELS 16     /* 4-bit code -> level table                              */
#define QLORA_DQ_LEVELS 256     /* 8-bit code -> constant level table                     */
#define QLORA_MAX_RANK 256      /* largest adapter rank r accepted                        */

typedef uint16_t qlora_bf16;    /* bf16 bit pattern                                       */
typedef void *qlora_stream_t;   /* a cudaStream_t                                         */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = 1,        /* a required pointer is NULL                               */
  QLORA_ERR_SHAPE = 2,       /* a size is out of range or not a multiple it must be      */
  QLORA_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned                  */
  QLORA_ERR_RANGE = 4,       /* a scalar (r, alpha) is out of range                      */
  QLORA_ERR_CUDA = 5,        /* a CUDA runtime/driver call or a launch failed            */
  QLORA_ERR_UNSUPPORTED = 6, /* the current device is not sm_100                         */
  QLORA_ERR_WORKSPACE = 7,   /* workspace NULL or smaller than qlora_workspace_bytes     */
  QLORA_ERR_TABLE = 8        /* a code table is not finite and strictly ascending, or the
                                NF4 table has no exact 0.0f                              */
} qlora_status;

/* Human-readable name of a status (static string). */
QLORA_API const char *qlora_status_string(qlora_status s);

/* QLORA_ABI_VERSION of the built library. */
QLORA_API int qlora_abi_version(void);

/*
 * The library's default code tables (host, no device work).
 *
 * qlora_nf4_levels: the 16 ascending NF4 levels — standard-normal quantiles
 * rescaled to [-1, 1] with an exact zero, equal probability mass per level
 * on each side (promptingindex.com "4-bit NormalFloat"; DL0087 formulation
 * list). Sixteen is even, so the split is 7 negative, 0, 8 positive; the
 * outermost probability is delta = ((1 - 1/30) + (1 - 1/32)) / 2.
 * qlora_dq_levels: the 256 ascending 8-bit constant levels k/255 (the pages
 * fix only "8-bit"; an unsigned linear map is taken, the constants being
 * non-negative). Any other ascending tables may be passed to the calls.
 */
QLORA_API void qlora_nf4_levels(float out[16]);
QLORA_API void qlora_dq_levels(float out[256]);

/*
 * Alternative code tables (host, no device work) for the comparison the
 * pages make: 4-bit NormalFloat against the uniform 4-bit types it
 * outperforms (promptingindex.com "Finetuning 65B Models on a Single GPU",
 * section "4-bit NormalFloat"; intvml.com "DL0087 QLoRA", component 1).
 * Each is an ordinary input of the calls below (a table swap):
 *   qlora_int4_levels        i / 7 for i = -8..7 (absmax 4-bit integers; -8/7
 *                            lies below -1 and is never the nearest level)
 *   qlora_fp4_levels         the E2M1 values (0, 0.5, 1, 1.5, 2, 3, 4, 6 and
 *                            negatives) / 6, +0 once, plus an unused 8/6
 *   qlora_dq_signed_levels   (2k - 255) / 255: a signed linear 8-bit map
 *   qlora_dq_dynamic_levels  0, then 2^-e (1 - m/64) for (e, m) = divmod(j, 32),
 *                            j = 0..254, ascending: 8 octaves of 32 levels
 * Every value is computed in double precision and rounded once to float.
 */
QLORA_API void qlora_int4_levels(float out[16]);
QLORA_API void qlora_fp4_levels(float out[16]);
QLORA_API void qlora_dq_signed_levels(float out[256]);
QLORA_API void qlora_dq_dynamic_levels(float out[256]);

/*
 * Bytes of scratch that qlora_linear_fwd / qlora_linear_bwd need for this
 * shape (the larger of the two). Returns 0 for shapes the calls reject.
 */
QLORA_API size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Blockwise NF4 quantization (DL0087 components 1-2; sandgarden.com "QLoRA",
 * workflow step "Load and Quantize").
 *   W       device bf16 [N, K]
 *   nf4     host float[16], ascending, finite, containing 0.0f
 *   packed  device uint8 [N*K/2]: element 2j in the low nibble of byte j,
 *           element 2j+1 in the high nibble
 *   absmax  device float [N*K/64]: c_b = max |w| over the 64 consecutive
 *           row-major elements of block b
 * Code of an element: the count of fp32 midpoints (L[i]+L[i+1])*0.5f that
 * lie strictly below x = w / c_b (IEEE fp32 division); a block of zeros
 * encodes x = 0.
 * Requires N >= 1, K >= 64, K % 64 == 0, 16-byte aligned W, packed, absmax.
 */
QLORA_API qlora_status qlora_quantize_nf4(const qlora_bf16 *W, int64_t N, int64_t K, const float nf4[16],
                                uint8_t *packed, float *absmax, qlora_stream_t stream);

/*
 * Double quantization of the absmax constants (DL0087 component 3;
 * promptingindex.com "Double Quantization and Paged Optimizers").
 *   absmax  device float [nb] (non-negative)
 *   t8      host float[256], ascending, finite
 *   q       device uint8 [nb]: nearest 8-bit level of c / S_g (same
 *           midpoint rule as the NF4 code; a group of zeros encodes 0)
 *   scale2  device float [ceil(nb/256)]: S_g = max of the 256 consecutive
 *           constants of group g (the last group may be shorter; groups
 *           straddle weight rows)
 * Requires nb >= 1, 16-byte aligned pointers.
 */
QLORA_API qlora_status qlora_double_quant(const float *absmax, int64_t nb, const float t8[256],
                                uint8_t *q, float *scale2, qlora_stream_t stream);

/*
 * Quantize and double-quantize in one pass (DL0087 components (2) and (3)):
 * the same packed codes, q and scale2 as qlora_quantize_nf4 followed by
 * qlora_double_quant, bit for bit, from one kernel in which a CTA owns whole
 * second-level groups (256 blocks), so the fp32 block constants stay on
 * chip. absmax: device fp32 [N*K/64] receiving the block constants, or NULL
 * (not written). Same requirements and errors as the two calls.
 */
QLORA_API qlora_status qlora_quantize_dq(const qlora_bf16 *W, int64_t N, int64_t K, const float nf4[16],
                              const float t8[256], uint8_t *packed, uint8_t *q, float *scale2,
                              float *absmax, qlora_stream_t stream);

/*
 * Dequantization to bf16 (DL0087, opening paragraph and Figure 1):
 *   W_out[e] = bf16_rne( nf4[code_e] * c'_b ),  c'_b = t8[q_b] * scale2[b/256],
 * both products in fp32. Bit-identical to the bf16 weight the two linear
 * calls feed to their tensor-core MMAs (they never write it to memory).
 *   packed, q, scale2 as produced above; W_out device bf16 [N, K].
 */
QLORA_API qlora_status qlora_dequant(const uint8_t *packed, const uint8_t *q, const float *scale2,
                           int64_t N, int64_t K, const float nf4[16], const float t8[256],
                           qlora_bf16 *W_out, qlora_stream_t stream);

/*
 * QLoRA linear forward (DL0087 Figure 1 and formulation list):
 *   Y = X W'^T + s (X A) B,   s = alpha / r,
 * W' the dequantized weight, rebuilt tile by tile inside the GEMM mainloop.
 *   X [M, K], A [K, r], B [r, N], Y [M, N]: device bf16.
 *   XA_out: device bf16 [M, r] receiving X A (unscaled) for the backward, or
 *           NULL.
 *   workspace: device scratch of at least qlora_workspace_bytes(M, N, K, r).
 * Accumulation in fp32; (X A) is rounded to bf16 (times s) before its
 * rank-r product. Requires M >= 1, N % 64 == 0, K % 64 == 0, N, K >= 64,
 * 1 <= r <= 256, r % 8 == 0, alpha finite, 16-byte aligned pointers.
 * With M <= 16 tokens the product is memory-bound and runs as a single pass
 * over the packed weight that dequantizes in registers; W' (the bf16 weight
 * the MMAs see) is the same bit pattern on both paths.
 */
QLORA_API qlora_status qlora_linear_fwd(const uint8_t *packed, const uint8_t *q, const float *scale2,
                              const float nf4[16], const float t8[256],
                              int64_t M, int64_t N, int64_t K,
                              const qlora_bf16 *X, const qlora_bf16 *A, const qlora_bf16 *B,
                              int r, float alpha, qlora_bf16 *Y, qlora_bf16 *XA_out,
                              void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * QLoRA linear backward through the frozen base (DL0087 component 4;
 * sandgarden.com workflow "Fine-Tune the Adapters"): W' is dequantized
 * again inside the mainloop (recompute, no stored bf16 copy) and gradients
 * stop at the adapters — there is no dW.
 *   G  = dY B^T
 *   dX = dY W' + s G A^T
 *   dA = s X^T G
 *   dB = s (X A)^T dY
 *   X [M, K], dY [M, N], A [K, r], B [r, N]: device bf16.
 *   XA: device bf16 [M, r] saved by the forward, or NULL to recompute X A.
 *   dX [M, K], dA [K, r], dB [r, N]: device bf16 outputs. They must not
 *   overlap any input or each other: the dA/dB kernel runs concurrently with
 *   the tail of the dX GEMM (the call still completes, in stream order, only
 *   after every output is written).
 * Same requirements as qlora_linear_fwd.
 */
QLORA_API qlora_status qlora_linear_bwd(const uint8_t *packed, const uint8_t *q, const float *scale2,
                              const float nf4[16], const float t8[256],
                              int64_t M, int64_t N, int64_t K,
                              const qlora_bf16 *X, const qlora_bf16 *dY,
                              const qlora_bf16 *A, const qlora_bf16 *B, const qlora_bf16 *XA,
                              int r, float alpha, qlora_bf16 *dX, qlora_bf16 *dA, qlora_bf16 *dB,
                              void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * Compute type of the 16-bit tensors of a call (systemoverflow.com "QLoRA:
 * Efficient Finetuning of Quantized LLMs at Extreme Scale": the adapters and
 * the computation run in 16-bit float or bfloat16). With QLORA_F16 every
 * 16-bit operand and output is IEEE binary16 instead of bf16: the
 * dequantized weight is W'[e] = f16_rne(nf4[code_e] * c'_b) (fp32 product;
 * magnitudes beyond 65504 round to +-inf, small ones to fp16 subnormals),
 * the tensor-core MMAs take fp16 A and B, accumulation stays fp32 and every
 * output (including X A and the scaled s X A the low-rank step uses) is
 * rounded to fp16. The packed codes and constants are the same for both.
 */
typedef enum { QLORA_BF16 = 0, QLORA_F16 = 1 } qlora_dtype;

/*
 * qlora_dequant, qlora_linear_fwd and qlora_linear_bwd with the compute type
 * as an argument; the 16-bit pointers are bf16 or fp16 bit patterns as
 * `dtype` says. Same requirements, ownership and error behaviour as the bf16
 * calls above (which are these with QLORA_BF16); a dtype other than the two
 * values returns QLORA_ERR_RANGE and launches nothing.
 */
QLORA_API qlora_status qlora_dequant_dt(const uint8_t *packed, const uint8_t *q, const float *scale2,
                              int64_t N, int64_t K, const float nf4[16], const float t8[256],
                              qlora_dtype dtype, void *W_out, qlora_stream_t stream);
QLORA_API qlora_status qlora_linear_fwd_dt(const uint8_t *packed, const uint8_t *q, const float *scale2,
                              const float nf4[16], const float t8[256], qlora_dtype dtype,
                              int64_t M, int64_t N, int64_t K,
                              const void *X, const void *A, const void *B,
                              int r, float alpha, void *Y, void *XA_out,
                              void *workspace, size_t workspace_bytes, qlora_stream_t stream);
QLORA_API qlora_status qlora_linear_bwd_dt(const uint8_t *packed, const uint8_t *q, const float *scale2,
                              const float nf4[16], const float t8[256], qlora_dtype dtype,
                              int64_t M, int64_t N, int64_t K,
                              const void *X, const void *dY, const void *A, const void *B, const void *XA,
                              int r, float alpha, void *dX, void *dA, void *dB,
                              void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * The device error word of the current device: bit 0 = a bounded pipeline
 * wait ran out (the kernel returned early; its outputs are undefined).
 * Synchronizes the device. clear != 0 resets the word. Returns 0xFFFFFFFF if
 * the word cannot be read.
 */
QLORA_API uint32_t qlora_device_error(int clear);

/*
 * Self-test of the failure path (no counterpart on the pages): launches one
 * kernel whose single wait can never complete. After the bounded-wait limit
 * (about 2 s) it gives up, sets bit 0 of the device error word and returns,
 * exactly as a pipeline wait that ran out would; nothing traps or faults and
 * the device stays usable. Asynchronous on `stream`; read the result with
 * qlora_device_error.
 */
QLORA_API qlora_status qlora_selftest_bounded_wait(qlora_stream_t stream);

/*
 * Host-side allocation fault injection (no counterpart on the pages; the
 * paged optimizers exist so that a memory spike does not end the run, and
 * this lets a test make the library's own allocations fail without touching
 * the GPU). After `skip` more resource allocations succeed, the next `n`
 * fail with the driver's out-of-memory result, without calling the driver.
 * The library's resource allocations are the managed optimizer state of
 * qlora_paged_adamw_create, and the side streams and fork/join events that
 * the block executor creates on a thread's first qlora_block_fwd /
 * qlora_block_bwd on a device (in the order: fork event, then per side
 * stream the stream and its join event). The failing call returns
 * QLORA_ERR_CUDA, launches nothing, frees what it had made and leaves no
 * half-built state: the same call succeeds once the injected failures are
 * used up. n <= 0 cancels the pending failures. Thread-safe; returns the
 * number of injected failures that were still pending before this call.
 */
QLORA_API int qlora_debug_fail_allocs(int skip, int n);

/*
 * Forward without a caller workspace (the QLoRA pages have no counterpart:
 * this is an integration convenience, not part of the method).
 *
 * Same arguments and result as qlora_linear_fwd, minus the workspace. It is
 * for callers that cannot allocate device memory at all: code running as a
 * plugin inside a host framework that owns every device allocation, or a
 * latency-bound loop that must never enter the allocator. Its scratch is a
 * static device array of QLORA_NOALLOC_SCRATCH_BYTES compiled into the
 * library (each GPU that loads the library keeps it until the process
 * exits); the call itself allocates nothing.
 *   - A shape whose forward scratch (qlora_workspace_bytes' forward share)
 *     exceeds QLORA_NOALLOC_SCRATCH_BYTES returns QLORA_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - Every call on a device shares the one array and it keeps the previous
 *     call's contents (nothing in it needs to start at zero). Calls whose
 *     kernels overlap on the GPU (different streams, no ordering) race on
 *     it: order them.
 */
#define QLORA_NOALLOC_SCRATCH_BYTES (8u << 20)
QLORA_API qlora_status qlora_linear_fwd_noalloc(const uint8_t *packed, const uint8_t *q,
                                                const float *scale2, const float nf4[16],
                                                const float t8[256], int64_t M, int64_t N, int64_t K,
                                                const qlora_bf16 *X, const qlora_bf16 *A,
                                                const qlora_bf16 *B, int r, float alpha, qlora_bf16 *Y,
                                                qlora_bf16 *XA_out, qlora_stream_t stream);

/*
 * Decoder-block chaining (promptingindex.com "QLoRA: Finetuning 65B Models on
 * a Single GPU", "LoRA placement": adapters on every linear of the block;
 * systemoverflow.com "QLoRA ... at Extreme Scale": gradient checkpointing
 * trades recomputation for memory). One call runs all linears of a decoder
 * block (for LLaMA: q, k, v, o, gate, up, down), each a qlora_linear_fwd or
 * qlora_linear_bwd, spread round-robin over QLORA_BLOCK_STREAMS streams (the
 * caller's stream and library-owned ones that fork from it and join back
 * into it with events), so that one linear's low-rank (skinny) kernels and
 * GEMM tail overlap the next linear's GEMM. The call is asynchronous on
 * `stream`, ordered after earlier work on it, and everything it launches is
 * complete, in stream order, before later work on `stream`; it can be
 * captured into a CUDA graph (after one uncaptured call, which sets up the
 * library's kernels and streams).
 *
 * Recompute schedule (`save_xa`): 1 = the forward writes X A of every linear
 * to desc.XA and the backward reads it; 0 = the forward saves nothing and
 * the backward recomputes X A. The base weight is dequantized again in the
 * backward in both (it is never stored in 16-bit form).
 *
 * desc[i]: packed, q, scale2 (the quantized base), N, K, X [M, K], A [K, r],
 *   B [r, N], Y [M, N] (forward output), XA [M, r] (save_xa = 1), dY
 *   [M, N], dX [M, K], dA [K, r], dB [r, N] (backward). Pointers a pass does
 *   not use may be NULL. The linears must not share any output buffer.
 * workspace: at least qlora_block_workspace_bytes(n, desc, M, r) bytes.
 * Errors: as the per-linear calls (the first failing linear's status is
 * returned; linears before it have been launched).
 */
#define QLORA_BLOCK_STREAMS 2
typedef struct {
  const uint8_t *packed;
  const uint8_t *q;
  const float *scale2;
  int64_t N, K;
  const void *X, *A, *B;
  void *Y, *XA;
  const void *dY;
  void *dX, *dA, *dB;
} qlora_linear_desc;
QLORA_API size_t qlora_block_workspace_bytes(int n, const qlora_linear_desc *desc, int64_t M, int r);
QLORA_API qlora_status qlora_block_fwd(int n, const qlora_linear_desc *desc, const float nf4[16],
                                       const float t8[256], qlora_dtype dtype, int64_t M, int r, float alpha,
                                       int save_xa, void *workspace, size_t workspace_bytes,
                                       qlora_stream_t stream);
QLORA_API qlora_status qlora_block_bwd(int n, const qlora_linear_desc *desc, const float nf4[16],
                                       const float t8[256], qlora_dtype dtype, int64_t M, int r, float alpha,
                                       int save_xa, void *workspace, size_t workspace_bytes,
                                       qlora_stream_t stream);

/*
 * Paged AdamW for the adapters (intvml.com "DL0087 QLoRA: 4-bit Quantized
 * LoRA", component (5) "Paged Optimizers"; promptingindex.com "QLoRA:
 * Finetuning 65B Models on a Single GPU", "Double Quantization and Paged
 * Optimizers"): the optimizer state sits in CUDA unified (managed) memory,
 * so it can be paged out to host RAM when device memory runs short and
 * back when it frees up, instead of failing the step.
 *
 * State per adapter element: an fp32 master copy of the 16-bit parameter and
 * the two fp32 moments m, v (12 bytes), in one managed allocation that the
 * handle owns. The update is AdamW with decoupled weight decay (Loshchilov
 * and Hutter, ICLR 2019, Algorithm 2) in fp32:
 *   p <- p (1 - lr wd); m <- b1 m + (1 - b1) g; v <- b2 v + (1 - b2) g^2;
 *   p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)
 * and the 16-bit parameter is then p rounded to nearest even.
 *
 * Placement: before each step the library reads the device's free memory
 * (cudaMemGetInfo) and calls qlora_paged_adamw_placement. Paging out sets
 * the preferred location to the host, lets the device map the pages, and
 * prefetches them to the host; the step then reads and writes the state
 * across the host link. Paging in sets the preferred location to the
 * device and prefetches the pages back. Where the device does not support
 * concurrent managed access the hints are skipped and the driver migrates
 * on demand.
 *
 * create:  nseg tensors (1 <= nseg), counts[s] >= 1 elements each (host
 *          array); *out receives the handle. QLORA_ERR_CUDA if the managed
 *          allocation fails.
 * init:    params[s]: device 16-bit tensors (host array of nseg pointers);
 *          master <- params, m = v = 0. Asynchronous on `stream`.
 * step:    grads[s]: device 16-bit gradients, same shapes; t >= 1 the step
 *          number; lr >= 0, 0 <= beta1, beta2 < 1, eps > 0, wd >= 0, all
 *          finite (else QLORA_ERR_RANGE). Writes params[s] and the state.
 *          Asynchronous on `stream`; the state must not be read by the host
 *          until the stream is synchronized.
 * set_reserve: device bytes the placement keeps free for other work
 *          (default 0).
 * placement: pure policy, exported for tests: 1 (host) or 0 (device) for a
 *          state of state_bytes given free device bytes and the reserve;
 *          `current` is the present location (0 or 1). On the device it
 *          stays until free < reserve; on the host it comes back once
 *          free >= state_bytes + reserve.
 * location: 0 or 1, where the last step placed the state.
 * state:   the managed pointers of the master copy and the moments (fp32,
 *          concatenated over the segments in order); host-readable once the
 *          stream is synchronized. Owned by the handle.
 * destroy: frees the state (synchronizes the device first); NULL is a no-op.
 */
typedef struct qlora_paged_adamw qlora_paged_adamw;
QLORA_API qlora_status qlora_paged_adamw_create(int nseg, const int64_t *counts, qlora_paged_adamw **out);
QLORA_API void qlora_paged_adamw_destroy(qlora_paged_adamw *opt);
QLORA_API qlora_status qlora_paged_adamw_init(qlora_paged_adamw *opt, void *const *params, qlora_dtype dtype,
                                              qlora_stream_t stream);
QLORA_API qlora_status qlora_paged_adamw_step(qlora_paged_adamw *opt, void *const *params,
                                              const void *const *grads, qlora_dtype dtype, int64_t t, float lr,
                                              float beta1, float beta2, float eps, float weight_decay,
                                              qlora_stream_t stream);
QLORA_API qlora_status qlora_paged_adamw_set_reserve(qlora_paged_adamw *opt, size_t reserve_bytes);
QLORA_API int qlora_paged_adamw_placement(size_t free_bytes, size_t state_bytes, size_t reserve_bytes,
                                          int current);
QLORA_API int qlora_paged_adamw_location(const qlora_paged_adamw *opt);
QLORA_API size_t qlora_paged_adamw_state_bytes(const qlora_paged_adamw *opt);
QLORA_API qlora_status qlora_paged_adamw_state(const qlora_paged_adamw *opt, float **master, float **m,
                                               float **v);

/*
 * Measurement instrumentation (no counterpart on the pages).
 *
 * qlora_set_trace_events: when both are non-NULL, the next qlora_linear_fwd
 * and qlora_linear_bwd calls on this host thread record `start` (a
 * cudaEvent_t) on their stream just before their fused dequant-GEMM kernel
 * (for M <= 16 tokens: the register-dequant weight stream) and `stop` just
 * after it, so a caller can time that kernel alone with
 * cudaEventElapsedTime. Pass NULL, NULL to stop. The events stay owned by the
 * caller.
 * qlora_launch_count: the number of kernels this library has launched in
 * this process (all devices, all threads).
 */
QLORA_API void qlora_set_trace_events(void *start, void *stop);
QLORA_API uint64_t qlora_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H_ */
