/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: the QLoRA frozen-NF4 linear layer
 * on NVIDIA B200 (sm_100a).
 *
 * The layer (page citations give the page title and section):
 *   - The frozen base weight W [N, K] (PyTorch Linear layout, out x in) is
 *     stored as 4-bit NormalFloat: 16 levels at N(0,1) quantiles normalised
 *     to [-1, 1] ("QLoRA Guide", NF4 vs uniform INT4; "Qlora Expert", Core
 *     Concept), one absmax constant per block of 64 consecutive weights
 *     ("QLoRA Implementation Details (2025 Edition)", Step 1, NF4 Math), and
 *     the block constants themselves quantized to 8 bit ("QLoRA: The 4-bit
 *     Revolution", 2. Double Quantization), here as int8 codes with an fp32
 *     scale and mean per group of 256 block constants.
 *   - Every forward and backward dequantizes to bf16 on the fly inside the
 *     matrix product; the bf16 copy is never stored ("QLORA: Efficient
 *     Finetuning of Quantized LLMs", Notes).
 *   - A bf16 LoRA branch is added: Y = X W'^T + s (X A^T) B^T with
 *     s = alpha / r ("QLoRA Guide", Forward pass; "QLoRA Implementation
 *     Details (2025 Edition)", Step 4).  Only A and B receive gradients
 *     ("QLoRA Guide", Forward pass: the dequantized W is a constant for
 *     autograd), so the backward returns dX, dA and dB and never dW.
 *
 * Conventions for every entry point:
 *   - bf16 values are passed as raw 16-bit patterns (qlora_bf16).
 *   - Every tensor is dense row-major.  Pointers marked "device" must be
 *     device (or managed) memory of the current CUDA device; the caller owns
 *     all memory, the library never allocates or frees and holds no state
 *     except a per-process copy of the codebook it computes on first use.
 *   - Work is enqueued on `stream` (NULL = the legacy default stream) and
 *     the call returns without synchronizing.  Results are valid once the
 *     stream reaches that point.  Inputs may be written by work enqueued
 *     just before the call on the same stream: kernels launched with
 *     programmatic dependent launch, which may start while the kernel ahead
 *     of them is still running, read none of the caller's memory before that
 *     kernel has completed (before it they only prefetch into L2, which is
 *     coherent).
 *   - The return value is QLORA_OK (0) or a negative QLORA_ERR_* code.  All
 *     argument checks run before anything is launched; a rejected call
 *     launches nothing and writes nothing.  No C++ exception crosses the ABI.
 *   - Weights and activations must be finite.
 *   - Device-side waits are bounded: a kernel that gives up sets a sticky
 *     status word read by qlora_device_status() instead of hanging.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qlora_bf16;            /* raw bf16 bit pattern */
typedef struct CUstream_st* qlora_stream_t;   /* a cudaStream_t */

#define QLORA_NF4_BLOCK 64              /* weights per absmax block */
#define QLORA_DQ_GROUP 256              /* block constants per double-quant group */
#define QLORA_MAX_RANK 256              /* largest LoRA rank accepted */
#define QLORA_MAX_K (1 << 21)           /* largest K (input features) of the linear layer: keeps every
                                           launch's grid within CUDA's limits */

enum {
    QLORA_OK = 0,
    QLORA_ERR_NULL = -1,        /* a required pointer is NULL */
    QLORA_ERR_SHAPE = -2,       /* M, N or K <= 0, K % 64 != 0, K > QLORA_MAX_K (linear layer), or a
                                   size overflows */
    QLORA_ERR_RANK = -3,        /* r outside [1, QLORA_MAX_RANK] */
    QLORA_ERR_ALIGN = -4,       /* a pointer is not 16-byte aligned */
    QLORA_ERR_WORKSPACE = -5,   /* workspace NULL or smaller than qlora_workspace_bytes() */
    QLORA_ERR_DEVICE = -6,      /* current device is not compute capability 10.0 */
    QLORA_ERR_LAUNCH = -7,      /* a CUDA launch or runtime call failed */
    QLORA_ERR_TIMEOUT = -8,     /* a device-side bounded wait gave up (see qlora_device_status) */
    QLORA_ERR_VALUE = -9,       /* a scalar argument is not finite, or an unknown quant_type */
    QLORA_ERR_SCRATCH = -10     /* needs more than QLORA_NOALLOC_SCRATCH_BYTES (no-alloc entry point) */
};

/* 4-bit quant types ("Qlora Expert", Hyperparameter Guidance: the 4-bit
 * quant type is "nf4" or "fp4"; "QLoRA Guide", FAQs: NF4 vs FP4). */
#define QLORA_QUANT_NF4 0   /* NormalFloat: 16 levels at N(0,1) quantiles (nf4_codebook) */
#define QLORA_QUANT_FP4 1   /* E2M1 4-bit float over its largest magnitude (quant4_codebook) */

/* Quantized weight: all device pointers, caller-owned.
 *   packed [N, K/2] uint8: byte j of row n holds element 2j in its high
 *                          nibble and element 2j+1 in its low nibble; a
 *                          nibble indexes the quant type's 16-entry table L
 *                          (nf4_codebook / quant4_codebook).
 *   codes  [N*K/64] int8 : code of block b = flat weights [64b, 64b+64)
 *   scale  [G] fp32, mean [G] fp32, G = ceil(N*K/64 / 256): group g covers
 *                          blocks [256g, 256g+256) of the flattened weight.
 *   The constant of block b is c'_b = fmaf((float)codes[b], scale[b/256],
 *   mean[b/256]) and the dequantized weight is bf16_rne(L[nibble] * c'_b).
 *   packed must be 16-byte aligned; codes, scale and mean 4-byte aligned (the
 *   fused kernels copy the codes as whole 32-bit words: N % 8 == 0 makes the
 *   code count a multiple of 8). */
typedef struct {
    const uint8_t* packed;
    const int8_t* codes;
    const float* scale;
    const float* mean;
    int64_t N;
    int64_t K;
    int32_t quant_type;     /* QLORA_QUANT_NF4 or QLORA_QUANT_FP4: which 16-entry table L the nibbles
                               index; any other value is rejected with QLORA_ERR_VALUE */
} nf4dq_weight;

/* The 16 NF4 levels in fp32, ascending (out16[0] = -1, out16[7] = 0,
 * out16[15] = +1): 8 positive normal quantiles at the first 8 of 9 evenly
 * spaced probabilities from delta = ((1-1/32)+(1-1/30))/2 down to 1/2, 7
 * negative ones at the first 7 of 8, and an exact zero, divided by the
 * largest (the pages give only "levels at N(0,1) quantiles"; this is the
 * construction of the QLoRA paper they cite).  Host memory; no GPU needed. */
QLORA_API int nf4_codebook(float out16[16]);

/* The 16 levels of a quant type in fp32, indexed by nibble.  NF4: as
 * nf4_codebook.  FP4 (a reading: the pages name the type but give no
 * values): the E2M1 value of the nibble's bit pattern (bit 3 sign, bits 2..1
 * exponent with bias 1, bit 0 mantissa; exponent 0 is subnormal: 0 or 0.5),
 * divided by the largest magnitude 6 in double and rounded once to fp32:
 * +-{0, 1/12, 1/6, 1/4, 1/3, 1/2, 2/3, 1}; nibbles 0 and 8 are +0 and -0.
 * Host memory; returns QLORA_ERR_VALUE for another quant_type. */
QLORA_API int quant4_codebook(int quant_type, float out16[16]);

/* Element counts of a quantized [N, K] weight (host only, no GPU needed).
 * Any output pointer may be NULL. */
QLORA_API int nf4dq_sizes(int64_t N, int64_t K, int64_t* packed_bytes, int64_t* n_blocks, int64_t* n_groups);

/* Quantize a bf16 weight W [N, K] (device) to NF4 with double-quantized
 * constants ("Qlora Expert", Core Concept 1-2; "QLoRA Implementation
 * Details (2025 Edition)", Step 1).  Per block: c_b = max |w|; each weight
 * goes to the level nearest w / c_b (IEEE fp32 division; exactly halfway
 * goes to the lower level; c_b = 0 gives the zero level 7).  Per group:
 * mean_g = fl32(S / n_g) with S the fp64 pairwise sum (stride 128..1) of
 * the group's constants, scale_g = fl32(max |c_b - mean_g| / 127),
 * code_b = clamp(rint((c_b - mean_g) / scale_g), -127, 127) (0 when
 * scale_g = 0).  Outputs (device, caller-allocated, sizes from
 * nf4dq_sizes): packed, codes, scale, mean.  W and packed must be 16-byte
 * aligned.  Requires K % 64 == 0. */
QLORA_API int nf4_quantize_dq(const qlora_bf16* W, int64_t N, int64_t K, uint8_t* packed, int8_t* codes,
                    float* scale, float* mean, qlora_stream_t stream);

/* nf4_quantize_dq for either quant type.  The encoder is the same nearest-
 * level rule over that type's distinct levels in ascending order (thresholds
 * halfway between neighbours, in fp32; exactly on a threshold goes to the
 * lower level); the nibble written is the level's index in the table of
 * quant4_codebook.  For FP4 a zero (and every weight of an all-zero block)
 * is written as +0 (nibble 0).  quant_type other than NF4 / FP4:
 * QLORA_ERR_VALUE. */
QLORA_API int quant4_quantize_dq(const qlora_bf16* W, int64_t N, int64_t K, int quant_type, uint8_t* packed,
                                 int8_t* codes, float* scale, float* mean, qlora_stream_t stream);

/* Dequantize to a dense bf16 W' [N, K] (device, 16-byte aligned)
 * ("QLORA: Efficient Finetuning of Quantized LLMs", Notes: dequantize to
 * BF16).  Bit-exact with the definition under nf4dq_weight. */
QLORA_API int nf4_dequant(const nf4dq_weight* w, qlora_bf16* W_out, qlora_stream_t stream);

/* Dequantize-and-merge ("Qlora Expert", When to Use and Common Pitfalls: a
 * dense model is obtained by dequantize-and-merge, since merging into the
 * 4-bit weight is impossible -- merging requires dequantization; "QLoRA
 * Implementation Details (2025 Edition)", Step 7: merge for inference).
 * The dense bf16 weight of the adapted layer:
 *   W_out[n, k] = bf16_rne( fmaf(scaling, d[n, k], w'[n, k]) )
 *   d[n, k]     = sum over j = 0 .. r-1 of B[n, j] * A[j, k], accumulated in
 *                 fp32 as d = fmaf(B[n, j], A[j, k], d) from d = 0 in
 *                 increasing j (a fixed order, so the result is reproducible
 *                 bit for bit)
 *   w'[n, k]    = the dequantized weight bf16_rne(L[q] * c'_b) of nf4_dequant.
 * A [r, K] bf16 (16-byte aligned), B [N, r] bf16, W_out [N, K] bf16
 * (16-byte aligned), all device.  1 <= r <= QLORA_MAX_RANK; any N >= 1;
 * K % 64 == 0, K <= QLORA_MAX_K.  With B = 0 the result equals nf4_dequant's
 * in value.  Non-finite scaling: QLORA_ERR_VALUE. */
QLORA_API int nf4_dequant_merge(const nf4dq_weight* w, const qlora_bf16* A, const qlora_bf16* B, int r,
                                float scaling, qlora_bf16* W_out, qlora_stream_t stream);

/* One AdamW step of LoRA adapter parameters with 8-bit moment states
 * ("Qlora Expert", Hyperparameter Guidance: paged_adamw_8bit, 8-bit Adam to
 * cut optimizer memory; "QLoRA Implementation Details (2025 Edition)", Step
 * 5: Paged Optimizer).  The paging itself (unified memory) is left to the
 * caller's allocator; this is the step.  The pages give no state encoding;
 * this library's reading:
 *   - states m and v are stored per block of QLORA_ADAM_BLOCK consecutive
 *     parameters as one fp32 scale and one FP8 E4M3 code per parameter
 *     (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, largest 448):
 *     value = fl32(e4m3(code) * scale), scale = fl32(absmax / 448),
 *     code = e4m3 round-to-nearest-even of fl32(value * fl32(448 / absmax)),
 *     saturating at 448; code 0 when absmax = 0.  All-zero codes and scales
 *     are the initial (zero) state.
 *   - the update, every operation one IEEE fp32 rounding in this order:
 *       m = b1*m + omb1*g;  v = b2*v + omb2*(g*g);  mh = m*rbc1;  vh = v*rbc2;
 *       u = mh/(sqrt(vh) + eps) + weight_decay*p;  p = bf16_rne(p - lr*u)
 *     with omb = fl32(1 - b), rbc = fl32(1 / (1 - b^step)) computed in double
 *     on the host; then each block's m and v are requantized with its new
 *     absmax.
 * p [n] bf16 (in/out, 16-byte aligned), g [n] bf16 gradient (16-byte
 * aligned), m_code, v_code [n] (in/out, 8-byte aligned), m_scale, v_scale
 * [ceil(n / QLORA_ADAM_BLOCK)] fp32 (in/out), all device.  step >= 1 is the
 * 1-based step count.  Errors: non-finite lr/eps/weight_decay or a beta
 * outside [0, 1) -> QLORA_ERR_VALUE; n <= 0 -> QLORA_ERR_SHAPE. */
#define QLORA_ADAM_BLOCK 256
QLORA_API int adamw_8bit_step(qlora_bf16* p, const qlora_bf16* g, int64_t n, uint8_t* m_code, float* m_scale,
                              uint8_t* v_code, float* v_scale, int64_t step, float lr, float beta1, float beta2,
                              float eps, float weight_decay, qlora_stream_t stream);

/* Bytes of device workspace that qlora_linear_fwd / qlora_linear_bwd need
 * for these sizes (0 is never returned for valid sizes; returns 0 for
 * invalid ones).  The same workspace may be reused by calls that run one
 * after another on one stream; calls that overlap on the GPU need separate
 * workspaces. */
QLORA_API size_t qlora_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/* Forward ("QLoRA Guide", Forward pass / Dequant + LoRA path):
 *   T = X A^T            [M, r]  (fp32 accumulation)
 *   Y = X W'^T + s T B^T [M, N]  (fp32 accumulation, one bf16 rounding)
 * X [M, K] bf16, A [r, K] bf16, B [N, r] bf16, Y [M, N] bf16 (all device).
 * T_out [M, r] bf16 may be NULL; when given it receives bf16(T) for reuse
 * by the backward.  s = scaling (alpha / r).  ws: device workspace of at
 * least qlora_workspace_bytes(M, N, K, r) bytes, 256-byte aligned.
 * X, Y must be 16-byte aligned.  Requires K % 64 == 0, K <= QLORA_MAX_K and
 * N % 8 == 0. */
QLORA_API int qlora_linear_fwd(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                     const qlora_bf16* B, int r, float scaling, qlora_bf16* Y, qlora_bf16* T_out,
                     void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Backward of <Y, dY> ("QLoRA Guide", Forward pass: only A and B receive
 * gradients; "QLORA: Efficient Finetuning of Quantized LLMs", Notes):
 *   U  = dY B                    [M, r]
 *   dX = dY W' + s U A           [M, K]
 *   dA = s U^T X                 [r, K]
 *   dB = s dY^T T, T = X A^T     [N, r]
 * No gradient is computed for the frozen base weight.  T may be NULL (it is
 * then recomputed from X and A) or the bf16 T_out of the forward.
 * dX, dA, dB: device bf16 outputs (fp32 accumulation).  Same alignment and
 * workspace rules as qlora_linear_fwd. */
QLORA_API int qlora_linear_bwd(const qlora_bf16* X, const qlora_bf16* dY, int64_t M, const nf4dq_weight* w,
                     const qlora_bf16* A, const qlora_bf16* B, int r, float scaling, const qlora_bf16* T,
                     qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB, void* ws, size_t ws_bytes,
                     qlora_stream_t stream);

/* LoRA dropout ("Qlora Expert", Implementation Pattern: lora_dropout=0.05;
 * "QLoRA Implementation Details (2025 Edition)", Step 4: lora_dropout=0.1).
 * The pages give only the rate; this library's reading: dropout on the LoRA
 * branch's input, the base path unchanged,
 *   Y  = X W'^T + s (Xd A^T) B^T,  T = Xd A^T,  Xd = X * keep * c,
 *   c  = fl32(1 / (1 - p)),
 * and its backward under the same mask:
 *   U = dY B,  dX = dY W' + s (U A) * keep * c,  dA = s U^T Xd,  dB = s dY^T T.
 * The kernels keep X * keep (exact in bf16) and apply c in fp32 to the
 * accumulated T and dA and to the LoRA term of dX.
 * Element e = m K + k of X is kept iff field >= llrint(p * 2^16), field
 * being 16-bit field (e mod 16) (field 4i + j = bits 16j..16j+15 of output
 * i) of the Philox4x64-10 output (Salmon et al., SC 2011) for counter
 * (e div 16, offset, 0, 0) and key (seed, 0).  The forward and the backward
 * of one step must be given the same (dropout_p, seed, offset); T given to
 * the backward is the T_out of that forward.
 * Arguments, layouts and errors are those of qlora_linear_fwd / _bwd, plus:
 * 0 <= dropout_p < 1 (else QLORA_ERR_VALUE; 0 drops nothing), and the
 * workspace must hold qlora_dropout_workspace_bytes(M, N, K, r) bytes (the
 * regular workspace plus the dropped copy of X and its keep bitmask). */
QLORA_API size_t qlora_dropout_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
QLORA_API int qlora_linear_fwd_dropout(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                                       const qlora_bf16* B, int r, float scaling, float dropout_p, uint64_t seed,
                                       uint64_t offset, qlora_bf16* Y, qlora_bf16* T_out, void* ws, size_t ws_bytes,
                                       qlora_stream_t stream);
QLORA_API int qlora_linear_bwd_dropout(const qlora_bf16* X, const qlora_bf16* dY, int64_t M, const nf4dq_weight* w,
                                       const qlora_bf16* A, const qlora_bf16* B, int r, float scaling,
                                       float dropout_p, uint64_t seed, uint64_t offset, const qlora_bf16* T,
                                       qlora_bf16* dX, qlora_bf16* dA, qlora_bf16* dB, void* ws, size_t ws_bytes,
                                       qlora_stream_t stream);

/* Human-readable text for a status code (static storage). */
QLORA_API const char* qlora_status_string(int status);

/* Sticky device status of the current device: QLORA_OK, or QLORA_ERR_TIMEOUT
 * if a kernel's bounded wait gave up since the last reset.  Synchronizes the
 * current device.  reset != 0 clears it afterwards. */
QLORA_API int qlora_device_status(int reset);

/* Which kernel family the last successful fwd/bwd call on this thread
 * dispatched to (for tests and benchmarks): 1 = small-M tensor-core GEMV
 * kernels (M <= 32), 2 = tcgen05 fused dequant-GEMM on one SM per tile
 * (32 < M <= 128), 3 = the same on SM pairs (cta_group::2, M > 128). */
QLORA_API int qlora_last_path(void);

/* Schedule of the SM-pair kernel (no counterpart on the pages; for tests; no
 * device work).  qlora_pair_schedule: for M tokens, an n_out-wide output
 * (N forward, K backward), `pairs` SM pairs and the direction (bwd != 0),
 * writes the token tiles of 256 per weight stage (*mt), the tile count
 * (*ntiles) and 1 to *stream_k when the (tile, reduction step) units are dealt
 * to the pairs stream-K, else 0.  qlora_pair_spans: the spans that pair `pair`
 * of `npairs` takes of ntiles x nsteps units under stream-K, in the order it
 * takes them: out[3 i] = tile, out[3 i + 1] = first step, out[3 i + 2] = end
 * step (exclusive); writes at most max_spans and returns the span count.
 * Both return QLORA_ERR_VALUE (or QLORA_ERR_NULL) on a bad argument. */
QLORA_API int qlora_pair_schedule(int64_t M, int64_t n_out, int pairs, int bwd, int* mt, int64_t* ntiles,
                                  int* stream_k);
QLORA_API int qlora_pair_spans(int64_t ntiles, int nsteps, int pair, int npairs, int64_t* out, int max_spans);

/* Measurement hooks (no counterpart on the pages; used by benchmarks).
 * qlora_launch_count: number of kernels this library has launched in this
 * process so far (all threads).  qlora_set_kernel_events: the next
 * qlora_linear_fwd / qlora_linear_bwd call on this thread records `before`
 * (a cudaEvent_t) on its stream right before its fused dequant-GEMM kernel
 * and `after` right after it, then forgets both; pass NULL, NULL to clear.
 * For M <= 32 the pair brackets the fused kernel together with the small
 * kernels chained to it (forward: GEMV, T, finish; backward: U / dB, then
 * dY W').  An event between two kernels ends the programmatic-launch overlap
 * between them, so a timed call runs a little slower than an untimed one. */
QLORA_API long long qlora_launch_count(void);
QLORA_API int qlora_set_kernel_events(void* before, void* after);

/* qlora_linear_fwd_noalloc -- the paper has no counterpart; this is a
 * convenience of this library.
 *
 * The same forward as qlora_linear_fwd, for callers that cannot allocate
 * device memory: code running where another allocator owns all of the
 * device's memory (a serving engine that reserved its pool at start-up),
 * or code called back from inside a framework that forbids allocating on
 * its hot path.  Instead of a caller-provided workspace it uses one scratch
 * array of QLORA_NOALLOC_SCRATCH_BYTES that the library defines statically
 * in device memory; every GPU that loads the library holds that array until
 * the process exits.  Nothing is allocated or freed by this call.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Calls whose workspace need (qlora_workspace_bytes) exceeds
 *     QLORA_NOALLOC_SCRATCH_BYTES return QLORA_ERR_SCRATCH and launch
 *     nothing.  Decode-sized calls fit: M <= 16 with 70B-model projections
 *     (up to 28672 x 8192, r <= 64), M <= 32 up to 11008 x 4096; M = 32 with
 *     a 28672-row weight needs ~12 MiB and is rejected.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race on it and must be serialized by the
 *     caller.  Nothing in the scratch needs to be zeroed between calls.
 * Arguments, layouts and the other errors are those of qlora_linear_fwd. */
#define QLORA_NOALLOC_SCRATCH_BYTES (8u << 20)
QLORA_API int qlora_linear_fwd_noalloc(const qlora_bf16* X, int64_t M, const nf4dq_weight* w, const qlora_bf16* A,
                                       const qlora_bf16* B, int r, float scaling, qlora_bf16* Y, qlora_bf16* T_out,
                                       qlora_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
