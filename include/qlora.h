/* qlora.h -- C ABI of the B200 (sm_100a) library for the forward and backward pass of an
 * unmerged-LoRA linear layer whose frozen base weight stays in 4-bit storage.
 *
 * The layer ("Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §2 "The math":
 * y = W x + (alpha/r) B A x, the scaling "part of the layer" wherever BA appears; §3 "The setup":
 * the 4-bit base is dequantised to bf16 on the fly, the matmul computed and the dequantised tensor
 * discarded), written for a batch of M rows with s = alpha/r (or alpha/sqrt(r)):
 *
 *   T  = X A^T                    Y  = X deq(W)^T + s T B^T
 *   U  = dY B                     dX = dY deq(W) + s U A
 *   dA = s U^T X                  dB = s dY^T T
 *
 * dA and dB follow "Training LLMs on a Budget", §2 "Initialization matters" (dL/dA = B^T dL/dy x^T,
 * dL/dB = dL/dy x^T A^T); there is no dW: the base is frozen ("Quantized weights, full precision:
 * The math behind 75% cheaper fine-tuning", "Backward pass and optimizer step in training").
 * deq(W) is computed inside the GEMM kernels; no bf16 copy of W is ever written to device memory.
 *
 * Shapes and layouts (row-major, last index contiguous):
 *   X [M,K], Y [M,N], dY [M,N], dX [M,K], A [r,K], B [N,r], T/U [M,r], dA [r,K], dB [N,r]: bf16
 *   (PyTorch's nn.Linear convention: W is [N = out, K = in]).
 *
 * Conventions shared by every entry point:
 *   - Pointers are device pointers unless stated otherwise; the caller owns every buffer.  The
 *     library never allocates, frees or synchronises on the compute path; all work is enqueued
 *     on `stream`.
 *   - Arguments are validated before anything is enqueued; a failed check returns
 *     QLORA_ERR_INVALID_ARG / QLORA_ERR_UNSUPPORTED / QLORA_ERR_WORKSPACE and enqueues nothing.
 *     A failed launch returns QLORA_ERR_CUDA.  Device-side pipeline waits are bounded: if one ever
 *     gives up, the kernel records QLORA_ERR_DEVICE_TIMEOUT in the workspace and ends, and
 *     qlora_get_device_status() reports it.
 *   - Shape limits: K % 64 == 0, N % 16 == 0, K >= 64, N >= 16, M >= 0 (M == 0 is a no-op that
 *     still overwrites dA and dB with zeros), r in {8, 16, 32, 64}; every pointer 16-byte aligned
 *     (with M == 0 the [M, ...] activation pointers may be NULL).  Grouped ops: 1 <= E <= 1024.
 *   - Outputs are overwritten, never accumulated (gradient accumulation across micro-batches is the
 *     caller's job).  Results are deterministic: the same inputs (and workspace size) give
 *     bitwise-identical outputs.
 *   - Calls that share a workspace must be ordered on one stream.
 *   - Host threads may call the library concurrently.  Its process-wide state is small: per-device
 *     caches filled once (SM count, kernel shared-memory attributes, set on a kernel's first launch
 *     on a device and not again: a cudaDeviceReset discards them, so do not reset a device that
 *     the library has run on and use it again in the same process), a pool of events and a side
 *     stream per device used to order the backward pass's dA/dB launch (mutex-guarded), the launch
 *     counter (atomic) and the opt-in profiling record (qlora_profile_*, mutex-guarded); the
 *     fixed scratch of qlora_linear_fwd_noalloc is shared by all its callers (see there).
 */
#ifndef QLORA_H_
#define QLORA_H_

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

typedef struct CUstream_st* qlora_stream_t; /* a cudaStream_t; NULL = the legacy default stream */

typedef enum {
  /* NF4: 16 normal-quantile levels times one fp32 absmax per 64 weights along K
   * ("Training LLMs on a Budget", §3 "The three QLoRA tricks", items 1 and 2). */
  QLORA_FMT_NF4 = 0,
  /* MXFP4: E2M1 elements times one E8M0 scale 2^(e-127) per 32 along K
   * ("Fine-Tuning 4-Bit Models: Adapting a Base That Only Ships Quantized", "Case 2: An NVFP4
   * deployment checkpoint is what you were handed"). */
  QLORA_FMT_MXFP4 = 1,
  /* NVFP4: E2M1 elements times one E4M3 scale per 16 along K, times one fp32 tensor scale
   * (same page and section: "a per-block FP8 scale over 16-element micro-blocks"). */
  QLORA_FMT_NVFP4 = 2,
  /* NF4 with double quantisation: as NF4, the absmax of each 64-block stored as an 8-bit E4M3
   * code times an fp32 second-level scale shared by 256 consecutive first-level codes
   * ("Training LLMs on a Budget", §3 "The three QLoRA tricks", item 2).  4.127 bits/weight. */
  QLORA_FMT_NF4_DQ = 3
} qlora_format_t;

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,    /* a NULL/misaligned pointer or a shape outside the limits */
  QLORA_ERR_UNSUPPORTED = 2,    /* a valid request this build does not implement (e.g. rank) */
  QLORA_ERR_WORKSPACE = 3,      /* workspace NULL, misaligned or too small (qlora_workspace_size) */
  QLORA_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed (launch, tensor map) */
  QLORA_ERR_DEVICE_TIMEOUT = 5  /* a bounded device-side wait gave up (kernel ended early) */
} qlora_status_t;

/* One frozen 4-bit weight W [N,K] (row n = output feature, K contiguous).
 *   codes  [N, K/2] uint8: element 2j of a row in the low nibble of byte j, 2j+1 in the high.
 *   scales NF4: float [N, K/64]; MXFP4: uint8 E8M0 [N, K/32]; NVFP4: uint8 E4M3 [N, K/16];
 *          NF4_DQ: uint8 E4M3 first-level codes [N, K/64].
 *          Block b of row n covers k in [b*bs, (b+1)*bs).
 *   tensor_scale NVFP4: device float* holding the decode multiplier (grouped: [E] values);
 *          NULL for the other formats.  It must be finite and non-zero.
 *   scales2 NF4_DQ: device float [G] second-level scales, G = ceil(N * (K/64) / 256); scale g
 *          serves first-level codes [256 g, 256 g + 256) of the row-major [N, K/64] array
 *          (grouped: [E, G], per expert).  NULL for the other formats.
 * Decode of element (n,k) with code c: NF4 bf16(fp32(level[c] * absmax)); NF4_DQ the same with
 * absmax = fp32(e4m3(c1) * scales2[g]); MXFP4 bf16(e2m1(c) * 2^(e-127)); NVFP4
 * bf16(fp32(fp32(e2m1(c) * e4m3(s)) * tensor_scale)), every
 * multiply binary32 round-to-nearest-even without flush-to-zero.  The kernels apply the NVFP4
 * tensor scale to the fp32 accumulator rather than to each element (it is uniform over W); the
 * per-element micro-block decode is exact.
 * For the grouped entry points codes/scales are stacked [E, N, ...]. */
typedef struct {
  int32_t fmt; /* qlora_format_t */
  int32_t reserved;
  int64_t N, K;
  const uint8_t* codes;
  const void* scales;
  const float* tensor_scale;
  const float* scales2;
} qlora_weight_t;

typedef enum {
  QLORA_OP_FWD = 0,
  QLORA_OP_BWD = 1,
  QLORA_OP_GROUPED_FWD = 2,
  QLORA_OP_GROUPED_BWD = 3,
  QLORA_OP_FWD_W4A8 = 4       /* qlora_linear_fwd_w4a8 */
} qlora_op_t;

/* Bytes of device workspace `op` needs for these shapes (E = number of experts for the grouped
 * ops, ignored otherwise; for the grouped ops M is the total row count).  Returns 0 for invalid
 * arguments.  A workspace sized for an op and shapes also serves smaller M.  For one layer of at
 * most 256 rows the size includes the fp32 split partials of the short-batch kernels (tens of MB
 * for a 14336 x 4096 weight); a call whose workspace lacks room for them (e.g. one sized for
 * more than 256 rows, which need none) runs the tiled kernels instead: the same results up to
 * the order of fp32 additions.  The training calls reject only a workspace smaller than the
 * part without those partials (QLORA_ERR_WORKSPACE). */
QLORA_API size_t qlora_workspace_size(int op, const qlora_weight_t* W, int64_t M, int r, int E);

/* Zero the workspace's 8192-byte header (device status word, the tiled kernel's tile ticket and
 * the arrival counters of the split reductions, which every launch leaves at zero).  Call once
 * after allocating a workspace (or zero its first 8192 bytes yourself), and again after a
 * QLORA_ERR_DEVICE_TIMEOUT.  Async on stream. */
QLORA_API qlora_status_t qlora_workspace_init(void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Forward: Y = X deq(W)^T + s (X A^T) B^T.  Two launches: T = X A^T (written to T_save when not
 * NULL, for the backward pass), then the fused dequant-GEMM whose epilogue adds s T B^T.
 *   W: frozen weight (host struct, device arrays); X [M,K], A [r,K], B [N,r]; Y [M,N] out;
 *   T_save [M,r] out or NULL; scale = s; ws/ws_bytes: workspace (>= qlora_workspace_size(FWD)). */
QLORA_API qlora_status_t qlora_linear_fwd(const qlora_weight_t* W, const void* X, const void* A,
                                const void* B, void* Y, void* T_save, int64_t M, int r,
                                float scale, void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Backward: dX = dY deq(W) + s (dY B) A, dA = s (dY B)^T X, dB = s dY^T T.
 *   T [M,r]: the forward's T_save, or NULL to recompute it from X and A.
 *   dX [M,K] out or NULL (skip the input gradient); dA [r,K] and dB [N,r] out (overwritten). */
QLORA_API qlora_status_t qlora_linear_bwd(const qlora_weight_t* W, const void* X, const void* A,
                                const void* B, const void* T, const void* dY, void* dX, void* dA,
                                void* dB, int64_t M, int r, float scale, void* ws, size_t ws_bytes,
                                qlora_stream_t stream);

/* Grouped (mixture-of-experts) forward: expert e applies its own W_e, A_e, B_e to rows
 * [offsets[e], offsets[e+1]) of the expert-packed X ("Quantized weights, full precision", "LoRA
 * operations and quantization": LoRA on the mxfp4 experts of an MoE model).
 *   W: one struct describing the stacked weights (codes [E,N,K/2], scales [E,N,K/bs],
 *   tensor_scale [E] for NVFP4); d_offsets: device int32 [E+1], exclusive prefix sum,
 *   offsets[0] = 0, offsets[E] = M_total, non-decreasing (checked on the device: a violation is
 *   reported as QLORA_ERR_INVALID_ARG by qlora_get_device_status); A [E,r,K], B [E,N,r];
 *   X [M_total,K]; Y [M_total,N]; T_save [M_total,r] or NULL. */
QLORA_API qlora_status_t qlora_grouped_fwd(const qlora_weight_t* W, int E, const int32_t* d_offsets,
                                 int64_t M_total, const void* X, const void* A, const void* B,
                                 void* Y, void* T_save, int r, float scale, void* ws,
                                 size_t ws_bytes, qlora_stream_t stream);

/* Grouped backward: per expert as qlora_linear_bwd; dA [E,r,K], dB [E,N,r] (experts with no rows
 * get zeros); dX [M_total,K] or NULL; T [M_total,r] or NULL (recompute). */
QLORA_API qlora_status_t qlora_grouped_bwd(const qlora_weight_t* W, int E, const int32_t* d_offsets,
                                 int64_t M_total, const void* X, const void* A, const void* B,
                                 const void* T, const void* dY, void* dX, void* dA, void* dB,
                                 int r, float scale, void* ws, size_t ws_bytes,
                                 qlora_stream_t stream);

/* Forward without a workspace: the same computation as qlora_linear_fwd, for callers
 * that cannot allocate device memory where they run the layer -- for example runtimes that
 * allocate everything at start-up and forbid allocation on the step path (an allocation can
 * synchronise the device and fragment its memory), or plain C callers with no allocator of their
 * own.  The paper has no counterpart of this entry point; it only changes who provides scratch.
 *   Scratch is a fixed 4 MiB array inside the library (every GPU that loads the library holds it
 *   until the process exits): 256 bytes of status, the [M,r] bf16 operand Zs and, when T_save is
 *   NULL, an [M,r] bf16 T.  It always runs the tiled kernels, so for M > 256 its results are
 *   bitwise those of qlora_linear_fwd; shorter batches, which qlora_linear_fwd runs through the
 *   weight-streaming kernel, differ from them in rounding only.  A call fits when
 *   256 + Z <= 4 MiB with T_save, or 256 + 2 Z <= 4 MiB without, where Z = 2*M*r bytes rounded up
 *   to a multiple of 256: M*r <= 2,097,024 with T_save, or M*r <= 1,048,448 without (for r = 64:
 *   M <= 32766 and M <= 16382).  Larger sizes are rejected with QLORA_ERR_WORKSPACE before
 *   anything is enqueued.
 *   The call allocates nothing (no cudaMalloc/cudaFree, no allocating library routine); it clears
 *   the status word on `stream` each call.
 *   The first call on each device looks up the array's device address (cudaGetSymbolAddress) with
 *   that device current; make that first call before any stream capture.
 *   Every call uses the same array and leaves its contents behind: calls whose work overlaps on
 *   the GPU (other streams, other threads) race on it, so order them on one stream.
 *   A device-side wait that gives up ends the kernel early and records QLORA_ERR_DEVICE_TIMEOUT
 *   in the array's status word; read it with qlora_linear_fwd_noalloc_status.
 * Arguments and their checks are those of qlora_linear_fwd, minus the workspace (M = 0 is a
 * no-op returning QLORA_OK and accepts NULL X and Y). */
QLORA_API qlora_status_t qlora_linear_fwd_noalloc(const qlora_weight_t* W, const void* X,
                                                  const void* A, const void* B, void* Y,
                                                  void* T_save, int64_t M, int r, float scale,
                                                  qlora_stream_t stream);

/* Opt-in native block-scaled forward for MXFP4 weights (W4A8), an inference-style variant of
 * qlora_linear_fwd ("Quantized weights, full precision", "LoRA operations and quantization":
 * Blackwell's mxfp4-native ops; "Fine-Tuning 4-Bit Models", "Case 3": a W4AFP8 variant):
 *   Y = deq8(X) deq(W)^T + s (X A^T) B^T
 * deq8(X) is X quantised to MXFP8 as qlora_mxfp8_quantize does; deq(W) is the exact product of
 * each E2M1 code and its E8M0 block scale (not rounded to bf16).  The tensor cores multiply the
 * stored 4-bit codes by the 8-bit activation codes with both block scales, accumulating in fp32
 * (tcgen05.mma kind::mxf8f6f4 block_scale); the LoRA term is the bf16 one of qlora_linear_fwd
 * (T = X A^T from the bf16 X, written to T_save when not NULL).  Y therefore differs from
 * qlora_linear_fwd by the activation quantisation (each element of X moves by up to 2^-4 of its
 * magnitude); the backward pass stays qlora_linear_bwd.  Three launches: quantise X, T, GEMM.
 *   W: MXFP4 only, K % 128 == 0 (others: QLORA_ERR_UNSUPPORTED); W->codes 32-byte aligned.
 *   Other arguments and limits as qlora_linear_fwd; ws >= qlora_workspace_size(
 *   QLORA_OP_FWD_W4A8), which holds Zs, T (when T_save is NULL), the E4M3 codes of X [M,K] and
 *   their scales [M,K/32].  M = 0 is a no-op. */
QLORA_API qlora_status_t qlora_linear_fwd_w4a8(const qlora_weight_t* W, const void* X,
                                               const void* A, const void* B, void* Y,
                                               void* T_save, int64_t M, int r, float scale,
                                               void* ws, size_t ws_bytes, qlora_stream_t stream);

/* Quantise X [M,K] bf16 to MXFP8: codes [M,K] uint8 E4M3 and scales [M,K/32] uint8 E8M0, one per
 * 32 consecutive elements along K.  The pages fix no activation format or rule; this is the OCP MX
 * shared-exponent rule, as the weight encoder uses for MXFP4: per block e = clamp(floor(log2 amax)
 * - 8 + 127, 0, 254) (8 = E4M3's largest normal exponent; 0 for an all-zero block), element =
 * the nearest E4M3 value of x / 2^(e-127), ties to the even code, magnitudes saturating at 448,
 * the sign dropped when the magnitude rounds to zero.  Requires K % 128 == 0 and 16-byte aligned
 * pointers (M = 0 is a no-op).  X must be finite.  Async on stream; used by qlora_linear_fwd_w4a8
 * and exported for testing. */
QLORA_API qlora_status_t qlora_mxfp8_quantize(const void* X, int64_t M, int64_t K, void* codes,
                                              void* scales, qlora_stream_t stream);

/* Synchronise `stream` and read the status word of qlora_linear_fwd_noalloc's fixed scratch on
 * the current device: QLORA_OK, or the device-side error of the last no-alloc call (each call
 * clears it when it starts).  Allocates nothing.  Not for the compute path. */
QLORA_API qlora_status_t qlora_linear_fwd_noalloc_status(qlora_stream_t stream);

/* Synchronise `stream` and read the workspace's device status word (QLORA_OK or the first
 * device-side error recorded since qlora_workspace_init).  Not for the compute path. */
QLORA_API qlora_status_t qlora_get_device_status(void* ws, qlora_stream_t stream);

/* Test-only: decode the whole weight through the kernels' own dequant stage (TMA code loads,
 * register decode, swizzled shared-memory tile) and write it un-swizzled as bf16 [N,K] to `out`
 * (N*K*2 bytes).  transposed = 0 uses the forward tiling (K-major operand tile), 1 the dX tiling
 * (MN-major operand tile); 2 and 3 run the short-batch kernels' decoders (batches of up to 64
 * rows: 2 the forward's register / tensor-memory form, 3 the dX shared-memory form; not for
 * NF4_DQ, which those kernels do not take) -- their NVFP4 elements are written times 2^-8, as
 * those kernels use them.  NVFP4 is written WITHOUT the tensor scale (the kernels apply it in the
 * epilogue).  This is the one call that writes a bf16 weight to memory: it exists to check the
 * decode bit for bit and is never used by the layer. */
QLORA_API qlora_status_t qlora_debug_dequant(const qlora_weight_t* W, int transposed, void* out,
                                   qlora_stream_t stream);

/* Test-only: run a kernel that waits on a barrier nothing ever completes, with a wait limit of
 * about limit_us microseconds, to check that bounded waits end with QLORA_ERR_DEVICE_TIMEOUT
 * recorded in the workspace instead of hanging. */
QLORA_API qlora_status_t qlora_debug_wait_timeout(void* ws, size_t ws_bytes, int limit_us,
                                        qlora_stream_t stream);

/* Quantise a float weight once, before training ("Training LLMs on a Budget", §3 "The setup"):
 * v [N,K] (row-major, device; fp32, or bf16 when v_is_bf16) into the
 * storage W describes (fmt, N, K and device pointers codes, scales, tensor_scale for NVFP4,
 * scales2 for NF4_DQ; the arrays are written although the struct declares them const).  One
 * weight per call: an expert stack is quantised one expert at a time, each with its own slice of
 * the arrays.  Errors: QLORA_ERR_INVALID_ARG for a shape or pointer outside the weight limits
 * every entry point applies (N % 16, K % 64, 16-byte aligned codes and scales) or a v that is
 * NULL or not 16-byte aligned; QLORA_ERR_CUDA for a failed launch.  The pages give no rounding rules; these are the
 * library's (the oracle's `oracle_encode` states them the same way):
 *   NF4    absmax = max |v| of the 64-block; code = the number of NF4 level midpoints below
 *          v / absmax (binary64), ties to the lower code; an all-zero block is all code 7.
 *   NF4_DQ as NF4 against the decoded absmax fp32(e4m3(c1) * s2), s2 = fp32(group max / 448) per
 *          256 consecutive blocks (1 for an all-zero group), c1 = nearest E4M3 of absmax / s2.
 *   MXFP4  e = clamp(floor(log2 amax) - 2 + 127, 0, 254) (0 for a zero block); code = nearest
 *          E2M1 of v / 2^(e-127), ties to the even code, saturating at 6.
 *   NVFP4  tensor_scale = fp32(max |v| / 2688) (1 for a zero tensor); block scale = nearest E4M3
 *          of amax / (6 tensor_scale); code = nearest E2M1 of v / (e4m3(s_b) tensor_scale).
 *   Quotients binary64, E4M3 ties to the even code, saturating at 448.  v must be finite.
 * Async on stream (NVFP4: three launches, the tensor scale's slot used in between). */
QLORA_API qlora_status_t qlora_quantize(const qlora_weight_t* W, const void* v, int v_is_bf16,
                                        qlora_stream_t stream);

/* Merge a trained adapter into a stored weight and requantise ("Training LLMs on a Budget",
 * §2 "Deployment: keep or merge"; "Fine-Tuning 4-Bit Models", "Case 2" and "Case 3"):
 * W_out = Q(deq(W) + scale B A),
 * with Q the rules of qlora_quantize in W_out's format (any format, same N and K).  The merged
 * value of (n,k) is fp32(deq(W)[n,k] + scale * sum_j B[n,j] A[j,k]), the sum over j = 0..r-1 in
 * order, every product and sum in binary64; it is written to `merged` [N,K] fp32 (device,
 * caller-owned scratch, kept as an output: the adapter signal lost to requantisation is
 * deq(W_out) - merged).  A [r,K], B [N,r] bf16; 1 <= r <= 1024.  Async on stream. */
QLORA_API qlora_status_t qlora_merge_requantize(const qlora_weight_t* W, const void* A,
                                                const void* B, int r, float scale,
                                                const qlora_weight_t* W_out, float* merged,
                                                qlora_stream_t stream);

/* LoftQ initialisation of the adapter for a quantised base ("Training LLMs on a Budget: LoRA,
 * QLoRA, and LoftQ", §4 "The algorithm: alternating quantization and SVD"): starting from
 * B A = 0, `iters` rounds of  Q_t = quantise(W - scale B_{t-1} A_{t-1})  (the rules of
 * qlora_quantize, in Q's format)  then  scale B_t A_t = the rank-r truncated SVD U_r S_r V_r^T of
 * R_t = W - deq(Q_t), split as B_t = U_r sqrt(S_r / scale), A_t = sqrt(S_r / scale) V_r^T.
 *   W       [N,K] fp32, device (N, K from Q); not modified.
 *   Q       receives the last quantisation Q_iters (its storage is written).
 *   A_out   [r,K] bf16, B_out [N,r] bf16 (device): A_iters, B_iters rounded to bf16 once at the end.
 *   errs    [iters+1] fp32, device: errs[0] = ||W - deq(Q_1)||_F (the plain QLoRA start, B = 0),
 *           errs[t] = ||W - deq(Q_t) - scale B_t A_t||_F with the unrounded factors.
 *   sigma   [r] fp32, device, or NULL: the top r singular values of the last residual.
 *   1 <= r <= min(96, N, K); 1 <= iters <= 64; scale > 0; N*K <= 2^31.
 * The SVD is randomized subspace iteration (l = min(r + 16, 96, N, K) columns, a Rademacher test
 * matrix from SplitMix64(seed), `power_iters` in [0, 16] rounds of R R^T, Rayleigh-Ritz) in fp32
 * with fp64 l x l eigenproblems: exact for a residual of rank <= l, and within the usual
 * randomized-SVD bound otherwise (more power iterations bring it closer to the truncated SVD).
 * Deterministic for a given seed.  work: device scratch of qlora_loftq_workspace_size(N, K, r)
 * bytes (256-byte aligned; about 4 N K bytes).  Async on stream.  Errors as qlora_quantize, plus
 * QLORA_ERR_WORKSPACE for a short workspace. */
QLORA_API size_t qlora_loftq_workspace_size(int64_t N, int64_t K, int r);
QLORA_API qlora_status_t qlora_loftq(const float* W, const qlora_weight_t* Q, int r, float scale,
                                     int iters, int power_iters, uint64_t seed, void* A_out,
                                     void* B_out, float* errs, float* sigma, void* work,
                                     size_t work_bytes, qlora_stream_t stream);

/* Benchmark support: measure the decode throughput of the short-batch kernels' dequant stage
 * (the decoder that streams the 4-bit weight at batches of up to 64 rows) on every SM -- 512
 * threads per SM, each decoding `iters` 64-element items into a shared-memory operand tile -- and
 * return the mean decoded weights per SM clock cycle in *weights_per_clock_per_sm.  fmt: QLORA_FMT_*; 1 <= iters
 * <= 2^20.  Synchronises the device and allocates two small device buffers; not for the compute
 * path.  The result is the ceiling of the short-batch path, where every weight is decoded for a
 * few activation rows. */
QLORA_API qlora_status_t qlora_debug_decode_rate(int fmt, int iters,
                                                 double* weights_per_clock_per_sm);

/* Profiling support for benchmarks.  qlora_launch_count() is the number of kernels this library
 * has launched in the process (always counted).  While profiling is enabled, every launch is also
 * bracketed by two CUDA events recorded on its stream (up to 65536 launches; events are created by
 * qlora_profile_enable, never on the compute path); qlora_profile_read synchronises on them and
 * returns, per kernel kind, the launch count and total milliseconds.  Kinds: "fused_fwd",
 * "fused_dx", "lora_down_T", "lora_down_U", "lora_wgrad" (grouped variants add "grouped_"),
 * "stream_fwd", "stream_dx", "stream_reduce" (batches of 65-256 rows), "short_fwd", "short_dx"
 * (batches of up to 64 rows).
 * Host-side bookkeeping only; the compute path is unchanged when profiling is off. */
QLORA_API int64_t qlora_launch_count(void);
QLORA_API qlora_status_t qlora_profile_enable(int enable);
QLORA_API qlora_status_t qlora_profile_reset(void);
/* Fills up to max_kinds entries; returns the number of kinds through *n_kinds. */
QLORA_API qlora_status_t qlora_profile_read(int max_kinds, int* n_kinds, const char** names,
                                            int* counts, double* total_ms);

/* A short English description of a status code (static storage). */
QLORA_API const char* qlora_status_string(qlora_status_t status);

/* Build identification: "<version> sm_100a". */
QLORA_API const char* qlora_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_H_ */
