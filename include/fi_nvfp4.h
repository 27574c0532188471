/*
 * fi_nvfp4.h - bf16 activations x NVFP4 weights (mm_bf16_fp4) on NVIDIA B200 (sm_100a).
 *
 * The operation, after "perf(gemm): split-K, occupancy, and m=1 stream-GEMV decode tactics
 * for mm_bf16_fp4" (flashinfer PR #4038), Description:
 *
 *     out[m, n] = A[m, k] . dequant(W[n, k])^T
 *
 * with A in bf16 and W in NVFP4: E2M1 4-bit codes packed two per byte, one E4M3 scale per
 * 16 contiguous k, one fp32 scale for the whole tensor; fp32 accumulation, bf16 output.
 * Split-K tactics write fp32 partials that a second kernel sums in a fixed order, so
 * results are bitwise deterministic run to run (PR #4038, "What it does"); within one
 * tactic a row's bits do not depend on m (the batch-invariant property of the FlashInfer
 * v0.7.4 article, in its section on why identical bits matter).
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library never frees
 *    or retains them beyond the call. Calls are asynchronous on `stream` (NULL = legacy
 *    default stream) and never synchronise the host.
 *  - bf16 tensors are passed as uint16_t bit patterns; layouts are row-major, dense.
 *  - NVFP4 layout (the canonical one of PR #4038's GEMV commit message: packed
 *    [N, K/2] codes with linear E4M3 scales): Wq is uint8 [n, k/2], byte j of a row holds
 *    code 2j in bits 0-3 and code 2j+1 in bits 4-7; Wscale is uint8 [n, k/16] of E4M3
 *    codes, row-major (linear, unswizzled); gscale points to one fp32 in device memory (so
 *    calls can be captured in a CUDA graph without a host read).
 *  - Return value: FI_OK (0) or a negative fi_status. On error nothing was launched and a
 *    message is available from fi_last_error() (thread-local). A CUDA launch failure
 *    returns FI_ERR_CUDA after other work of the same call may already be queued.
 *  - Supported device: compute capability 10.0 (B200, sm_100a); other devices return
 *    FI_ERR_UNSUPPORTED_ARCH.
 */
#ifndef FI_NVFP4_H_
#define FI_NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FI_API __attribute__((visibility("default")))
#else
#define FI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so this header needs no CUDA headers. */
typedef struct CUstream_st* fi_stream_t;

typedef enum {
  FI_OK = 0,
  FI_ERR_INVALID_ARG = -1,       /* null / misaligned pointer, negative size, bad tactic */
  FI_ERR_UNSUPPORTED_SHAPE = -2, /* k not a multiple of 32, m beyond the tactic's range */
  FI_ERR_UNSUPPORTED_ARCH = -3,  /* current device is not compute capability 10.0 */
  FI_ERR_WORKSPACE = -4,         /* split-K workspace missing or too small */
  FI_ERR_CUDA = -5               /* a CUDA runtime call or launch failed */
} fi_status;

/* ------------------------------------------------------------------------- tactics
 * A tactic is a 32-bit code built by FI_TACTIC(kind, splits, ctas_per_sm, variant):
 *   kind         FI_KIND_GEMV (streaming GEMV, 1 <= m <= 32) or FI_KIND_MMA (tcgen05
 *                tensor-core GEMM, 1 <= m <= 256, k a multiple of 64);
 *   splits       number of K partitions S (1..4095); 0 = device-sized ("knee") split:
 *                the smallest S that gives the device enough concurrent weight streams
 *                (PR #4038, Description, "What it does": the device-sized GEMV split).
 *                MMA: 1..k/64 splits of whole 64-k steps; 0 = the split with the fewest
 *                waves of steps for one CTA per SM (partials and the reduce counted);
 *   ctas_per_sm  CTAs per SM the grid is sized for (PR #4038, Description, "What it
 *                does": occupancy tactics); 0 = automatic. GEMV stream pipeline: 1 = one
 *                16-warp CTA per SM, 2 = two 8-warp CTAs per SM; ring pipeline: 1..15.
 *                MMA: 0 or 1;
 *   variant      GEMV: low nibble = weight rows computed together by one warp (stream
 *                pipeline 1, 2 or 4; ring pipeline 1, 2, 4 or 8, at most 16 / m rounded to a
 *                power of two; 0 = automatic); high nibble = pipeline (0 = automatic:
 *                1, or 2 where the activations do not fit a half SM; at m = 1 with S > 1
 *                and automatic rows, 4 with two CTAs per SM where k % 256 != 0, else 1 with
 *                4 rows per item, where those row groups still give every SM 4 warps;
 *                1 = per-warp
 *                asynchronous copies, 2 = producer-warp ring, 3 = per-warp
 *                copies in one half-SM CTA per SM, so that consecutive calls overlap, with
 *                an L2 prefetch of weights up to 40 MB; its CTAs-per-SM field is ignored;
 *                4 = weights loaded straight to registers, 1 or 2 rows per warp;
 *                5 = the lean form of 1 for m = 1: k % 256 == 0 and every split's k/32 chunks
 *                a multiple of 32, 1, 2 or 4 rows per item). At m = 1 the automatic pipeline is
 *                5 wherever it applies.
 *                MMA: where the activations are converted to the tensor core's f16 operand
 *                (the same arithmetic and bits either way): 1 = a prepass kernel into the
 *                workspace; 2 = inside the MMA kernel, into shared memory (m <= 128 and the
 *                split's k range x 16-row-padded m fits next to the weight ring, else
 *                FI_ERR_UNSUPPORTED_SHAPE); 0 = automatic: 2 for one-wave grids at m <= 8
 *                with at most 28 64-k steps per split, else 1. Resolves to 1 or 2.
 *                The default table: for the shapes the library's cold-L2 tuner measured (the
 *                generated csrc/tactic_table.inc, per SM count and bucket of m), its pick;
 *                otherwise at m = 1, 3 for weights up to 12 MB, else 4 where k % 256 != 0, 5
 *                where k % 2048 == 0, 1 otherwise.
 * Only `kind` and the resolved S change the arithmetic: two tactics with the same kind
 * and S give bitwise identical outputs (whatever their pipeline, rows or CTAs), and for a
 * fixed tactic every output row is bitwise independent of m. Both kinds form every product
 * exactly and accumulate in fp32; GEMV and MMA results differ in their last bits because
 * they group and order the fp32 additions differently (the GEMV sums each 16-block's products
 * in element order, then adds the block sum times its scale; the MMA accumulates 64-k steps
 * of pre-scaled weights in the tensor core).
 * FI_TACTIC_DEFAULT (-1) selects from the built-in per-shape
 * table (PR #4038, Description, "What it does": the untuned m=1 route to the GEMV); the
 * table's choice of kind and S depends on m, so the default is batch-invariant only
 * within the m range of one table entry.
 */
#define FI_KIND_GEMV 0
#define FI_KIND_MMA 1
#define FI_TACTIC_DEFAULT ((int64_t)-1)
#define FI_TACTIC(kind, splits, ctas_per_sm, variant)                          \
  ((int64_t)(((int64_t)(kind) << 24) | ((int64_t)(splits) << 12) |             \
             ((int64_t)(ctas_per_sm) << 8) | (int64_t)(variant)))
#define FI_TACTIC_KIND(t) ((int)(((t) >> 24) & 0xF))
#define FI_TACTIC_SPLITS(t) ((int)(((t) >> 12) & 0xFFF))
#define FI_TACTIC_CTAS(t) ((int)(((t) >> 8) & 0xF))
#define FI_TACTIC_VARIANT(t) ((int)((t) & 0xFF))

/* A tactic resolved for one shape and device (host-side description). */
typedef struct {
  int32_t kind;        /* FI_KIND_GEMV or FI_KIND_MMA */
  int32_t splits;      /* resolved S >= 1 */
  int32_t ctas_per_sm; /* resolved co-resident CTAs per SM */
  int32_t variant;     /* resolved variant (GEMV: rows per warp | pipeline << 4; MMA: 1 prepass, 2 in-kernel) */
  int32_t grid_x;      /* CTAs along n */
  int32_t grid_y;      /* CTAs along k (= splits) */
  int32_t threads;     /* threads per CTA */
  int32_t smem_bytes;  /* dynamic shared memory per CTA */
  int64_t workspace_bytes; /* scratch: GEMV fp32 partials (0 if S == 1); MMA variant 1: f16 A and its scales,
                              then partials if S > 1; MMA variant 2: partials if S > 1 */
} fi_tactic_info;

/* Output element types (the op writes bf16 by default; PR #4038's commits add an fp16 output
 * through the GEMV path, covered by its test of fp16 GEMV output). */
typedef enum { FI_DTYPE_BF16 = 0, FI_DTYPE_F16 = 1 } fi_dtype;

/* ------------------------------------------------------------------ entry points */

/*
 * Quantise fp32 weights to NVFP4 (the weight-preparation step; not on the timed path).
 *   W       device fp32 [n, k], row-major, 16-byte aligned.
 *   Wq      device uint8 [n, k/2] (output), 16-byte aligned.
 *   Wscale  device uint8 [n, k/16] (output), 16-byte aligned.
 *   gscale  device fp32 [1] (output); also used as scratch by the call.
 * Recipe: gscale = amax(|W|) / (448*6) (one fp32 division); for each 16-block
 * sf = E4M3_rn_satfinite((amax_block / 6) / gscale); denom = sf * gscale;
 * code = E2M1_rn_satfinite(w / denom) with the sign of w, or 0 for the whole block when
 * denom == 0. All arithmetic is IEEE fp32 round-to-nearest-even, so the result is
 * bit-identical to a CPU implementation of the same steps. Inputs must be finite.
 * Preconditions: n >= 0, k >= 0, k % 16 == 0 (n == 0 or k == 0 writes gscale = 0).
 */
FI_API int fi_nvfp4_pack_weights(const float* W, int64_t n, int64_t k, uint8_t* Wq,
                          uint8_t* Wscale, float* gscale, fi_stream_t stream);

/*
 * out[m, n] = bf16_rn(gscale * sum_k A[m, k] * e2m1(Wq) * e4m3(Wscale)), with exact products
 * and fp32 accumulation (see the tactic notes above for the order of the additions)
 * (PR #4038, Description).
 *   A       device bf16 bits [m, k], 16-byte aligned.
 *   Wq, Wscale, gscale  NVFP4 weights as produced by fi_nvfp4_pack_weights; Wq and Wscale
 *           16-byte aligned. The weights are read with bulk asynchronous copies that may
 *           start before the kernel that precedes this call on `stream` has finished
 *           (programmatic dependent launch): Wq, Wscale must not be written by that kernel.
 *           A and gscale are read, and out written, only after it has completed.
 *   out     device bf16 bits [m, n], 2-byte aligned; must not overlap the inputs.
 *   tactic  FI_TACTIC_DEFAULT or an FI_TACTIC(...) code (see above).
 * Preconditions: m >= 0, n >= 0, k >= 0, k % 32 == 0; m <= 32 for GEMV tactics and
 * m <= 256 with k % 64 == 0 for MMA tactics (FI_ERR_UNSUPPORTED_SHAPE otherwise). m == 0
 * or n == 0 is a no-op; k == 0 writes zeros.
 * Workspace: a GEMV call with S > 1 needs fi_mm_workspace_bytes() bytes of device memory
 * for fp32 partials; an MMA call with activation variant 1 needs them for its f16 copy of A
 * (each row and K split times a power of two), those scales and, when S > 1, the fp32
 * partials; variant 2 only for the partials. It uses the buffer registered with
 * fi_set_workspace() for the current device (FI_ERR_WORKSPACE if that is too small); if
 * none is registered, the library allocates one with cudaMalloc (growing it when needed)
 * and keeps it until process exit, except while `stream` is capturing a CUDA graph,
 * where it returns FI_ERR_WORKSPACE instead of allocating.
 * The per-device workspace is shared: calls that may overlap on different streams must
 * use fi_mm_bf16_fp4_ex with separate workspaces.
 */
FI_API int fi_mm_bf16_fp4(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale,
                   const float* gscale, uint16_t* out, int64_t m, int64_t n, int64_t k,
                   int64_t tactic, fi_stream_t stream);

/*
 * fi_mm_bf16_fp4 with a caller-provided split-K workspace (device, 256-byte aligned,
 * at least fi_mm_workspace_bytes() bytes; may be NULL when that is 0). Never allocates.
 */
FI_API int fi_mm_bf16_fp4_ex(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale,
                      const float* gscale, uint16_t* out, int64_t m, int64_t n, int64_t k,
                      int64_t tactic, void* workspace, size_t workspace_bytes,
                      fi_stream_t stream);

/*
 * fi_mm_bf16_fp4 with a choice of output type (PR #4038, the commit that covers fp16 output
 * through the GEMV path): out_dtype FI_DTYPE_BF16 writes bf16 bits as fi_mm_bf16_fp4 does,
 * FI_DTYPE_F16 writes IEEE binary16 bits, rounded to nearest even from the same fp32 value
 * (magnitudes of 65520 and more become +-inf). Every tactic and kind supports both; the fp32
 * arithmetic before the final rounding is the same, so the two outputs of one tactic are the
 * two roundings of one fp32 result.
 *   out        device [m, n] of 16-bit elements, 2-byte aligned.
 *   workspace  NULL: the per-device workspace of fi_mm_bf16_fp4 (registered or allocated, with
 *              its rules under stream capture); otherwise as fi_mm_bf16_fp4_ex.
 * Other arguments, preconditions and errors are those of fi_mm_bf16_fp4 / fi_mm_bf16_fp4_ex;
 * an out_dtype other than the two above returns FI_ERR_INVALID_ARG.
 */
FI_API int fi_mm_bf16_fp4_out(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale,
                       const float* gscale, uint16_t* out, int out_dtype, int64_t m, int64_t n,
                       int64_t k, int64_t tactic, void* workspace, size_t workspace_bytes,
                       fi_stream_t stream);

/*
 * fi_mm_bf16_fp4 without any device allocation. The paper has no counterpart: this entry
 * point exists for users of this library who may not allocate GPU memory at call time, such
 * as an operator plugin inside a serving engine that has already reserved the device's memory
 * for weights and the KV cache, or a component whose memory plan is fixed at start-up and
 * that owns no buffer it could pass to fi_mm_bf16_fp4_ex. fi_mm_bf16_fp4 would cudaMalloc its
 * workspace on first use; this variant keeps the workspace (the split-K fp32 partials, and
 * for MMA tactics of variant 1 the f16 copy of the activations) in a static device array compiled into
 * the library instead: FI_NOALLOC_SCRATCH_BYTES (4 MiB) on every GPU that loads the library,
 * held until the process exits.
 * Arguments, tactics, preconditions and results are those of fi_mm_bf16_fp4.
 * Limit: the resolved tactic's fi_mm_workspace_bytes() (GEMV: 4 * splits * m * n; MMA: about
 * 2 * m * k for variant 1, plus 4 * splits * m * n when split) must not exceed FI_NOALLOC_SCRATCH_BYTES; a
 * larger call returns FI_ERR_WORKSPACE and launches nothing. Single-split GEMV tactics use no
 * scratch. With FI_TACTIC_DEFAULT, a default whose scratch would not fit is replaced by the
 * same kind with the largest smaller split that fits (for a GEMV, with the default's pipeline
 * where that resolves at the smaller split, else the automatic one; a single split needs no
 * scratch), so its bits may differ from fi_mm_bf16_fp4's default for that shape.
 * Set-up: the first call on a device that reaches a launch looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first call before any
 * stream capture begins.
 * Sharing: all calls on a device use the same array, and it keeps the last call's contents.
 * Nothing in it needs to start at zero (each split writes all of its partials before the
 * reduce reads them; the MMA path writes its whole activation copy before reading it), but
 * calls whose kernels can overlap on the GPU (different streams, parallel graph branches)
 * race on it and must be serialised by the caller.
 * Never calls cudaMalloc, cudaFree or any other allocating routine.
 */
#define FI_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
FI_API int fi_mm_bf16_fp4_noalloc(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale,
                           const float* gscale, uint16_t* out, int64_t m, int64_t n, int64_t k,
                           int64_t tactic, fi_stream_t stream);

/*
 * Fixed-order split-K reduction (PR #4038, Description, "What it does": the split-K item):
 * for every element e of [m, n],
 *     s = ((p[0][e] + p[1][e]) + p[2][e]) + ...   (fp32, s = 0 .. splits-1 in order)
 *     out[e] = bf16_rn(s * gscale[0])             (fp32 product)
 *   partials  device fp32 [splits, m, n], 16-byte aligned.
 *   gscale    device fp32 [1].
 *   out       device bf16 bits [m, n], 2-byte aligned.
 * Preconditions: 1 <= splits <= 4095, m >= 0, n >= 0.
 */
FI_API int fi_splitk_reduce(const float* partials, int64_t splits, int64_t m, int64_t n,
                     const float* gscale, uint16_t* out, fi_stream_t stream);

/* fi_splitk_reduce with a choice of output type: out = round(s * gscale[0]) to bf16
 * (FI_DTYPE_BF16) or to IEEE binary16 (FI_DTYPE_F16, round to nearest even, +-inf from 65520
 * on); FI_ERR_INVALID_ARG for any other out_dtype. */
FI_API int fi_splitk_reduce_out(const float* partials, int64_t splits, int64_t m, int64_t n,
                         const float* gscale, uint16_t* out, int out_dtype, fi_stream_t stream);

/* --------------------------------------------------------------- host helpers
 * These run on the host only and never launch work. `num_sms` <= 0 means "query the
 * current device" (which then must exist); a positive value describes a device without
 * touching CUDA, so the tactic logic can be inspected on any machine.
 */

/* Resolve a tactic (or FI_TACTIC_DEFAULT) for a shape. Returns FI_OK and fills *info,
 * or an error status (invalid code, unsupported m for the kind, ...). */
FI_API int fi_resolve_tactic(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms,
                      fi_tactic_info* info);

/* The tactic FI_TACTIC_DEFAULT resolves to (the per-shape table). Negative on error. */
FI_API int64_t fi_default_tactic(int64_t m, int64_t n, int64_t k, int num_sms);

/* Enumerate the valid tactics for a shape into out[0 .. cap-1]; returns how many exist
 * (which may exceed cap), or a negative status. The menu: splits {1, 2, 4, 8, device-sized}
 * for every GEMV pipeline (stream and ring also at one and two rows per warp, the stream
 * pipeline also at two CTAs per SM) and for the MMA; codes resolving to the same launch are
 * listed once, codes the shape does not support are left out. */
FI_API int fi_list_tactics(int64_t m, int64_t n, int64_t k, int num_sms, int64_t* out, int cap);

/* Workspace bytes a call with this shape and tactic needs (GEMV: 0 when S == 1; MMA: the
 * f16 activations and their row scales, then the fp32 partials when S > 1), or 0 for an
 * invalid tactic. */
FI_API size_t fi_mm_workspace_bytes(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms);

/* Register a caller-owned split-K workspace for the current device (device pointer,
 * 256-byte aligned; NULL with bytes == 0 unregisters it). The library frees any buffer it
 * allocated itself for that device. The caller keeps ownership of `ptr` and must keep it
 * alive while calls that use it may run. */
FI_API int fi_set_workspace(void* ptr, size_t bytes);

/* ------------------------------------------------------------ failure detection
 * Every mbarrier wait inside the kernels (the ring pipeline's and the MMA path's) is bounded
 * in time: when a wait runs out, the kernel records a bit in a sticky per-device error word,
 * stops computing, lets its in-flight copies land and returns; the outputs of that call are
 * then undefined. (The stream pipeline has no waits between threads: each thread waits only
 * for its own copies.) The library has no counterpart on the pages; it exists so that a stuck
 * pipeline ends with an error instead of a hung GPU.
 */

/* Read and clear the current device's sticky kernel error word (0 = no error): bit 0 a
 * consumer (decode) wait, bit 1 a producer wait, bit 2 a final drain, bit 3 (MMA) a drain
 * before exit, bit 4 (MMA) the epilogue's wait ran out. Synchronizes the device. */
FI_API int fi_get_device_error(unsigned* code);

/* Test hooks. FI_DEBUG_STALL_PRODUCER: the producers of the next `value` launches (the ring
 * pipeline's producer warp, the MMA path's producers) issue no copies, so their waits run out
 * (exercises the path above without a GPU fault; stream-pipeline launches have no producer
 * and still count down).
 * FI_DEBUG_WAIT_TIMEOUT_NS: limit of every kernel wait in ns (default 1e9). */
#define FI_DEBUG_STALL_PRODUCER 1
#define FI_DEBUG_WAIT_TIMEOUT_NS 2
FI_API int fi_debug_set(int key, int64_t value);

/* Message describing the last error on this host thread ("" if none). */
FI_API const char* fi_last_error(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
FI_API int fi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FI_NVFP4_H_ */
