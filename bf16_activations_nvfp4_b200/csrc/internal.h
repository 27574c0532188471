// Host-side internals shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fi_nvfp4.h"

namespace fi {

constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------- error reporting
int set_error(int status, const char* fmt, ...);
int set_cuda_error(const char* what);  // reads and clears cudaGetLastError()
void clear_error();

// SM count of the current device (cached per device).
int device_sm_count();

// TMA tensor map over `base` (rank dims, innermost first; strides in bytes of dims 1..rank-1;
// box extents per dim), no interleave, 256-byte L2 promotion, zero fill out of bounds.
int encode_tensor_map(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const uint64_t* dims,
                      const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle);

// ------------------------------------------------------------------------ GEMV
constexpr int kGemvConsumerWarps = 16;                    // warps that decode and multiply
constexpr int kGemvThreads = (kGemvConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kChunkK = 32;                                // k per lane per step (16 code bytes)
constexpr int kGemvMaxM = 32;
constexpr int kSmemBudget = 227 * 1024 - 1024;             // dynamic shared memory per CTA we allow
constexpr int kGemvMaxStages = 16;
constexpr int kGemvStageTarget = 16 * 1024;                // preferred bytes per ring stage

// The per-warp async-copy pipeline: one CTA of 16 warps per SM, or two of 8 warps.
constexpr int kStreamMaxThreads = 512;
constexpr int kStreamIters = 2;                            // chunk iterations per work item
constexpr int kStreamCellBytes = 32 * 16 + 32 * 4;         // one iteration of one row: code cells + scale words
constexpr int kStreamHalfBudget = 228 * 1024 / 2 - 1024;   // dynamic shared memory per CTA, two CTAs per SM
// pipelines (the high nibble of the GEMV tactic variant)
constexpr int kPipeAuto = 0, kPipeStream = 1, kPipeRing = 2, kPipeOverlap = 3, kPipeReg = 4, kPipeLean = 5;
constexpr int kRegDepth = 4;   // register pipeline: chunk iterations in flight per warp
constexpr int kLeanIters = 2;  // lean stream pipeline: chunk iterations per work item

// Activation rows the GEMV kernel instance for m is compiled for (1, 2, 4, ..., 32).
inline int gemv_mt(int64_t m) {
  int mt = 1;
  while (mt < m) mt *= 2;
  return mt;
}

__host__ __device__ inline int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// Bytes of one row of E4M3 scales in a ring stage of `slab` chunks: the copied superset starts
// up to 14 bytes before the row's first scale and is rounded to 16 bytes at both ends. Shared
// by the host's shared-memory layout and the kernel, so both always agree.
__host__ __device__ inline int64_t gemv_scales_stride(int64_t slab) { return round_up(slab * 2 + 28, 16); }

// Most weight rows a ring stage holds for the kernel instance of MT activation rows (bounded
// by the accumulator registers, RMAX * MT <= 16).
__host__ __device__ constexpr int gemv_rmax(int mt) { return mt >= 16 ? 1 : (16 / mt > 8 ? 8 : 16 / mt); }
int gemv_rows_per_stage_max(int64_t m);

// Launch geometry of the GEMV for one shape and tactic (computed on the host).
struct GemvGeometry {
  int pipeline;  // kPipeStream or kPipeRing
  int S, RS, stages, ctas_per_sm, grid_x, grid_y, threads;
  int64_t stage_bytes, off_as, off_bar, off_ring, smem_bytes;
};
// Returns FI_OK and fills g, or FI_ERR_UNSUPPORTED_SHAPE when the activations of m rows over
// a split leave no room for two ring stages of one weight row in shared memory. rs_req is
// the requested rows per stage (0 = as many as fit the stage target).
int gemv_geometry(int64_t m, int64_t n, int64_t k, int S, int rs_req, int ctas_per_sm, int sms, GemvGeometry* g);
// The same for the per-warp async-copy pipeline: R rows per item (0 = automatic), ring slots
// per warp (4, else 2 when the activations leave room for only two).
int gemv_stream_geometry(int64_t m, int64_t n, int64_t k, int S, int r_req, int ctas_per_sm, int sms,
                         GemvGeometry* g, bool overlap = false);

struct GemvArgs {
  const uint16_t* A;
  const uint8_t* Wq;
  const uint8_t* Ws;
  const float* gscale;
  uint16_t* out;       // used when splits == 1
  int out_f16;         // out holds f16 (1) or bf16 (0)
  float* partials;     // [splits, m, n] when splits > 1
  int64_t m, n, k;
  int pipeline;        // kPipeStream or kPipeRing
  int splits;          // S: global K splits (grid.y)
  int rows_per_stage;  // RS: consecutive weight rows per ring stage (one consumer warp each)
  int stages;          // NST: ring stages (stream pipeline: slots per warp)
  int grid_x;          // CTAs per split
  int threads;         // threads per CTA
  int pdl;             // launch with programmatic stream serialization
  int scale16;         // stream pipeline: copy the E4M3 scales in aligned 16-byte pieces (k % 256 == 0, splits on 8 chunks)
  int prefetch_l2;     // stream pipeline: each warp asks the L2 to prefetch its whole weight range first
  int debug_stall;     // test hook: the producer issues nothing (consumer waits time out)
  int64_t stage_bytes, off_as, off_bar, off_ring, smem_bytes;
  uint64_t timeout_ns; // limit of every mbarrier wait
};
int launch_gemv(const GemvArgs& a, cudaStream_t stream);
int gemv_read_error(unsigned* bits);

// ------------------------------------------------------------------------- MMA
// Tensor-core path: one CTA per kMmaTileRows weight rows, 64 k per pipeline step. The
// activations are converted to f16 times a power of two per (row, K split): either by a prepass
// kernel into the workspace (a16 [m_pad, k], then rs [splits, m_pad] fp32 at the next 256-byte
// boundary, then the split-K partials) or, when the split's slice fits shared memory next to the
// raw-code ring ("resident" mode, m_pad <= kMmaTmemMaxM), by the kernel's decode warps into
// shared memory, in which case the workspace holds only the partials.
constexpr int kMmaTileRows = 256;
constexpr int kMmaKStep = 64;
constexpr int kMmaMaxM = 256;
constexpr int kMmaThreads = 24 * 32;
inline int mma_m_pad(int64_t m) { return (int)((m + 15) / 16 * 16); }
inline int64_t mma_rs_offset(int64_t m, int64_t k) { return round_up((int64_t)mma_m_pad(m) * k * 2, 256); }
inline int64_t mma_workspace_bytes(int64_t m, int64_t k, int64_t splits) {
  return mma_rs_offset(m, k) + (int64_t)mma_m_pad(m) * 4 * splits;
}
// split-K partials [splits, m, n] fp32 follow the activations at the next 256-byte boundary
inline int64_t mma_partials_offset(int64_t m, int64_t k, int64_t splits) {
  return round_up(mma_workspace_bytes(m, k, splits), 256);
}
// operand stages (decoded weights + activation tile of one 64-k step): as many as fit, 2..4
constexpr int kMmaMaxOpStages = 4;
// m_pad <= kMmaTmemMaxM: the decoded weights live in tensor memory, a stage is the activation
// tile only; above, a stage also holds the decoded weight tile in shared memory
constexpr int kMmaTmemMaxM = 128;
inline int64_t mma_stage_bytes(int m_pad) {
  return (m_pad <= kMmaTmemMaxM ? 0 : (int64_t)kMmaTileRows * 128) + round_up((int64_t)m_pad * 128, 1024);
}
int mma_op_stages(int m_pad);
int64_t mma_smem_bytes(int m_pad);
// Resident mode: the bytes of a split's activation slice (steps x m_pad x 128, the largest split
// of `splits` over k/64 steps) and of the row scales after it; the mode is taken when
// m_pad <= kMmaTmemMaxM and it fits shared memory next to the raw-code ring.
int64_t mma_resident_act_bytes(int m_pad, int64_t k, int splits);
inline int64_t mma_resident_extra_bytes(int m_pad) { return round_up((int64_t)m_pad * 4, 16); }
bool mma_act_resident(int m_pad, int64_t k, int splits);
int64_t mma_resident_smem_bytes(int m_pad, int64_t k, int splits);

struct MmaArgs {
  const uint16_t* A;
  const uint8_t* Wq;
  const uint8_t* Ws;
  const float* gscale;
  uint16_t* out;
  int out_f16;    // out holds f16 (1) or bf16 (0)
  uint16_t* a16;  // workspace: f16 activations [m_pad, k]
  float* rs;      // workspace: per-row inverse scales [m_pad]
  int64_t m, n, k;
  int m_pad;
  int splits;           // K splits (grid.y); > 1 writes fp32 partials [splits, m, n] to `partials`
  float* partials;
  int op_stages;        // operand stages in shared memory (mma_op_stages)
  uint32_t stage_bytes; // bytes of one operand stage (mma_stage_bytes; 0 in resident mode)
  int act_resident;     // the decode warps convert the split's activations into shared memory
  uint32_t act_bytes;   // resident mode: bytes of the activation slice (mma_resident_act_bytes)
  uint32_t act_extra_bytes;  // resident mode: row scales (mma_resident_extra_bytes)
  int debug_stall;      // test hook: the producer issues nothing (the waits time out)
  unsigned* err;        // the device error word
  uint64_t timeout_ns;  // limit of every mbarrier wait
};
int launch_mma(const MmaArgs& a, cudaStream_t stream);
// Device address of the sticky kernel error word on the current device (looked up once).
unsigned* device_error_word();

// ---------------------------------------------------------------------- reduce
int launch_splitk_reduce(const float* partials, int splits, int64_t m, int64_t n,
                         const float* gscale, uint16_t* out, bool out_f16, bool pdl, cudaStream_t stream);

// ------------------------------------------------------------------------ pack
int launch_pack(const float* W, int64_t n, int64_t k, uint8_t* Wq, uint8_t* Wscale,
                float* gscale, cudaStream_t stream);

}  // namespace fi
