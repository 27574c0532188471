// Host-side internals shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
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

// ------------------------------------------------------------------------ GEMV
// Geometry shared by the tactic resolver and the GEMV launcher.
constexpr int kGemvWarps = 8;                 // warps per CTA
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kChunkK = 32;                   // k per lane per step (16 code bytes)
constexpr int kWarpK = 32 * kChunkK;          // k per warp step (512 code bytes)
constexpr int kGemvMaxM = 32;
constexpr int kSmemBudget = 200 * 1024;       // dynamic shared memory we allow per CTA

// Activation rows the GEMV kernel instance for m is compiled for (1, 2, 4, ..., 32).
inline int gemv_mt(int64_t m) {
  int mt = 1;
  while (mt < m) mt *= 2;
  return mt;
}

// Shared memory the GEMV needs: m activation rows over klen k as f16, padded to whole warp
// steps of 1024 k, plus one fp32 power-of-two scale per 16-block, plus the in-CTA split-K
// combine buffer (2 parities x 8 warps x R rows x MT activation rows, fp32).
inline int64_t gemv_smem_bytes(int64_t m, int64_t klen, int R) {
  const int64_t padded = (klen + 1023) / 1024 * 1024;
  return m * padded * 2 + m * (klen / 16) * 4 + 2 * 8 * (int64_t)R * gemv_mt(m) * 4;
}

struct GemvArgs {
  const uint16_t* A;
  const uint8_t* Wq;
  const uint8_t* Ws;
  const float* gscale;
  uint16_t* out;       // used when splits == 1
  float* partials;     // [splits, m, n] when splits > 1
  int64_t m, n, k;
  int splits;         // S: global K splits (grid.y)
  int kw;             // KW: warps sharing one row group inside a CTA (1, 2, 4, 8)
  int rows_per_warp;  // R
  int grid_x;         // CTAs per split wanted by the tactic (capped by occupancy at launch)
  int ctas_per_sm;
  int num_sms;
  int smem_bytes;
  int pdl;            // launch with programmatic stream serialization
};
int launch_gemv(const GemvArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------------- reduce
int launch_splitk_reduce(const float* partials, int splits, int64_t m, int64_t n,
                         const float* gscale, uint16_t* out, bool pdl, cudaStream_t stream);

// ------------------------------------------------------------------------ pack
int launch_pack(const float* W, int64_t n, int64_t k, uint8_t* Wq, uint8_t* Wscale,
                float* gscale, cudaStream_t stream);

}  // namespace fi
