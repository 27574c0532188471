// Fixed-order split-K reduction (PR #4038, Description, "What it does": the split-K item;
// each split leaves an fp32 partial and a second, PDL-chained kernel adds the partials in
// one fixed order, which makes the result repeat bit for bit from run to run).
//
//   out[e] = round( (((p[0][e] + p[1][e]) + p[2][e]) + ...) * gscale )   all fp32
//
// round() is to nearest even into bf16, or into f16 for the optional fp16 output (PR #4038's
// commit covering fp16 output through the GEMV path).
//
// HBM-bound elementwise pass: each thread owns 4 consecutive elements (16-byte loads of
// every partial, one 8-byte store), the grid covers the [m, n] output once. Launched with
// programmatic stream serialization after the split-K producer: the CTAs may become
// resident early and block in griddepcontrol.wait until the producer grid has completed
// and its writes are visible.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace fi {

template <bool F16>
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ partials,
                                                             int splits, int64_t mn,
                                                             const float* __restrict__ gscale,
                                                             uint16_t* __restrict__ out,
                                                             bool vec4) {
  pdl_launch_dependents();
  pdl_wait();
  const float g = *gscale;
  const int64_t e0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 4;
  if (e0 >= mn) return;
  if (vec4 && e0 + 4 <= mn) {
    float4 s = *reinterpret_cast<const float4*>(partials + e0);
    for (int p = 1; p < splits; ++p) {
      const float4 v = *reinterpret_cast<const float4*>(partials + (int64_t)p * mn + e0);
      s.x = __fadd_rn(s.x, v.x);
      s.y = __fadd_rn(s.y, v.y);
      s.z = __fadd_rn(s.z, v.z);
      s.w = __fadd_rn(s.w, v.w);
    }
    const uint32_t lo = (uint32_t)f32_to_out(__fmul_rn(s.x, g), F16) |
                        ((uint32_t)f32_to_out(__fmul_rn(s.y, g), F16) << 16);
    const uint32_t hi = (uint32_t)f32_to_out(__fmul_rn(s.z, g), F16) |
                        ((uint32_t)f32_to_out(__fmul_rn(s.w, g), F16) << 16);
    *reinterpret_cast<uint2*>(out + e0) = make_uint2(lo, hi);
  } else {
    for (int64_t e = e0; e < e0 + 4 && e < mn; ++e) {
      float s = partials[e];
      for (int p = 1; p < splits; ++p) s = __fadd_rn(s, partials[(int64_t)p * mn + e]);
      out[e] = f32_to_out(__fmul_rn(s, g), F16);
    }
  }
}

int launch_splitk_reduce(const float* partials, int splits, int64_t m, int64_t n,
                         const float* gscale, uint16_t* out, bool out_f16, bool pdl, cudaStream_t stream) {
  const int64_t mn = m * n;
  if (mn == 0) return FI_OK;
  const bool vec4 = (mn % 4 == 0) && ((reinterpret_cast<uintptr_t>(partials) & 15) == 0) &&
                    ((reinterpret_cast<uintptr_t>(out) & 7) == 0);
  const int64_t blocks = ((mn + 3) / 4 + 255) / 256;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, out_f16 ? splitk_reduce_kernel<true> : splitk_reduce_kernel<false>, partials, splits,
                         mn, gscale, out, vec4) != cudaSuccess)
    return set_cuda_error("splitk_reduce_kernel launch");
  return FI_OK;
}

}  // namespace fi
