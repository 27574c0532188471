// NVFP4 weight quantisation and packing (weight preparation, off the timed path).
//
// Recipe (the format named in PR #4038's Description - E2M1 codes, E4M3 scales per 16 k,
// one fp32 tensor scale - with the quantisation steps this library is specified with):
//   gscale  = amax(|W|) / 2688                      (2688 = 448 * 6, fp32 division)
//   sf_b    = E4M3_rn_sat((amax_b / 6) / gscale)    (per 16-element block b of a row)
//   denom_b = sf_b * gscale
//   code_i  = E2M1_rn_sat(w_i / denom_b), sign of w_i; all codes 0 when denom_b == 0.
// Three launches: amax (atomicMax on the fp32 bit pattern, exact and order-free), the
// per-block quantiser, and a one-thread kernel that turns amax into gscale in place.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace fi {

__global__ void __launch_bounds__(256) pack_amax_kernel(const float4* __restrict__ W4, int64_t n4,
                                                         unsigned int* __restrict__ amax_bits) {
  float m = 0.0f;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = W4[i];
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float warp_max[8];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, warp_max[w]);
    // non-negative floats order like their bit patterns
    atomicMax(amax_bits, __float_as_uint(m));
  }
}

// One thread per 16-element block.
__global__ void __launch_bounds__(256) pack_quant_kernel(const float* __restrict__ W, int64_t n,
                                                          int64_t k, const float* __restrict__ amax,
                                                          uint8_t* __restrict__ Wq,
                                                          uint8_t* __restrict__ Wscale) {
  const int64_t blocks_per_row = k / 16;
  const int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (b >= n * blocks_per_row) return;
  const float g = __fdiv_rn(*amax, 2688.0f);
  const float4* src = reinterpret_cast<const float4*>(W + b * 16);
  float x[16];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const float4 t = src[v];
    x[4 * v + 0] = t.x;
    x[4 * v + 1] = t.y;
    x[4 * v + 2] = t.z;
    x[4 * v + 3] = t.w;
  }
  float bmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(x[i]));
  uint32_t sf_code = 0;
  if (g != 0.0f) {
    const float t = __fdiv_rn(bmax, 6.0f);
    sf_code = f32_to_e4m3(__fdiv_rn(t, g));
  }
  const float sf_val = f16_lo_to_f32(e4m3x2_to_f16x2(sf_code));
  const float denom = __fmul_rn(sf_val, g);
  uint32_t lo = 0, hi = 0;
  if (denom != 0.0f) {
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      lo |= f32x2_to_e2m1x2(__fdiv_rn(x[i], denom), __fdiv_rn(x[i + 1], denom)) << (4 * i);
      hi |= f32x2_to_e2m1x2(__fdiv_rn(x[8 + i], denom), __fdiv_rn(x[8 + i + 1], denom)) << (4 * i);
    }
  }
  *reinterpret_cast<uint2*>(Wq + b * 8) = make_uint2(lo, hi);
  Wscale[b] = (uint8_t)sf_code;
}

__global__ void pack_finalize_kernel(float* gscale) {
  // the slot held amax(|W|) as written by pack_amax_kernel
  *gscale = __fdiv_rn(*gscale, 2688.0f);
}

int launch_pack(const float* W, int64_t n, int64_t k, uint8_t* Wq, uint8_t* Wscale,
                float* gscale, cudaStream_t stream) {
  if (cudaMemsetAsync(gscale, 0, sizeof(float), stream) != cudaSuccess)
    return set_cuda_error("cudaMemsetAsync(gscale)");
  const int64_t count = n * k;
  if (count == 0) return FI_OK;
  const int sms = device_sm_count();
  const int64_t n4 = count / 4;  // k % 16 == 0, so count % 4 == 0
  int64_t grid = (n4 + 255) / 256;
  if (grid > (int64_t)sms * 8) grid = (int64_t)sms * 8;
  pack_amax_kernel<<<(unsigned)grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(W), n4,
                                                       reinterpret_cast<unsigned int*>(gscale));
  if (cudaGetLastError() != cudaSuccess) return set_cuda_error("pack_amax_kernel launch");
  const int64_t nblocks = n * (k / 16);
  const int64_t qgrid = (nblocks + 255) / 256;
  if (qgrid > 0x7fffffffLL) return set_error(FI_ERR_UNSUPPORTED_SHAPE, "weight tensor too large");
  pack_quant_kernel<<<(unsigned)qgrid, 256, 0, stream>>>(W, n, k, gscale, Wq, Wscale);
  if (cudaGetLastError() != cudaSuccess) return set_cuda_error("pack_quant_kernel launch");
  pack_finalize_kernel<<<1, 1, 0, stream>>>(gscale);
  if (cudaGetLastError() != cudaSuccess) return set_cuda_error("pack_finalize_kernel launch");
  return FI_OK;
}

}  // namespace fi
