// Streaming GEMV for bf16 activations x NVFP4 weights, m <= 32 (sm_100a).
//
// After PR #4038's streaming GEMV ("weights stream from global memory to registers with
// latency hidden by warp count", "one output row per warp, warp-shuffle reduction", and the
// v2 commit's "A-in-SMEM staging" lever for m > 1), re-designed for B200:
//
//  * Grid (G, S): blockIdx.y is the global K split s; the G CTAs of a split take balanced,
//    contiguous ranges of weight row groups (R rows each) and persist over them.
//  * Inside a CTA the 8 warps form 8/KW slots of KW warps. The KW warps of a slot share one
//    row group and split its k range KW ways (in-CTA split-K); their partials are combined
//    through shared memory in fixed order kw = 0..KW-1, so narrow-n shapes fill the GPU
//    without a second kernel.
//  * A warp streams R rows at once: lane L reads the 16 code bytes (32 k, two scale blocks) of
//    chunk t*32+L with one coalesced 128-bit load per row plus the two E4M3 scale bytes. D steps
//    are kept in flight in a register ring, across row-group boundaries, and the first D are
//    issued before the activations are staged, so the weight stream starts at once.
//  * The CTA stages A[0:m, split] in shared memory as f16 with one power-of-two scale per
//    16-block (block floating point). A bf16 value has 8 significant bits, so the f16 copy is
//    exact for every element within 2^28 of its block maximum; smaller ones are rounded at
//    2^-39 of the block maximum.
//  * Decode is the hardware cvt.rn.f16x2.e2m1x2 (two codes per instruction, exact) and the dot
//    product the mixed-precision fma.rn.f32.f16 (f16 x f16 product, fp32 accumulate), one
//    instruction per code; an 8-bit-significand activation times an E2M1 value is exact, so the
//    only roundings are fp32 accumulation steps.
//  * Per 16-block: p = sum_{i in block} a_i * e2m1_i (sequential, fp32), then
//    acc = fma(p, sf_w * sf_a, acc). Lanes combine through a fixed xor butterfly (every lane
//    ends with the same bits), then the KW warps in fixed order. The k order of every output is
//    fixed by (k, S, KW) alone: bits do not depend on m, R, D, G or the CTAs per SM.
//  * S == 1 writes bf16_rn(acc * gscale); S > 1 writes the fp32 partial for the fixed-order
//    reduce kernel.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace fi {

namespace {

// Stage A[0:m, kbase : kbase + klen] as f16 (scaled per 16-block) plus fp32 block scales.
__device__ __forceinline__ void stage_activations(const uint16_t* __restrict__ A, int64_t k, int m,
                                                  int64_t kbase, int klen, uint32_t* Ah, float* As) {
  const int blocks_per_row = klen / 16;
  const int nblk = m * blocks_per_row;
  for (int bi = threadIdx.x; bi < nblk; bi += blockDim.x) {
    const int r = bi / blocks_per_row;
    const int b = bi - r * blocks_per_row;
    const uint16_t* src = A + (int64_t)r * k + kbase + (int64_t)b * 16;
    const uint4 v0 = ldg_v4(src);
    const uint4 v1 = ldg_v4(src + 8);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t e = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      e = max(e, (w[i] >> 7) & 0xFFu);
      e = max(e, (w[i] >> 23) & 0xFFu);
    }
    // scale the block maximum into [2^14, 2^15): biased exponent E -> shift 141 - E
    int sh = 141 - (int)e;
    sh = sh < -126 ? -126 : (sh > 126 ? 126 : sh);
    const float up = __uint_as_float((uint32_t)(sh + 127) << 23);
    const float down = __uint_as_float((uint32_t)(127 - sh) << 23);
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float lo = __uint_as_float(w[i] << 16) * up;
      const float hi = __uint_as_float(w[i] & 0xFFFF0000u) * up;
      h[i] = f32x2_to_f16x2(lo, hi);
    }
    uint4* dst = reinterpret_cast<uint4*>(Ah + (int64_t)r * (klen / 2) + b * 8);
    dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
    dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
    As[r * blocks_per_row + b] = down;
  }
}

// Sum of 16 products a_i * w_i (8 f16x2 words each), sequential in element order.
__device__ __forceinline__ float dot16(const uint32_t* a, const uint32_t* w) {
  float p = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    p = fma_lo_f16(a[i], w[i], p);
    p = fma_hi_f16(a[i], w[i], p);
  }
  return p;
}

template <int R>
struct Step {
  uint4 q[R];
  uint32_t sc[R];
};

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace

template <int MT, int R, int D>
__global__ void __launch_bounds__(kGemvThreads) gemv_nvfp4_kernel(GemvArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // let a PDL-launched split-K reduce get scheduled; it waits for this grid to finish
  pdl_launch_dependents();

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int m = (int)p.m;
  const int64_t n = p.n, k = p.k;
  const int S = p.splits;
  const int s = blockIdx.y;
  const int KW = p.kw;
  const int NS = kGemvWarps / KW;  // row-group slots per CTA
  const int slot = warp / KW;
  const int kw = warp - slot * KW;

  // K range of this split (in 32-k chunks) and of this warp inside it
  const int64_t C = k / kChunkK;
  const int64_t c0 = (int64_t)s * C / S;
  const int nch = (int)((int64_t)(s + 1) * C / S - c0);
  const int klen = nch * kChunkK;
  const int w0 = kw * nch / KW;
  const int wch = (kw + 1) * nch / KW - w0;
  // at least one (possibly empty) step per row group, so every warp of a slot meets the
  // slot's barrier once per row group even when its share of k is empty
  const int T = wch > 0 ? (wch + 31) / 32 : 1;

  // row groups of this CTA, and of this warp's slot
  const int64_t RG = (n + R - 1) / R;
  const int64_t rg_lo = (int64_t)blockIdx.x * RG / gridDim.x;
  const int64_t rg_hi = (int64_t)(blockIdx.x + 1) * RG / gridDim.x;
  const int nrg = (rg_lo + slot < rg_hi) ? (int)((rg_hi - rg_lo - slot + NS - 1) / NS) : 0;
  const int F = nrg * T;

  uint32_t* Ah = reinterpret_cast<uint32_t*>(smem);
  float* As = reinterpret_cast<float*>(smem + (int64_t)m * klen * 2);
  float* comb = As + m * (klen / 16);  // [2][NS][KW][R*MT], used when KW > 1

  const uint8_t* wq_base = p.Wq + (c0 + w0) * 16;
  const uint8_t* ws_base = p.Ws + (c0 + w0) * 2;
  const int64_t wq_row = k / 2, ws_row = k / 16;

  auto load_step = [&](Step<R>& st, int li, int lt) {
    const int c = lt * 32 + lane;
    const bool ok = li < nrg && c < wch;
    const int64_t j0 = (rg_lo + slot + (int64_t)li * NS) * R;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      if (ok && j0 + i < n) {
        st.q[i] = ldg_stream_v4(wq_base + (j0 + i) * wq_row + (int64_t)c * 16);
        st.sc[i] = ldg_stream_u16(ws_base + (j0 + i) * ws_row + (int64_t)c * 2);
      } else {
        st.q[i] = make_uint4(0, 0, 0, 0);
        st.sc[i] = 0;
      }
    }
  };

  // prologue: put the first D steps of the weight stream in flight, then stage A
  Step<R> ring[D];
  int li = 0, lt = 0;
#pragma unroll
  for (int d = 0; d < D; ++d) {
    load_step(ring[d], li, lt);
    if (++lt == T) { lt = 0; ++li; }
  }
  stage_activations(p.A, k, m, c0 * kChunkK, klen, Ah, As);
  __syncthreads();

  const float g = (S == 1) ? *p.gscale : 1.0f;
  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;

  int ci = 0, ct = 0;
  for (int f0 = 0; f0 < F; f0 += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (f0 + d < F) {
        Step<R>& cur = ring[d];
        const int c = ct * 32 + lane;
        if (c < wch) {
          uint32_t wf[R][16];
          float sw[R][2];
#pragma unroll
          for (int i = 0; i < R; ++i) {
            const uint32_t words[4] = {cur.q[i].x, cur.q[i].y, cur.q[i].z, cur.q[i].w};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              wf[i][wd * 4 + 0] = e2m1x2_byte_to_f16x2<0>(words[wd]);
              wf[i][wd * 4 + 1] = e2m1x2_byte_to_f16x2<1>(words[wd]);
              wf[i][wd * 4 + 2] = e2m1x2_byte_to_f16x2<2>(words[wd]);
              wf[i][wd * 4 + 3] = e2m1x2_byte_to_f16x2<3>(words[wd]);
            }
            const uint32_t sh = e4m3x2_to_f16x2(cur.sc[i]);
            sw[i][0] = f16_lo_to_f32(sh);
            sw[i][1] = f16_hi_to_f32(sh);
          }
          const int ca = w0 + c;  // chunk index inside the staged split
#pragma unroll
          for (int r = 0; r < MT; ++r) {
            if (r < m) {
              const uint4* ap = reinterpret_cast<const uint4*>(Ah + (int64_t)r * (klen / 2) + ca * 16);
              const uint4 a0 = ap[0], a1 = ap[1], a2 = ap[2], a3 = ap[3];
              const uint32_t a[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                      a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
              const float2 sa = *reinterpret_cast<const float2*>(As + r * (klen / 16) + ca * 2);
#pragma unroll
              for (int i = 0; i < R; ++i) {
                const float p0 = dot16(a, wf[i]);
                const float p1 = dot16(a + 8, wf[i] + 8);
                acc[i][r] = fmaf(p0, sw[i][0] * sa.x, acc[i][r]);
                acc[i][r] = fmaf(p1, sw[i][1] * sa.y, acc[i][r]);
              }
            }
          }
        }
        // refill this ring slot with the step D ahead (predicated off past the end)
        load_step(cur, li, lt);
        if (++lt == T) { lt = 0; ++li; }

        if (ct == T - 1) {
          // row group ci is complete: reduce over lanes, then over the slot's KW warps
          const int64_t j0 = (rg_lo + slot + (int64_t)ci * NS) * R;
          const int par = ci & 1;
#pragma unroll
          for (int i = 0; i < R; ++i) {
#pragma unroll
            for (int r = 0; r < MT; ++r) {
              float v = acc[i][r];
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
              acc[i][r] = v;
            }
          }
          if (KW > 1) {
            float* mine = comb + ((par * NS + slot) * KW + kw) * (R * MT);
#pragma unroll
            for (int i = 0; i < R; ++i)
#pragma unroll
              for (int r = 0; r < MT; ++r)
                if (lane == ((i * MT + r) & 31)) mine[i * MT + r] = acc[i][r];
            named_barrier(1 + slot, KW * 32);
            if (kw == 0) {
              const float* all = comb + (par * NS + slot) * KW * (R * MT);
#pragma unroll
              for (int i = 0; i < R; ++i)
#pragma unroll
                for (int r = 0; r < MT; ++r) {
                  float v = acc[i][r];
                  for (int q = 1; q < KW; ++q) v += all[q * (R * MT) + i * MT + r];
                  acc[i][r] = v;
                }
            }
          }
          if (KW == 1 || kw == 0) {
#pragma unroll
            for (int i = 0; i < R; ++i) {
              const int64_t j = j0 + i;
#pragma unroll
              for (int r = 0; r < MT; ++r) {
                if (r < m && j < n && lane == ((i * MT + r) & 31)) {
                  if (S == 1)
                    p.out[(int64_t)r * n + j] = f32_to_bf16_rn(acc[i][r] * g);
                  else
                    p.partials[((int64_t)s * m + r) * n + j] = acc[i][r];
                }
              }
            }
          }
#pragma unroll
          for (int i = 0; i < R; ++i)
#pragma unroll
            for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
        }
        if (++ct == T) { ct = 0; ++ci; }
      }
    }
  }
}

namespace {

template <typename K>
int occupancy(K kern, int smem_bytes) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGemvThreads, smem_bytes) != cudaSuccess) {
    cudaGetLastError();
    return 1;
  }
  return occ > 0 ? occ : 1;
}

template <int MT, int R, int D>
int launch_one(const GemvArgs& a, cudaStream_t stream) {
  auto kern = gemv_nvfp4_kernel<MT, R, D>;
  // the opt-in shared memory limit is a per-device function attribute; raise it once
  static int configured[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_cuda_error("cudaGetDevice");
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return set_cuda_error("cudaFuncSetAttribute(gemv smem)");
    configured[dev] = 1;
  }
  // the grid is persistent: never ask for more CTAs than fit at once
  const int occ = occupancy(kern, a.smem_bytes);
  const int ctas = a.ctas_per_sm < occ ? a.ctas_per_sm : occ;
  int64_t gx = (int64_t)a.num_sms * ctas / a.splits;
  if (gx < 1) gx = 1;
  if (gx > a.grid_x) gx = a.grid_x;
  dim3 grid((unsigned)gx, (unsigned)a.splits);
  kern<<<grid, kGemvThreads, a.smem_bytes, stream>>>(a);
  if (cudaGetLastError() != cudaSuccess) return set_cuda_error("gemv kernel launch");
  return FI_OK;
}

template <int MT>
int launch_rows(const GemvArgs& a, cudaStream_t stream) {
  constexpr int D1 = MT <= 4 ? 4 : 2;
  switch (a.rows_per_warp) {
    case 1: return launch_one<MT, 1, D1>(a, stream);
    case 2: return launch_one<MT, 2, 2>(a, stream);
    case 4: return launch_one<MT, 4, 2>(a, stream);
    default: return set_error(FI_ERR_INVALID_ARG, "GEMV rows per warp must be 1, 2 or 4");
  }
}

}  // namespace

int launch_gemv(const GemvArgs& a, cudaStream_t stream) {
  if (a.m <= 1) return launch_rows<1>(a, stream);
  if (a.m <= 2) return launch_rows<2>(a, stream);
  if (a.m <= 4) return launch_rows<4>(a, stream);
  if (a.m <= 8) return launch_rows<8>(a, stream);
  if (a.m <= 16) return launch_rows<16>(a, stream);
  if (a.m <= 32) return launch_rows<32>(a, stream);
  return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV supports m <= %d", kGemvMaxM);
}

}  // namespace fi
