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

// Shared-memory image of the activations for one K split, laid out for conflict-free reads:
// chunk c (32 k) of row r lives in 4 16-byte quads at uint4 index
//     ((r * G + c / 32) * 4 + q) * 32 + c % 32,        G = ceil(nch / 32)
// so the 32 lanes of a warp, reading chunks 32t .. 32t+31, touch 512 contiguous bytes per
// quad. Values are f16 with one power-of-two scale per 16-block (fp32, linear As[r][2c+h]).
__device__ __forceinline__ void stage_activations(const uint16_t* __restrict__ A, int64_t k, int m,
                                                  int64_t kbase, int nch, uint4* Ah4, float* As) {
  const int G = (nch + 31) / 32;
  const int blocks_per_row = nch * 2;
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
    const int c = b >> 1, half = b & 1;
    uint4* dst = Ah4 + ((int64_t)(r * G + c / 32) * 4 + 2 * half) * 32 + (c % 32);
    dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
    dst[32] = make_uint4(h[4], h[5], h[6], h[7]);
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

// Occupancy target per instance (register budget per thread = 65536 / (256 * CTAs)): the
// small-m streaming instances keep three CTAs (24 warps) per SM resident.
template <int MT, int R>
constexpr int gemv_min_ctas() {
  return (MT * R <= 2) ? 3 : (MT * R <= 8 && MT <= 4) ? 2 : 1;
}

template <int MT, int R, int D>
__global__ void __launch_bounds__(kGemvThreads, gemv_min_ctas<MT, R>()) gemv_nvfp4_kernel(GemvArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // a PDL-launched successor (the split-K reduce, or the next op) may be scheduled now; it
  // waits for this grid's completion before touching what this grid writes
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
  const int G = (nch + 31) / 32;
  const int w0 = kw * nch / KW;
  const int wch = (kw + 1) * nch / KW - w0;
  // at least one (possibly empty) step per row group, so every warp of a slot meets the
  // slot's barrier once per row group even when its share of k is empty
  const int T = wch > 0 ? (wch + 31) / 32 : 1;
  const int climit = wch - lane;  // step t is live for this lane iff 32 * t < climit

  // row groups of this CTA, and of this warp's slot
  const int64_t RG = (n + R - 1) / R;
  const int64_t rg_lo = (int64_t)blockIdx.x * RG / gridDim.x;
  const int64_t rg_hi = (int64_t)(blockIdx.x + 1) * RG / gridDim.x;
  const int nrg = (rg_lo + slot < rg_hi) ? (int)((rg_hi - rg_lo - slot + NS - 1) / NS) : 0;
  const int F = nrg * T;

  uint4* Ah4 = reinterpret_cast<uint4*>(smem);
  float* As = reinterpret_cast<float*>(smem + (int64_t)m * G * 32 * 64);
  float* comb = As + m * nch * 2;  // [2][NS][KW][R*MT], used when KW > 1

  // load cursor: one pointer per row, advanced 32 chunks per step and jumped to the next
  // row group of this slot (NS * R rows further) after T steps
  const int64_t rs_q = k / 2, rs_s = k / 16;
  const uint8_t* lq[R];
  const uint8_t* ls[R];
  {
    const int64_t j0 = (rg_lo + slot) * R;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      lq[i] = p.Wq + (j0 + i) * rs_q + (c0 + w0 + lane) * 16;
      ls[i] = p.Ws + (j0 + i) * rs_s + (c0 + w0 + lane) * 2;
    }
  }
  const int64_t jump_q = (int64_t)NS * R * rs_q - (int64_t)T * 32 * 16;
  const int64_t jump_s = (int64_t)NS * R * rs_s - (int64_t)T * 32 * 2;
  // rows of the row group being fetched that exist (0 once past this warp's row groups)
  int64_t l_left = nrg > 0 ? n - (rg_lo + slot) * R : 0;
  int l_t = 0, l_g = 0;
  auto issue = [&](Step<R>& st) {
    const bool live = 32 * l_t < climit && l_g < nrg;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      if (live && i < l_left) {
        st.q[i] = ldg_stream_v4(lq[i]);
        st.sc[i] = ldg_stream_u16(ls[i]);
      } else {
        st.q[i] = make_uint4(0, 0, 0, 0);
        st.sc[i] = 0;
      }
      lq[i] += 32 * 16;
      ls[i] += 32 * 2;
    }
    if (++l_t == T) {
      l_t = 0;
      ++l_g;
      l_left -= (int64_t)NS * R;
#pragma unroll
      for (int i = 0; i < R; ++i) {
        lq[i] += jump_q;
        ls[i] += jump_s;
      }
    }
  };

  // prologue: put the first D steps of the weight stream in flight (weights are never written
  // by the preceding kernel), then wait for the producer of A and stage it
  Step<R> ring[D];
#pragma unroll
  for (int d = 0; d < D; ++d) issue(ring[d]);
  pdl_wait();
  stage_activations(p.A, k, m, c0 * kChunkK, nch, Ah4, As);
  __syncthreads();

  const float g = (S == 1) ? *p.gscale : 1.0f;
  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;

  // compute cursor: this lane's activation quads and block scales for step t
  const int ca0 = w0 + lane;
  const uint4* a_base = Ah4 + (int64_t)(ca0 / 32) * 4 * 32 + (ca0 % 32);
  const float2* s_base = reinterpret_cast<const float2*>(As) + ca0;
  int ct = 0, cg = 0;
  for (int f0 = 0; f0 < F; f0 += D) {
#pragma unroll
    for (int d = 0; d < D; ++d) {
      if (f0 + d < F) {
        Step<R>& cur = ring[d];
        if (MT == 1 && 32 * ct < climit) {
          // one activation row: decode each weight word straight into the FMAs (same
          // element order as below, fewer live registers)
          const uint4* ap = a_base + (int64_t)ct * 4 * 32;
          const uint4 a0 = ap[0], a1 = ap[32], a2 = ap[64], a3 = ap[96];
          const uint32_t a[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                  a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
          const float2 sa = s_base[ct * 32];
#pragma unroll
          for (int i = 0; i < R; ++i) {
            const uint32_t words[4] = {cur.q[i].x, cur.q[i].y, cur.q[i].z, cur.q[i].w};
            float pb[2] = {0.0f, 0.0f};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const uint32_t h0 = e2m1x2_byte_to_f16x2<0>(words[wd]);
              const uint32_t h1 = e2m1x2_byte_to_f16x2<1>(words[wd]);
              const uint32_t h2 = e2m1x2_byte_to_f16x2<2>(words[wd]);
              const uint32_t h3 = e2m1x2_byte_to_f16x2<3>(words[wd]);
              float& pp = pb[wd >> 1];
              pp = fma_lo_f16(a[wd * 4 + 0], h0, pp);
              pp = fma_hi_f16(a[wd * 4 + 0], h0, pp);
              pp = fma_lo_f16(a[wd * 4 + 1], h1, pp);
              pp = fma_hi_f16(a[wd * 4 + 1], h1, pp);
              pp = fma_lo_f16(a[wd * 4 + 2], h2, pp);
              pp = fma_hi_f16(a[wd * 4 + 2], h2, pp);
              pp = fma_lo_f16(a[wd * 4 + 3], h3, pp);
              pp = fma_hi_f16(a[wd * 4 + 3], h3, pp);
            }
            const uint32_t sh = e4m3x2_to_f16x2(cur.sc[i]);
            acc[i][0] = fmaf(pb[0], f16_lo_to_f32(sh) * sa.x, acc[i][0]);
            acc[i][0] = fmaf(pb[1], f16_hi_to_f32(sh) * sa.y, acc[i][0]);
          }
        } else if (MT > 1 && 32 * ct < climit) {
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
#pragma unroll
          for (int r = 0; r < MT; ++r) {
            if (r < m) {
              const uint4* ap = a_base + ((int64_t)r * G + ct) * 4 * 32;
              const uint4 a0 = ap[0], a1 = ap[32], a2 = ap[64], a3 = ap[96];
              const uint32_t a[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                      a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
              const float2 sa = s_base[r * nch + ct * 32];
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
        issue(cur);

        if (ct == T - 1) {
          // row group cg is complete: reduce over lanes, then over the slot's KW warps
          const int64_t j0 = (rg_lo + slot + (int64_t)cg * NS) * R;
          const int par = cg & 1;
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
        if (++ct == T) {
          ct = 0;
          ++cg;
        }
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)gx, (unsigned)a.splits);
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return set_cuda_error("gemv kernel launch");
  return FI_OK;
}

template <int MT>
int launch_rows(const GemvArgs& a, cudaStream_t stream) {
  constexpr int D1 = MT <= 4 ? 4 : 2;
  switch (a.rows_per_warp) {
    case 1: return launch_one<MT, 1, D1>(a, stream);
    case 2: return launch_one<MT, 2, 2>(a, stream);
    case 4:
      if constexpr (MT <= 16) return launch_one<MT, 4, 2>(a, stream);
      return set_error(FI_ERR_INVALID_ARG, "GEMV with 4 rows per warp supports m <= 16");
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
