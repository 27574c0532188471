// Streaming GEMV for bf16 activations x NVFP4 weights, m <= 32 (sm_100a).
//
// After the streaming GEMV of PR #4038 (Description, "What it does", and its GEMV commit
// messages: weights go from global memory straight to registers with many warps covering
// the latency, each output row is reduced across a warp with shuffles, and a later commit
// stages the activations in shared memory), re-designed for B200, where an m=1 GEMV has to
// keep ~100 KB of weights in flight per SM to run at HBM speed. Four pipelines share the
// activation staging, the work split and the per-chunk arithmetic, so for one K split S they
// give bitwise identical outputs:
//
//  * Stream pipeline (gemv_stream_kernel, the default): every warp streams its own rows with
//    per-thread cp.async into its own shared-memory ring; a lane copies exactly the cells it
//    computes and waits only for its own copies (cp.async.wait_group), so there is no wait
//    between threads. A straight-line fast path covers splits whose chunks are a multiple of
//    64 (k = 4096, 14336 at S = 1). The overlapped variant sizes the CTAs for half an SM but
//    launches one per SM, so the next call's CTAs are resident beside them, and prefetches
//    each warp's weights into L2 first.
//  * Register pipeline (gemv_reg_kernel): the pages' own design, weights straight to registers
//    with 16-byte loads, a ring of D chunk iterations in flight per warp.
//  * Ring pipeline (gemv_nvfp4_kernel): one producer warp per CTA streams whole rows with bulk
//    copies (cp.async.bulk, completion counted on an mbarrier) into an NST-stage ring; 16
//    consumer warps decode from it. Its waits are bounded (below); it also runs k = 65536 at
//    m = 1, whose activations do not fit the other pipelines' shared memory.
//  * Programmatic dependent launch. Weights are never written by the preceding kernel, so each
//    pipeline issues its first weight copies before the grid-dependency wait and stages the
//    activations after it.
//  * Work. Grid (G, S): blockIdx.y is the K split s; the warps of a split own balanced,
//    contiguous groups of weight rows (ring pipeline: CTAs own row ranges and warps take
//    stages in turn), so a row is always computed by one warp and the activations it loads
//    once per chunk serve all rows of its group.
//  * Arithmetic (fixed by k and S alone, hence bitwise identical for every m, pipeline, rows
//    per group, CTA shape and grid): A is staged as f16 with one power-of-two scale sf_a per
//    16-block that puts the block maximum in [2^9, 2^10) (exact for every element within 2^26
//    of its block maximum); codes are decoded by cvt.rn.f16x2.e2m1x2 (exact). Per 16-block, the
//    16 products (each exact in fp32) are summed in fp32 by the mixed-precision fma.rn.f32.f16,
//    the even and the odd elements in two chains in element order, t = even + odd, and
//    acc = fma(t, sw * sf_a, acc) with sw the block's E4M3 scale. Lane L takes chunks L, L+32, L+64, ... of the split; the lanes combine through a
//    fixed xor butterfly (all lanes end with the same bits). S == 1 writes bf16_rn(acc *
//    gscale); S > 1 writes fp32 partials for the reduce kernel.
//  * Bounded waits (ring pipeline). Every mbarrier wait gives up after a time limit
//    (%globaltimer): it sets a device error flag and a CTA-wide abort flag, the CTA finishes
//    its control flow without computing, and the producer waits (bounded) for the copies it
//    issued before exiting.
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "sync.cuh"

namespace fi {

// Sticky device error word: bit 0 = a consumer wait timed out, bit 1 = a producer wait timed
// out, bit 2 = the producer's final drain timed out (ring pipeline; the MMA path uses bits 0-4
// likewise). Read and cleared by gemv_read_error().
__device__ unsigned int g_gemv_error = 0;

namespace {

// Wait for phase `parity` of `bar` (bounded; see sync.cuh), recording timeouts in g_gemv_error.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t timeout_ns, unsigned err_bit) {
  return fi::mbar_wait_bounded(bar, parity, abort_flag, timeout_ns, &g_gemv_error, err_bit);
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ void stage_block(const uint4 v0, const uint4 v1, int r, int b, int GA, int blocks_per_row,
                                            uint4* Ah4, float* As) {
  const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  // largest magnitude of the block: with the sign bits cleared, bf16 bit patterns order as
  // unsigned 16-bit integers, two per packed max
  uint32_t mx = w[0] & 0x7FFF7FFFu;
#pragma unroll
  for (int i = 1; i < 8; ++i) asm("max.u16x2 %0, %0, %1;" : "+r"(mx) : "r"(w[i] & 0x7FFF7FFFu));
  const uint32_t e = max((mx >> 7) & 0xFFu, mx >> 23);
  int sh = 136 - (int)e;  // biased exponent E -> block maximum in [2^9, 2^10)
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
  uint4* dst = Ah4 + ((int64_t)(r * GA + c / 32) * 4 + 2 * half) * 32 + (c % 32);
  dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
  dst[32] = make_uint4(h[4], h[5], h[6], h[7]);
  As[r * blocks_per_row + b] = down;
}

// Stage A[0:m, kbase : kbase + 32*nch] for the consumer warps. Layout for conflict-free reads:
// chunk c (32 k) of row r is 4 16-byte quads at uint4 index ((r * GA + c / 32) * 4 + q) * 32 +
// c % 32 (GA = ceil(nch / 32)), so a warp reading 32 consecutive chunks touches 512
// contiguous bytes per quad. Values are f16 scaled by a power of two per 16-block that puts
// the block maximum in [2^9, 2^10); As[r][b] holds the inverse scale. A thread loads up to four
// of its blocks before converting any, so their global-memory latencies overlap.
template <int U = 4>
__device__ __forceinline__ void stage_activations(const uint16_t* __restrict__ A, int64_t k, int m,
                                                  int64_t kbase, int nch, uint4* Ah4, float* As, int tid,
                                                  int nthreads) {
  const int GA = (nch + 31) / 32;
  const int blocks_per_row = nch * 2;
  const int nblk = m * blocks_per_row;
  for (int b0 = tid; b0 < nblk; b0 += U * nthreads) {
    uint4 v[U][2];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int bi = b0 + u * nthreads;
      if (bi < nblk) {
        const int r = bi / blocks_per_row;
        const uint16_t* src = A + (int64_t)r * k + kbase + (int64_t)(bi - r * blocks_per_row) * 16;
        v[u][0] = ldg_v4(src);
        v[u][1] = ldg_v4(src + 8);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int bi = b0 + u * nthreads;
      if (bi < nblk) {
        const int r = bi / blocks_per_row;
        stage_block(v[u][0], v[u][1], r, bi - r * blocks_per_row, GA, blocks_per_row, Ah4, As);
      }
    }
  }
}

// The 16 products of one 16-block summed in fp32: a and w hold the block's 8 f16 pairs
// (element 2j in the low half of word j). Each product of two f16 values is exact in fp32; the
// mixed-precision fma.rn.f32.f16 adds it to a running fp32 sum with one round-to-nearest-even.
// The even elements and the odd elements are summed in two chains, each in element order
// (two chains halve the dependent-latency path), and the block's sum is even + odd.
__device__ __forceinline__ float block_dot(const uint32_t* a, const uint32_t* w) {
  float te, to;
  asm("{\n .reg .b16 al, ah, wl, wh;\n mov.b32 {al, ah}, %2;\n mov.b32 {wl, wh}, %3;\n"
      " fma.rn.f32.f16 %0, al, wl, 0f00000000;\n fma.rn.f32.f16 %1, ah, wh, 0f00000000;\n}"
      : "=f"(te), "=f"(to)
      : "r"(a[0]), "r"(w[0]));
#pragma unroll
  for (int i = 1; i < 8; ++i)
    asm("{\n .reg .b16 al, ah, wl, wh;\n mov.b32 {al, ah}, %2;\n mov.b32 {wl, wh}, %3;\n"
        " fma.rn.f32.f16 %0, al, wl, %0;\n fma.rn.f32.f16 %1, ah, wh, %1;\n}"
        : "+f"(te), "+f"(to)
        : "r"(a[i]), "r"(w[i]));
  return __fadd_rn(te, to);
}

// One 32-k chunk of one weight row against one activation row: av the chunk's 16 staged f16
// pairs, sa its two activation block scales (powers of two), wf the decoded codes, sh the two
// E4M3 block scales as f16x2. Per block, acc = fma(t, sw * sa, acc) with t the block's fp32 dot
// product (sw * sa is exact: sa is a power of two). Every pipeline calls this, so their bits
// agree.
__device__ __forceinline__ float chunk_acc(const uint32_t (&av)[16], float2 sa, const uint32_t (&wf)[16], uint32_t sh,
                                           float acc) {
  const float t0 = block_dot(av, wf);
  const float t1 = block_dot(av + 8, wf + 8);
  acc = fmaf(t0, __fmul_rn(f16_lo_to_f32(sh), sa.x), acc);
  return fmaf(t1, __fmul_rn(f16_hi_to_f32(sh), sa.y), acc);
}

// Decode one 16-byte code quad (32 E2M1 codes) into 16 f16x2 words.
__device__ __forceinline__ void decode32(const uint4 q, uint32_t* wf) {
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    wf[wd * 4 + 0] = e2m1x2_byte_to_f16x2<0>(words[wd]);
    wf[wd * 4 + 1] = e2m1x2_byte_to_f16x2<1>(words[wd]);
    wf[wd * 4 + 2] = e2m1x2_byte_to_f16x2<2>(words[wd]);
    wf[wd * 4 + 3] = e2m1x2_byte_to_f16x2<3>(words[wd]);
  }
}

// NR weight rows of a ring stage against MT activation rows: lane L takes chunks L, L+32, ...
// of the split; the activations loaded for a chunk serve all NR rows. Row i's codes start at
// shared address code0 + i * cstride and its E4M3 scales at sbase + i * sstride + ((off0 + i *
// doff) & 15) (the scales sit at their source offset within 16-byte aligned copies); a_s / as_s
// are the shared addresses of the staged activations and their scales; acc[i][r] accumulates
// in fp32.
template <int MT, int NR>
__device__ __forceinline__ void stage_rows(uint32_t code0, int cstride, uint32_t sbase, int sstride, uint32_t off0,
                                           uint32_t doff, uint32_t a_s, uint32_t as_s, int m, int nch, int GA,
                                           int lane, float (&acc)[NR][MT]) {
  const uint32_t a_row = (uint32_t)GA * 4 * 32 * 16;  // bytes per activation row
  const uint32_t as_row = (uint32_t)nch * 8;
  uint32_t scale0[NR];
#pragma unroll
  for (int i = 0; i < NR; ++i) scale0[i] = sbase + (uint32_t)(i * sstride) + ((off0 + (uint32_t)i * doff) & 15u);
  for (int c = lane; c < nch; c += 32) {
    const uint32_t ap = a_s + (uint32_t)(((c >> 5) * 4 * 32 + (c & 31)) * 16);
    const uint32_t sp = as_s + (uint32_t)c * 8;
    if (MT == 1) {
      const uint4 a0 = lds_v4(ap), a1 = lds_v4(ap + 512), a2 = lds_v4(ap + 1024), a3 = lds_v4(ap + 1536);
      const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                               a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
      const float2 sa = lds_f2(sp);
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const uint4 cq = lds_v4(code0 + (uint32_t)(i * cstride + c * 16));
        const uint32_t sc = lds_u16(scale0[i] + (uint32_t)(c * 2));
        uint32_t wf[16];
        decode32(cq, wf);
        acc[i][0] = chunk_acc(av, sa, wf, e4m3x2_to_f16x2(sc), acc[i][0]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        const uint4 cq = lds_v4(code0 + (uint32_t)(i * cstride + c * 16));
        const uint32_t sc = lds_u16(scale0[i] + (uint32_t)(c * 2));
        uint32_t wf[16];
        decode32(cq, wf);
        const uint32_t sh = e4m3x2_to_f16x2(sc);
#pragma unroll
        for (int r = 0; r < MT; ++r) {
          if (r < m) {
            const uint32_t apr = ap + (uint32_t)r * a_row;
            const uint4 a0 = lds_v4(apr), a1 = lds_v4(apr + 512), a2 = lds_v4(apr + 1024), a3 = lds_v4(apr + 1536);
            const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                     a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
            acc[i][r] = chunk_acc(av, lds_f2(sp + (uint32_t)r * as_row), wf, sh, acc[i][r]);
          }
        }
      }
    }
  }
}

// Combine the lanes of acc (fixed xor butterfly: every lane ends with the same bits) and
// write rows j0 .. j0+rows-1: round(acc * g) to the output type (bf16, or f16) when S == 1,
// else the fp32 partial of split s.
template <int MT, int NR>
__device__ __forceinline__ void finish_rows(float (&acc)[NR][MT], const GemvArgs& p, int64_t j0, int rows, int m,
                                            int S, int s, float g, int lane, bool write) {
#pragma unroll
  for (int i = 0; i < NR; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r) {
      float v = acc[i][r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[i][r] = v;
    }
  if (!write) return;
#pragma unroll
  for (int i = 0; i < NR; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r)
      if (i < rows && r < m && lane == ((i * MT + r) & 31)) {
        const int64_t j = j0 + i;
        if (S == 1)
          p.out[(int64_t)r * p.n + j] = f32_to_out(acc[i][r] * g, p.out_f16 != 0);
        else
          p.partials[((int64_t)s * m + r) * p.n + j] = acc[i][r];
      }
}

}  // namespace

template <int MT, int RS>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_nvfp4_kernel(GemvArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ volatile int abort_flag;

  constexpr int NC = kGemvConsumerWarps;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const bool producer = warp == NC;
  const int m = (int)p.m;
  const int64_t n = p.n, k = p.k;
  const int S = p.splits;
  const int s = blockIdx.y;
  const int NST = p.stages;

  // K range of this split, in 32-k chunks
  const int64_t C = k / kChunkK;
  const int64_t c0 = (int64_t)s * C / S;
  const int nch = (int)((int64_t)(s + 1) * C / S - c0);

  // rows of this CTA, RS per ring stage
  const int64_t r_lo = (int64_t)blockIdx.x * n / gridDim.x;
  const int64_t r_hi = (int64_t)(blockIdx.x + 1) * n / gridDim.x;
  const int64_t Q = (r_hi - r_lo + RS - 1) / RS;  // ring stages of this CTA

  // shared memory carve-up (offsets computed on the host, 128-byte aligned)
  uint4* Ah4 = reinterpret_cast<uint4*>(smem);
  float* As = reinterpret_cast<float*>(smem + p.off_as);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* empty = full + NST;
  uint8_t* ring = smem + p.off_ring;
  const uint32_t ring_s = smem_addr(ring), a_s = smem_addr(Ah4), as_s = smem_addr(As);
  const int codes_stride = nch * 16;  // bytes per row of codes in a stage (rows are adjacent)
  const int scales_off = RS * codes_stride;
  // S == 1: one contiguous superset of the rows' scales; S > 1: one superset per row
  const int scales_stride = (int)gemv_scales_stride(nch);

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NC);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // a PDL-launched successor may be scheduled now; it waits for this grid's completion
  pdl_launch_dependents();

  const int64_t rs_q = k / 2, rs_s = k / 16;
  const int64_t scale_bytes_total = n * rs_s;

  if (producer) {
    // ------------------------------------------------------------------ producer warp
    if (lane == 0 && !p.debug_stall) {
      int64_t issued = 0;
      for (int64_t q = 0; q < Q; ++q) {
        const int slot = (int)(q % NST);
        if (q >= NST && !mbar_wait_bounded(&empty[slot], (uint32_t)((q / NST - 1) & 1), &abort_flag,
                                           p.timeout_ns, 2u))
          break;
        const int64_t j0 = r_lo + q * RS;
        const int rows = (int)min((int64_t)RS, r_hi - j0);
        uint8_t* stage = ring + (int64_t)slot * p.stage_bytes;
        uint8_t* sdst = stage + scales_off;
        if (S == 1) {
          const int64_t st = j0 * rs_s, en = (j0 + rows) * rs_s;
          const int64_t al = st & ~(int64_t)15, ae = (en + 15) & ~(int64_t)15;
          uint32_t bytes = (uint32_t)(rows * rs_q);
          const bool plain = ae > scale_bytes_total;
          if (plain) {
            for (int64_t b = al; b < en; ++b) sdst[b - al] = p.Ws[b];
          } else {
            bytes += (uint32_t)(ae - al);
          }
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_g2s(stage, p.Wq + j0 * rs_q, (uint32_t)(rows * rs_q), &full[slot]);
          if (!plain) bulk_g2s(sdst, p.Ws + al, (uint32_t)(ae - al), &full[slot]);
        } else {
          uint32_t bytes = 0;
          for (int r = 0; r < rows; ++r) {
            const int64_t st = (j0 + r) * rs_s + c0 * 2;
            const int64_t al = st & ~(int64_t)15, ae = (st + (int64_t)nch * 2 + 15) & ~(int64_t)15;
            if (ae > scale_bytes_total) {
              uint8_t* dst = sdst + r * scales_stride;
              for (int64_t b = al; b < st + (int64_t)nch * 2; ++b) dst[b - al] = p.Ws[b];
            } else {
              bytes += (uint32_t)(ae - al);
            }
            bytes += (uint32_t)nch * 16;
          }
          mbar_arrive_expect_tx(&full[slot], bytes);
          for (int r = 0; r < rows; ++r) {
            const int64_t j = j0 + r;
            bulk_g2s(stage + r * codes_stride, p.Wq + j * rs_q + c0 * 16, (uint32_t)nch * 16, &full[slot]);
            const int64_t st = j * rs_s + c0 * 2;
            const int64_t al = st & ~(int64_t)15, ae = (st + (int64_t)nch * 2 + 15) & ~(int64_t)15;
            if (ae <= scale_bytes_total)
              bulk_g2s(sdst + r * scales_stride, p.Ws + al, (uint32_t)(ae - al), &full[slot]);
          }
        }
        issued = q + 1;
      }
      // drain: every copy this CTA issued must have landed before the CTA exits
      const int64_t first = issued > NST ? issued - NST : 0;
      for (int64_t q = first; q < issued; ++q)
        mbar_wait_bounded(&full[q % NST], (uint32_t)((q / NST) & 1), &abort_flag, p.timeout_ns, 4u);
    }
    return;
  }

  // -------------------------------------------------------------------- consumer warps
  pdl_wait();
  const int GA = (nch + 31) / 32;
  stage_activations(p.A, k, m, c0 * kChunkK, nch, Ah4, As, tid, NC * 32);
  named_barrier(1, NC * 32);
  const float g = (S == 1) ? *p.gscale : 1.0f;

  // Every consumer warp passes every stage in order and releases it (the empty barrier counts
  // all NC warps), but only warp q % NC computes stage q. A slot therefore never runs more than
  // one phase ahead of any warp waiting on it, which the parity-based waits require.
  for (int64_t q = 0; q < Q; ++q) {
    const int slot = (int)(q % NST);
    const bool ok = mbar_wait_bounded(&full[slot], (uint32_t)((q / NST) & 1), &abort_flag, p.timeout_ns, 1u);
    if (q % NC != warp) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
      continue;
    }
    const int64_t j0 = r_lo + q * RS;
    const int rows = (int)min((int64_t)RS, r_hi - j0);
    const uint32_t stage_s = ring_s + (uint32_t)slot * (uint32_t)p.stage_bytes;
    // row i's scales: S == 1 copies the rows' contiguous scales as one aligned superset (stride
    // k/16); S > 1 copies an aligned superset per row (stride scales_stride). Either way row i's
    // scales sit at offset ((j0 + i) * k/16 + c0 * 2) & 15 within its part of the stage.
    const uint32_t sbase = stage_s + (uint32_t)scales_off;
    const int sstride = S == 1 ? (int)rs_s : scales_stride;
    const uint32_t off0 = (uint32_t)((j0 * rs_s + c0 * 2) & 15);
    const uint32_t doff = S == 1 ? 0u : (uint32_t)(rs_s & 15);
    const bool write = ok && !abort_flag;
    if (rows == RS) {
      float acc[RS][MT];
#pragma unroll
      for (int i = 0; i < RS; ++i)
#pragma unroll
        for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
      if (ok)
        stage_rows<MT, RS>(stage_s, codes_stride, sbase, sstride, off0, doff, a_s, as_s, m, nch, GA, lane, acc);
      finish_rows<MT, RS>(acc, p, j0, RS, m, S, s, g, lane, write);
    } else {
      // the CTA's last, partial stage: one row at a time
      for (int i = 0; i < rows; ++i) {
        float acc[1][MT];
#pragma unroll
        for (int r = 0; r < MT; ++r) acc[0][r] = 0.0f;
        if (ok)
          stage_rows<MT, 1>(stage_s + (uint32_t)(i * codes_stride), codes_stride,
                            sbase + (uint32_t)(i * sstride) + ((off0 + (uint32_t)i * doff) & 15u), 0, 0u, 0u,
                            a_s, as_s, m, nch, GA, lane, acc);
        finish_rows<MT, 1>(acc, p, j0 + i, 1, m, S, s, g, lane, write);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }
}

// ============================================================ per-warp async-copy pipeline
//
// The second GEMV pipeline. Every warp streams its own weight rows with per-thread
// asynchronous copies (cp.async, the load/store-unit path of ordinary loads) into its own ring
// of NS shared-memory slots, and computes from there. There is no producer warp and no barrier
// between warps: lane L copies exactly the 16-byte code cells (and the scale bytes) of the
// chunks it computes, so each thread waits only for its own copies (cp.async.wait_group, a
// hardware wait that costs no issue slots and cannot outlive the copies). A slot holds R
// weight rows at one chunk iteration: row i's cell of lane L at i*512 + L*16, and the 4-byte
// aligned word holding the lane's two E4M3 scale bytes at R*512 + i*128 + L*4.
//
// The work item of a warp is (row group, chunk iteration t): chunk c = 32 t + L of the split
// for R consecutive rows. Items run in order, each lane taking chunks L, L+32, ... of every
// row in increasing order with the same per-chunk arithmetic as the other pipelines, so all
// of them give bitwise identical results for the same S.
//
// A CTA is 8 warps and at most about half of an SM's shared memory and registers, so the
// CTAs of the next programmatically dependent launch can become resident beside it and start
// their weight stream while this one finishes.

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Hint the L2 to fetch [p, p + bytes) from DRAM (bulk prefetch: no destination, no completion;
// p and bytes multiples of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Lane 0 of a warp asks the L2 to prefetch the warp's whole weight range (codes and scales of
// rows r_lo .. r_hi-1 over the split): the copies into shared memory then hit in L2. Called
// before the grid-dependency wait, so the DRAM stream runs during the wait and the preceding
// kernel's tail. Ranges are trimmed to whole 16-byte pieces inside the tensors.
__device__ __forceinline__ void prefetch_rows_l2(const GemvArgs& p, int64_t r_lo, int64_t r_hi, int64_t c0, int nch) {
  const int64_t rs_q = p.k / 2, rs_s = p.k / 16;
  auto range = [](const uint8_t* base, int64_t lo, int64_t hi) {
    lo = (lo + 15) & ~(int64_t)15;
    hi &= ~(int64_t)15;
    for (int64_t a = lo; a < hi; a += 32768) prefetch_l2_bulk(base + a, (uint32_t)min((int64_t)32768, hi - a));
  };
  if (p.splits == 1) {  // the warp's rows are one contiguous range of each tensor
    range(p.Wq, r_lo * rs_q, r_hi * rs_q);
    range(p.Ws, r_lo * rs_s, r_hi * rs_s);
  } else {
    for (int64_t j = r_lo; j < r_hi; ++j) {
      range(p.Wq, j * rs_q + c0 * 16, j * rs_q + (c0 + nch) * 16);
      range(p.Ws, j * rs_s + c0 * 2, j * rs_s + (c0 + nch) * 2);
    }
  }
}

__device__ __forceinline__ void sts_u16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"((unsigned short)v) : "memory");
}

// One chunk of the split for R weight rows against MT activation rows. code_s is the lane's
// cell of row 0 in the slot, scale_s + soff[i] the address of the lane's two scale bytes of row
// i (rows 128 bytes apart); ap / sp are the lane's staged activations of the chunk (4 quads 512
// bytes apart) and their two block scales, for activation row 0 (rows a_row / as_row apart).
// Every weight row is computed without a branch, so the compiler can interleave the rows'
// independent chains; rows of a partial group compute on stale cells and are never written.
template <int MT, int R, int CS = 512, int SS = 128>
__device__ __forceinline__ void item_rows(uint32_t code_s, uint32_t scale_s, const uint32_t (&soff)[R], uint32_t ap,
                                          uint32_t sp, uint32_t a_row, uint32_t as_row, int m,
                                          float (&acc)[R][MT]) {
  if (MT == 1) {
    const uint4 a0 = lds_v4(ap), a1 = lds_v4(ap + 512), a2 = lds_v4(ap + 1024), a3 = lds_v4(ap + 1536);
    const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                             a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
    const float2 sa = lds_f2(sp);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const uint4 cq = lds_v4(code_s + (uint32_t)(i * CS));
      const uint32_t sc = lds_u16(scale_s + (uint32_t)(i * SS) + soff[i]);
      uint32_t wf[16];
      decode32(cq, wf);
      acc[i][0] = chunk_acc(av, sa, wf, e4m3x2_to_f16x2(sc), acc[i][0]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const uint4 cq = lds_v4(code_s + (uint32_t)(i * CS));
      const uint32_t sc = lds_u16(scale_s + (uint32_t)(i * SS) + soff[i]);
      uint32_t wf[16];
      decode32(cq, wf);
      const uint32_t sh = e4m3x2_to_f16x2(sc);
#pragma unroll
      for (int r = 0; r < MT; ++r) {
        if (r < m) {
          const uint32_t apr = ap + (uint32_t)r * a_row;
          const uint4 a0 = lds_v4(apr), a1 = lds_v4(apr + 512), a2 = lds_v4(apr + 1024), a3 = lds_v4(apr + 1536);
          const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                   a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
          acc[i][r] = chunk_acc(av, lds_f2(sp + (uint32_t)r * as_row), wf, sh, acc[i][r]);
        }
      }
    }
  }
}

template <int MT, int R, int NS>
__global__ void __launch_bounds__(kStreamMaxThreads, 1) gemv_stream_kernel(GemvArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TI = kStreamIters;  // chunk iterations per work item
  constexpr uint32_t kSlot = (uint32_t)(TI * R) * kStreamCellBytes;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int NW = (int)(blockDim.x >> 5);
  const int m = (int)p.m;
  const int64_t n = p.n, k = p.k;
  const int S = p.splits;
  const int s = blockIdx.y;

  // K range of this split, in 32-k chunks; chunk iterations of a row; items of a row group
  const int64_t C = k / kChunkK;
  const int64_t c0 = (int64_t)s * C / S;
  const int nch = (int)((int64_t)(s + 1) * C / S - c0);
  const int T = (nch + 31) / 32;
  const int TT = (T + TI - 1) / TI;

  // rows of this warp: whole groups of R rows, balanced over all warps of the split (only the
  // matrix's last group can be partial)
  const int64_t GW = (int64_t)gridDim.x * NW;
  const int64_t gw = (int64_t)blockIdx.x * NW + warp;
  const int64_t ngr = (n + R - 1) / R;
  const int64_t g_lo = gw * ngr / GW, g_hi = (gw + 1) * ngr / GW;
  const int64_t r_lo = g_lo * R, r_hi = min(n, g_hi * R);
  const int Q = (int)(g_hi - g_lo) * TT;  // items of this warp

  const int64_t rs_q = k / 2, rs_s = k / 16;
  const uint8_t* const ws_end = p.Ws + n * rs_s;
  const uint32_t a_s = smem_addr(smem), as_s = smem_addr(smem + p.off_as);
  // this warp's ring: NS slots; in a slot, the cell of (iteration ti, row i) for lane L at
  // (ti*R + i)*512 + L*16, and the scale cell of (ti, i) at TI*R*512 + (ti*R + i)*128
  const uint32_t ring = smem_addr(smem + p.off_ring) + (uint32_t)warp * NS * kSlot;
  const uint32_t my_code = ring + (uint32_t)lane * 16;
  const uint32_t scale_area = ring + (uint32_t)(TI * R) * 512;
  const int64_t lane_k = (c0 + lane) * 2;  // the lane's first scale byte within a row's split
  // Scale copies. s16 (k % 256 == 0 and every split starts and ends on 8 chunks, so a row's
  // scales of one iteration are four aligned 16-byte pieces): lane L < 4*TI*R copies piece pc
  // of (iteration ti_L, row i_L) of every item into the first 64 bytes of that cell, and lane
  // L's two bytes of a cell sit at 2L. Otherwise every lane copies the 4-byte aligned word
  // holding its two bytes to cell + 4L.
  const bool s16 = p.scale16 != 0;
  const int pc = lane & 3, i_l = (lane >> 2) % R, ti_l = lane / (4 * R);
  const bool s_lane = lane < 4 * TI * R;
  const uint32_t my_scale = scale_area + (s16 ? 0u : (uint32_t)lane * 4);
  const uint32_t my_s16 = scale_area + (uint32_t)((ti_l * R + i_l) * 128 + pc * 16);

  pdl_launch_dependents();
  if (p.prefetch_l2 && lane == 0 && r_lo < r_hi) prefetch_rows_l2(p, r_lo, r_hi, c0, nch);

  // compute cursor constants: the lane's staged activations of chunk 32 t + L sit at a_s +
  // t*2048 + L*16 and their block scales at as_s + t*256 + L*8
  const int GA = (nch + 31) / 32;
  const uint32_t a_row = (uint32_t)GA * 2048, as_row = (uint32_t)nch * 8;
  const uint32_t a_lane = a_s + (uint32_t)lane * 16, as_lane = as_s + (uint32_t)lane * 8;

  // ---- Fast path (16-byte scale pieces and whole items: the split's chunks are a multiple of
  // 32*TI, which the serving shapes meet). Every item has every lane and iteration, so the loop
  // is straight-line: copies are predicated per row (only the matrix's last group can be
  // partial), and the issue cursor moves by one of two constant strides (next item of the
  // row group, or the first item of the next group). (Per-warp tensor copies of whole items
  // cost fewer instructions but measured slower on B200: 9.5 against 9.1 us at 4096 x 14336.)
  if (s16 && nch % (32 * TI) == 0) {
    const uint8_t* qi[R];
#pragma unroll
    for (int i = 0; i < R; ++i) qi[i] = p.Wq + (r_lo + i) * rs_q + (c0 + lane) * 16;
    const uint8_t* si = p.Ws + (r_lo + i_l) * rs_s + c0 * 2 + ti_l * 64 + pc * 16;
    const int64_t dq = (int64_t)R * rs_q - (int64_t)(TT - 1) * TI * 512;  // to the next group
    const int64_t ds = (int64_t)R * rs_s - (int64_t)(TT - 1) * TI * 64;
    int64_t j0_i = r_lo;
    int itt_i = 0, iq = 0;
    auto issue_fast = [&](uint32_t uo) {
      const bool live = iq < Q;
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const bool rv = live && j0_i + i < r_hi;
#pragma unroll
        for (int ti = 0; ti < TI; ++ti)
          if (rv) cp_async_16(my_code + uo + (uint32_t)((ti * R + i) * 512), qi[i] + ti * 512);
      }
      if (s_lane && live && j0_i + i_l < r_hi) cp_async_16(my_s16 + uo, si);
      cp_async_commit();
      const bool wrap = itt_i == TT - 1;
      itt_i = wrap ? 0 : itt_i + 1;
#pragma unroll
      for (int i = 0; i < R; ++i) qi[i] += wrap ? dq : (int64_t)TI * 512;
      si += wrap ? ds : (int64_t)TI * 64;
      j0_i += wrap ? R : 0;
      ++iq;
    };
#pragma unroll
    for (int u = 0; u < NS; ++u) issue_fast((uint32_t)u * kSlot);

    pdl_wait();
    stage_activations(p.A, k, m, c0 * kChunkK, nch, reinterpret_cast<uint4*>(smem),
                      reinterpret_cast<float*>(smem + p.off_as), tid, (int)blockDim.x);
    __syncthreads();
    const float g = (S == 1) ? *p.gscale : 1.0f;

    float acc[R][MT];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
    const uint32_t zoff[R] = {};  // the lane's scale bytes sit at cell + 2L for every row
    const uint32_t sbase = scale_area + (uint32_t)lane * 2;
    int64_t j0 = r_lo;
    int ctt = 0;
    uint32_t uo = 0, ac = a_lane, asc = as_lane;
    for (int q_ = 0; q_ < Q; ++q_) {
      cp_async_wait<NS - 1>();  // this lane's copies of item q_ have landed
#pragma unroll
      for (int ti = 0; ti < TI; ++ti)
        item_rows<MT, R>(my_code + uo + (uint32_t)(ti * R * 512), sbase + uo + (uint32_t)(ti * R * 128), zoff,
                         ac + (uint32_t)ti * 2048, asc + (uint32_t)ti * 256, a_row, as_row, m, acc);
      issue_fast(uo);  // refill the slot just read with item q_ + NS
      ac += TI * 2048;
      asc += TI * 256;
      if (++ctt == TT) {
        finish_rows<MT, R>(acc, p, j0, (int)min((int64_t)R, r_hi - j0), m, S, s, g, lane, true);
#pragma unroll
        for (int i = 0; i < R; ++i)
#pragma unroll
          for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
        ctt = 0;
        ac = a_lane;
        asc = as_lane;
        j0 += R;
      }
      uo = (uo == (uint32_t)(NS - 1) * kSlot) ? 0u : uo + kSlot;
    }
    cp_async_wait<0>();
    return;
  }

  // ---- General path (any k, any split)

  // ---- issue cursor: item iq = (group ig, item itt of the row group). Row i's code pointer
  // q[i] (this lane's cell at the item's first iteration) advances by TI*512 bytes per item;
  // the scale pointer sp (s16: this lane's piece; else the 4-byte word of row 0, row i at
  // sdel[i] beyond it) by TI*64.
  int ig = 0, itt = 0, iq = 0;
  const uint8_t* q[R];
  const uint8_t* sp = nullptr;
  uint32_t sdel[R];
  int irows = 0;
  bool iedge = false;  // the group holds the tensor's last scale pair and its size is 2 mod 4
  auto issue_group = [&]() {
    const int64_t j0 = r_lo + (int64_t)ig * R;
    irows = (int)max((int64_t)0, min((int64_t)R, r_hi - j0));
#pragma unroll
    for (int i = 0; i < R; ++i) q[i] = p.Wq + (j0 + (i < irows ? i : 0)) * rs_q + (c0 + lane) * 16;
    if (s16) {
      sp = p.Ws + (j0 + (i_l < irows ? i_l : 0)) * rs_s + c0 * 2 + ti_l * 64 + pc * 16;
    } else {
      const int64_t x0 = j0 * rs_s + lane_k;
      sp = p.Ws + (x0 & ~(int64_t)3);
#pragma unroll
      for (int i = 0; i < R; ++i) sdel[i] = (uint32_t)(((x0 + i * rs_s) & ~(int64_t)3) - (x0 & ~(int64_t)3));
      iedge = (n * rs_s) % 4 != 0 && j0 + irows >= n;
    }
  };
  // copy item iq into the slot at byte offset uo; always commits one group (empty past the
  // warp's last item) so that wait_group counts stay uniform
  auto issue = [&](uint32_t uo) {
    if (iq < Q) {
      const int t0 = itt * TI;
      if (irows == R && (t0 + TI) * 32 <= nch) {  // warp-uniform: no row or lane is cut
#pragma unroll
        for (int ti = 0; ti < TI; ++ti)
#pragma unroll
          for (int i = 0; i < R; ++i) cp_async_16(my_code + uo + (uint32_t)((ti * R + i) * 512), q[i] + ti * 512);
        if (s16 && s_lane) cp_async_16(my_s16 + uo, sp);
      } else {
#pragma unroll
        for (int ti = 0; ti < TI; ++ti)
          if ((t0 + ti) * 32 + lane < nch) {
#pragma unroll
            for (int i = 0; i < R; ++i)
              if (i < irows) cp_async_16(my_code + uo + (uint32_t)((ti * R + i) * 512), q[i] + ti * 512);
          }
        if (s16 && s_lane && i_l < irows && (t0 + ti_l) * 32 + pc * 8 < nch) cp_async_16(my_s16 + uo, sp);
      }
      if (!s16) {
#pragma unroll
        for (int ti = 0; ti < TI; ++ti) {
          if ((t0 + ti) * 32 + lane < nch) {
            const uint32_t sdst = my_scale + uo + (uint32_t)(ti * R * 128);
#pragma unroll
            for (int i = 0; i < R; ++i) {
              if (i < irows) {
                const uint8_t* w = sp + sdel[i] + ti * 64;
                if (!iedge || w + 4 <= ws_end) {
                  cp_async_4(sdst + (uint32_t)(i * 128), w);
                } else {  // the tensor's last scale pair when its size is 2 mod 4: plain load
                  const uint32_t off = (uint32_t)(((r_lo + (int64_t)ig * R + i) * rs_s + lane_k) & 2);
                  sts_u16(sdst + (uint32_t)(i * 128) + off, ldg_stream_u16(w + off));
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < R; ++i) q[i] += TI * 512;
      sp += TI * 64;
      ++iq;
      if (++itt == TT) {
        itt = 0;
        ++ig;
        issue_group();
      }
    }
    cp_async_commit();
  };

  // prologue: the first NS items (weights only: they do not depend on the preceding kernel)
  issue_group();
#pragma unroll
  for (int u = 0; u < NS; ++u) issue((uint32_t)u * kSlot);

  pdl_wait();
  stage_activations(p.A, k, m, c0 * kChunkK, nch, reinterpret_cast<uint4*>(smem),
                    reinterpret_cast<float*>(smem + p.off_as), tid, (int)blockDim.x);
  __syncthreads();
  const float g = (S == 1) ? *p.gscale : 1.0f;

  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
  int64_t j0 = r_lo;
  int ctt = 0;
  uint32_t uo = 0;  // byte offset of the slot being computed
  uint32_t ac = a_lane, asc = as_lane;  // the item's first iteration
  // the lane's scale bytes within a cell, beyond my_scale (the same for every chunk of a row):
  // 2L with 16-byte scale copies, else 0 or 2 within the lane's word
  uint32_t soff[R];
#pragma unroll
  for (int i = 0; i < R; ++i) soff[i] = s16 ? (uint32_t)lane * 2 : (uint32_t)(((j0 + i) * rs_s + lane_k) & 2);
  for (int q_ = 0; q_ < Q; ++q_) {
    cp_async_wait<NS - 1>();  // this lane's copies of item q_ have landed
    const int t0 = ctt * TI;
    if ((t0 + TI) * 32 <= nch) {  // warp-uniform: every lane has every chunk of the item
#pragma unroll
      for (int ti = 0; ti < TI; ++ti)
        item_rows<MT, R>(my_code + uo + (uint32_t)(ti * R * 512), my_scale + uo + (uint32_t)(ti * R * 128), soff,
                         ac + (uint32_t)ti * 2048, asc + (uint32_t)ti * 256, a_row, as_row, m, acc);
    } else {
#pragma unroll
      for (int ti = 0; ti < TI; ++ti)
        if ((t0 + ti) * 32 + lane < nch)
          item_rows<MT, R>(my_code + uo + (uint32_t)(ti * R * 512), my_scale + uo + (uint32_t)(ti * R * 128), soff,
                           ac + (uint32_t)ti * 2048, asc + (uint32_t)ti * 256, a_row, as_row, m, acc);
    }
    // refill the slot just read with item q_ + NS (the reads above are complete: their
    // results have been consumed)
    issue(uo);
    ac += TI * 2048;
    asc += TI * 256;
    if (++ctt == TT) {
      finish_rows<MT, R>(acc, p, j0, (int)min((int64_t)R, r_hi - j0), m, S, s, g, lane, true);
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
      ctt = 0;
      ac = a_lane;
      asc = as_lane;
      j0 += R;
#pragma unroll
      for (int i = 0; i < R; ++i) soff[i] = s16 ? (uint32_t)lane * 2 : (uint32_t)(((j0 + i) * rs_s + lane_k) & 2);
    }
    uo = (uo == (uint32_t)(NS - 1) * kSlot) ? 0u : uo + kSlot;
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------------------
// Lean stream pipeline (pipeline 5, m = 1). The stream pipeline's per-lane asynchronous
// copies, cut to what decode needs: one activation row, k % 256 == 0, and splits of whole 32-k
// chunk iterations. A slot holds R rows x TI chunk iterations: row i's cells of iteration ti
// at (i * TI + ti) * 512 (lane L's at + 16 L) and its scales at R * TI * 512 + (i * TI + ti) * 64
// (lane L's two bytes at + 2 L); a row group's last item may hold fewer iterations. The item
// loop is unrolled over the NS slots of the warp's ring, so every shared-memory address of the
// inner loop is a per-item base plus a compile-time offset, and the copy cursor is one pointer
// per tensor. The activations of the split are staged once per CTA; grid.y is the K split, as in
// the other pipelines.
template <int R, int NS>
__global__ void __launch_bounds__(kStreamMaxThreads, 1) gemv_lean_kernel(GemvArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int TI = kLeanIters;
  constexpr uint32_t kCodes = (uint32_t)(R * TI * 512), kSlot = kCodes + (uint32_t)(R * TI * 64);
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int NW = (int)(blockDim.x >> 5);
  const int64_t n = p.n, k = p.k;
  const int S = p.splits;
  const int s = blockIdx.y;

  const int64_t C = k / kChunkK;
  const int64_t c0 = (int64_t)s * C / S;
  const int nch = (int)((int64_t)(s + 1) * C / S - c0);  // a multiple of 32
  const int T = nch / 32;                               // chunk iterations of a row
  const int TT = (T + TI - 1) / TI;                     // items of a row group

  const int64_t GW = (int64_t)gridDim.x * NW;
  const int64_t gw = (int64_t)blockIdx.x * NW + warp;
  const int64_t ngr = (n + R - 1) / R;
  const int64_t g_lo = gw * ngr / GW, g_hi = (gw + 1) * ngr / GW;
  const int64_t r_lo = g_lo * R, r_hi = min(n, g_hi * R);
  const int Q = (int)(g_hi - g_lo) * TT;

  const int64_t rs_q = k / 2, rs_s = k / 16;
  const uint32_t ring = smem_addr(smem + p.off_ring) + (uint32_t)warp * NS * kSlot;
  const uint32_t my_code = ring + (uint32_t)lane * 16;
  // scale pieces: lane L < 4 * TI * R copies bytes [16 (L % 4TI), +16) of row L / 4TI's item
  // range (TI * 64 bytes) to kCodes + 16 L of the slot; the piece belongs to iteration (L % 4TI) / 4
  const bool s_lane = lane < 4 * TI * R;
  const int i_l = lane / (4 * TI), ti_l = (lane % (4 * TI)) / 4;
  const uint32_t my_s16 = ring + kCodes + (uint32_t)lane * 16;

  // ---- copy cursor: code cell of row 0 for this lane, this lane's scale piece, rows present
  const uint8_t* gq = p.Wq + r_lo * rs_q + (c0 + lane) * 16;
  const uint8_t* gs = p.Ws + (r_lo + (s_lane ? i_l : 0)) * rs_s + c0 * 2 + (lane % (4 * TI)) * 16;
  // from the end of a group's last item to the next group's first (every item advances the
  // cursor by TI iterations, a short last item included)
  const int64_t dq = (int64_t)R * rs_q - (int64_t)TT * TI * 512;
  const int64_t ds = (int64_t)R * rs_s - (int64_t)TT * TI * 64;
  int rows_i = (int)min((int64_t)R, r_hi - r_lo);  // rows of the group being copied
  int itt = 0, iq = 0;
  auto issue = [&](uint32_t off) {
    if (iq < Q) {
      const int tin = min(TI, T - itt * TI);  // iterations of this item
#pragma unroll
      for (int i = 0; i < R; ++i)
        if (i < rows_i)
#pragma unroll
          for (int ti = 0; ti < TI; ++ti)
            if (ti < tin) cp_async_16(my_code + off + (uint32_t)((i * TI + ti) * 512), gq + i * rs_q + ti * 512);
      if (s_lane && i_l < rows_i && ti_l < tin) cp_async_16(my_s16 + off, gs);
      gq += TI * 512;
      gs += TI * 64;
      if (++itt == TT) {
        itt = 0;
        gq += dq;
        gs += ds;
        rows_i = (int)min((int64_t)R, r_hi - (r_lo + (int64_t)(iq / TT + 1) * R));
      }
      ++iq;
    }
    cp_async_commit();
  };
  pdl_launch_dependents();
#pragma unroll
  for (int u = 0; u < NS; ++u) issue((uint32_t)u * kSlot);

  pdl_wait();
  {  // the split's activations (one activation row), staged once per CTA
    const int GA = (nch + 31) / 32;
    uint4* Ah4 = reinterpret_cast<uint4*>(smem);
    float* As = reinterpret_cast<float*>(smem + p.off_as);
    const uint16_t* src = p.A + c0 * kChunkK;
    for (int b = tid; b < 2 * nch; b += (int)blockDim.x) {
      const uint4 v0 = ldg_v4(src + b * 16), v1 = ldg_v4(src + b * 16 + 8);
      stage_block(v0, v1, 0, b, GA, 2 * nch, Ah4, As);
    }
  }
  __syncthreads();
  const float g = (S == 1) ? *p.gscale : 1.0f;

  const uint32_t a_lane = smem_addr(smem) + (uint32_t)lane * 16;
  const uint32_t as_lane = smem_addr(smem + p.off_as) + (uint32_t)lane * 8;
  const uint32_t sc_lane = ring + kCodes + (uint32_t)lane * 2;
  const uint32_t zoff[R] = {};
  float acc[R][1];
#pragma unroll
  for (int i = 0; i < R; ++i) acc[i][0] = 0.0f;
  int64_t j0 = r_lo;
  int ctt = 0;
  uint32_t ac = a_lane, asc = as_lane;
  for (int q0 = 0; q0 < Q; q0 += NS) {
#pragma unroll
    for (int u = 0; u < NS; ++u) {
      if (q0 + u < Q) {
        cp_async_wait<NS - 1>();  // this lane's copies of item q0 + u have landed
        const int tin = min(TI, T - ctt * TI);
#pragma unroll
        for (int ti = 0; ti < TI; ++ti)
          if (ti < tin)
            item_rows<1, R, TI * 512, TI * 64>(my_code + (uint32_t)(u * kSlot + ti * 512),
                                               sc_lane + (uint32_t)(u * kSlot + ti * 64), zoff,
                                               ac + (uint32_t)ti * 2048, asc + (uint32_t)ti * 256, 0, 0, 1, acc);
        issue((uint32_t)u * kSlot);  // refill the slot just read with item q0 + u + NS
        ac += TI * 2048;
        asc += TI * 256;
        if (++ctt == TT) {
          finish_rows<1, R>(acc, p, j0, (int)min((int64_t)R, r_hi - j0), 1, S, s, g, lane, true);
#pragma unroll
          for (int i = 0; i < R; ++i) acc[i][0] = 0.0f;
          ctt = 0;
          ac = a_lane;
          asc = as_lane;
          j0 += R;
        }
      }
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------------------
// Register pipeline (pipeline 4): the weights go from global memory straight to registers
// with 16-byte loads, as in the pages' streaming GEMV; nothing is copied to shared memory but
// the staged activations. Each warp keeps the loads of its next D chunk iterations in flight
// in a register ring (the loop is unrolled by D so every ring index is static). Same rows per
// warp, lane-to-chunk mapping and per-chunk arithmetic as the other pipelines, so the same
// bits for the same S.

// One chunk of R weight rows from registers (codes cq[i], the lane's two scale bytes sc[i]).
template <int MT, int R>
__device__ __forceinline__ void chunk_rows_reg(const uint4 (&cq)[R], const uint32_t (&sc)[R], uint32_t ap,
                                               uint32_t sp, uint32_t a_row, uint32_t as_row, int m,
                                               float (&acc)[R][MT]) {
  if (MT == 1) {
    const uint4 a0 = lds_v4(ap), a1 = lds_v4(ap + 512), a2 = lds_v4(ap + 1024), a3 = lds_v4(ap + 1536);
    const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                             a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
    const float2 sa = lds_f2(sp);
#pragma unroll
    for (int i = 0; i < R; ++i) {
      uint32_t wf[16];
      decode32(cq[i], wf);
      acc[i][0] = chunk_acc(av, sa, wf, e4m3x2_to_f16x2(sc[i]), acc[i][0]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      uint32_t wf[16];
      decode32(cq[i], wf);
      const uint32_t sh = e4m3x2_to_f16x2(sc[i]);
#pragma unroll
      for (int r = 0; r < MT; ++r) {
        if (r < m) {
          const uint32_t apr = ap + (uint32_t)r * a_row;
          const uint4 a0 = lds_v4(apr), a1 = lds_v4(apr + 512), a2 = lds_v4(apr + 1024), a3 = lds_v4(apr + 1536);
          const uint32_t av[16] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w,
                                   a2.x, a2.y, a2.z, a2.w, a3.x, a3.y, a3.z, a3.w};
          acc[i][r] = chunk_acc(av, lds_f2(sp + (uint32_t)r * as_row), wf, sh, acc[i][r]);
        }
      }
    }
  }
}

template <int MT, int R, int D>
__global__ void __launch_bounds__(kStreamMaxThreads, 1) gemv_reg_kernel(GemvArgs p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int NW = (int)(blockDim.x >> 5);
  const int m = (int)p.m;
  const int64_t n = p.n, k = p.k;
  const int S = p.splits;
  const int s = blockIdx.y;

  const int64_t C = k / kChunkK;
  const int64_t c0 = (int64_t)s * C / S;
  const int nch = (int)((int64_t)(s + 1) * C / S - c0);
  const int T = (nch + 31) / 32;  // chunk iterations of a row

  // rows of this warp: whole groups of R rows, balanced over all warps of the split
  const int64_t GW = (int64_t)gridDim.x * NW;
  const int64_t gw = (int64_t)blockIdx.x * NW + warp;
  const int64_t ngr = (n + R - 1) / R;
  const int64_t g_lo = gw * ngr / GW, g_hi = (gw + 1) * ngr / GW;
  const int64_t r_lo = g_lo * R, r_hi = min(n, g_hi * R);
  const int Q = (int)(g_hi - g_lo) * T;  // chunk iterations of this warp, row group by row group

  const int64_t rs_q = k / 2, rs_s = k / 16;
  pdl_launch_dependents();
  if (p.prefetch_l2 && lane == 0 && r_lo < r_hi) prefetch_rows_l2(p, r_lo, r_hi, c0, nch);

  // ---- load cursor: iteration (group lg, chunk iteration lt); row i's code and scale pointers
  // for this lane's chunk
  int lt = 0, iq = 0;
  int64_t lj0 = r_lo;
  const uint8_t* qp[R];
  const uint8_t* spp[R];
  auto load_group = [&]() {
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const int64_t j = min(lj0 + i, n - 1);  // rows past n load row n-1 and are never written
      qp[i] = p.Wq + j * rs_q + (c0 + lane) * 16;
      spp[i] = p.Ws + j * rs_s + (c0 + lane) * 2;
    }
  };
  uint4 rq[D][R];
  uint32_t rsc[D][R];
  // load iteration iq into ring slot u (u compile-time at every call site)
  auto load = [&](uint4 (&q)[R], uint32_t (&sc)[R]) {
    if (iq < Q && lt * 32 + lane < nch) {
#pragma unroll
      for (int i = 0; i < R; ++i) {
        q[i] = ldg_stream_v4(qp[i]);
        sc[i] = ldg_stream_u16(spp[i]);
      }
    }
    if (iq < Q) {
#pragma unroll
      for (int i = 0; i < R; ++i) {
        qp[i] += 512;
        spp[i] += 64;
      }
      if (++lt == T) {
        lt = 0;
        lj0 += R;
        load_group();
      }
    }
    ++iq;
  };
  load_group();
#pragma unroll
  for (int u = 0; u < D; ++u) load(rq[u], rsc[u]);

  pdl_wait();
  stage_activations(p.A, k, m, c0 * kChunkK, nch, reinterpret_cast<uint4*>(smem),
                    reinterpret_cast<float*>(smem + p.off_as), tid, (int)blockDim.x);
  __syncthreads();
  const float g = (S == 1) ? *p.gscale : 1.0f;

  const int GA = (nch + 31) / 32;
  const uint32_t a_row = (uint32_t)GA * 2048, as_row = (uint32_t)nch * 8;
  const uint32_t a_lane = smem_addr(smem) + (uint32_t)lane * 16;
  const uint32_t as_lane = smem_addr(smem + p.off_as) + (uint32_t)lane * 8;
  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
  int64_t j0 = r_lo;
  int ct = 0;
  uint32_t ac = a_lane, asc = as_lane;
  for (int q0 = 0; q0 < Q; q0 += D) {
#pragma unroll
    for (int u = 0; u < D; ++u) {
      if (q0 + u < Q) {
        if (ct * 32 + lane < nch) chunk_rows_reg<MT, R>(rq[u], rsc[u], ac, asc, a_row, as_row, m, acc);
        load(rq[u], rsc[u]);  // the slot's registers are consumed: refill with iteration q0 + u + D
        ac += 2048;
        asc += 256;
        if (++ct == T) {
          finish_rows<MT, R>(acc, p, j0, (int)min((int64_t)R, r_hi - j0), m, S, s, g, lane, true);
#pragma unroll
          for (int i = 0; i < R; ++i)
#pragma unroll
            for (int r = 0; r < MT; ++r) acc[i][r] = 0.0f;
          ct = 0;
          ac = a_lane;
          asc = as_lane;
          j0 += R;
        }
      }
    }
  }
}

namespace {

template <int MT, int RS>
int launch_one(const GemvArgs& a, cudaStream_t stream) {
  auto kern = gemv_nvfp4_kernel<MT, RS>;
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.grid_x, (unsigned)a.splits);
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

template <int MT, int R, int NS>
int launch_stream_one(const GemvArgs& a, cudaStream_t stream) {
  auto kern = gemv_stream_kernel<MT, R, NS>;
  static int configured[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_cuda_error("cudaGetDevice");
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return set_cuda_error("cudaFuncSetAttribute(gemv stream smem)");
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.grid_x, (unsigned)a.splits);
  cfg.blockDim = dim3((unsigned)a.threads);
  cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return set_cuda_error("gemv stream kernel launch");
  return FI_OK;
}

template <int MT, int R>
int launch_reg(const GemvArgs& a, cudaStream_t stream) {
  auto kern = gemv_reg_kernel<MT, R, kRegDepth>;
  static int configured[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_cuda_error("cudaGetDevice");
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return set_cuda_error("cudaFuncSetAttribute(gemv register smem)");
    configured[dev] = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.grid_x, (unsigned)a.splits);
  cfg.blockDim = dim3((unsigned)a.threads);
  cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return set_cuda_error("gemv register kernel launch");
  return FI_OK;
}

template <int R>
int launch_lean(const GemvArgs& a, cudaStream_t stream) {
  auto kern = a.stages == 4 ? gemv_lean_kernel<R, 4> : gemv_lean_kernel<R, 2>;
  static int configured[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return set_cuda_error("cudaGetDevice");
  if (!(configured[dev] & (a.stages == 4 ? 1 : 2))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return set_cuda_error("cudaFuncSetAttribute(gemv lean smem)");
    configured[dev] |= a.stages == 4 ? 1 : 2;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)a.grid_x, (unsigned)a.splits);
  cfg.blockDim = dim3((unsigned)a.threads);
  cfg.dynamicSmemBytes = (size_t)a.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return set_cuda_error("gemv lean kernel launch");
  return FI_OK;
}

template <int MT, int R>
int launch_stream_ns(const GemvArgs& a, cudaStream_t stream) {
  if (a.pipeline == kPipeLean) {
    if constexpr (MT == 1) return launch_lean<R>(a, stream);
    return set_error(FI_ERR_INVALID_ARG, "GEMV lean pipeline: m = 1 only");
  }
  if (a.pipeline == kPipeReg) {
    if constexpr (R <= 2) return launch_reg<MT, R>(a, stream);  // R = 4 would spill the register ring
    return set_error(FI_ERR_INVALID_ARG, "GEMV register pipeline: at most 2 rows per warp");
  }
  if (a.stages == 4) return launch_stream_one<MT, R, 4>(a, stream);
  if (a.stages == 2) return launch_stream_one<MT, R, 2>(a, stream);
  return set_error(FI_ERR_INVALID_ARG, "GEMV stream pipeline: %d slots per warp is not available", a.stages);
}

template <int MT>
int launch_stream_r(const GemvArgs& a, cudaStream_t stream) {
  switch (a.rows_per_stage) {
    case 1: return launch_stream_ns<MT, 1>(a, stream);
    case 2:
      if constexpr (gemv_rmax(MT) >= 2) return launch_stream_ns<MT, 2>(a, stream);
      break;
    case 4:
      if constexpr (gemv_rmax(MT) >= 4) return launch_stream_ns<MT, 4>(a, stream);
      break;
    default: break;
  }
  return set_error(FI_ERR_INVALID_ARG, "GEMV rows per item %d is not available for m=%lld", a.rows_per_stage,
                   (long long)a.m);
}

template <int MT>
int launch_rs(const GemvArgs& a, cudaStream_t stream) {
  switch (a.rows_per_stage) {
    case 1: return launch_one<MT, 1>(a, stream);
    case 2:
      if constexpr (gemv_rmax(MT) >= 2) return launch_one<MT, 2>(a, stream);
      break;
    case 4:
      if constexpr (gemv_rmax(MT) >= 4) return launch_one<MT, 4>(a, stream);
      break;
    case 8:
      if constexpr (gemv_rmax(MT) >= 8) return launch_one<MT, 8>(a, stream);
      break;
    default: break;
  }
  return set_error(FI_ERR_INVALID_ARG, "GEMV rows per stage %d is not available for m=%lld", a.rows_per_stage,
                   (long long)a.m);
}

}  // namespace

int gemv_rows_per_stage_max(int64_t m) { return gemv_rmax(gemv_mt(m)); }

namespace {
template <int MT>
int launch_mt(const GemvArgs& a, cudaStream_t stream) {
  return a.pipeline == kPipeRing ? launch_rs<MT>(a, stream) : launch_stream_r<MT>(a, stream);
}
}  // namespace

int launch_gemv(const GemvArgs& a, cudaStream_t stream) {
  if (a.m <= 1) return launch_mt<1>(a, stream);
  if (a.m <= 2) return launch_mt<2>(a, stream);
  if (a.m <= 4) return launch_mt<4>(a, stream);
  if (a.m <= 8) return launch_mt<8>(a, stream);
  if (a.m <= 16) return launch_mt<16>(a, stream);
  if (a.m <= 32) return launch_mt<32>(a, stream);
  return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV supports m <= %d", kGemvMaxM);
}

unsigned* device_error_word() {
  static unsigned* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_gemv_error) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<unsigned*>(p);
  }
  return addr[dev];
}

int gemv_read_error(unsigned* bits) {
  unsigned v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_error, sizeof(v)) != cudaSuccess)
    return set_cuda_error("cudaMemcpyFromSymbol(gemv error)");
  if (v && cudaMemcpyToSymbol(g_gemv_error, &zero, sizeof(zero)) != cudaSuccess)
    return set_cuda_error("cudaMemcpyToSymbol(gemv error)");
  *bits = v;
  return FI_OK;
}

}  // namespace fi
