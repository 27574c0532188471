// Tensor-core path for bf16 activations x NVFP4 weights (sm_100a, tcgen05 + TMA + TMEM).
//
// After PR #4038's MMA path (Description, "What it does": the GEMV reads the same packed
// operands as the MMA kernel, so the tactic can pick either per shape), re-designed for B200:
//
//  * Operands. tcgen05.mma kind::f16 needs both operands of one 16-bit type. The weights are
//    decoded to f16 (every E2M1 value times its E4M3 block scale is exact in f16: at most 6
//    significant bits, magnitudes 2^-10 .. 2688); the activations are converted once per call
//    to f16 times a power of two per (row, K split) that puts the maximum of the row's split
//    range in [2^14, 2^15) (exact for every element within 2^29 of that maximum), so the tensor
//    core accumulates sum_k W'[i][k] * A'[j][k] in fp32 and one factor per (row, split) undoes
//    the scale. The conversion runs in act_to_f16_kernel into the workspace, or, when the
//    split's slice fits shared memory (m_pad <= 128), in otherwise idle warps at kernel start
//    ("resident" activations: no second launch and no per-step activation copies); both use
//    the same arithmetic and give the same bits.
//  * Roles (one CTA per 256 weight rows, 24 warps):
//      warp 0      TMA producer of the raw codes of the tile (256 rows x 32 bytes per 64-k step)
//                  into a 4-stage ring, issued before the grid-dependency wait (weights never
//                  depend on the preceding kernel);
//      warp 18     TMA producer of the f16 activation tiles (m_pad rows x 64 k, 128-byte
//                  swizzled) into the operand stages (2 to 4, as many as shared memory holds);
//                  with resident activations it copies the split's bf16 tiles once instead and
//                  converts them with warps 19-22;
//      warps 2-17  decode: two threads per weight row (32 k each), codes -> f16
//                  (cvt.rn.f16x2.e2m1x2) times the block scale (exact f16 multiply), written to
//                  tensor memory (m_pad <= 128; the loop runs over groups of 4 steps with
//                  compile-time stage indices) or to shared memory in the 128-byte-swizzled
//                  K-major layout the MMA reads; the block scales are loaded 8-11 steps ahead;
//      warps 1, 23 the MMAs, one thread each, one M = 128 half of the tile each (warp 1 also
//                  allocates TMEM): per 64-k step 4 K=16 steps, N = m_pad, accumulating in
//                  TMEM; tcgen05.commit frees the stage once both halves have read it;
//      warps 19-22 epilogue: tcgen05.ld of the accumulator, out[j][i] = round(D[i][j] *
//                  rs[j] * gscale) to bf16 (or f16); with resident activations they first
//                  convert them (warp 18 too), while the decode warps start on the weights.
//  * The weight tile is decoded once per call (the activations, m_pad <= 256 rows, are one MMA
//    N tile), so the decode work is one cvt and one f16 multiply per two codes.
//  * Every wait is bounded (see sync.cuh); on a timeout the roles stop, the MMA issuer and the
//    producer drain what they issued, and TMEM is freed before the CTA exits.
//
// Arithmetic order: fixed by k (64-k steps in order, K=16 sub-steps in order) and independent
// of m, so for a fixed tactic a row's bits do not depend on m (an output element depends only
// on its weight row and activation row); results are deterministic run to run.
#include <cstdint>
#include <algorithm>
#include <cstring>

#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sync.cuh"

namespace fi {

namespace {

constexpr int kWarpTma = 0, kWarpMma = 1, kWarpDq0 = 2, kDqWarps = 16, kWarpAct = 18, kWarpEpi0 = 19, kEpiWarps = 4,
              kWarpMma2 = 23;
static_assert((kWarpMma2 + 1) * 32 == kMmaThreads, "warp roles cover the CTA");
static_assert(kWarpDq0 + kDqWarps == kWarpAct && kWarpAct + 1 == kWarpEpi0 && kDqWarps * 32 == 2 * kMmaTileRows,
              "two decode threads per tile row");
// resident activations: converted by the activation producer and epilogue warps (18-22)
constexpr int kConvWarps = kEpiWarps + 1;
static_assert(kWarpAct + kConvWarps == kWarpMma2, "converting warps: 18 .. 22");
constexpr int kRawStages = 4;
constexpr uint32_t kRawBytes = kMmaTileRows * 32;  // 256 rows x 32 code bytes
constexpr uint32_t kWopBytes = kMmaTileRows * 128;  // 256 rows x 64 f16, 128-byte swizzled
// barriers: raw_full, raw_empty, then act_full, op_full, op_empty per operand stage, tmem_full,
// and one drain barrier per MMA-issuing thread
constexpr int kNumBars = 2 * kRawStages + 3 * kMmaMaxOpStages + 3;

// Shared-memory matrix descriptor of a K-major tile with 128-byte rows in the 128-byte swizzle
// (8-row atoms of 1024 bytes): start address >> 4 in bits 0-13, leading-dimension offset 1
// (unused for swizzled K-major), stride-dimension offset 1024 >> 4 in bits 32-45, descriptor
// version 1 in bits 46-47, swizzle mode 2 (128 bytes) in bits 61-63.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1), f16 A and B (bits 7-9,
// 10-12 = 0), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__device__ __forceinline__ uint32_t f16_idesc(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// tcgen05.mma with the A operand (the weights) in tensor memory at a_tmem.
__device__ __forceinline__ void umma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane (32x32b shape: the warp's 32 lanes
// from the lane in taddr, which must be the warp's own quarter), as two 8-column stores (on B200
// the decode loop ran 2-5% faster this way than with one 16-column store or four 4-column ones).
__device__ __forceinline__ void tmem_st16_halves(uint32_t taddr, const uint32_t (&v)[16]) {
#pragma unroll
  for (int q = 0; q < 2; ++q)
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr + q * 8),
                 "r"(v[8 * q]), "r"(v[8 * q + 1]), "r"(v[8 * q + 2]), "r"(v[8 * q + 3]), "r"(v[8 * q + 4]),
                 "r"(v[8 * q + 5]), "r"(v[8 * q + 6]), "r"(v[8 * q + 7])
                 : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint4 lds_v4m(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The four bytes of a 32-bit word (8 E2M1 codes, low nibble first) as four f16x2 pairs, in
// byte order, with one unpack of the word for all four conversions. Exact.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2,
                                                  uint32_t& h3) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}

// One thread's 32 k of a step: 16 code bytes (blocks 2hb, 2hb+1 of the row) and the two E4M3
// scales in the low 16 bits of sc2 -> 16 f16 pairs (code value times its block scale, exact).
__device__ __forceinline__ void decode_step(const uint4 c0, uint32_t sc2, uint32_t (&hv)[16]) {
  const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
  for (int bb = 0; bb < 2; ++bb) {  // 16-k block 2hb + bb: words 2bb, 2bb+1
    const uint32_t sf2 = e4m3x2_to_f16x2(__byte_perm(sc2, 0u, (uint32_t)(bb | (bb << 4))));
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t h[4];
      e2m1x8_to_f16x2x4(words[2 * bb + q], h[0], h[1], h[2], h[3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) hv[8 * bb + 4 * q + i] = hmul2(h[i], sf2);
    }
  }
}

// Wait that ignores the abort flag (used to drain copies and MMAs in flight before exit).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, unsigned* err) {
  volatile int never = 0;
  mbar_wait_bounded(bar, parity, &never, timeout_ns, err, 8u);
}

}  // namespace

// The activation conversion shared by the prepass kernel and the kernel's resident mode, so
// that both give the same bits. Per (activation row, K split): the largest biased exponent of
// the row's bf16 values over the split's k range sets a power of two that puts the maximum in
// [2^14, 2^15); every value times it is rounded to f16, and the epilogue multiplies by the
// inverse (exact).
__device__ __forceinline__ uint32_t bf16x8_max_exp(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t e = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) e = max(e, max((w[q] >> 7) & 0xFFu, (w[q] >> 23) & 0xFFu));
  return e;
}

__device__ __forceinline__ int act_shift(uint32_t e_max) {
  const int sh = 141 - (int)e_max;  // biased exponent E of the maximum -> [2^14, 2^15)
  return sh < -126 ? -126 : (sh > 126 ? 126 : sh);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 v, float up) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t h[4];
#pragma unroll
  for (int q = 0; q < 4; ++q)
    h[q] = f32x2_to_f16x2(__uint_as_float(w[q] << 16) * up, __uint_as_float(w[q] & 0xFFFF0000u) * up);
  return make_uint4(h[0], h[1], h[2], h[3]);
}

// A[m, k] bf16 -> a16[m_pad, k] f16, block (row, split) over the split's k range (64-k steps
// [s KS/S, (s+1) KS/S)), scaled by the per-(row, split) power of two above; rs[split][row] =
// the inverse scale. Rows m .. m_pad-1 are zero.
__global__ void __launch_bounds__(256) act_to_f16_kernel(const uint16_t* __restrict__ A, int64_t m, int64_t k,
                                                         uint16_t* __restrict__ a16, float* __restrict__ rs) {
  pdl_launch_dependents();
  pdl_wait();
  const int64_t row = blockIdx.x;
  const int m_pad = (int)gridDim.x, S = (int)gridDim.y, sp = (int)blockIdx.y;
  const int64_t KS_all = k / kMmaKStep;
  const int64_t kb = sp * KS_all / S * kMmaKStep, ke = (sp + 1) * KS_all / S * kMmaKStep;
  const int tid = threadIdx.x;
  uint4* dst = reinterpret_cast<uint4*>(a16 + row * k + kb);
  const int64_t n8 = (ke - kb) / 8;  // 16-byte groups of the row's split range
  if (row >= m) {
    for (int64_t i = tid; i < n8; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) rs[(int64_t)sp * m_pad + row] = 0.0f;
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(A + row * k + kb);
  uint32_t e = 0;
  for (int64_t i = tid; i < n8; i += blockDim.x) e = max(e, bf16x8_max_exp(ldg_v4(src + i)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
  __shared__ uint32_t red[8];
  if ((tid & 31) == 0) red[tid >> 5] = e;
  __syncthreads();
  e = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) e = max(e, red[w]);
  const int sh = act_shift(e);
  const float up = __uint_as_float((uint32_t)(sh + 127) << 23);
  for (int64_t i = tid; i < n8; i += blockDim.x) dst[i] = bf16x8_to_f16x8(ldg_v4(src + i), up);
  if (tid == 0) rs[(int64_t)sp * m_pad + row] = __uint_as_float((uint32_t)(127 - sh) << 23);
}

// TA: the decoded weights go to tensor memory (tcgen05.st) and the MMAs read A from there
// (m_pad <= 128: the accumulator takes 2 m_pad <= 256 columns, the A stages columns 256-511);
// otherwise they go to shared memory in the 128-byte swizzle.
template <bool TA>
__global__ void __launch_bounds__(kMmaThreads, 1)
    mma_nvfp4_kernel(const MmaArgs p, const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_w) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ volatile int abort_flag;
  __shared__ uint32_t tmem_slot;
  // 1024-byte aligned base for the swizzled tiles: the raw-code ring, then NST operand stages
  // (decoded weights, then activations, each stage stage_bytes; 0 with resident activations),
  // then the resident slice and its row scales (act_bytes + act_extra_bytes, else 0), then
  // the barriers
  const int NST = p.op_stages;
  const uint32_t stage_bytes = p.stage_bytes;
  const uint32_t raw_s = smem_addr(smem_raw);
  const uint32_t base = (raw_s + 1023u) & ~1023u;
  uint8_t* const basep = smem_raw + (base - raw_s);
  // resident activations (p.act_resident): the split's whole f16 activation slice, one
  // 128-byte-swizzled tile of m_pad rows x 64 k per step, then the per-row inverse scales
  const bool resident = p.act_resident != 0;
  const uint32_t act_res = base + kRawStages * kRawBytes + (uint32_t)NST * stage_bytes;
  float* const rs_res = reinterpret_cast<float*>(basep + kRawStages * kRawBytes + (uint32_t)NST * stage_bytes +
                                                 p.act_bytes);
  uint64_t* const bars = reinterpret_cast<uint64_t*>(basep + kRawStages * kRawBytes + (uint32_t)NST * stage_bytes +
                                                     p.act_bytes + p.act_extra_bytes);
  uint64_t* const raw_full = bars;
  uint64_t* const raw_empty = bars + kRawStages;
  uint64_t* const act_full = bars + 2 * kRawStages;
  uint64_t* const op_full = act_full + kMmaMaxOpStages;
  uint64_t* const op_empty = op_full + kMmaMaxOpStages;
  uint64_t* const tmem_full = op_empty + kMmaMaxOpStages;
  uint64_t* const drain = tmem_full + 1;
  auto raw_addr = [&](int st) { return base + (uint32_t)st * kRawBytes; };
  auto wop_addr = [&](int st) { return base + kRawStages * kRawBytes + (uint32_t)st * stage_bytes; };
  auto act_addr = [&](int st) { return wop_addr(st) + (TA ? 0u : kWopBytes); };
  // TA: columns of the A operand of stage st, half h (32 columns: 64 k as f16 pairs)
  auto a_col = [&](int st, int h) { return 256u + (uint32_t)st * 64u + (uint32_t)h * 32u; };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n = p.n, k = p.k;
  const int m = (int)p.m, N = p.m_pad;
  // split blockIdx.y of gridDim.y takes the 64-k steps [ks0, ks0 + KS) in order
  const int KS_all = (int)(k / kMmaKStep), S = (int)gridDim.y, sp = (int)blockIdx.y;
  const int ks0 = (int)((int64_t)sp * KS_all / S);
  const int KS = (int)((int64_t)(sp + 1) * KS_all / S) - ks0;
  const int64_t w0 = (int64_t)blockIdx.x * kMmaTileRows;
  const uint32_t ncols = TA ? 512u : (N <= 16 ? 32u : (N <= 64 ? 128u : (N <= 128 ? 256u : 512u)));  // >= 2N

  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < kRawStages; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], kDqWarps);
    }
    for (int i = 0; i < NST; ++i) {
      // resident mode: act_full[0] completes once, when the converting warps are done, and
      // act_full[1] once, when the copies of the split's bf16 activations have landed
      mbar_init(&act_full[i], resident && i == 0 ? kConvWarps : 1);
      mbar_init(&op_full[i], kDqWarps);
      mbar_init(&op_empty[i], 2);  // both MMA issuers commit
    }
    mbar_init(tmem_full, 2);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_slot;
  pdl_launch_dependents();

  if (resident && warp >= kWarpAct && warp < kWarpAct + kConvWarps) {
    // ----------------------------------------------------------- resident activations
    // The activation producer and epilogue warps (idle until the accumulator is complete)
    // convert the split's activations while the decode warps start on the weights. Each warp
    // owns whole rows (no atomics, no barrier between warps): A over k [64 ks0, 64 (ks0 + KS))
    // lands as bf16 in the swizzled tiles the MMA reads (one 128-byte-swizzled tile of N rows x
    // 64 k per step, one TMA copy each, all in flight at once; rows m..N-1 zero), then each
    // row's largest exponent over the split (a warp reduction), then the in-place conversion
    // to f16 with the per-(row, split) scale (the prepass kernel's arithmetic). A is written
    // by the preceding kernel.
    pdl_wait();
    const int cw = warp - kWarpAct;   // 0 .. kConvWarps - 1: this warp converts rows cw, cw + 5, ...
    const int per_row = KS * 8;       // 16-byte pieces of a row's split range
    if (cw == 0 && lane == 0) {
      // the split's bf16 tiles, one TMA copy per step (rows m..N-1 read as zeros)
      mbar_arrive_expect_tx(&act_full[1], (uint32_t)KS * (uint32_t)(N * 128));
      for (int s = 0; s < KS; ++s)
        tma_load_2d(act_res + (uint32_t)s * (uint32_t)(N * 128), &tmap_a, (ks0 + s) * kMmaKStep, 0,
                    smem_addr(&act_full[1]));
    }
    auto piece_addr = [&](int j, int c) {
      const int st = c >> 3, cc = c & 7;  // step, 16-byte chunk within the row's 128 bytes
      return act_res + (uint32_t)st * (uint32_t)(N * 128) + (uint32_t)(j >> 3) * 1024u + (uint32_t)(j & 7) * 128u +
             ((uint32_t)(cc ^ (j & 7)) << 4);
    };
    // every copy must land before the conversion reads it or the CTA exits, abort or not
    drain_wait(&act_full[1], 0u, p.timeout_ns, p.err);
    for (int j = cw; j < N; j += kConvWarps) {
      if (j >= m) {
        if (lane == 0) rs_res[j] = 0.0f;
        continue;
      }
      uint32_t e = 0;
#pragma unroll 4
      for (int c = lane; c < per_row; c += 32) e = max(e, bf16x8_max_exp(lds_v4m(piece_addr(j, c))));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
      const int sh = act_shift(e);
      const float up = __uint_as_float((uint32_t)(sh + 127) << 23);
#pragma unroll 4
      for (int c = lane; c < per_row; c += 32) {
        const uint32_t a = piece_addr(j, c);
        const uint4 h = bf16x8_to_f16x8(lds_v4m(a), up);
        sts_v4(a, h.x, h.y, h.z, h.w);
      }
      if (lane == 0) rs_res[j] = __uint_as_float((uint32_t)(127 - sh) << 23);
    }
    // make the generic-proxy stores visible to the tensor core (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&act_full[0]);
  }

  if (warp == kWarpTma) {
    // ------------------------------------------------------------------------ producers
    // one thread streams the raw codes, gated by the decode warps freeing raw stages (the
    // activation tiles have their own warp: two lanes of one warp in divergent loops with
    // suspending waits progress one at a time, which serialised the two streams)
    if (lane == 0 && !p.debug_stall) {
      int issued = 0;
      const int pro = KS < kRawStages ? KS : kRawStages;
      for (int s = 0; s < pro; ++s) {
        mbar_arrive_expect_tx(&raw_full[s], kRawBytes);
        tma_load_2d(raw_addr(s), &tmap_w, (ks0 + s) * 32, (int)w0, smem_addr(&raw_full[s]));
        ++issued;
      }
      for (int s = 0; s + kRawStages < KS && !abort_flag; ++s) {
        const int rs = s % kRawStages;
        if (!mbar_wait_bounded(&raw_empty[rs], (uint32_t)((s / kRawStages) & 1), &abort_flag, p.timeout_ns, p.err,
                               2u))
          break;
        mbar_arrive_expect_tx(&raw_full[rs], kRawBytes);
        tma_load_2d(raw_addr(rs), &tmap_w, (ks0 + s + kRawStages) * 32, (int)w0, smem_addr(&raw_full[rs]));
        ++issued;
      }
      // drain: every copy issued must have landed before the CTA exits
      for (int s = issued - kRawStages < 0 ? 0 : issued - kRawStages; s < issued; ++s)
        drain_wait(&raw_full[s % kRawStages], (uint32_t)((s / kRawStages) & 1), p.timeout_ns, p.err);
    }
  } else if (warp == kWarpAct) {
    // --------------------------------------------------------------- activation producer
    // one thread streams the f16 activation tiles, gated by the MMAs freeing operand stages
    if (lane == 0 && !p.debug_stall && !resident) {
      pdl_wait();  // the activations come from the conversion kernel launched just before
      int issued = 0, os = 0;
      uint32_t ph = 0;  // phase of op_empty[os] to wait for once every stage has been used
      for (int s = 0; s < KS && !abort_flag; ++s) {
        if (s >= NST && !mbar_wait_bounded(&op_empty[os], ph, &abort_flag, p.timeout_ns, p.err, 2u)) break;
        mbar_arrive_expect_tx(&act_full[os], (uint32_t)N * 128u);
        tma_load_2d(act_addr(os), &tmap_a, (ks0 + s) * kMmaKStep, 0, smem_addr(&act_full[os]));
        ++issued;
        if (++os == NST) {
          os = 0;
          if (s >= NST) ph ^= 1u;
        }
      }
      for (int s = issued - NST < 0 ? 0 : issued - NST; s < issued; ++s)
        drain_wait(&act_full[s % NST], (uint32_t)((s / NST) & 1), p.timeout_ns, p.err);
    }
  } else if (warp >= kWarpDq0 && warp < kWarpDq0 + kDqWarps) {
    // -------------------------------------------------------------------------- decode
    // shared-memory operand: two threads per row (adjacent lanes), blocks 2hb, 2hb+1 each.
    // TA: a warp may only reach its own quarter of the TMEM lanes, so warp w takes rows
    // h*128 + 32(w % 4) + lane of half h and k half hb, (h, hb) from the warp's index among
    // the four decode warps of its quarter.
    const int dq = (warp - kWarpDq0) >> 2;
    const int tq = warp & 3;
    const int r = TA ? (dq & 1) * 128 + tq * 32 + lane : (tid - kWarpDq0 * 32) >> 1;  // tile row, 0 .. 255
    const int hb = TA ? dq >> 1 : tid & 1;  // this thread's half of the step: blocks 2hb, 2hb+1
    const int64_t row = w0 + r;
    const bool valid = row < n;
    const int64_t rs_s = k / 16;
    const uint8_t* srow = p.Ws + (valid ? row : 0) * rs_s + (int64_t)ks0 * 4;  // the split's first step
    const uint32_t wdst = (uint32_t)(r >> 7) * (kWopBytes / 2) + (uint32_t)(r & 127) * 128u;
    const uint32_t swz = (uint32_t)(r & 7);
    // The row's four E4M3 scales of step s are the 4 bytes at srow + 4s. They are loaded in
    // groups of 4 steps, three groups ahead of their use, so the global-memory latency of the
    // scales (cold: they are read once per call) is off the per-step path.
    const bool al16 = rs_s % 16 == 0 && ks0 % 4 == 0;
    auto load_group = [&](int gi) -> uint4 {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      const int s0 = gi * 4;
      if (valid && s0 < KS) {
        if (al16 && s0 + 3 < KS) {
          v = ldg_v4(srow + s0 * 4);
        } else {
          v.x = ldg_u32(srow + s0 * 4);
          if (s0 + 1 < KS) v.y = ldg_u32(srow + s0 * 4 + 4);
          if (s0 + 2 < KS) v.z = ldg_u32(srow + s0 * 4 + 8);
          if (s0 + 3 < KS) v.w = ldg_u32(srow + s0 * 4 + 12);
        }
      }
      return v;
    };
    uint4 sg0 = load_group(0), sg1 = load_group(1), sg2 = load_group(2);
    if constexpr (TA) {
      // Four operand stages (the host guarantees NST == kRawStages == 4 here), so the loop runs
      // over groups of 4 steps with the step's stage, barriers, scale word and tensor-memory
      // columns fixed at compile time; a group's 4 scale words were loaded 8-11 steps ahead.
      // The decode warps' instruction issue paces a step at small m (B200 counters: cutting
      // the integer work per step from 63 to 28 instructions per thread took 4096 x 14336 at
      // m = 8 from 22.0 to 20.4 us), so the per-step bookkeeping is kept to a minimum.
      static_assert(kRawStages == 4 && kMmaMaxOpStages == 4, "one group = one pass over both rings");
      const uint32_t raw_row = base + (uint32_t)r * 32u + (uint32_t)hb * 16u;
      const uint32_t tm_row = tmem + ((uint32_t)(tq * 32) << 16) + a_col(0, r >> 7) + (uint32_t)hb * 16u;
      bool run = true;
      for (int s0 = 0; s0 < KS && run; s0 += 4) {
        const uint32_t par = (uint32_t)((s0 >> 2) & 1);  // raw_full phase; op_empty waits for par ^ 1
        const uint4 scg = sg0;
        sg0 = sg1;
        sg1 = sg2;
        sg2 = load_group(s0 / 4 + 3);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (s0 + j >= KS) break;
          // One step per pass (pairing two steps per wait and store cut instructions but lost
          // overlap). Fast path: both phases already complete for every lane (one test each and
          // one vote); else every lane waits, bounded, and the warp continues only if all of
          // them saw both.
          const bool fast = mbar_try_wait(&raw_full[j], par) && (s0 == 0 || mbar_try_wait(&op_empty[j], par ^ 1u));
          if (!__all_sync(0xffffffffu, fast)) {
            const bool ok = mbar_wait_bounded(&raw_full[j], par, &abort_flag, p.timeout_ns, p.err, 1u) &&
                            (s0 == 0 || mbar_wait_bounded(&op_empty[j], par ^ 1u, &abort_flag, p.timeout_ns, p.err, 1u));
            if (!__all_sync(0xffffffffu, ok)) {
              run = false;
              break;
            }
          }
          const uint4 c0 = lds_v4m(raw_row + (uint32_t)j * kRawBytes);
          const uint32_t sc4 = j == 0 ? scg.x : (j == 1 ? scg.y : (j == 2 ? scg.z : scg.w));
          uint32_t hv[16];
          decode_step(c0, hb ? (sc4 >> 16) : sc4, hv);
          // lane r & 127 of half r >> 7: columns a_col + 16 hb .. + 15 hold k 32 hb .. 32 hb + 31
          tmem_st16_halves(tm_row + (uint32_t)j * 64u, hv);
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&op_full[j]);
            mbar_arrive(&raw_empty[j]);
          }
        }
      }
    } else {
      int os = 0;        // operand stage of step s
      uint32_t eph = 0;  // phase of op_empty[os] to wait for (steps s >= NST)
      for (int s = 0; s < KS; ++s) {
        const int rsn = s % kRawStages;
        const int sj = s & 3;
        const uint32_t sc4 = sj == 0 ? sg0.x : (sj == 1 ? sg0.y : (sj == 2 ? sg0.z : sg0.w));
        if (sj == 3) {
          sg0 = sg1;
          sg1 = sg2;
          sg2 = load_group(s / 4 + 3);
        }
        // every lane waits; the warp continues only if all of them saw both phases (a timeout is
        // seen lane by lane, and the warp must stay converged for __syncwarp below)
        const bool ok =
            mbar_wait_bounded(&raw_full[rsn], (uint32_t)((s / kRawStages) & 1), &abort_flag, p.timeout_ns, p.err, 1u) &&
            (s < NST || mbar_wait_bounded(&op_empty[os], eph, &abort_flag, p.timeout_ns, p.err, 1u));
        if (!__all_sync(0xffffffffu, ok)) break;
        const uint4 c0 = lds_v4m(raw_addr(rsn) + (uint32_t)r * 32u + (uint32_t)hb * 16u);
        uint32_t hv[16];  // the 32 k of this thread as f16 pairs, in k order
        decode_step(c0, hb ? (sc4 >> 16) : sc4, hv);
        const uint32_t dst = wop_addr(os) + wdst;
#pragma unroll
        for (int c = 0; c < 4; ++c)  // chunk 4hb + c of the row (8 k each), 128-byte swizzle
          sts_v4(dst + (((4u * (uint32_t)hb + (uint32_t)c) ^ swz) << 4), hv[4 * c], hv[4 * c + 1], hv[4 * c + 2],
                 hv[4 * c + 3]);
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&op_full[os]);
          mbar_arrive(&raw_empty[rsn]);
        }
        if (++os == NST) {
          os = 0;
          if (s >= NST) eph ^= 1u;
        }
      }
    }
  } else if (warp == kWarpMma || warp == kWarpMma2) {
    // ----------------------------------------------------------------------------- MMA
    // Two issuing threads, one per M = 128 half of the tile (disjoint TMEM columns, same
    // activation operand): at small N the issue of MMA instructions by one thread, not the
    // tensor core, set the pace. Each commits to the stage's op_empty (count 2), to tmem_full
    // (count 2) and to its own drain barrier.
    if (lane == 0) {
      const int h = warp == kWarpMma ? 0 : 1;
      const uint32_t idesc = f16_idesc(128, N);
      // the descriptors differ only in the start-address field: a constant high part plus a
      // 32-bit running start (address >> 4) per stage
      const uint64_t desc_fixed = sw128_desc(0);
      const uint32_t a_first = (wop_addr(0) >> 4) & 0x3FFFu, a_stride = stage_bytes >> 4;
      constexpr uint32_t kHalf = kWopBytes / 2 / 16, kAct = kWopBytes / 16;  // in 16-byte units
      uint32_t a_lo = a_first;
      // resident mode: step s's activation tile at act_res + s * N * 128 (in 16-byte units)
      uint32_t b_res = (act_res >> 4) & 0x3FFFu;
      const uint32_t b_res_step = (uint32_t)N * 8u;
      int os = 0;
      uint32_t par = 0;  // phase of act_full[os] and op_full[os] for step s
      bool go = !resident || mbar_wait_bounded(&act_full[0], 0u, &abort_flag, p.timeout_ns, p.err, 4u);
      for (int s = 0; s < KS && go; ++s) {
        if (!resident && !mbar_wait_bounded(&act_full[os], par, &abort_flag, p.timeout_ns, p.err, 4u)) break;
        if (!mbar_wait_bounded(&op_full[os], par, &abort_flag, p.timeout_ns, p.err, 4u)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t acc0 = s != 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < kMmaKStep / 16; ++kk) {
          if constexpr (TA) {
            const uint64_t bdesc = desc_fixed | (uint64_t)((resident ? b_res : a_lo) + (uint32_t)kk * 2u);
            umma_f16_ta(tmem + (uint32_t)(h * N), tmem + a_col(os, h) + (uint32_t)kk * 8u, bdesc, idesc,
                        kk != 0 ? 1u : acc0);
          } else {
            const uint64_t bdesc = desc_fixed | (uint64_t)(a_lo + kAct + (uint32_t)kk * 2u);
            const uint64_t adesc = desc_fixed | (uint64_t)(a_lo + (uint32_t)h * kHalf + (uint32_t)kk * 2u);
            umma_f16(tmem + (uint32_t)(h * N), adesc, bdesc, idesc, kk != 0 ? 1u : acc0);
          }
        }
        umma_commit(&op_empty[os]);  // frees the stage when these MMAs have read it
        a_lo += a_stride;
        b_res += b_res_step;
        if (++os == NST) {
          os = 0;
          par ^= 1u;
          a_lo = a_first;
        }
      }
      umma_commit(tmem_full);  // the accumulator is complete when every MMA issued has finished
      umma_commit(&drain[h]);
      drain_wait(&drain[h], 0, p.timeout_ns, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------ epilogue
    pdl_wait();
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int i = q * 32 + lane;
    // warp-uniform: the TMEM loads below are collective over the warp
    // resident mode: the row scales come from the converting warps (wait for all of them)
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(tmem_full, 0, &abort_flag, p.timeout_ns, p.err, 16u) &&
                                                (!resident || mbar_wait_bounded(&act_full[0], 0u, &abort_flag,
                                                                                p.timeout_ns, p.err, 16u)) &&
                                                !abort_flag);
    const float* const rsp = resident ? rs_res : p.rs + (int64_t)sp * N;  // this split's inverse row scales
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok) {
      const float g = *p.gscale;
      // S > 1: this split's fp32 partials D * rs[j] (exact: rs is a power of two), summed in
      // split order by the reduce kernel; S == 1: round(D * rs[j] * gscale) to the output type
      float* const part = S > 1 ? p.partials + (int64_t)sp * m * n : nullptr;
      for (int h = 0; h < 2; ++h) {
        const int64_t row = w0 + h * 128 + i;
        for (int j0 = 0; j0 < N; j0 += 16) {
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * N + j0), v);
          if (row < n) {
            if (part == nullptr) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int j = j0 + jj;
                if (j < m)
                  p.out[(int64_t)j * n + row] = f32_to_out(__fmul_rn(__fmul_rn(v[jj], rsp[j]), g), p.out_f16 != 0);
              }
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int j = j0 + jj;
                if (j < m) part[(int64_t)j * n + row] = __fmul_rn(v[jj], rsp[j]);
              }
            }
          }
        }
      }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  }

  __syncthreads();
  if (warp == kWarpMma) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

// ---------------------------------------------------------------------------- host side

namespace {

int encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {row_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  return encode_tensor_map(map, type, 2, base, dims, strides, box, swizzle);
}

}  // namespace

int mma_op_stages(int m_pad) {
  const int64_t per = mma_stage_bytes(m_pad);
  const int64_t room = kSmemBudget - 1024 - (int64_t)kRawStages * kRawBytes - kNumBars * 8;
  // with the weights in tensor memory, its columns 256-511 hold at most 4 stages of A
  return (int)std::max<int64_t>(2, std::min<int64_t>(kMmaMaxOpStages, room / per));
}

int64_t mma_smem_bytes(int m_pad) {
  return 1024 + (int64_t)kRawStages * kRawBytes + (int64_t)mma_op_stages(m_pad) * mma_stage_bytes(m_pad) +
         kNumBars * 8;
}

int64_t mma_resident_act_bytes(int m_pad, int64_t k, int splits) {
  const int64_t KS_all = k / kMmaKStep;
  const int64_t ks_max = splits > 0 ? (KS_all + splits - 1) / splits : KS_all;  // the largest split
  return ks_max * (int64_t)m_pad * 128;
}

int64_t mma_resident_smem_bytes(int m_pad, int64_t k, int splits) {
  return 1024 + (int64_t)kRawStages * kRawBytes + mma_resident_act_bytes(m_pad, k, splits) +
         mma_resident_extra_bytes(m_pad) + kNumBars * 8;
}

bool mma_act_resident(int m_pad, int64_t k, int splits) {
  return m_pad <= kMmaTmemMaxM && k >= kMmaKStep && mma_resident_smem_bytes(m_pad, k, splits) <= kSmemBudget;
}

int launch_mma(const MmaArgs& a, cudaStream_t stream) {
  if (a.k % kMmaKStep != 0 || a.m_pad < 16 || a.m_pad > kMmaMaxM || a.m_pad % 16 != 0)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "MMA path: k must be a multiple of %d and m <= %d", kMmaKStep,
                     kMmaMaxM);
  if (a.splits < 1 || a.splits > a.k / kMmaKStep || (a.splits > 1 && !a.partials))
    return set_error(FI_ERR_INVALID_ARG, "MMA path: %d splits for k=%lld", a.splits, (long long)a.k);
  const bool resident = a.act_resident != 0;
  if (a.m_pad <= kMmaTmemMaxM && a.op_stages != kMmaMaxOpStages)
    return set_error(FI_ERR_INVALID_ARG, "MMA path: weights in tensor memory need %d operand stages, got %d",
                     kMmaMaxOpStages, a.op_stages);
  if (resident) {
    if (!mma_act_resident(a.m_pad, a.k, a.splits) || a.op_stages != kMmaMaxOpStages || a.stage_bytes != 0 ||
        (int64_t)a.act_bytes != mma_resident_act_bytes(a.m_pad, a.k, a.splits) ||
        (int64_t)a.act_extra_bytes != mma_resident_extra_bytes(a.m_pad))
      return set_error(FI_ERR_INVALID_ARG, "MMA path: resident activations do not fit m_pad=%d, k=%lld, %d splits",
                       a.m_pad, (long long)a.k, a.splits);
  } else if (a.op_stages < 2 || a.op_stages > kMmaMaxOpStages || (int64_t)a.stage_bytes != mma_stage_bytes(a.m_pad) ||
             a.act_bytes != 0 || a.act_extra_bytes != 0) {
    return set_error(FI_ERR_INVALID_ARG, "MMA path: %d operand stages of %u bytes do not match m_pad=%d", a.op_stages,
                     a.stage_bytes, a.m_pad);
  }
  CUtensorMap tmap_a, tmap_w;
  int rc = FI_OK;
  if (resident) {
    // activations: bf16 [m, k] as they come, box 64 k x m_pad rows (rows past m read as zero),
    // 128-byte swizzle: the layout of the MMA's B operand, converted in place by the kernel
    rc = encode_2d(&tmap_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.A, (uint64_t)a.k, (uint64_t)a.m, (uint64_t)a.k * 2,
                   kMmaKStep, (uint32_t)a.m_pad, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FI_OK) return rc;
  } else {
    // activations: f16 [m_pad, k], box 64 k x m_pad rows, 128-byte swizzle (the MMA's B operand)
    rc = encode_2d(&tmap_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.a16, (uint64_t)a.k, (uint64_t)a.m_pad,
                   (uint64_t)a.k * 2, kMmaKStep, (uint32_t)a.m_pad, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc != FI_OK) return rc;
  }
  // packed codes: u8 [n, k/2], box 32 bytes x 256 rows (rows past n read as zero codes)
  rc = encode_2d(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, (uint64_t)(a.k / 2), (uint64_t)a.n,
                 (uint64_t)(a.k / 2), 32, kMmaTileRows, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (rc != FI_OK) return rc;

  const bool ta = a.m_pad <= kMmaTmemMaxM;
  auto kern = ta ? mma_nvfp4_kernel<true> : mma_nvfp4_kernel<false>;
  static int configured[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return set_cuda_error("cudaGetDevice");
  if (!(configured[dev] & (ta ? 2 : 1))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget) != cudaSuccess)
      return set_cuda_error("cudaFuncSetAttribute(mma smem)");
    configured[dev] |= ta ? 2 : 1;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  if (!resident) {
    cudaLaunchConfig_t pre = {};
    pre.gridDim = dim3((unsigned)a.m_pad, (unsigned)a.splits);
    pre.blockDim = dim3(256);
    pre.stream = stream;
    pre.attrs = attr;
    pre.numAttrs = 1;
    if (cudaLaunchKernelEx(&pre, act_to_f16_kernel, a.A, a.m, a.k, a.a16, a.rs) != cudaSuccess)
      return set_cuda_error("act_to_f16_kernel launch");
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((a.n + kMmaTileRows - 1) / kMmaTileRows), (unsigned)a.splits);
  cfg.blockDim = dim3(kMmaThreads);
  // at most one CTA per SM: with the weights in tensor memory a CTA takes all 512 columns, and
  // a second CTA on the SM would wait in its allocation
  const int64_t smem = resident ? mma_resident_smem_bytes(a.m_pad, a.k, a.splits) : mma_smem_bytes(a.m_pad);
  cfg.dynamicSmemBytes = (size_t)std::max<int64_t>(smem, kSmemBudget / 2 + 4096);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a, tmap_a, tmap_w) != cudaSuccess)
    return set_cuda_error("mma_nvfp4_kernel launch");
  return FI_OK;
}

}  // namespace fi
