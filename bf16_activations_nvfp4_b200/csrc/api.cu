// C-ABI entry points: argument checks, the tactic table, the split-K workspace, launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>

#include "fi_nvfp4.h"
#include "internal.h"

namespace fi {

// -------------------------------------------------------------------- errors

namespace {
thread_local char g_err[512] = "";
}

int set_error(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return status;
}

int set_cuda_error(const char* what) {
  const cudaError_t e = cudaGetLastError();
  snprintf(g_err, sizeof(g_err), "%s: %s", what, cudaGetErrorString(e));
  return FI_ERR_CUDA;
}

void clear_error() { g_err[0] = '\0'; }

// --------------------------------------------------------------- device facts

namespace {
std::mutex g_dev_mu;
int g_sms[kMaxDevices] = {};
int g_arch_ok[kMaxDevices] = {};  // 0 unknown, 1 ok, -1 unsupported
}  // namespace

static int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return set_cuda_error("cudaGetDevice");
  if (*dev < 0 || *dev >= kMaxDevices) return set_error(FI_ERR_INVALID_ARG, "device id %d out of range", *dev);
  return FI_OK;
}

int device_sm_count() {
  int dev = 0;
  if (current_device(&dev) != FI_OK) return 0;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_sms[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      set_cuda_error("cudaDeviceGetAttribute(SM count)");
      return 0;
    }
    g_sms[dev] = v;
  }
  return g_sms[dev];
}

static int check_arch() {
  int dev = 0;
  const int rc = current_device(&dev);
  if (rc != FI_OK) return rc;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return set_cuda_error("cudaDeviceGetAttribute(compute capability)");
    g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    if (g_arch_ok[dev] < 0)
      return set_error(FI_ERR_UNSUPPORTED_ARCH,
                       "device %d has compute capability %d.%d; this library is built for sm_100a (10.0)",
                       dev, major, minor);
  }
  if (g_arch_ok[dev] < 0)
    return set_error(FI_ERR_UNSUPPORTED_ARCH, "device %d is not compute capability 10.0", dev);
  return FI_OK;
}

// ----------------------------------------------------------------- tactics

// Largest m the default table sends to the GEMV. Measured on B200 (cold L2, PDL-chained
// graphs): the split-K MMA path is faster from m = 8 on every serving shape (4096 x 14336 at
// m = 8: 25.6 against 47.5 us; at m = 32: 29.6 against 176 us) and level at m = 4; the GEMV
// keeps m = 1..4.
constexpr int64_t kDefaultGemvMaxM = 4;

int gemv_geometry(int64_t m, int64_t n, int64_t k, int S, int rs_req, int ctas_per_sm, int sms, GemvGeometry* g) {
  const int64_t C = k / kChunkK;
  const int64_t nch = (C + S - 1) / S;  // chunks of the largest split
  const int ctas = ctas_per_sm > 0 ? ctas_per_sm : 1;
  const int64_t per_cta = std::min<int64_t>(kSmemBudget, (228 * 1024) / ctas - 2048);
  const int64_t a_bytes = round_up(m * ((nch + 31) / 32) * 2048, 128);
  const int64_t as_bytes = round_up(m * nch * 8, 128);
  const int64_t bar_bytes = round_up(2 * kGemvMaxStages * 8, 128);
  const int64_t fixed = a_bytes + as_bytes + bar_bytes;
  const int64_t avail = per_cta - fixed;
  // a stage: rs rows of codes, then their scales (one contiguous superset when S == 1, one
  // superset per row otherwise), as the kernel lays them out
  auto stage_of = [&](int64_t rs) {
    const int64_t scales = S == 1 ? round_up(rs * nch * 2 + 30, 16) : rs * gemv_scales_stride(nch);
    return round_up(rs * nch * 16 + scales, 128);
  };
  const int rmax = gemv_rows_per_stage_max(m);
  int64_t rs = rs_req;
  if (rs == 0) {
    rs = 1;
    while (rs * 2 <= rmax && stage_of(rs * 2) <= kGemvStageTarget) rs *= 2;
  }
  if (rs < 1 || rs > rmax || (rs & (rs - 1)) != 0)
    return set_error(FI_ERR_INVALID_ARG, "GEMV rows per stage must be a power of two in 1..%d for m=%lld", rmax,
                     (long long)m);
  const int64_t stage_bytes = stage_of(rs);
  const int64_t stages = std::min<int64_t>(kGemvMaxStages, avail > 0 ? avail / stage_bytes : 0);
  if (stages < 2)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV: m=%lld over %lld k per split leaves no room for the weight ring in shared "
                     "memory; use more splits",
                     (long long)m, (long long)(nch * kChunkK));
  int64_t gx = std::max<int64_t>(1, (int64_t)sms * ctas / S);
  if (gx > n) gx = std::max<int64_t>(1, n);
  g->pipeline = kPipeRing;
  g->threads = kGemvThreads;
  g->S = S;
  g->RS = (int)rs;
  g->stages = (int)stages;
  g->ctas_per_sm = ctas;
  g->grid_x = (int)gx;
  g->stage_bytes = stage_bytes;
  g->off_as = a_bytes;
  g->off_bar = a_bytes + as_bytes;
  g->off_ring = fixed;
  g->smem_bytes = fixed + stages * stage_bytes;
  return FI_OK;
}

// Per-warp async-copy pipeline. ctas_per_sm 1: one CTA of 16 warps per SM with the whole
// shared memory; 2: two CTAs of 8 warps per SM with half of it each. A CTA holds the split's
// activations and, per warp, NS slots of kStreamIters chunk iterations x R rows x 32 lanes x
// (16 code bytes + a 4-byte scale word). The grid never has more warps than row groups.
// Automatic choices (measured on B200 at m = 1): from n = 64 rows per SM on, two 8-warp CTAs per
// SM with four rows per item; below that, one 16-warp CTA per SM with two rows per item.
static bool stream_wide(int64_t n, int sms) { return n >= (int64_t)sms * 64; }

// overlap: CTAs sized for half an SM, but only one per SM, so that the next call's CTAs (launched
// early by programmatic dependent launch) are resident beside them and prefetch their weights.
int gemv_stream_geometry(int64_t m, int64_t n, int64_t k, int S, int r_req, int ctas_per_sm, int sms,
                         GemvGeometry* g, bool overlap) {
  const int64_t C = k / kChunkK;
  const int64_t nch = (C + S - 1) / S;  // chunks of the largest split
  // automatic CTA shape: two half-SM CTAs per SM for wide n, and at m = 1 (where the activations
  // always fit half an SM) when the 2-row groups fill two CTAs of at least 4 warps on every SM;
  // measured at m = 1: 4096 x 14336 8.78 us on 293 CTAs of 7 warps (R = 2) against 9.1 us on
  // 147 CTAs of 14; 2048 x 7168 (1024 groups) 4.98 us on 256 CTAs of 4 warps, which leave 40
  // SMs with one CTA, against 4.35 us on 147 CTAs of 7
  const bool wide = stream_wide(n, sms);
  const bool fill2 = m == 1 && (n + 1) / 2 >= (int64_t)sms * 2 * 4;
  const int ctas = overlap ? 2 : (ctas_per_sm > 0 ? ctas_per_sm : (wide || fill2 ? 2 : 1));
  if (ctas > 2) return set_error(FI_ERR_INVALID_ARG, "GEMV stream pipeline: at most 2 CTAs per SM");
  int nw = ctas == 1 ? 16 : 8;
  const int64_t budget = ctas == 1 ? kSmemBudget : kStreamHalfBudget;
  const int64_t a_bytes = round_up(m * ((nch + 31) / 32) * 2048, 128);
  const int64_t as_bytes = round_up(m * nch * 8, 128);
  const int rmax = std::min(4, gemv_rows_per_stage_max(m));  // registers: at most 4 rows per item
  int64_t r = r_req;
  if (r == 0) r = std::min(ctas == 2 && !overlap && wide ? 4 : 2, rmax);
  if (r < 1 || r > rmax || (r & (r - 1)) != 0)
    return set_error(FI_ERR_INVALID_ARG, "GEMV rows per item must be a power of two in 1..%d for m=%lld", rmax,
                     (long long)m);
  const int64_t slot = (int64_t)kStreamIters * r * kStreamCellBytes;
  const int64_t fixed = a_bytes + as_bytes;
  // Rows go to warps in whole groups of r. When the groups of a split would fill fewer than
  // its share of CTA slots, the CTAs get fewer warps (at least 4) so that the work spreads over
  // every SM (4096 x 14336 at m = 1: 2048 groups of 2 rows on 147 CTAs of 14 warps instead of
  // 128 CTAs of 16).
  const int64_t groups = (n + r - 1) / r;
  const int64_t gx_cap = std::max<int64_t>(1, (int64_t)sms * (overlap ? 1 : ctas) / S);
  if ((groups + nw - 1) / nw < gx_cap) nw = (int)std::max<int64_t>(4, (groups + gx_cap - 1) / gx_cap);
  int ns = 4;
  if (fixed + (int64_t)nw * ns * slot > budget) ns = 2;
  if (fixed + (int64_t)nw * ns * slot > budget)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV: m=%lld over %lld k per split leaves no room for the weight slots in shared memory; "
                     "use more splits",
                     (long long)m, (long long)(nch * kChunkK));
  const int64_t gx = std::max<int64_t>(1, std::min<int64_t>(gx_cap, (groups + nw - 1) / nw));
  g->pipeline = overlap ? kPipeOverlap : kPipeStream;
  g->threads = nw * 32;
  g->S = S;
  g->RS = (int)r;
  g->stages = ns;
  g->ctas_per_sm = ctas;
  g->grid_x = (int)gx;
  g->stage_bytes = slot;
  g->off_as = a_bytes;
  g->off_ring = fixed;
  g->off_bar = fixed;
  g->smem_bytes = fixed + (int64_t)nw * ns * slot;
  return FI_OK;
}

// Register pipeline: shared memory holds only the staged activations; each warp keeps
// kRegDepth chunk iterations of its rows in registers. CTAs of up to 16 warps (one per SM) or
// up to 8 (two per SM), spread over every SM like the stream pipeline's.
static int gemv_reg_geometry(int64_t m, int64_t n, int64_t k, int S, int r_req, int ctas_per_sm, int sms,
                             GemvGeometry* g) {
  const int64_t C = k / kChunkK;
  const int64_t nch = (C + S - 1) / S;
  const int ctas = ctas_per_sm > 0 ? ctas_per_sm : 1;
  if (ctas > 2) return set_error(FI_ERR_INVALID_ARG, "GEMV register pipeline: at most 2 CTAs per SM");
  int nw = ctas == 1 ? 16 : 8;
  const int64_t budget = ctas == 1 ? kSmemBudget : kStreamHalfBudget;
  const int64_t a_bytes = round_up(m * ((nch + 31) / 32) * 2048, 128);
  const int64_t as_bytes = round_up(m * nch * 8, 128);
  if (a_bytes + as_bytes > budget)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV: m=%lld over %lld k per split does not fit shared memory; use more splits", (long long)m,
                     (long long)(nch * kChunkK));
  const int rmax = std::min(2, gemv_rows_per_stage_max(m));  // the register ring of 4 rows would spill
  int64_t r = r_req ? r_req : rmax;
  if (r < 1 || r > rmax || (r & (r - 1)) != 0)
    return set_error(FI_ERR_INVALID_ARG, "GEMV rows per warp must be a power of two in 1..%d for m=%lld", rmax,
                     (long long)m);
  const int64_t groups = (n + r - 1) / r;
  const int64_t gx_cap = std::max<int64_t>(1, (int64_t)sms * ctas / S);
  if ((groups + nw - 1) / nw < gx_cap) nw = (int)std::max<int64_t>(4, (groups + gx_cap - 1) / gx_cap);
  g->pipeline = kPipeReg;
  g->threads = nw * 32;
  g->S = S;
  g->RS = (int)r;
  g->stages = kRegDepth;
  g->ctas_per_sm = ctas;
  g->grid_x = (int)std::max<int64_t>(1, std::min<int64_t>(gx_cap, (groups + nw - 1) / nw));
  g->stage_bytes = 0;
  g->off_as = a_bytes;
  g->off_bar = a_bytes + as_bytes;
  g->off_ring = a_bytes + as_bytes;
  g->smem_bytes = a_bytes + as_bytes;
  return FI_OK;
}

// Lean stream pipeline (m = 1 only): the stream pipeline's CTA shapes and row groups, with
// per-warp rings of NS slots of R rows x kLeanIters chunk iterations (codes and scales, 576
// bytes per row and iteration); a row group's last item may hold a single iteration. Needs
// k % 256 == 0 and every split a whole number of 32-chunk iterations ((k/32) % (32 S) == 0).
static int gemv_lean_geometry(int64_t m, int64_t n, int64_t k, int S, int r_req, int ctas_per_sm, int sms,
                              GemvGeometry* g) {
  if (m != 1)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV lean pipeline: m = 1 only (got m=%lld)", (long long)m);
  const int64_t C = k / kChunkK;
  if (k % 256 != 0 || C % (32 * (int64_t)S) != 0)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV lean pipeline: needs k %% 256 == 0 and k/32 a multiple of 32 * splits (k=%lld, splits=%d)",
                     (long long)k, S);
  const int64_t nch = C / S;
  const bool wide = stream_wide(n, sms);
  const bool fill2 = (n + 1) / 2 >= (int64_t)sms * 2 * 4;
  const int ctas = ctas_per_sm > 0 ? ctas_per_sm : (wide || fill2 ? 2 : 1);
  if (ctas > 2) return set_error(FI_ERR_INVALID_ARG, "GEMV lean pipeline: at most 2 CTAs per SM");
  int nw = ctas == 1 ? 16 : 8;
  const int64_t budget = ctas == 1 ? kSmemBudget : kStreamHalfBudget;
  const int64_t a_bytes = round_up(((nch + 31) / 32) * 2048, 128);
  const int64_t as_bytes = round_up(nch * 8, 128);
  int64_t r = r_req;
  if (r == 0) r = ctas == 2 && wide ? 4 : 2;
  if (r != 1 && r != 2 && r != 4)
    return set_error(FI_ERR_INVALID_ARG, "GEMV lean pipeline: 1, 2 or 4 rows per item (got %lld)", (long long)r);
  const int64_t slot = (int64_t)kLeanIters * r * 576;
  const int64_t groups = (n + r - 1) / r;
  const int64_t gx_cap = std::max<int64_t>(1, (int64_t)sms * ctas / S);
  if ((groups + nw - 1) / nw < gx_cap) nw = (int)std::max<int64_t>(4, (groups + gx_cap - 1) / gx_cap);
  const int64_t fixed = a_bytes + as_bytes;
  int ns = 4;
  if (fixed + (int64_t)nw * ns * slot > budget) ns = 2;
  if (fixed + (int64_t)nw * ns * slot > budget)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV lean pipeline: %lld k per split leave no room for the weight slots; use more splits",
                     (long long)(nch * kChunkK));
  g->pipeline = kPipeLean;
  g->threads = nw * 32;
  g->S = S;
  g->RS = (int)r;
  g->stages = ns;
  g->ctas_per_sm = ctas;
  g->grid_x = (int)std::max<int64_t>(1, std::min<int64_t>(gx_cap, (groups + nw - 1) / nw));
  g->grid_y = S;
  g->stage_bytes = slot;
  g->off_as = a_bytes;
  g->off_bar = fixed;
  g->off_ring = fixed;
  g->smem_bytes = fixed + (int64_t)nw * ns * slot;
  return FI_OK;
}

static int geometry_for(int pipe, int64_t m, int64_t n, int64_t k, int S, int r, int ctas, int sms, GemvGeometry* g) {
  if (pipe == kPipeRing) return gemv_geometry(m, n, k, S, r, ctas, sms, g);
  if (pipe == kPipeReg) return gemv_reg_geometry(m, n, k, S, r, ctas, sms, g);
  if (pipe == kPipeLean) return gemv_lean_geometry(m, n, k, S, r, ctas, sms, g);
  return gemv_stream_geometry(m, n, k, S, r, ctas, sms, g, pipe == kPipeOverlap);
}

// Device-sized split (PR #4038, Description, "What it does": the device-sized GEMV split): the fewest splits S
// that give every SM a CTA with rows to stream while `m_fit` activation rows of a split fit
// the shared-memory staging next to the weight ring. Depends on (n, k, SMs, R, m_fit) only.
static int gemv_knee(int pipe, int64_t n, int64_t k, int sms, int64_t m_fit, int rs, int ctas, int* S_out) {
  const int64_t C = k / kChunkK;
  const int64_t maxS = std::max<int64_t>(1, std::min<int64_t>(C, 4095));
  for (int64_t S = 1; S <= maxS; ++S) {
    GemvGeometry g{};
    if (geometry_for(pipe, m_fit, n, k, (int)S, rs, ctas, sms, &g) != FI_OK) continue;
    // enough: the splits' warps cover at least 40% of the SMs' warp slots (16 per SM; the ring
    // pipeline's CTAs always have 16 consumer warps). Measured on B200: idle warp slots cost
    // less than a second kernel and the partials' traffic until well below that (2048 x 7168
    // at m = 1 ran faster on 64 CTAs of 16 warps than split in two).
    const int64_t warps = (int64_t)g.grid_x * (pipe == kPipeRing ? 16 : g.threads / 32);
    const int64_t slots = pipe == kPipeRing ? (int64_t)sms * g.ctas_per_sm * 16 : (int64_t)sms * 16;
    const bool enough = warps * S * 5 >= slots * 2;
    const bool last = S == maxS || (C / (S + 1)) < 32;  // a split keeps at least one warp step
    if (enough || last) {
      *S_out = (int)S;
      clear_error();
      return FI_OK;
    }
  }
  return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV: no split count fits m=%lld in shared memory", (long long)m_fit);
}

static int resolve(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms, fi_tactic_info* out);

// The measured table (generated by the package's cold-L2 tuner, tune.py): per (n, k, SM count)
// and bucket of m, the tactic that was fastest on this GPU model. Shapes and devices it does not
// list take the built-in rules below.
struct TunedTactic {
  int64_t n, k;
  int32_t m_lo, m_hi, sms;
  int64_t tactic;
  double us;  // measured mean us per call (documentation only)
};
#include "tactic_table.inc"

static int64_t tuned_tactic(int64_t m, int64_t n, int64_t k, int sms) {
  for (const TunedTactic& e : kTunedTactics)
    if (e.n == n && e.k == k && e.sms == sms && m >= e.m_lo && m <= e.m_hi) return e.tactic;
  return -1;
}

// The built-in table. m = 1, 2..4 and 5..256 are separate buckets: the tactic (and so the bits
// of a row) is the same for every m inside a bucket.
static int64_t default_tactic_impl(int64_t m, int64_t n, int64_t k, int num_sms) {
  const int64_t tuned = tuned_tactic(m, n, k, num_sms);
  if (tuned >= 0) return tuned;
  if (m <= kDefaultGemvMaxM) {
    const int64_t m_fit = m <= 1 ? 1 : kDefaultGemvMaxM;
    // stream pipeline with its automatic CTA shape and rows per item (see gemv_stream_geometry);
    // weights of at most 12 MB take the overlapped variant (half-SM CTAs, one per SM, weights
    // prefetched into L2 while the preceding call computes). Measured on B200 at m = 1 in
    // PDL-chained graphs: 2048 x 7168 4.03 against 4.33 us, 4096 x 4096 3.73 against 4.19 us;
    // from 15 MB on the whole-SM CTAs were faster.
    // Where k % 256 != 0 the stream pipeline takes its general path (4-byte scale words, lane
    // predicates): there the register pipeline with two CTAs per SM was faster (10304 x 2688:
    // 6.60 against 7.46 us).
    // At m = 1 with k a multiple of 2048, the lean stream pipeline (measured on B200, cold L2,
    // PDL-chained graphs: 4096 x 14336 9.45-9.97 against 9.65-10.0 us, 14336 x 4096 9.26-9.37
    // against 9.4-9.6 us on different boxes).
    const bool small = n * (k / 2 + k / 16) <= ((int64_t)12 << 20);
    const bool lean = m <= 1 && k % (kChunkK * 32 * kLeanIters) == 0;
    const int pipe = small ? kPipeOverlap : (k % 256 != 0 ? kPipeReg : (lean ? kPipeLean : kPipeStream));
    const int ctas = pipe == kPipeReg ? 2 : 0;
    int S = 1;
    if (gemv_knee(pipe, n, k, num_sms, m_fit, 0, ctas, &S) != FI_OK) S = 1;
    return FI_TACTIC(FI_KIND_GEMV, S, ctas, pipe << 4);
  }
  return FI_TACTIC(FI_KIND_MMA, 0, 0, 0);  // device-sized K split
}

// GEMV variant byte: low nibble = weight rows computed together by one warp (ring pipeline:
// rows per ring stage; the others: rows per work item; 0 = automatic); high nibble = the
// pipeline (0 = automatic: stream, or ring when the activations do not fit; 1 = stream, 2 =
// ring, 3 = overlapped stream, 4 = register). Every pipeline gives the same bits for the same
// S. Splits 0 = device-sized, resolved for m <= 32 so that the resolved S (and
// the bits) never depend on m.
static int resolve_gemv(int64_t m, int64_t n, int64_t k, int S_req, int ctas_req, int var,
                        int sms, fi_tactic_info* out) {
  if (m > kGemvMaxM)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV tactics support m <= %d (got m=%lld)",
                     kGemvMaxM, (long long)m);
  const int64_t C = k / kChunkK;
  const int ctas = ctas_req;  // 0 = the pipeline's automatic choice
  const int rsel = var & 0xF;
  const bool pipe_auto = (var >> 4) == kPipeAuto;
  int pipe = pipe_auto ? kPipeStream : var >> 4;
  if (var < 0 || pipe > kPipeLean || rsel > 8)
    return set_error(FI_ERR_INVALID_ARG,
                     "GEMV variant 0x%x: rows must be 0, 1, 2, 4 or 8 and the pipeline 0 to 5", var);
  int S = S_req;
  if (S == 0) {
    // the lean pipeline takes m = 1 only, so its split is sized for one activation row
    const int rc = gemv_knee(pipe, n, k, sms, pipe == kPipeLean ? 1 : kGemvMaxM, 0, ctas, &S);
    if (rc != FI_OK) return rc;
  } else if (C > 0 && S > C) {
    return set_error(FI_ERR_INVALID_ARG, "splits=%lld exceeds k/32=%lld", (long long)S, (long long)C);
  }
  GemvGeometry g{};
  if (C == 0) {  // k == 0: nothing to stream; the caller writes zeros
    memset(&g, 0, sizeof(g));
    g.pipeline = pipe;
    g.S = 1;
    g.RS = 1;
    g.ctas_per_sm = ctas ? ctas : 1;
    g.grid_x = 1;
    g.threads = pipe == kPipeRing ? kGemvThreads : kStreamMaxThreads;
  } else {
    int rc = FI_ERR_UNSUPPORTED_SHAPE;
    // the automatic pipeline at m = 1 with a K split: each warp's share of a split is short, and
    // more weight bytes per warp item pay. Where k % 256 != 0 the register pipeline (two rows,
    // two CTAs per SM unless asked otherwise), else the stream pipeline with four rows per item;
    // only where those row groups, over all splits, still give every SM at least 4 warps (as on
    // the serving shapes, n >= 2048, that the measurement covers). Measured on B200 at S in
    // {2, 4, 8}: 3-22% less time per call than two rows per stream item, never more than 1%
    // slower. Same bits: only the pipeline changes.
    const bool reg_rule = k % 256 != 0;
    const int64_t rule_warps = (n + (reg_rule ? 1 : 3)) / (reg_rule ? 2 : 4) * S;
    // at m = 1 the automatic pipeline is the lean stream pipeline wherever its whole items fit
    // the split (measured on B200 at S = 1: 4096 x 14336 9.45 against 10.0 us, 14336 x 4096
    // 9.26 against 9.6 us); the bits are those of any other pipeline at the same S
    if (pipe_auto && m == 1) {
      rc = geometry_for(kPipeLean, m, n, k, S, rsel, ctas, sms, &g);
      if (rc != FI_OK) clear_error();
    }
    if (rc != FI_OK && pipe_auto && m == 1 && S > 1 && rsel == 0 && rule_warps >= 4 * (int64_t)sms) {
      rc = reg_rule ? geometry_for(kPipeReg, m, n, k, S, 0, ctas ? ctas : 2, sms, &g)
                    : geometry_for(kPipeStream, m, n, k, S, 4, ctas, sms, &g);
      if (rc != FI_OK) clear_error();
    }
    if (rc != FI_OK) rc = geometry_for(pipe, m, n, k, S, rsel, ctas, sms, &g);
    // the automatic pipeline takes the ring (a whole SM's shared memory) when the activations
    // do not fit the stream pipeline's half SM; both give the same bits for the same S
    if (rc == FI_ERR_UNSUPPORTED_SHAPE && pipe_auto) {
      rc = geometry_for(kPipeRing, m, n, k, S, rsel, ctas, sms, &g);
      if (rc == FI_OK) clear_error();
    }
    if (rc != FI_OK) return rc;
  }
  out->kind = FI_KIND_GEMV;
  out->splits = g.S;
  out->ctas_per_sm = g.ctas_per_sm;
  out->variant = g.RS | (g.pipeline << 4);
  out->grid_x = g.grid_x;
  out->grid_y = g.S;
  out->threads = g.threads;
  out->smem_bytes = (int32_t)g.smem_bytes;
  out->workspace_bytes = g.S > 1 ? (int64_t)g.S * m * n * (int64_t)sizeof(float) : 0;
  return FI_OK;
}

// MMA tactic: splits 1..k/64 (0 = device-sized), CTAs per SM 0 or 1, variant 0 (automatic), 1
// (activations converted by a prepass kernel into the workspace) or 2 (converted by the kernel
// into shared memory, "resident"; only where the split's slice fits, m <= 128). Every CTA then
// converts its split's slice while its decode warps start on the weights; that saves the
// prepass launch (about 3 us in a chained sequence of calls on B200) but costs the CTA time in
// proportion to its rows x steps, once per wave. Measured on B200 (resident against prepass,
// us per call): 4096 x 4096, S = 8: 9.5 / 10.9 at m = 4, 10.0 / 11.0 at m = 8, 11.0 / 11.7 at
// m = 16; 4096 x 14336, S = 8 (28 steps): 18.9 / 20.1 at m = 4, 19.6 / 20.4 at m = 8, 22.0 /
// 21.2 at m = 16, 26.6 / 23.0 at m = 32; 2048 x 7168, S = 8: 11.7 / 12.5 at m = 4, 14.8 / 12.9
// at m = 16; 14336 x 4096, S = 2 (32 steps): 20.7 / 20.3 at m = 8. So automatic takes it for
// one-wave grids (tiles x S <= SMs) with m <= 8 and at most 28 steps per split. Needs m <= 256
// and k a multiple of 64; the workspace holds the f16
// activations and their (row, split) scales in prepass mode, then the [S, m, n] fp32 partials
// when S > 1. Both modes give the same bits.
static int resolve_mma(int64_t m, int64_t n, int64_t k, int S_req, int ctas_req, int var, int sms,
                       fi_tactic_info* out) {
  if (m > kMmaMaxM)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "MMA tactics support m <= %d (got m=%lld)", kMmaMaxM, (long long)m);
  if (k % kMmaKStep != 0)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "MMA tactics need k to be a multiple of %d (got k=%lld)", kMmaKStep,
                     (long long)k);
  if (ctas_req > 1 || var > 2)
    return set_error(FI_ERR_INVALID_ARG, "MMA tactics take CTAs per SM 0/1 and variant 0, 1 or 2");
  const int64_t tiles = std::max<int64_t>(1, (n + kMmaTileRows - 1) / kMmaTileRows);
  const int64_t KS = k / kMmaKStep;
  int64_t S = S_req;
  if (S > 1 && S > KS)
    return set_error(FI_ERR_INVALID_ARG, "splits=%lld exceeds k/%d=%lld", (long long)S, kMmaKStep, (long long)KS);
  if (S == 0) {
    // device-sized split: one CTA per SM, so a launch of tiles * S CTAs takes ceil(tiles * S /
    // sms) waves of ceil(KS / S) steps plus about 4 steps of per-CTA start and epilogue. A
    // split adds 3 steps for the reduce launch and the partials' write and read (2 S m n 4
    // bytes at about 4 MB per step, a step being about 0.6 us measured on B200). Take the S
    // (1..16) of least cost. The partials are costed at m = kMmaMaxM whatever the call's m, so
    // that S (and with it a row's bits) depends on (n, k, SMs) alone: the device-sized code is
    // batch-invariant like every other tactic code.
    S = 1;
    double best = -1.0;
    const double m_cost = (double)kMmaMaxM;
    for (int64_t c = 1; c <= std::min<int64_t>(16, std::max<int64_t>(1, KS)); ++c) {
      const double cost = (double)((tiles * c + sms - 1) / sms) * (double)((KS + c - 1) / c + 4) +
                          (c > 1 ? 3.0 + 2.0 * (double)c * m_cost * (double)n * 4.0 / 4.0e6 : 0.0);
      if (best < 0 || cost < best) {
        best = cost;
        S = c;
      }
    }
  }
  if (S < 1) S = 1;
  const int m_pad = mma_m_pad(std::max<int64_t>(m, 1));
  const bool fits = mma_act_resident(m_pad, k, (int)S);
  if (var == 2 && !fits)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "MMA resident activations: m=%lld rows of %lld k over %lld splits do not fit shared memory",
                     (long long)m, (long long)k, (long long)S);
  const int64_t steps = (KS + S - 1) / S;
  const bool resident = var == 2 || (var == 0 && fits && tiles * S <= sms && m <= 8 && steps <= 28);
  out->kind = FI_KIND_MMA;
  out->splits = (int32_t)S;
  out->ctas_per_sm = 1;
  out->variant = resident ? 2 : 1;
  out->grid_x = (int32_t)tiles;
  out->grid_y = (int32_t)S;
  out->threads = kMmaThreads;
  out->smem_bytes = (int32_t)(resident ? mma_resident_smem_bytes(m_pad, k, (int)S) : mma_smem_bytes(m_pad));
  if (m <= 0 || k <= 0)
    out->workspace_bytes = 0;
  else if (resident)
    out->workspace_bytes = S > 1 ? S * m * n * 4 : 0;
  else
    out->workspace_bytes = S > 1 ? mma_partials_offset(m, k, S) + S * m * n * 4 : mma_workspace_bytes(m, k, S);
  return FI_OK;
}

static int resolve(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms, fi_tactic_info* out) {
  if (m < 0 || n < 0 || k < 0) return set_error(FI_ERR_INVALID_ARG, "negative size");
  if (k % 32 != 0) return set_error(FI_ERR_UNSUPPORTED_SHAPE, "k=%lld is not a multiple of 32", (long long)k);
  if (num_sms <= 0) return set_error(FI_ERR_INVALID_ARG, "SM count unavailable");
  if (tactic == FI_TACTIC_DEFAULT) tactic = default_tactic_impl(m, n, k, num_sms);
  if (tactic < 0 || tactic >= ((int64_t)1 << 28))
    return set_error(FI_ERR_INVALID_ARG, "invalid tactic code %lld", (long long)tactic);
  const int kind = FI_TACTIC_KIND(tactic);
  const int S = FI_TACTIC_SPLITS(tactic);
  const int ctas = FI_TACTIC_CTAS(tactic);
  const int var = FI_TACTIC_VARIANT(tactic);
  memset(out, 0, sizeof(*out));
  if (kind == FI_KIND_GEMV) return resolve_gemv(m, n, k, S, ctas, var, num_sms, out);
  if (kind == FI_KIND_MMA) return resolve_mma(m, n, k, S, ctas, var, num_sms, out);
  return set_error(FI_ERR_INVALID_ARG, "unknown tactic kind %d", kind);
}

static int sms_or_device(int num_sms) {
  if (num_sms > 0) return num_sms;
  return device_sm_count();
}

// -------------------------------------------------------------- workspace

namespace {
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  bool owned = false;
};
std::mutex g_ws_mu;
Workspace g_ws[kMaxDevices];
}  // namespace

static int get_workspace(size_t need, cudaStream_t stream, void** ptr) {
  int dev = 0;
  int rc = current_device(&dev);
  if (rc != FI_OK) return rc;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace& w = g_ws[dev];
  if (w.bytes >= need && w.ptr) {
    *ptr = w.ptr;
    return FI_OK;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return set_cuda_error("cudaStreamIsCapturing");
  if (cap != cudaStreamCaptureStatusNone)
    return set_error(FI_ERR_WORKSPACE,
                     "split-K needs %zu B of workspace; register one with fi_set_workspace before capturing",
                     need);
  if (!w.owned && w.ptr)
    return set_error(FI_ERR_WORKSPACE, "registered workspace has %zu B, the call needs %zu B", w.bytes, need);
  if (w.owned && w.ptr) {
    if (cudaFree(w.ptr) != cudaSuccess) return set_cuda_error("cudaFree(workspace)");
    w.ptr = nullptr;
    w.bytes = 0;
  }
  size_t bytes = need < ((size_t)16 << 20) ? ((size_t)16 << 20) : need;
  if (cudaMalloc(&w.ptr, bytes) != cudaSuccess) {
    w.ptr = nullptr;
    return set_cuda_error("cudaMalloc(workspace)");
  }
  w.bytes = bytes;
  w.owned = true;
  *ptr = w.ptr;
  return FI_OK;
}

// ------------------------------------------------------------------ test hooks

namespace {
// launches whose producer warp is told to issue nothing (consumer waits then time out)
std::atomic<int> g_debug_stall_launches{0};
// limit of every mbarrier wait inside the kernels
std::atomic<uint64_t> g_wait_timeout_ns{1000000000ull};
}  // namespace

// ------------------------------------------------------------------ checks

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static int mm_run(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                  uint16_t* out, int out_dtype, int64_t m, int64_t n, int64_t k, int64_t tactic, void* workspace,
                  size_t workspace_bytes, bool use_registered, cudaStream_t stream) {
  clear_error();
  if (out_dtype != FI_DTYPE_BF16 && out_dtype != FI_DTYPE_F16)
    return set_error(FI_ERR_INVALID_ARG, "out_dtype %d is neither FI_DTYPE_BF16 nor FI_DTYPE_F16", out_dtype);
  const bool out_f16 = out_dtype == FI_DTYPE_F16;
  if (m < 0 || n < 0 || k < 0) return set_error(FI_ERR_INVALID_ARG, "negative size");
  if (k % 32 != 0) return set_error(FI_ERR_UNSUPPORTED_SHAPE, "k=%lld is not a multiple of 32", (long long)k);
  if (m == 0 || n == 0) return FI_OK;
  if (k == 0) {  // the empty sum: out = 0; A and the weights are empty and may be null
    if (!out) return set_error(FI_ERR_INVALID_ARG, "null pointer argument");
    int rc0 = check_arch();
    if (rc0 != FI_OK) return rc0;
    if (cudaMemsetAsync(out, 0, (size_t)(m * n) * sizeof(uint16_t), stream) != cudaSuccess)
      return set_cuda_error("cudaMemsetAsync(out)");
    return FI_OK;
  }
  if (!A || !Wq || !Wscale || !gscale || !out) return set_error(FI_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(A, 16) || !aligned(Wq, 16) || !aligned(Wscale, 16))
    return set_error(FI_ERR_INVALID_ARG, "A, Wq and Wscale must be 16-byte aligned");
  if (!aligned(out, 2) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "out must be 2-byte and gscale 4-byte aligned");
  int rc = check_arch();
  if (rc != FI_OK) return rc;
  const int sms = device_sm_count();
  if (sms <= 0) return FI_ERR_CUDA;
  fi_tactic_info info;
  rc = resolve(m, n, k, tactic, sms, &info);
  if (rc != FI_OK) return rc;
  float* partials = nullptr;
  if (info.workspace_bytes > 0) {
    const size_t need = (size_t)info.workspace_bytes;
    if (use_registered) {
      void* p = nullptr;
      rc = get_workspace(need, stream, &p);
      if (rc != FI_OK) return rc;
      partials = static_cast<float*>(p);
    } else {
      if (!workspace || workspace_bytes < need)
        return set_error(FI_ERR_WORKSPACE, "workspace of %zu B given, %zu B needed", workspace_bytes, need);
      if (!aligned(workspace, 256)) return set_error(FI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
      partials = static_cast<float*>(workspace);
    }
  }
  if (info.kind == FI_KIND_GEMV) {
    GemvGeometry g{};
    rc = geometry_for(info.variant >> 4, m, n, k, info.splits, info.variant & 0xF, info.ctas_per_sm, sms, &g);
    if (rc != FI_OK) return rc;
    GemvArgs a;
    memset(&a, 0, sizeof(a));
    a.A = A;
    a.Wq = Wq;
    a.Ws = Wscale;
    a.gscale = gscale;
    a.out = out;
    a.out_f16 = out_f16 ? 1 : 0;
    a.partials = partials;
    a.m = m;
    a.n = n;
    a.k = k;
    a.pipeline = g.pipeline;
    a.splits = g.S;
    a.rows_per_stage = g.RS;
    a.stages = g.stages;
    a.grid_x = g.grid_x;
    a.threads = g.threads;
    a.pdl = 1;
    // whole aligned 16-byte scale pieces per row and iteration: k % 256 == 0 and every split
    // boundary on a multiple of 8 chunks
    a.scale16 = k % 256 == 0 && (k / kChunkK) % (8 * (int64_t)g.S) == 0 ? 1 : 0;
    // overlapped pipeline: weights that fit the L2 with room to spare (two consecutive calls'
    // worth) are prefetched into it whole at kernel start, while the preceding call computes
    a.prefetch_l2 = g.pipeline == kPipeOverlap && n * (k / 2 + k / 16) <= ((int64_t)40 << 20) ? 1 : 0;
    a.debug_stall = g_debug_stall_launches > 0 ? 1 : 0;
    if (g_debug_stall_launches > 0) --g_debug_stall_launches;
    a.stage_bytes = g.stage_bytes;
    a.off_as = g.off_as;
    a.off_bar = g.off_bar;
    a.off_ring = g.off_ring;
    a.smem_bytes = g.smem_bytes;
    a.timeout_ns = g_wait_timeout_ns;
    rc = launch_gemv(a, stream);
    if (rc != FI_OK) return rc;
  } else {
    MmaArgs a;
    memset(&a, 0, sizeof(a));
    a.A = A;
    a.Wq = Wq;
    a.Ws = Wscale;
    a.gscale = gscale;
    a.out = out;
    a.out_f16 = out_f16 ? 1 : 0;
    uint8_t* ws = reinterpret_cast<uint8_t*>(partials);
    a.m = m;
    a.n = n;
    a.k = k;
    a.m_pad = mma_m_pad(m);
    a.splits = info.splits;
    a.act_resident = info.variant == 2 ? 1 : 0;
    if (a.act_resident) {
      // the kernel converts the activations into shared memory: the workspace is the partials
      a.partials = reinterpret_cast<float*>(ws);
      a.op_stages = kMmaMaxOpStages;
      a.stage_bytes = 0;
      a.act_bytes = (uint32_t)mma_resident_act_bytes(a.m_pad, k, info.splits);
      a.act_extra_bytes = (uint32_t)mma_resident_extra_bytes(a.m_pad);
    } else {
      a.a16 = reinterpret_cast<uint16_t*>(ws);
      a.rs = reinterpret_cast<float*>(ws + mma_rs_offset(m, k));
      a.partials = reinterpret_cast<float*>(ws + mma_partials_offset(m, k, info.splits));
      a.op_stages = mma_op_stages(a.m_pad);
      a.stage_bytes = (uint32_t)mma_stage_bytes(a.m_pad);
    }
    a.debug_stall = g_debug_stall_launches > 0 ? 1 : 0;
    if (g_debug_stall_launches > 0) --g_debug_stall_launches;
    a.err = device_error_word();
    if (!a.err) return set_cuda_error("cudaGetSymbolAddress(device error word)");
    a.timeout_ns = g_wait_timeout_ns;
    rc = launch_mma(a, stream);
    if (rc != FI_OK) return rc;
    if (info.splits > 1)
      return launch_splitk_reduce(a.partials, info.splits, m, n, gscale, out, out_f16, true, stream);
    return FI_OK;
  }
  if (info.splits > 1) return launch_splitk_reduce(partials, info.splits, m, n, gscale, out, out_f16, true, stream);
  return FI_OK;
}

}  // namespace fi

using namespace fi;

extern "C" {

int fi_nvfp4_pack_weights(const float* W, int64_t n, int64_t k, uint8_t* Wq, uint8_t* Wscale,
                          float* gscale, fi_stream_t stream) {
  clear_error();
  if (n < 0 || k < 0) return set_error(FI_ERR_INVALID_ARG, "negative size");
  if (k % 16 != 0) return set_error(FI_ERR_UNSUPPORTED_SHAPE, "k=%lld is not a multiple of 16", (long long)k);
  if (!gscale) return set_error(FI_ERR_INVALID_ARG, "gscale must not be null");
  if (n * k > 0 && (!W || !Wq || !Wscale)) return set_error(FI_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(Wscale, 16) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "W, Wq and Wscale must be 16-byte, gscale 4-byte aligned");
  const int rc = check_arch();
  if (rc != FI_OK) return rc;
  return launch_pack(W, n, k, Wq, Wscale, gscale, reinterpret_cast<cudaStream_t>(stream));
}

int fi_mm_bf16_fp4(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                   uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, fi_stream_t stream) {
  return mm_run(A, Wq, Wscale, gscale, out, FI_DTYPE_BF16, m, n, k, tactic, nullptr, 0, true,
                reinterpret_cast<cudaStream_t>(stream));
}

int fi_mm_bf16_fp4_ex(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                      uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, void* workspace,
                      size_t workspace_bytes, fi_stream_t stream) {
  return mm_run(A, Wq, Wscale, gscale, out, FI_DTYPE_BF16, m, n, k, tactic, workspace, workspace_bytes, false,
                reinterpret_cast<cudaStream_t>(stream));
}

int fi_mm_bf16_fp4_out(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                       uint16_t* out, int out_dtype, int64_t m, int64_t n, int64_t k, int64_t tactic,
                       void* workspace, size_t workspace_bytes, fi_stream_t stream) {
  return mm_run(A, Wq, Wscale, gscale, out, out_dtype, m, n, k, tactic, workspace, workspace_bytes,
                workspace == nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int fi_splitk_reduce(const float* partials, int64_t splits, int64_t m, int64_t n, const float* gscale,
                     uint16_t* out, fi_stream_t stream) {
  return fi_splitk_reduce_out(partials, splits, m, n, gscale, out, FI_DTYPE_BF16, stream);
}

int fi_splitk_reduce_out(const float* partials, int64_t splits, int64_t m, int64_t n, const float* gscale,
                         uint16_t* out, int out_dtype, fi_stream_t stream) {
  clear_error();
  if (out_dtype != FI_DTYPE_BF16 && out_dtype != FI_DTYPE_F16)
    return set_error(FI_ERR_INVALID_ARG, "out_dtype %d is neither FI_DTYPE_BF16 nor FI_DTYPE_F16", out_dtype);
  if (m < 0 || n < 0) return set_error(FI_ERR_INVALID_ARG, "negative size");
  if (splits < 1 || splits > 4095) return set_error(FI_ERR_INVALID_ARG, "splits must be in [1, 4095]");
  if (m == 0 || n == 0) return FI_OK;
  if (!partials || !gscale || !out) return set_error(FI_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(partials, 16) || !aligned(out, 2) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "partials must be 16-byte, out 2-byte aligned");
  const int rc = check_arch();
  if (rc != FI_OK) return rc;
  return launch_splitk_reduce(partials, (int)splits, m, n, gscale, out, out_dtype == FI_DTYPE_F16, false,
                              reinterpret_cast<cudaStream_t>(stream));
}

int fi_resolve_tactic(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms, fi_tactic_info* info) {
  clear_error();
  if (!info) return set_error(FI_ERR_INVALID_ARG, "info must not be null");
  const int sms = sms_or_device(num_sms);
  if (sms <= 0) return set_error(FI_ERR_CUDA, "no device to query the SM count from");
  return resolve(m, n, k, tactic, sms, info);
}

int64_t fi_default_tactic(int64_t m, int64_t n, int64_t k, int num_sms) {
  clear_error();
  const int sms = sms_or_device(num_sms);
  if (sms <= 0) return set_error(FI_ERR_CUDA, "no device to query the SM count from");
  return default_tactic_impl(m, n, k, sms);
}

int fi_list_tactics(int64_t m, int64_t n, int64_t k, int num_sms, int64_t* out, int cap) {
  clear_error();
  const int sms = sms_or_device(num_sms);
  if (sms <= 0) return set_error(FI_ERR_CUDA, "no device to query the SM count from");
  // the split menu {1, 2, 4, 8, device-sized} on the stream and ring pipelines, each with the
  // automatic row count and with one and two rows per warp; the stream pipeline also with two
  // CTAs per SM; the overlapped and register pipelines; the MMA. Entries resolving to the same
  // launch are listed once
  int64_t cand[64];
  int nc = 0;
  const int splits[] = {1, 2, 4, 8, 0};
  for (int pipe : {kPipeStream, kPipeRing})
    for (int R : {0, 1, 2})
      for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 0, R | (pipe << 4));
  for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 2, kPipeStream << 4);
  for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 0, kPipeOverlap << 4);
  for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 0, kPipeReg << 4);
  for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 0, kPipeLean << 4);
  for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_MMA, S, 0, 0);
  fi_tactic_info seen[64];
  int nseen = 0, count = 0;
  for (int c = 0; c < nc; ++c) {
    fi_tactic_info info;
    if (resolve(m, n, k, cand[c], sms, &info) != FI_OK) continue;
    bool dup = false;
    for (int i = 0; i < nseen; ++i)
      dup |= seen[i].kind == info.kind && seen[i].splits == info.splits && seen[i].variant == info.variant &&
             seen[i].ctas_per_sm == info.ctas_per_sm;
    if (dup) continue;
    seen[nseen++] = info;
    if (count < cap && out) out[count] = cand[c];
    ++count;
  }
  clear_error();
  return count;
}

size_t fi_mm_workspace_bytes(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms) {
  const int sms = sms_or_device(num_sms);
  if (sms <= 0) return 0;
  fi_tactic_info info;
  if (resolve(m, n, k, tactic, sms, &info) != FI_OK) return 0;
  return (size_t)info.workspace_bytes;
}

int fi_set_workspace(void* ptr, size_t bytes) {
  clear_error();
  if ((ptr == nullptr) != (bytes == 0)) return set_error(FI_ERR_INVALID_ARG, "ptr and bytes must both be set or both be 0");
  if (ptr && !aligned(ptr, 256)) return set_error(FI_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  int dev = 0;
  const int rc = current_device(&dev);
  if (rc != FI_OK) return rc;
  std::lock_guard<std::mutex> lk(g_ws_mu);
  Workspace& w = g_ws[dev];
  if (w.owned && w.ptr && cudaFree(w.ptr) != cudaSuccess) return set_cuda_error("cudaFree(workspace)");
  w.ptr = ptr;
  w.bytes = bytes;
  w.owned = false;
  return FI_OK;
}

int fi_get_device_error(unsigned* code) {
  clear_error();
  if (!code) return set_error(FI_ERR_INVALID_ARG, "code must not be null");
  *code = 0;
  const int rc = check_arch();
  if (rc != FI_OK) return rc;
  return gemv_read_error(code);
}

int fi_debug_set(int key, int64_t value) {
  clear_error();
  switch (key) {
    case FI_DEBUG_STALL_PRODUCER:
      if (value < 0) return set_error(FI_ERR_INVALID_ARG, "launch count must be >= 0");
      g_debug_stall_launches = (int)value;
      return FI_OK;
    case FI_DEBUG_WAIT_TIMEOUT_NS:
      if (value <= 0) return set_error(FI_ERR_INVALID_ARG, "timeout must be > 0 ns");
      g_wait_timeout_ns = (uint64_t)value;
      return FI_OK;
    default:
      return set_error(FI_ERR_INVALID_ARG, "unknown debug key %d", key);
  }
}

const char* fi_last_error(void) { return g_err; }

int fi_version(void) { return 100; }

}  // extern "C"
