// C-ABI entry points: argument checks, the tactic table, the split-K workspace, launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>
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

// Device-sized parallelism: enough weight-streaming warps on every SM to keep HBM busy
// (PR #4038 measured saturation at ~20 warps/SM on SM12x and sized split-K from the device).
constexpr int kKneeWarpsPerSm = 20;
// A warp keeps at least this many 32-k chunks of a row (one full warp step) so that its
// lanes have work when the k range is divided among warps or splits.
constexpr int64_t kMinChunksPerWarp = 32;
// Shared memory per CTA the device-sized split aims for (three CTAs per SM fit).
constexpr int64_t kKneeSmemPerCta = 72 * 1024;
// Largest m the default table sends to the GEMV.
constexpr int64_t kDefaultGemvMaxM = 32;

static int gemv_default_rows(int64_t n) { return n >= 4096 ? 2 : 1; }

// Smallest power of two KW <= maxKW (and <= 8) with RG * KW * S >= target.
static int64_t auto_kw(int64_t RG, int64_t S, int64_t C, int64_t target) {
  int64_t KW = 1;
  while (KW < 8 && RG * KW * S < target && (C / S) / (KW * 2) >= kMinChunksPerWarp) KW *= 2;
  return KW;
}

// Device-sized split for rows-per-warp R: the in-CTA split KW first (no second kernel), then
// the fewest global splits S that reach the target warp count, raised until `m_fit`
// activation rows of a split fit the shared-memory staging. Depends on (n, k, SMs, m_fit).
static void gemv_knee(int64_t n, int64_t k, int sms, int64_t m_fit, int R, int64_t KW_req, int64_t* S_out,
                      int64_t* KW_out) {
  const int64_t C = k / kChunkK;
  const int64_t RG = (n + R - 1) / R;
  const int64_t target = (int64_t)kKneeWarpsPerSm * sms;
  const int64_t KW = KW_req ? KW_req : auto_kw(RG, 1, C, target);
  const int64_t want = (target + RG * KW - 1) / (RG * KW > 0 ? RG * KW : 1);
  int64_t cap = C / (kMinChunksPerWarp * KW);
  if (cap < 1) cap = 1;
  int64_t S = want < 1 ? 1 : (want > cap ? cap : want);
  while (S < C && gemv_smem_bytes(m_fit, ((C + S - 1) / S) * kChunkK, R) > kKneeSmemPerCta) ++S;
  *S_out = S;
  *KW_out = KW;
}

static int resolve(int64_t m, int64_t n, int64_t k, int64_t tactic, int num_sms, fi_tactic_info* out);

// The built-in table. m = 1, 2..8 and 9..32 are separate buckets: the tactic (and so the bits
// of a row) is the same for every m inside a bucket.
static int64_t default_tactic_impl(int64_t m, int64_t n, int64_t k, int num_sms) {
  if (m <= kDefaultGemvMaxM) {
    const int64_t m_fit = m <= 1 ? 1 : (m <= 8 ? 8 : kGemvMaxM);
    const int R = (m_fit > 16 && gemv_default_rows(n) > 2) ? 2 : gemv_default_rows(n);
    int64_t S = 1, KW = 1;
    gemv_knee(n, k, num_sms, m_fit, R, 0, &S, &KW);
    return FI_TACTIC(FI_KIND_GEMV, S, 0, R | (KW << 4));
  }
  return FI_TACTIC(FI_KIND_MMA, 1, 0, 0);
}

// GEMV variant byte: low nibble R (weight rows per warp), high nibble KW (warps per row
// group inside a CTA); 0 in either means automatic. Splits 0 = device-sized, resolved for
// m <= 32 so that the resolved S (and the bits) never depend on m.
static int resolve_gemv(int64_t m, int64_t n, int64_t k, int S_req, int ctas_req, int var,
                        int sms, fi_tactic_info* out) {
  if (m > kGemvMaxM)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "GEMV tactics support m <= %d (got m=%lld)",
                     kGemvMaxM, (long long)m);
  const int R = (var & 0xF) ? (var & 0xF) : gemv_default_rows(n);
  if (R != 1 && R != 2 && R != 4)
    return set_error(FI_ERR_INVALID_ARG, "GEMV rows per warp must be 0 (auto), 1, 2 or 4");
  if (R == 4 && m > 16)
    return set_error(FI_ERR_INVALID_ARG, "GEMV with 4 rows per warp supports m <= 16");
  const int KW_req = var >> 4;
  if (KW_req != 0 && KW_req != 1 && KW_req != 2 && KW_req != 4 && KW_req != 8)
    return set_error(FI_ERR_INVALID_ARG, "GEMV warps per row group must be 0 (auto), 1, 2, 4 or 8");
  const int64_t C = k / kChunkK;
  const int64_t RG = (n + R - 1) / R;
  int64_t KW = KW_req;
  int64_t S = S_req;
  if (S == 0) {
    gemv_knee(n, k, sms, kGemvMaxM, R, KW_req, &S, &KW);
  } else {
    if (C > 0 && S > C)
      return set_error(FI_ERR_INVALID_ARG, "splits=%lld exceeds k/32=%lld", (long long)S, (long long)C);
    if (KW == 0) KW = auto_kw(RG, S, C, (int64_t)kKneeWarpsPerSm * sms);
  }
  if (S < 1) S = 1;
  if (C > 0 && KW > C / S)
    return set_error(FI_ERR_INVALID_ARG, "warps per row group (%lld) exceeds the %lld k-chunks of a split",
                     (long long)KW, (long long)(C / S));
  const int64_t klen_max = ((C + S - 1) / S) * kChunkK;
  const int64_t smem = gemv_smem_bytes(m, klen_max, R);
  if (smem > kSmemBudget)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE,
                     "GEMV: m=%lld with k/splits=%lld needs %lld B of shared memory (> %d); use more splits",
                     (long long)m, (long long)klen_max, (long long)smem, kSmemBudget);
  int ctas = ctas_req;
  if (ctas == 0) {
    // leave room on every SM for the PDL-launched reduce when the tactic splits
    ctas = S > 1 ? 3 : 4;
    const int fit = (int)((227 * 1024) / (smem + 1024));
    if (ctas > fit) ctas = fit;
    if (ctas < 1) ctas = 1;
  }
  const int64_t NS = kGemvWarps / KW;
  const int64_t cta_rows = (RG + NS - 1) / NS;
  int64_t slots = ((int64_t)sms * ctas) / S;
  if (slots < 1) slots = 1;
  const int64_t grid_x = cta_rows < slots ? cta_rows : slots;
  out->kind = FI_KIND_GEMV;
  out->splits = (int32_t)S;
  out->ctas_per_sm = ctas;
  out->variant = (int32_t)(R | (KW << 4));
  out->grid_x = (int32_t)(grid_x > 0 ? grid_x : 1);
  out->grid_y = (int32_t)S;
  out->threads = kGemvThreads;
  out->smem_bytes = (int32_t)smem;
  out->workspace_bytes = S > 1 ? S * m * n * (int64_t)sizeof(float) : 0;
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
  if (kind == FI_KIND_MMA)
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "MMA tactics are not available in this build");
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

// ------------------------------------------------------------------ checks

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

static int mm_run(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                  uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, void* workspace,
                  size_t workspace_bytes, bool use_registered, cudaStream_t stream) {
  clear_error();
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
  if (!aligned(A, 16) || !aligned(Wq, 16)) return set_error(FI_ERR_INVALID_ARG, "A and Wq must be 16-byte aligned");
  if (!aligned(Wscale, 2) || !aligned(out, 2) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "Wscale/out must be 2-byte and gscale 4-byte aligned");
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
    GemvArgs a;
    a.A = A;
    a.Wq = Wq;
    a.Ws = Wscale;
    a.gscale = gscale;
    a.out = out;
    a.partials = partials;
    a.m = m;
    a.n = n;
    a.k = k;
    a.splits = info.splits;
    a.kw = info.variant >> 4;
    a.rows_per_warp = info.variant & 0xF;
    a.grid_x = info.grid_x;
    a.ctas_per_sm = info.ctas_per_sm;
    a.num_sms = sms;
    a.smem_bytes = info.smem_bytes;
    a.pdl = 1;
    rc = launch_gemv(a, stream);
    if (rc != FI_OK) return rc;
  } else {
    return set_error(FI_ERR_UNSUPPORTED_SHAPE, "MMA tactics are not available in this build");
  }
  if (info.splits > 1) return launch_splitk_reduce(partials, info.splits, m, n, gscale, out, true, stream);
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
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(Wscale, 8) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "W/Wq must be 16-byte, Wscale 8-byte, gscale 4-byte aligned");
  const int rc = check_arch();
  if (rc != FI_OK) return rc;
  return launch_pack(W, n, k, Wq, Wscale, gscale, reinterpret_cast<cudaStream_t>(stream));
}

int fi_mm_bf16_fp4(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                   uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, fi_stream_t stream) {
  return mm_run(A, Wq, Wscale, gscale, out, m, n, k, tactic, nullptr, 0, true,
                reinterpret_cast<cudaStream_t>(stream));
}

int fi_mm_bf16_fp4_ex(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                      uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, void* workspace,
                      size_t workspace_bytes, fi_stream_t stream) {
  return mm_run(A, Wq, Wscale, gscale, out, m, n, k, tactic, workspace, workspace_bytes, false,
                reinterpret_cast<cudaStream_t>(stream));
}

int fi_splitk_reduce(const float* partials, int64_t splits, int64_t m, int64_t n, const float* gscale,
                     uint16_t* out, fi_stream_t stream) {
  clear_error();
  if (m < 0 || n < 0) return set_error(FI_ERR_INVALID_ARG, "negative size");
  if (splits < 1 || splits > 4095) return set_error(FI_ERR_INVALID_ARG, "splits must be in [1, 4095]");
  if (m == 0 || n == 0) return FI_OK;
  if (!partials || !gscale || !out) return set_error(FI_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(partials, 16) || !aligned(out, 2) || !aligned(gscale, 4))
    return set_error(FI_ERR_INVALID_ARG, "partials must be 16-byte, out 2-byte aligned");
  const int rc = check_arch();
  if (rc != FI_OK) return rc;
  return launch_splitk_reduce(partials, (int)splits, m, n, gscale, out, false,
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
  // the split menu {1, 2, 4, 8, device-sized} for each rows-per-warp choice, plus every
  // in-CTA split for one row per warp; entries resolving to the same launch are listed once
  int64_t cand[32];
  int nc = 0;
  const int splits[] = {1, 2, 4, 8, 0};
  for (int R : {1, 2, 4})
    for (int S : splits) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, S, 0, R);
  for (int KW : {1, 2, 4, 8}) cand[nc++] = FI_TACTIC(FI_KIND_GEMV, 1, 0, 1 | (KW << 4));
  fi_tactic_info seen[32];
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

const char* fi_last_error(void) { return g_err; }

int fi_version(void) { return 100; }

}  // extern "C"
