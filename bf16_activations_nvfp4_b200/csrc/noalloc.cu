// fi_mm_bf16_fp4 for callers that must not allocate device memory.
//
// The split-K tactics need fp32 partials in global memory. fi_mm_bf16_fp4 allocates that
// workspace with cudaMalloc on first use and fi_mm_bf16_fp4_ex takes one from the caller, but
// some callers can do neither: an operator plugin inside a serving engine that has reserved
// all device memory for weights and the KV cache up front (an extra cudaMalloc fails, or
// fragments the pool the engine manages), or a component whose memory plan is fixed when the
// process starts and which owns no buffer it could lend. For them this file keeps the partials
// in a static device array that is part of the library image: every GPU that loads the library
// holds kNoAllocScratchBytes of it until the process exits, and no call allocates anything.
//
// Host code cannot use the array's name as a device address (on the host it names a stand-in
// object), so the entry point looks up the device address once per device with
// cudaGetSymbolAddress, with that device current, and passes that pointer to the kernels.
#include <cstdint>
#include <mutex>

#include "fi_nvfp4.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = FI_NOALLOC_SCRATCH_BYTES;
static_assert(kNoAllocScratchBytes % 256 == 0, "scratch size must keep 256-byte granularity");

}  // namespace

// The shared split-K scratch: at most kNoAllocScratchBytes / 4 fp32 partials (splits * m * n).
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_addr[fi::kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up on first use).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fi::set_cuda_error("cudaGetDevice");
  if (dev < 0 || dev >= fi::kMaxDevices)
    return fi::set_error(FI_ERR_INVALID_ARG, "device %d is beyond the library's limit of %d devices", dev,
                         fi::kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return fi::set_error(FI_ERR_CUDA, "cudaGetSymbolAddress(no-alloc scratch) on device %d: %s", dev,
                           cudaGetErrorString(e));
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FI_OK;
}

}  // namespace

extern "C" {

int fi_mm_bf16_fp4_noalloc(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, const float* gscale,
                           uint16_t* out, int64_t m, int64_t n, int64_t k, int64_t tactic, fi_stream_t stream) {
  // Empty problems, k == 0 and invalid sizes need no scratch: the regular checks answer them.
  if (m <= 0 || n <= 0 || k <= 0 || k % 32 != 0)
    return fi_mm_bf16_fp4_ex(A, Wq, Wscale, gscale, out, m, n, k, tactic, nullptr, 0, stream);
  // The default tactic whose scratch would not fit takes, with the same kind, the largest
  // split below its own that fits (the split changes the bits, as any split does).
  // Validity comes from fi_resolve_tactic: a single-split GEMV is valid with no scratch at all.
  // A GEMV keeps the default's pipeline where that fits the smaller split, else takes the
  // automatic pipeline (which falls back to the producer-warp ring when the activations of a
  // longer split do not fit the other pipelines' shared memory); the bits depend on S only.
  if (tactic == FI_TACTIC_DEFAULT && fi_mm_workspace_bytes(m, n, k, tactic, 0) > kNoAllocScratchBytes) {
    fi_tactic_info info;
    if (fi_resolve_tactic(m, n, k, tactic, 0, &info) == FI_OK) {
      for (int S = info.splits - 1; S >= 1 && tactic == FI_TACTIC_DEFAULT; --S) {
        const int pipe_bits = info.kind == FI_KIND_GEMV ? (info.variant >> 4) << 4 : 0;
        for (int v : {pipe_bits, 0}) {
          const int64_t t = FI_TACTIC(info.kind, S, 0, v);
          fi_tactic_info ti;
          if (fi_resolve_tactic(m, n, k, t, 0, &ti) == FI_OK &&
              (size_t)ti.workspace_bytes <= kNoAllocScratchBytes) {
            tactic = t;
            break;
          }
        }
      }
    }
  }
  // Refuse, before any launch, a call whose partials would not fit the static scratch. (An
  // invalid tactic reports 0 here and is rejected with its own message below.)
  const size_t need = fi_mm_workspace_bytes(m, n, k, tactic, 0);
  if (need > kNoAllocScratchBytes)
    return fi::set_error(FI_ERR_WORKSPACE,
                         "split-K partials of this call need %zu B, but the allocation-free entry point's static "
                         "scratch holds %zu B (splits * m * n <= %zu); use fewer splits or fi_mm_bf16_fp4_ex",
                         need, kNoAllocScratchBytes, kNoAllocScratchBytes / sizeof(float));
  void* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != FI_OK) return rc;
  return fi_mm_bf16_fp4_ex(A, Wq, Wscale, gscale, out, m, n, k, tactic, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
