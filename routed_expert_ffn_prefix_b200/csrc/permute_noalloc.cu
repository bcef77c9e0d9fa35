// permute_noalloc.cu -- moe_permute for callers that cannot allocate device memory.
//
// Some callers can't hand the library a workspace: a serving loop that
// reserves all device memory at start-up and forbids allocation afterwards,
// a plugin running inside another framework that owns every device
// allocation, or code that must not trigger the implicit device-wide
// synchronisation cudaMalloc/cudaFree can cause.  This entry point runs the
// same permutation kernels as moe_permute, with their scratch (the
// per-block expert histograms) in a fixed-size array compiled into the
// library instead of a caller-provided workspace.
#include <mutex>

#include "kernels.h"

namespace {

constexpr long long kNoallocMaxSlots = 131072;  // T * k
// Per-block histograms for the largest accepted problem: one row of E counts
// per block of kPermuteChunk slots, 128 rows x 1024 experts = 128 Ki int32
// (512 KiB), resident on every device that loads the library until the
// process exits.
constexpr size_t kScratchInts =
    (size_t)((kNoallocMaxSlots + moe::kPermuteChunk - 1) / moe::kPermuteChunk) * moe::kMaxExperts;
static_assert(kScratchInts == 128u * 1024u, "scratch sized for 131072 slots over 1024 experts");

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

// The device address of the array, looked up per device and per context:
// the host-side symbol is only a stand-in, never a device address, and a
// device reset (cudaDeviceReset) reloads the library's module in a new
// context, which can move the array.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct Cached {
  unsigned long long ctx_id;
  int32_t* addr;
};
constexpr int kDevices = moe::kMaxDevices;
std::mutex g_mutex;
Cached g_cache[kDevices] = {};
CtxGetCurrentFn g_get_ctx = nullptr;
CtxGetIdFn g_get_id = nullptr;

bool driver_fns() {
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_ctx = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return g_get_ctx != nullptr && g_get_id != nullptr;
}

// Device address of the scratch array for device `dev` (current), looked up
// with cudaGetSymbolAddress the first time a context of that device calls.
moe_status_t scratch_address(int dev, int32_t** out) {
  if (dev < 0 || dev >= kDevices) return MOE_ERR_INVALID_ARG;
  if (!driver_fns()) return MOE_ERR_CUDA;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr || g_get_id(ctx, &id) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  Cached& c = g_cache[dev];
  if (c.addr == nullptr || c.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) {
      c = Cached{};
      return MOE_ERR_CUDA;
    }
    c = Cached{id, static_cast<int32_t*>(p)};
  }
  *out = c.addr;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_ids, int T, int E, int k, int32_t* counts,
                                            int32_t* offsets, int32_t* sorted_token_ids, int32_t* inv_perm,
                                            void* stream) {
  if (!topk_ids || !counts || !offsets || !sorted_token_ids || !inv_perm) return MOE_ERR_INVALID_ARG;
  // The library's own limits, as moe_permute applies them.
  if (T < 1 || E < 1 || E > moe::kMaxExperts || k < 1 || k > E || k > moe::kMaxK) return MOE_ERR_INVALID_ARG;
  const uintptr_t mis = (reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(counts) |
                         reinterpret_cast<uintptr_t>(offsets) | reinterpret_cast<uintptr_t>(sorted_token_ids) |
                         reinterpret_cast<uintptr_t>(inv_perm)) & 15u;
  if (mis) return MOE_ERR_ALIGNMENT;
  // Batches beyond the built-in scratch are refused before anything is enqueued.
  if ((long long)T * k > kNoallocMaxSlots) return MOE_ERR_WORKSPACE;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_ARCH;
  int32_t* scratch = nullptr;
  const moe_status_t st = scratch_address(dev, &scratch);
  if (st != MOE_OK) return st;
  // Every histogram row the kernels read is written first in the same call,
  // so nothing has to be cleared; no device status word is kept here.
  const cudaError_t err = moe::launch_permute(topk_ids, T, E, k, counts, offsets, sorted_token_ids, inv_perm,
                                              scratch, nullptr, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
