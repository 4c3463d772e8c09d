// moe_permute_static_scratch: the dispatch counting sort of moe_permute,
// with its scratch memory held in a fixed device array compiled into this
// library instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point
// where they route tokens. Three examples:
//   - a process whose device memory is entirely owned by a pool, where
//     cudaMalloc would fail or fragment it;
//   - a latency-critical loop that cannot afford the implicit device
//     synchronisation of cudaMalloc/cudaFree;
//   - a plug-in host that gives its extensions no allocator.
// Such a caller still owns its inputs and outputs; only the scratch comes
// from here.
//
// Cost and limits:
//   * The array below is 4 MiB.  Every GPU that loads this library reserves
//     it from module load until the process exits, whether or not the
//     entry point is ever called.
//   * It holds the per-chunk expert counts and their prefix sums:
//     2 x M x ceil(T*k / 512) int32.  Requests with
//     M * ceil(T*k / 512) > kStaticPermScratchInts are rejected with
//     MOE_ERR_UNSUPPORTED before anything is launched.
//   * All calls on a device share the one array.  The kernels overwrite
//     every scratch entry they read (nothing has to start at zero), so a
//     call never sees stale data from the previous call.  But two calls
//     whose kernels overlap on the GPU (different streams without ordering
//     between them) race on the array and may produce wrong results.
//   * The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current, and records it with
//     the device's current context.  A later call in a different context
//     (after cudaDeviceReset, for instance) looks it up again.  Make the
//     first call on a device before any stream capture begins.
#include <atomic>
#include <mutex>

#include "kernels.cuh"

namespace {

constexpr size_t kStaticPermScratchInts = size_t(1) << 19;  // per array: 2 MiB

// [0, kStaticPermScratchInts): per-chunk counts; [kStaticPermScratchInts, 2x): their bases.
static __device__ __align__(256) int32_t g_perm_scratch[2 * kStaticPermScratchInts];

constexpr int kMaxDevices = 64;
std::mutex g_addr_mutex;
int32_t* g_addr[kMaxDevices] = {nullptr};
CUcontext g_ctx[kMaxDevices] = {nullptr};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point table (the
// library links no driver library directly).
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

CUcontext current_context() {
  CUcontext c = nullptr;
  const CtxGetCurrentFn fn = ctx_get_current();
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_perm_scratch on the current device.  The host-side
// symbol `g_perm_scratch` is only a stand-in, not a device address, so the
// kernels get this pointer instead.  It is looked up once per device and
// context: a context created anew (the module loaded again) may place the
// array elsewhere.
moe_status_t scratch_address(int32_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_addr_mutex);
  CUcontext ctx = current_context();
  if (g_addr[dev] == nullptr || ctx == nullptr || ctx != g_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_perm_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_addr[dev] = static_cast<int32_t*>(p);
    g_ctx[dev] = current_context();  // the lookup makes the device's context current
  }
  *out = g_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_static_scratch(const int32_t* topk_idx, const float* topk_w, int T,
                                                   int k, int M, int32_t* counts, int32_t* offsets,
                                                   int32_t* slot_of, int32_t* row_token, float* row_w,
                                                   int32_t* device_status, void* stream) {
  using namespace moe;
  if (T < 0 || k < 1 || M < 1 || k > M) return MOE_ERR_INVALID_ARG;
  if (M > kMaxExperts || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(M) * perm_num_chunks(pairs) > static_cast<long long>(kStaticPermScratchInts))
    return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_w || !slot_of || !row_token || !row_w)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  int32_t* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (device_status != nullptr && cudaMemsetAsync(device_status, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (T == 0) {
    if (cudaMemsetAsync(counts, 0, static_cast<size_t>(M) * 4, s) != cudaSuccess ||
        cudaMemsetAsync(offsets, 0, static_cast<size_t>(M + 1) * 4, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const cudaError_t e = launch_permute(topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token,
                                       row_w, scratch, scratch + kStaticPermScratchInts, device_status, s);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
