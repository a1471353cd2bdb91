// qsa_forward_noalloc: the forward pass for callers that cannot allocate device
// memory.  Some callers have no way to obtain a workspace: for example a plugin
// loaded into a host application that owns the device allocator and gives its
// extensions no allocation hook, or a latency-critical path that must not call
// cudaMalloc because it can synchronise the device and take unbounded time.
// This entry point keeps its scratch (the per-row sorted route lists that the
// forward kernel consumes) in a fixed array compiled into the library, so the
// caller passes only inputs and outputs.
#include <climits>
#include <cmath>
#include <mutex>

#include "qsa.h"
#include "qsa_device.cuh"
#include "qsa_internal.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch array.  Every GPU that loads this library holds it until the
// process exits; every call on a device shares that device's copy.
static __device__ __align__(256) unsigned char g_noalloc_scratch[QSA_NOALLOC_SCRATCH_BYTES];

std::mutex g_mutex;
// Per device: the context the address was taken in (its process-unique ID) and
// the address.  A context is destroyed by cudaDeviceReset, and the runtime makes
// a new one (with the module loaded again, possibly elsewhere) on the next call,
// so an address is reused only while the context it came from is current.
unsigned long long g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_ptr[kMaxDevices] = {};

// Driver calls reached through the runtime (no link against libcuda): the
// current context and its ID, which CUDA never gives to a second context.
using CtxGetCurrentFn = int (*)(void**);
using CtxGetIdFn = int (*)(void*, unsigned long long*);

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult r1 = cudaDriverEntryPointSymbolNotFound, r2 = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &r1) == cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &r2) == cudaSuccess &&
        r1 == cudaDriverEntryPointSuccess && r2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    looked_up = true;
  }
  if (get_current == nullptr || get_id == nullptr) return false;
  void* ctx = nullptr;
  if (get_current(&ctx) != 0 || ctx == nullptr) return false;
  return get_id(ctx, id) == 0 && *id != 0;
}

// Device address of the scratch array in the current context.  In host code the
// array's name only stands in for the symbol, so the address must come from
// cudaGetSymbolAddress with the device current.  It is looked up once per device
// and context: the first call on a device (and the first after a device reset)
// does it, and that call should come before any stream capture.  Should the
// context ID be unavailable, it is looked up on every call (a host-side lookup
// that allocates nothing).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) && g_scratch_ptr[dev] != nullptr && g_scratch_ctx[dev] == ctx) {
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
  }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // makes the device's context current if it was not
  if (e != cudaSuccess) return e;
  g_scratch_ptr[dev] = p;
  g_scratch_ctx[dev] = current_context_id(&ctx) ? ctx : 0;
  *out = p;
  return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Status for sizes outside the supported envelope, in the order qsa_forward checks them.
qsa_status_t size_status(int64_t T, int64_t T_kv, int H, int G, int n_sel) {
  if (T < 1 || T_kv < 1 || n_sel < 1 || n_sel > 16384 || G < 1 || H < 1) return QSA_ERR_INVALID_ARGUMENT;
  if (T_kv > INT32_MAX || T > INT32_MAX / n_sel || T > (int64_t{1} << 30)) return QSA_ERR_INVALID_ARGUMENT;
  if (H % G != 0 || H / G != qsa::kHeadsPerGroup) return QSA_ERR_UNSUPPORTED;
  return QSA_ERR_INVALID_ARGUMENT;
}

}  // namespace

extern "C" qsa_status_t qsa_forward_noalloc(const void* q, const void* k, const void* v, const int32_t* routes,
                                            int64_t T, int64_t T_kv, int H, int G, int n_sel, float scale,
                                            void* out, float* lse, qsa_stream_t stream) {
  if (!q || !k || !v || !routes || !out || !lse) return QSA_ERR_INVALID_ARGUMENT;
  const size_t need = qsa_forward_workspace_size(T, T_kv, H, G, n_sel);
  if (need == 0) return size_status(T, T_kv, H, G, n_sel);
  if (!(scale > 0.f) || !std::isfinite(scale)) return QSA_ERR_INVALID_ARGUMENT;
  const auto aligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(routes, 4) ||
      !aligned(lse, 4))
    return QSA_ERR_MISALIGNED;
  if (need > QSA_NOALLOC_SCRATCH_BYTES) return QSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return QSA_ERR_CUDA;
  // Scratch layout (the same as qsa_forward's workspace): a status word, row
  // counts [T] int32, then the sorted route lists [T, n_sel] int32.  The route
  // kernel overwrites every value the forward kernel reads (and zeroes the status
  // word), so nothing needs clearing between calls.
  unsigned char* base = static_cast<unsigned char*>(scratch);
  int* status = reinterpret_cast<int*>(base);
  int32_t* row_cnt = reinterpret_cast<int32_t*>(base + 256);
  int32_t* row_cols = reinterpret_cast<int32_t*>(base + 256 + align256(static_cast<size_t>(T) * 4));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (qsa::launch_route_rows(routes, T, T_kv, n_sel, row_cnt, row_cols, nullptr, 2, status, nullptr, nullptr, nullptr,
                             H, nullptr, s) != cudaSuccess)
    return QSA_ERR_CUDA;
  if (qsa::launch_forward(q, k, v, row_cnt, row_cols, T, G, n_sel, scale, out, lse, status, s) != cudaSuccess)
    return QSA_ERR_CUDA;
  return QSA_OK;
}
