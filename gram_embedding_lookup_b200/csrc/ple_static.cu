// ple_embed_static: the lookup half of the layer (n-gram row IDs, then row
// gather and dequantisation) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run the layer:
// serving engines that reserve the whole device budget for their own caching
// allocator at start-up (so a later cudaMalloc fails or fragments the pool),
// and allocation-free runtimes that forbid device allocation after
// initialisation. They also cannot create a handle, because ple_create
// allocates. This entry point takes every input and the output from the
// caller and keeps its only intermediate (the row IDs) in a fixed array that
// lives in the library image.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "ple.h"
#include "ple_internal.h"

namespace {

// Row IDs of one call, [PLE_STATIC_MAX_TOKENS][2], and the device status word.
// Every GPU that loads the library holds these until the process exits.
static __device__ __align__(256) int32_t g_static_ids[2 * PLE_STATIC_MAX_TOKENS];
static __device__ __align__(256) int32_t g_static_status[64];

constexpr int kMaxDevices = 64;
constexpr int32_t kMaxRowDim = 65536;   // the widest row the gather's index arithmetic is sized for

// The arrays' device addresses, looked up once per device and context. In host
// code the arrays' names are host-side stand-ins, not device addresses; the
// addresses come from cudaGetSymbolAddress with the device current. After
// cudaDeviceReset the library's image is loaded into a new context at other
// addresses, so the cache is keyed by the context's unique ID and the lookup
// runs again when that ID changes.
struct DeviceScratch {
  unsigned long long ctx_id = 0;
  int32_t* ids = nullptr;
  int32_t* status = nullptr;
};
std::mutex g_setup_mutex;
DeviceScratch g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique ID of the current context (0 if the driver cannot say). The runtime
// call before it makes sure the device's primary context exists.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa{}, qb{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    cudaGetLastError();
  });
  if (get_current == nullptr || get_id == nullptr || cudaFree(nullptr) != cudaSuccess) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

ple_status static_scratch(int32_t** ids, int32_t** status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLE_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceScratch& d = g_scratch[dev];
  if (d.ids == nullptr || ctx == 0 || ctx != d.ctx_id) {
    void* a = nullptr;
    void* b = nullptr;
    if (cudaGetSymbolAddress(&a, g_static_ids) != cudaSuccess ||
        cudaGetSymbolAddress(&b, g_static_status) != cudaSuccess || a == nullptr || b == nullptr) {
      cudaGetLastError();
      d = DeviceScratch{};
      return PLE_ERR_CUDA;
    }
    d.ctx_id = ctx;
    d.ids = static_cast<int32_t*>(a);
    d.status = static_cast<int32_t*>(b);
  }
  *ids = d.ids;
  *status = d.status;
  return PLE_OK;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

extern "C" ple_status ple_embed_static(const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                                       const int32_t* hist, const uint8_t* table, const float* scales,
                                       int64_t rows0, int64_t rows1, int32_t row_dim, int32_t vocab, void* e_out,
                                       int32_t* status_out, cudaStream_t stream) {
  if (T < 0 || S < 1 || vocab <= 0 || row_dim <= 0 || rows0 <= 0 || rows1 <= 0 || rows0 >= (int64_t(1) << 31) ||
      rows1 >= (int64_t(1) << 31))
    return PLE_ERR_INVALID_ARG;
  if (T > PLE_STATIC_MAX_TOKENS) return PLE_ERR_SHAPE;
  if (row_dim % 16 != 0 || row_dim > kMaxRowDim) return PLE_ERR_UNSUPPORTED;
  if (status_out != nullptr && !aligned(status_out, 4)) return PLE_ERR_ALIGN;
  if (T == 0) {
    // nothing to look up; the caller's status word still reports this call
    if (status_out != nullptr && cudaMemsetAsync(status_out, 0, sizeof(int32_t), stream) != cudaSuccess)
      return PLE_ERR_CUDA;
    return PLE_OK;
  }
  if (tokens == nullptr || offsets == nullptr || table == nullptr || scales == nullptr || e_out == nullptr)
    return PLE_ERR_INVALID_ARG;
  if (!aligned(tokens, 4) || !aligned(offsets, 4) || (hist && !aligned(hist, 4)) || !aligned(table, 16) ||
      !aligned(scales, 4) || !aligned(e_out, 16) || (status_out && !aligned(status_out, 4)))
    return PLE_ERR_ALIGN;

  int32_t* ids = nullptr;
  int32_t* status = nullptr;
  ple_status st = static_scratch(&ids, &status);
  if (st != PLE_OK) return st;
  // the status word keeps the previous call's value: clear it first
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return PLE_ERR_CUDA;

  ple::PrepareArgs pa{};
  pa.tokens = tokens;
  pa.T = T;
  pa.offsets = offsets;
  pa.S = S;
  pa.hist = hist;
  pa.vocab = vocab;
  pa.rows0 = rows0;
  pa.rows1 = rows1;
  pa.ids = ids;
  pa.H = 0;
  pa.status = status;
  if (ple::launch_prepare(pa, stream) != cudaSuccess) return PLE_ERR_CUDA;
  if (ple::launch_gather(ids, T, ple::TableRef{table, nullptr, scales, 0, row_dim, 0, 0}, rows0, rows1, row_dim,
                        static_cast<__half*>(e_out), false, stream) != cudaSuccess)
    return PLE_ERR_CUDA;
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return PLE_ERR_CUDA;
  return PLE_OK;
}
