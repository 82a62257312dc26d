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
std::mutex g_setup_mutex;
int32_t* g_ids_ptr[kMaxDevices] = {};
int32_t* g_status_ptr[kMaxDevices] = {};

// Device addresses of the arrays on the current device. In host code the
// arrays' names are host-side stand-ins, not device addresses; the addresses
// come from cudaGetSymbolAddress, looked up once per device.
ple_status static_scratch(int32_t** ids, int32_t** status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PLE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_ids_ptr[dev] == nullptr) {
    void* a = nullptr;
    void* b = nullptr;
    if (cudaGetSymbolAddress(&a, g_static_ids) != cudaSuccess ||
        cudaGetSymbolAddress(&b, g_static_status) != cudaSuccess || a == nullptr || b == nullptr) {
      cudaGetLastError();
      return PLE_ERR_CUDA;
    }
    g_ids_ptr[dev] = static_cast<int32_t*>(a);
    g_status_ptr[dev] = static_cast<int32_t*>(b);
  }
  *ids = g_ids_ptr[dev];
  *status = g_status_ptr[dev];
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
  if (row_dim % 16 != 0) return PLE_ERR_UNSUPPORTED;
  if (T == 0) return PLE_OK;
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
  if (ple::launch_gather(ids, T, ple::TableRef{table, nullptr, scales, 0}, rows0, rows1, row_dim,
                        static_cast<__half*>(e_out), false, stream) != cudaSuccess)
    return PLE_ERR_CUDA;
  if (status_out != nullptr &&
      cudaMemcpyAsync(status_out, status, sizeof(int32_t), cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return PLE_ERR_CUDA;
  return PLE_OK;
}
