// Device-side filler for the synthetic PLE table (input generation only).
//
// Fills table u8[2][R][D] (FP8-E4M3 codes, uniform over the 254 finite codes)
// and scales f32[2][R] (uniform in [0.01, 0.1)), or the NVFP4 variant's packed
// codes and block scales, from the counter-based
// splitmix64 generator (Steele, Lea and Flood, OOPSLA 2014). Element i of
// stream `tag` is mix(base(seed, tag) + (i + 1) * GAMMA) with
// base(seed, tag) = mix(seed ^ (tag << 32)). The host generator in
// ple_inputs/__init__.py implements the same definition; tests compare the two
// bit for bit on sampled rows. Nothing here computes any part of the layer.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;
constexpr uint32_t kTagCodes = 1;
constexpr uint32_t kTagScales = 2;
constexpr uint32_t kTagNvCodes = 3;    // NVFP4 table: packed E2M1 code bytes
constexpr uint32_t kTagNvBlocks = 4;   // NVFP4 table: E4M3 block-scale bytes
constexpr uint32_t kNvBlockBase = 0x30;

__host__ __device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ __forceinline__ uint64_t stream_base(uint64_t seed, uint32_t tag) {
  return sm64_mix(seed ^ (static_cast<uint64_t>(tag) << 32));
}

// Uniform map onto the 254 finite E4M3 codes: i in [0,254), skip 0x7F.
__device__ __forceinline__ uint32_t draw_code(uint64_t u) {
  const uint32_t i = static_cast<uint32_t>(((u >> 32) * 254ull) >> 32);
  return i + (i >= 127u ? 1u : 0u);
}

__global__ void fill_codes_kernel(uint8_t* __restrict__ table, uint64_t n16, uint64_t base) {
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t c = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < n16; c += stride) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t v = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const uint64_t i = c * 16 + q * 4 + b;
        v |= draw_code(sm64_mix(base + (i + 1) * kGamma)) << (8 * b);
      }
      w[q] = v;
    }
    reinterpret_cast<uint4*>(table)[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

__global__ void fill_scales_kernel(float* __restrict__ scales, uint64_t n, uint64_t base) {
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t u = sm64_mix(base + (i + 1) * kGamma);
    const double f = static_cast<double>(u >> 40) * 0x1p-24;          // exact
    scales[i] = __double2float_rn(__dadd_rn(0.01, __dmul_rn(0.09, f)));  // no contraction
  }
}

// Byte i of a flat array: the draw's top byte (mode 0, packed E2M1 codes) or
// kNvBlockBase + its top 4 bits (mode 1, E4M3 block scales 0.5 .. 1.875).
__global__ void fill_nv_bytes_kernel(uint32_t* __restrict__ dst, uint64_t n4, uint64_t base, int mode) {
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t c = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < n4; c += stride) {
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint64_t i = c * 4 + b;
      const uint64_t u = sm64_mix(base + (i + 1) * kGamma);
      const uint32_t byte = mode == 0 ? static_cast<uint32_t>(u >> 56) : kNvBlockBase + static_cast<uint32_t>(u >> 60);
      v |= byte << (8 * b);
    }
    dst[c] = v;
  }
}

// The same bytes stored row by row: word w of row r (row_words = 9D/64 words)
// is code word w of the row (w < D/8) or block-scale word w - D/8, each drawn
// from the counter index it has in its own flat array.
__global__ void fill_nv_rows_kernel(uint32_t* __restrict__ dst, uint64_t rows, int32_t row_dim, uint64_t code_base,
                                    uint64_t block_base) {
  const uint64_t cw = static_cast<uint64_t>(row_dim / 8), bw = static_cast<uint64_t>(row_dim / 64);
  const uint64_t row_words = cw + bw, n4 = rows * row_words;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t c = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < n4; c += stride) {
    const uint64_t r = c / row_words, k = c - r * row_words;
    const bool code = k < cw;
    const uint64_t first = code ? (r * cw + k) * 4 : (r * bw + (k - cw)) * 4;
    const uint64_t base = code ? code_base : block_base;
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint64_t u = sm64_mix(base + (first + b + 1) * kGamma);
      const uint32_t byte = code ? static_cast<uint32_t>(u >> 56) : kNvBlockBase + static_cast<uint32_t>(u >> 60);
      v |= byte << (8 * b);
    }
    dst[c] = v;
  }
}

}  // namespace

extern "C" uint64_t ple_synth_stream_base(uint64_t seed, uint32_t tag) {
  return stream_base(seed, tag);
}

// Returns 0 on success, else the CUDA error code (or cudaErrorInvalidValue for bad sizes).
extern "C" int ple_synth_fill_table(uint8_t* table, float* scales, int64_t rows_per_order,
                                    int32_t row_dim, uint64_t seed, cudaStream_t stream) {
  if (table == nullptr || scales == nullptr || rows_per_order <= 0 || row_dim <= 0 ||
      (row_dim % 16) != 0 || (reinterpret_cast<uintptr_t>(table) % 16) != 0) {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  const uint64_t nbytes = 2ull * static_cast<uint64_t>(rows_per_order) * static_cast<uint64_t>(row_dim);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  fill_codes_kernel<<<sms * 8, 256, 0, stream>>>(table, nbytes / 16, stream_base(seed, kTagCodes));
  fill_scales_kernel<<<sms * 2, 256, 0, stream>>>(scales, 2ull * static_cast<uint64_t>(rows_per_order),
                                                  stream_base(seed, kTagScales));
  return static_cast<int>(cudaGetLastError());
}

// NVFP4 table: codes u8[2][R][D/2], block scales u8[2][R][D/16], scales f32[2][R]
// (the FP8 table's scale stream). Returns 0 on success, else a CUDA error code.
extern "C" int ple_synth_fill_nvfp4(uint8_t* codes, uint8_t* blocks, float* scales, int64_t rows_per_order,
                                    int32_t row_dim, uint64_t seed, cudaStream_t stream) {
  if (codes == nullptr || blocks == nullptr || scales == nullptr || rows_per_order <= 0 || row_dim <= 0 ||
      (row_dim % 64) != 0 || (reinterpret_cast<uintptr_t>(codes) % 4) != 0 ||
      (reinterpret_cast<uintptr_t>(blocks) % 4) != 0) {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  const uint64_t rows = 2ull * static_cast<uint64_t>(rows_per_order);
  const uint64_t code_bytes = rows * static_cast<uint64_t>(row_dim / 2);
  const uint64_t block_bytes = rows * static_cast<uint64_t>(row_dim / 16);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  fill_nv_bytes_kernel<<<sms * 8, 256, 0, stream>>>(reinterpret_cast<uint32_t*>(codes), code_bytes / 4,
                                                    stream_base(seed, kTagNvCodes), 0);
  fill_nv_bytes_kernel<<<sms * 8, 256, 0, stream>>>(reinterpret_cast<uint32_t*>(blocks), block_bytes / 4,
                                                    stream_base(seed, kTagNvBlocks), 1);
  fill_scales_kernel<<<sms * 2, 256, 0, stream>>>(scales, rows, stream_base(seed, kTagScales));
  return static_cast<int>(cudaGetLastError());
}

// The NVFP4 table stored row by row (rows u8[2][R][9D/16]: each row's D/2 code
// bytes, then its D/16 block-scale bytes), with the same contents as
// ple_synth_fill_nvfp4, and scales f32[2][R]. Returns 0 or a CUDA error code.
extern "C" int ple_synth_fill_nvfp4_rows(uint8_t* rows, float* scales, int64_t rows_per_order, int32_t row_dim,
                                         uint64_t seed, cudaStream_t stream) {
  if (rows == nullptr || scales == nullptr || rows_per_order <= 0 || row_dim <= 0 || (row_dim % 64) != 0 ||
      (reinterpret_cast<uintptr_t>(rows) % 4) != 0) {
    return static_cast<int>(cudaErrorInvalidValue);
  }
  const uint64_t n = 2ull * static_cast<uint64_t>(rows_per_order);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  fill_nv_rows_kernel<<<sms * 8, 256, 0, stream>>>(reinterpret_cast<uint32_t*>(rows), n, row_dim,
                                                   stream_base(seed, kTagNvCodes), stream_base(seed, kTagNvBlocks));
  fill_scales_kernel<<<sms * 2, 256, 0, stream>>>(scales, n, stream_base(seed, kTagScales));
  return static_cast<int>(cudaGetLastError());
}
