// Decode and speculative-verify steps for small batches (B sequences of q new
// tokens each, token t = b*q + i).
//
// Decode is latency-bound: new n-grams depend on the token just produced
// (DGX Spark report, "推理流程": each decode step depends on the token just
// generated), while the rows and the lookup need no hidden state (same report,
// section "n-gram embedding 是一条附加的条件记忆路径"). An 8-token step reads
// 41 KB of rows and 13.1 MB of W_proj and does 105 MFLOP, so its time is the
// W_proj stream and a chain of round trips. The step is two kernels:
//
//   decode_embed_kernel (tokens and token history only): one block per token
//     hashes the token's contexts, gathers and dequantises its rows into
//     e[t] (fp16, the same rounding as the prefill path) and writes the
//     token's metadata; given the hidden states it also computes the gate.
//     It runs with nothing in front of it but the step's inputs.
//
//   decode_proj_kernel (T <= 16): one CTA per SM owns a contiguous range of
//     8-channel groups with the whole K. Its share of W_proj (at most 24 rows
//     of fp16, 123 KB at D = 2560) is requested by bulk copies before it waits
//     for the embed kernel (programmatic dependent launch), so the W_proj
//     stream runs under the embed kernel. After the wait it copies e, takes
//     the gates, runs the products on mma.sync m16n8k16 (tokens x channels,
//     fp16 inputs, fp32 accumulation; eight warps split K and add their sums
//     in warp order in shared memory), then the conv against the carried
//     state, the residual and the state commit for its own channels. No
//     partial sum leaves the CTA and no CTA waits for another, and every sum
//     is taken in a fixed order, so the result is the same bits on every run.
//
// A CTA reads hidden only at its own channels (residual) unless it has to
// compute the gates itself, so with precomputed gates out may alias hidden.
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <algorithm>

#include "ple_device.cuh"
#include "ple_internal.h"

namespace ple {
namespace {

constexpr uint64_t kQ0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kQ1 = 0xC2B2AE3D27D4EB4Full;
constexpr uint64_t kQ2 = 0x165667B19E3779F9ull;
constexpr uint64_t kHeadMix = 0xFF51AFD7ED558CCDull;   // separates the 8 hash heads of an order
constexpr int kHeads = 16;                             // multi-head layout: 2 orders x 8 heads

__device__ __forceinline__ uint64_t ctx_of(int32_t tok) {
  return static_cast<uint64_t>(static_cast<uint32_t>(tok)) + 1ull;
}

// x mod m for m < 2^31 by Barrett reduction with magic = floor((2^64 - 1) / m):
// the quotient estimate umulhi(x, magic) is at most 2 below floor(x / m).
__device__ __forceinline__ uint64_t mod_barrett(uint64_t x, uint64_t m, uint64_t magic) {
  uint64_t r = x - __umul64hi(x, magic) * m;
  if (r >= m) r -= m;
  if (r >= m) r -= m;
  return r;
}

// ------------------------------------------------------------------ embed: rows, metadata, gate
// FMT: 0 = E4M3 rows (two orders), 1 = NVFP4 rows, 2 = the multi-head E4M3 layout.
// Thread j of the block takes 16-code chunks j, j + blockDim, ... of the
// token's row (of all 16 head rows side by side for FMT 2); warp 0 also
// computes the gate.
template <int FMT>
__global__ void __launch_bounds__(512) decode_embed_kernel(const DecodeEmbedArgs a) {
  constexpr bool NV = FMT == 1;
  pdl_launch_dependents();             // the projection's prologue (its W_proj copies) may start now
  pdl_wait();                          // tokens, history and hidden may come from the previous kernel
  const int t = blockIdx.x;
  const int b = t / a.q, i = t - b * a.q;
  const int lane = threadIdx.x & 31;
  const bool gate_warp0 = a.hidden != nullptr && threadIdx.x < 32;
  const int H8 = a.H / 8;
  const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
  uint4 hv[kEmbedH4];
  if (gate_warp0) {                    // the gate's loads go out first: they need no row ID
#pragma unroll
    for (int r = 0; r < kEmbedH4; ++r) {
      const int j = lane + 32 * r;
      if (j < H8) hv[r] = ld_stream_v4(hrow + j);
    }
  }
  const int32_t tok = a.tokens[t];
  if (threadIdx.x == 0 && (tok < 0 || tok >= a.vocab)) set_status(a.status, PLE_ERR_RANGE);
  const int32_t h0 = a.hist[2 * b], h1 = a.hist[2 * b + 1];
  auto carried = [](int32_t h) -> uint64_t { return h < 0 ? 0ull : ctx_of(h); };
  const uint64_t x0 = ctx_of(tok);
  const uint64_t x1 = i >= 1 ? ctx_of(a.tokens[t - 1]) : carried(h1);
  const uint64_t x2 = i >= 2 ? ctx_of(a.tokens[t - 2]) : (i == 1 ? carried(h1) : carried(h0));
  const uint64_t k2 = (x0 * kQ0) ^ (x1 * kQ1);
  const uint64_t k3 = k2 ^ (x2 * kQ2);
  const int nch = a.D / 16;
  uint4* erow = reinterpret_cast<uint4*>(a.e + static_cast<int64_t>(t) * a.D);
  if constexpr (FMT == 2) {
    // chunk j of the token comes from head row j / (chunks per head): head hh of
    // order hh / 8 reads sub-table hh at fold(k_n ^ (hh % 8) * kHeadMix) mod rows
    const int hd = a.D / kHeads, cph = hd / 16;
    for (int j = threadIdx.x; j < nch; j += blockDim.x) {
      const int hh = j / cph;
      const uint64_t k = ((hh >> 3) ? k3 : k2) ^ (static_cast<uint64_t>(hh & 7) * kHeadMix);
      const int64_t row = static_cast<int64_t>(hh) * a.rows0 +
                          static_cast<int64_t>(mod_barrett(k ^ (k >> 32), a.rows0, a.magic0));
      const uint4 v = ld_stream_v4(a.table + row * hd + (j - hh * cph) * 16);
      uint4 o0, o1;
      deq16_one(v, __ldg(a.scales + row), o0, o1);
      erow[2 * j] = o0;
      erow[2 * j + 1] = o1;
    }
  } else {
    const int64_t r0 = static_cast<int64_t>(mod_barrett(k2 ^ (k2 >> 32), a.rows0, a.magic0));
    const int64_t r1 = a.rows0 + static_cast<int64_t>(mod_barrett(k3 ^ (k3 >> 32), a.rows1, a.magic1));
    const float s0 = __ldg(a.scales + r0), s1 = __ldg(a.scales + r1);
    for (int j = threadIdx.x; j < nch; j += blockDim.x) {
      const RowChunk<NV> x = load_chunk<NV>(a.table, a.blocks, r0, a.D, j);
      const RowChunk<NV> y = load_chunk<NV>(a.table, a.blocks, r1, a.D, j);
      uint4 o0, o1;
      deq_chunk<NV>(x, y, s0, s1, o0, o1);
      erow[2 * j] = o0;
      erow[2 * j + 1] = o1;
    }
  }
  if (threadIdx.x < 32) {
    const float g = gate_warp0 ? gate_warp(hv, hrow, reinterpret_cast<const uint4*>(a.w_gate), H8, lane) : 0.f;
    if (lane == 0) {
      TokMeta m;
      m.g = g;
      m.seq = b;
      m.pos = i;
      m.flags = i == a.q - 1 ? kFlagLast : 0;
      a.meta[t] = m;
    }
  }
}

// ------------------------------------------------------------------ projection and the rest (T <= 16)
constexpr int kPjWarps = 8;
constexpr int kPjThreads = kPjWarps * 32;
constexpr int kPjMaxTok = 16;          // the mma's M: tokens
constexpr int kPjGroup = 8;            // the mma's N: channels per group
constexpr int kPjMaxGroups = 3;        // groups per CTA (24 channels)
constexpr int kPjMaxChan = kPjGroup * kPjMaxGroups;
constexpr int kSmemLimit = 227 * 1024;

struct __align__(16) ProjSmem {
  float red[kPjWarps][kPjMaxGroups][kPjMaxTok][kPjGroup];   // per-warp sums over the warp's K range
  float res[kPjMaxTok][kPjMaxChan];                         // hidden at this CTA's channels
  float cst[kPjMaxTok][3][kPjMaxChan];                      // carried conv state at this CTA's channels
  float g[kPjMaxTok];                                       // gates
  uint64_t bar_w[kPjWarps];                                 // W_proj pieces of warp w's K range
  uint64_t bar_e[kPjWarps];                                 // e pieces of warp w's K range
};

// K-steps (16 values of K) of warp w: [ks_begin(w), ks_begin(w + 1)).
__host__ __device__ __forceinline__ int ks_begin(int w, int KS) { return w * KS / kPjWarps; }

// Dynamic shared memory, from a 128-byte aligned base: W_proj rows
// [max_groups * 8][D + 8] fp16, e rows [T][D + 8] fp16 (rows padded by 16
// bytes: conflict-free ldmatrix), then ProjSmem.
size_t proj_smem_bytes(int max_groups, int32_t D, int T) {
  return 128 + static_cast<size_t>(max_groups * kPjGroup + T) * (D + 8) * sizeof(__half) + sizeof(ProjSmem);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kPjThreads, 1) decode_proj_kernel(const DecodeProjArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_s + 127u) & ~127u) - raw_s);
  const int T = a.B * a.q;
  const int ldr = a.D + 8;                                   // fp16 per shared-memory row
  __half* ws = reinterpret_cast<__half*>(base);              // [max_groups * 8][ldr]
  __half* es = ws + static_cast<int64_t>(a.max_groups) * kPjGroup * ldr;   // [T][ldr]
  ProjSmem* sm = reinterpret_cast<ProjSmem*>(es + static_cast<int64_t>(T) * ldr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G8 = a.H / kPjGroup;
  const int g0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * G8 / gridDim.x);
  const int g1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * G8 / gridDim.x);
  const int ng = g1 - g0, c0 = g0 * kPjGroup, nch = ng * kPjGroup;
  const int KS = a.D / 16;
  const int kb = ks_begin(warp, KS), ke = ks_begin(warp + 1, KS);
  const uint32_t piece = static_cast<uint32_t>(ke - kb) * 32u;   // bytes of one row in this warp's K range

  if (tid == 0) {
    for (int w = 0; w < kPjWarps; ++w) {
      mbar_init(smem_u32(&sm->bar_w[w]), 1);
      mbar_init(smem_u32(&sm->bar_e[w]), 1);
    }
    fence_barrier_init();
  }
  __syncthreads();

  // ---- 1. before the wait: this warp's K range of the CTA's W_proj rows (constant
  //         since ple_create), and the conv taps of this thread's items
  if (piece > 0) {
    const uint32_t bw = smem_u32(&sm->bar_w[warp]);
    if (lane == 0) mbar_arrive_expect_tx(bw, piece * nch);
    __syncwarp();
    for (int r = lane; r < nch; r += 32)
      bulk_load(smem_u32(ws + r * ldr + kb * 16), a.w16 + static_cast<int64_t>(c0 + r) * a.D + kb * 16, piece, bw);
  }
  const int n_items = a.B * nch;                             // (sequence b, channel c) pairs
  float4 cw[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int it = tid + k * kPjThreads;
    if (it < n_items) cw[k] = __ldg(reinterpret_cast<const float4*>(a.conv_w) + c0 + it % nch);
  }
  pdl_launch_dependents();
  pdl_wait();                                                // e, meta, hidden and the state are ready

  // ---- 2. e pieces; gates; residual and state at this CTA's channels
  if (piece > 0) {
    const uint32_t be = smem_u32(&sm->bar_e[warp]);
    if (lane == 0) mbar_arrive_expect_tx(be, piece * T);
    __syncwarp();
    for (int r = lane; r < T; r += 32)
      bulk_load(smem_u32(es + r * ldr + kb * 16), a.e + static_cast<int64_t>(r) * a.D + kb * 16, piece, be);
  }
  for (int it = tid; it < T * nch; it += kPjThreads) {
    const int t = it / nch, c = it - (it / nch) * nch;
    sm->res[t][c] = __bfloat162float(a.hidden[static_cast<int64_t>(t) * a.H + c0 + c]);
  }
  for (int it = tid; it < a.B * 3 * nch; it += kPjThreads) {
    const int bk = it / nch, c = it - bk * nch;
    sm->cst[bk / 3][bk % 3][c] = a.conv_state[static_cast<int64_t>(bk) * a.H + c0 + c];
  }
  if (a.gate_ready) {
    if (tid < T) sm->g[tid] = a.meta[tid].g;
  } else {
    const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
    for (int t = warp; t < T; t += kPjWarps) {
      const float g = gate_warp_row(reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H), wg,
                                    a.H / 8, lane);
      if (lane == 0) sm->g[t] = g;
    }
  }

  // ---- 3. products over this warp's K range: tokens (A, rows of e) x channels
  //         (B, rows of W_proj), one accumulator per 8-channel group
  float acc[kPjMaxGroups][4];
#pragma unroll
  for (int g = 0; g < kPjMaxGroups; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
  bool ok = true;
  if (piece > 0) {
    ok = mbar_wait(smem_u32(&sm->bar_w[warp]), 0) && mbar_wait(smem_u32(&sm->bar_e[warp]), 0);
    if (!ok && lane == 0) set_status(a.status, PLE_ERR_TIMEOUT);
  }
  if (ok) {
    // ldmatrix.x4 for A: matrix m = lane / 8 covers token rows (m & 1) * 8 + 0..7 and
    // K offset (m >> 1) * 8; rows past T repeat the last token (their sums are unused)
    const int am = lane >> 3;
    const int arow = min((lane & 7) + ((am & 1) << 3), T - 1);
    const uint32_t a_addr = smem_u32(es + arow * ldr + kb * 16 + ((am >> 1) << 3));
    // ldmatrix.x2 for B: lanes 0..15 address channel rows 0..7 at K offsets 0 and 8
    const uint32_t b_addr = smem_u32(ws + (lane & 7) * ldr + kb * 16 + (((lane >> 3) & 1) << 3));
    const uint32_t group_bytes = kPjGroup * ldr * 2;
    for (int ks = 0; ks < ke - kb; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a_addr + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int g = 0; g < kPjMaxGroups; ++g) {
        if (g < ng) {
          uint32_t b0, b1;
          ldmatrix_x2(b_addr + g * group_bytes + ks * 32, b0, b1);
          mma_16816(acc[g], a0, a1, a2, a3, b0, b1);
        }
      }
    }
  }
  // C layout: (token gq, channels 2tq, 2tq+1) and (token gq + 8, the same channels)
  {
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int g = 0; g < kPjMaxGroups; ++g) {
      float (&rw)[kPjMaxTok][kPjGroup] = sm->red[warp][g];
      rw[gq][2 * tq] = acc[g][0];
      rw[gq][2 * tq + 1] = acc[g][1];
      rw[gq + 8][2 * tq] = acc[g][2];
      rw[gq + 8][2 * tq + 1] = acc[g][3];
    }
  }
  __syncthreads();

  // ---- 4. per (sequence b, channel c): sum over the warps in order, gate, conv
  //         against the carried state, residual, state after n_commit[b] tokens
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int it = tid + k * kPjThreads;
    if (it >= n_items) break;
    const int b = it / nch, c = it - (it / nch) * nch;
    const int g = c >> 3, cc = c & 7;
    const int ch = c0 + c;
    int32_t ncb = a.n_commit ? a.n_commit[b] : a.q;
    if (ncb < 1 || ncb > a.q) {
      if (c == 0 && blockIdx.x == 0) set_status(a.status, PLE_ERR_RANGE);
      ncb = max(1, min(ncb, a.q));
    }
    float w0 = sm->cst[b][0][c], w1 = sm->cst[b][1][c], w2 = sm->cst[b][2][c];
    float k0 = w0, k1 = w1, k2 = w2;
    const float4 cwt = cw[k];
    for (int i = 0; i < a.q; ++i) {
      const int t = b * a.q + i;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kPjWarps; ++w) v += sm->red[w][g][t][cc];
      const float u = sm->g[t] * v;
      const float y = cwt.x * w0 + cwt.y * w1 + cwt.z * w2 + cwt.w * u;
      w0 = w1;
      w1 = w2;
      w2 = u;
      const int64_t idx = static_cast<int64_t>(t) * a.H + ch;
      const float o = sm->res[t][c] + y;
      if (a.out_f32) reinterpret_cast<float*>(a.out)[idx] = o;
      else reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(o);
      if (i == ncb - 1) {
        k0 = w0;
        k1 = w1;
        k2 = w2;
      }
    }
    float* cs = a.conv_state + static_cast<int64_t>(b) * 3 * a.H + ch;
    cs[0] = k0;
    cs[a.H] = k1;
    cs[2 * a.H] = k2;
  }
  // ---- 5. the new token history: the last two committed tokens (the embed
  //         kernel, the only reader of the old one, has completed)
  if (blockIdx.x == 0 && tid < a.B) {
    const int b = tid;
    const int32_t ncb = max(1, min(a.n_commit ? a.n_commit[b] : a.q, a.q));
    const int32_t* tkp = a.tokens + static_cast<int64_t>(b) * a.q;
    const int32_t n1 = tkp[ncb - 1];
    const int32_t n0 = ncb >= 2 ? tkp[ncb - 2] : a.hist[2 * b + 1];
    a.hist[2 * b] = n0;
    a.hist[2 * b + 1] = n1;
  }
}

template <typename Kernel, typename Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, const Args& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace

uint64_t barrett_magic(int64_t m) { return ~0ull / static_cast<uint64_t>(m); }

cudaError_t launch_decode_embed(const DecodeEmbedArgs& a, cudaStream_t stream) {
  const int T = a.B * a.q;
  const int nch = a.D / 16;
  const int threads = std::min(512, std::max(32, (nch + 31) / 32 * 32));
  const dim3 grid(T), block(threads);
  if (a.format == PLE_TABLE_E4M3_HEADS) return launch_pdl(decode_embed_kernel<2>, grid, block, 0, a, stream);
  if (a.format == PLE_TABLE_NVFP4) return launch_pdl(decode_embed_kernel<1>, grid, block, 0, a, stream);
  return launch_pdl(decode_embed_kernel<0>, grid, block, 0, a, stream);
}

bool decode_proj_plan(int32_t H, int32_t D, int32_t num_sms, DecodeProjPlan* plan) {
  if (H % kPjGroup != 0 || D % 16 != 0 || num_sms < 1) return false;
  const int32_t G8 = H / kPjGroup;
  const int32_t grid = std::min(num_sms, G8);
  const int32_t max_groups = (G8 + grid - 1) / grid;
  if (max_groups > kPjMaxGroups) return false;
  if (proj_smem_bytes(max_groups, D, kPjMaxTok) > static_cast<size_t>(kSmemLimit)) return false;
  plan->grid = grid;
  plan->max_groups = max_groups;
  return true;
}

bool decode_proj_supported(int32_t B, int32_t q) { return static_cast<int64_t>(B) * q <= kPjMaxTok; }

cudaError_t launch_decode_proj(const DecodeProjArgs& a, const DecodeProjPlan& plan, cudaStream_t stream) {
  static PerDeviceOnce configured;
  const cudaError_t e = configured.run([] {
    return cudaFuncSetAttribute(decode_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
  });
  if (e != cudaSuccess) return e;
  DecodeProjArgs b = a;
  b.max_groups = plan.max_groups;
  return launch_pdl(decode_proj_kernel, dim3(plan.grid), dim3(kPjThreads),
                    proj_smem_bytes(plan.max_groups, a.D, a.B * a.q), b, stream);
}

}  // namespace ple
