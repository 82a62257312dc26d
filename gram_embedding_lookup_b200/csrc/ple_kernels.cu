// libple kernels other than the projection: the prepare stage (sequence map,
// n-gram row IDs, sigmoid gate), the row gather with E4M3 dequantisation, the
// one-time W_proj conversion, and the combine kernels used after a split-K
// projection (small batches and decode steps).
//
// The n-gram definition follows the DGX Spark deployment report
// ("【Qwen3.8-Flash-Next 端侧部署】01-模型架构与整体方案", section
// "n-gram embedding 是一条附加的条件记忆路径": IDs from token IDs, positions and
// sequence boundaries only) and the RTX 3090 llama.cpp report (section
// "n-gram表格": the last few tokens are hashed into bigram and trigram rows).
// The concrete hash is the one stated in include/ple.h.
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

constexpr uint64_t kP0 = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kP1 = 0xC2B2AE3D27D4EB4Full;
constexpr uint64_t kP2 = 0x165667B19E3779F9ull;

__device__ __forceinline__ uint64_t context_of(int32_t tok) {
  return static_cast<uint64_t>(static_cast<uint32_t>(tok)) + 1ull;
}

__device__ __forceinline__ uint64_t fold64(uint64_t k) { return k ^ (k >> 32); }

// x mod m for m < 2^31 by Barrett reduction with magic = floor((2^64 - 1) / m):
// the quotient estimate umulhi(x, magic) is at most 2 below floor(x / m).
__device__ __forceinline__ uint64_t mod_barrett(uint64_t x, uint64_t m, uint64_t magic) {
  uint64_t r = x - __umul64hi(x, magic) * m;
  if (r >= m) r -= m;
  if (r >= m) r -= m;
  return r;
}

PrepareArgs with_magic(const PrepareArgs& in) {
  PrepareArgs a = in;
  a.magic0 = ~0ull / static_cast<uint64_t>(a.rows0);
  a.magic1 = ~0ull / static_cast<uint64_t>(a.rows1);
  return a;
}

// Sequence, position and last-token flag of token t. `report` decides which
// caller records a range error.
__device__ __forceinline__ void sequence_of(const PrepareArgs& a, int t, bool report, int32_t& s, int32_t& pos,
                                            int32_t& last) {
  if (a.uniform_q > 0) {
    s = t / a.uniform_q;
    pos = t - s * a.uniform_q;
    last = (pos == a.uniform_q - 1);
    return;
  }
  int lo = 0, hi = a.S - 1;
  while (lo < hi) {                           // largest s with offsets[s] <= t
    const int mid = (lo + hi + 1) >> 1;
    if (a.offsets[mid] <= t) lo = mid; else hi = mid - 1;
  }
  s = lo;
  const int32_t begin = a.offsets[s];
  const int32_t end = a.offsets[s + 1];
  pos = t - begin;
  if (pos < 0 || t >= end) {                  // inconsistent offsets: keep every access in bounds
    if (report) set_status(a.status, PLE_ERR_RANGE);
    pos = max(0, min(pos, t));
  }
  last = (t == end - 1);
}

// The bigram and trigram keys of token t at position pos of sequence s. Before
// the sequence start the carried history, or nothing, stands in.
__device__ __forceinline__ void keys_of(const PrepareArgs& a, int t, int32_t s, int32_t pos, bool report,
                                        uint64_t& k2, uint64_t& k3) {
  const int32_t tok = a.tokens[t];
  if (report && (tok < 0 || tok >= a.vocab)) set_status(a.status, PLE_ERR_RANGE);
  const uint64_t x0 = context_of(tok);
  auto carried = [&](int k) -> uint64_t {     // the token k places before the sequence start
    if (a.hist == nullptr) return 0ull;
    const int32_t h = a.hist[2 * s + (2 - k)];
    return h < 0 ? 0ull : context_of(h);
  };
  const uint64_t x1 = pos >= 1 ? context_of(a.tokens[t - 1]) : carried(1);
  const uint64_t x2 = pos >= 2 ? context_of(a.tokens[t - 2]) : (pos == 1 ? carried(1) : carried(2));
  k2 = (x0 * kP0) ^ (x1 * kP1);
  k3 = k2 ^ (x2 * kP2);
}

// Sequence, position, last-token flag and the bigram and trigram keys of token
// t (every lane of the calling warp computes the same values; lane 0 reports
// errors).
__device__ __forceinline__ void sequence_and_keys(const PrepareArgs& a, int t, int lane, int32_t& s, int32_t& pos,
                                                  int32_t& last, uint64_t& k2, uint64_t& k3) {
  sequence_of(a, t, lane == 0, s, pos, last);
  keys_of(a, t, s, pos, lane == 0, k2, k3);
}

__device__ __forceinline__ void sequence_and_rows(const PrepareArgs& a, int t, int lane, int32_t& s, int32_t& pos,
                                                  int32_t& last, int32_t& r0, int32_t& r1) {
  uint64_t k2, k3;
  sequence_and_keys(a, t, lane, s, pos, last, k2, k3);
  r0 = static_cast<int32_t>(mod_barrett(fold64(k2), static_cast<uint64_t>(a.rows0), a.magic0));
  r1 = static_cast<int32_t>(mod_barrett(fold64(k3), static_cast<uint64_t>(a.rows1), a.magic1));
}

// The state and offsets work of the prepare / embed kernels, by threads
// [0, nthr) of blocks sb of nsb (tid: the calling thread's index among them).
__device__ __forceinline__ void state_blocks(const PrepareArgs& a, int sb, int nsb, int tid, int nthr) {
  if (sb == 0 && a.uniform_q == 0) {
    // offsets must start at 0, end at T and be non-decreasing
    if (tid == 0 && (a.offsets[0] != 0 || a.offsets[a.S] != a.T)) set_status(a.status, PLE_ERR_RANGE);
    for (int s = tid; s < a.S; s += nthr)
      if (a.offsets[s] > a.offsets[s + 1]) set_status(a.status, PLE_ERR_RANGE);
  }
  if (a.conv_in != nullptr) {
    const int64_t n4 = static_cast<int64_t>(a.S) * 3 * a.H / 4;
    const float4* src = reinterpret_cast<const float4*>(a.conv_in);
    float4* dst = reinterpret_cast<float4*>(a.conv_copy);
    for (int64_t i = static_cast<int64_t>(sb) * nthr + tid; i < n4;
         i += static_cast<int64_t>(nsb) * nthr)
      dst[i] = src[i];
  }
  if (a.hist_new != nullptr && sb == 0) {
    for (int s = tid; s < a.S; s += nthr) {
      int32_t begin, end;
      if (a.uniform_q > 0) { begin = s * a.uniform_q; end = begin + a.uniform_q; }
      else { begin = a.offsets[s]; end = a.offsets[s + 1]; }
      end = min(max(end, 0), a.T);
      begin = min(max(begin, 0), end);
      const int32_t len = end - begin;
      const int32_t h0 = a.hist ? a.hist[2 * s] : -1;
      const int32_t h1 = a.hist ? a.hist[2 * s + 1] : -1;
      int32_t n0, n1;
      if (len >= 2) { n0 = a.tokens[end - 2]; n1 = a.tokens[end - 1]; }
      else if (len == 1) { n0 = h1; n1 = a.tokens[end - 1]; }
      else { n0 = h0; n1 = h1; }
      a.hist_new[2 * s] = n0;
      a.hist_new[2 * s + 1] = n1;
    }
  }
}

// ------------------------------------------------------------------ prepare
constexpr int kPrepWarps = 8;   // one warp per token, 8 tokens per block

__global__ void __launch_bounds__(256) prepare_kernel(const PrepareArgs a, int token_blocks) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (static_cast<int>(blockIdx.x) >= token_blocks) {
    state_blocks(a, blockIdx.x - token_blocks, gridDim.x - token_blocks, threadIdx.x, blockDim.x);
    return;
  }

  const int t = blockIdx.x * kPrepWarps + warp;
  if (t >= a.T) return;
  int32_t s, pos, last, r0, r1;
  sequence_and_rows(a, t, lane, s, pos, last, r0, r1);
  if (lane == 0) reinterpret_cast<int2*>(a.ids)[t] = make_int2(r0, r1);
  if (a.meta == nullptr) return;

  // ---- gate: g = sigmoid(w_gate . h_t), fp32 accumulation, warp reduction
  const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
  const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
  float acc = 0.f;
  for (int j = lane; j < a.H / 8; j += 32) {
    const uint4 hv = hrow[j];
    const uint4 wv = __ldg(wg + j);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hv);
    const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 hf = __bfloat1622float2(h2[q]);
      const float2 wf = __bfloat1622float2(w2[q]);
      acc = fmaf(hf.x, wf.x, acc);
      acc = fmaf(hf.y, wf.y, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    TokMeta m;
    m.g = 1.0f / (1.0f + expf(-acc));
    m.seq = s;
    m.pos = pos;
    m.flags = last ? kFlagLast : 0;
    a.meta[t] = m;
  }
}

// ------------------------------------------------------------------ gather
template <bool NV>
__global__ void __launch_bounds__(256) gather_kernel(const int2* __restrict__ ids, int32_t T, const TableRef t,
                                                     int64_t rows0, int64_t rows1, int32_t D,
                                                     __half* __restrict__ e, int reduce_ids) {
  const int chunks = D >> 4;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= static_cast<int64_t>(T) * chunks) return;
  const int32_t tk = static_cast<int32_t>(g / chunks);
  const int32_t c = static_cast<int32_t>(g - static_cast<int64_t>(tk) * chunks);
  int2 id = ids[tk];
  if (reduce_ids) {
    id.x = static_cast<int32_t>(static_cast<uint32_t>(id.x) % static_cast<uint32_t>(rows0));
    id.y = static_cast<int32_t>(static_cast<uint32_t>(id.y) % static_cast<uint32_t>(rows1));
  }
  const int64_t row0 = id.x;
  const int64_t row1 = rows0 + id.y;
  const RowChunk<NV> a = load_chunk<NV>(t.codes, t.blocks, row0, t.cs, t.bs, c);
  const RowChunk<NV> b = load_chunk<NV>(t.codes, t.blocks, row1, t.cs, t.bs, c);
  const float s0 = __ldg(t.scales + row0);
  const float s1 = __ldg(t.scales + row1);
  uint4 o0, o1;
  deq_chunk<NV>(a, b, s0, s1, o0, o1);
  uint4* dst = reinterpret_cast<uint4*>(e + static_cast<int64_t>(tk) * D + c * 16);
  dst[0] = o0;
  dst[1] = o1;
}

// ------------------------------------------------------------------ embed (prepare + gather)
constexpr int kEmbedD16 = 5;    // 16-code chunks per lane and row held in registers (rows <= 2560 codes)

// ------------------------------------------------------------------ gate (after ple_prepare)
// The gate of a batch whose IDs, rows and metadata ple_prepare left in the
// scratch: one warp per token writes meta[t].g. Blocks past token_blocks take
// the snapshot of the carried conv state, as the embed kernel's state work does.
__global__ void __launch_bounds__(256) gate_kernel(const PrepareArgs a, int token_blocks) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (static_cast<int>(blockIdx.x) >= token_blocks) {
    if (a.conv_in != nullptr) {
      const int64_t n4 = static_cast<int64_t>(a.S) * 3 * a.H / 4;
      const float4* src = reinterpret_cast<const float4*>(a.conv_in);
      float4* dst = reinterpret_cast<float4*>(a.conv_copy);
      const int sb = blockIdx.x - token_blocks, nsb = gridDim.x - token_blocks;
      for (int64_t i = static_cast<int64_t>(sb) * blockDim.x + threadIdx.x; i < n4;
           i += static_cast<int64_t>(nsb) * blockDim.x)
        dst[i] = src[i];
    }
    return;
  }
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  const int H8 = a.H / 8;
  const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
  uint4 hv[kEmbedH4];
#pragma unroll
  for (int r = 0; r < kEmbedH4; ++r) {
    const int j = lane + 32 * r;
    if (j < H8) hv[r] = ld_stream_v4(hrow + j);
  }
  const float g = gate_warp(hv, hrow, reinterpret_cast<const uint4*>(a.w_gate), H8, lane);
  if (lane == 0) a.meta[t].g = g;
}

// ------------------------------------------------------------------ multi-head layout
// The row geometry of the SSD-stream model card ("Qwen3.8 Flash-Next NVFP4 -
// SSD Stream", section "技术细节": 16 table lookups per token, 160-byte rows):
// 8 hash heads per order; head j of order n reads sub-table 8n + j at row
// fold(k_n ^ j * kHeadMix) mod rows (head 0 is the two-order row), and e is the
// 16 dequantised rows side by side.
constexpr uint64_t kHeadMix = 0xFF51AFD7ED558CCDull;   // odd constant separating the heads
constexpr int kHeads = 16;

// One warp per token. Lane l < 16 owns head l: its row ID and its row's scale;
// the gather then spreads the token's D / 16 chunks of 16 codes over the lanes,
// each taking its chunk's row and scale from the owning lane. Blocks past
// token_blocks do the offsets check and the state work.
__global__ void __launch_bounds__(256) embed_heads_kernel(const PrepareArgs a, const TableRef tab, int32_t D,
                                                          __half* __restrict__ e, int token_blocks) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (static_cast<int>(blockIdx.x) >= token_blocks) {
    state_blocks(a, blockIdx.x - token_blocks, gridDim.x - token_blocks, threadIdx.x, blockDim.x);
    return;
  }
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  int32_t s, pos, last;
  uint64_t k2, k3;
  sequence_and_keys(a, t, lane, s, pos, last, k2, k3);
  const int hh = lane & (kHeads - 1);
  const uint64_t k = ((hh >> 3) ? k3 : k2) ^ (static_cast<uint64_t>(hh & 7) * kHeadMix);
  const int32_t row = static_cast<int32_t>(mod_barrett(fold64(k), static_cast<uint64_t>(a.rows0), a.magic0));
  if (lane < kHeads) a.ids[static_cast<int64_t>(t) * kHeads + lane] = row;
  if (a.meta != nullptr) {
    float g = 0.f;
    if (a.hidden != nullptr) {
      const int H8 = a.H / 8;
      const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
      uint4 hv[kEmbedH4];
#pragma unroll
      for (int r = 0; r < kEmbedH4; ++r) {
        const int j = lane + 32 * r;
        if (j < H8) hv[r] = ld_stream_v4(hrow + j);
      }
      g = gate_warp(hv, hrow, reinterpret_cast<const uint4*>(a.w_gate), H8, lane);
    }
    if (lane == 0) {
      TokMeta m;
      m.g = g;
      m.seq = s;
      m.pos = pos;
      m.flags = last ? kFlagLast : 0;
      a.meta[t] = m;
    }
  }
  if (e == nullptr) return;
  const int hd = D / kHeads;                 // codes per head row
  const int cph = hd / 16;                   // 16-code chunks per head row
  const int nch = D / 16;
  const int64_t srow = static_cast<int64_t>(hh) * a.rows0 + row;
  const float sc = __ldg(tab.scales + srow);
  for (int base = 0; base < nch; base += 32) {
    const int c = base + lane;
    const int h = min(c, nch - 1) / cph;
    const int r = __shfl_sync(0xffffffffu, row, h);
    const float sh = __shfl_sync(0xffffffffu, sc, h);
    if (c < nch) {
      const int cc = c - h * cph;
      const uint4 v = ld_stream_v4(tab.codes + (static_cast<int64_t>(h) * a.rows0 + r) * hd + cc * 16);
      uint4 o0, o1;
      deq16_one(v, sh, o0, o1);
      uint4* dst = reinterpret_cast<uint4*>(e + static_cast<int64_t>(t) * D + c * 16);
      dst[0] = o0;
      dst[1] = o1;
    }
  }
}

// Gather stage of the multi-head layout: one thread per 16-code chunk.
__global__ void __launch_bounds__(256) gather_heads_kernel(const int32_t* __restrict__ ids, int32_t T,
                                                           const TableRef t, int64_t rows, int32_t D,
                                                           __half* __restrict__ e) {
  const int nch = D / 16;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= static_cast<int64_t>(T) * nch) return;
  const int32_t tk = static_cast<int32_t>(g / nch);
  const int c = static_cast<int>(g - static_cast<int64_t>(tk) * nch);
  const int hd = D / kHeads;
  const int cph = hd / 16;
  const int h = c / cph;
  const int cc = c - h * cph;
  const uint32_t r = static_cast<uint32_t>(ids[static_cast<int64_t>(tk) * kHeads + h]) % static_cast<uint32_t>(rows);
  const int64_t row = static_cast<int64_t>(h) * rows + r;
  const uint4 v = ld_stream_v4(t.codes + row * hd + cc * 16);
  uint4 o0, o1;
  deq16_one(v, __ldg(t.scales + row), o0, o1);
  uint4* dst = reinterpret_cast<uint4*>(e + static_cast<int64_t>(tk) * D + c * 16);
  dst[0] = o0;
  dst[1] = o1;
}

// ------------------------------------------------------------------ embed, pipelined
// n-gram row IDs, the gate dot product over h_t, and the row gather with E4M3
// dequantisation into fp16 e_t, in one pass over HBM. One persistent CTA per
// SM takes a contiguous range of tokens. Its
// producer warp computes the row IDs of 30 tokens at a time (a lane per token)
// into a ring of kPipeBatches batches in shared memory. Each of the 15
// consumer warps takes two tokens of every batch and issues all of a token's
// loads at once: its hidden row and its two table rows (plain 16-byte loads,
// which keep more bytes in flight per SM than bulk copies of single rows do).
// Then come the gate dot product (fp32, lane-strided, then a warp reduction),
// the dequantisation into fp16 e_t and the metadata (with e null the rows are
// skipped: the gather-fused projection reads them itself). Batches go through the
// ring in order, so every parity wait is for the phase after the one last
// released.
constexpr int kPipeConsumers = 15;                   // 16 warps in all: 128 registers per thread
constexpr int kPipeThreads = 32 * (1 + kPipeConsumers);
constexpr int kPipeBatch = 2 * kPipeConsumers;       // tokens per batch: 2 per consumer warp
static_assert(kPipeBatch <= 32, "a producer lane per token of a batch");
constexpr int kPipeBatches = 4;                      // batches in the ring

struct PipeTok {                                     // per token, written by the producer
  int32_t r0, r1, seq, pos, flags, pad0, pad1, pad2;
};

struct PipeSmem {
  PipeTok tok[kPipeBatches][kPipeBatch];
  uint64_t full[kPipeBatches];                       // producer -> consumers (count 1)
  uint64_t empty[kPipeBatches];                      // consumers -> producer (count kPipeConsumers)
};

template <bool NV>
__global__ void __launch_bounds__(kPipeThreads, 1)
    embed_pipe_kernel(const PrepareArgs a, const TableRef tab, int32_t D, __half* __restrict__ e) {
  __shared__ PipeSmem sm;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * a.T / gridDim.x);
  const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * a.T / gridDim.x);
  const int n = t1 - t0;
  const int nb = (n + kPipeBatch - 1) / kPipeBatch;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPipeBatches; ++i) {
      mbar_init(smem_u32(&sm.full[i]), 1);
      mbar_init(smem_u32(&sm.empty[i]), kPipeConsumers);
    }
    fence_barrier_init();
  }
  __syncthreads();
  // the projection may start its prologue on SMs this kernel leaves; it reads
  // the rows, gates and state only after this grid has completed
  pdl_launch_dependents();

  if (warp == 0) {
    // ---- producer: row IDs, a lane per token
    for (int b = 0; b < nb; ++b) {
      const int slot = b % kPipeBatches, round = b / kPipeBatches;
      if (round > 0 && !mbar_wait(smem_u32(&sm.empty[slot]), (round - 1) & 1)) {
        if (lane == 0) set_status(a.status, PLE_ERR_TIMEOUT);
        break;
      }
      const int k = b * kPipeBatch + lane;
      if (lane < kPipeBatch && k < n) {
        int32_t s, pos, last, r0, r1;
        sequence_and_rows(a, t0 + k, 0, s, pos, last, r0, r1);
        reinterpret_cast<int2*>(a.ids)[t0 + k] = make_int2(r0, r1);
        PipeTok& pt = sm.tok[slot][lane];
        pt.r0 = r0;
        pt.r1 = r1;
        pt.seq = s;
        pt.pos = pos;
        pt.flags = last ? kFlagLast : 0;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.full[slot]));
    }
  } else {
    // ---- consumers: two tokens of every batch, lane-parallel within the warp.
    //      A token's hidden row does not depend on its row IDs, so its loads
    //      are issued right after the warp's previous gate, before the wait for
    //      the token's batch (the first time, the conv-state snapshot, the new
    //      token history and the offsets check run meanwhile). Every warp waits
    //      for every batch, so that its release of a slot always counts in the
    //      slot's current round.
    const int cw = warp - 1;
    const int H8 = a.H / 8;
    const int D16 = D / 16;
    const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
    const bool with_gate = a.hidden != nullptr;       // null: ple_prepare, the gate comes later
    const bool with_rows = e != nullptr;              // null: the projection gathers the rows itself
    // hv holds the hidden row of the warp's next token; it is loaded as soon as
    // the previous token's gate has used it, so the load runs under that
    // token's dequantisation and stores (and, for a batch's first token, under
    // the wait for the batch's row IDs)
    uint4 hv[kEmbedH4];
    auto load_hidden = [&](int t) {
      const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
#pragma unroll
      for (int r = 0; r < kEmbedH4; ++r) {
        const int j = lane + 32 * r;
        if (j < H8) hv[r] = ld_stream_v4(hrow + j);
      }
    };
    // the k-th token (in the CTA's range) this warp handles after token k
    auto next_token = [&](int b, int half) {
      return half + 1 < kPipeBatch / kPipeConsumers ? b * kPipeBatch + cw + kPipeConsumers * (half + 1)
                                                    : (b + 1) * kPipeBatch + cw;
    };
    if (with_gate && cw < n) load_hidden(t0 + cw);
    bool state_done = false;
    for (int b = 0; b < nb; ++b) {
      const int slot = b % kPipeBatches, round = b / kPipeBatches;
      RowChunk<NV> ca[kEmbedD16], cb[kEmbedD16];
      if (!state_done) {
        state_blocks(a, blockIdx.x, gridDim.x, threadIdx.x - 32, blockDim.x - 32);
        state_done = true;
      }
      if (!mbar_wait(smem_u32(&sm.full[slot]), round & 1)) {
        if (lane == 0) set_status(a.status, PLE_ERR_TIMEOUT);
        break;
      }
#pragma unroll 1
      for (int half = 0; half < kPipeBatch / kPipeConsumers; ++half) {
        const int i = cw + kPipeConsumers * half;
        const int k = b * kPipeBatch + i;
        if (k >= n) break;                                   // warp-uniform
        const int t = t0 + k;
        const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
        const PipeTok pt = sm.tok[slot][i];
        const int64_t ra = pt.r0, rb = a.rows0 + pt.r1;
#pragma unroll
        for (int r = 0; r < kEmbedD16; ++r) {
          const int j = lane + 32 * r;
          if (with_rows && j < D16) {
            ca[r] = load_chunk<NV>(tab.codes, tab.blocks, ra, tab.cs, tab.bs, j);
            cb[r] = load_chunk<NV>(tab.codes, tab.blocks, rb, tab.cs, tab.bs, j);
          }
        }
        const float s0 = with_rows ? __ldg(tab.scales + ra) : 0.f;
        const float s1 = with_rows ? __ldg(tab.scales + rb) : 0.f;
        const float g = with_gate ? gate_warp(hv, hrow, wg, H8, lane) : 0.f;
        const int kn = next_token(b, half);
        if (with_gate && kn < n) load_hidden(t0 + kn);
        if (lane == 0) {
          TokMeta m;
          m.g = g;
          m.seq = pt.seq;
          m.pos = pt.pos;
          m.flags = pt.flags;
          a.meta[t] = m;
        }
        if (!with_rows) continue;                            // warp-uniform
        // e_t = deq(bigram row) + deq(trigram row), fp16
        uint4* erow = reinterpret_cast<uint4*>(e + static_cast<int64_t>(t) * D);
        auto emit = [&](int j, const RowChunk<NV>& x, const RowChunk<NV>& y) {
          uint4 o0, o1;
          deq_chunk<NV>(x, y, s0, s1, o0, o1);
          erow[2 * j] = o0;
          erow[2 * j + 1] = o1;
        };
#pragma unroll
        for (int r = 0; r < kEmbedD16; ++r) {
          const int j = lane + 32 * r;
          if (j < D16) emit(j, ca[r], cb[r]);
        }
        for (int j = lane + 32 * kEmbedD16; j < D16; j += 32)
          emit(j, load_chunk<NV>(tab.codes, tab.blocks, ra, tab.cs, tab.bs, j), load_chunk<NV>(tab.codes, tab.blocks, rb, tab.cs, tab.bs, j));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.empty[slot]));
    }
    if (!state_done) state_blocks(a, blockIdx.x, gridDim.x, threadIdx.x - 32, blockDim.x - 32);
  }
}

// ------------------------------------------------------------------ embed as independent work units
// The same results as embed_pipe_kernel, from two launches whose work units do
// not wait on one another, for large batches.
//
// ids_meta_kernel: a thread per token computes the sequence map, the row IDs
// and the token's sequence, position and last-token flag (the gate field of
// the metadata is left to the gate blocks), and extra blocks do the state
// work. It lets the next grid launch at once.
//
// embed_split_kernel (launched as that grid's programmatic dependent): the
// gate blocks come first, a warp per token; they stream h and write g with no
// wait, since h does not depend on the IDs, and so cover the IDs kernel's
// latency. The gather blocks follow: each waits for the IDs, then a thread
// dequantises one 16-code chunk of both rows into e. Both kinds of block hold
// at most 40 registers per thread (the gate loads h in two halves), so six
// blocks fit on an SM. They walk the tokens from
// the end, so the first tokens' rows are the last written and still in L2 when
// the projection starts on them. A gather block waiting for the IDs grid means
// this grid completes only after that one, which the projection relies on; a
// grid of gate blocks alone waits in its gate blocks.
constexpr int kIdsThreads = 256;
constexpr int kSplitThreads = 256;
constexpr int kSplitGateTokens = kSplitThreads / 32;          // tokens per gate block
constexpr int kSplitBlocksPerSm = 6;                          // 40 registers per thread
constexpr int kSplitMinTokens = 4096;                        // below this the one-kernel form is faster

// FMT: 0 = E4M3 rows (two orders, ids [T][2]), 1 = NVFP4 (the same IDs), 2 = the
// multi-head layout (ids [T][16], a.rows0 rows per head sub-table).
template <int FMT>
__global__ void __launch_bounds__(kIdsThreads) ids_meta_kernel(const PrepareArgs a, int token_blocks) {
  pdl_launch_dependents();
  if (static_cast<int>(blockIdx.x) >= token_blocks) {
    state_blocks(a, blockIdx.x - token_blocks, gridDim.x - token_blocks, threadIdx.x, blockDim.x);
    return;
  }
  const int t = blockIdx.x * kIdsThreads + threadIdx.x;
  if (t >= a.T) return;
  int32_t s, pos, last;
  sequence_of(a, t, true, s, pos, last);
  uint64_t k2, k3;
  keys_of(a, t, s, pos, true, k2, k3);
  if constexpr (FMT == 2) {
    int32_t r[kHeads];
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
      const uint64_t k = ((hh >> 3) ? k3 : k2) ^ (static_cast<uint64_t>(hh & 7) * kHeadMix);
      r[hh] = static_cast<int32_t>(mod_barrett(fold64(k), static_cast<uint64_t>(a.rows0), a.magic0));
    }
    int4* dst = reinterpret_cast<int4*>(a.ids + static_cast<int64_t>(t) * kHeads);
#pragma unroll
    for (int q4 = 0; q4 < kHeads / 4; ++q4) dst[q4] = make_int4(r[4 * q4], r[4 * q4 + 1], r[4 * q4 + 2], r[4 * q4 + 3]);
  } else {
    const int32_t r0 = static_cast<int32_t>(mod_barrett(fold64(k2), static_cast<uint64_t>(a.rows0), a.magic0));
    const int32_t r1 = static_cast<int32_t>(mod_barrett(fold64(k3), static_cast<uint64_t>(a.rows1), a.magic1));
    reinterpret_cast<int2*>(a.ids)[t] = make_int2(r0, r1);
  }
  if (a.meta == nullptr) return;
  if (a.hidden == nullptr) {                  // no gate blocks: the gate field is written later, by the gate kernel
    TokMeta m;
    m.g = 0.f;
    m.seq = s;
    m.pos = pos;
    m.flags = last ? kFlagLast : 0;
    a.meta[t] = m;
  } else {                                    // every field but g, which a gate block writes meanwhile
    int32_t* m = reinterpret_cast<int32_t*>(a.meta + t);
    m[1] = s;
    reinterpret_cast<int2*>(m)[1] = make_int2(pos, last ? kFlagLast : 0);
  }
}

// Gather units of a token: E4M3 and the multi-head layout one 16-code chunk per
// thread; NVFP4 two chunks (16 bytes of packed codes and 2 block-scale bytes
// per row), so that each load is as wide as an E4M3 thread's.
template <int FMT> constexpr int kSplitChunksPerThread = FMT == 1 ? 2 : 1;

template <int FMT>
__global__ void __launch_bounds__(kSplitThreads, kSplitBlocksPerSm)
    embed_split_kernel(const PrepareArgs a, const TableRef tab, int32_t D, __half* __restrict__ e, int32_t n_gate,
                       int32_t n_blocks) {
  pdl_launch_dependents();
  const int64_t b = blockIdx.x;
  if (b < n_gate) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = static_cast<int>(b) * kSplitGateTokens + warp;
    if (t < a.T) {
      const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
      const float g = gate_warp_halves(hrow, reinterpret_cast<const uint4*>(a.w_gate), a.H / 8, lane);
      if (lane == 0) a.meta[t].g = g;
    }
    if (n_blocks == n_gate) pdl_wait();                          // no gather block waits for the IDs grid
    return;
  }
  pdl_wait();                                                    // the row IDs
  constexpr int CPT = kSplitChunksPerThread<FMT>;
  const int units = D / (16 * CPT);                              // per token
  const int64_t idx = (n_blocks - 1 - b) * kSplitThreads + threadIdx.x;
  if (idx >= static_cast<int64_t>(a.T) * units) return;
  const int32_t t = static_cast<int32_t>(idx / units);
  const int c = static_cast<int>(idx - static_cast<int64_t>(t) * units);
  uint4* dst = reinterpret_cast<uint4*>(e + idx * 16 * CPT);
  if constexpr (FMT == 2) {
    const int hd = D / kHeads, cph = hd / 16, hh = c / cph;
    const int64_t row = static_cast<int64_t>(hh) * a.rows0 + a.ids[static_cast<int64_t>(t) * kHeads + hh];
    const uint4 v = ld_stream_v4(tab.codes + row * hd + (c - hh * cph) * 16);
    uint4 o0, o1;
    deq16_one(v, __ldg(tab.scales + row), o0, o1);
    dst[0] = o0;
    dst[1] = o1;
  } else {
    const int2 id = reinterpret_cast<const int2*>(a.ids)[t];
    const int64_t row0 = id.x, row1 = a.rows0 + id.y;
    const float sa = __ldg(tab.scales + row0);
    const float sb = __ldg(tab.scales + row1);
    if constexpr (FMT == 1) {
      // elements [32c, 32c + 32): 16 bytes of codes and 2 block-scale bytes per row
      const uint4 xa = ld_stream_v4(tab.codes + row0 * tab.cs + 16 * c);
      const uint4 xb = ld_stream_v4(tab.codes + row1 * tab.cs + 16 * c);
      const uint32_t ba = ld_stream_u16(tab.blocks + row0 * tab.bs + 2 * c);
      const uint32_t bb = ld_stream_u16(tab.blocks + row1 * tab.bs + 2 * c);
      uint4 o0, o1, o2, o3;
      deq16_nv(make_uint2(xa.x, xa.y), make_uint2(xb.x, xb.y), ba & 0xFFu, bb & 0xFFu, sa, sb, o0, o1);
      deq16_nv(make_uint2(xa.z, xa.w), make_uint2(xb.z, xb.w), ba >> 8, bb >> 8, sa, sb, o2, o3);
      dst[0] = o0;
      dst[1] = o1;
      dst[2] = o2;
      dst[3] = o3;
    } else {
      const RowChunk<false> ca = load_chunk<false>(tab.codes, tab.blocks, row0, tab.cs, tab.bs, c);
      const RowChunk<false> cb = load_chunk<false>(tab.codes, tab.blocks, row1, tab.cs, tab.bs, c);
      uint4 o0, o1;
      deq_chunk<false>(ca, cb, sa, sb, o0, o1);
      dst[0] = o0;
      dst[1] = o1;
    }
  }
}

// ------------------------------------------------------------------ embed as a bulk-copy pipeline
// The gather and gate blocks of embed_split_kernel as one persistent kernel
// (2 CTAs per SM), after ids_meta_kernel, for the two-order layouts (E4M3,
// NVFP4) when the rows and hidden rows start on 16-byte boundaries. (The
// multi-head layout's 16 rows of 160 bytes per token keep the producer warp
// busier than the split kernel's loads: it stays on embed_split_kernel.) Per CTA a ring of token stages, each the
// token's rows (codes and, for NVFP4, block scales), its hidden row and a
// header with the row scales:
//   warp 0, producer: row IDs and scales of 32 tokens at a time (the next 32
//     IDs in flight meanwhile); per token, when its stage is free, the bytes
//     to expect, the bulk copies (cp.async.bulk) of the rows (NVFP4: codes and
//     block scales apart) and the hidden row, the header, then its arrival on
//     the stage's full barrier;
//   warps 1-5, consumers: warp w takes the CTA's tokens w, w + 5, ..., each
//     whole: the rows dequantised into e (a lane per 16-code chunk, 16-byte
//     stores), then the gate from the staged hidden row in the order every
//     gate path takes its sums. Warp w owns stages 2w and 2w + 1, so it meets
//     each stage's phases in order.
// The copy engine keeps about 200 KB per SM in flight, where a thread per
// chunk holds 32 bytes. CTA c takes tokens T - 1 - c, T - 1 - c - grid, ...:
// the first tokens' rows are the last written, still in L2 when the
// projection starts on them. Every wait is bounded and taken alike by a whole
// warp; past the limit the status records a timeout, an abort flag releases
// the other waits, and the producer waits (bounded) for the copies it issued
// before the CTA leaves.
constexpr int kBkConsWarps = 5;
constexpr int kBkStagesPerWarp = 2;
constexpr int kBkStages = kBkConsWarps * kBkStagesPerWarp;
constexpr int kBkThreads = 32 * (1 + kBkConsWarps);
constexpr int kBkCtasPerSm = 2;
constexpr uint32_t kBkHeader = 16;          // the two fp32 row scales (and padding)

// Token k of a CTA: consumer warp k % 5, stage 2 (k % 5) + (k / 5) % 2, the
// (k / 10)-th use of that stage.
__host__ __device__ __forceinline__ int bk_stage(int k) {
  return (k % kBkConsWarps) * kBkStagesPerWarp + (k / kBkConsWarps) % kBkStagesPerWarp;
}

template <int FMT>
__host__ __device__ __forceinline__ uint32_t bk_codes_bytes(int32_t D) {
  return FMT == 1 ? 2u * static_cast<uint32_t>(D / 2 + D / 16) : 2u * D;
}

template <int FMT>
__host__ __device__ __forceinline__ uint32_t bk_stage_bytes(int32_t D, int32_t H, bool gate) {
  return ((bk_codes_bytes<FMT>(D) + 15u) & ~15u) + (gate ? 2u * H : 0u) + kBkHeader;
}

__device__ __forceinline__ bool bk_wait(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag, int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long start = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - start > kWaitLimitCycles) {
      set_status(status, PLE_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(kBkThreads, kBkCtasPerSm)
    embed_bulk_kernel(const PrepareArgs a, const TableRef tab, int32_t D, __half* __restrict__ e, int32_t gate) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kBkStages], empty[kBkStages];
  __shared__ int32_t abort_word;
  volatile int32_t* abort_flag = &abort_word;
  static_assert(FMT == 0 || FMT == 1, "two-order layouts only");
  constexpr int kRowsN = 2;                                  // rows (and scales) per token
  constexpr uint32_t kStageUses = kBkStages;                 // tokens between two uses of a stage
  const uint32_t hid_off = (bk_codes_bytes<FMT>(D) + 15u) & ~15u;
  const uint32_t hdr_off = hid_off + (gate ? 2u * a.H : 0u);
  const uint32_t SB = hdr_off + kBkHeader;
  const uint32_t tx = bk_codes_bytes<FMT>(D) + (gate ? 2u * a.H : 0u);   // bytes a token's copies bring
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, G = gridDim.x;
  const int nk = c < a.T ? (a.T - 1 - c) / G + 1 : 0;       // this CTA's tokens
  auto tok = [&](int k) { return a.T - 1 - (c + k * G); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBkStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    pdl_wait();                                              // the row IDs
    // lane l: the two row IDs of token k0 + l
    int32_t cur[kRowsN], nxt[kRowsN];
    auto load_ids = [&](int k0, int32_t (&v)[kRowsN]) {
      const int k = k0 + lane;
      if (k < nk) {
        const int2 x = reinterpret_cast<const int2*>(a.ids)[tok(k)];
        v[0] = x.x;
        v[1] = x.y;
      } else {
#pragma unroll
        for (int r = 0; r < kRowsN; ++r) v[r] = 0;
      }
    };
    auto global_row = [&](int r, int32_t id) -> int64_t {   // row r of a token: its global row
      return r == 0 ? static_cast<int64_t>(id) : a.rows0 + id;
    };
    load_ids(0, cur);
    int issued = 0;
    bool stop = false;                                       // warp-uniform
    for (int k0 = 0; k0 < nk && !stop; k0 += 32) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      if (k0 + 32 < nk) load_ids(k0 + 32, nxt);
      float sc[kRowsN];                                       // lane l: the row scales of token k0 + l
#pragma unroll
      for (int r = 0; r < kRowsN; ++r) sc[r] = k0 + lane < nk ? __ldg(tab.scales + global_row(r, cur[r])) : 0.f;
      for (int j = 0; j < 32 && k0 + j < nk; ++j) {
        const int k = k0 + j, s = bk_stage(k);
        if (k >= kBkStages &&
            !__all_sync(0xffffffffu, bk_wait(smem_u32(&empty[s]), (k / kStageUses - 1) & 1, abort_flag, a.status))) {
          stop = true;
          break;
        }
        const int t = tok(k);
        uint8_t* st = smem + static_cast<size_t>(s) * SB;
        const uint32_t fb = smem_u32(&full[s]);
        if (lane == 0) mbar_expect_tx(fb, tx);
        __syncwarp();
        // lane r < kRowsN copies row r of token k
        int32_t id = 0;
#pragma unroll
        for (int r = 0; r < kRowsN; ++r) {
          const int32_t v = __shfl_sync(0xffffffffu, cur[r], j);
          if (lane == r) id = v;
        }
        if (lane < kRowsN) {
          const int64_t row = global_row(lane, id);
          if constexpr (FMT == 1) {
            // the row's D/2 code bytes, then its D/16 block-scale bytes: one copy
            // when the table keeps them side by side
            const uint32_t o = lane * static_cast<uint32_t>(D / 2 + D / 16);
            if (tab.nv_rows) {
              bulk_load(smem_u32(st + o), tab.codes + row * tab.cs, static_cast<uint32_t>(D / 2 + D / 16), fb);
            } else {
              bulk_load(smem_u32(st + o), tab.codes + row * tab.cs, static_cast<uint32_t>(D / 2), fb);
              bulk_load(smem_u32(st + o + D / 2), tab.blocks + row * tab.bs, static_cast<uint32_t>(D / 16), fb);
            }
          } else {
            bulk_load(smem_u32(st + lane * D), tab.codes + row * D, static_cast<uint32_t>(D), fb);
          }
        }
        if (gate && lane == 31)
          bulk_load(smem_u32(st + hid_off), a.hidden + static_cast<int64_t>(t) * a.H, 2u * a.H, fb);
        // the header: lane r < kRowsN writes row r's scale
        float* hdr = reinterpret_cast<float*>(st + hdr_off);
#pragma unroll
        for (int r = 0; r < kRowsN; ++r) {
          const float v = __shfl_sync(0xffffffffu, sc[r], j);
          if (lane == r) hdr[r] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(fb);
        issued = k + 1;
      }
#pragma unroll
      for (int r = 0; r < kRowsN; ++r) cur[r] = nxt[r];
    }
    // copies in flight land before the CTA's shared memory is released
    for (int k = max(0, issued - kBkStages); k < issued; ++k) {
      const long long start = clock64();
      while (!mbar_try_wait(smem_u32(&full[bk_stage(k)]), (k / kStageUses) & 1) && clock64() - start < kWaitLimitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int w = warp - 1;
    const int units = D / 16;
    const int H8 = a.H / 8;
    const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
    uint4 wv[kEmbedH4];
    if (gate) {
#pragma unroll
      for (int r = 0; r < kEmbedH4; ++r) {
        const int j = lane + 32 * r;
        if (j < H8) wv[r] = __ldg(wg + j);
      }
    }
    for (int k = w; k < nk; k += kBkConsWarps) {
      const int s = bk_stage(k);
      if (!__all_sync(0xffffffffu, bk_wait(smem_u32(&full[s]), (k / kStageUses) & 1, abort_flag, a.status))) break;
      const uint8_t* st = smem + static_cast<size_t>(s) * SB;
      const float* hdr = reinterpret_cast<const float*>(st + hdr_off);   // the two row scales
      const int t = tok(k);
      // the rows -> e: lane l takes chunks l, l + 32, ...
      uint4* dst = reinterpret_cast<uint4*>(e + static_cast<int64_t>(t) * D);
#pragma unroll 5
      for (int j = lane; j < units; j += 32) {
        uint4 o0, o1;
        if constexpr (FMT == 1) {
          const uint32_t rb = static_cast<uint32_t>(D / 2 + D / 16);
          const uint2 ca = *reinterpret_cast<const uint2*>(st + j * 8);
          const uint2 cb = *reinterpret_cast<const uint2*>(st + rb + j * 8);
          deq16_nv(ca, cb, st[D / 2 + j], st[rb + D / 2 + j], hdr[0], hdr[1], o0, o1);
        } else {
          deq16(*reinterpret_cast<const uint4*>(st + j * 16), *reinterpret_cast<const uint4*>(st + D + j * 16),
                hdr[0], hdr[1], o0, o1);
        }
        dst[2 * j] = o0;
        dst[2 * j + 1] = o1;
      }
      if (gate) {
        const uint4* hv = reinterpret_cast<const uint4*>(st + hid_off);
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kEmbedH4; ++r) {
          const int j = lane + 32 * r;
          if (j < H8) gate_dot8(acc, hv[j], wv[r]);
        }
        for (int j = lane + 32 * kEmbedH4; j < H8; j += 32) gate_dot8(acc, hv[j], __ldg(wg + j));
        const float g = gate_finish(acc);
        if (lane == 0) a.meta[t].g = g;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
  }
}

// ------------------------------------------------------------------ bounded-wait self-test
// One warp waits, through the same bounded wait the library's kernels use, on
// an mbarrier that expects one arrival nobody makes. The wait runs out after
// `limit` cycles; the kernel then records PLE_ERR_TIMEOUT and returns.
__global__ void wait_selftest_kernel(int32_t* status, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (!mbar_wait(smem_u32(&bar), 0, limit) && threadIdx.x == 0) set_status(status, PLE_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ W_proj conversion
__global__ void convert_w_kernel(const __nv_bfloat16* __restrict__ w, int32_t D, int32_t H,
                                 __half* __restrict__ w16, int32_t* bad) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int k = k0 + i, j = j0 + threadIdx.x;
    float v = 0.f;
    if (k < D && j < H) v = __bfloat162float(w[static_cast<int64_t>(k) * H + j]);
    if (!(fabsf(v) <= 65504.f)) atomicExch(bad, 1);   // also catches NaN
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int j = j0 + i, k = k0 + threadIdx.x;
    if (k < D && j < H) w16[static_cast<int64_t>(j) * D + k] = __float2half_rn(tile[threadIdx.x][i]);
  }
}

// ------------------------------------------------------------------ combine (packed batch)
__device__ __forceinline__ void store_out(void* out, int32_t out_f32, int64_t idx, float v) {
  if (out_f32) reinterpret_cast<float*>(out)[idx] = v;
  else reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

__global__ void __launch_bounds__(128) combine_forward_kernel(const CombineArgs a) {
  const int32_t t = blockIdx.y;
  const int32_t j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= a.H || t >= a.T) return;
  pdl_wait();                                  // the partial sums come from the projection
  const TokMeta mt = a.meta[t];
  float u[4];                          // u[k] = u_{t-3+k}
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int lag = 3 - k;
    if (mt.pos - lag >= 0) {
      const int32_t tk = t - lag;
      float v = 0.f;
      for (int sp = 0; sp < a.k_splits; ++sp)
        v += a.partial[(static_cast<int64_t>(sp) * a.T + tk) * a.H + j];
      u[k] = a.meta[tk].g * v;
    } else {
      u[k] = a.conv0 ? a.conv0[(static_cast<int64_t>(mt.seq) * 3 + (3 + mt.pos - lag)) * a.H + j] : 0.f;
    }
  }
  const float4 cw = reinterpret_cast<const float4*>(a.conv_w)[j];
  const float y = cw.x * u[0] + cw.y * u[1] + cw.z * u[2] + cw.w * u[3];
  const int64_t idx = static_cast<int64_t>(t) * a.H + j;
  store_out(a.out, a.out_f32, idx, __bfloat162float(a.hidden[idx]) + y);
  if (a.conv_state != nullptr && (mt.flags & kFlagLast)) {
    float* cs = a.conv_state + static_cast<int64_t>(mt.seq) * 3 * a.H + j;
    cs[0] = u[1];
    cs[a.H] = u[2];
    cs[2 * a.H] = u[3];
    if (j == 0) {
      a.hist_state[2 * mt.seq] = a.hist_new[2 * mt.seq];
      a.hist_state[2 * mt.seq + 1] = a.hist_new[2 * mt.seq + 1];
    }
  }
}

// ------------------------------------------------------------------ combine (decode step)
__global__ void __launch_bounds__(128) combine_decode_kernel(const DecodeCombineArgs a) {
  const int32_t b = blockIdx.y;
  const int32_t j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= a.H || b >= a.B) return;
  pdl_wait();                                  // the partial sums come from the projection
  int32_t nc = a.n_commit ? a.n_commit[b] : a.q;
  if (nc < 1 || nc > a.q) {
    if (j == 0) set_status(a.status, PLE_ERR_RANGE);
    nc = max(1, min(nc, a.q));
  }
  float* cs = a.conv_state + static_cast<int64_t>(b) * 3 * a.H + j;
  float w0 = cs[0], w1 = cs[a.H], w2 = cs[2 * a.H];
  float c0 = w0, c1 = w1, c2 = w2;
  const float4 cw = reinterpret_cast<const float4*>(a.conv_w)[j];
  for (int i = 0; i < a.q; ++i) {
    const int32_t t = b * a.q + i;
    const int32_t T = a.B * a.q;
    float v = 0.f;
    for (int sp = 0; sp < a.k_splits; ++sp) v += a.partial[(static_cast<int64_t>(sp) * T + t) * a.H + j];
    const float u = a.meta[t].g * v;
    const float y = cw.x * w0 + cw.y * w1 + cw.z * w2 + cw.w * u;
    w0 = w1; w1 = w2; w2 = u;
    const int64_t idx = static_cast<int64_t>(t) * a.H + j;
    store_out(a.out, a.out_f32, idx, __bfloat162float(a.hidden[idx]) + y);
    if (i == nc - 1) { c0 = w0; c1 = w1; c2 = w2; }
  }
  cs[0] = c0;
  cs[a.H] = c1;
  cs[2 * a.H] = c2;
  if (j == 0) {
    // last two committed tokens, taking carried ones when fewer than two were committed
    const int32_t* tk = a.tokens + static_cast<int64_t>(b) * a.q;
    const int32_t h0 = a.hist[2 * b], h1 = a.hist[2 * b + 1];
    const int32_t n1 = tk[nc - 1];
    const int32_t n0 = nc >= 2 ? tk[nc - 2] : h1;
    (void)h0;
    a.hist[2 * b] = n0;
    a.hist[2 * b + 1] = n1;
  }
}

// The kernels that run in a chain with a projection or under programmatic
// dependent launch take the largest shared-memory carveout (prefer_max_shared).
cudaError_t configure_chain_kernels() {
  static PerDeviceOnce configured;
  return configured.run([] {
    cudaError_t r = cudaSuccess;
    auto set = [&r](auto kernel) {
      if (r == cudaSuccess) r = prefer_max_shared(kernel);
    };
    set(ids_meta_kernel<0>);
    set(ids_meta_kernel<1>);
    set(ids_meta_kernel<2>);
    set(embed_split_kernel<0>);
    set(embed_split_kernel<1>);
    set(embed_split_kernel<2>);
    set(embed_pipe_kernel<false>);
    set(embed_pipe_kernel<true>);
    set(embed_heads_kernel);
    set(gate_kernel);
    set(combine_forward_kernel);
    set(combine_decode_kernel);
    return r;
  });
}

}  // namespace

cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t stream) {
  const int token_blocks = (a.T + kPrepWarps - 1) / kPrepWarps;
  int state_blocks = 1;
  if (a.conv_in != nullptr) {
    const int64_t n4 = static_cast<int64_t>(a.S) * 3 * a.H / 4;
    const int64_t want = (n4 + 255) / 256;
    state_blocks = static_cast<int>(want < 1 ? 1 : (want > 148 ? 148 : want));
  }
  prepare_kernel<<<token_blocks + state_blocks, 256, 0, stream>>>(with_magic(a), token_blocks);
  return cudaGetLastError();
}

// The embed of a batch of kSplitMinTokens or more as two launches (all table
// formats): the IDs kernel, then the gate and gather blocks as its dependent.
// Whether embed_bulk_kernel<FMT> (FMT 0 or 1) takes the rows and gates of a
// batch: every bulk copy starts on a 16-byte boundary and is a multiple of 16
// bytes, and kBkCtasPerSm CTAs with kBkStages stages fit an SM's shared memory.
constexpr size_t kBkSmemPerCta = 112 * 1024;

template <int FMT>
bool embed_bulk_ok(const PrepareArgs& a, const TableRef& table, int32_t D, const __half* e, bool gate) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (e == nullptr || !al16(e) || !al16(table.codes)) return false;
  if (FMT == 0 ? D % 16 != 0 : D % 256 != 0) return false;   // NVFP4: D / 16 block-scale bytes per row
  if (FMT == 1 && (!al16(table.blocks) || table.cs % 16 != 0 || table.bs % 16 != 0)) return false;
  if (gate && (a.H % 8 != 0 || !al16(a.hidden) || !al16(a.w_gate))) return false;
  return static_cast<size_t>(kBkStages) * bk_stage_bytes<FMT>(D, a.H, gate) <= kBkSmemPerCta;
}

template <int FMT>
cudaError_t launch_embed_split(const PrepareArgs& a, const TableRef& table, int32_t D, __half* e,
                               int32_t num_sms, cudaStream_t stream, int* kernels) {
  const PrepareArgs am = with_magic(a);
  const int token_blocks = (a.T + kIdsThreads - 1) / kIdsThreads;
  int sblocks = 1;
  if (a.conv_in != nullptr) {
    const int64_t want = (static_cast<int64_t>(a.S) * 3 * a.H / 4 + kIdsThreads - 1) / kIdsThreads;
    sblocks = static_cast<int>(want < 1 ? 1 : (want > 148 ? 148 : want));
  }
  ids_meta_kernel<FMT><<<token_blocks + sblocks, kIdsThreads, 0, stream>>>(am, token_blocks);
  cudaError_t r = cudaGetLastError();
  if (r != cudaSuccess) return r;
  const bool gate = a.hidden != nullptr && a.meta != nullptr;
  if constexpr (FMT != 2) {
  if (embed_bulk_ok<FMT>(a, table, D, e, gate)) {
    static PerDeviceOnce configured;
    r = configured.run([] {
      cudaError_t x = cudaFuncSetAttribute(embed_bulk_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kBkSmemPerCta));
      return x == cudaSuccess ? prefer_max_shared(embed_bulk_kernel<FMT>) : x;
    });
    if (r != cudaSuccess) return r;
    if (kernels != nullptr) *kernels = 2;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(static_cast<int64_t>(kBkCtasPerSm) * num_sms, a.T)));
    cfg.blockDim = dim3(kBkThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(kBkStages) * bk_stage_bytes<FMT>(D, a.H, gate);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, embed_bulk_kernel<FMT>, am, table, D, e, gate ? 1 : 0);
  }
  }
  const int64_t units = static_cast<int64_t>(a.T) * (D / (16 * kSplitChunksPerThread<FMT>));
  const int64_t n_gate = gate ? (a.T + kSplitGateTokens - 1) / kSplitGateTokens : 0;
  const int64_t n_gather = e != nullptr ? (units + kSplitThreads - 1) / kSplitThreads : 0;
  if (n_gate + n_gather == 0) return cudaSuccess;
  if (kernels != nullptr) *kernels = 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_gate + n_gather));
  cfg.blockDim = dim3(kSplitThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int32_t ng = static_cast<int32_t>(n_gate), nblk = static_cast<int32_t>(n_gate + n_gather);
  return cudaLaunchKernelEx(&cfg, embed_split_kernel<FMT>, am, table, D, e, ng, nblk);
}

cudaError_t launch_embed(const PrepareArgs& a, const TableRef& table, int32_t D, __half* e, int32_t num_sms,
                         cudaStream_t stream, int* kernels) {
  if (kernels != nullptr) *kernels = 1;
  const cudaError_t cfg_err = configure_chain_kernels();
  if (cfg_err != cudaSuccess) return cfg_err;
  if (a.T >= kSplitMinTokens) {
    if (table.nvfp4) return launch_embed_split<1>(a, table, D, e, num_sms, stream, kernels);
    return launch_embed_split<0>(a, table, D, e, num_sms, stream, kernels);
  }
  const bool state = a.conv_in != nullptr || a.hist_new != nullptr;
  // small batches spread over the SMs: a few tokens per CTA, no warp taking two in turn
  const int grid = state ? num_sms : std::min<int>(num_sms, a.T);
  if (table.nvfp4)
    embed_pipe_kernel<true><<<grid, kPipeThreads, 0, stream>>>(with_magic(a), table, D, e);
  else
    embed_pipe_kernel<false><<<grid, kPipeThreads, 0, stream>>>(with_magic(a), table, D, e);
  return cudaGetLastError();
}

cudaError_t launch_embed_heads(const PrepareArgs& a, const TableRef& table, int32_t D, __half* e, int32_t num_sms,
                               cudaStream_t stream, int* kernels) {
  if (kernels != nullptr) *kernels = 1;
  const cudaError_t cfg_err = configure_chain_kernels();
  if (cfg_err != cudaSuccess) return cfg_err;
  if (a.T >= kSplitMinTokens && a.ids != nullptr) return launch_embed_split<2>(a, table, D, e, num_sms, stream, kernels);
  const int token_blocks = (a.T + 7) / 8;
  int sblocks = 1;
  if (a.conv_in != nullptr) {
    const int64_t want = (static_cast<int64_t>(a.S) * 3 * a.H / 4 + 255) / 256;
    sblocks = static_cast<int>(want < 1 ? 1 : (want > 148 ? 148 : want));
  }
  embed_heads_kernel<<<token_blocks + sblocks, 256, 0, stream>>>(with_magic(a), table, D, e, token_blocks);
  return cudaGetLastError();
}

cudaError_t launch_gather_heads(const int32_t* ids, int32_t T, const TableRef& table, int64_t rows, int32_t D,
                                __half* e, cudaStream_t stream) {
  const int64_t threads = static_cast<int64_t>(T) * (D / 16);
  gather_heads_kernel<<<static_cast<int>((threads + 255) / 256), 256, 0, stream>>>(ids, T, table, rows, D, e);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int32_t* status, long long limit_cycles, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit_cycles);
  return cudaGetLastError();
}

cudaError_t launch_gate(const PrepareArgs& a, cudaStream_t stream) {
  const cudaError_t cfg_err = configure_chain_kernels();
  if (cfg_err != cudaSuccess) return cfg_err;
  const int token_blocks = (a.T + 7) / 8;
  int state_blocks = 0;
  if (a.conv_in != nullptr) {
    const int64_t want = (static_cast<int64_t>(a.S) * 3 * a.H / 4 + 255) / 256;
    state_blocks = static_cast<int>(want < 1 ? 1 : (want > 148 ? 148 : want));
  }
  gate_kernel<<<token_blocks + state_blocks, 256, 0, stream>>>(a, token_blocks);
  return cudaGetLastError();
}

cudaError_t launch_gather(const int32_t* ids, int32_t T, const TableRef& table, int64_t rows0, int64_t rows1,
                          int32_t D, __half* e, bool reduce_ids, cudaStream_t stream) {
  const int64_t threads = static_cast<int64_t>(T) * (D / 16);
  const int blocks = static_cast<int>((threads + 255) / 256);
  const int2* id2 = reinterpret_cast<const int2*>(ids);
  if (table.nvfp4)
    gather_kernel<true><<<blocks, 256, 0, stream>>>(id2, T, table, rows0, rows1, D, e, reduce_ids ? 1 : 0);
  else
    gather_kernel<false><<<blocks, 256, 0, stream>>>(id2, T, table, rows0, rows1, D, e, reduce_ids ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_convert_w(const __nv_bfloat16* w, int32_t D, int32_t H, __half* w16, int32_t* bad,
                             cudaStream_t stream) {
  dim3 grid((H + 31) / 32, (D + 31) / 32), block(32, 8);
  convert_w_kernel<<<grid, block, 0, stream>>>(w, D, H, w16, bad);
  return cudaGetLastError();
}

// Combine kernels start under programmatic dependent launch: their blocks wait
// for the projection before they read anything it writes.
template <typename Kernel, typename Args>
cudaError_t launch_after_projection(Kernel kernel, dim3 grid, const Args& a, cudaStream_t stream) {
  const cudaError_t cfg_err = configure_chain_kernels();
  if (cfg_err != cudaSuccess) return cfg_err;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_combine_forward(const CombineArgs& a, cudaStream_t stream) {
  return launch_after_projection(combine_forward_kernel, dim3((a.H + 127) / 128, a.T), a, stream);
}

cudaError_t launch_combine_decode(const DecodeCombineArgs& a, cudaStream_t stream) {
  return launch_after_projection(combine_decode_kernel, dim3((a.H + 127) / 128, a.B), a, stream);
}

}  // namespace ple
