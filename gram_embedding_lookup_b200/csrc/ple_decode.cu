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
//     of fp16, 123 KB at D = 2560) is requested by 16-byte cp.async from every
//     lane (each warp copies the K range it multiplies; bulk copies of such
//     short pieces measured slower) before it waits for the embed kernel
//     (programmatic dependent launch), so the W_proj stream runs under the
//     embed kernel. After the wait it copies e the same way, takes
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

constexpr int kTwoOrderMaxTok = 8;     // two-order steps: order 0 of token t in row t, order 1 in row t + 8

// 16 codes of one row as exact fp16 values: E4M3 codes as they are; NVFP4
// codes times their block scale (an E2M1 value times an E4M3 value has at most
// 6 significant bits and lies in the fp16 range, so the product is exact).
template <bool NV>
__device__ __forceinline__ void codes_to_f16(const RowChunk<NV>& x, uint4& o0, uint4& o1) {
  uint32_t h[8];
  if constexpr (NV) {
    const __half2 bs = __float2half2_rn(e4m3x2_cvt(x.b & 0xFFu).x);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t w = k < 4 ? x.c.x : x.c.y;
      const __half2 v = __hmul2(e2m1x2_cvt(w >> (8 * (k & 3))), bs);
      h[k] = *reinterpret_cast<const uint32_t*>(&v);
    }
  } else {
    const uint32_t w[4] = {x.c.x, x.c.y, x.c.z, x.c.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[k >> 1] >> (16 * (k & 1))) & 0xFFFFu), __NV_E4M3);
      h[k] = *reinterpret_cast<const uint32_t*>(&r);
    }
  }
  o0 = make_uint4(h[0], h[1], h[2], h[3]);
  o1 = make_uint4(h[4], h[5], h[6], h[7]);
}

// ------------------------------------------------------------------ embed: rows, metadata, gate
// FMT: 0 = E4M3 rows (two orders), 1 = NVFP4 rows, 2 = the multi-head E4M3 layout.
// Thread j of the block takes 16-code chunks j, j + blockDim, ... of the
// token's row (of all 16 head rows side by side for FMT 2); warp 0 also
// computes the gate.
constexpr int kEmbedThreads = 256;    // most threads of a decode_embed_kernel block

template <int FMT>
__global__ void __launch_bounds__(kEmbedThreads) decode_embed_kernel(const DecodeEmbedArgs a) {
  constexpr bool NV = FMT == 1;
  pdl_launch_dependents();             // the projection's prologue (its W_proj copies) may start now
  if (a.w16 != nullptr && threadIdx.x < 32) {
    // this block's share of W_proj into L2 (16 KB pieces, one lane each), spread
    // over every block of the grid, which has a block per SM at least: the
    // projection after this kernel then reads it from L2, and when the step is
    // prepared ahead of its hidden states the stream is off the step's path
    const int64_t pieces = (a.w16_bytes + 16383) / 16384;
    const int64_t p0 = pieces * blockIdx.x / gridDim.x, p1 = pieces * (blockIdx.x + 1) / gridDim.x;
    const uint8_t* wb = reinterpret_cast<const uint8_t*>(a.w16);
    for (int64_t pc = p0 + threadIdx.x; pc < p1; pc += 32) {
      const int64_t off = pc * 16384;
      const int64_t left = a.w16_bytes - off;
      bulk_prefetch_l2(wb + off, static_cast<uint32_t>(left < 16384 ? left : 16384));
    }
  }
  if (static_cast<int>(blockIdx.x) >= a.B * a.q) return;    // a prefetch-only block
  const int t = blockIdx.x;
  const int b = t / a.q, i = t - b * a.q;
  const int lane = threadIdx.x & 31;
  const bool gate_warp0 = a.hidden != nullptr && threadIdx.x < 32;
  const int H8 = a.H / 8;
  const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
  uint4 wv[kEmbedH4];
  if (gate_warp0) {                    // w_gate is a weight: load it before the wait
#pragma unroll
    for (int r = 0; r < kEmbedH4; ++r) {
      const int j = lane + 32 * r;
      if (j < H8) wv[r] = __ldg(wg + j);
    }
  }
  pdl_wait();                          // tokens, history and hidden may come from the previous kernel
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
    if (a.codes2) {
      // the two rows as exact fp16 codes (rows t and t + 8 of e), the scales apart
      uint4* crow1 = reinterpret_cast<uint4*>(a.e + static_cast<int64_t>(t + kTwoOrderMaxTok) * a.D);
      for (int j = threadIdx.x; j < nch; j += blockDim.x) {
        const RowChunk<NV> x = load_chunk<NV>(a.table, a.blocks, r0, a.cs, a.bs, j);
        const RowChunk<NV> y = load_chunk<NV>(a.table, a.blocks, r1, a.cs, a.bs, j);
        uint4 o0, o1;
        codes_to_f16<NV>(x, o0, o1);
        erow[2 * j] = o0;
        erow[2 * j + 1] = o1;
        codes_to_f16<NV>(y, o0, o1);
        crow1[2 * j] = o0;
        crow1[2 * j + 1] = o1;
      }
      if (threadIdx.x == 0) reinterpret_cast<float2*>(a.row_scales)[t] = make_float2(s0, s1);
    } else {
      for (int j = threadIdx.x; j < nch; j += blockDim.x) {
        const RowChunk<NV> x = load_chunk<NV>(a.table, a.blocks, r0, a.cs, a.bs, j);
        const RowChunk<NV> y = load_chunk<NV>(a.table, a.blocks, r1, a.cs, a.bs, j);
        uint4 o0, o1;
        deq_chunk<NV>(x, y, s0, s1, o0, o1);
        erow[2 * j] = o0;
        erow[2 * j + 1] = o1;
      }
    }
  }
  if (threadIdx.x < 32) {
    const float g = gate_warp0 ? gate_warp_pre(hv, wv, hrow, wg, H8, lane) : 0.f;
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
  float cst[kPjMaxTok][3][kPjMaxChan];                      // carried conv state at this CTA's channels
  __nv_bfloat16 res[kPjMaxTok][kPjMaxChan];                 // hidden at this CTA's channels
  TokMeta meta[kPjMaxTok];                                  // gates (prepared steps)
  float g[kPjMaxTok];                                       // gates
  int32_t tok[kPjMaxTok];                                   // the step's tokens
  int32_t hist[kPjMaxTok][2];                               // the token history before the step
  int32_t nc[kPjMaxTok];                                    // n_commit
  int64_t rid[kPjMaxTok][2];                                // fused steps: global rows of the two orders
  float sc[kPjMaxTok][2];                                   // two-order steps: the rows' scales
  int32_t rid16[kPjMaxTok][kHeads];                         // fused steps, multi-head layout
  uint64_t wbar;                                            // W_proj rows landed
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

// How the kernel gets the step's rows:
//   kRowsE      from e (fp16 e_t, decode_embed_kernel);
//   kRowsHash   it hashes the tokens and gathers and dequantises e_t itself;
//   kRowsHash2  it hashes the tokens and gathers the two orders' codes as exact
//               fp16 A rows (token t's order-0 row in A row t, order-1 row in A
//               row t + 8, T <= 8), the row scales applied after the products:
//               v_t = s0 * (codes0 . W) + s1 * (codes1 . W);
//   kRowsCodes2 the same with the codes and row scales decode_embed_kernel wrote.
// The two-order forms leave no rounding of e_t to fp16 and cost one
// conversion per code pair instead of a fused multiply-add and a rounding per
// element; a step gives the same bits through ple_decode_step and
// ple_decode_prepare + ple_decode_step_prepared.
constexpr int kRowsE = 0, kRowsHash = 1, kRowsHash2 = 2, kRowsCodes2 = 3;

// FMT = 0, 1, 2: E4M3, NVFP4 or multi-head table (unused with kRowsE).
template <int FMT, int MODE>
__global__ void __launch_bounds__(kPjThreads, 1) decode_proj_kernel(const DecodeProjArgs a) {
  constexpr bool FUSED = MODE == kRowsHash || MODE == kRowsHash2;   // the kernel reads the history itself
  constexpr bool TWO = MODE == kRowsHash2 || MODE == kRowsCodes2;
  constexpr bool COPIED = MODE == kRowsE || MODE == kRowsCodes2;      // rows from decode_embed_kernel
  static_assert(!TWO || FMT != 2, "the multi-head rows carry a scale per head: no two-order form");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_s + 127u) & ~127u) - raw_s);
  const int T = a.B * a.q;
  const int ldr = a.D + 8;                                   // fp16 per shared-memory row
  __half* ws = reinterpret_cast<__half*>(base);              // [max_groups * 8][ldr]
  __half* es = ws + static_cast<int64_t>(a.max_groups) * kPjGroup * ldr;   // [T][ldr]
  ProjSmem* sm = reinterpret_cast<ProjSmem*>(es + static_cast<int64_t>(TWO ? kPjMaxTok : T) * ldr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G8 = a.H / kPjGroup;
  const int g0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * G8 / gridDim.x);
  const int g1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * G8 / gridDim.x);
  const int ng = g1 - g0, c0 = g0 * kPjGroup, nch = ng * kPjGroup;
  const int KS = a.D / 16;
  const int kb = ks_begin(warp, KS), ke = ks_begin(warp + 1, KS);

  // ---- 1. the CTA's W_proj rows (constant since ple_create) by bulk copies,
  //         lane r of the last warp copying row r, counted in bytes on wbar:
  //         issued before the wait, so that under programmatic dependent launch
  //         they run under the kernel before, and without holding any warp, so
  //         that the hashing starts at once. Before the wait also the conv taps
  //         of this lane's channel and, when the gates are computed here, w_gate.
  const int kchunks = (ke - kb) * 2;                         // 16-byte chunks of one row in this warp's K range
  const bool second = lane + 32 < kchunks;
  const uint32_t wbar = smem_u32(&sm->wbar);
  if (warp == kPjWarps - 1) {
    if (lane == 0) {
      mbar_init(wbar, 1);
      fence_barrier_init();
      mbar_arrive_expect_tx(wbar, static_cast<uint32_t>(nch) * a.D * 2u);
    }
    __syncwarp();
    for (int r = lane; r < nch; r += 32)
      bulk_load(smem_u32(ws + r * ldr), a.w16 + static_cast<int64_t>(c0 + r) * a.D, a.D * 2u, wbar);
  }
  // items: (sequence b, channel c), warp w takes sequences w, w + 8, ..., lane c
  float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane < nch) cw = __ldg(reinterpret_cast<const float4*>(a.conv_w) + c0 + lane);
  const int H8 = a.H / 8;
  const uint4* wg = reinterpret_cast<const uint4*>(a.w_gate);
  uint4 wv[kEmbedH4];
  if (!a.gate_ready) {
#pragma unroll
    for (int r = 0; r < kEmbedH4; ++r) {
      const int j = lane + 32 * r;
      if (j < H8) wv[r] = __ldg(wg + j);
    }
  }
  pdl_launch_dependents();
  pdl_wait();                                                // tokens, e, meta, hidden and the state are ready

  // ---- 2. everything the step reads, in one round trip: the rows or codes
  //         decode_embed_kernel wrote (this warp's K range) and the codes' row
  //         scales; residual, state, gates, tokens, history and n_commit into
  //         shared memory by cp.async
  if constexpr (COPIED) {
    // this warp's K range of the rows (two-order: rows t and t + 8 of token t)
    if (lane < kchunks) {
      for (int r = 0; r < (TWO ? kPjMaxTok : T); ++r) {
        if (TWO && (r & 7) >= T) continue;
        const __half* src = a.e + static_cast<int64_t>(r) * a.D + kb * 16 + lane * 8;
        const uint32_t dst = smem_u32(es + r * ldr + kb * 16 + lane * 8);
        cp_async_16(dst, src);
        if (second) cp_async_16(dst + 512, src + 256);
      }
    }
    if (TWO && tid < 2 * T) cp_async_4(smem_u32(&sm->sc[tid >> 1][tid & 1]), a.row_scales + tid);
  }
  {
    // hidden at this CTA's channels: ng 16-byte pieces per token
    for (int x = tid; x < T * ng; x += kPjThreads) {
      const int t = x / ng, p = x - t * ng;
      cp_async_16(smem_u32(&sm->res[t][p * 8]), a.hidden + static_cast<int64_t>(t) * a.H + c0 + p * 8);
    }
    // carried conv state: 2 ng 16-byte pieces per (sequence, tap)
    const int pc = 2 * ng;
    for (int x = tid; x < a.B * 3 * pc; x += kPjThreads) {
      const int bk = x / pc, p = x - bk * pc;
      cp_async_16(smem_u32(&sm->cst[bk / 3][bk % 3][p * 4]), a.conv_state + static_cast<int64_t>(bk) * a.H + c0 + p * 4);
    }
    if (tid < T) {
      if (a.gate_ready) cp_async_16(smem_u32(&sm->meta[tid]), a.meta + tid);
      cp_async_4(smem_u32(&sm->tok[tid]), a.tokens + tid);
    }
    if (tid < a.B) {
      cp_async_4(smem_u32(&sm->hist[tid][0]), a.hist + 2 * tid);
      cp_async_4(smem_u32(&sm->hist[tid][1]), a.hist + 2 * tid + 1);
      if (a.n_commit) cp_async_4(smem_u32(&sm->nc[tid]), a.n_commit + tid);
    }
  }
  cp_async_commit();
  uint4 hv[kEmbedH4];
  if (!a.gate_ready && warp < T) {                           // the gate loads need no row ID
#pragma unroll
    for (int r = 0; r < kEmbedH4; ++r) {
      const int j = lane + 32 * r;
      if (j < H8) hv[r] = ld_stream_v4(reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(warp) * a.H) + j);
    }
  }
  // gates: warp w takes tokens w, w + 8, ... (its first token's hidden row is in
  // flight already); computed while the row IDs are found, before any row is read
  auto gates = [&] {
    if (!a.gate_ready) {
      for (int t = warp; t < T; t += kPjWarps) {
        const uint4* hrow = reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H);
        if (t != warp) {
#pragma unroll
          for (int r = 0; r < kEmbedH4; ++r) {
            const int j = lane + 32 * r;
            if (j < H8) hv[r] = ld_stream_v4(hrow + j);
          }
        }
        const float g = gate_warp_pre(hv, wv, hrow, wg, H8, lane);
        if (lane == 0) sm->g[t] = g;
      }
    }
  };
  int32_t ticket = -1;
  float s_two[2] = {0.f, 0.f};                               // two-order forms: this thread's token's row scales
  if constexpr (FUSED) {
    // row IDs: thread t hashes token t (for the multi-head layout, thread (t, head))
    constexpr int kIdsPerTok = FMT == 2 ? kHeads : 1;
    const bool hasher = tid < T * kIdsPerTok;
    const int t = hasher ? tid / kIdsPerTok : 0, hh = hasher ? tid - t * kIdsPerTok : 0;
    const int b = t / a.q, i = t - b * a.q;
    int32_t tok = 0, p1 = -1, p2 = -1;                       // the token, then the one or two before it
    if (hasher) {
      tok = a.tokens[t];
      p1 = i >= 1 ? a.tokens[t - 1] : a.hist[2 * b + 1];
      p2 = i >= 2 ? a.tokens[t - 2] : (i == 1 ? a.hist[2 * b + 1] : a.hist[2 * b]);
    }
    if (hasher) {
      if (blockIdx.x == 0 && hh == 0 && (tok < 0 || tok >= a.vocab)) set_status(a.status, PLE_ERR_RANGE);
      // inside the sequence every context is a token (+1); before it, a carried entry < 0 is absent
      const uint64_t x0 = ctx_of(tok);
      const uint64_t x1 = (i >= 1 || p1 >= 0) ? ctx_of(p1) : 0ull;
      const uint64_t x2 = (i >= 2 || p2 >= 0) ? ctx_of(p2) : 0ull;
      const uint64_t k2 = (x0 * kQ0) ^ (x1 * kQ1);
      const uint64_t k3 = k2 ^ (x2 * kQ2);
      if constexpr (FMT == 2) {
        const uint64_t k = ((hh >> 3) ? k3 : k2) ^ (static_cast<uint64_t>(hh & 7) * kHeadMix);
        sm->rid16[t][hh] = static_cast<int32_t>(mod_barrett(k ^ (k >> 32), a.rows0, a.magic0));
      } else {
        const int64_t r0 = static_cast<int64_t>(mod_barrett(k2 ^ (k2 >> 32), a.rows0, a.magic0));
        const int64_t r1 = a.rows0 + static_cast<int64_t>(mod_barrett(k3 ^ (k3 >> 32), a.rows1, a.magic1));
        sm->rid[t][0] = r0;
        sm->rid[t][1] = r1;
        if constexpr (TWO) {
          s_two[0] = __ldg(a.scales + r0);
          s_two[1] = __ldg(a.scales + r1);
        }
      }
    }
    gates();                                                 // under the hash's loads
    __syncthreads();                                         // row IDs ready: this CTA has read the history
    // count this CTA in; the last CTA to arrive writes the new history at the end,
    // when no CTA of the grid can still read the old one (the ticket is used only then)
    if (tid == 0) ticket = atomicAdd(a.step_count, 1);
  }
  if constexpr (MODE == kRowsHash2) {
    // this warp's K range (chunks of 16 codes, lane l takes chunk kb + l) of A
    // rows r = 0..15: token r & 7, order r >> 3; all 16 rows' loads in flight
    // before any is used (from a cold L2 the gather is one HBM round trip)
    const int nck = ke - kb;
    RowChunk<FMT == 1> x[kPjMaxTok];
#pragma unroll
    for (int rr = 0; rr < kPjMaxTok; ++rr) {
      const int t = rr & 7;
      if (t < T && lane < nck) x[rr] = load_chunk<FMT == 1>(a.table, a.blocks, sm->rid[t][rr >> 3], a.cs, a.bs, kb + lane);
    }
#pragma unroll
    for (int rr = 0; rr < kPjMaxTok; ++rr) {
      const int t = rr & 7;
      if (t < T && lane < nck) {
        uint4 o0, o1;
        codes_to_f16<FMT == 1>(x[rr], o0, o1);
        uint4* dst = reinterpret_cast<uint4*>(es + rr * ldr + (kb + lane) * 16);
        dst[0] = o0;
        dst[1] = o1;
      }
    }
    if (tid < T) {
      sm->sc[tid][0] = s_two[0];
      sm->sc[tid][1] = s_two[1];
    }
  } else if constexpr (FUSED) {
    // this warp's K range (chunks of 16 codes) of every token's rows, dequantised
    // into e rows in shared memory: lane l takes tasks l, l + 32, ... of
    // (token, chunk), all of a batch's loads in flight before any is used
    constexpr int kBatch = 5;
    const int nck = ke - kb;
    const int tasks = T * nck;
    for (int x0 = 0; x0 < tasks; x0 += 32 * kBatch) {
      RowChunk<FMT == 1> ra[kBatch], rb[kBatch];
      float sa[kBatch], sb[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        const int x = x0 + lane + 32 * r;
        if (x < tasks) {
          const int t = x / nck, j = kb + (x - t * nck);
          if constexpr (FMT == 2) {
            const int hd = a.D / kHeads, cph = hd / 16, hh = j / cph;
            const int64_t row = static_cast<int64_t>(hh) * a.rows0 + sm->rid16[t][hh];
            ra[r].c = ld_stream_v4(a.table + row * hd + (j - hh * cph) * 16);
            sa[r] = __ldg(a.scales + row);
          } else {
            const int64_t r0 = sm->rid[t][0], r1 = sm->rid[t][1];
            ra[r] = load_chunk<FMT == 1>(a.table, a.blocks, r0, a.cs, a.bs, j);
            rb[r] = load_chunk<FMT == 1>(a.table, a.blocks, r1, a.cs, a.bs, j);
            sa[r] = __ldg(a.scales + r0);
            sb[r] = __ldg(a.scales + r1);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kBatch; ++r) {
        const int x = x0 + lane + 32 * r;
        if (x < tasks) {
          const int t = x / nck, j = kb + (x - t * nck);
          uint4 o0, o1;
          if constexpr (FMT == 2) deq16_one(ra[r].c, sa[r], o0, o1);
          else deq_chunk<FMT == 1>(ra[r], rb[r], sa[r], sb[r], o0, o1);
          uint4* dst = reinterpret_cast<uint4*>(es + t * ldr + j * 16);
          dst[0] = o0;
          dst[1] = o1;
        }
      }
    }
  }
  if constexpr (COPIED) gates();
  cp_async_wait_all();
  __syncthreads();                                           // every copy and every e row has landed
  if (a.gate_ready && tid < T) sm->g[tid] = sm->meta[tid].g;

  // W_proj has landed (bounded: past the limit the status records a timeout and
  // the products are skipped)
  const bool w_ok = mbar_wait(wbar, 0);
  if (!w_ok && tid == 0) set_status(a.status, PLE_ERR_TIMEOUT);

  // ---- 3. products over this warp's K range: tokens (A, rows of e) x channels
  //         (B, rows of W_proj), one accumulator per 8-channel group
  float acc[kPjMaxGroups][4];
#pragma unroll
  for (int g = 0; g < kPjMaxGroups; ++g) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0.f;
  if (w_ok) {
    // ldmatrix.x4 for A: matrix m = lane / 8 covers token rows (m & 1) * 8 + 0..7 and
    // K offset (m >> 1) * 8; rows past T repeat the last token (their sums are unused)
    const int am = lane >> 3;
    const int lrow = (lane & 7) + ((am & 1) << 3);
    const int arow = TWO ? (min(lrow & 7, T - 1) | (lrow & 8)) : min(lrow, T - 1);
    const uint32_t a_addr = smem_u32(es + arow * ldr + kb * 16 + ((am >> 1) << 3));
    // ldmatrix.x2 for B: lanes 0..15 address channel rows 0..7 at K offsets 0 and 8
    const uint32_t b_addr = smem_u32(ws + (lane & 7) * ldr + kb * 16 + (((lane >> 3) & 1) << 3));
    const uint32_t group_bytes = kPjGroup * ldr * 2;
#pragma unroll 4
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
  if (lane < nch) {
    const int c = lane, g = c >> 3, cc = c & 7;
    const int ch = c0 + c;
    for (int b = warp; b < a.B; b += kPjWarps) {
      int32_t ncb = a.n_commit ? sm->nc[b] : a.q;
      if (ncb < 1 || ncb > a.q) {
        if (c == 0 && blockIdx.x == 0) set_status(a.status, PLE_ERR_RANGE);
        ncb = max(1, min(ncb, a.q));
      }
      float w0 = sm->cst[b][0][c], w1 = sm->cst[b][1][c], w2 = sm->cst[b][2][c];
      float k0 = w0, k1 = w1, k2 = w2;
      for (int i = 0; i < a.q; ++i) {
        const int t = b * a.q + i;
        float v = 0.f;
        if constexpr (TWO) {
          float v0 = 0.f, v1 = 0.f;
#pragma unroll
          for (int w = 0; w < kPjWarps; ++w) {
            v0 += sm->red[w][g][t][cc];
            v1 += sm->red[w][g][t + 8][cc];
          }
          v = sm->sc[t][0] * v0 + sm->sc[t][1] * v1;
        } else {
#pragma unroll
          for (int w = 0; w < kPjWarps; ++w) v += sm->red[w][g][t][cc];
        }
        const float u = sm->g[t] * v;
        const float y = cw.x * w0 + cw.y * w1 + cw.z * w2 + cw.w * u;
        w0 = w1;
        w1 = w2;
        w2 = u;
        const int64_t idx = static_cast<int64_t>(t) * a.H + ch;
        const float o = __bfloat162float(sm->res[t][c]) + y;
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
  }
  // ---- 5. the new token history: the last two committed tokens, written by one
  //         thread once every reader of the old one is done with it (fused: the
  //         last CTA past its hashing; otherwise the embed kernel read it)
  if (tid == 0 && (FUSED ? ticket == static_cast<int32_t>(gridDim.x) - 1 : blockIdx.x == 0)) {
    for (int b = 0; b < a.B; ++b) {
      const int32_t ncb = max(1, min(a.n_commit ? sm->nc[b] : a.q, a.q));
      const int32_t n1 = sm->tok[b * a.q + ncb - 1];
      const int32_t n0 = ncb >= 2 ? sm->tok[b * a.q + ncb - 2] : sm->hist[b][1];
      a.hist[2 * b] = n0;
      a.hist[2 * b + 1] = n1;
    }
    if (FUSED) *a.step_count = 0;                            // ready for the next step
  }
  if (!w_ok) mbar_wait(wbar, 0);                             // copies in flight land before the CTA leaves
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
  static PerDeviceOnce configured;
  const cudaError_t r = configured.run([] {
    cudaError_t x = prefer_max_shared(decode_embed_kernel<0>);
    if (x == cudaSuccess) x = prefer_max_shared(decode_embed_kernel<1>);
    if (x == cudaSuccess) x = prefer_max_shared(decode_embed_kernel<2>);
    return x;
  });
  if (r != cudaSuccess) return r;
  const int T = a.B * a.q;
  const int nch = a.D / 16;
  const int threads = std::min(kEmbedThreads, std::max(32, (nch + 31) / 32 * 32));
  const dim3 grid(a.w16 != nullptr ? std::max(T, a.prefetch_blocks) : T), block(threads);
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

bool decode_two_order(int32_t T, int32_t format) {
  return T <= kTwoOrderMaxTok && (format == PLE_TABLE_E4M3 || format == PLE_TABLE_NVFP4);
}

cudaError_t launch_decode_proj(const DecodeProjArgs& a, const DecodeProjPlan& plan, cudaStream_t stream) {
  static PerDeviceOnce configured;
  const cudaError_t e = configured.run([] {
    cudaError_t x = cudaSuccess;
    auto set = [&x](auto kernel) {
      if (x == cudaSuccess)
        x = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
      if (x == cudaSuccess) x = prefer_max_shared(kernel);
    };
    set(decode_proj_kernel<0, kRowsE>);
    set(decode_proj_kernel<0, kRowsHash>);
    set(decode_proj_kernel<1, kRowsHash>);
    set(decode_proj_kernel<2, kRowsHash>);
    set(decode_proj_kernel<0, kRowsHash2>);
    set(decode_proj_kernel<1, kRowsHash2>);
    set(decode_proj_kernel<0, kRowsCodes2>);
    return x;
  });
  if (e != cudaSuccess) return e;
  DecodeProjArgs b = a;
  b.max_groups = plan.max_groups;
  const int T = a.B * a.q;
  const bool two = decode_two_order(T, a.format);
  const size_t smem = proj_smem_bytes(plan.max_groups, a.D, two ? kPjMaxTok : T);
  const dim3 grid(plan.grid), block(kPjThreads);
  const bool nv = a.format == PLE_TABLE_NVFP4;
  if (a.e != nullptr) {                                      // rows or codes from decode_embed_kernel
    if (!two) return launch_pdl(decode_proj_kernel<0, kRowsE>, grid, block, smem, b, stream);
    return launch_pdl(decode_proj_kernel<0, kRowsCodes2>, grid, block, smem, b, stream);
  }
  if (two) {
    if (nv) return launch_pdl(decode_proj_kernel<1, kRowsHash2>, grid, block, smem, b, stream);
    return launch_pdl(decode_proj_kernel<0, kRowsHash2>, grid, block, smem, b, stream);
  }
  if (a.format == PLE_TABLE_E4M3_HEADS) return launch_pdl(decode_proj_kernel<2, kRowsHash>, grid, block, smem, b, stream);
  if (nv) return launch_pdl(decode_proj_kernel<1, kRowsHash>, grid, block, smem, b, stream);
  return launch_pdl(decode_proj_kernel<0, kRowsHash>, grid, block, smem, b, stream);
}

}  // namespace ple
