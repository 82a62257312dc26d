// One decode / speculative-verify step for small batches (B * q <= 16 tokens)
// in a single kernel: n-gram row IDs, gate, row gather and dequantisation,
// projection, conv against the carried state, residual and state commit.
//
// Decode is latency-bound: new n-grams depend on the token just produced
// (DGX Spark report, "推理流程": each decode step depends on the token just
// generated). The work per step is tiny (8 tokens: 41 KB of rows, 105 MFLOP)
// next to the 13.1 MB of W_proj that every step streams, so the step is one
// kernel with no intermediate tensors, one CTA per SM:
//   - the projection [H x D] is cut into units of 16 channels x 64 K-values
//     (2 KB of fp16 W_proj, one TMA box); the CTAs take equal, contiguous runs
//     of the units in channel-major order, so every SM streams the same share
//     of W_proj and a run covers at most three 16-channel tiles;
//   - the W_proj units are requested first, before the kernel waits for the
//     previous kernel in the stream (programmatic dependent launch), so that
//     this fetch overlaps the previous step's tail;
//   - every CTA computes the T row-ID pairs and gates and gathers and
//     dequantises the T row pairs into shared memory (the same rounding to fp16
//     as the prefill path), all warps sharing the loads; for the multi-head
//     layout, 16 head rows per token (a thread per token and head hashes),
//     dequantised row by row and laid side by side;
//   - the 16 x T x 64 products of a unit run on the tensor cores with mma.sync
//     m16n8k16 (fp16 inputs, fp32 accumulation), the W_proj operand read with
//     ldmatrix from the 128-byte-swizzled TMA tiles;
//   - a CTA writes its sum for each tile it touches into a fixed slot; the CTA
//     that completes a tile (a per-tile unit counter) adds the slots in slot
//     order, so the result does not depend on arrival order, and runs the conv,
//     the residual and the state commit for the tile's 16 channels;
//   - the CTA that completes the last tile writes the new token history, since
//     every CTA reads the old one before it contributes to any tile.
// Every CTA reads whole rows of hidden for the gates, so out must not alias
// hidden here (an in-place step takes the multi-kernel path).
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

constexpr int kChan = 16;                       // channels per tile (the mma's M)
constexpr int kMaxTok = 16;                     // tokens per step (two mma N-blocks of 8)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kUnitK = 64;                      // K-values per unit: one 128-byte swizzle row
constexpr int kUnitBytes = kChan * kUnitK * 2;  // 2 KB
constexpr int kMaxUnits = 64;                   // units per CTA
constexpr int kMaxLocalTiles = 3;
constexpr int kSmemLimit = 227 * 1024;

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

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}


// Unit partition: CTA b of G owns units [u0(b), u0(b + 1)) with u0(b) = b * U / G;
// the owner of unit u is the largest b with u0(b) <= u. 32-bit: the host
// checks that (U + 1) * G fits.
__host__ __device__ __forceinline__ int32_t unit_begin(int32_t b, int32_t U, int32_t G) { return b * U / G; }
__host__ __device__ __forceinline__ int32_t unit_owner(int32_t u, int32_t U, int32_t G) {
  return ((u + 1) * G - 1) / U;
}

struct __align__(16) DecodeSmem {
  float red[kMaxLocalTiles][kWarps][kChan][kMaxTok];   // per-warp tile sums
  float v[kMaxTok][kChan];                             // a finished tile's projection
  float res[kMaxTok][kChan];                           // and its residual (hidden)
  float gacc[kMaxTok];                                 // gate pre-activations
  int64_t rid[kMaxTok][2];                             // row IDs (into the stacked table)
  int32_t rid16[kMaxTok][kHeads];                      // multi-head layout: row of each head
  uint64_t bar[kMaxUnits];                             // one mbarrier per W_proj unit
  int32_t fin[kMaxLocalTiles];
  int32_t last;
};
static_assert(sizeof(DecodeSmem) % 16 == 0, "the e rows follow the struct at a 16-byte offset");

// Dynamic shared memory, from a 1024-byte aligned base: W_proj units
// [units][16][128 B] (TMA 128-byte swizzle), DecodeSmem, e [16][D + 8] fp16,
// w_gate [H] bf16.
size_t smem_bytes(int units, int32_t D, int32_t H) {
  return 1024 + static_cast<size_t>(units) * kUnitBytes + sizeof(DecodeSmem) +
         static_cast<size_t>(kMaxTok) * (D + 8) * sizeof(__half) + static_cast<size_t>(H) * sizeof(__nv_bfloat16);
}

// FMT: 0 = E4M3 rows (two orders), 1 = NVFP4 rows, 2 = the multi-head E4M3 layout.
template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_small_kernel(const __grid_constant__ CUtensorMap tmap_w, const DecodeSmallArgs a) {
  constexpr bool NV = FMT == 1;
  constexpr bool HEADS = FMT == 2;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const uint32_t wt_s = smem_u32(base);
  DecodeSmem* sm = reinterpret_cast<DecodeSmem*>(base + a.units_max * kUnitBytes);
  const int ldE = a.D + 8;                                  // padded row: conflict-free B loads
  __half* e16 = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(sm) + sizeof(DecodeSmem));
  __nv_bfloat16* wg_s = reinterpret_cast<__nv_bfloat16*>(e16 + kMaxTok * ldE);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int T = a.B * a.q;
  const int KC = a.D / kUnitK;
  const int ntiles = a.H / kChan;
  const int U = ntiles * KC;
  const int G = gridDim.x;
  const int u0 = unit_begin(blockIdx.x, U, G), u1 = unit_begin(blockIdx.x + 1, U, G);
  const int nunits = u1 - u0;                               // >= 1 (host plan)
  const int ct_first = u0 / KC;
  const int n_local = (u1 - 1) / KC - ct_first + 1;
  const int c = threadIdx.x & (kChan - 1), tk = threadIdx.x >> 4;   // 256 threads = 16 tokens x 16 channels

  // ---- 1. before the wait: request this CTA's W_proj units (warp 0, a unit per
  //         lane), stage w_gate, load the conv taps of this CTA's tiles
  if (warp == 0) {
    for (int i = lane; i < nunits; i += 32) mbar_init(smem_u32(&sm->bar[i]), 1);
    fence_barrier_init();
    __syncwarp();
    if (lane == 0) tma_prefetch_desc(&tmap_w);
    for (int i = lane; i < nunits; i += 32) {
      const int u = u0 + i;
      const int ct = u / KC;
      const uint32_t bar = smem_u32(&sm->bar[i]);
      mbar_arrive_expect_tx(bar, kUnitBytes);
      tma_load_2d(wt_s + i * kUnitBytes, &tmap_w, (u - ct * KC) * kUnitK, ct * kChan, bar);
    }
  }
  for (int j = threadIdx.x; j < a.H / 8; j += kThreads)
    reinterpret_cast<uint4*>(wg_s)[j] = __ldg(reinterpret_cast<const uint4*>(a.w_gate) + j);
  if (threadIdx.x < kMaxTok) sm->gacc[threadIdx.x] = 0.f;
  if (threadIdx.x == 0) sm->last = 0;
  const bool conv_thread = threadIdx.x < a.B * kChan;       // (sequence tk, channel c)
  float4 cw[kMaxLocalTiles];
#pragma unroll
  for (int cl = 0; cl < kMaxLocalTiles; ++cl)
    if (conv_thread && cl < n_local) cw[cl] = __ldg(reinterpret_cast<const float4*>(a.conv_w) + (ct_first + cl) * kChan + c);
  __syncthreads();                                          // w_gate staged, gate sums zeroed
  pdl_launch_dependents();
  // tokens, hidden and the state may come from the previous kernel in the stream
  pdl_wait();

  // ---- 2. loads the epilogue needs, then row IDs (a thread per token), gates and rows (all warps)
  float cst[kMaxLocalTiles][3];                             // conv state of (sequence tk, channel c)
  float res[kMaxLocalTiles];                                // hidden of (token tk, channel c)
#pragma unroll
  for (int cl = 0; cl < kMaxLocalTiles; ++cl) {
    if (cl < n_local) {
      const int ch = (ct_first + cl) * kChan + c;
      if (conv_thread) {
        const float* cs = a.conv_state + static_cast<int64_t>(tk) * 3 * a.H + ch;
        cst[cl][0] = cs[0];
        cst[cl][1] = cs[a.H];
        cst[cl][2] = cs[2 * a.H];
      }
      if (tk < T) res[cl] = __bfloat162float(a.hidden[static_cast<int64_t>(tk) * a.H + ch]);
    }
  }
  int32_t nc = a.q;
  if (conv_thread && a.n_commit) nc = a.n_commit[tk];
  const int hv8 = a.H / 8;                                  // uint4 per hidden row
  const int nsg = (hv8 + 31) / 32;                          // 32-lane segments per hidden row
  const int dv16 = a.D / 16;                                // uint4 per table row
  const int nsr = (dv16 + 31) / 32;                         // 32-lane segments per table row
  constexpr int kGateBatch = 10;                            // hidden segments in flight per lane
  constexpr int kRowBatch = 10;                             // row segments in flight per lane
  // gate: warp w takes a contiguous run of the T * nsg hidden segments, so that
  // it reduces across lanes once per token it touches
  const int gtot = T * nsg, gpw = (gtot + kWarps - 1) / kWarps;
  const int gs0 = min(gtot, warp * gpw), gs1 = min(gtot, gs0 + gpw);
  auto gate_load = [&](uint4 (&hv)[kGateBatch], int first) {
#pragma unroll
    for (int r = 0; r < kGateBatch; ++r) {
      const int s = gs0 + first + r;
      const int t = s / nsg, j = (s - t * nsg) * 32 + lane;
      if (s < gs1 && j < hv8) hv[r] = __ldg(reinterpret_cast<const uint4*>(a.hidden + static_cast<int64_t>(t) * a.H) + j);
    }
  };
  auto gate_flush = [&](float acc, int t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicAdd(&sm->gacc[t], acc);
  };
  auto gate_use = [&](const uint4 (&hv)[kGateBatch], int first) {
    float acc = 0.f;
    int tcur = -1;
#pragma unroll
    for (int r = 0; r < kGateBatch; ++r) {
      const int s = gs0 + first + r;
      if (s >= gs1) break;                                  // warp-uniform
      const int t = s / nsg, j = (s - t * nsg) * 32 + lane;
      if (t != tcur) {
        if (tcur >= 0) gate_flush(acc, tcur);
        acc = 0.f;
        tcur = t;
      }
      if (j < hv8) {
        const uint4 wq = reinterpret_cast<const uint4*>(wg_s)[j];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hv[r]);
        const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&wq);
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          const float2 hf = __bfloat1622float2(h2[qq]);
          const float2 wf = __bfloat1622float2(w2[qq]);
          acc = fmaf(hf.x, wf.x, acc);
          acc = fmaf(hf.y, wf.y, acc);
        }
      }
    }
    if (tcur >= 0) gate_flush(acc, tcur);
  };
  {
    uint4 hv[kGateBatch];
    gate_load(hv, 0);
    if (threadIdx.x < (HEADS ? T * kHeads : T)) {
      const int t = HEADS ? threadIdx.x / kHeads : threadIdx.x;
      const int hh = HEADS ? threadIdx.x % kHeads : 0;
      const int b = t / a.q, i = t - b * a.q;
      const int32_t tok = a.tokens[t];
      if (blockIdx.x == 0 && hh == 0 && (tok < 0 || tok >= a.vocab)) set_status(a.status, PLE_ERR_RANGE);
      const int32_t h0 = a.hist[2 * b], h1 = a.hist[2 * b + 1];
      auto carried = [](int32_t h) -> uint64_t { return h < 0 ? 0ull : ctx_of(h); };
      const uint64_t x0 = ctx_of(tok);
      const uint64_t x1 = i >= 1 ? ctx_of(a.tokens[t - 1]) : carried(h1);
      const uint64_t x2 = i >= 2 ? ctx_of(a.tokens[t - 2]) : (i == 1 ? carried(h1) : carried(h0));
      const uint64_t k2 = (x0 * kQ0) ^ (x1 * kQ1);
      const uint64_t k3 = k2 ^ (x2 * kQ2);
      if constexpr (HEADS) {
        // head hh of order hh / 8 reads sub-table hh: fold(k_n ^ (hh % 8) * kHeadMix) mod rows
        const uint64_t k = ((hh >> 3) ? k3 : k2) ^ (static_cast<uint64_t>(hh & 7) * kHeadMix);
        sm->rid16[t][hh] = static_cast<int32_t>(mod_barrett(k ^ (k >> 32), a.rows0, a.magic0));
      } else {
        const int64_t r0 = static_cast<int64_t>(mod_barrett(k2 ^ (k2 >> 32), a.rows0, a.magic0));
        const int64_t r1 = a.rows0 + static_cast<int64_t>(mod_barrett(k3 ^ (k3 >> 32), a.rows1, a.magic1));
        sm->rid[t][0] = r0;
        sm->rid[t][1] = r1;
      }
    }
    gate_use(hv, 0);
  }
  __syncthreads();                                          // row IDs ready
  const int row_segs = (T * nsr + kWarps - 1) / kWarps;     // per warp
  if constexpr (HEADS) {
    // chunk j of a token (16 codes) comes from head row j / (chunks per head)
    const int hd = a.D / kHeads, cph = hd / 16;
    for (int first = 0; first < row_segs; first += kRowBatch) {
      uint4 xh[kRowBatch];
      float sh[kRowBatch];
#pragma unroll
      for (int r = 0; r < kRowBatch; ++r) {
        const int s = warp + kWarps * (first + r);
        const int t = s / nsr, j = (s - t * nsr) * 32 + lane;
        if (t < T && j < dv16) {
          const int h = j / cph;
          const int64_t row = static_cast<int64_t>(h) * a.rows0 + sm->rid16[t][h];
          xh[r] = ld_stream_v4(a.table + row * hd + (j - h * cph) * 16);
          sh[r] = __ldg(a.scales + row);
        }
      }
#pragma unroll
      for (int r = 0; r < kRowBatch; ++r) {
        const int s = warp + kWarps * (first + r);
        const int t = s / nsr, j = (s - t * nsr) * 32 + lane;
        if (t < T && j < dv16) {
          uint4 lo, hi;
          deq16_one(xh[r], sh[r], lo, hi);
          uint4* dst = reinterpret_cast<uint4*>(e16 + t * ldE + 16 * j);
          dst[0] = lo;
          dst[1] = hi;
        }
      }
    }
  }
  for (int first = 0; first < (HEADS ? 0 : row_segs); first += kRowBatch) {
    RowChunk<NV> xa[kRowBatch], xb[kRowBatch];
    float sa[kRowBatch], sb[kRowBatch];
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      const int s = warp + kWarps * (first + r);
      const int t = s / nsr, j = (s - t * nsr) * 32 + lane;
      if (t < T && j < dv16) {
        const int64_t ra = sm->rid[t][0], rb = sm->rid[t][1];
        xa[r] = load_chunk<NV>(a.table, a.blocks, ra, a.D, j);
        xb[r] = load_chunk<NV>(a.table, a.blocks, rb, a.D, j);
        sa[r] = __ldg(a.scales + ra);
        sb[r] = __ldg(a.scales + rb);
      }
    }
#pragma unroll
    for (int r = 0; r < kRowBatch; ++r) {
      const int s = warp + kWarps * (first + r);
      const int t = s / nsr, j = (s - t * nsr) * 32 + lane;
      if (t < T && j < dv16) {
        uint4 lo, hi;
        deq_chunk<NV>(xa[r], xb[r], sa[r], sb[r], lo, hi);
        uint4* dst = reinterpret_cast<uint4*>(e16 + t * ldE + 16 * j);
        dst[0] = lo;
        dst[1] = hi;
      }
    }
  }
  for (int first = kGateBatch; first < gs1 - gs0; first += kGateBatch) {
    uint4 hv[kGateBatch];
    gate_load(hv, first);
    gate_use(hv, first);
  }
  __syncthreads();                                          // e and the gate sums complete

  // ---- 3. projection: per local tile, this warp's units (local index warp, warp + 8, ...)
  const int gq = lane >> 2, tq = lane & 3;
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);      // ldmatrix row of this lane's address
  const int lchunk = lane >> 4;                             // and its 16-byte chunk within a k-step
  for (int cl = 0; cl < n_local; ++cl) {
    const int ct = ct_first + cl;
    const int ib = max(u0, ct * KC) - u0, ie = min(u1, (ct + 1) * KC) - u0;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    // local unit indices i in [ib, ie) with i % 8 == warp
    for (int i = ib + ((warp - ib) % kWarps + kWarps) % kWarps; i < ie; i += kWarps) {
      if (!mbar_wait(smem_u32(&sm->bar[i]), 0)) {
        if (lane == 0) set_status(a.status, PLE_ERR_TIMEOUT);
        break;
      }
      const int k0 = (u0 + i - ct * KC) * kUnitK;
      const uint32_t tile = wt_s + i * kUnitBytes + lrow * 128;
#pragma unroll
      for (int ks = 0; ks < kUnitK / 16; ++ks) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(tile + (((2 * ks + lchunk) ^ (lrow & 7)) << 4), a0, a1, a2, a3);
        const int k = k0 + ks * 16 + 2 * tq;
        const uint32_t* e0 = reinterpret_cast<const uint32_t*>(e16 + gq * ldE + k);
        if (T > 8) {
          const uint32_t* e1 = reinterpret_cast<const uint32_t*>(e16 + (gq + 8) * ldE + k);
          mma_16816(d0, a0, a1, a2, a3, e0[0], e0[4]);
          mma_16816(d1, a0, a1, a2, a3, e1[0], e1[4]);
        } else if (ks & 1) {                                // one N-block: two accumulation chains
          mma_16816(d1, a0, a1, a2, a3, e0[0], e0[4]);
        } else {
          mma_16816(d0, a0, a1, a2, a3, e0[0], e0[4]);
        }
      }
    }
    if (T <= 8) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        d0[q] += d1[q];
        d1[q] = 0.f;
      }
    }
    // C layout: (channel gq, tokens 2tq, 2tq+1) and (channel gq + 8, same tokens)
    float (&rw)[kChan][kMaxTok] = sm->red[cl][warp];
    rw[gq][2 * tq] = d0[0];
    rw[gq][2 * tq + 1] = d0[1];
    rw[gq + 8][2 * tq] = d0[2];
    rw[gq + 8][2 * tq + 1] = d0[3];
    rw[gq][8 + 2 * tq] = d1[0];
    rw[gq][8 + 2 * tq + 1] = d1[1];
    rw[gq + 8][8 + 2 * tq] = d1[2];
    rw[gq + 8][8 + 2 * tq + 1] = d1[3];
  }
  __syncthreads();

  // ---- 4. this CTA's tile sums into their slots; count the units in. The tile
  //         that completes the last tile also knows that every CTA has read the
  //         old token history (each reads it before it counts any unit).
  for (int cl = 0; cl < n_local; ++cl) {
    const int ct = ct_first + cl;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += sm->red[cl][w][c][tk];
    const int slot = blockIdx.x - unit_owner(ct * KC, U, G);
    a.partial[(static_cast<int64_t>(ct) * a.slots + slot) * (kChan * kMaxTok) + tk * kChan + c] = v;
  }
  __syncthreads();
  if (threadIdx.x < n_local) {                              // one thread per local tile
    const int cl = threadIdx.x;
    const int ct = ct_first + cl;
    const int mine = min(u1, (ct + 1) * KC) - max(u0, ct * KC);
    __threadfence();                                        // the CTA's slot writes before the count
    const int32_t fin = atomicAdd(a.tile_count + ct, mine) + mine == KC;
    sm->fin[cl] = fin;
    if (fin) {
      __threadfence();                                      // every slot of the tile before its reads
      a.tile_count[ct] = 0;                                 // ready for the next step
      if (atomicAdd(a.tiles_done, 1) == ntiles - 1) {
        *a.tiles_done = 0;
        sm->last = 1;
      }
    }
  }
  __syncthreads();
  if (sm->last && threadIdx.x < a.B) {                      // new token history
    const int b = threadIdx.x;
    const int32_t ncb = max(1, min(a.n_commit ? a.n_commit[b] : a.q, a.q));
    const int32_t* tkp = a.tokens + static_cast<int64_t>(b) * a.q;
    const int32_t n1 = tkp[ncb - 1];
    const int32_t n0 = ncb >= 2 ? tkp[ncb - 2] : a.hist[2 * b + 1];
    a.hist[2 * b] = n0;
    a.hist[2 * b + 1] = n1;
  }

  // ---- 5. tiles this CTA completed: slot sum, conv against the state, residual, commit
#pragma unroll
  for (int cl = 0; cl < kMaxLocalTiles; ++cl) {
    if (cl < n_local && sm->fin[cl]) {                      // block-uniform
      const int ct = ct_first + cl;
      const int s_first = unit_owner(ct * KC, U, G);
      const int n_slots = unit_owner((ct + 1) * KC - 1, U, G) - s_first + 1;
      const float* p = a.partial + static_cast<int64_t>(ct) * a.slots * (kChan * kMaxTok) + tk * kChan + c;
      float v = 0.f;
      for (int s = 0; s < n_slots; ++s) v += __ldcg(p + s * (kChan * kMaxTok));
      sm->v[tk][c] = v;
      if (tk < T) sm->res[tk][c] = res[cl];
      __syncthreads();
      if (conv_thread) {
        const int b = tk;
        const int ch = ct * kChan + c;
        int32_t ncb = nc;
        if (ncb < 1 || ncb > a.q) {
          if (c == 0 && ct == 0) set_status(a.status, PLE_ERR_RANGE);
          ncb = max(1, min(ncb, a.q));
        }
        float w0 = cst[cl][0], w1 = cst[cl][1], w2 = cst[cl][2];
        float k0 = w0, k1 = w1, k2 = w2;
        const float4 cwt = cw[cl];
        for (int i = 0; i < a.q; ++i) {
          const int t = b * a.q + i;
          const float g = 1.0f / (1.0f + expf(-sm->gacc[t]));
          const float u = g * sm->v[t][c];
          const float y = cwt.x * w0 + cwt.y * w1 + cwt.z * w2 + cwt.w * u;
          w0 = w1; w1 = w2; w2 = u;
          const int64_t idx = static_cast<int64_t>(t) * a.H + ch;
          const float o = sm->res[t][c] + y;
          if (a.out_f32) reinterpret_cast<float*>(a.out)[idx] = o;
          else reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(o);
          if (i == ncb - 1) { k0 = w0; k1 = w1; k2 = w2; }
        }
        float* cs = a.conv_state + static_cast<int64_t>(b) * 3 * a.H + ch;
        cs[0] = k0;
        cs[a.H] = k1;
        cs[2 * a.H] = k2;
      }
      __syncthreads();                                      // v and res are reused by the next tile
    }
  }
}

}  // namespace

bool decode_small_plan(int32_t H, int32_t D, int32_t num_sms, DecodePlan* plan) {
  if (H % kChan != 0 || D % kUnitK != 0 || num_sms < 1) return false;
  const int64_t KC = D / kUnitK;
  const int64_t U64 = static_cast<int64_t>(H / kChan) * KC;
  const int64_t G64 = std::min<int64_t>(num_sms, U64);
  if ((U64 + 1) * G64 >= (int64_t(1) << 31)) return false;       // 32-bit unit arithmetic in the kernel
  const int32_t U = static_cast<int32_t>(U64), G = static_cast<int32_t>(G64);
  int units_max = 0, slots = 0;
  for (int32_t b = 0; b < G; ++b) {
    const int32_t u0 = unit_begin(b, U, G), u1 = unit_begin(b + 1, U, G);
    if (u1 <= u0) return false;                                    // G <= U: every CTA owns a unit
    units_max = std::max<int>(units_max, u1 - u0);
    if ((u1 - 1) / KC - u0 / KC + 1 > kMaxLocalTiles) return false;
    if (unit_owner(u0, U, G) != b || unit_owner(u1 - 1, U, G) != b) return false;
  }
  for (int32_t ct = 0; ct < H / kChan; ++ct) {
    const int32_t first = static_cast<int32_t>(ct * KC), last = static_cast<int32_t>((ct + 1) * KC - 1);
    slots = std::max<int>(slots, unit_owner(last, U, G) - unit_owner(first, U, G) + 1);
  }
  if (units_max > kMaxUnits || smem_bytes(units_max, D, H) > static_cast<size_t>(kSmemLimit)) return false;
  plan->grid = G;
  plan->units_max = units_max;
  plan->slots = slots;
  return true;
}

bool decode_small_supported(int32_t B, int32_t q) { return B * q <= kMaxTok; }

int64_t decode_small_partial_elems(const DecodePlan& plan, int32_t H) {
  return static_cast<int64_t>(H / kChan) * plan.slots * kChan * kMaxTok;
}

uint64_t barrett_magic(int64_t m) { return ~0ull / static_cast<uint64_t>(m); }

cudaError_t launch_decode_small(const CUtensorMap& tmap_w, const DecodeSmallArgs& a, int32_t grid,
                                cudaStream_t stream) {
  static PerDeviceOnce configured;
  const cudaError_t e = configured.run([] {
    cudaError_t r = cudaFuncSetAttribute(decode_small_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemLimit);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(decode_small_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(decode_small_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    return r;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes(a.units_max, a.D, a.H);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.heads) return cudaLaunchKernelEx(&cfg, decode_small_kernel<2>, tmap_w, a);
  if (a.nvfp4) return cudaLaunchKernelEx(&cfg, decode_small_kernel<1>, tmap_w, a);
  return cudaLaunchKernelEx(&cfg, decode_small_kernel<0>, tmap_w, a);
}

}  // namespace ple
