// Decode and speculative-verify steps of 17 to 256 tokens (the MTP shape of the
// Thor T5000 report's launch flags and acceptance table: 64 sequences x 3
// tokens, 1 accepted + 2 drafts) after decode_embed_kernel: the projection on
// the tensor cores (tcgen05, accumulators in TMEM) split along K, with the
// split sums, gate, conv against the carried state, residual and state commit
// in the same kernel.
//
// Shape: 192 tokens x 2560 x 2560 is 2.5 GFLOP against 13.1 MB of W_proj and
// 1 MB of rows. Per SM the bound is operand traffic, so the grid is 20
// channel tiles (M = 128, operand A = fp16 W_proj, K-major) x 7 K-splits
// (operand B = the step's fp16 rows e, N = the step's tokens): 140 CTAs, one
// per SM, each with 94 KB of W_proj and 140 KB of e. Each operand arrives two
// K-blocks per TMA copy (3-D boxes of 32 KB and more, which the copy engine
// delivers faster per SM than single K-blocks). The first stages' W_proj
// copies are issued before the programmatic wait, under the embed kernel.
//
// The K-split CTAs of a channel tile write their fp32 sums to a scratch slab
// ([tile][split][token][128 channels], coalesced), count themselves in at the
// tile's counter and wait (bounded) until all have. Every CTA then takes an
// equal share of the step's sequences: for its tile's 128 channels it adds
// the splits' sums in split order (the same bits on every run), applies the
// gate from the embed kernel, runs the conv along the sequence's q tokens
// from the carried state, adds the residual and commits the state after
// n_commit[b] tokens. The last CTA of a tile to finish resets the tile's
// counters for the next step. The CTAs of a tile wait for one another, so the
// grid never exceeds the SM count (one CTA per SM by its shared memory); a CTA
// that still waits after about a second records PLE_ERR_TIMEOUT and leaves.
//
// Warp roles (320 threads): warp 0 issues the TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2-9 run the epilogue (two per TMEM lane quarter,
// each taking every other 32-token column block).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>

#include "ple_device.cuh"
#include "ple_internal.h"

namespace ple {
namespace {

constexpr int kMtM = 128;                 // channels per CTA (TMEM lanes)
constexpr int kMtBK = 64;                 // K per stage: one 128-byte swizzled row of fp16
constexpr int kMtUmmaK = 16;
constexpr int kMtThreads = 320;
constexpr int kMtTmaWarp = 0;
constexpr int kMtMmaWarp = 1;
constexpr int kMtEpiWarp0 = 2;
constexpr int kMtEpiThreads = 256;
constexpr int kMtStages = 5;              // most stages; fewer when 256 tokens do not leave room
constexpr uint32_t kMtAStage = kMtM * kMtBK * 2;   // 16 KB: W_proj of one K-block
constexpr int kMtKbs = 2;                 // K-blocks per stage: each operand arrives as one 3-D TMA box of two
constexpr uint32_t kMtTmemCols = 256;
constexpr int kMtSmemLimit = 226 * 1024;  // dynamic; the per-block maximum (227 KB) includes the static word

struct MtBars {
  uint64_t full[kMtStages];
  uint64_t empty[kMtStages];
  uint64_t tfull;
  uint64_t staged;          // the split sums of a chunk of sequences landed
  uint32_t tmem_base;
  int32_t abort_flag;
};

// Bytes of one stage: two K-blocks of W_proj (A) and of the step's rows (B,
// n_pad rows of 128 bytes per K-block).
size_t mtp_stage_bytes(int n_pad) {
  return static_cast<size_t>(kMtKbs) * (kMtAStage + static_cast<size_t>(n_pad) * kMtBK * 2);
}

// Dynamic shared memory from a 1024-byte aligned base: A stages, B stages, then
// the barriers.
size_t mtp_smem_bytes(int n_pad, int stages) {
  return 1024 + static_cast<size_t>(stages) * mtp_stage_bytes(n_pad) + sizeof(MtBars);
}

int mtp_stages(int n_pad) {
  int s = kMtStages;
  while (s > 2 && mtp_smem_bytes(n_pad, s) > static_cast<size_t>(kMtSmemLimit)) --s;
  return s;
}

__device__ __forceinline__ int32_t ld_acquire(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag, int32_t* status) {
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

__global__ void __launch_bounds__(kMtThreads, 1)
    mtp_proj_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_e,
                    const MtpProjArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array (an integer
  // round trip would hide the address space, and plain loads from it would be
  // generic ones)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int S = a.stages;
  const uint32_t b_kb = static_cast<uint32_t>(a.n_pad) * kMtBK * 2;   // B bytes of one K-block
  const uint32_t a_stage = kMtKbs * kMtAStage, b_stage = kMtKbs * b_kb;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + S * a_stage;
  MtBars* bars = reinterpret_cast<MtBars*>(smem + S * (a_stage + b_stage));
  volatile int32_t* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x % a.m_tiles, ks = blockIdx.x / a.m_tiles;
  const int kb0 = ks * a.num_kb / a.k_splits, kb1 = (ks + 1) * a.num_kb / a.k_splits;
  const int nkb = kb1 - kb0;
  const int nst = (nkb + kMtKbs - 1) / kMtKbs;             // stage loads (the last may hold one K-block)
  const int T = a.B * a.q;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->tfull), 1);
    mbar_init(smem_u32(&bars->staged), 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMtMmaWarp) {
    tmem_alloc(smem_u32(&bars->tmem_base), kMtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == kMtTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_e);
      // 3-D boxes {64, rows, 2 K-blocks}: a second K-block past the tensor is
      // zero-filled, one past this split's K range is loaded and not used
      const uint32_t tx = a_stage + b_stage;
      const int pre = min(nst, S);
      // W_proj of the first stages does not depend on the previous kernel
      for (int i = 0; i < pre; ++i) {
        const uint32_t fb = smem_u32(&bars->full[i]);
        mbar_arrive_expect_tx(fb, tx);
        tma_load_3d(sA + i * a_stage, &tmap_w, 0, m * kMtM, kb0 + kMtKbs * i, fb);
      }
      pdl_launch_dependents();
      pdl_wait();                                             // e comes from the embed kernel
      for (int i = 0; i < pre; ++i)
        tma_load_3d(sB + i * b_stage, &tmap_e, 0, 0, kb0 + kMtKbs * i, smem_u32(&bars->full[i]));
      int issued = pre;
      for (int i = pre; i < nst; ++i) {
        const int stage = i % S;
        const uint32_t round = static_cast<uint32_t>(i / S);
        if (!wait_bar(smem_u32(&bars->empty[stage]), (round - 1) & 1, abort_flag, a.status)) break;
        const uint32_t fb = smem_u32(&bars->full[stage]);
        mbar_arrive_expect_tx(fb, tx);
        tma_load_3d(sA + stage * a_stage, &tmap_w, 0, m * kMtM, kb0 + kMtKbs * i, fb);
        tma_load_3d(sB + stage * b_stage, &tmap_e, 0, 0, kb0 + kMtKbs * i, fb);
        issued = i + 1;
      }
      // copies in flight land before the CTA's shared memory is released
      for (int i = max(0, issued - S); i < issued; ++i) {
        const long long start = clock64();
        while (!mbar_try_wait(smem_u32(&bars->full[i % S]), static_cast<uint32_t>(i / S) & 1) &&
               clock64() - start < kWaitLimitCycles) {
        }
      }
    } else {
      pdl_launch_dependents();
    }
  } else if (warp == kMtMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    pdl_launch_dependents();
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(kMtM, a.n_pad);
      bool ok = true;
      for (int i = 0; i < nst; ++i) {
        const int stage = i % S;
        if (!wait_bar(smem_u32(&bars->full[stage]), static_cast<uint32_t>(i / S) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int hk = 0; hk < kMtKbs; ++hk) {
          if (kMtKbs * i + hk >= nkb) break;                  // the box's second K-block is past this split
          const uint64_t adesc = sdesc_k_sw128(sA + stage * a_stage + hk * kMtAStage);
          const uint64_t bdesc = sdesc_k_sw128(sB + stage * b_stage + hk * b_kb);
#pragma unroll
          for (int k = 0; k < kMtBK / kMtUmmaK; ++k)
            mma_f16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (i > 0 || hk > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(smem_u32(&bars->empty[stage]));
      }
      if (ok) mma_commit(smem_u32(&bars->tfull));
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-9)
    const int et = threadIdx.x - 32 * kMtEpiWarp0;          // 0..255
    const int quarter = warp & 3, half = (warp - kMtEpiWarp0) >> 2;
    const int row = quarter * 32 + lane;                     // TMEM lane: channel inside the tile
    // in the split sums: lane c4 of each warp takes channels 4 c4 .. 4 c4 + 3 of
    // the tile, warp ph (0..7) every 8th token or sequence from ph
    const int c4 = et & 31, ph = et >> 5;
    const float4 cw0 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + m * kMtM + 4 * c4);
    const float4 cw1 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + m * kMtM + 4 * c4 + 1);
    const float4 cw2 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + m * kMtM + 4 * c4 + 2);
    const float4 cw3 = __ldg(reinterpret_cast<const float4*>(a.conv_w) + m * kMtM + 4 * c4 + 3);
    pdl_launch_dependents();
    pdl_wait();                                              // gates, hidden and the state are ready
    // the new token history, while the products run (the embed kernel, the only
    // reader of the old one, has completed)
    if (blockIdx.x == 0) {
      for (int b = et; b < a.B; b += kMtEpiThreads) {
        const int32_t ncb = max(1, min(a.n_commit ? a.n_commit[b] : a.q, a.q));
        const int32_t* tkp = a.tokens + static_cast<int64_t>(b) * a.q;
        const int32_t n1 = tkp[ncb - 1];
        const int32_t n0 = ncb >= 2 ? tkp[ncb - 2] : a.hist[2 * b + 1];
        a.hist[2 * b] = n0;
        a.hist[2 * b + 1] = n1;
      }
    }
    float* slab = a.partial + static_cast<int64_t>(m) * a.k_splits * a.n_pad * kMtM;
    bool ok = wait_bar(smem_u32(&bars->tfull), 0, abort_flag, a.status);
    if (ok) {
      // this split's sums [T][128] into shared memory (the operand stages are
      // free: every MMA has completed), then to the slab in one bulk copy
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      float* St = reinterpret_cast<float*>(smem);
      for (int c = half; c * 32 < T; c += 2) {
        float v[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(c * 32), v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < T) St[(c * 32 + j) * kMtM + row] = v[j];
      }
      fence_proxy_async_smem();                              // the bulk copy reads these writes
    }
    tc_fence_before();
    ok = !named_bar_or(1, kMtEpiThreads, !ok);              // one decision for the whole epilogue
    // This CTA's share of the sequences, all 128 channels of the tile, runs in
    // chunks of whole sequences. Everything a chunk needs goes into shared memory
    // at once: the splits' sums by bulk copies (from the start of the staging
    // area), hidden at the tile's channels, the gates, the carried state and
    // n_commit by cp.async (the side arrays, at the end of the area), so a chunk
    // costs one round trip to L2. The first chunk's side arrays need no split
    // sums: they are loaded now, under the meet, when they clear this split's
    // sums on their way out.
    const int b0 = ks * a.B / a.k_splits, b1 = (ks + 1) * a.B / a.k_splits;
    const uint32_t region = static_cast<uint32_t>(S) * (a_stage + b_stage);
    const uint32_t per_seq = static_cast<uint32_t>(a.q) * (a.k_splits * 512u + 256u + 16u) + 3u * 512u + 32u;
    const int max_seqs = max(1, static_cast<int>(region / per_seq));
    auto side_bytes = [&](int ns) -> uint32_t {
      return (static_cast<uint32_t>(ns) * (a.q * 272u + 3u * 512u + 4u) + 15u) & ~15u;
    };
    // threads [first, first + n) of the epilogue issue the side loads
    auto load_side = [&](int bc, int ns, int first, int n) {
      const int nt = ns * a.q, t0 = bc * a.q;
      const int lt = et - first;
      if (lt < 0) return;
      uint8_t* Hs = smem + region - side_bytes(ns);               // [nt][128] bf16
      uint8_t* Ms = Hs + static_cast<size_t>(nt) * 256;          // [nt] TokMeta
      uint8_t* Cs = Ms + static_cast<size_t>(nt) * 16;           // [ns][3][128] f32
      uint8_t* Ns = Cs + static_cast<size_t>(ns) * 3 * 512;      // [ns] n_commit
      for (int x = lt; x < nt * 16; x += n) {
        const int tk = x >> 4, c16 = x & 15;
        cp_async_16(smem_u32(Hs + tk * 256 + c16 * 16), a.hidden + static_cast<int64_t>(t0 + tk) * a.H + m * kMtM + c16 * 8);
      }
      for (int x = lt; x < nt; x += n) cp_async_16(smem_u32(Ms + x * 16), a.meta + t0 + x);
      for (int x = lt; x < ns * 3 * 32; x += n) {
        const int r3 = x >> 5, c32 = x & 31;
        cp_async_16(smem_u32(Cs + r3 * 512 + c32 * 16),
                    a.conv_state + (static_cast<int64_t>(bc) * 3 + r3) * a.H + m * kMtM + c32 * 4);
      }
      if (a.n_commit != nullptr)
        for (int x = lt; x < ns; x += n) cp_async_4(smem_u32(Ns + x * 4), a.n_commit + bc + x);
      cp_async_commit();
    };
    const bool side_early = ok && b0 < b1 &&
                            region - side_bytes(min(max_seqs, b1 - b0)) >= static_cast<uint32_t>(T) * 512u;
    if (side_early) load_side(b0, min(max_seqs, b1 - b0), 32, kMtEpiThreads - 32);   // not warp 2: it counts in
    // ---- the tile's splits meet: count in, wait (bounded) for the others
    __shared__ int32_t go;
    if (et == 0) {
      if (ok) {
        bulk_store(slab + static_cast<int64_t>(ks) * a.n_pad * kMtM, smem_u32(smem), static_cast<uint32_t>(T) * 512u);
        bulk_commit_group();
        bulk_wait_group<0>();
        fence_proxy_async_global();                          // the copy's writes before the count
        __threadfence();
      }
      int32_t arrived = ok ? atomicAdd(a.tile_count + m, 1) + 1 : 0;
      const long long start = clock64();
      while (ok && arrived < a.k_splits) {
        if (clock64() - start > kWaitLimitCycles || *abort_flag) {
          set_status(a.status, PLE_ERR_TIMEOUT);
          ok = false;
          break;
        }
        arrived = ld_acquire(a.tile_count + m);
      }
      go = ok ? 1 : 0;
    }
    named_bar_sync(1, kMtEpiThreads);
    if (go) {
      const uint32_t staged_bar = smem_u32(&bars->staged);
      uint32_t chunk_parity = 0;
      for (int bc = b0; bc < b1 && go; bc += max_seqs) {
        const int ns = min(max_seqs, b1 - bc);
        const int nt = ns * a.q, t0 = bc * a.q;
        uint8_t* P = smem;                                           // [k_splits][nt][128] f32
        uint8_t* Hs = smem + region - side_bytes(ns);                // the side arrays, as load_side puts them
        uint8_t* Ms = Hs + static_cast<size_t>(nt) * 256;
        uint8_t* Cs = Ms + static_cast<size_t>(nt) * 16;
        uint8_t* Ns = Cs + static_cast<size_t>(ns) * 3 * 512;
        if (et < 32) {                                     // lane sp of warp 2 copies split sp
          if (et == 0) mbar_arrive_expect_tx(staged_bar, static_cast<uint32_t>(a.k_splits) * nt * 512u);
          __syncwarp();
          if (et < a.k_splits) {
            fence_proxy_async_global();                    // after the acquire: the others' sums
            bulk_load(smem_u32(P + static_cast<size_t>(et) * nt * 512),
                      slab + (static_cast<int64_t>(et) * a.n_pad + t0) * kMtM, static_cast<uint32_t>(nt) * 512u,
                      staged_bar);
          }
        }
        if (!(side_early && bc == b0)) load_side(bc, ns, 0, kMtEpiThreads);
        cp_async_wait_all();
        named_bar_sync(1, kMtEpiThreads);
        const bool landed = wait_bar(staged_bar, chunk_parity, abort_flag, a.status);
        if (named_bar_or(1, kMtEpiThreads, !landed)) break;  // every thread leaves, or none
        chunk_parity ^= 1;
        const float4* P4 = reinterpret_cast<const float4*>(P);      // [k_splits][nt][32] float4
        const uint2* H4 = reinterpret_cast<const uint2*>(Hs);       // [nt][32]: 4 bf16
        const TokMeta* Mm = reinterpret_cast<const TokMeta*>(Ms);
        const float4* C4 = reinterpret_cast<const float4*>(Cs);     // [ns][3][32]
        float4* U4 = reinterpret_cast<float4*>(P);                  // u into split 0's slots
        // With 128-bit accesses each thread runs 4 channels, and a batch of 4 of
        // its tokens keeps that many loads in flight; loads are unconditional (an
        // index past the chunk reads its last token again).
        // 1. the gated sums u: the splits' sums added in split order
        for (int tq = ph; tq < nt; tq += 4 * 8) {
          int tk[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) tk[j] = min(tq + 8 * j, nt - 1);
          float4 v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
          for (int sp = 0; sp < a.k_splits; ++sp) {
            const float4* ps = P4 + sp * nt * 32 + c4;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float4 x = ps[tk[j] * 32];
              v[j].x += x.x;
              v[j].y += x.y;
              v[j].z += x.z;
              v[j].w += x.w;
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float g = Mm[tk[j]].g;
            if (tq + 8 * j < nt) U4[tk[j] * 32 + c4] = make_float4(g * v[j].x, g * v[j].y, g * v[j].z, g * v[j].w);
          }
        }
        named_bar_sync(1, kMtEpiThreads);                  // every u of the chunk is in place
        // 2. the outputs: the conv reads the sequence's extended stream (three
        //    carried entries, then its tokens' u); token i taps entries i, i + 1,
        //    i + 2 and its own u
        auto ext = [&](int sb, int e) -> float4 {          // entry e of sequence sb's stream
          return e < 3 ? C4[(sb * 3 + e) * 32 + c4] : U4[(sb * a.q + e - 3) * 32 + c4];
        };
        for (int tq = ph; tq < nt; tq += 4 * 8) {
          float4 x0[4], x1[4], x2[4], xu[4];
          uint2 hv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int tc = min(tq + 8 * j, nt - 1);
            const int sb = tc / a.q, i = tc - sb * a.q;
            x0[j] = ext(sb, i);
            x1[j] = ext(sb, i + 1);
            x2[j] = ext(sb, i + 2);
            xu[j] = ext(sb, i + 3);
            hv[j] = H4[tc * 32 + c4];
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (tq + 8 * j < nt) {
              const float2 h01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hv[j].x));
              const float2 h23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hv[j].y));
              const float o0 = h01.x + (cw0.x * x0[j].x + cw0.y * x1[j].x + cw0.z * x2[j].x + cw0.w * xu[j].x);
              const float o1 = h01.y + (cw1.x * x0[j].y + cw1.y * x1[j].y + cw1.z * x2[j].y + cw1.w * xu[j].y);
              const float o2 = h23.x + (cw2.x * x0[j].z + cw2.y * x1[j].z + cw2.z * x2[j].z + cw2.w * xu[j].z);
              const float o3 = h23.y + (cw3.x * x0[j].w + cw3.y * x1[j].w + cw3.z * x2[j].w + cw3.w * xu[j].w);
              const int64_t idx = static_cast<int64_t>(t0 + tq + 8 * j) * a.H + m * kMtM + 4 * c4;
              if (a.out_f32) {
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + idx) = make_float4(o0, o1, o2, o3);
              } else {
                const __nv_bfloat162 b01 = __floats2bfloat162_rn(o0, o1), b23 = __floats2bfloat162_rn(o2, o3);
                uint2 w;
                w.x = *reinterpret_cast<const uint32_t*>(&b01);
                w.y = *reinterpret_cast<const uint32_t*>(&b23);
                *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + idx) = w;
              }
            }
          }
        }
        // 3. the carried state: the three entries of the extended stream that end
        //    at the sequence's last committed token
        for (int sq = ph; sq < ns; sq += 8) {
          int32_t ncb = a.n_commit ? reinterpret_cast<const int32_t*>(Ns)[sq] : a.q;
          if (ncb < 1 || ncb > a.q) {
            if (c4 == 0 && m == 0) set_status(a.status, PLE_ERR_RANGE);
            ncb = max(1, min(ncb, a.q));
          }
          const float4 k0 = ext(sq, ncb), k1 = ext(sq, ncb + 1), k2 = ext(sq, ncb + 2);
          float4* cs = reinterpret_cast<float4*>(a.conv_state + static_cast<int64_t>(bc + sq) * 3 * a.H + m * kMtM) + c4;
          cs[0] = k0;
          cs[a.H / 4] = k1;
          cs[2 * (a.H / 4)] = k2;
        }
        named_bar_sync(1, kMtEpiThreads);                  // the staging area is reused by the next chunk
      }
      named_bar_sync(1, kMtEpiThreads);
      // the last CTA of the tile to get here resets its counters for the next step
      if (et == 0 && atomicAdd(a.tile_done + m, 1) == a.k_splits - 1) {
        a.tile_count[m] = 0;
        a.tile_done[m] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMtMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMtTmemCols);
  }
}

}  // namespace

bool mtp_proj_plan(int32_t H, int32_t D, int32_t num_sms, MtpPlan* plan) {
  if (H % kMtM != 0 || D % kMtBK != 0 || num_sms < 1) return false;
  const int32_t m_tiles = H / kMtM, num_kb = D / kMtBK;
  if (m_tiles > num_sms) return false;
  const int32_t k_splits = std::max(1, std::min(std::min(num_kb, num_sms / m_tiles), kMtpMaxSplits));
  if (mtp_smem_bytes(kMtpMaxTokens, mtp_stages(kMtpMaxTokens)) > static_cast<size_t>(kMtSmemLimit)) return false;
  plan->m_tiles = m_tiles;
  plan->k_splits = k_splits;
  plan->num_kb = num_kb;
  return true;
}

int64_t mtp_partial_elems(const MtpPlan& plan) {
  return static_cast<int64_t>(plan.m_tiles) * plan.k_splits * kMtpMaxTokens * kMtM;
}

cudaError_t launch_mtp_proj(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const MtpProjArgs& a,
                            cudaStream_t stream) {
  static PerDeviceOnce configured;
  const cudaError_t e = configured.run([] {
    const cudaError_t x =
        cudaFuncSetAttribute(mtp_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMtSmemLimit);
    return x == cudaSuccess ? prefer_max_shared(mtp_proj_kernel) : x;
  });
  if (e != cudaSuccess) return e;
  MtpProjArgs b = a;
  b.stages = mtp_stages(a.n_pad);
  // the split's sums [T][128] f32 pass through the operand stages on their way out
  if (static_cast<size_t>(a.B) * a.q * 512u > static_cast<size_t>(b.stages) * mtp_stage_bytes(a.n_pad))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(a.m_tiles * a.k_splits);
  cfg.blockDim = dim3(kMtThreads);
  cfg.dynamicSmemBytes = mtp_smem_bytes(a.n_pad, b.stages);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mtp_proj_kernel, tmap_w, tmap_e, b);
}

}  // namespace ple
