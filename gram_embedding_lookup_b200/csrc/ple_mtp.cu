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
// per SM, each with 94 KB of W_proj and 140 KB of e. The first stages' W_proj
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
// Warp roles (192 threads): warp 0 issues the TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2-5 (one TMEM lane quarter each) run the
// epilogue.
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
constexpr int kMtThreads = 192;
constexpr int kMtTmaWarp = 0;
constexpr int kMtMmaWarp = 1;
constexpr int kMtEpiWarp0 = 2;
constexpr int kMtEpiThreads = 128;
constexpr int kMtStages = 5;              // most stages; fewer when 256 tokens do not leave room
constexpr uint32_t kMtAStage = kMtM * kMtBK * 2;   // 16 KB
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

// Dynamic shared memory from a 1024-byte aligned base: A stages, B stages
// (n_pad rows of 128 bytes each), then the barriers.
size_t mtp_smem_bytes(int n_pad, int stages) {
  return 1024 + static_cast<size_t>(stages) * (kMtAStage + static_cast<size_t>(n_pad) * kMtBK * 2) + sizeof(MtBars);
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
  const uint32_t b_stage = static_cast<uint32_t>(a.n_pad) * kMtBK * 2;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + S * kMtAStage;
  MtBars* bars = reinterpret_cast<MtBars*>(smem + S * (kMtAStage + b_stage));
  volatile int32_t* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x % a.m_tiles, ks = blockIdx.x / a.m_tiles;
  const int kb0 = ks * a.num_kb / a.k_splits, kb1 = (ks + 1) * a.num_kb / a.k_splits;
  const int nkb = kb1 - kb0;
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
      const uint32_t tx = kMtAStage + b_stage;
      const int pre = min(nkb, S);
      // W_proj of the first stages does not depend on the previous kernel
      for (int i = 0; i < pre; ++i) {
        const uint32_t fb = smem_u32(&bars->full[i]);
        mbar_arrive_expect_tx(fb, tx);
        tma_load_2d(sA + i * kMtAStage, &tmap_w, (kb0 + i) * kMtBK, m * kMtM, fb);
      }
      pdl_launch_dependents();
      pdl_wait();                                             // e comes from the embed kernel
      for (int i = 0; i < pre; ++i)
        tma_load_2d(sB + i * b_stage, &tmap_e, (kb0 + i) * kMtBK, 0, smem_u32(&bars->full[i]));
      int issued = pre;
      for (int i = pre; i < nkb; ++i) {
        const int stage = i % S;
        const uint32_t round = static_cast<uint32_t>(i / S);
        if (!wait_bar(smem_u32(&bars->empty[stage]), (round - 1) & 1, abort_flag, a.status)) break;
        const uint32_t fb = smem_u32(&bars->full[stage]);
        mbar_arrive_expect_tx(fb, tx);
        tma_load_2d(sA + stage * kMtAStage, &tmap_w, (kb0 + i) * kMtBK, m * kMtM, fb);
        tma_load_2d(sB + stage * b_stage, &tmap_e, (kb0 + i) * kMtBK, 0, fb);
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
      for (int i = 0; i < nkb; ++i) {
        const int stage = i % S;
        if (!wait_bar(smem_u32(&bars->full[stage]), static_cast<uint32_t>(i / S) & 1, abort_flag, a.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t adesc = sdesc_k_sw128(sA + stage * kMtAStage);
        const uint64_t bdesc = sdesc_k_sw128(sB + stage * b_stage);
#pragma unroll
        for (int k = 0; k < kMtBK / kMtUmmaK; ++k)
          mma_f16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bars->empty[stage]));
      }
      if (ok) mma_commit(smem_u32(&bars->tfull));
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2-5)
    const int et = threadIdx.x - 32 * kMtEpiWarp0;          // 0..127
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                     // channel inside the tile
    const int ch = m * kMtM + row;
    const float4 cw = __ldg(reinterpret_cast<const float4*>(a.conv_w) + ch);
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
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      float* mine = slab + static_cast<int64_t>(ks) * a.n_pad * kMtM + row;
      for (int c = 0; c * 32 < T; ++c) {
        float v[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(c * 32), v);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c * 32 + j < T) __stcg(mine + static_cast<int64_t>(c * 32 + j) * kMtM, v[j]);
      }
    }
    tc_fence_before();
    // ---- the tile's splits meet: count in, wait (bounded) for the others
    __threadfence();
    named_bar_sync(1, kMtEpiThreads);
    __shared__ int32_t go;
    if (et == 0) {
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
      // ---- this CTA's share of the sequences, all 128 channels of the tile, in chunks
      //      of whole sequences. Everything a chunk needs goes into shared memory at
      //      once (the operand stages are free: every MMA has completed): the
      //      splits' sums by bulk copies, hidden at the tile's channels, the gates
      //      and the carried state by 16-byte cp.async, so a chunk costs one round
      //      trip to L2. Then each thread runs its channel.
      const int b0 = ks * a.B / a.k_splits, b1 = (ks + 1) * a.B / a.k_splits;
      const uint32_t region = static_cast<uint32_t>(S) * (kMtAStage + b_stage);
      const uint32_t per_seq = static_cast<uint32_t>(a.q) * (a.k_splits * 512u + 256u + 16u) + 3u * 512u + 4u;
      const int max_seqs = max(1, static_cast<int>(region / per_seq));
      const uint32_t staged_bar = smem_u32(&bars->staged);
      uint32_t chunk_parity = 0;
      for (int bc = b0; bc < b1 && go; bc += max_seqs) {
        const int ns = min(max_seqs, b1 - bc);
        const int nt = ns * a.q, t0 = bc * a.q;
        uint8_t* P = smem;                                           // [k_splits][nt][128] f32
        uint8_t* Hs = P + static_cast<size_t>(a.k_splits) * nt * 512;   // [nt][128] bf16
        uint8_t* Ms = Hs + static_cast<size_t>(nt) * 256;              // [nt] TokMeta
        uint8_t* Cs = Ms + static_cast<size_t>(nt) * 16;               // [ns][3][128] f32
        uint8_t* Ns = Cs + static_cast<size_t>(ns) * 3 * 512;          // [ns] n_commit
        if (et == 0) {
          mbar_arrive_expect_tx(staged_bar, static_cast<uint32_t>(a.k_splits) * nt * 512u);
          for (int sp = 0; sp < a.k_splits; ++sp)
            bulk_load(smem_u32(P + static_cast<size_t>(sp) * nt * 512),
                      slab + (static_cast<int64_t>(sp) * a.n_pad + t0) * kMtM, static_cast<uint32_t>(nt) * 512u,
                      staged_bar);
        }
        for (int x = et; x < nt * 16; x += kMtEpiThreads) {
          const int tk = x >> 4, c16 = x & 15;
          cp_async_16(smem_u32(Hs + tk * 256 + c16 * 16),
                      a.hidden + static_cast<int64_t>(t0 + tk) * a.H + m * kMtM + c16 * 8);
        }
        for (int x = et; x < nt; x += kMtEpiThreads) cp_async_16(smem_u32(Ms + x * 16), a.meta + t0 + x);
        for (int x = et; x < ns * 3 * 32; x += kMtEpiThreads) {
          const int r3 = x >> 5, c32 = x & 31;
          cp_async_16(smem_u32(Cs + r3 * 512 + c32 * 16),
                      a.conv_state + (static_cast<int64_t>(bc) * 3 + r3) * a.H + m * kMtM + c32 * 4);
        }
        if (a.n_commit != nullptr)
          for (int x = et; x < ns; x += kMtEpiThreads) cp_async_4(smem_u32(Ns + x * 4), a.n_commit + bc + x);
        cp_async_commit();
        cp_async_wait_all();
        named_bar_sync(1, kMtEpiThreads);
        if (!wait_bar(staged_bar, chunk_parity, abort_flag, a.status)) break;
        chunk_parity ^= 1;
        const float* Pf = reinterpret_cast<const float*>(P);
        const __nv_bfloat16* Hb = reinterpret_cast<const __nv_bfloat16*>(Hs);
        const TokMeta* Mm = reinterpret_cast<const TokMeta*>(Ms);
        const float* Cf = reinterpret_cast<const float*>(Cs);
        // Each thread owns its channel's row of every staged array, so the three
        // passes below need no barrier between them. With one epilogue warp per
        // scheduler, each pass keeps a batch of tokens' loads in flight before any
        // of them is used. 1. The gated sums u: 16 tokens at a time, the splits'
        // sums added in split order; u overwrites split 0's slot.
        // The loads of a batch are unconditional (a token index past the chunk
        // reads the chunk's last token again), so that no branch splits them.
        float* Uf = reinterpret_cast<float*>(P);
        for (int tq = 0; tq < nt; tq += 16) {
          int off[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) off[j] = min(tq + j, nt - 1) * kMtM + row;
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
#pragma unroll 2
          for (int sp = 0; sp < a.k_splits; ++sp) {
            const float* ps = Pf + sp * nt * kMtM;
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] += ps[off[j]];
          }
          float g[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) g[j] = Mm[min(tq + j, nt - 1)].g;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (tq + j < nt) Uf[off[j]] = g[j] * v[j];
        }
        // 2. the outputs, 8 tokens at a time: the conv reads the sequence's
        //    extended stream (three carried entries, then its tokens' u), token i
        //    taps entries i, i + 1, i + 2 and its own u
        {
          int sb = 0, i = 0;                               // sequence and position of token tq
          for (int tq = 0; tq < nt; tq += 8) {
            float e0[8], e1[8], e2[8], u[8], hv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              // past the chunk's end: the last token's entries again (unused)
              const int tc = min(tq + j, nt - 1);
              const int ic = tq + j < nt ? i : a.q - 1, sc = tq + j < nt ? sb : ns - 1;
              const float* xc = Cf + sc * 3 * kMtM + row;
              const float* xu = Uf + (tc - ic) * kMtM + row;
              e0[j] = *(ic >= 3 ? xu + (ic - 3) * kMtM : xc + ic * kMtM);
              e1[j] = *(ic >= 2 ? xu + (ic - 2) * kMtM : xc + (ic + 1) * kMtM);
              e2[j] = *(ic >= 1 ? xu + (ic - 1) * kMtM : xc + (ic + 2) * kMtM);
              u[j] = xu[ic * kMtM];
              hv[j] = __bfloat162float(Hb[tc * kMtM + row]);
              if (++i == a.q) {
                i = 0;
                ++sb;
              }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (tq + j < nt) {
                const float y = cw.x * e0[j] + cw.y * e1[j] + cw.z * e2[j] + cw.w * u[j];
                const int64_t idx = static_cast<int64_t>(t0 + tq + j) * a.H + ch;
                const float o = hv[j] + y;
                if (a.out_f32) reinterpret_cast<float*>(a.out)[idx] = o;
                else reinterpret_cast<__nv_bfloat16*>(a.out)[idx] = __float2bfloat16_rn(o);
              }
            }
          }
        }
        // 3. the carried state, 4 sequences at a time: the three entries of the
        //    extended stream that end at the sequence's last committed token
        for (int sq = 0; sq < ns; sq += 4) {
          float k[4][3];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int sb = min(sq + j, ns - 1);
            int32_t ncb = a.n_commit ? reinterpret_cast<const int32_t*>(Ns)[sb] : a.q;
            if (ncb < 1 || ncb > a.q) {
              if (et == 0 && m == 0) set_status(a.status, PLE_ERR_RANGE);
              ncb = max(1, min(ncb, a.q));
            }
            const float* xc = Cf + sb * 3 * kMtM + row;
            const float* xu = Uf + sb * a.q * kMtM + row;
#pragma unroll
            for (int r = 0; r < 3; ++r) k[j][r] = *(ncb + r >= 3 ? xu + (ncb + r - 3) * kMtM : xc + (ncb + r) * kMtM);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (sq + j < ns) {
              float* cs = a.conv_state + static_cast<int64_t>(bc + sq + j) * 3 * a.H + ch;
              cs[0] = k[j][0];
              cs[a.H] = k[j][1];
              cs[2 * a.H] = k[j][2];
            }
          }
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
