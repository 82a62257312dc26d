// Projection of the gathered n-gram embeddings onto the hidden size on the
// fifth-generation tensor cores (tcgen05, accumulators in TMEM), with the
// layer's tail fused into the epilogue: sigmoid gate, width-4 causal
// depthwise conv along the sequence, residual add, carried state.
//
// "Projection" and "gating" / "short convolution" are the steps the DGX Spark
// deployment report lists after dequantisation ("【Qwen3.8-Flash-Next
// 端侧部署】01-模型架构与整体方案", section "n-gram embedding
// 是一条附加的条件记忆路径").
//
// Orientation (swap-AB): the MMA's M dimension is the hidden channel (128 per
// tile, operand A = fp16 W_proj^T, K-major) and N is the token (up to 256 per
// tile, operand B = the fp16 embeddings e, K-major). In TMEM a thread of the
// epilogue then owns one channel and sees consecutive tokens in consecutive
// columns, so the conv along the sequence is a sliding window in registers,
// and every global load/store of the epilogue is coalesced across channels.
//
// Conv halo: a fused tile covers 256 token rows but outputs the last 253;
// its first 3 rows are recomputed so that the conv window is complete.
//
// Epilogue data path (fused): h arrives by TMA in 32-token chunks into a
// 3-deep ring; each thread adds its channel's conv output and, for bf16
// output, writes the result back into the same shared-memory chunk, which a
// TMA store then writes to `out` (fp32 output is stored directly). Chunks in
// which no token starts a sequence or ends one with state take a branch-free
// path.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues tcgen05.mma, warps 2-5 run the epilogue (one TMEM lane quarter each).
// The grid is persistent (one CTA per SM), accumulators are double-buffered
// (2 x 256 TMEM columns), the K pipeline has 4 stages of 64.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ple_device.cuh"
#include "ple_internal.h"

namespace ple {
namespace {

constexpr int BM = 128;            // channels per tile (MMA M)
constexpr int BK = 64;             // K per stage: one 128-byte swizzled row of fp16
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int BN_MAX = 256;        // tokens per tile (MMA N)
constexpr int EPI_CHUNK = 32;      // tokens per TMEM load in the epilogue
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_STAGE = BM * BK * 2;          // 16 KB
constexpr uint32_t B_STAGE = BN_MAX * BK * 2;      // 32 KB
constexpr uint32_t H_CHUNK = EPI_CHUNK * BM * 2;   // 8 KB (bf16 h, 32 tokens x 128 channels)
constexpr uint32_t H_BUFS = 3;                     // ring of h / output chunks

constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + STAGES * A_STAGE;
constexpr uint32_t OFF_H = OFF_B + STAGES * B_STAGE;
constexpr uint32_t OFF_META = OFF_H + H_BUFS * H_CHUNK;
constexpr uint32_t OFF_FLAGS = OFF_META + BN_MAX * 16;
constexpr uint32_t OFF_BAR = OFF_FLAGS + 64;
constexpr uint32_t SMEM_USED = OFF_BAR + 256;
static_assert(SMEM_USED + 1024 <= static_cast<uint32_t>(kGemmSmemBytes), "smem layout");

struct SmemBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t hfull[H_BUFS];
  uint32_t tmem_base;
  int32_t abort_flag;
};
static_assert(sizeof(SmemBars) <= 256, "barrier block");

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                              int32_t* status) {
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

__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& m, int& n, int& ks) {
  m = tile % p.m_tiles;
  const int rest = tile / p.m_tiles;
  n = rest % p.n_tiles;
  ks = rest / p.n_tiles;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_e,
            const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_o,
            const __grid_constant__ CUtensorMap tmap_o_head, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemBars* bars = reinterpret_cast<SmemBars*>(smem + OFF_BAR);
  volatile int32_t* abort_flag = &bars->abort_flag;
  const uint32_t sA = smem_u32(smem + OFF_A);
  const uint32_t sB = smem_u32(smem + OFF_B);
  const uint32_t sH = smem_u32(smem + OFF_H);
  TokMeta* meta_s = reinterpret_cast<TokMeta*>(smem + OFF_META);
  uint32_t* chunk_flags = reinterpret_cast<uint32_t*>(smem + OFF_FLAGS);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = p.m_tiles * p.n_tiles * p.k_splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bars->tfull[a]), 1);
      mbar_init(smem_u32(&bars->tempty[a]), EPI_THREADS);
    }
    for (uint32_t b = 0; b < H_BUFS; ++b) mbar_init(smem_u32(&bars->hfull[b]), 1);
    bars->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      tma_prefetch_desc(&tmap_e);
      uint32_t stage = 0, phase = 0;
      uint32_t issued_parity[STAGES];
      bool issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
      const uint32_t tx_bytes = A_STAGE + static_cast<uint32_t>(p.n_tok) * BK * 2;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        int m, n, ks;
        tile_coords(p, tile, m, n, ks);
        const int tok0 = p.tok_origin + n * p.tok_stride;
        const int kb0 = ks * p.num_kb / p.k_splits, kb1 = (ks + 1) * p.num_kb / p.k_splits;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(smem_u32(&bars->empty[stage]), phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t fb = smem_u32(&bars->full[stage]);
          mbar_arrive_expect_tx(fb, tx_bytes);
          tma_load_2d(sA + stage * A_STAGE, &tmap_w, kb * BK, m * BM, fb);
          tma_load_2d(sB + stage * B_STAGE, &tmap_e, kb * BK, tok0, fb);
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // let copies already in flight land before the CTA's shared memory is released
        for (int s = 0; s < STAGES; ++s) {
          if (!issued[s]) continue;
          const long long start = clock64();
          while (!mbar_try_wait(smem_u32(&bars->full[s]), issued_parity[s]) &&
                 clock64() - start < kWaitLimitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(BM, p.n_tok);
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
        int m, n, ks;
        tile_coords(p, tile, m, n, ks);
        (void)m; (void)n;
        const int kb0 = ks * p.num_kb / p.k_splits, kb1 = (ks + 1) * p.num_kb / p.k_splits;
        const int acc = it & 1;
        const uint32_t acc_parity = (it >> 1) & 1;
        if (!wait_or_abort(smem_u32(&bars->tempty[acc]), acc_parity ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(acc * BN_MAX);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_or_abort(smem_u32(&bars->full[stage]), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sdesc_k_sw128(sA + stage * A_STAGE);
          const uint64_t bdesc = sdesc_k_sw128(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            // advance 16 fp16 = 32 bytes along K inside the swizzled row: +2 in the >>4 address field
            mma_f16(tmem_d, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          mma_commit(smem_u32(&bars->empty[stage]));
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(smem_u32(&bars->tfull[acc]));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;                 // TMEM lanes [32*quarter, 32*quarter+32)
    const int row = quarter * 32 + lane;          // channel inside the tile
    const int et = threadIdx.x - 64;              // 0..127
    const int nchunks = (p.n_tok + EPI_CHUNK - 1) / EPI_CHUNK;
    const bool tma_out = p.fused && !p.out_f32;   // bf16 output leaves through TMA stores
    uint32_t hchunk = 0;                          // h chunks consumed so far (ring position)
    uint32_t h_pending = 0;                       // ring buffers with a load in flight (abort path)
    uint32_t h_pend_par = 0;                      // and the phase parity each of those loads completes
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++it) {
      int m, n, ks;
      tile_coords(p, tile, m, n, ks);
      const int tok0 = p.tok_origin + n * p.tok_stride;
      const int ch = m * BM + row;
      const int acc = it & 1;
      const uint32_t acc_parity = (it >> 1) & 1;

      if (p.fused) {
        // token metadata of the tile, and per 32-token chunk a flag telling
        // whether any token needs more than the plain sliding window
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int i = et + k * EPI_THREADS;
          const int t = tok0 + i;
          TokMeta mt;
          if (t >= 0 && t < p.T) mt = p.meta[t];
          else { mt.g = 0.f; mt.seq = 0; mt.pos = -1; mt.flags = 0; }
          meta_s[i] = mt;
          const bool special = mt.pos <= 0 || ((mt.flags & kFlagLast) && p.conv_state != nullptr) ||
                               (!tma_out && i < p.halo);
          const unsigned b = __ballot_sync(0xffffffffu, special);
          if (lane == 0) chunk_flags[(et >> 5) + 4 * k] = b;
        }
        if (et == 0) {
          bulk_wait_group_read<1>();              // the two oldest ring buffers are no longer being stored
          for (int b = 0; b < 2 && b < nchunks; ++b) {
            const uint32_t buf = (hchunk + b) % H_BUFS;
            const uint32_t hb = smem_u32(&bars->hfull[buf]);
            mbar_arrive_expect_tx(hb, H_CHUNK);
            tma_load_2d(sH + buf * H_CHUNK, &tmap_h, m * BM, tok0 + b * EPI_CHUNK, hb);
            h_pending |= 1u << buf;
            h_pend_par = (h_pend_par & ~(1u << buf)) | ((((hchunk + b) / H_BUFS) & 1u) << buf);
          }
        }
        named_bar_sync(1, EPI_THREADS);
      }

      if (!wait_or_abort(smem_u32(&bars->tfull[acc]), acc_parity, abort_flag, p.status)) { ok = false; break; }
      tc_fence_after();

      float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
      if (p.fused) cw = reinterpret_cast<const float4*>(p.conv_w)[ch];
      float w0 = 0.f, w1 = 0.f, w2 = 0.f;      // u_{t-3}, u_{t-2}, u_{t-1}
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN_MAX);

      for (int c = 0; c < nchunks; ++c) {
        float v[32];
        tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(c * EPI_CHUNK), v);
        if (p.fused) {
          const uint32_t gc = hchunk + c;
          const uint32_t buf = gc % H_BUFS;
          if (!wait_or_abort(smem_u32(&bars->hfull[buf]), (gc / H_BUFS) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          h_pending &= ~(1u << buf);
          __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(smem + OFF_H + buf * H_CHUNK);
          const TokMeta* mc = meta_s + c * EPI_CHUNK;
          if (chunk_flags[c] == 0) {
            // every token valid, none starts a sequence, no state to write
#pragma unroll
            for (int i = 0; i < EPI_CHUNK; ++i) {
              const float u = mc[i].g * v[i];
              const float y = cw.x * w0 + cw.y * w1 + cw.z * w2 + cw.w * u;
              w0 = w1; w1 = w2; w2 = u;
              const float o = __bfloat162float(hs[i * BM + row]) + y;
              if (tma_out) {
                hs[i * BM + row] = __float2bfloat16_rn(o);
              } else {
                const int t = tok0 + c * EPI_CHUNK + i;
                reinterpret_cast<float*>(p.out)[static_cast<int64_t>(t) * p.H + ch] = o;
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < EPI_CHUNK; ++i) {
              const int tl = c * EPI_CHUNK + i;
              const TokMeta mt = mc[i];
              if (mt.pos < 0) continue;            // outside [0, T): same for the whole warp
              const float u = mt.g * v[i];
              if (mt.pos == 0) {                   // sequence start: carried state or zeros
                if (p.conv0 != nullptr) {
                  const float* c0 = p.conv0 + static_cast<int64_t>(mt.seq) * 3 * p.H + ch;
                  w0 = c0[0]; w1 = c0[p.H]; w2 = c0[2 * p.H];
                } else {
                  w0 = w1 = w2 = 0.f;
                }
              }
              const float y = cw.x * w0 + cw.y * w1 + cw.z * w2 + cw.w * u;
              w0 = w1; w1 = w2; w2 = u;
              if (tl >= p.halo) {
                const float o = __bfloat162float(hs[i * BM + row]) + y;
                if (tma_out) {
                  hs[i * BM + row] = __float2bfloat16_rn(o);
                } else {
                  const int t = tok0 + tl;
                  reinterpret_cast<float*>(p.out)[static_cast<int64_t>(t) * p.H + ch] = o;
                }
                if (p.conv_state != nullptr && (mt.flags & kFlagLast)) {
                  float* cs = p.conv_state + static_cast<int64_t>(mt.seq) * 3 * p.H + ch;
                  cs[0] = w0; cs[p.H] = w1; cs[2 * p.H] = w2;
                  if (ch == 0) {
                    p.hist_state[2 * mt.seq] = p.hist_new[2 * mt.seq];
                    p.hist_state[2 * mt.seq + 1] = p.hist_new[2 * mt.seq + 1];
                  }
                }
              }
            }
          }
          if (tma_out) fence_proxy_async_smem();   // make the smem writes visible to the TMA store
          named_bar_sync(1, EPI_THREADS);
          if (et == 0) {
            if (tma_out) {
              // the first chunk of a tile starts with the halo rows, which belong to the previous tile
              if (c == 0 && p.halo > 0)
                tma_store_2d(&tmap_o_head, sH + buf * H_CHUNK + p.halo * BM * 2, m * BM, tok0 + p.halo);
              else
                tma_store_2d(&tmap_o, sH + buf * H_CHUNK, m * BM, tok0 + c * EPI_CHUNK);
              bulk_commit_group();
            }
            if (c + 2 < nchunks) {
              bulk_wait_group_read<1>();            // buffer (gc + 2) % 3 was stored one group ago
              const uint32_t nb = (gc + 2) % H_BUFS;
              const uint32_t hbar = smem_u32(&bars->hfull[nb]);
              mbar_arrive_expect_tx(hbar, H_CHUNK);
              tma_load_2d(sH + nb * H_CHUNK, &tmap_h, m * BM, tok0 + (c + 2) * EPI_CHUNK, hbar);
              h_pending |= 1u << nb;
              h_pend_par = (h_pend_par & ~(1u << nb)) | ((((gc + 2) / H_BUFS) & 1u) << nb);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < EPI_CHUNK; ++i) {
            const int tl = c * EPI_CHUNK + i;
            const int t = tok0 + tl;
            if (tl < p.n_tok && t < p.T)
              p.partial[(static_cast<int64_t>(ks) * p.T + t) * p.H + ch] = v[i];
          }
        }
      }
      if (!ok) break;
      if (p.fused) hchunk += nchunks;
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->tempty[acc]));
      if (p.fused) named_bar_sync(1, EPI_THREADS);  // meta_s is rewritten by the next tile
    }
    if (et == 0) {
      if (!ok) {
        for (uint32_t b = 0; b < H_BUFS; ++b) {
          if (!(h_pending & (1u << b))) continue;
          const uint32_t par = (h_pend_par >> b) & 1u;
          const long long start = clock64();
          while (!mbar_try_wait(smem_u32(&bars->hfull[b]), par) && clock64() - start < kWaitLimitCycles) {
          }
        }
      }
      bulk_wait_group<0>();                      // output stores complete before the CTA exits
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const CUtensorMap& tmap_h,
                        const CUtensorMap& tmap_o, const CUtensorMap& tmap_o_head, const GemmParams& p, int grid,
                        cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  gemm_kernel<<<grid, NUM_THREADS, kGemmSmemBytes, stream>>>(tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, p);
  return cudaGetLastError();
}

}  // namespace ple
