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
// Orientation (swap-AB): the MMA's M dimension is the hidden channel
// (operand A = fp16 W_proj^T, K-major) and N is the token (up to 256 per tile,
// operand B = the fp16 embeddings e, K-major). In TMEM a thread of the
// epilogue then owns one channel and sees consecutive tokens in consecutive
// columns, so the conv along the sequence is a sliding window in registers,
// and every global load/store of the epilogue is coalesced across channels.
//
// Two forms share one epilogue:
//   - single-SM tiles (CTAS = 1): 128 channels x up to 256 tokens, 4 K-stages;
//     also runs the split-K variant that writes fp32 partials;
//   - SM-pair tiles (CTAS = 2, a cluster of two CTAs): 256 channels x 256
//     tokens. Each CTA loads its 128 channels of W and its 128 tokens of e;
//     the even CTA issues tcgen05.mma.cta_group::2 (M = 256), which reads the
//     other halves from the odd CTA's shared memory and writes each CTA's 128
//     channels into that CTA's TMEM. Per SM this halves the token-operand
//     traffic from L2, the bound of the single-SM form. 5 K-stages.
//
// Conv halo: a fused tile covers 256 token rows but outputs the last 253;
// its first 3 rows are recomputed so that the conv window is complete.
//
// Epilogue data path (fused): h arrives by TMA in 32-token chunks into a ring
// of shared-memory buffers (7 for SM pairs, 3 for single SMs) that runs ahead
// across tile boundaries. Each compute thread adds its channel's conv output
// and, for bf16 output, writes the result back into the same shared-memory
// chunk; the I/O warp then stores the chunk with one TMA store and refills
// the ring, so the compute warps never wait on TMA issue and need no barrier
// per chunk. fp32 output is stored directly. Chunks in which no token starts a
// sequence or ends one with state take a branch-free path.
//
// Warp roles (224 threads): warp 0 issues the operand TMA loads, warp 1 owns
// TMEM and issues tcgen05.mma (the even CTA of a pair only), warps 2-5 run
// the epilogue arithmetic (one TMEM lane quarter each), warp 6 moves the
// epilogue's h and output chunks. The grid is persistent (one CTA per SM),
// the accumulators are double-buffered (2 x 256 TMEM columns).
//
// Gather-fused form (SM pairs): the token operand never exists in HBM. A
// loader warp per CTA copies, for each K-stage, the 64 codes the stage takes
// from the two FP8 E4M3 table rows of each of the CTA's 128 tokens, and the
// rows' scales, into a ring of landing slots in shared memory (16-byte
// cp.async, completion counted on the slot's mbarrier). Eight converter warps
// dequantise each slot exactly as the embed kernel does (one helper) and store
// the fp16 result into the stage's 128-byte-swizzled B tile, fence the
// generic-proxy stores for the tensor core and arrive on the even CTA's full
// barrier (CTA-scope release: the data stays in the converter's own CTA),
// whose expected count covers the W TMA and the sixteen converter warps of
// the pair. Neither the loader nor the converters hold global loads in
// flight, so no fence or arrive waits on memory.
// Roles (512 threads): warps 0-3 the epilogue arithmetic, warp 4 the W TMA,
// warp 5 TMEM and MMA, warp 6 the epilogue I/O, warp 7 the row loader, warps
// 8-15 the converters.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ple_device.cuh"
#include "ple_internal.h"

namespace ple {
namespace {

constexpr int BM = 128;            // channels per CTA (TMEM lanes)
constexpr int BK = 64;             // K per stage: one 128-byte swizzled row of fp16
constexpr int UMMA_K = 16;
constexpr int BN_MAX = 256;        // tokens per tile (MMA N)
constexpr int EPI_CHUNK = 32;      // tokens per TMEM load in the epilogue
constexpr int CPT = BN_MAX / EPI_CHUNK;   // epilogue chunks per fused tile
constexpr int EPI_THREADS = 128;   // compute threads of the epilogue
constexpr int IO_WARP = 6;
constexpr int CONV_WARPS = 8;      // gather-fused form: converter warps per CTA (warps 8-15)
constexpr int CONV_WARP0 = 8;
constexpr int LOADER_WARP = 7;

// Warp roles of the two forms (GATHER = false: B by TMA from e; true: gathered).
template <bool GATHER>
struct Roles {
  static constexpr int THREADS = GATHER ? 512 : 224;
  static constexpr int TMA_WARP = GATHER ? 4 : 0;
  static constexpr int MMA_WARP = GATHER ? 5 : 1;
  static constexpr int EPI_WARP0 = GATHER ? 0 : 2;    // four epilogue warps from here
};
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t A_STAGE = BM * BK * 2;          // 16 KB
constexpr uint32_t H_CHUNK = EPI_CHUNK * BM * 2;   // 8 KB (bf16 h, 32 tokens x 128 channels)

template <int CTAS, bool GATHER = false>
struct Cfg {
  // K-blocks per stage: the SM-pair form fetches two K-blocks of each operand
  // per TMA copy (a 3-D box of 32 KB), which the copy engine delivers at about
  // 72 B/clk per SM against about 41 B/clk for two 16 KB boxes (measured)
  static constexpr int KBS = (!GATHER && CTAS == 2) ? 2 : 1;
  static constexpr int STAGES = GATHER ? 4 : (CTAS == 2 ? 3 : 4);
  static constexpr int HBUFS = GATHER ? 4 : 3;                   // ring of h / output chunks
  static constexpr int LSTAGES = GATHER ? 3 : 0;                  // landing slots of FP8 row segments
  static constexpr uint32_t B_ROWS = BN_MAX / CTAS;              // token rows of e held by one CTA
  static constexpr uint32_t A_BYTES = KBS * A_STAGE;             // W_proj bytes of a stage
  static constexpr uint32_t B_STAGE = KBS * B_ROWS * BK * 2;     // e bytes of a stage
  // landing slot: BK codes of each token's order-0 row, then of its order-1
  // row (64 bytes per token and order); the rows' scales of a tile go into one
  // of two buffers (by tile parity), 8 bytes per token
  static constexpr uint32_t L_CODES = B_ROWS * BK;               // 8 KB per order
  static constexpr uint32_t L_SLOT = 2 * L_CODES;
  static constexpr uint32_t S_BUF = B_ROWS * 8;
  static constexpr uint32_t OFF_A = 0;
  static constexpr uint32_t OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr uint32_t OFF_L = OFF_B + STAGES * B_STAGE;
  static constexpr uint32_t OFF_S = OFF_L + LSTAGES * L_SLOT;
  static constexpr uint32_t OFF_H = OFF_S + (GATHER ? 2 * S_BUF : 0);
  static constexpr uint32_t OFF_META = OFF_H + HBUFS * H_CHUNK;
  static constexpr uint32_t OFF_G = OFF_META + BN_MAX * 16;      // gates of the tile, one float per token
  static constexpr uint32_t OFF_FLAGS = OFF_G + BN_MAX * 4;
  static constexpr uint32_t OFF_BAR = OFF_FLAGS + 64;
  static constexpr uint32_t SMEM_USED = OFF_BAR + 512;
  static_assert(SMEM_USED + 1024 <= static_cast<uint32_t>(kGemmSmemBytes), "smem layout");
  static_assert(OFF_L % 1024 == 0 && L_SLOT % 128 == 0 && OFF_H % 128 == 0, "alignment of TMA destinations");
  static_assert(LSTAGES <= 8, "landing barriers");
};

template <int STAGES, int HBUFS>
struct SmemBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t hfull[HBUFS];    // h chunk landed (TMA)
  uint64_t cdone[HBUFS];    // compute threads finished the chunk in this buffer
  uint64_t lfull[8];        // gather-fused form: landing slot filled (every loader lane's copies landed)
  uint64_t lempty[8];       // landing slot read by every converter thread
  uint32_t tmem_base;
  int32_t abort_flag;
};
static_assert(sizeof(SmemBars<5, 7>) <= 512, "barrier block");

// CLUSTER: cluster-scope acquire (threads of the peer CTA arrive on the barrier).
template <bool CLUSTER = false>
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int32_t* abort_flag,
                                              int32_t* status) {
  auto test = [&] { return CLUSTER ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (test()) return true;
  const long long start = clock64();
  while (true) {
    if (test()) return true;
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

// Where this CTA's tiles are: tile number i of the CTA is unit + i * units.
struct TileWalk {
  int unit, units, total_tiles, rank, ctas;
  __device__ __forceinline__ bool coords(const GemmParams& p, int i, int& ch0, int& tok0) const {
    const int tile = unit + i * units;
    if (tile >= total_tiles) return false;
    int m, n, ks;
    tile_coords(p, tile, m, n, ks);
    ch0 = m * BM * ctas + rank * BM;
    tok0 = p.tok_origin + n * p.tok_stride;
    return true;
  }
};

// Token metadata of tile i for one compute thread's two tokens (et, et + 128).
__device__ __forceinline__ void load_meta(const GemmParams& p, const TileWalk& walk, int i, int et,
                                          TokMeta (&mt)[2]) {
  int ch0 = 0, tok0 = 0;
  const bool has = walk.coords(p, i, ch0, tok0);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int t = tok0 + et + k * EPI_THREADS;
    if (has && t >= 0 && t < p.T) mt[k] = p.meta[t];
    else { mt[k].g = 0.f; mt[k].seq = 0; mt[k].pos = -1; mt[k].flags = 0; }
  }
}

// The epilogue arithmetic of tile number `i` of this CTA (compute warps):
// TMEM -> gate, conv, residual -> out (fused), or TMEM -> fp32 partials
// (split-K). `q` is the running chunk number of the h stream. Returns false if
// a wait ran out.
template <int STAGES, int HBUFS, int EPI_W0>
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, uint8_t* smem, uint32_t off_h, uint32_t off_meta,
                                              uint32_t off_g, uint32_t off_flags, SmemBars<STAGES, HBUFS>* bars,
                                              volatile int32_t* abort_flag, const TileWalk& walk, int i, int ks,
                                              uint32_t tacc, uint32_t tfull_bar, uint32_t tfull_parity, uint32_t& q,
                                              TokMeta (&mt_next)[2]) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;                 // TMEM lanes [32*quarter, 32*quarter+32)
  const int row = quarter * 32 + lane;          // channel inside the CTA's 128
  const int et = threadIdx.x - 32 * EPI_W0;     // 0..127
  int ch0 = 0, tok0 = 0;
  walk.coords(p, i, ch0, tok0);
  const int ch = ch0 + row;
  const int nchunks = (p.n_tok + EPI_CHUNK - 1) / EPI_CHUNK;
  const bool tma_out = p.fused && !p.out_f32;   // bf16 output leaves through TMA stores
  TokMeta* meta_s = reinterpret_cast<TokMeta*>(smem + off_meta);
  float* g_s = reinterpret_cast<float*>(smem + off_g);
  uint32_t* chunk_flags = reinterpret_cast<uint32_t*>(smem + off_flags);

  if (p.fused) {
    // token metadata of the tile (loaded one tile ahead), and per 32-token chunk
    // a flag telling whether any token needs more than the plain sliding window
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int ti = et + k * EPI_THREADS;
      const TokMeta mt = mt_next[k];
      meta_s[ti] = mt;
      g_s[ti] = mt.g;
      const bool special = mt.pos <= 0 || ((mt.flags & kFlagLast) && p.conv_state != nullptr) ||
                           (!tma_out && ti < p.halo);
      const unsigned b = __ballot_sync(0xffffffffu, special);
      if (lane == 0) chunk_flags[(et >> 5) + 4 * k] = b;
    }
    load_meta(p, walk, i + 1, et, mt_next);     // the next tile's, while this one runs
    named_bar_sync(1, EPI_THREADS);
  }

  if (!wait_or_abort(tfull_bar, tfull_parity, abort_flag, p.status)) return false;
  tc_fence_after();

  float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
  if (p.fused) cw = reinterpret_cast<const float4*>(p.conv_w)[ch];
  float w0 = 0.f, w1 = 0.f, w2 = 0.f;          // u_{t-3}, u_{t-2}, u_{t-1}
  const uint32_t tbase = tacc + (static_cast<uint32_t>(quarter * 32) << 16);

  for (int c = 0; c < nchunks; ++c) {
    float v[32];
    tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>(c * EPI_CHUNK), v);
    if (p.fused) {
      const uint32_t buf = q % HBUFS;
      if (!wait_or_abort(smem_u32(&bars->hfull[buf]), (q / HBUFS) & 1, abort_flag, p.status)) return false;
      __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(smem + off_h + buf * H_CHUNK);
      if (chunk_flags[c] == 0) {
        // every token valid, none starts a sequence, no state to write:
        // first all loads, then the arithmetic
        float g[EPI_CHUNK], hf[EPI_CHUNK];
        const float4* g4 = reinterpret_cast<const float4*>(g_s + c * EPI_CHUNK);
#pragma unroll
        for (int j = 0; j < EPI_CHUNK / 4; ++j) {
          const float4 x = g4[j];
          g[4 * j] = x.x; g[4 * j + 1] = x.y; g[4 * j + 2] = x.z; g[4 * j + 3] = x.w;
        }
#pragma unroll
        for (int j = 0; j < EPI_CHUNK; ++j) hf[j] = __bfloat162float(hs[j * BM + row]);
#pragma unroll
        for (int j = 0; j < EPI_CHUNK; ++j) {
          const float u = g[j] * v[j];
          const float y = cw.x * w0 + cw.y * w1 + cw.z * w2 + cw.w * u;
          w0 = w1; w1 = w2; w2 = u;
          const float o = hf[j] + y;
          if (tma_out) {
            hs[j * BM + row] = __float2bfloat16_rn(o);
          } else {
            const int t = tok0 + c * EPI_CHUNK + j;
            reinterpret_cast<float*>(p.out)[static_cast<int64_t>(t) * p.H + ch] = o;
          }
        }
      } else {
        const TokMeta* mc = meta_s + c * EPI_CHUNK;
#pragma unroll
        for (int j = 0; j < EPI_CHUNK; ++j) {
          const int tl = c * EPI_CHUNK + j;
          const TokMeta mt = mc[j];
          if (mt.pos < 0) continue;            // outside [0, T): same for the whole warp
          const float u = mt.g * v[j];
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
            const float o = __bfloat162float(hs[j * BM + row]) + y;
            if (tma_out) {
              hs[j * BM + row] = __float2bfloat16_rn(o);
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
      if (tma_out) fence_proxy_async_smem();   // the TMA store reads these shared-memory writes
      mbar_arrive(smem_u32(&bars->cdone[buf]));
      ++q;
    } else {
#pragma unroll
      for (int j = 0; j < EPI_CHUNK; ++j) {
        const int tl = c * EPI_CHUNK + j;
        const int t = tok0 + tl;
        if (tl < p.n_tok && t < p.T)
          p.partial[(static_cast<int64_t>(ks) * p.T + t) * p.H + ch] = v[j];
      }
    }
  }
  tc_fence_before();
  return true;
}

// The I/O warp of the fused epilogue (one thread): keeps HBUFS - 1 h chunks
// loaded or in flight ahead of the compute threads, across tile boundaries,
// and stores each finished chunk of bf16 output with one TMA store.
template <int STAGES, int HBUFS>
__device__ __forceinline__ void epilogue_io(const GemmParams& p, uint32_t sH, SmemBars<STAGES, HBUFS>* bars,
                                            volatile int32_t* abort_flag, const CUtensorMap* tmap_h,
                                            const CUtensorMap* tmap_o, const CUtensorMap* tmap_o_head,
                                            const TileWalk& walk) {
  const bool tma_out = !p.out_f32;
  uint32_t issued = 0;                        // chunks whose h load has been issued
  uint32_t pending = 0, pend_par = 0;         // loads in flight per buffer (abort path)
  auto issue_upto = [&](uint32_t upto) {
    while (issued < upto) {
      int ch0, tok0;
      if (!walk.coords(p, static_cast<int>(issued / CPT), ch0, tok0)) return;   // past the last tile
      const uint32_t buf = issued % HBUFS;
      const uint32_t bar = smem_u32(&bars->hfull[buf]);
      mbar_arrive_expect_tx(bar, H_CHUNK);
      tma_load_2d(sH + buf * H_CHUNK, tmap_h, ch0, tok0 + static_cast<int>(issued % CPT) * EPI_CHUNK, bar);
      pending |= 1u << buf;
      pend_par = (pend_par & ~(1u << buf)) | (((issued / HBUFS) & 1u) << buf);
      ++issued;
    }
  };
  issue_upto(HBUFS - 1);
  bool ok = true;
  int ch0 = 0, tok0 = 0;
  for (int i = 0; ok && walk.coords(p, i, ch0, tok0); ++i) {
    for (int c = 0; c < CPT; ++c) {
      const uint32_t q = static_cast<uint32_t>(i * CPT + c);
      const uint32_t buf = q % HBUFS;
      if (!wait_or_abort(smem_u32(&bars->cdone[buf]), (q / HBUFS) & 1, abort_flag, p.status)) { ok = false; break; }
      pending &= ~(1u << buf);                // consumed, so its load had landed
      if (tma_out) {
        // the first chunk of a tile starts with the halo rows, which belong to the previous tile
        if (c == 0 && p.halo > 0)
          tma_store_2d(tmap_o_head, sH + buf * H_CHUNK + p.halo * BM * 2, ch0, tok0 + p.halo);
        else
          tma_store_2d(tmap_o, sH + buf * H_CHUNK, ch0, tok0 + c * EPI_CHUNK);
        bulk_commit_group();
      }
      bulk_wait_group_read<1>();              // the buffer refilled next was stored one group ago
      issue_upto(q + HBUFS);
    }
  }
  if (!ok) {
    for (int b = 0; b < HBUFS; ++b) {
      if (!(pending & (1u << b))) continue;
      const uint32_t par = (pend_par >> b) & 1u;
      const long long start = clock64();
      while (!mbar_try_wait(smem_u32(&bars->hfull[b]), par) && clock64() - start < kWaitLimitCycles) {
      }
    }
  }
  bulk_wait_group<0>();                        // output stores complete before the CTA exits
}

// First token row of this CTA in its tile number i (gather-fused form).
__device__ __forceinline__ int gather_first_token(const GemmParams& p, int unit, int units, int i, uint32_t rank) {
  int m, n, ks;
  tile_coords(p, unit + i * units, m, n, ks);
  return p.tok_origin + n * p.tok_stride + static_cast<int>(rank) * (BN_MAX / 2);
}

// The row loader of the gather-fused form (warp 7 of each CTA of a pair). Per
// K-stage it copies into the next landing slot the 64 codes the stage takes
// from the order-0 and order-1 rows of each of the CTA's 128 tokens (16-byte
// cp.async; four lanes cover one 64-byte row segment, so each instruction
// reads eight whole segments); with a tile's first stage it also copies the
// rows' scales (4-byte cp.async) into the scale buffer of the tile's parity.
// Lane l serves order (l / 4) % 2 of tokens l / 8 + 4k, k = 0..31; it reads
// those tokens' row IDs once per tile. Tokens outside [0, T) copy row 0 and
// are zeroed by the converters. A scale buffer is rewritten two tiles later,
// after the converters have read it (the loader runs at most LSTAGES <
// 2 num_kb stages ahead). Each lane arrives on the slot's barrier when its
// copies have landed, so the loader holds no loads in registers and never
// waits on memory except for the row IDs.
template <class C, int STAGES, int HBUFS>
__device__ __forceinline__ void gather_loader(const GemmParams& p, uint32_t sL, uint32_t sS, SmemBars<STAGES, HBUFS>* bars,
                                              volatile int32_t* abort_flag, int unit, int units, int total_tiles,
                                              uint32_t rank) {
  constexpr int LST = C::LSTAGES;
  const int lane = threadIdx.x & 31;
  const int piece = lane & 3;                          // 16-byte piece of the 64-byte segment
  const int ord = (lane >> 2) & 1;
  const int tok_lo = lane >> 3;                        // tokens tok_lo + 4k
  const bool scale_lane = piece == 0;                  // one lane per segment copies its scale
  const int my_tiles = (total_tiles - unit + units - 1) / units;
  const uint8_t* codes = p.codes + static_cast<int64_t>(16 * piece);
  const uint32_t dst_codes = static_cast<uint32_t>(ord) * C::L_CODES + static_cast<uint32_t>(tok_lo * BK + 16 * piece);
  const uint32_t dst_scale = sS + static_cast<uint32_t>(tok_lo * 8 + ord * 4);
  uint32_t ls = 0, lphase = 0;
  pdl_wait();                                          // the row IDs come from the previous kernel
  bool ok = true;
  for (int i = 0; i < my_tiles && ok; ++i) {
    const int t0 = gather_first_token(p, unit, units, i, rank) + tok_lo;
    int row[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int t = t0 + 4 * k;
      const bool valid = t >= 0 && t < p.T;
      const int* idp = reinterpret_cast<const int*>(p.ids + (valid ? t : 0)) + ord;
      row[k] = valid ? __ldg(idp) + (ord ? static_cast<int>(p.rows0) : 0) : 0;
    }
    for (int kb = 0; kb < p.num_kb; ++kb) {
      if (!wait_or_abort(smem_u32(&bars->lempty[ls]), lphase ^ 1, abort_flag, p.status)) { ok = false; break; }
      const uint32_t slot = sL + ls * C::L_SLOT;
      const int64_t koff = static_cast<int64_t>(kb) * BK;
#pragma unroll
      for (int k = 0; k < 32; ++k)
        cp_async_16(slot + dst_codes + static_cast<uint32_t>(k * 4 * BK), codes + static_cast<int64_t>(row[k]) * p.D + koff);
      if (kb == 0 && scale_lane) {                     // the tile's scales travel with its first stage
        const uint32_t sb = dst_scale + static_cast<uint32_t>(i & 1) * C::S_BUF;
#pragma unroll
        for (int k = 0; k < 32; ++k) cp_async_4(sb + static_cast<uint32_t>(k * 4 * 8), p.scales + row[k]);
      }
      cp_async_mbar_arrive_noinc(smem_u32(&bars->lfull[ls]));
      if (++ls == LST) { ls = 0; lphase ^= 1; }
    }
  }
  cp_async_wait_all();                                 // no copy lands after the CTA's shared memory is released
}

// The converters of the gather-fused form (warps 8-15 of each CTA of a pair).
// Thread (warp w, lane l) owns token rows r = 16w + l/4 and r + 8 of the CTA's
// 128 and the 16-code chunk c = l % 4 of the stage's 64 codes per row. Per
// stage it reads its codes and scales from the landing slot, releases the
// slot, dequantises 2 x 16 codes per row into fp16 and stores them at their
// 128-byte-swizzle positions (16-byte chunk index XOR row % 8) in the stage's
// B tile. Rows of tokens outside [0, T) are zero.
template <class C, int STAGES, int HBUFS>
__device__ __forceinline__ void gather_converter(const GemmParams& p, uint32_t sB, uint32_t sL, uint32_t sS,
                                                 SmemBars<STAGES, HBUFS>* bars, volatile int32_t* abort_flag,
                                                 int unit, int units, int total_tiles, uint32_t rank) {
  constexpr int LST = C::LSTAGES;
  const int cw = (threadIdx.x >> 5) - CONV_WARP0;
  const int lane = threadIdx.x & 31;
  const int c = lane & 3;
  const int r_lo = cw * 16 + (lane >> 2);             // rows r_lo and r_lo + 8
  const uint32_t swz = static_cast<uint32_t>(r_lo & 7);
  const uint32_t st0 = static_cast<uint32_t>(r_lo) * 128u + (((2u * c) ^ swz) << 4);
  const uint32_t st1 = static_cast<uint32_t>(r_lo) * 128u + (((2u * c + 1u) ^ swz) << 4);
  const uint32_t ld_codes = static_cast<uint32_t>(r_lo) * BK + 16u * c;
  const uint32_t ld_scale = sS + static_cast<uint32_t>(r_lo) * 8u;
  const int my_tiles = (total_tiles - unit + units - 1) / units;
  uint32_t ls = 0, lphase = 0, stage = 0, phase = 0;
  for (int i = 0; i < my_tiles; ++i) {
    const int t0 = gather_first_token(p, unit, units, i, rank) + r_lo;
    bool valid[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) valid[k] = t0 + 8 * k >= 0 && t0 + 8 * k < p.T;
    float2 sc[2];
    for (int kb = 0; kb < p.num_kb; ++kb) {
      if (!wait_or_abort(smem_u32(&bars->lfull[ls]), lphase, abort_flag, p.status)) return;
      const uint32_t slot = sL + ls * C::L_SLOT;
      uint4 a[2], b[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint32_t dr = static_cast<uint32_t>(k) * 8u;
        a[k] = ld_shared_v4(slot + ld_codes + dr * BK);
        b[k] = ld_shared_v4(slot + C::L_CODES + ld_codes + dr * BK);
        if (kb == 0) sc[k] = ld_shared_f2(ld_scale + static_cast<uint32_t>(i & 1) * C::S_BUF + dr * 8u);
      }
      mbar_arrive(smem_u32(&bars->lempty[ls]));       // the slot may be refilled
      if (++ls == LST) { ls = 0; lphase ^= 1; }
      if (!wait_or_abort(smem_u32(&bars->empty[stage]), phase ^ 1, abort_flag, p.status)) return;
      const uint32_t dst = sB + stage * C::B_STAGE;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint4 o0 = make_uint4(0u, 0u, 0u, 0u), o1 = make_uint4(0u, 0u, 0u, 0u);
        if (valid[k]) deq16(a[k], b[k], sc[k].x, sc[k].y, o0, o1);
        st_shared_v4(dst + st0 + k * 8 * 128, o0);
        st_shared_v4(dst + st1 + k * 8 * 128, o1);
      }
      fence_proxy_async_smem();                        // the tensor core reads these stores
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->full[stage]), 0));
      if (++stage == STAGES) { stage = 0; phase ^= 1; }
    }
  }
}

// GATHER = false: the token operand e comes by TMA (224 threads); true: the
// gather-fused form (512 threads, SM pairs only; tmap_e is not read).
template <int CTAS, bool GATHER>
__global__ void __launch_bounds__(Roles<GATHER>::THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_e,
            const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_o,
            const __grid_constant__ CUtensorMap tmap_o_head, const GemmParams p) {
  using C = Cfg<CTAS, GATHER>;
  using R = Roles<GATHER>;
  static_assert(!GATHER || CTAS == 2, "the gather-fused form runs on SM pairs");
  constexpr int STAGES = C::STAGES;
  constexpr int HBUFS = C::HBUFS;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array (an integer
  // round trip would hide the address space, and plain loads from it would be
  // generic ones)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  auto* bars = reinterpret_cast<SmemBars<STAGES, HBUFS>*>(smem + C::OFF_BAR);
  volatile int32_t* abort_flag = &bars->abort_flag;
  const uint32_t sA = smem_u32(smem + C::OFF_A);
  const uint32_t sB = smem_u32(smem + C::OFF_B);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = p.m_tiles * p.n_tiles * p.k_splits;
  const uint32_t rank = CTAS == 2 ? cluster_ctarank() : 0u;   // CTA inside the pair
  const bool leader = rank == 0;
  const int unit = blockIdx.x / CTAS;                         // pair (or CTA) index
  const int units = gridDim.x / CTAS;

  if (threadIdx.x == 0) {
    // full: the leader's W (and e) TMA arrive, plus one arrive per converter warp of the pair
    const uint32_t full_count = GATHER ? 1 + CONV_WARPS * CTAS : 1;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), full_count);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&bars->tfull[a]), 1);
      mbar_init(smem_u32(&bars->tempty[a]), EPI_THREADS * CTAS);
    }
    for (int b = 0; b < HBUFS; ++b) {
      mbar_init(smem_u32(&bars->hfull[b]), 1);
      mbar_init(smem_u32(&bars->cdone[b]), EPI_THREADS);
    }
    for (int l = 0; l < C::LSTAGES; ++l) {
      mbar_init(smem_u32(&bars->lfull[l]), 32);                 // every loader lane, once its copies land
      mbar_init(smem_u32(&bars->lempty[l]), 32 * CONV_WARPS);   // every converter thread
    }
    bars->abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == R::MMA_WARP) {
    if constexpr (CTAS == 2) {
      tmem_alloc_pair(smem_u32(&bars->tmem_base), TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CTAS == 2) cluster_sync();     // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;
  // a combine kernel after the split-K form may launch now; it waits for this grid
  pdl_launch_dependents();

  if (warp == R::TMA_WARP) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&tmap_w);
      if constexpr (!GATHER) tma_prefetch_desc(&tmap_e);
      uint32_t stage = 0, phase = 0;
      uint32_t issued_parity[STAGES];
      bool issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
      // bytes the even CTA's full barrier receives per stage (both CTAs' loads)
      const uint32_t tx_bytes =
          GATHER ? CTAS * A_STAGE : CTAS * C::KBS * (A_STAGE + static_cast<uint32_t>(p.n_tok / CTAS) * BK * 2);
      bool ok = true;
      bool e_ready = false;
      for (int tile = unit; tile < total_tiles && ok; tile += units) {
        int m, n, ks;
        tile_coords(p, tile, m, n, ks);
        const int tok0 = p.tok_origin + n * p.tok_stride;
        const int chA = m * BM * CTAS + static_cast<int>(rank) * BM;
        const int tokB = tok0 + static_cast<int>(rank) * (p.n_tok / CTAS);
        const int kb0 = ks * p.num_kb / p.k_splits, kb1 = (ks + 1) * p.num_kb / p.k_splits;
        for (int kb = kb0; kb < kb1; kb += C::KBS) {
          if (!wait_or_abort(smem_u32(&bars->empty[stage]), phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t fb = smem_u32(&bars->full[stage]);
          if (leader) mbar_arrive_expect_tx(fb, tx_bytes);
          if constexpr (C::KBS == 2) {
            // 3-D boxes {64, rows, 2 K-blocks}: a second K-block past the tensor is
            // zero-filled, one past this tile's K range is loaded and not used
            const uint32_t fb0 = mapa_shared(fb, 0);
            tma_load_3d_pair(sA + stage * C::A_BYTES, &tmap_w, 0, chA, kb, fb0);
            if (!e_ready) { pdl_wait(); e_ready = true; }     // e comes from the previous kernel
            tma_load_3d_pair(sB + stage * C::B_STAGE, &tmap_e, 0, tokB, kb, fb0);
          } else if constexpr (CTAS == 2) {
            const uint32_t fb0 = mapa_shared(fb, 0);
            tma_load_2d_pair(sA + stage * A_STAGE, &tmap_w, kb * BK, chA, fb0);
            if constexpr (!GATHER) {
              if (!e_ready) { pdl_wait(); e_ready = true; }   // e comes from the previous kernel
              tma_load_2d_pair(sB + stage * C::B_STAGE, &tmap_e, kb * BK, tokB, fb0);
            }
          } else {
            tma_load_2d(sA + stage * A_STAGE, &tmap_w, kb * BK, chA, fb);
            if (!e_ready) { pdl_wait(); e_ready = true; }
            tma_load_2d(sB + stage * C::B_STAGE, &tmap_e, kb * BK, tokB, fb);
          }
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      (void)e_ready;
      if (!ok && leader) {
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
  } else if (warp == R::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_f16_f32(BM * CTAS, p.n_tok);
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = unit; tile < total_tiles && ok; tile += units, ++it) {
        int m, n, ks;
        tile_coords(p, tile, m, n, ks);
        (void)m; (void)n;
        const int kb0 = ks * p.num_kb / p.k_splits, kb1 = (ks + 1) * p.num_kb / p.k_splits;
        const int acc = it & 1;
        const uint32_t acc_parity = (it >> 1) & 1;
        if (!wait_or_abort(smem_u32(&bars->tempty[acc]), acc_parity ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + static_cast<uint32_t>(acc * BN_MAX);
        for (int kb = kb0; kb < kb1; kb += C::KBS) {
          // gather-fused: the peer's converter warps arrive with cluster-scope release
          if (!wait_or_abort<GATHER>(smem_u32(&bars->full[stage]), phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int hk = 0; hk < C::KBS; ++hk) {
            if (kb + hk >= kb1) break;                          // the box's second K-block is past this tile's range
            const uint64_t adesc = sdesc_k_sw128(sA + stage * C::A_BYTES + hk * A_STAGE);
            // a box lands densely: its second K-block follows the first's n_tok / CTAS rows
            const uint64_t bdesc = sdesc_k_sw128(sB + stage * C::B_STAGE + hk * static_cast<uint32_t>(p.n_tok / CTAS) * BK * 2);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              // advance 16 fp16 = 32 bytes along K inside the swizzled row: +2 in the >>4 address field
              const uint32_t accum = (kb + hk > kb0 || k > 0) ? 1u : 0u;
              if constexpr (CTAS == 2)
                mma_f16_pair(tmem_d, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
              else
                mma_f16(tmem_d, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
            }
          }
          const uint32_t eb = smem_u32(&bars->empty[stage]);
          if constexpr (CTAS == 2) {
            mma_commit_pair(eb);                    // this CTA's producers
            mma_commit_pair(mapa_shared(eb, 1));    // the peer's producers
          } else {
            mma_commit(eb);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        const uint32_t fbar = smem_u32(&bars->tfull[acc]);
        if constexpr (CTAS == 2) {
          mma_commit_pair(fbar);
          mma_commit_pair(mapa_shared(fbar, 1));
        } else {
          mma_commit(fbar);
        }
      }
    }
  } else if (warp == IO_WARP) {
    // ------------------------------------------------------------ epilogue I/O (both CTAs)
    if (lane == 0 && p.fused) {
      const TileWalk walk{unit, units, total_tiles, static_cast<int>(rank), CTAS};
      epilogue_io<STAGES, HBUFS>(p, smem_u32(smem + C::OFF_H), bars, abort_flag, &tmap_h, &tmap_o, &tmap_o_head,
                                 walk);
    }
  } else if (warp >= R::EPI_WARP0 && warp < R::EPI_WARP0 + 4) {
    // ------------------------------------------------------------ epilogue arithmetic (four warps, both CTAs)
    const int et = threadIdx.x - 32 * R::EPI_WARP0;
    const TileWalk walk{unit, units, total_tiles, static_cast<int>(rank), CTAS};
    uint32_t q = 0;
    TokMeta mt_next[2];
    // metadata, gates, the state snapshot and the new history come from the
    // previous kernel; every output store happens after this wait
    pdl_wait();
    if (p.fused) load_meta(p, walk, 0, et, mt_next);
    int it = 0;
    bool ok = true;
    for (int tile = unit; tile < total_tiles && ok; tile += units, ++it) {
      int m, n, ks;
      tile_coords(p, tile, m, n, ks);
      const int acc = it & 1;
      ok = epilogue_tile<STAGES, HBUFS, R::EPI_WARP0>(p, smem, C::OFF_H, C::OFF_META, C::OFF_G, C::OFF_FLAGS, bars,
                                                      abort_flag, walk, it, ks,
                                                      tmem_base + static_cast<uint32_t>(acc * BN_MAX),
                                                      smem_u32(&bars->tfull[acc]), (it >> 1) & 1, q, mt_next);
      if (!ok) break;
      // the accumulator may be overwritten: tell the MMA issuer of the pair
      if constexpr (CTAS == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&bars->tempty[acc]), 0));
      else mbar_arrive(smem_u32(&bars->tempty[acc]));
      if (p.fused) named_bar_sync(1, EPI_THREADS);  // meta and flags are rewritten by the next tile
    }
  } else if constexpr (GATHER) {
    const uint32_t sL = smem_u32(smem + C::OFF_L);
    const uint32_t sS = smem_u32(smem + C::OFF_S);
    if (warp == LOADER_WARP) {
      // ------------------------------------------------------------ row loader (both CTAs)
      gather_loader<C>(p, sL, sS, bars, abort_flag, unit, units, total_tiles, rank);
    } else if (warp >= CONV_WARP0) {
      // ------------------------------------------------------------ converters (both CTAs)
      gather_converter<C>(p, sB, sL, sS, bars, abort_flag, unit, units, total_tiles, rank);
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (CTAS == 2) cluster_sync();     // neither CTA leaves while the pair still uses its memory
  if (warp == R::MMA_WARP) {
    tc_fence_after();
    if constexpr (CTAS == 2) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int CTAS, bool GATHER>
cudaError_t launch_gemm_impl(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const CUtensorMap& tmap_h,
                             const CUtensorMap& tmap_o, const CUtensorMap& tmap_o_head, const GemmParams& p, int grid,
                             cudaStream_t stream) {
  static PerDeviceOnce configured;
  const cudaError_t e = configured.run([] {
    const cudaError_t x = cudaFuncSetAttribute(gemm_kernel<CTAS, GATHER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kGemmSmemBytes);
    return x == cudaSuccess ? prefer_max_shared(gemm_kernel<CTAS, GATHER>) : x;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Roles<GATHER>::THREADS);
  // what the layout uses (plus the alignment slack), not the per-block maximum:
  // the few KB left let small kernels of another stream (the next batch's
  // ple_prepare_slot) share the SMs
  cfg.dynamicSmemBytes = Cfg<CTAS, GATHER>::SMEM_USED + 1024;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CTAS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the prologue, W_proj and h overlap the embed
  // kernel's tail (the kernel waits before it reads anything that kernel writes)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<CTAS, GATHER>, tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, p);
}

}  // namespace

bool gather_fused_supported(int32_t num_kb) { return 2 * num_kb > Cfg<2, true>::LSTAGES; }

cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const CUtensorMap& tmap_h,
                        const CUtensorMap& tmap_o, const CUtensorMap& tmap_o_head, const GemmParams& p, int grid,
                        int ctas, bool gather, cudaStream_t stream) {
  if (gather) {
    if (ctas != 2 || !p.fused || p.n_tok != BN_MAX || p.k_splits != 1 || !gather_fused_supported(p.num_kb))
      return cudaErrorInvalidValue;
    return launch_gemm_impl<2, true>(tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, p, grid, stream);
  }
  if (ctas == 2) return launch_gemm_impl<2, false>(tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, p, grid, stream);
  return launch_gemm_impl<1, false>(tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, p, grid, stream);
}

}  // namespace ple
