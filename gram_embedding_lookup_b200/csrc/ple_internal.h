// Host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "ple.h"

namespace ple {

struct TokMeta;

// Kernel attributes (such as the dynamic shared-memory limit) belong to the
// device that is current when they are set. PerDeviceOnce runs a setup once for
// every device a process uses (devices 0..63; others run it on every call).
class PerDeviceOnce {
 public:
  template <typename F>
  cudaError_t run(F&& setup) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t(1) << dev) : 0;
    if (bit != 0 && (done_.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = setup();
    if (e == cudaSuccess && bit != 0) done_.fetch_or(bit, std::memory_order_release);
    return e;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// Every kernel of the library asks for the largest shared-memory carveout, so
// that a kernel and its programmatic dependent (the projections take up to
// 227 KB of shared memory) can share an SM: an SM changes its L1/shared split
// only once it has drained.
template <typename Kernel>
cudaError_t prefer_max_shared(Kernel kernel) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              static_cast<int>(cudaSharedmemCarveoutMaxShared));
}

// The table as the kernels see it (ple_table_format in ple.h).
struct TableRef {
  const uint8_t* codes;        // E4M3: one byte per element; NVFP4: two E2M1 codes per byte
  const uint8_t* blocks;       // NVFP4: one E4M3 block scale per 16 elements; else null
  const float* scales;         // fp32 per row
  int32_t nvfp4;               // 1: PLE_TABLE_NVFP4 or PLE_TABLE_NVFP4_ROWS
  int32_t cs, bs;              // bytes from one row's codes (block scales) to the next row's
  int32_t nv_rows;             // 1: PLE_TABLE_NVFP4_ROWS (blocks = codes + D/2, one piece per row)
};

// Prepare stage: sequence map, n-gram row IDs, gate, state snapshot.
struct PrepareArgs {
  const int32_t* tokens;
  int32_t T;
  const int32_t* offsets;      // [S+1]; unused when uniform_q > 0
  int32_t S;
  int32_t uniform_q;           // > 0: sequence s covers tokens [s*q, (s+1)*q)
  const int32_t* hist;         // [S][2] or null
  int32_t vocab;
  int64_t rows0, rows1;
  uint64_t magic0, magic1;     // floor((2^64 - 1) / rows): set by the launchers
  int32_t* ids;                // [T][2]
  const __nv_bfloat16* hidden; // [T][H] (null: ids only)
  const __nv_bfloat16* w_gate; // [H]
  int32_t H;
  TokMeta* meta;               // [T] (null: ids only)
  const float* conv_in;        // [S][3][H] user state (null: none)
  float* conv_copy;            // [S][3][H] scratch snapshot of conv_in
  int32_t* hist_new;           // [S][2] state after each sequence (null: none)
  int32_t* status;
};
cudaError_t launch_prepare(const PrepareArgs& a, cudaStream_t stream);

// Prepare and gather fused (one pass over HBM): ids, metadata with the gate,
// and e[t] for the batch. num_sms sizes the persistent grid. With e null it
// writes only the ids and the metadata (the gather-fused projection follows).
cudaError_t launch_embed(const PrepareArgs& a, const TableRef& table, int32_t D, __half* e, int32_t num_sms,
                         cudaStream_t stream,
                         int* kernels = nullptr);

// The multi-head layout (PLE_TABLE_E4M3_HEADS): one warp per token computes the
// 16 head rows (ids [T][16]), the gate and metadata when a.meta is set, and
// e[t] (the 16 dequantised rows side by side) when e is set; extra blocks do
// the offsets check and the state work. a.rows0 is the rows per head sub-table.
cudaError_t launch_embed_heads(const PrepareArgs& a, const TableRef& table, int32_t D, __half* e, int32_t num_sms,
                               cudaStream_t stream, int* kernels = nullptr);

// Gather stage of the multi-head layout: ids [T][16] -> e [T][D].
cudaError_t launch_gather_heads(const int32_t* ids, int32_t T, const TableRef& table, int64_t rows, int32_t D,
                                __half* e, cudaStream_t stream);

// Failure-detection self-test: one bounded mbarrier wait that runs out after
// limit_cycles and records PLE_ERR_TIMEOUT in *status.
cudaError_t launch_wait_selftest(int32_t* status, long long limit_cycles, cudaStream_t stream);

// Gate of a prepared batch: meta[t].g from hidden (one warp per token), plus the
// conv-state snapshot when conv_in is set.
cudaError_t launch_gate(const PrepareArgs& a, cudaStream_t stream);

// Gather stage: e[t] = deq(row of order 0) + deq(row of order 1), fp16.
cudaError_t launch_gather(const int32_t* ids, int32_t T, const TableRef& table, int64_t rows0, int64_t rows1,
                          int32_t D, __half* e, bool reduce_ids, cudaStream_t stream);

// W_proj bf16 [D][H] -> fp16 [H][D]; *bad set to 1 when a value is outside the fp16 range.
cudaError_t launch_convert_w(const __nv_bfloat16* w, int32_t D, int32_t H, __half* w16, int32_t* bad,
                             cudaStream_t stream);

// Projection kernel (tcgen05).
struct GemmParams {
  int32_t T, H, D;
  int32_t n_tok;         // tokens per tile (MMA N): multiple of 16, <= 256
  int32_t tok_stride;    // token step between consecutive token tiles
  int32_t tok_origin;    // first token of tile 0 (negative: halo before token 0)
  int32_t halo;          // leading rows of a tile that are not output (fused mode)
  int32_t m_tiles, n_tiles, k_splits, num_kb;
  int32_t fused;         // 1: gate+conv+residual epilogue, 0: write fp32 partials
  const TokMeta* meta;
  const float* conv_w;
  const float* conv0;    // state snapshot [S][3][H] or null (fresh)
  float* conv_state;     // [S][3][H] written at each sequence's last token, or null
  int32_t* hist_state;   // [S][2] or null
  const int32_t* hist_new;
  void* out;
  int32_t out_f32;
  float* partial;        // [k_splits][T][H]
  int32_t* status;
  // gather-fused form only: the kernel builds the token operand itself from
  // the E4M3 table rows named by ids
  const int2* ids;       // [T] (row of order 0, row of order 1)
  const uint8_t* codes;  // [2][R][D]; order 1 starts at row rows0
  const float* scales;   // [2][R]
  int64_t rows0;
};
constexpr int kGemmSmemBytes = 227 * 1024;   // the sm_100 per-block maximum
// tmap_o / tmap_o_head: bf16 output tiles of 32 and of 29 tokens (the first
// chunk of a fused tile without its halo rows).
// ctas = 2: SM-pair tiles (clusters of two CTAs, 256 channels per tile, grid even,
// m_tiles = hidden / 256, tmap_e boxes of n_tok / 2 rows); ctas = 1: single-SM tiles.
// gather = true (ctas = 2, fused, n_tok = 256 only): the token operand is
// gathered and dequantised from the table inside the kernel (p.ids, p.codes,
// p.scales, p.rows0); tmap_e is not read.
cudaError_t launch_gemm(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const CUtensorMap& tmap_h,
                        const CUtensorMap& tmap_o, const CUtensorMap& tmap_o_head, const GemmParams& p, int grid,
                        int ctas, bool gather, cudaStream_t stream);
// Whether the gather-fused form takes rows of num_kb K-stages (64 codes each).
bool gather_fused_supported(int32_t num_kb);

// Combine split-K partials + gate + conv + residual (+ state) for a packed batch.
struct CombineArgs {
  int32_t T, H, k_splits;
  const float* partial;
  const TokMeta* meta;
  const __nv_bfloat16* hidden;
  const float* conv_w;
  const float* conv0;      // snapshot or null
  float* conv_state;       // null: no state
  int32_t* hist_state;
  const int32_t* hist_new;
  void* out;
  int32_t out_f32;
};
cudaError_t launch_combine_forward(const CombineArgs& a, cudaStream_t stream);

// Decode-step combine: B sequences of q tokens, commit the first n_commit[b].
struct DecodeCombineArgs {
  int32_t B, q, H, k_splits;
  const float* partial;
  const TokMeta* meta;
  const __nv_bfloat16* hidden;
  const float* conv_w;
  const int32_t* tokens;   // [B][q]
  int32_t* hist;           // [B][2] in/out
  float* conv_state;       // [B][3][H] in/out
  const int32_t* n_commit; // [B] or null
  void* out;
  int32_t out_f32;
  int32_t* status;
};
cudaError_t launch_combine_decode(const DecodeCombineArgs& a, cudaStream_t stream);

// Decode / speculative-verify steps: B sequences of q tokens (token t = b*q + i).
//
// decode_embed_kernel needs only the tokens and the token history: one block
// per token computes the token's n-gram rows and writes the dequantised rows to
// e[t] (fp16 [T][D]) and the token's metadata (sequence b, position i, last
// flag); with hidden set it also writes the gate meta[t].g (through gate_warp).
struct DecodeEmbedArgs {
  const int32_t* tokens;   // [B][q]
  int32_t B, q;
  const int32_t* hist;     // [B][2]: token t-2, t-1 before the step; < 0 = absent
  int32_t vocab;
  int64_t rows0, rows1;    // rows per sub-table (E4M3_HEADS: rows0 per head)
  uint64_t magic0, magic1; // barrett_magic(rows0), barrett_magic(rows1)
  const uint8_t* table;
  const uint8_t* blocks;   // NVFP4 block scales (null otherwise)
  const float* scales;
  int32_t cs, bs;          // row strides in bytes of the codes and the block scales (TableRef)
  int32_t format;          // ple_table_format (PLE_TABLE_NVFP4 for both NVFP4 layouts)
  int32_t D, H;
  const __nv_bfloat16* hidden;   // [T][H], or null: the gate is computed later
  const __nv_bfloat16* w_gate;
  __half* e;               // [T][D]; with codes2, [16][D]: token t's two rows as exact fp16 codes in rows t and t + 8
  float* row_scales;       // with codes2: [T][2], the two rows' scales
  int32_t codes2;          // 1: e takes the codes and row_scales the scales (decode_two_order steps)
  TokMeta* meta;           // [T]
  const __half* w16;       // fp16 W_proj, prefetched into L2 for the kernel after this one (null: none)
  int64_t w16_bytes;
  int32_t prefetch_blocks; // the grid has at least this many blocks (past T: prefetch only)
  int32_t* status;
};
cudaError_t launch_decode_embed(const DecodeEmbedArgs& a, cudaStream_t stream);
uint64_t barrett_magic(int64_t m);
// Steps of up to 8 tokens of a two-order table (E4M3 or NVFP4) run the
// channel-split kernel on exact codes with the row scales after the products.
bool decode_two_order(int32_t T, int32_t format);

// decode_proj_kernel, for steps of B * q <= 16 tokens: the projection, gate,
// conv against the carried state, residual and state commit, one CTA per SM.
// CTA b owns a contiguous range of 8-channel groups with the whole K, so no
// partial sums cross CTAs and no CTA waits for another. With e null the
// kernel also computes the row IDs and gathers, in each warp, the K range of
// every token's rows that the warp multiplies (the whole step in one kernel);
// otherwise it reads what decode_embed_kernel wrote: the rows, or for
// decode_two_order steps the codes and row scales. Up to 8 tokens of a
// two-order table run as 16 mma rows of exact codes (order 0 and order 1 of
// each token) with the row scales applied after the products.
struct DecodeProjArgs {
  const int32_t* tokens;   // [B][q] (the rows of a fused step, and the new token history)
  int32_t B, q;
  int32_t* hist;           // [B][2] in/out
  float* conv_state;       // [B][3][H] in/out
  const int32_t* n_commit; // [B] or null
  const __half* w16;       // fp16 W_proj [H][D] (K-major)
  const __half* e;         // from decode_embed_kernel ([T][D] rows, or [16][D] codes), or null: the kernel
                           // gathers the rows itself
  const float* row_scales; // [T][2] from decode_embed_kernel (with e, decode_two_order steps)
  const TokMeta* meta;     // [T]
  int32_t gate_ready;      // 1: meta[t].g holds the gate; 0: each CTA computes it from hidden
  // the table, for a step whose rows the kernel gathers itself (e null)
  int32_t vocab;
  int64_t rows0, rows1;
  uint64_t magic0, magic1;
  const uint8_t* table;
  const uint8_t* blocks;
  const float* scales;
  int32_t cs, bs;          // row strides in bytes of the codes and the block scales (TableRef)
  int32_t format;          // ple_table_format (PLE_TABLE_NVFP4 for both NVFP4 layouts)
  int32_t* step_count;     // fused steps: CTAs past their hashing, zero between launches
  const __nv_bfloat16* hidden;
  const __nv_bfloat16* w_gate;
  const float* conv_w;
  void* out;
  int32_t out_f32;
  int32_t H, D;
  int32_t max_groups;      // DecodeProjPlan::max_groups
  int32_t* status;
};
struct DecodeProjPlan {
  int32_t grid;            // CTAs (at most one per SM)
  int32_t max_groups;      // most 8-channel groups one CTA owns
};
// False when the layer shape does not fit the kernel (steps then run split-K).
bool decode_proj_plan(int32_t H, int32_t D, int32_t num_sms, DecodeProjPlan* plan);
bool decode_proj_supported(int32_t B, int32_t q);
cudaError_t launch_decode_proj(const DecodeProjArgs& a, const DecodeProjPlan& plan, cudaStream_t stream);

// mtp_proj_kernel, for steps of 17..kMtpMaxTokens tokens after
// decode_embed_kernel (gates in meta): a split-K tcgen05 projection whose
// K-split CTAs meet at a per-tile counter, then each adds the splits' sums in
// order for its share of the sequences and runs gate, conv, residual and state
// commit. Its CTAs wait for one another, so the grid (m_tiles * k_splits) never
// exceeds the SM count.
constexpr int kMtpMaxTokens = 256;
constexpr int kMtpMaxQ = 16;       // tokens per sequence: a chunk of whole sequences fits the staging area
constexpr int kMtpMaxSplits = 8;
struct MtpPlan {
  int32_t m_tiles;         // hidden / 128
  int32_t k_splits;        // CTAs per channel tile
  int32_t num_kb;          // row_dim / 64
};
struct MtpProjArgs {
  const int32_t* tokens;   // [B][q]
  int32_t B, q;
  int32_t* hist;           // [B][2] in/out
  float* conv_state;       // [B][3][H] in/out
  const int32_t* n_commit; // [B] or null
  const TokMeta* meta;     // [T]: gates
  const __nv_bfloat16* hidden;
  const float* conv_w;
  void* out;
  int32_t out_f32;
  int32_t H;
  int32_t m_tiles, k_splits, num_kb;
  int32_t n_pad;           // T rounded up to 16 (the MMA's N)
  int32_t stages;          // set by the launcher
  float* partial;          // [m_tiles][k_splits][kMtpMaxTokens][128]
  int32_t* tile_count;     // [m_tiles], zero between launches
  int32_t* tile_done;      // [m_tiles], zero between launches
  int32_t* status;
};
bool mtp_proj_plan(int32_t H, int32_t D, int32_t num_sms, MtpPlan* plan);
int64_t mtp_partial_elems(const MtpPlan& plan);
// tmap_w: fp16 W_proj [H][D], box 64 x 128, 128-byte swizzle; tmap_e: fp16 e
// [T][D], box 64 x n_pad, 128-byte swizzle.
cudaError_t launch_mtp_proj(const CUtensorMap& tmap_w, const CUtensorMap& tmap_e, const MtpProjArgs& a,
                            cudaStream_t stream);

}  // namespace ple
