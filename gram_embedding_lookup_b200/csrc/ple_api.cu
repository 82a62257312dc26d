// The C ABI of libple: handle life cycle, host-side argument checks, launch
// planning and per-stage timing. Every step of the layer runs in the kernels
// of ple_kernels.cu and ple_gemm.cu; nothing here computes on the host.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <new>
#include <vector>

#include "ple.h"
#include "ple_device.cuh"
#include "ple_internal.h"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

constexpr int kTileM = 128;       // channels per projection tile
constexpr int kTileK = 64;        // K per pipeline stage
constexpr int kFusedRows = 256;   // token rows of a fused tile
constexpr int kHalo = 3;          // conv taps before the current token

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

struct Plan {
  bool fused;
  int n_tok, tok_stride, tok_origin, halo, n_tiles, k_splits;
  int ctas;   // 2: SM-pair tiles of 256 channels; 1: single-SM tiles of 128
};

}  // namespace

struct ple_handle {
  ple_config cfg{};
  ple_weights w{};
  int device = 0;
  int num_sms = 148;
  __half* w16 = nullptr;
  // the batch scratch (rows, IDs, metadata, new history): set 0 serves
  // ple_forward, the decode steps and prepare slot 0; set 1 (with
  // prepare_slots == 2) only prepare slot 1
  struct Scratch {
    __half* e = nullptr;
    int32_t* ids = nullptr;
    ple::TokMeta* meta = nullptr;
    int32_t* hist_new = nullptr;
    float* row_scales = nullptr;   // decode steps of up to 8 tokens: [T][2] the two rows' scales
  } scratch[2];
  __half*& e = scratch[0].e;
  int32_t*& ids = scratch[0].ids;
  ple::TokMeta*& meta = scratch[0].meta;
  int32_t*& hist_new = scratch[0].hist_new;
  float* partial = nullptr;
  int64_t partial_elems = 0;
  float* conv0 = nullptr;
  int32_t* status = nullptr;     // [0]: sticky status
  bool decode_proj = false;      // the channel-split decode projection fits this shape and device
  ple::DecodeProjPlan decode_plan{};
  bool mtp = false;              // the split-K decode projection with in-kernel sums fits
  ple::MtpPlan mtp_plan{};
  float* mtp_partial = nullptr;  // its split sums
  int32_t* mtp_counts = nullptr; // its per-tile counters [2][m_tiles], zero between launches
  EncodeTiledFn encode = nullptr;
  CUtensorMap tmap_w{};          // fp16 W_proj, boxes of 64 K x 128 channels
  CUtensorMap tmap_w_kb2{};      // the same as 3-D boxes of two K-blocks (the SM-pair projection)
  int32_t forward_path = 0;
  struct Prepared {        // the batch ple_prepare left in a scratch set (ids, e, meta, hist_new)
    bool valid = false;
    int32_t T = 0, S = 0;
    bool with_hist = false;
  } prepared_slot[2];
  Prepared& prepared = prepared_slot[0];
  struct PreparedDecode {  // the step ple_decode_prepare left in the scratch (e, meta)
    bool valid = false;
    int32_t B = 0, q = 0;
    const int32_t* tokens = nullptr;
    const int32_t* hist = nullptr;
    bool small = false;    // the channel-split kernel takes the step (chosen when prepared)
  } prepared_decode;
  bool profiling = false;
  struct Rec { int stage; cudaEvent_t a, b; };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> free_events;
  double stage_ms[PLE_NUM_STAGES] = {0, 0, 0, 0};
  int64_t stage_launches[PLE_NUM_STAGES] = {0, 0, 0, 0};
  int64_t launches = 0;
};

namespace {

Plan plan_projection(const ple_handle* h, int T, int path, int64_t partial_cap) {
  const int m_tiles = h->cfg.hidden / kTileM;
  const int num_kb = h->cfg.row_dim / kTileK;
  const int fused_tiles_n = ceil_div(T, kFusedRows - kHalo);
  bool fused = (path == 1 || path == 3 || path == 4) ||
               (path == 0 && static_cast<int64_t>(m_tiles) * fused_tiles_n >= h->num_sms);
  if (!fused) {
    const int n_tok = std::min(256, ceil_div(T, 16) * 16);
    const int n_tiles = ceil_div(T, n_tok);
    const int tiles = m_tiles * n_tiles;
    int ks = std::max(1, std::min(h->num_sms / std::max(tiles, 1), std::min(num_kb, 16)));
    while (ks > 1 && static_cast<int64_t>(ks) * T * h->cfg.hidden > partial_cap) --ks;
    if (static_cast<int64_t>(T) * h->cfg.hidden <= partial_cap)
      return Plan{false, n_tok, n_tok, 0, 0, n_tiles, ks, 1};
    fused = true;   // no room for partials: fall back to the fused path
  }
  const int ctas = (path != 3 && h->cfg.hidden % (2 * kTileM) == 0 && h->num_sms >= 2) ? 2 : 1;
  return Plan{true, kFusedRows, kFusedRows - kHalo, -kHalo, kHalo, fused_tiles_n, 1, ctas};
}

// Whether ple_forward on T tokens runs the gather-fused projection (the token
// operand gathered from the table inside the projection kernel, never written
// to HBM): path 4, E4M3 tables, SM-pair tiles. It is not the automatic choice:
// the kernel dequantises each token's rows once per 256-channel tile (ten
// times at hidden 2560) inside the tensor-bound kernel, and measures slower
// than the embed kernel followed by the TMA-fed projection.
bool gather_fused(const ple_handle* h, int T) {
  if (h->forward_path != 4 || h->cfg.table_format != PLE_TABLE_E4M3) return false;
  if (h->cfg.rows[0] + h->cfg.rows[1] >= (int64_t(1) << 31)) return false;   // rows are int32 in the kernel
  if (!ple::gather_fused_supported(h->cfg.row_dim / kTileK)) return false;
  const Plan pl = plan_projection(h, T, 4, h->partial_elems);
  return pl.fused && pl.ctas == 2;
}

cudaEvent_t take_event(ple_handle* h) {
  if (!h->free_events.empty()) {
    cudaEvent_t e = h->free_events.back();
    h->free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

template <class F>
ple_status run_stage(ple_handle* h, int stage, cudaStream_t s, F&& launch) {
  cudaEvent_t a = nullptr, b = nullptr;
  if (h->profiling) {
    a = take_event(h);
    b = take_event(h);
    cudaEventRecord(a, s);
  }
  const cudaError_t err = launch();
  if (err != cudaSuccess) return PLE_ERR_CUDA;
  ++h->launches;
  if (h->profiling) {
    cudaEventRecord(b, s);
    h->pending.push_back({stage, a, b});
  }
  return PLE_OK;
}

bool encode_2d(ple_handle* h, CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = h->encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// A K-major fp16 operand [outer][K] as a 3-D tensor {64 elements, outer, K / 64}
// (a row's K-blocks 128 bytes apart), boxes of {64, box_outer, 2}: two K-blocks
// per copy, each landing as its own 128-byte-swizzled tile.
bool encode_kb2(ple_handle* h, CUtensorMap* map, const void* base, uint64_t K, uint64_t outer, uint32_t box_outer) {
  const cuuint64_t dims[3] = {64, outer, K / 64};
  const cuuint64_t strides[2] = {K * 2, 128};
  const cuuint32_t box[3] = {64, box_outer, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = h->encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// True when the current device is not the handle's (its memory and kernels live there).
bool wrong_device(const ple_handle* h) {
  int dev = -1;
  return cudaGetDevice(&dev) != cudaSuccess || dev != h->device;
}

bool heads_layout(const ple_handle* h) { return h->cfg.table_format == PLE_TABLE_E4M3_HEADS; }
int ids_per_token(const ple_config& c) { return c.table_format == PLE_TABLE_E4M3_HEADS ? 16 : 2; }

// The kernels computing the row IDs (and, as the arguments ask, gate, metadata,
// state and e) for the handle's table layout.
cudaError_t launch_embed_for(ple_handle* h, const ple::PrepareArgs& pa, __half* e, cudaStream_t stream);

// The format the kernels see: both NVFP4 layouts are PLE_TABLE_NVFP4 there,
// told apart by the row strides of TableRef.
int32_t kernel_format(const ple_config& c) {
  return c.table_format == PLE_TABLE_NVFP4_ROWS ? static_cast<int32_t>(PLE_TABLE_NVFP4) : c.table_format;
}

ple::TableRef table_ref(const ple_handle* h) {
  const ple_config& c = h->cfg;
  const int32_t D = c.row_dim;
  ple::TableRef t{h->w.table, nullptr, h->w.scales, 0, D, 0, 0};
  if (c.table_format == PLE_TABLE_NVFP4) {
    t.blocks = h->w.block_scales;
    t.nvfp4 = 1;
    t.cs = D / 2;
    t.bs = D / 16;
  } else if (c.table_format == PLE_TABLE_NVFP4_ROWS) {
    t.blocks = h->w.table + D / 2;                      // each row's block scales follow its codes
    t.nvfp4 = 1;
    t.cs = t.bs = D / 2 + D / 16;
    t.nv_rows = 1;
  }
  return t;
}

cudaError_t launch_embed_for(ple_handle* h, const ple::PrepareArgs& pa, __half* e, cudaStream_t stream) {
  int kernels = 1;
  const cudaError_t r = heads_layout(h)
                            ? ple::launch_embed_heads(pa, table_ref(h), h->cfg.row_dim, e, h->num_sms, stream, &kernels)
                            : ple::launch_embed(pa, table_ref(h), h->cfg.row_dim, e, h->num_sms, stream, &kernels);
  h->launches += kernels - 1;           // the stage counts one launch; large batches take two kernels
  return r;
}

void free_all(ple_handle* h) {
  cudaFree(h->w16);
  for (auto& sc : h->scratch) {
    cudaFree(sc.e);
    cudaFree(sc.ids);
    cudaFree(sc.meta);
    cudaFree(sc.hist_new);
    cudaFree(sc.row_scales);
  }
  cudaFree(h->partial);
  cudaFree(h->conv0);
  cudaFree(h->status);
  cudaFree(h->mtp_partial);
  cudaFree(h->mtp_counts);
  for (auto& r : h->pending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->free_events) cudaEventDestroy(e);
}

ple_status run_projection(ple_handle* h, const ple_handle::Scratch& sc, int32_t T, int32_t S, int32_t uniform_q,
                          const void* hidden, void* out, ple_out_dtype dtype, const ple_state* state, int32_t* dec_hist,
                          float* dec_conv, const int32_t* tokens, const int32_t* n_commit, bool gather,
                          cudaStream_t stream);

// Runs prepare + gather + projection (+ combine) for a packed batch.
ple_status run_layer(ple_handle* h, const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                     const void* hidden, void* out, ple_out_dtype dtype, const ple_state* state, cudaStream_t stream) {
  const ple_config& c = h->cfg;
  ple::PrepareArgs pa{};
  pa.tokens = tokens;
  pa.T = T;
  pa.offsets = offsets;
  pa.S = S;
  pa.hist = state ? state->hist : nullptr;
  pa.vocab = c.vocab;
  pa.rows0 = c.rows[0];
  pa.rows1 = c.rows[1];
  pa.ids = h->ids;
  pa.hidden = static_cast<const __nv_bfloat16*>(hidden);
  pa.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
  pa.H = c.hidden;
  pa.meta = h->meta;
  if (state != nullptr) {
    pa.conv_in = state->conv;
    pa.conv_copy = h->conv0;
    pa.hist_new = h->hist_new;
  }
  pa.status = h->status;
  // row IDs, gate and the gathered, dequantised rows in one kernel; for the
  // gather-fused projection, IDs and gate only
  const bool gather = gather_fused(h, T);
  h->prepared.valid = false;            // the scratch now holds this call's batch
  h->prepared_decode.valid = false;
  const ple_status st = run_stage(h, PLE_STAGE_PREPARE, stream, [&] {
    return launch_embed_for(h, pa, gather ? nullptr : h->e, stream);
  });
  if (st != PLE_OK) return st;
  return run_projection(h, h->scratch[0], T, S, 0, hidden, out, dtype, state, nullptr, nullptr, nullptr, nullptr, gather,
                        stream);
}

// The projection and everything after it, on the rows, IDs and metadata in the
// handle's scratch (written by the embed kernel, or by ple_prepare plus the gate
// kernel). gather: the rows are not in the scratch; the projection gathers them
// from the table by the IDs.
ple_status run_projection(ple_handle* h, const ple_handle::Scratch& sc, int32_t T, int32_t S, int32_t uniform_q,
                          const void* hidden, void* out, ple_out_dtype dtype, const ple_state* state, int32_t* dec_hist,
                          float* dec_conv, const int32_t* tokens, const int32_t* n_commit, bool gather,
                          cudaStream_t stream) {
  const ple_config& c = h->cfg;
  const bool decode = uniform_q > 0;
  const Plan pl = plan_projection(h, T, decode ? 2 : (gather ? 4 : h->forward_path), h->partial_elems);
  if (gather && !(pl.fused && pl.ctas == 2)) return PLE_ERR_UNSUPPORTED;
  ple_status st = PLE_OK;
  CUtensorMap tmap_e{}, tmap_h{}, tmap_o{}, tmap_o_head{};
  const bool kb2 = pl.ctas == 2 && !gather;     // the SM-pair projection takes two K-blocks per copy
  if (kb2 ? !encode_kb2(h, &tmap_e, sc.e, c.row_dim, T, pl.n_tok / pl.ctas)
          : !encode_2d(h, &tmap_e, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, sc.e, c.row_dim, T,
                       static_cast<uint64_t>(c.row_dim) * 2, kTileK, pl.n_tok / pl.ctas, CU_TENSOR_MAP_SWIZZLE_128B))
    return PLE_ERR_CUDA;
  if (!encode_2d(h, &tmap_h, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, hidden, c.hidden, T,
                 static_cast<uint64_t>(c.hidden) * 2, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_NONE))
    return PLE_ERR_CUDA;

  if (pl.fused && dtype == PLE_OUT_BF16) {
    if (!encode_2d(h, &tmap_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, c.hidden, T,
                   static_cast<uint64_t>(c.hidden) * 2, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_2d(h, &tmap_o_head, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, c.hidden, T,
                   static_cast<uint64_t>(c.hidden) * 2, kTileM, 32 - kHalo, CU_TENSOR_MAP_SWIZZLE_NONE))
      return PLE_ERR_CUDA;
  }

  ple::GemmParams gp{};
  gp.T = T;
  gp.H = c.hidden;
  gp.D = c.row_dim;
  gp.n_tok = pl.n_tok;
  gp.tok_stride = pl.tok_stride;
  gp.tok_origin = pl.tok_origin;
  gp.halo = pl.halo;
  gp.m_tiles = c.hidden / (kTileM * pl.ctas);
  gp.n_tiles = pl.n_tiles;
  gp.k_splits = pl.k_splits;
  gp.num_kb = c.row_dim / kTileK;
  gp.fused = pl.fused ? 1 : 0;
  gp.meta = sc.meta;
  gp.conv_w = h->w.conv_w;
  gp.conv0 = (!decode && state) ? h->conv0 : nullptr;
  gp.conv_state = (!decode && state) ? state->conv : nullptr;
  gp.hist_state = (!decode && state) ? state->hist : nullptr;
  gp.hist_new = sc.hist_new;
  gp.out = out;
  gp.out_f32 = dtype == PLE_OUT_F32 ? 1 : 0;
  gp.partial = h->partial;
  gp.status = h->status;
  if (gather) {
    gp.ids = reinterpret_cast<const int2*>(sc.ids);
    gp.codes = h->w.table;
    gp.scales = h->w.scales;
    gp.rows0 = c.rows[0];
  }
  const int total = gp.m_tiles * gp.n_tiles * gp.k_splits;
  const int grid = pl.ctas == 2 ? 2 * std::min(total, h->num_sms / 2) : std::min(total, h->num_sms);
  st = run_stage(h, PLE_STAGE_GEMM, stream, [&] {
    return ple::launch_gemm(kb2 ? h->tmap_w_kb2 : h->tmap_w, tmap_e, tmap_h, tmap_o, tmap_o_head, gp, grid, pl.ctas,
                            gather, stream);
  });
  if (st != PLE_OK || pl.fused) return st;

  if (decode) {
    ple::DecodeCombineArgs da{};
    da.B = S;
    da.q = uniform_q;
    da.H = c.hidden;
    da.k_splits = pl.k_splits;
    da.partial = h->partial;
    da.meta = sc.meta;
    da.hidden = static_cast<const __nv_bfloat16*>(hidden);
    da.conv_w = h->w.conv_w;
    da.tokens = tokens;
    da.hist = dec_hist;
    da.conv_state = dec_conv;
    da.n_commit = n_commit;
    da.out = out;
    da.out_f32 = gp.out_f32;
    da.status = h->status;
    return run_stage(h, PLE_STAGE_COMBINE, stream, [&] { return ple::launch_combine_decode(da, stream); });
  }
  ple::CombineArgs ca{};
  ca.T = T;
  ca.H = c.hidden;
  ca.k_splits = pl.k_splits;
  ca.partial = h->partial;
  ca.meta = sc.meta;
  ca.hidden = static_cast<const __nv_bfloat16*>(hidden);
  ca.conv_w = h->w.conv_w;
  ca.conv0 = gp.conv0;
  ca.conv_state = gp.conv_state;
  ca.hist_state = gp.hist_state;
  ca.hist_new = sc.hist_new;
  ca.out = out;
  ca.out_f32 = gp.out_f32;
  return run_stage(h, PLE_STAGE_COMBINE, stream, [&] { return ple::launch_combine_forward(ca, stream); });
}

// Whether the channel-split kernel takes a decode step of B x q tokens.
bool decode_small(const ple_handle* h, int32_t B, int32_t q) {
  return h->forward_path != 2 && h->decode_proj && ple::decode_proj_supported(B, q);
}

// The tokens-only half of a decode step: rows into h->e (for a step the
// channel-split kernel takes on exact codes, the codes and row scales),
// metadata into h->meta, and the gates when hidden is given.
ple_status run_decode_embed(ple_handle* h, const int32_t* tokens, int32_t B, int32_t q, const int32_t* hist,
                            const void* hidden, bool small, cudaStream_t stream) {
  const ple_config& c = h->cfg;
  ple::DecodeEmbedArgs a{};
  a.tokens = tokens;
  a.B = B;
  a.q = q;
  a.hist = hist;
  a.vocab = c.vocab;
  a.rows0 = c.rows[0];
  a.rows1 = c.rows[1];
  a.magic0 = ple::barrett_magic(c.rows[0]);
  a.magic1 = ple::barrett_magic(c.rows[1]);
  const ple::TableRef tab = table_ref(h);
  a.table = tab.codes;
  a.blocks = tab.blocks;
  a.cs = tab.cs;
  a.bs = tab.bs;
  a.scales = h->w.scales;
  a.format = kernel_format(c);
  a.D = c.row_dim;
  a.H = c.hidden;
  a.hidden = static_cast<const __nv_bfloat16*>(hidden);
  a.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
  a.e = h->e;
  a.row_scales = h->scratch[0].row_scales;
  a.codes2 = small && ple::decode_two_order(B * q, kernel_format(c)) ? 1 : 0;
  a.meta = h->meta;
  a.w16 = h->w16;
  a.w16_bytes = static_cast<int64_t>(c.hidden) * c.row_dim * 2;
  a.prefetch_blocks = h->num_sms;
  a.status = h->status;
  return run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return ple::launch_decode_embed(a, stream); });
}

ple::DecodeProjArgs decode_proj_args(const ple_handle* h, const int32_t* tokens, int32_t B, int32_t q,
                                     const void* hidden, void* out, ple_out_dtype dtype, int32_t* hist,
                                     float* conv_state, const int32_t* n_commit);

// The hidden-dependent half of a decode step whose rows and metadata are in the
// scratch: the channel-split projection kernel for steps of up to 16 tokens
// (unless path 2 forces split-K), else the split-K projection and the decode
// combine. Without gates in the metadata, a gate kernel writes them first when
// the kernels after it cannot compute them (split-K, or out aliasing hidden).
ple_status run_decode_rest(ple_handle* h, const int32_t* tokens, int32_t B, int32_t q, const void* hidden, void* out,
                           ple_out_dtype dtype, int32_t* hist, float* conv_state, const int32_t* n_commit,
                           bool gate_ready, bool small, cudaStream_t stream) {
  const ple_config& c = h->cfg;
  const int32_t T = B * q;
  if (!gate_ready && (!small || out == hidden)) {
    ple::PrepareArgs ga{};
    ga.T = T;
    ga.S = B;
    ga.hidden = static_cast<const __nv_bfloat16*>(hidden);
    ga.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
    ga.H = c.hidden;
    ga.meta = h->meta;
    const ple_status st = run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return ple::launch_gate(ga, stream); });
    if (st != PLE_OK) return st;
    gate_ready = true;
  }
  if (!small && h->forward_path != 2 && h->mtp && T <= ple::kMtpMaxTokens && q <= ple::kMtpMaxQ) {
    const int n_pad = (T + 15) / 16 * 16;
    CUtensorMap tmap_e{};
    if (!encode_kb2(h, &tmap_e, h->e, c.row_dim, T, n_pad)) return PLE_ERR_CUDA;   // two K-blocks per copy
    ple::MtpProjArgs a{};
    a.tokens = tokens;
    a.B = B;
    a.q = q;
    a.hist = hist;
    a.conv_state = conv_state;
    a.n_commit = n_commit;
    a.meta = h->meta;
    a.hidden = static_cast<const __nv_bfloat16*>(hidden);
    a.conv_w = h->w.conv_w;
    a.out = out;
    a.out_f32 = dtype == PLE_OUT_F32 ? 1 : 0;
    a.H = c.hidden;
    a.m_tiles = h->mtp_plan.m_tiles;
    a.k_splits = h->mtp_plan.k_splits;
    a.num_kb = h->mtp_plan.num_kb;
    a.n_pad = n_pad;
    a.partial = h->mtp_partial;
    a.tile_count = h->mtp_counts;
    a.tile_done = h->mtp_counts + h->mtp_plan.m_tiles;
    a.status = h->status;
    return run_stage(h, PLE_STAGE_GEMM, stream, [&] { return ple::launch_mtp_proj(h->tmap_w_kb2, tmap_e, a, stream); });
  }
  if (!small)
    return run_projection(h, h->scratch[0], T, B, q, hidden, out, dtype, nullptr, hist, conv_state, tokens, n_commit,
                          false, stream);
  ple::DecodeProjArgs a = decode_proj_args(h, tokens, B, q, hidden, out, dtype, hist, conv_state, n_commit);
  a.e = h->e;
  a.row_scales = h->scratch[0].row_scales;
  a.meta = h->meta;
  a.gate_ready = gate_ready ? 1 : 0;
  return run_stage(h, PLE_STAGE_GEMM, stream, [&] { return ple::launch_decode_proj(a, h->decode_plan, stream); });
}

// The arguments of the channel-split decode kernel common to its two forms.
ple::DecodeProjArgs decode_proj_args(const ple_handle* h, const int32_t* tokens, int32_t B, int32_t q,
                                     const void* hidden, void* out, ple_out_dtype dtype, int32_t* hist,
                                     float* conv_state, const int32_t* n_commit) {
  const ple_config& c = h->cfg;
  ple::DecodeProjArgs a{};
  a.tokens = tokens;
  a.B = B;
  a.q = q;
  a.hist = hist;
  a.conv_state = conv_state;
  a.n_commit = n_commit;
  a.w16 = h->w16;
  a.hidden = static_cast<const __nv_bfloat16*>(hidden);
  a.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
  a.conv_w = h->w.conv_w;
  a.out = out;
  a.out_f32 = dtype == PLE_OUT_F32 ? 1 : 0;
  a.H = c.hidden;
  a.D = c.row_dim;
  a.vocab = c.vocab;
  a.rows0 = c.rows[0];
  a.rows1 = c.rows[1];
  a.magic0 = ple::barrett_magic(c.rows[0]);
  a.magic1 = ple::barrett_magic(c.rows[1]);
  const ple::TableRef tab = table_ref(h);
  a.table = tab.codes;
  a.blocks = tab.blocks;
  a.cs = tab.cs;
  a.bs = tab.bs;
  a.scales = h->w.scales;
  a.format = kernel_format(c);
  a.step_count = h->status + 1;
  a.status = h->status;
  return a;
}

// Host checks shared by the decode entry points.
ple_status check_decode_step(const ple_handle* h, int32_t B, int32_t q, const void* hidden, void* out,
                             ple_out_dtype out_dtype, const int32_t* hist, const float* conv_state,
                             const int32_t* n_commit) {
  if (out_dtype != PLE_OUT_BF16 && out_dtype != PLE_OUT_F32) return PLE_ERR_INVALID_ARG;
  if (B < 1 || q < 1 || B > h->cfg.max_seqs || static_cast<int64_t>(B) * q > h->cfg.max_tokens) return PLE_ERR_SHAPE;
  if (hidden == nullptr || out == nullptr || hist == nullptr || conv_state == nullptr) return PLE_ERR_INVALID_ARG;
  if (out == hidden && out_dtype != PLE_OUT_BF16) return PLE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(out, 16) || !aligned(hist, 4) || !aligned(conv_state, 16) ||
      (n_commit && !aligned(n_commit, 4)))
    return PLE_ERR_ALIGN;
  return PLE_OK;
}

}  // namespace

extern "C" {

const char* ple_status_string(ple_status s) {
  switch (s) {
    case PLE_OK: return "ok";
    case PLE_ERR_INVALID_ARG: return "invalid argument";
    case PLE_ERR_SHAPE: return "size outside the handle's configuration";
    case PLE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PLE_ERR_RANGE: return "token outside [0, vocab) or inconsistent offsets / n_commit";
    case PLE_ERR_OOM: return "device allocation failed";
    case PLE_ERR_CUDA: return "CUDA runtime error";
    case PLE_ERR_TIMEOUT: return "a bounded device wait ran out";
    case PLE_ERR_UNSUPPORTED: return "unsupported configuration";
  }
  return "unknown status";
}

ple_status ple_create(const ple_config* config, const ple_weights* weights, cudaStream_t stream, ple_handle** out) {
  if (config == nullptr || weights == nullptr || out == nullptr) return PLE_ERR_INVALID_ARG;
  *out = nullptr;
  const ple_config& c = *config;
  if ((c.table_format != PLE_TABLE_E4M3 && c.table_format != PLE_TABLE_NVFP4 &&
       c.table_format != PLE_TABLE_E4M3_HEADS && c.table_format != PLE_TABLE_NVFP4_ROWS) ||
      c.vocab <= 0 || c.hidden <= 0 || c.row_dim <= 0 || c.max_tokens <= 0 || c.max_seqs <= 0)
    return PLE_ERR_INVALID_ARG;
  if (c.prepare_slots < 0 || c.prepare_slots > 2) return PLE_ERR_INVALID_ARG;
  if (c.hidden % 128 != 0 || c.row_dim % 64 != 0) return PLE_ERR_UNSUPPORTED;
  if (c.table_format == PLE_TABLE_E4M3_HEADS) {
    // 16 head rows of row_dim / 16 codes, a whole number of 16-byte chunks each
    if (c.row_dim % 256 != 0) return PLE_ERR_UNSUPPORTED;
    if (c.rows[1] != c.rows[0]) return PLE_ERR_INVALID_ARG;
  }
  // rows of row_dim * 9/16 bytes: every row starts on a 16-byte boundary
  if (c.table_format == PLE_TABLE_NVFP4_ROWS && c.row_dim % 256 != 0) return PLE_ERR_UNSUPPORTED;
  for (int n = 0; n < 2; ++n)
    if (c.rows[n] <= 0 || c.rows[n] >= (int64_t(1) << 31)) return PLE_ERR_INVALID_ARG;
  if (weights->table == nullptr || weights->scales == nullptr || weights->w_proj == nullptr ||
      weights->w_gate == nullptr || weights->conv_w == nullptr)
    return PLE_ERR_INVALID_ARG;
  if (c.table_format == PLE_TABLE_NVFP4 && weights->block_scales == nullptr) return PLE_ERR_INVALID_ARG;
  if (c.table_format == PLE_TABLE_NVFP4_ROWS && weights->block_scales != nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(weights->table, 16) || !aligned(weights->w_proj, 16) || !aligned(weights->w_gate, 16) ||
      !aligned(weights->conv_w, 16) || !aligned(weights->scales, 4) ||
      (c.table_format == PLE_TABLE_NVFP4 && !aligned(weights->block_scales, 16)))
    return PLE_ERR_ALIGN;

  ple_handle* h = new (std::nothrow) ple_handle();
  if (h == nullptr) return PLE_ERR_OOM;
  h->cfg = c;
  h->w = *weights;
  cudaGetDevice(&h->device);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);

  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    delete h;
    return PLE_ERR_CUDA;
  }
  h->encode = reinterpret_cast<EncodeTiledFn>(fn);

  // partial-sum capacity: whatever the automatic plan needs up to max_tokens, and
  // at least one split of min(max_tokens, 4096) tokens (forced split-K path)
  int64_t cap = static_cast<int64_t>(std::min(c.max_tokens, 4096)) * c.hidden;
  for (int T = 1; T <= c.max_tokens; ++T) {
    const Plan p = plan_projection(h, T, 0, INT64_MAX);
    if (p.fused) continue;
    cap = std::max(cap, static_cast<int64_t>(p.k_splits) * T * c.hidden);
  }
  h->partial_elems = cap;

  const int64_t e_rows = std::max<int64_t>(c.max_tokens, 256);
  bool ok = cudaMalloc(&h->w16, static_cast<size_t>(c.row_dim) * c.hidden * 2) == cudaSuccess &&
            cudaMalloc(&h->partial, static_cast<size_t>(cap) * 4) == cudaSuccess &&
            cudaMalloc(&h->conv0, static_cast<size_t>(c.max_seqs) * 3 * c.hidden * 4) == cudaSuccess &&
            cudaMalloc(&h->status, 8) == cudaSuccess;
  for (int k = 0; k < (c.prepare_slots == 2 ? 2 : 1) && ok; ++k) {
    ple_handle::Scratch& sc = h->scratch[k];
    ok = cudaMalloc(&sc.e, static_cast<size_t>(e_rows) * c.row_dim * 2) == cudaSuccess &&
         cudaMalloc(&sc.ids, static_cast<size_t>(c.max_tokens) * ids_per_token(c) * 4) == cudaSuccess &&
         cudaMalloc(&sc.meta, static_cast<size_t>(c.max_tokens) * sizeof(ple::TokMeta)) == cudaSuccess &&
         cudaMalloc(&sc.hist_new, static_cast<size_t>(c.max_seqs) * 2 * 4) == cudaSuccess &&
         cudaMalloc(&sc.row_scales, 16 * 2 * 4) == cudaSuccess;
  }
  h->decode_proj = ple::decode_proj_plan(c.hidden, c.row_dim, h->num_sms, &h->decode_plan);
  h->mtp = ok && c.max_tokens > 16 && ple::mtp_proj_plan(c.hidden, c.row_dim, h->num_sms, &h->mtp_plan);
  if (h->mtp) {
    const size_t counts = static_cast<size_t>(2 * h->mtp_plan.m_tiles) * 4;
    ok = cudaMalloc(&h->mtp_partial, static_cast<size_t>(ple::mtp_partial_elems(h->mtp_plan)) * 4) == cudaSuccess &&
         cudaMalloc(&h->mtp_counts, counts) == cudaSuccess &&
         cudaMemsetAsync(h->mtp_counts, 0, counts, stream) == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    free_all(h);
    delete h;
    return PLE_ERR_OOM;
  }
  cudaMemsetAsync(h->status, 0, 8, stream);
  if (ple::launch_convert_w(static_cast<const __nv_bfloat16*>(weights->w_proj), c.row_dim, c.hidden, h->w16,
                            h->status, stream) != cudaSuccess) {
    free_all(h);
    delete h;
    return PLE_ERR_CUDA;
  }
  int32_t bad = 0;
  if (cudaMemcpyAsync(&bad, h->status, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess) {
    free_all(h);
    delete h;
    return PLE_ERR_CUDA;
  }
  if (bad != 0) {
    free_all(h);
    delete h;
    return PLE_ERR_UNSUPPORTED;
  }
  if (cudaMemsetAsync(h->status, 0, 4, stream) != cudaSuccess ||
      !encode_2d(h, &h->tmap_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, h->w16, c.row_dim, c.hidden,
                 static_cast<uint64_t>(c.row_dim) * 2, kTileK, kTileM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_kb2(h, &h->tmap_w_kb2, h->w16, c.row_dim, c.hidden, kTileM) ||
      cudaStreamSynchronize(stream) != cudaSuccess) {
    free_all(h);
    delete h;
    return PLE_ERR_CUDA;
  }
  *out = h;
  return PLE_OK;
}

ple_status ple_destroy(ple_handle* h) {
  if (h == nullptr) return PLE_ERR_INVALID_ARG;
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
  return PLE_OK;
}

ple_status ple_ngram_ids(ple_handle* h, const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                         const int32_t* hist, int32_t* ids, cudaStream_t stream) {
  if (h == nullptr || T < 0) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (S < 1 || S > h->cfg.max_seqs || T > h->cfg.max_tokens) return PLE_ERR_SHAPE;
  if (T == 0) return PLE_OK;
  if (tokens == nullptr || offsets == nullptr || ids == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(tokens, 4) || !aligned(offsets, 4) || !aligned(ids, 8) || (hist && !aligned(hist, 4)))
    return PLE_ERR_ALIGN;
  ple::PrepareArgs pa{};
  pa.tokens = tokens;
  pa.T = T;
  pa.offsets = offsets;
  pa.S = S;
  pa.hist = hist;
  pa.vocab = h->cfg.vocab;
  pa.rows0 = h->cfg.rows[0];
  pa.rows1 = h->cfg.rows[1];
  pa.ids = ids;
  pa.H = h->cfg.hidden;
  pa.status = h->status;
  if (heads_layout(h))            // [T][16]: the row IDs alone (no metadata, no rows)
    return run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return launch_embed_for(h, pa, nullptr, stream); });
  return run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return ple::launch_prepare(pa, stream); });
}

ple_status ple_gather_rows(ple_handle* h, const int32_t* ids, int32_t T, void* e_out, cudaStream_t stream) {
  if (h == nullptr || T < 0) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (T == 0) return PLE_OK;
  if (ids == nullptr || e_out == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(ids, 8) || !aligned(e_out, 16)) return PLE_ERR_ALIGN;
  const ple_config& c = h->cfg;
  if (heads_layout(h))
    return run_stage(h, PLE_STAGE_GATHER, stream, [&] {
      return ple::launch_gather_heads(ids, T, table_ref(h), c.rows[0], c.row_dim, static_cast<__half*>(e_out), stream);
    });
  return run_stage(h, PLE_STAGE_GATHER, stream, [&] {
    return ple::launch_gather(ids, T, table_ref(h), c.rows[0], c.rows[1], c.row_dim,
                              static_cast<__half*>(e_out), true, stream);
  });
}

ple_status ple_forward(ple_handle* h, const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                       const void* hidden, void* out, ple_out_dtype out_dtype, const ple_state* state,
                       cudaStream_t stream) {
  if (h == nullptr || T < 0) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (out_dtype != PLE_OUT_BF16 && out_dtype != PLE_OUT_F32) return PLE_ERR_INVALID_ARG;
  if (S < 1 || S > h->cfg.max_seqs || T > h->cfg.max_tokens) return PLE_ERR_SHAPE;
  if (T == 0) return PLE_OK;
  if (tokens == nullptr || offsets == nullptr || hidden == nullptr || out == nullptr) return PLE_ERR_INVALID_ARG;
  if (out == hidden && out_dtype != PLE_OUT_BF16) return PLE_ERR_INVALID_ARG;
  if (state != nullptr && (state->hist == nullptr || state->conv == nullptr)) return PLE_ERR_INVALID_ARG;
  if (!aligned(tokens, 4) || !aligned(offsets, 4) || !aligned(hidden, 16) || !aligned(out, 16) ||
      (state && (!aligned(state->hist, 4) || !aligned(state->conv, 16))))
    return PLE_ERR_ALIGN;
  return run_layer(h, tokens, T, offsets, S, hidden, out, out_dtype, state, stream);
}

ple_status ple_prepare_slot(ple_handle* h, int32_t slot, const int32_t* tokens, int32_t T, const int32_t* offsets,
                            int32_t S, const int32_t* hist, cudaStream_t stream) {
  if (h == nullptr || T < 0 || slot < 0 || slot > 1) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (h->scratch[slot].e == nullptr) return PLE_ERR_INVALID_ARG;      // slot 1 needs prepare_slots == 2
  if (S < 1 || S > h->cfg.max_seqs || T > h->cfg.max_tokens) return PLE_ERR_SHAPE;
  h->prepared_slot[slot].valid = false;
  if (slot == 0) h->prepared_decode.valid = false;
  if (T > 0) {
    if (tokens == nullptr || offsets == nullptr) return PLE_ERR_INVALID_ARG;
    if (!aligned(tokens, 4) || !aligned(offsets, 4) || (hist && !aligned(hist, 4))) return PLE_ERR_ALIGN;
    const ple_config& c = h->cfg;
    const ple_handle::Scratch& sc = h->scratch[slot];
    ple::PrepareArgs pa{};
    pa.tokens = tokens;
    pa.T = T;
    pa.offsets = offsets;
    pa.S = S;
    pa.hist = hist;
    pa.vocab = c.vocab;
    pa.rows0 = c.rows[0];
    pa.rows1 = c.rows[1];
    pa.ids = sc.ids;
    pa.hidden = nullptr;                 // the gate waits for ple_forward_prepared
    pa.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
    pa.H = c.hidden;
    pa.meta = sc.meta;
    pa.hist_new = sc.hist_new;
    pa.status = h->status;
    const ple_status st = run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return launch_embed_for(h, pa, sc.e, stream); });
    if (st != PLE_OK) return st;
  }
  ple_handle::Prepared& pr = h->prepared_slot[slot];
  pr.valid = true;
  pr.T = T;
  pr.S = S;
  pr.with_hist = hist != nullptr;
  return PLE_OK;
}

ple_status ple_prepare(ple_handle* h, const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                       const int32_t* hist, cudaStream_t stream) {
  return ple_prepare_slot(h, 0, tokens, T, offsets, S, hist, stream);
}

ple_status ple_forward_prepared_slot(ple_handle* h, int32_t slot, const void* hidden, void* out,
                                     ple_out_dtype out_dtype, const ple_state* state, cudaStream_t stream) {
  if (h == nullptr || slot < 0 || slot > 1 || !h->prepared_slot[slot].valid) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (out_dtype != PLE_OUT_BF16 && out_dtype != PLE_OUT_F32) return PLE_ERR_INVALID_ARG;
  const ple_handle::Prepared& pr = h->prepared_slot[slot];
  if ((state != nullptr) != pr.with_hist) return PLE_ERR_INVALID_ARG;
  const int32_t T = pr.T, S = pr.S;
  if (T == 0) return PLE_OK;
  if (hidden == nullptr || out == nullptr) return PLE_ERR_INVALID_ARG;
  if (out == hidden && out_dtype != PLE_OUT_BF16) return PLE_ERR_INVALID_ARG;
  if (state != nullptr && (state->hist == nullptr || state->conv == nullptr)) return PLE_ERR_INVALID_ARG;
  if (!aligned(hidden, 16) || !aligned(out, 16) || (state && (!aligned(state->hist, 4) || !aligned(state->conv, 16))))
    return PLE_ERR_ALIGN;
  const ple_config& c = h->cfg;
  const ple_handle::Scratch& sc = h->scratch[slot];
  ple::PrepareArgs ga{};
  ga.T = T;
  ga.S = S;
  ga.hidden = static_cast<const __nv_bfloat16*>(hidden);
  ga.w_gate = static_cast<const __nv_bfloat16*>(h->w.w_gate);
  ga.H = c.hidden;
  ga.meta = sc.meta;
  if (state != nullptr) {
    ga.conv_in = state->conv;
    ga.conv_copy = h->conv0;
  }
  const ple_status st = run_stage(h, PLE_STAGE_PREPARE, stream, [&] { return ple::launch_gate(ga, stream); });
  if (st != PLE_OK) return st;
  return run_projection(h, sc, T, S, 0, hidden, out, out_dtype, state, nullptr, nullptr, nullptr, nullptr, false,
                        stream);
}

ple_status ple_forward_prepared(ple_handle* h, const void* hidden, void* out, ple_out_dtype out_dtype,
                                const ple_state* state, cudaStream_t stream) {
  return ple_forward_prepared_slot(h, 0, hidden, out, out_dtype, state, stream);
}

ple_status ple_decode_step(ple_handle* h, const int32_t* tokens, int32_t B, int32_t q, const void* hidden, void* out,
                           ple_out_dtype out_dtype, int32_t* hist, float* conv_state, const int32_t* n_commit,
                           cudaStream_t stream) {
  if (h == nullptr) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  const ple_status chk = check_decode_step(h, B, q, hidden, out, out_dtype, hist, conv_state, n_commit);
  if (chk != PLE_OK) return chk;
  if (tokens == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(tokens, 4)) return PLE_ERR_ALIGN;
  h->prepared.valid = false;
  h->prepared_decode.valid = false;
  const bool small = decode_small(h, B, q);
  if (small && out != hidden) {
    // the whole step in one kernel: each CTA hashes the tokens and gathers the
    // K range of the rows it multiplies, and computes the gates
    ple::DecodeProjArgs a = decode_proj_args(h, tokens, B, q, hidden, out, out_dtype, hist, conv_state, n_commit);
    a.e = nullptr;
    a.meta = nullptr;
    a.gate_ready = 0;
    return run_stage(h, PLE_STAGE_GEMM, stream, [&] { return ple::launch_decode_proj(a, h->decode_plan, stream); });
  }
  const ple_status st = run_decode_embed(h, tokens, B, q, hist, hidden, small, stream);
  if (st != PLE_OK) return st;
  return run_decode_rest(h, tokens, B, q, hidden, out, out_dtype, hist, conv_state, n_commit, true, small, stream);
}

ple_status ple_decode_prepare(ple_handle* h, const int32_t* tokens, int32_t B, int32_t q, const int32_t* hist,
                              cudaStream_t stream) {
  if (h == nullptr) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  if (B < 1 || q < 1 || B > h->cfg.max_seqs || static_cast<int64_t>(B) * q > h->cfg.max_tokens) return PLE_ERR_SHAPE;
  if (tokens == nullptr || hist == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(tokens, 4) || !aligned(hist, 4)) return PLE_ERR_ALIGN;
  h->prepared.valid = false;
  h->prepared_decode.valid = false;
  const bool small = decode_small(h, B, q);
  const ple_status st = run_decode_embed(h, tokens, B, q, hist, nullptr, small, stream);
  if (st != PLE_OK) return st;
  h->prepared_decode = {true, B, q, tokens, hist, small};
  return PLE_OK;
}

ple_status ple_decode_step_prepared(ple_handle* h, const void* hidden, void* out, ple_out_dtype out_dtype,
                                    int32_t* hist, float* conv_state, const int32_t* n_commit, cudaStream_t stream) {
  if (h == nullptr || !h->prepared_decode.valid) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  const ple_handle::PreparedDecode pd = h->prepared_decode;
  if (hist != pd.hist) return PLE_ERR_INVALID_ARG;
  const ple_status chk = check_decode_step(h, pd.B, pd.q, hidden, out, out_dtype, hist, conv_state, n_commit);
  if (chk != PLE_OK) return chk;
  h->prepared_decode.valid = false;     // the state advances: the rows belong to this step only
  return run_decode_rest(h, pd.tokens, pd.B, pd.q, hidden, out, out_dtype, hist, conv_state, n_commit, false,
                         pd.small, stream);
}

ple_status ple_get_error(ple_handle* h) {
  if (h == nullptr) return PLE_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return PLE_ERR_CUDA;
  int32_t s = 0;
  if (cudaMemcpy(&s, h->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return PLE_ERR_CUDA;
  if (cudaMemset(h->status, 0, 4) != cudaSuccess) return PLE_ERR_CUDA;
  return static_cast<ple_status>(s);
}

ple_status ple_set_profiling(ple_handle* h, int32_t enable) {
  if (h == nullptr) return PLE_ERR_INVALID_ARG;
  h->profiling = enable != 0;
  return PLE_OK;
}

ple_status ple_get_stage_times(ple_handle* h, float* ms, int64_t* launches) {
  if (h == nullptr || ms == nullptr || launches == nullptr) return PLE_ERR_INVALID_ARG;
  double acc[PLE_NUM_STAGES] = {0, 0, 0, 0};
  int64_t cnt[PLE_NUM_STAGES] = {0, 0, 0, 0};
  ple_status st = PLE_OK;
  for (auto& r : h->pending) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) st = PLE_ERR_CUDA;
    acc[r.stage] += t;
    cnt[r.stage] += 1;
    h->free_events.push_back(r.a);
    h->free_events.push_back(r.b);
  }
  h->pending.clear();
  for (int i = 0; i < PLE_NUM_STAGES; ++i) {
    ms[i] = static_cast<float>(acc[i]);
    launches[i] = cnt[i];
  }
  return st;
}

ple_status ple_set_forward_path(ple_handle* h, int32_t path) {
  if (h == nullptr || path < 0 || path > 4) return PLE_ERR_INVALID_ARG;
  h->forward_path = path;
  return PLE_OK;
}

int64_t ple_launch_count(const ple_handle* h) { return h ? h->launches : -1; }

ple_status ple_wait_selftest(ple_handle* h, int64_t limit_cycles, cudaStream_t stream) {
  if (h == nullptr || limit_cycles <= 0 || limit_cycles > ple::kWaitLimitCycles) return PLE_ERR_INVALID_ARG;
  if (wrong_device(h)) return PLE_ERR_INVALID_ARG;
  return ple::launch_wait_selftest(h->status, limit_cycles, stream) == cudaSuccess ? PLE_OK : PLE_ERR_CUDA;
}

}  // extern "C"
