/*
 * libple — the n-gram embedding ("PLE") layer of Qwen3.8 Flash-Next on one B200.
 *
 * What the layer computes is described in the DGX Spark deployment report
 * ("【Qwen3.8-Flash-Next 端侧部署】01-模型架构与整体方案", section
 * "n-gram embedding 是一条附加的条件记忆路径"): from raw token IDs,
 * positions and sequence boundaries the engine derives n-gram IDs, reads the
 * matching rows of a large FP8 table, and the rows go through
 * dequantisation, projection, gating and a short convolution before they are
 * merged into the hidden states. The RTX 3090 llama.cpp report (section
 * "n-gram表格") adds that rows are keyed by hashing the last few tokens,
 * bigram and trigram entries, and depend only on the text.
 *
 * The pages leave the hash, the scale layout and the gate open; this library
 * fixes them as follows (all arithmetic is integer or IEEE fp32 unless noted):
 *   context  x = (uint64)(uint32)token + 1; 0 for a position before the
 *            sequence start with no carried history (a carried entry < 0 is
 *            absent). Every token gets one bigram row and one trigram row.
 *   keys     k2 = x_t*0x9E3779B97F4A7C15 ^ x_{t-1}*0xC2B2AE3D27D4EB4F,
 *            k3 = k2 ^ x_{t-2}*0x165667B19E3779F9   (wrap-around mod 2^64)
 *   rows     row_n = (k_n ^ (k_n >> 32)) mod rows[n]  (unsigned 64-bit)
 *   embed    e_t[k] = E4M3(table[0][row_2][k])*scales[0][row_2]
 *                   + E4M3(table[1][row_3][k])*scales[1][row_3]
 *            or, for an NVFP4 table (see ple_table_format),
 *            e_t[k] = E2M1(code[0][row_2][k])*E4M3(block[0][row_2][k/16])*scales[0][row_2]
 *                   + (the same for order 1 and row_3)
 *   project  v_t = e_t W_proj            (W_proj bf16 [row_dim][hidden])
 *   gate     g_t = sigmoid(w_gate . h_t) (one scalar per token)
 *   conv     y_t[j] = sum_{k=0..3} conv_w[j][k] * u_{t-3+k}[j],  u = g v,
 *            u before a fresh sequence = 0, else the carried state
 *   residual out_t = h_t + y_t
 *
 * Precision: the GPU rounds e_t to fp16 (computed in fp32) and multiplies it
 * with an fp16 copy of W_proj on the tensor cores with fp32 accumulation;
 * everything after the projection is fp32. Against a float64 evaluation the
 * fp32 output stays within max |err| 2e-2 and relative L2 error 1e-3 on the
 * workloads the tests cover.
 *
 * Conventions for every call below:
 *   - pointers are DEVICE pointers unless stated otherwise; all calls are
 *     asynchronous and ordered on the given stream (cudaStream_t, 0 = legacy);
 *   - argument errors are detected on the host before anything is launched,
 *     and the call returns the error without side effects;
 *   - errors that only the device can see (token outside [0, vocab),
 *     inconsistent offsets, an internal wait that ran out) set a sticky status
 *     word in the handle, read and cleared by ple_get_error();
 *   - a handle is used by one stream at a time, with the device it was
 *     created on current (another current device gives PLE_ERR_INVALID_ARG).
 */
#ifndef PLE_H_
#define PLE_H_

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PLE_OK = 0,
  PLE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum, forbidden aliasing */
  PLE_ERR_SHAPE = 2,         /* a size is outside what the handle was created for */
  PLE_ERR_ALIGN = 3,         /* a pointer is not 16-byte aligned */
  PLE_ERR_RANGE = 4,         /* (device) token outside [0, vocab) or inconsistent offsets */
  PLE_ERR_OOM = 5,           /* device allocation failed in ple_create */
  PLE_ERR_CUDA = 6,          /* a CUDA runtime call failed */
  PLE_ERR_TIMEOUT = 7,       /* (device) a bounded internal wait ran out; outputs invalid */
  PLE_ERR_UNSUPPORTED = 8    /* configuration the kernels do not support (e.g. |W_proj| > 65504) */
} ple_status;

typedef enum { PLE_OUT_BF16 = 0, PLE_OUT_F32 = 1 } ple_out_dtype;

/* Table formats.
 *   PLE_TABLE_E4M3: one FP8 E4M3 ("fn") code per element and one fp32 scale per
 *     row (51.2 GB at 2 x 10,000,048 rows of 2560).
 *   PLE_TABLE_NVFP4: the capacity variant of the pages, about 26.82 GiB against
 *     95.37 GiB in BF16 (deletoe.com page, section "第三条路：把 PLE 也量化，能塞下，
 *     但不够快"; DGX Spark report, sections "运行时内存占用" and "小结": a packed
 *     table of NVFP4 codes and FP8 scales). The layout is not on the pages;
 *     this library reads it as FP4 E2M1 codes, two per byte with the low
 *     nibble first, one E4M3 block scale per 16 elements, and the same fp32
 *     scale per row as the E4M3 table.
 *   PLE_TABLE_E4M3_HEADS: the row geometry of the SSD-stream model card
 *     ("Qwen3.8 Flash-Next NVFP4 - SSD Stream", section "技术细节": 16 table
 *     lookups per token, 160-byte FP8 rows). 16 sub-tables (8 hash heads per
 *     order) of rows[0] rows of row_dim/16 E4M3 codes, one fp32 scale per row;
 *     head j of order n (sub-table 8n + j) takes row
 *     (k ^ (k >> 32)) mod rows[0] with k = k_n ^ (j * 0xFF51AFD7ED558CCD) mod 2^64
 *     (k_n the order's key below; head 0 is the two-order row), and e is the
 *     16 dequantised rows side by side in sub-table order. rows[1] must equal
 *     rows[0]; row_dim % 256 == 0. The same 51,200,245,760 bytes hold
 *     16 x 20,000,096 rows of 160. Row IDs are [T][16] for this format.
 *   PLE_TABLE_NVFP4_ROWS: the contents of PLE_TABLE_NVFP4 (the same codes,
 *     block scales and row scales, the same results bit for bit) stored row by
 *     row: each row's row_dim/2 code bytes followed by its row_dim/16
 *     block-scale bytes, row_dim*9/16 contiguous bytes per row. A token's row
 *     is then one piece of memory, which the prefill embed fetches with one
 *     copy instead of two. block_scales must be NULL; row_dim % 256 == 0. */
typedef enum {
  PLE_TABLE_E4M3 = 0,
  PLE_TABLE_NVFP4 = 1,
  PLE_TABLE_E4M3_HEADS = 2,
  PLE_TABLE_NVFP4_ROWS = 3
} ple_table_format;

/* Sizes fixed at creation. hidden % 128 == 0, row_dim % 64 == 0,
 * 0 < rows[n] < 2^31. max_tokens bounds T of every call (and B*q of a decode
 * step); max_seqs bounds S (and B). prepare_slots: 0 or 1 = one batch scratch;
 * 2 = a second one for ple_prepare_slot / ple_forward_prepared_slot slot 1
 * (max_tokens * row_dim * 2 bytes more). */
typedef struct {
  int32_t vocab;
  int32_t hidden;
  int32_t row_dim;
  int32_t max_tokens;
  int32_t max_seqs;
  int32_t table_format;      /* ple_table_format */
  int32_t prepare_slots;     /* 0, 1 or 2 */
  int64_t rows[2];           /* rows of the bigram (0) and trigram (1) sub-tables */
} ple_config;

/* Parameters. All are BORROWED: they must stay valid and unchanged for the
 * handle's lifetime, except w_proj, which is read once by ple_create. */
typedef struct {
  const uint8_t* table;      /* E4M3: one code per element; sub-table n, row r at byte
                                offset (n*rows[0] + r)*row_dim ([2][rows][row_dim] when
                                rows[0] == rows[1]).
                                NVFP4: packed E2M1 codes, element 2i in the low nibble of
                                byte i of the row; row r of sub-table n at byte offset
                                (n*rows[0] + r)*row_dim/2.
                                E4M3_HEADS: sub-table h (0..15), row r at byte offset
                                (h*rows[0] + r)*(row_dim/16).
                                NVFP4_ROWS: row r of sub-table n at byte offset
                                (n*rows[0] + r)*row_dim*9/16: its packed codes as for
                                NVFP4, then at row_dim/2 its block scales as for
                                block_scales below. 16-byte aligned */
  const float* scales;       /* fp32 per-row scales; sub-table n, row r at n*rows[0] + r */
  const void* w_proj;        /* bf16 [row_dim][hidden], row-major */
  const void* w_gate;        /* bf16 [hidden] */
  const float* conv_w;       /* fp32 [hidden][4]; tap 3 multiplies the current token */
  const uint8_t* block_scales; /* NVFP4 only (NULL for the other formats): E4M3 scale of elements
                                [16j, 16j+16) of row r of sub-table n at byte offset
                                (n*rows[0] + r)*row_dim/16 + j; 16-byte aligned */
} ple_weights;

/* Per-sequence carried state (caller-owned, device memory). */
typedef struct {
  int32_t* hist;             /* [S][2]: token t-2, token t-1 before the sequence; < 0 = absent */
  float* conv;               /* [S][3][hidden]: u_{t-3}, u_{t-2}, u_{t-1} */
} ple_state;

typedef struct ple_handle ple_handle;

/* Creates a handle on the current device. Allocates the handle's own device
 * memory (an fp16 K-major copy of W_proj and scratch sized by max_tokens and
 * max_seqs) and converts W_proj on `stream`; synchronises `stream`.
 * Returns PLE_ERR_UNSUPPORTED if some |W_proj| exceeds the fp16 range. */
ple_status ple_create(const ple_config* config, const ple_weights* weights,
                      cudaStream_t stream, ple_handle** out);

/* Frees the handle and its device memory (synchronises the device first). */
ple_status ple_destroy(ple_handle* handle);

/* N-gram row IDs only. tokens int32 [T]; offsets int32 [S+1] with
 * offsets[0] = 0, offsets[S] = T, non-decreasing (sequence s covers
 * [offsets[s], offsets[s+1])); hist int32 [S][2] or NULL (all absent);
 * ids int32 [T][2] receives (bigram row, trigram row), each in [0, rows[n]);
 * for PLE_TABLE_E4M3_HEADS, ids int32 [T][16] receives the 16 head rows. */
ple_status ple_ngram_ids(ple_handle* handle, const int32_t* tokens, int32_t T,
                         const int32_t* offsets, int32_t S, const int32_t* hist,
                         int32_t* ids, cudaStream_t stream);

/* The gather stage alone: e_out fp16 [T][row_dim] receives e_t (see top of
 * file, in the handle's table format) for the given row IDs int32 [T][2]
 * ([T][16] for PLE_TABLE_E4M3_HEADS). IDs must be in range (the call reduces
 * them mod rows[n] so that no access leaves the table). */
ple_status ple_gather_rows(ple_handle* handle, const int32_t* ids, int32_t T,
                           void* e_out, cudaStream_t stream);

/* The layer on a packed batch (prefill or one chunk of a chunked prefill).
 * hidden bf16 [T][hidden]; out [T][hidden] of `out_dtype`, may equal hidden
 * only with PLE_OUT_BF16 (in-place residual add). state == NULL: every
 * sequence starts fresh and no state is written. Otherwise state->hist and
 * state->conv ([S] entries) are read as the state before each sequence and
 * overwritten with the state after it (unchanged for an empty sequence).
 * T == 0 is allowed and does nothing. */
ple_status ple_forward(ple_handle* handle, const int32_t* tokens, int32_t T,
                       const int32_t* offsets, int32_t S, const void* hidden, void* out,
                       ple_out_dtype out_dtype, const ple_state* state, cudaStream_t stream);

/* The layer in two calls, for callers that know the tokens before the hidden
 * states: the n-gram IDs and the row lookup need no hidden state (DGX Spark
 * report, section "n-gram embedding 是一条附加的条件记忆路径"), so
 * ple_prepare can run on a side stream while earlier layers compute hidden,
 * and ple_forward_prepared then does the rest: the gate, the projection, the
 * conv, the residual and the state.
 *
 * ple_prepare takes the arguments of ple_forward that do not depend on hidden
 * (hist = the state's hist, or NULL for fresh sequences) and leaves the row
 * IDs, the dequantised rows and the per-token metadata in the handle's
 * scratch. ple_forward_prepared takes hidden, out, out_dtype and state as in
 * ple_forward, for the batch last prepared on the handle. The result equals
 * ple_forward's bit for bit.
 *   - state must be non-NULL exactly when ple_prepare got a hist, and
 *     state->hist must hold the values ple_prepare read; otherwise
 *     PLE_ERR_INVALID_ARG.
 *   - ple_forward_prepared without a prepared batch returns
 *     PLE_ERR_INVALID_ARG. ple_forward and ple_decode_step reuse the scratch
 *     and discard the prepared batch. A prepared batch stays usable for
 *     further ple_forward_prepared calls (other hidden states) until then.
 *   - The two calls may use different streams; ordering them (an event) is
 *     the caller's job. */
ple_status ple_prepare(ple_handle* handle, const int32_t* tokens, int32_t T,
                       const int32_t* offsets, int32_t S, const int32_t* hist, cudaStream_t stream);
ple_status ple_forward_prepared(ple_handle* handle, const void* hidden, void* out,
                                ple_out_dtype out_dtype, const ple_state* state, cudaStream_t stream);

/* The same two calls on one of two batch slots, so that the next batch can be
 * prepared while the current one is projected: the Thor report's SSD tier
 * ("第四条路：让 47.68 GiB PLE 留在 SSD") and the SSD-stream model card
 * ("技术细节") fetch rows while earlier work runs and wait only when fetching
 * is slower. ple_prepare / ple_forward_prepared are slot 0. Slot 1 exists when
 * the handle was created with prepare_slots == 2 (else PLE_ERR_INVALID_ARG).
 *   - Each slot holds its own rows, IDs, metadata and new token history; a
 *     slot's prepared batch stays usable until the next ple_prepare_slot on
 *     the same slot. ple_forward, ple_prepare and the decode calls use slot
 *     0's scratch and discard slot 0's batch only.
 *   - ple_prepare_slot(s) may run on another stream at the same time as
 *     ple_forward_prepared_slot(1 - s); the caller orders the calls on the
 *     same slot (events), and runs the hidden-dependent calls (forward,
 *     forward_prepared, decode steps) on one stream at a time.
 *   - Results equal ple_forward's bit for bit. */
ple_status ple_prepare_slot(ple_handle* handle, int32_t slot, const int32_t* tokens, int32_t T,
                            const int32_t* offsets, int32_t S, const int32_t* hist, cudaStream_t stream);
ple_status ple_forward_prepared_slot(ple_handle* handle, int32_t slot, const void* hidden, void* out,
                                     ple_out_dtype out_dtype, const ple_state* state, cudaStream_t stream);

/* One decode / speculative-verify step: B sequences with q new tokens each.
 * tokens int32 [B][q]; hidden bf16 [B*q][hidden]; out [B*q][hidden];
 * hist int32 [B][2] and conv_state fp32 [B][3][hidden] are read and updated.
 * out may equal hidden only with PLE_OUT_BF16 (in-place residual add).
 * Outputs are computed for all q tokens; the state advances by the first
 * n_commit[b] tokens of sequence b (1 <= n_commit[b] <= q; NULL means q),
 * i.e. accepted draft tokens are committed and rejected ones rolled back. */
ple_status ple_decode_step(ple_handle* handle, const int32_t* tokens, int32_t B, int32_t q,
                           const void* hidden, void* out, ple_out_dtype out_dtype,
                           int32_t* hist, float* conv_state, const int32_t* n_commit,
                           cudaStream_t stream);

/* The decode step in two calls, for callers that know a step's tokens before
 * its hidden states. The n-gram IDs and the row lookup need no hidden state
 * (DGX Spark report, section "n-gram embedding 是一条附加的条件记忆路径"), and
 * the SSD-stream model card ("Qwen3.8 Flash-Next NVFP4 - SSD Stream", section
 * "技术细节") fetches the rows before the model reaches the block that uses
 * them. ple_decode_prepare takes the tokens [B][q] and the token history
 * hist [B][2] that ple_decode_step would take, and leaves the step's rows
 * and per-token metadata in the handle's scratch: for a step of up to 8
 * tokens of an E4M3 or NVFP4 table, each token's two rows as exact fp16 codes
 * with their two row scales (the step then reads them in one round trip and
 * applies the scales after the products, as ple_decode_step does); otherwise
 * the dequantised rows. The form is chosen here, with the path selection of
 * ple_set_forward_path in force at this call.
 * ple_decode_step_prepared then takes the rest of ple_decode_step's arguments
 * and runs the gate, the projection, the conv, the residual and the state
 * update. Together they give ple_decode_step's result bit for bit.
 *   - hist must be the buffer ple_decode_prepare read, unchanged in between;
 *     ple_decode_step_prepared updates it. Another pointer gives
 *     PLE_ERR_INVALID_ARG.
 *   - tokens must stay valid and unchanged until ple_decode_step_prepared has
 *     run: it reads them for the new token history.
 *   - ple_decode_step_prepared consumes the prepared step. ple_forward,
 *     ple_prepare, ple_decode_step and another ple_decode_prepare discard it.
 *     Without a prepared step the call returns PLE_ERR_INVALID_ARG.
 *   - The two calls may use different streams; ordering them (an event) is the
 *     caller's job. */
ple_status ple_decode_prepare(ple_handle* handle, const int32_t* tokens, int32_t B, int32_t q, const int32_t* hist,
                              cudaStream_t stream);
ple_status ple_decode_step_prepared(ple_handle* handle, const void* hidden, void* out, ple_out_dtype out_dtype,
                                    int32_t* hist, float* conv_state, const int32_t* n_commit, cudaStream_t stream);

/* ---- lookup without allocation ------------------------------------------
 * The pages have no counterpart of this entry point; it exists for callers of
 * this library that cannot allocate device memory where they run the layer:
 * serving engines whose caching allocator reserves the whole device budget at
 * start-up (a later cudaMalloc fails or fragments that pool), and runtimes
 * that forbid device allocation after initialisation. Such callers cannot
 * create a handle either, since ple_create allocates.
 *
 * ple_embed_static computes the n-gram row IDs of a packed batch (as
 * ple_ngram_ids) and gathers and dequantises the rows of an E4M3 table
 * (PLE_TABLE_E4M3 layout) into e_out fp16
 * [T][row_dim] (as ple_gather_rows). It allocates nothing: the row IDs live in
 * a fixed array inside the library image, PLE_STATIC_MAX_TOKENS x 2 int32
 * (128 KiB), which every GPU that loads the library holds until the process
 * exits. The caller passes all inputs and the output; table and scales are
 * laid out as in ple_weights, with rows0 / rows1 rows in the two sub-tables.
 *   - T > PLE_STATIC_MAX_TOKENS returns PLE_ERR_SHAPE; nothing is launched.
 *     row_dim must be a multiple of 16 and at most 65536 (else
 *     PLE_ERR_UNSUPPORTED).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. After cudaDeviceReset the next call on that
 *     device looks the address up again (the library image then lives in a
 *     new context), so that call too belongs outside a capture.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents. Calls that overlap on the GPU (other streams, other threads)
 *     race on it: order them on one stream.
 *   - status_out (device int32, may be NULL) receives the call's device status:
 *     PLE_ERR_RANGE for a token outside [0, vocab) or inconsistent offsets,
 *     else PLE_OK. Every call that returns PLE_OK writes it, T == 0 included
 *     (which launches nothing else and writes PLE_OK). */
#define PLE_STATIC_MAX_TOKENS 16384
ple_status ple_embed_static(const int32_t* tokens, int32_t T, const int32_t* offsets, int32_t S,
                            const int32_t* hist, const uint8_t* table, const float* scales,
                            int64_t rows0, int64_t rows1, int32_t row_dim, int32_t vocab, void* e_out,
                            int32_t* status_out, cudaStream_t stream);

/* Synchronises the device, returns the sticky device status and clears it. */
ple_status ple_get_error(ple_handle* handle);

/* Static description of a status code. */
const char* ple_status_string(ple_status status);

/* ---- measurement and test controls -------------------------------------- */

/* Kernel stages of the library, in launch order within a call. In
 * ple_forward and ple_decode_step the PREPARE stage also gathers and
 * dequantises the rows, except on the gather-fused path, where the GEMM stage
 * does. In ple_forward, PREPARE is one fused kernel, or, for a batch of 4,096
 * tokens or more, a row-ID kernel followed by the gate-and-gather kernel. In
 * a decode step it is the kernel of the step's tokens (rows, metadata, gates),
 * and for a step of up to 16 tokens GEMM is one kernel that also does the
 * gate, conv, residual and state (no COMBINE). ple_prepare, ple_decode_prepare
 * and the gate kernels of the prepared forms count as PREPARE too. GATHER
 * counts ple_gather_rows. */
enum { PLE_STAGE_PREPARE = 0, PLE_STAGE_GATHER = 1, PLE_STAGE_GEMM = 2, PLE_STAGE_COMBINE = 3,
       PLE_NUM_STAGES = 4 };

/* enable != 0: record CUDA events around every stage the handle runs (on the
 * call's stream) so that ple_get_stage_times can report them. */
ple_status ple_set_profiling(ple_handle* handle, int32_t enable);

/* Synchronises the recorded events and writes, per stage, the summed time in
 * milliseconds (ms[PLE_NUM_STAGES]) and the number of times the stage ran
 * (launches[PLE_NUM_STAGES]) since the last call; then resets the counters.
 * ple_launch_count counts kernels. */
ple_status ple_get_stage_times(ple_handle* handle, float* ms, int64_t* launches);

/* Path selection. For ple_forward: 0 = automatic, 1 = fused epilogue
 * (gate, conv and residual inside the projection kernel, conv halo
 * recomputed per tile; SM-pair tiles of 256 channels when hidden % 256 == 0),
 * 2 = split-K projection followed by a combine kernel, 3 = fused epilogue with
 * single-SM tiles of 128 channels, 4 = as 1, but with the row gather and
 * dequantisation inside the projection kernel: the first kernel computes only
 * the row IDs and the gate, and the projection reads the FP8 rows itself into
 * its shared-memory operand tiles, so the fp16 rows never reach HBM (E4M3
 * tables, SM-pair tiles, row_dim >= 128; elsewhere path 4 runs as
 * path 1). Paths 1 and 4 give identical bits; path 4 is never chosen
 * automatically, because on B200 it is slower (each token's rows are
 * dequantised once per 256-channel tile inside the tensor-bound kernel). For ple_decode_step: steps of B * q <= 16 tokens
 * run the channel-split projection kernel (every CTA owns whole output
 * channels, no partial sums cross CTAs) unless path is 2, which forces the
 * split-K projection and its combine kernel. */
ple_status ple_set_forward_path(ple_handle* handle, int32_t path);

/* Total number of kernels the handle has launched since creation. */
int64_t ple_launch_count(const ple_handle* handle);

/* Failure-detection self-test. Every wait inside the library's kernels is
 * bounded: when one runs out, the kernel records PLE_ERR_TIMEOUT in the
 * handle's sticky status, abandons its work and returns, so the CUDA context
 * stays usable and ple_get_error reports the failure. This call exercises that
 * path on demand: it launches one small kernel (stream-ordered) whose wait on
 * an mbarrier that nothing completes runs out after limit_cycles SM cycles
 * (0 < limit_cycles <= 2e9, about one second at B200 clocks). Returns
 * PLE_ERR_INVALID_ARG for a null handle or a limit out of range. */
ple_status ple_wait_selftest(ple_handle* handle, int64_t limit_cycles, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PLE_H_ */
