"""CPU oracle for the PLE n-gram embedding layer.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import or call this module. The GPU library never uses it;
it shares no code, table or constant generator with the CUDA path.

What the layer computes, and where the pages say so
---------------------------------------------------
The only prose definition is in the DGX Spark deployment report
("【Qwen3.8-Flash-Next 端侧部署】01-模型架构与整体方案", mengman.github.io,
section "n-gram embedding 是一条附加的条件记忆路径"): the engine keeps the raw
token IDs, positions and sequence boundaries, derives n-gram IDs from them,
reads the matching vectors from the big table, and the looked-up vectors go
through dequantisation, projection, gating and a short convolution before
they are merged into the hidden states on the GPU. The same section says the
ID computation and the lookup need no hidden state, while the merge does.
The RTX 3090 llama.cpp report (reactapp.top, section "n-gram表格") adds that
rows are keyed by hashing the last few tokens, that there are about 20 M
bigram and trigram entries, and that the needed rows depend only on the text.
The table is FP8 (bittide.aicompass.dev model card, "模型简介").

The pages give neither the hash, the scale layout, the gate form nor the conv
details. The readings fixed here (each marked READING) are:

* C-1  sequence s covers tokens [offsets[s], offsets[s+1]); no n-gram and no
       conv tap crosses a sequence boundary.
* C-2  context value of a token is x = uint32(token) + 1; a position before
       the sequence start with no carried history has x = 0, so every token
       gets both an order-2 (bigram) and an order-3 (trigram) row. A carried
       history entry < 0 is absent.
* C-3  keys, wrap-around mod 2**64:  k2 = x_t*P0 ^ x_{t-1}*P1,
       k3 = k2 ^ x_{t-2}*P2, with P0 the 64-bit golden-ratio constant of
       Knuth's multiplicative hashing and P1, P2 two odd 64-bit constants
       (the published xxHash64 primes 2 and 3).
* C-4  fold(k) = k ^ (k >> 32);  row_n = fold(k_n) mod R_n.
* C-5  FP8 codes are OCP E4M3 "fn" (bias 7, no infinities, 0x7F/0xFF NaN).
* C-6  one fp32 scale per row per order; deq = decode(code) * scale.
* C-7  the two orders are summed: e = deq(bigram row) + deq(trigram row).
* C-8  scalar gate per token: g_t = sigmoid(sum_j w_gate[j] * h_t[j]).
* C-9  depthwise causal conv of width 4 on u = g * v, no bias:
       y_t[j] = sum_{k=0..3} cw[j][k] * u_{t-3+k}[j]; tap 3 is the current
       token; u before a fresh sequence is 0, else the carried state.
* C-10 out = h + y.
* C-12 carried state: the last two tokens and the last three u rows.
* C-16 the NVFP4 table variant: FP4 E2M1 codes, two per byte (low nibble
       first), an E4M3 scale per 16 codes and the C-6 row scale.
* C-17 the multi-head row layout (the SSD-stream model card's geometry: 16
       table lookups per token of 160-byte rows): 8 heads per order, head j of
       order n reads sub-table 8n + j at row fold(k_n ^ j*HEAD_MIX) mod R'
       (head 0 is the C-4 row), each row carries its own scale, and e is the
       16 dequantised rows concatenated in head order.

Precision: every step is evaluated in float64 (library matmul for the
projection and the gate dot product); the caller rounds the float64 result
to fp32 or bf16 with ``to_f32`` / ``to_bf16_bits``.
"""
from __future__ import annotations

import math

import numpy as np

_U64 = np.uint64
_MASK64 = (1 << 64) - 1

# C-3 constants (READING): odd 64-bit multipliers.
P0 = 0x9E3779B97F4A7C15
P1 = 0xC2B2AE3D27D4EB4F
P2 = 0x165667B19E3779F9


# --------------------------------------------------------------------------------------
# C-5  FP8 E4M3 ("fn") decoding, closed form
# --------------------------------------------------------------------------------------
def e4m3_decode(code: int) -> float:
    """Value of one E4M3 byte: sign bit, 4 exponent bits (bias 7), 3 mantissa bits.

    exponent field 0: (-1)^s * (m/8) * 2^-6   (subnormal)
    otherwise:        (-1)^s * (1 + m/8) * 2^(e-7)
    0x7F and 0xFF are NaN; the format has no infinities (max finite 448)."""
    code = int(code) & 0xFF
    s = code >> 7
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        mag = (m / 8.0) * 2.0 ** -6
    else:
        mag = (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


E4M3_VALUES = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)


# --------------------------------------------------------------------------------------
# C-16  NVFP4 table rows (READING): FP4 E2M1 codes with an E4M3 scale per 16 codes
# --------------------------------------------------------------------------------------
# The pages' capacity variant quantises the PLE table to NVFP4, about 26.82 GiB
# against 95.37 GiB in BF16 (deletoe.com page, section "第三条路：把 PLE 也量化，
# 能塞下，但不够快"; DGX Spark report, section "运行时内存占用"), a packed table of
# "NVFP4 code" and "FP8 scale" (DGX Spark report, section "小结"). 26.82 GiB for
# the same 51.2 G elements is 4.5 bits per element: a 4-bit code per element and
# an 8-bit scale per 16 elements. The layout is not on the pages; this build
# reads it as: codes u8 [2][R][D/2], element 2i in the low nibble of byte i and
# element 2i+1 in the high nibble; block scales E4M3 u8 [2][R][D/16], block j
# covering elements [16j, 16j+16); and the per-row fp32 scale of C-6 kept as
# the outer factor:  deq[k] = e2m1(code_k) * e4m3(block_scale[k // 16]) * scale.

def e2m1_decode(code: int) -> float:
    """Value of one FP4 E2M1 code: sign bit, 2 exponent bits (bias 1), 1 mantissa bit.

    exponent field 0: (-1)^s * m * 0.5   (subnormal; m = 0 is zero)
    otherwise:        (-1)^s * (1 + m/2) * 2^(e-1)
    The format has no infinities and no NaN (max magnitude 6)."""
    code = int(code) & 0xF
    s = code >> 3
    e = (code >> 1) & 0x3
    m = code & 0x1
    mag = m * 0.5 if e == 0 else (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return -mag if s else mag


E2M1_VALUES = np.array([e2m1_decode(c) for c in range(16)], dtype=np.float64)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    """uint8 [..., D/2] of two codes per byte -> uint8 codes [..., D] (low nibble first)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequantise_nvfp4(packed: np.ndarray, block_scales: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """deq[i][k] = e2m1(code[i][k]) * e4m3(block_scales[i][k // 16]) * scales[i]   (C-16)."""
    codes = unpack_fp4(packed)
    blocks = E4M3_VALUES[np.asarray(block_scales, dtype=np.uint8)]
    per_elem = np.repeat(blocks, 16, axis=-1)
    return E2M1_VALUES[codes] * per_elem * np.asarray(scales, np.float64)[:, None]


# --------------------------------------------------------------------------------------
# bf16 / fp32 conversions of the oracle's own
# --------------------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to fp32 (nearest), then fp32 to bf16 with round-to-nearest-even."""
    b = to_f32(x).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    return ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


# --------------------------------------------------------------------------------------
# C-1  sequence map
# --------------------------------------------------------------------------------------
def sequence_map(offsets: np.ndarray, n_tokens: int):
    """For each token t: its sequence s (offsets[s] <= t < offsets[s+1]) and its
    position p = t - offsets[s] inside that sequence."""
    offsets = np.asarray(offsets, dtype=np.int64)
    t = np.arange(n_tokens, dtype=np.int64)
    seq = np.searchsorted(offsets, t, side="right") - 1
    pos = t - offsets[seq]
    return seq, pos


# --------------------------------------------------------------------------------------
# C-2  n-gram contexts
# --------------------------------------------------------------------------------------
def _context_value(token: int) -> int:
    return (int(token) & 0xFFFFFFFF) + 1


def ngram_contexts(tokens, offsets, hist=None):
    """x_t, x_{t-1}, x_{t-2} for every token as Python ints (C-2).

    ``hist`` (optional, [S][2]) holds the two tokens before each sequence's
    first token (index 0 = t-2, index 1 = t-1); negative entries are absent."""
    tokens = np.asarray(tokens).reshape(-1)
    T = tokens.shape[0]
    seq, pos = sequence_map(offsets, T)
    x0 = [0] * T
    x1 = [0] * T
    x2 = [0] * T
    for t in range(T):
        s, p = int(seq[t]), int(pos[t])
        x0[t] = _context_value(tokens[t])

        def carried(k):  # the token k places before the sequence start (k = 1 or 2)
            if hist is None:
                return 0
            h = int(hist[s][2 - k])
            return 0 if h < 0 else _context_value(h)

        x1[t] = _context_value(tokens[t - 1]) if p >= 1 else carried(1)
        if p >= 2:
            x2[t] = _context_value(tokens[t - 2])
        elif p == 1:
            x2[t] = carried(1)
        else:
            x2[t] = carried(2)
    return x0, x1, x2


# --------------------------------------------------------------------------------------
# C-3 / C-4  keys and row IDs
# --------------------------------------------------------------------------------------
def ngram_keys(x0: int, x1: int, x2: int):
    """Bigram and trigram keys of one token (arbitrary-precision ints, reduced mod 2^64)."""
    k2 = ((x0 * P0) & _MASK64) ^ ((x1 * P1) & _MASK64)
    k3 = k2 ^ ((x2 * P2) & _MASK64)
    return k2, k3


def fold(k: int) -> int:
    return k ^ (k >> 32)


def ngram_ids(tokens, offsets, rows, hist=None) -> np.ndarray:
    """Row IDs [T][2] (bigram row in sub-table 0, trigram row in sub-table 1)."""
    R0, R1 = (rows, rows) if np.isscalar(rows) else rows
    x0, x1, x2 = ngram_contexts(tokens, offsets, hist)
    ids = np.zeros((len(x0), 2), dtype=np.int64)
    for t in range(len(x0)):
        k2, k3 = ngram_keys(x0[t], x1[t], x2[t])
        ids[t, 0] = fold(k2) % int(R0)
        ids[t, 1] = fold(k3) % int(R1)
    return ids


# --------------------------------------------------------------------------------------
# C-17  the multi-head row layout (READING)
# --------------------------------------------------------------------------------------
# The SSD-stream model card (bittide.aicompass.dev mirror, section "技术细节")
# says the model makes 16 deterministic table lookups per generated token and
# that each FP8 row is 160 bytes; the same card gives the table as one file of
# 51,200,245,760 bytes, which is 16 sub-tables x 20,000,096 rows x 160 bytes.
# The main reading of this build (C-13) keeps 2 lookups of 2560-byte rows; this
# variant reads the card literally: each order (bigram, trigram) has 8 hash
# heads, head j of order n owns sub-table 8n + j, and the 16 rows of a token,
# each dequantised with its own row scale, are concatenated in head order to
# the 2560-wide e (16 x 160). Heads are separated by xor-ing a per-head
# multiple of an odd constant into the order's key before the fold, so head 0
# is exactly the C-4 row.

HEADS_PER_ORDER = 8
HEAD_MIX = 0xFF51AFD7ED558CCD   # odd 64-bit constant (MurmurHash3's 64-bit finaliser multiplier)


def ngram_ids_heads(tokens, offsets, rows_per_head, hist=None, heads=HEADS_PER_ORDER) -> np.ndarray:
    """Row IDs [T][2 * heads]: column n * heads + j is head j of order n (C-17)."""
    x0, x1, x2 = ngram_contexts(tokens, offsets, hist)
    R = int(rows_per_head)
    ids = np.zeros((len(x0), 2 * heads), dtype=np.int64)
    for t in range(len(x0)):
        keys = ngram_keys(x0[t], x1[t], x2[t])
        for n in range(2):
            for j in range(heads):
                ids[t, n * heads + j] = fold(keys[n] ^ ((j * HEAD_MIX) & _MASK64)) % R
    return ids


def row_ids(tokens, offsets, rows, hist, table) -> np.ndarray:
    """The token's row IDs for the table's layout: [T][2] (C-4) or [T][16] (C-17)."""
    if getattr(table, "format", "e4m3") == "heads":
        return ngram_ids_heads(tokens, offsets, rows if np.isscalar(rows) else rows[0], hist,
                               table.heads_per_order)
    return ngram_ids(tokens, offsets, rows, hist)


# --------------------------------------------------------------------------------------
# C-5..C-7  gather, dequantise, sum the orders
# --------------------------------------------------------------------------------------
def dequantise(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """deq[i][k] = decode(codes[i][k]) * scales[i]   (C-6)."""
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)] * np.asarray(scales, np.float64)[:, None]


def table_rows(table, order: int, rows) -> np.ndarray:
    """Dequantised rows of sub-table ``order`` (C-6 for an FP8 table, C-16 for NVFP4).

    ``table`` supplies ``codes(order, rows)`` and ``scales(order, rows)``, and for
    ``table.format == "nvfp4"`` also ``block_scales(order, rows)``."""
    if getattr(table, "format", "e4m3") == "nvfp4":
        return dequantise_nvfp4(table.codes(order, rows), table.block_scales(order, rows),
                                table.scales(order, rows))
    return dequantise(table.codes(order, rows), table.scales(order, rows))


def embed(table, ids: np.ndarray) -> np.ndarray:
    """e_t = deq(bigram row of t) + deq(trigram row of t)   (C-7); for the
    multi-head layout the 16 dequantised rows side by side in head order (C-17)."""
    ids = np.asarray(ids, dtype=np.int64)
    if getattr(table, "format", "e4m3") == "heads":
        return np.concatenate([dequantise(table.codes(h, ids[:, h]), table.scales(h, ids[:, h]))
                               for h in range(ids.shape[1])], axis=1)
    return table_rows(table, 0, ids[:, 0]) + table_rows(table, 1, ids[:, 1])


class ArrayTable:
    """A table held in arrays: codes uint8 [2][R][D], scales float32 [2][R]."""

    def __init__(self, codes: np.ndarray, scales: np.ndarray):
        self._codes = codes
        self._scales = scales

    def codes(self, order, rows):
        return self._codes[order][np.asarray(rows, dtype=np.int64)]

    def scales(self, order, rows):
        return self._scales[order][np.asarray(rows, dtype=np.int64)]


class HeadsArrayTable(ArrayTable):
    """A multi-head table held in arrays (C-17): codes uint8 [2 * heads][R'][D / (2 * heads)],
    scales float32 [2 * heads][R']; ``codes(h, rows)`` reads sub-table h."""

    format = "heads"

    def __init__(self, codes: np.ndarray, scales: np.ndarray, heads_per_order: int = HEADS_PER_ORDER):
        super().__init__(codes, scales)
        self.heads_per_order = heads_per_order


class Nvfp4ArrayTable(ArrayTable):
    """An NVFP4 table held in arrays (C-16): packed codes uint8 [2][R][D/2], block
    scales uint8 (E4M3) [2][R][D/16], row scales float32 [2][R]."""

    format = "nvfp4"

    def __init__(self, codes: np.ndarray, block_scales: np.ndarray, scales: np.ndarray):
        super().__init__(codes, scales)
        self._block_scales = block_scales

    def block_scales(self, order, rows):
        return self._block_scales[order][np.asarray(rows, dtype=np.int64)]


# --------------------------------------------------------------------------------------
# projection, gate, short conv, residual
# --------------------------------------------------------------------------------------
def project(e: np.ndarray, w_proj: np.ndarray) -> np.ndarray:
    """v_t = e_t W_proj, W_proj of shape [row_dim][hidden] (library matmul, float64)."""
    return np.asarray(e, np.float64) @ np.asarray(w_proj, np.float64)


def gate(h: np.ndarray, w_gate: np.ndarray) -> np.ndarray:
    """g_t = sigmoid(w_gate . h_t)   (C-8)."""
    a = np.asarray(h, np.float64) @ np.asarray(w_gate, np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-a))


def short_conv(u_hist: np.ndarray, conv_w: np.ndarray) -> np.ndarray:
    """Causal depthwise conv of width 4 over one sequence (C-9).

    ``u_hist`` is [3 + L][H]: the three u rows before the sequence (carried state
    or zeros) followed by the sequence's own L rows. Returns y [L][H] with
    y_t = sum_k cw[:, k] * u_{t-3+k}."""
    L = u_hist.shape[0] - 3
    cw = np.asarray(conv_w, np.float64)
    y = np.zeros((L, u_hist.shape[1]), dtype=np.float64)
    for k in range(4):
        y += cw[:, k][None, :] * u_hist[k:k + L]
    return y


# --------------------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------------------
def ple_forward(tokens, offsets, hidden_bits, w_proj_bits, w_gate_bits, conv_w, table,
                rows, hist=None, conv_state=None, sample=None):
    """The PLE layer on a packed batch.

    tokens int [T]; offsets int [S+1]; hidden_bits bf16 bits [T][H];
    w_proj_bits bf16 bits [D][H]; w_gate_bits bf16 bits [H]; conv_w f32 [H][4];
    hist int [S][2] or None; conv_state float [S][3][H] or None (zeros).

    ``sample`` (optional): token indices whose outputs are wanted; only the
    rows those outputs depend on are gathered and projected.

    ``rows`` is the rows per order (C-4), or per head sub-table for a table of
    the multi-head layout (C-17).

    Returns a dict: ``ids`` [T][2] ([T][16] for C-17); ``out`` float64 [len(sample) or T][H];
    ``hist_out`` [S][2] and ``conv_out`` [S][3][H] (the state after each sequence).
    """
    tokens = np.asarray(tokens).reshape(-1)
    offsets = np.asarray(offsets, dtype=np.int64)
    T = tokens.shape[0]
    S = offsets.shape[0] - 1
    ids = row_ids(tokens, offsets, rows, hist, table)
    seq, pos = sequence_map(offsets, T)
    H = np.asarray(w_gate_bits).shape[0]
    conv0 = np.zeros((S, 3, H)) if conv_state is None else np.asarray(conv_state, np.float64)

    want = np.arange(T) if sample is None else np.asarray(sample, dtype=np.int64)
    # tokens whose u is needed: each wanted token and up to 3 predecessors in its
    # sequence, and the last 3 tokens of every sequence (for the end state)
    need = set()
    for t in want:
        for k in range(4):
            if pos[t] - k >= 0:
                need.add(int(t) - k)
    for s in range(S):
        for t in range(max(int(offsets[s]), int(offsets[s + 1]) - 3), int(offsets[s + 1])):
            need.add(t)
    need = np.array(sorted(need), dtype=np.int64)
    idx_of = {int(t): i for i, t in enumerate(need)}

    h_need = bf16_bits_to_f64(np.asarray(hidden_bits)[need])
    e = embed(table, ids[need])
    v = project(e, bf16_bits_to_f64(w_proj_bits))
    g = gate(h_need, bf16_bits_to_f64(w_gate_bits))
    u = g[:, None] * v

    out = np.zeros((len(want), H), dtype=np.float64)
    for i, t in enumerate(want):
        t = int(t)
        s, p = int(seq[t]), int(pos[t])
        window = np.zeros((4, H))
        for k in range(4):           # window[3-k] = u_{t-k}
            if p - k >= 0:
                window[3 - k] = u[idx_of[t - k]]
            else:
                window[3 - k] = conv0[s][3 + (p - k)]
        y = short_conv(window, conv_w)[0]
        out[i] = bf16_bits_to_f64(np.asarray(hidden_bits)[t]) + y

    u_full = np.zeros((T, H))
    u_full[need] = u
    res = dict(ids=ids, out=out)
    res["hist_out"], res["conv_out"] = end_state(tokens, offsets, u_full, hist, conv0)
    return res


def end_state(tokens, offsets, u, hist, conv0, lengths=None):
    """State after each sequence (C-12): the last two tokens (with carried ones
    if the sequence is shorter than two) and the last three u rows (with carried
    ones if it is shorter than three). ``lengths[s]`` (optional) commits only
    the first lengths[s] tokens of sequence s."""
    offsets = np.asarray(offsets, dtype=np.int64)
    S = offsets.shape[0] - 1
    H = u.shape[1]
    hist_out = np.full((S, 2), -1, dtype=np.int64)
    conv_out = np.zeros((S, 3, H))
    for s in range(S):
        a = int(offsets[s])
        n = int(offsets[s + 1]) - a if lengths is None else int(lengths[s])
        prev_tok = [-1, -1] if hist is None else [int(hist[s][0]), int(hist[s][1])]
        toks = prev_tok + [int(x) for x in tokens[a:a + n]]
        hist_out[s] = toks[-2:]
        rows = np.concatenate([conv0[s], u[a:a + n]], axis=0)
        conv_out[s] = rows[-3:]
    return hist_out, conv_out


def ple_decode_step(tokens_bq, hidden_bits, w_proj_bits, w_gate_bits, conv_w, table, rows,
                    hist, conv_state, n_commit=None):
    """One decode / MTP-verify step: B sequences with q new tokens each.

    Outputs are produced for all q tokens of every sequence; the carried state
    advances by the first n_commit[b] tokens only (None = all q)."""
    tokens_bq = np.asarray(tokens_bq)
    B, q = tokens_bq.shape
    offsets = np.arange(B + 1, dtype=np.int64) * q
    flat = tokens_bq.reshape(-1)
    res = ple_forward(flat, offsets, hidden_bits, w_proj_bits, w_gate_bits, conv_w, table,
                      rows, hist=hist, conv_state=conv_state)
    # recompute u for the state update (the same definition as inside ple_forward)
    ids = res["ids"]
    u = gate(bf16_bits_to_f64(hidden_bits), bf16_bits_to_f64(w_gate_bits))[:, None] * \
        project(embed(table, ids), bf16_bits_to_f64(w_proj_bits))
    lengths = np.full(B, q) if n_commit is None else np.asarray(n_commit)
    hist_out, conv_out = end_state(flat, offsets, u, hist,
                                   np.asarray(conv_state, np.float64), lengths=lengths)
    return dict(ids=ids, out=res["out"], hist_out=hist_out, conv_out=conv_out)
