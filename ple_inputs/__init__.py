"""Seeded synthetic inputs for the PLE n-gram embedding layer.

This module is shared by the CPU oracle's tests and by the GPU tests / bench.
It holds *input generation only*: workload shapes, token streams, hidden
states, weights and the synthetic FP8 table. It contains none of the layer's
arithmetic (no hashing of n-grams, no dequantisation, no projection, gate,
convolution or residual).

The FP8 table of the full-scale workloads is 51,200,245,760 bytes, far too big
to build on the host, so its bytes are defined by a counter-based generator
(splitmix64, Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014): element ``i`` of stream ``tag`` is
``mix(base(seed, tag) + (i + 1) * GAMMA)``, the i-th output of a splitmix64
sequence. The host implementation below regenerates any rows on demand; the
CUDA implementation in ``csrc/ple_synth.cu`` fills the whole table in device
memory. Both follow this definition and are cross-checked bit for bit.

Workload sizes follow the deployment reports on Qwen3.8 Flash-Next's n-gram
embedding ("PLE"): a 51,200,245,760-byte FP8 table (deletoe.com page,
"第四条路" section; bittide.aicompass.dev page, "模型简介"), hidden size 2560,
prefill chunks of 16,384 tokens (kipfel.ltd page, section 5, launch flags),
MTP with 2 speculative tokens and per-position acceptance 0.68-0.73 / 0.42-0.47
(kipfel.ltd page, thorbench table).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "GAMMA", "splitmix64_stream", "table_codes", "table_scales", "SynthTable",
    "f32_to_bf16_bits", "Weights", "make_weights", "tokens_uniform", "tokens_zipf",
    "hidden_bf16", "WORKLOADS", "Workload", "workload", "prefill_batch",
    "decode_batch", "long_chunks", "mtp_session", "fill_table_device", "nv_table_codes",
    "nv_table_block_scales", "SynthNvTable", "fill_nv_table_device",
]

_U64 = np.uint64
GAMMA = 0x9E3779B97F4A7C15          # splitmix64 increment (odd 64-bit golden ratio)
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB
TAG_CODES = 1
TAG_SCALES = 2
TAG_NV_CODES = 3                     # NVFP4 table: packed E2M1 code bytes
TAG_NV_BLOCKS = 4                    # NVFP4 table: E4M3 block-scale bytes
NV_BLOCK_BASE = 0x30                 # block-scale codes 0x30..0x3F: E4M3 0.5 .. 1.875
N_FINITE_E4M3 = 254                  # 256 codes minus the two NaN codes 0x7F / 0xFF


def _mix(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on uint64 arrays (wrap-around arithmetic)."""
    z = np.asarray(z, dtype=_U64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> _U64(30))) * _U64(_MIX1)
        z = (z ^ (z >> _U64(27))) * _U64(_MIX2)
    return z ^ (z >> _U64(31))


def stream_base(seed: int, tag: int) -> int:
    """Starting state of stream ``tag`` for ``seed``."""
    s = (int(seed) ^ (int(tag) << 32)) & 0xFFFFFFFFFFFFFFFF
    return int(_mix(np.array([s], dtype=_U64))[0])


def splitmix64_stream(seed: int, tag: int, index: np.ndarray) -> np.ndarray:
    """Element ``index`` (uint64 array) of the splitmix64 sequence of (seed, tag)."""
    base = _U64(stream_base(seed, tag))
    idx = np.asarray(index, dtype=_U64)
    with np.errstate(over="ignore"):
        z = base + (idx + _U64(1)) * _U64(GAMMA)
    return _mix(z)


def _u64_to_code(u: np.ndarray) -> np.ndarray:
    """Map uint64 draws uniformly onto the 254 finite E4M3 byte codes.

    ``i = ((u >> 32) * 254) >> 32`` lies in [0, 254); codes 0x00..0x7E take
    i < 127 and codes 0x80..0xFE take the rest, skipping the NaN code 0x7F.
    """
    with np.errstate(over="ignore"):
        i = ((u >> _U64(32)) * _U64(N_FINITE_E4M3)) >> _U64(32)
    i = i.astype(np.int64)
    return (i + (i >= 127)).astype(np.uint8)


def _u64_to_scale(u: np.ndarray) -> np.ndarray:
    """Map uint64 draws onto fp32 scales in [0.01, 0.1): float32(0.01 + 0.09 * f),
    f = (u >> 40) / 2**24, evaluated in double and rounded once to fp32."""
    f = (u >> _U64(40)).astype(np.float64) * (2.0 ** -24)
    return (0.01 + 0.09 * f).astype(np.float32)


def table_codes(seed: int, rows_per_order: int, row_dim: int, order: int,
                rows: np.ndarray) -> np.ndarray:
    """FP8 codes of the given rows of sub-table ``order``: uint8 [len(rows)][row_dim].

    Byte k of row r of order n has counter index ((n * R + r) * D + k)."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    base = (np.int64(order) * np.int64(rows_per_order) + rows) * np.int64(row_dim)
    idx = base[:, None] + np.arange(row_dim, dtype=np.int64)[None, :]
    return _u64_to_code(splitmix64_stream(seed, TAG_CODES, idx.astype(_U64)))


def table_scales(seed: int, rows_per_order: int, order: int,
                 rows: np.ndarray) -> np.ndarray:
    """Per-row fp32 scales of the given rows of sub-table ``order``."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    idx = np.int64(order) * np.int64(rows_per_order) + rows
    return _u64_to_scale(splitmix64_stream(seed, TAG_SCALES, idx.astype(_U64)))


def nv_table_codes(seed: int, rows_per_order: int, row_dim: int, order: int,
                   rows: np.ndarray) -> np.ndarray:
    """Packed NVFP4 code bytes (two E2M1 codes each, all 16 codes equally likely)
    of the given rows of sub-table ``order``: uint8 [len(rows)][row_dim / 2].

    Byte k of row r of order n is the top byte of counter index ((n * R + r) * D/2 + k)."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    half = row_dim // 2
    base = (np.int64(order) * np.int64(rows_per_order) + rows) * np.int64(half)
    idx = base[:, None] + np.arange(half, dtype=np.int64)[None, :]
    return (splitmix64_stream(seed, TAG_NV_CODES, idx.astype(_U64)) >> _U64(56)).astype(np.uint8)


def nv_table_block_scales(seed: int, rows_per_order: int, row_dim: int, order: int,
                          rows: np.ndarray) -> np.ndarray:
    """E4M3 block-scale bytes (codes 0x30..0x3F, i.e. 0.5 .. 1.875) of the given rows:
    uint8 [len(rows)][row_dim / 16]. Byte j of row r of order n is drawn from counter
    index ((n * R + r) * D/16 + j): NV_BLOCK_BASE + the draw's top 4 bits."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    nb = row_dim // 16
    base = (np.int64(order) * np.int64(rows_per_order) + rows) * np.int64(nb)
    idx = base[:, None] + np.arange(nb, dtype=np.int64)[None, :]
    u = splitmix64_stream(seed, TAG_NV_BLOCKS, idx.astype(_U64))
    return (np.uint64(NV_BLOCK_BASE) + (u >> _U64(60))).astype(np.uint8)


@dataclass
class SynthTable:
    """Host view of the synthetic table [2][R][D] + scales [2][R] (rows made on demand)."""
    seed: int
    rows_per_order: int
    row_dim: int

    def codes(self, order: int, rows) -> np.ndarray:
        return table_codes(self.seed, self.rows_per_order, self.row_dim, order, rows)

    def scales(self, order: int, rows) -> np.ndarray:
        return table_scales(self.seed, self.rows_per_order, order, rows)

    def full(self):
        """The whole table as arrays (small tables only)."""
        r = np.arange(self.rows_per_order)
        if self.rows_per_order * self.row_dim > (1 << 28):
            raise ValueError("table too large to materialise on the host")
        codes = np.stack([self.codes(0, r), self.codes(1, r)])
        scales = np.stack([self.scales(0, r), self.scales(1, r)])
        return codes, scales


@dataclass
class SynthHeadsTable:
    """Host view of a synthetic table of the multi-head layout: 2 * heads sub-tables
    of ``rows_per_head`` rows of ``head_dim`` FP8 codes, one fp32 scale per row.
    Code k of row r of sub-table h has counter index ((h * R' + r) * head_dim + k),
    so the bytes are those of the [2][heads * R'][head_dim] table the device filler
    writes."""
    seed: int
    rows_per_head: int
    head_dim: int
    heads_per_order: int = 8
    format: str = "heads"

    def codes(self, head: int, rows) -> np.ndarray:
        return table_codes(self.seed, self.rows_per_head, self.head_dim, head, rows)

    def scales(self, head: int, rows) -> np.ndarray:
        return table_scales(self.seed, self.rows_per_head, head, rows)

    def full(self):
        """codes [2 * heads][R'][head_dim], scales [2 * heads][R'] (small tables only)."""
        r = np.arange(self.rows_per_head)
        n = 2 * self.heads_per_order
        if n * self.rows_per_head * self.head_dim > (1 << 28):
            raise ValueError("table too large to materialise on the host")
        return (np.stack([self.codes(h, r) for h in range(n)]), np.stack([self.scales(h, r) for h in range(n)]))


@dataclass
class SynthNvTable:
    """Host view of a synthetic NVFP4 table: packed codes [2][R][D/2], E4M3 block
    scales [2][R][D/16] and the same per-row fp32 scales as the FP8 table."""
    seed: int
    rows_per_order: int
    row_dim: int
    format: str = "nvfp4"

    def codes(self, order: int, rows) -> np.ndarray:
        return nv_table_codes(self.seed, self.rows_per_order, self.row_dim, order, rows)

    def block_scales(self, order: int, rows) -> np.ndarray:
        return nv_table_block_scales(self.seed, self.rows_per_order, self.row_dim, order, rows)

    def scales(self, order: int, rows) -> np.ndarray:
        return table_scales(self.seed, self.rows_per_order, order, rows)

    def packed_rows(self, order: int, rows) -> np.ndarray:
        """The given rows as the row-by-row layout stores them: uint8 [len(rows)][9D/16],
        each row's D/2 code bytes followed by its D/16 block-scale bytes."""
        return np.concatenate([self.codes(order, rows), self.block_scales(order, rows)], axis=1)

    def full(self):
        """The whole table as arrays (small tables only): codes, block scales, scales."""
        r = np.arange(self.rows_per_order)
        if self.rows_per_order * self.row_dim > (1 << 28):
            raise ValueError("table too large to materialise on the host")
        return (np.stack([self.codes(0, r), self.codes(1, r)]),
                np.stack([self.block_scales(0, r), self.block_scales(1, r)]),
                np.stack([self.scales(0, r), self.scales(1, r)]))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest even) and return the uint16 bit patterns.
    Used to make bf16 inputs; inputs are finite by construction."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    # finite inputs only: the largest finite pattern plus 0x8000 stays below 2**32
    b = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return b.astype(np.uint16)


@dataclass
class Weights:
    """Layer parameters as stored for the library: bf16 bit patterns / fp32."""
    w_proj: np.ndarray   # uint16 (bf16 bits) [D][H]
    w_gate: np.ndarray   # uint16 (bf16 bits) [H]
    conv_w: np.ndarray   # float32 [H][4]; tap 3 multiplies the current token


def make_weights(seed: int, row_dim: int, hidden: int) -> Weights:
    """W_proj and w_gate ~ N(0, 0.02) in bf16; conv taps ~ N(0, 0.5) in fp32."""
    rng = np.random.default_rng([seed, 101])
    w_proj = f32_to_bf16_bits(rng.normal(0.0, 0.02, size=(row_dim, hidden)).astype(np.float32))
    w_gate = f32_to_bf16_bits(rng.normal(0.0, 0.02, size=(hidden,)).astype(np.float32))
    conv_w = rng.normal(0.0, 0.5, size=(hidden, 4)).astype(np.float32)
    return Weights(w_proj, w_gate, conv_w)


def tokens_uniform(rng: np.random.Generator, n: int, vocab: int) -> np.ndarray:
    return rng.integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


_ZIPF_CDF: dict = {}


def tokens_zipf(rng: np.random.Generator, n: int, vocab: int, s: float = 1.1) -> np.ndarray:
    """Zipf(s) truncated to the vocabulary: P(rank k) ~ k^-s, token = k - 1
    (inverse-CDF draw). A stand-in for text, whose frequent n-grams repeat rows."""
    key = (vocab, s)
    if key not in _ZIPF_CDF:
        w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
        c = np.cumsum(w)
        _ZIPF_CDF[key] = c / c[-1]
    cdf = _ZIPF_CDF[key]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int32)


def hidden_bf16(rng: np.random.Generator, n_tokens: int, hidden: int) -> np.ndarray:
    """Hidden states ~ N(0, 1) rounded to bf16: uint16 bits [n_tokens][hidden]."""
    return f32_to_bf16_bits(rng.standard_normal((n_tokens, hidden), dtype=np.float32))


@dataclass(frozen=True)
class Workload:
    name: str
    vocab: int
    rows_per_order: int
    row_dim: int
    hidden: int
    table_seed: int
    seed: int
    extra: dict = field(default_factory=dict, hash=False, compare=False)

    def table(self) -> SynthTable:
        return SynthTable(self.table_seed, self.rows_per_order, self.row_dim)

    def heads_table(self, heads_per_order: int = 8) -> "SynthHeadsTable":
        """The table of the multi-head layout: rows_per_order is then the rows per
        head sub-table, and row_dim the width of e (2 * heads rows side by side)."""
        return SynthHeadsTable(self.table_seed, self.rows_per_order, self.row_dim // (2 * heads_per_order),
                               heads_per_order)

    def weights(self) -> Weights:
        return make_weights(self.table_seed, self.row_dim, self.hidden)

    @property
    def table_bytes(self) -> int:
        return 2 * self.rows_per_order * self.row_dim


FULL_VOCAB = 248_320
FULL_ROWS = 10_000_048
FULL_DIM = 2560
FULL_TABLE_SEED = 1      # one table and one set of weights for every full-scale workload

WORKLOADS = {
    "tiny": Workload("tiny", 1000, 4096, 64, 128, table_seed=0, seed=0,
                     extra=dict(T=256)),
    "decode": Workload("decode", FULL_VOCAB, FULL_ROWS, FULL_DIM, FULL_DIM,
                       FULL_TABLE_SEED, seed=1, extra=dict(B=8, q=1)),
    "prefill": Workload("prefill", FULL_VOCAB, FULL_ROWS, FULL_DIM, FULL_DIM,
                        FULL_TABLE_SEED, seed=2,
                        extra=dict(lengths=(1000, 3384, 4000, 8000))),
    "long": Workload("long", FULL_VOCAB, FULL_ROWS, FULL_DIM, FULL_DIM,
                     FULL_TABLE_SEED, seed=3, extra=dict(total=262_144, chunk=16_384)),
    "mtp": Workload("mtp", FULL_VOCAB, FULL_ROWS, FULL_DIM, FULL_DIM,
                    FULL_TABLE_SEED, seed=4,
                    extra=dict(B=64, q=3, steps=100, shared=19, prefix=512,
                               p_accept=(0.70, 0.45))),
}


# The multi-head layout (16 sub-tables of 20,000,096 rows x 160 codes: the same
# 51,200,245,760 bytes as the two-order table) and a small one for the tests.
HEADS_FULL_ROWS = 20_000_096
HEADS_WORKLOADS = {
    "heads_tiny": Workload("heads_tiny", 1000, 512, 256, 128, table_seed=5, seed=5),
    "heads_full": Workload("heads_full", FULL_VOCAB, HEADS_FULL_ROWS, FULL_DIM, FULL_DIM, FULL_TABLE_SEED, seed=6),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name] if name in WORKLOADS else HEADS_WORKLOADS[name]


def prefill_batch(w: Workload, variant: int = 0, lengths=None, zipf: bool = True):
    """Packed prefill batch: tokens int32 [T], offsets int32 [S+1], hidden bf16 bits [T][H]."""
    rng = np.random.default_rng([w.seed, 7, variant])
    lengths = list(lengths if lengths is not None else w.extra.get("lengths", (w.extra.get("T", 256),)))
    offsets = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    T = int(offsets[-1])
    if zipf:
        tokens = tokens_zipf(rng, T, w.vocab)
    else:
        tokens = tokens_uniform(rng, T, w.vocab)
    hidden = hidden_bf16(rng, T, w.hidden)
    return tokens, offsets, hidden


def tiny_batch(w: Workload):
    """One sequence of T uniform tokens (the tiny workload)."""
    rng = np.random.default_rng([w.seed, 7])
    T = w.extra["T"]
    tokens = tokens_uniform(rng, T, w.vocab)
    offsets = np.array([0, T], dtype=np.int32)
    hidden = hidden_bf16(rng, T, w.hidden)
    return tokens, offsets, hidden


def decode_batch(w: Workload, variant: int = 0, B=None, q=None):
    """Decode step: tokens int32 [B][q], hidden [B*q][H], carried history int32 [B][2]
    (two uniform tokens) and conv state float32 [B][3][H] ~ N(0, 1)."""
    rng = np.random.default_rng([w.seed, 11, variant])
    B = B or w.extra["B"]
    q = q or w.extra["q"]
    tokens = tokens_uniform(rng, B * q, w.vocab).reshape(B, q)
    hist = tokens_uniform(rng, 2 * B, w.vocab).reshape(B, 2)
    conv = rng.standard_normal((B, 3, w.hidden), dtype=np.float32)
    hidden = hidden_bf16(rng, B * q, w.hidden)
    return tokens, hidden, hist, conv


def long_chunks(w: Workload, n_chunks=None, chunk=None):
    """The long-context sequence (uniform tokens): yields (tokens [chunk], hidden [chunk][H])."""
    chunk = chunk or w.extra["chunk"]
    n_chunks = n_chunks or w.extra["total"] // chunk
    rng = np.random.default_rng([w.seed, 13])
    for _ in range(n_chunks):
        yield tokens_uniform(rng, chunk, w.vocab), hidden_bf16(rng, chunk, w.hidden)


def mtp_session(w: Workload, steps=None, B=None, q=None, prefix=None):
    """MTP-style decode session.

    Returns a dict with the prompts (int32 [B][prefix]), and per step the tokens
    int32 [B][q], hidden bf16 bits [B*q][H] and n_commit int32 [B].
    The first ``shared`` sequences share one Zipf prompt, identical
    continuations and identical hidden states (duplicated greedy requests);
    the rest are independent Zipf.
    n_commit = 1 + Bern(0.70) * (1 + Bern(0.45)) per sequence and step, from the
    per-position draft acceptance measured on the kipfel.ltd page (section 6).
    """
    B = B or w.extra["B"]
    q = q or w.extra["q"]
    steps = steps or w.extra["steps"]
    prefix = prefix or w.extra["prefix"]
    shared = min(w.extra["shared"], B)
    p1, p2 = w.extra["p_accept"]
    rng = np.random.default_rng([w.seed, 17])
    prompts = tokens_zipf(rng, B * prefix, w.vocab).reshape(B, prefix)
    prompts[:shared] = prompts[0]
    prompt_hidden = hidden_bf16(rng, B * prefix, w.hidden).reshape(B, prefix, w.hidden)
    prompt_hidden[:shared] = prompt_hidden[0]
    prompt_hidden = prompt_hidden.reshape(B * prefix, w.hidden)
    out_steps = []
    for _ in range(steps):
        toks = tokens_zipf(rng, B * q, w.vocab).reshape(B, q)
        toks[:shared] = toks[0]
        acc1 = rng.random(B) < p1
        acc2 = rng.random(B) < p2
        n_commit = (1 + acc1 * (1 + acc2)).astype(np.int32)
        n_commit[:shared] = n_commit[0]
        n_commit = np.minimum(n_commit, q)
        hid = hidden_bf16(rng, B * q, w.hidden).reshape(B, q, w.hidden)
        hid[:shared] = hid[0]                 # duplicated requests see identical hidden states
        out_steps.append((toks, hid.reshape(B * q, w.hidden), n_commit))
    return dict(prompts=prompts, prompt_hidden=prompt_hidden, steps=out_steps)


# --------------------------------------------------------------------------------------
# Device-side table filler (CUDA, built into ple_inputs/libple_synth.so)
# --------------------------------------------------------------------------------------
_SYNTH_LIB = None


def _synth_lib():
    global _SYNTH_LIB
    if _SYNTH_LIB is None:
        path = os.path.join(os.path.dirname(__file__), "libple_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.ple_synth_fill_table.restype = ctypes.c_int
        lib.ple_synth_fill_table.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int32, ctypes.c_uint64, ctypes.c_void_p]
        lib.ple_synth_fill_nvfp4.restype = ctypes.c_int
        lib.ple_synth_fill_nvfp4.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                             ctypes.c_int32, ctypes.c_uint64, ctypes.c_void_p]
        lib.ple_synth_fill_nvfp4_rows.restype = ctypes.c_int
        lib.ple_synth_fill_nvfp4_rows.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                                  ctypes.c_uint64, ctypes.c_void_p]
        lib.ple_synth_stream_base.restype = ctypes.c_uint64
        lib.ple_synth_stream_base.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
        _SYNTH_LIB = lib
    return _SYNTH_LIB


def fill_nv_table_device(codes_ptr: int, block_ptr: int, scales_ptr: int, rows_per_order: int,
                         row_dim: int, seed: int, stream: int = 0) -> None:
    """Fill a device NVFP4 table: codes u8[2][R][D/2], block scales u8[2][R][D/16], scales f32[2][R]."""
    rc = _synth_lib().ple_synth_fill_nvfp4(ctypes.c_void_p(codes_ptr), ctypes.c_void_p(block_ptr),
                                           ctypes.c_void_p(scales_ptr), rows_per_order, row_dim, seed,
                                           ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ple_synth_fill_nvfp4 failed with CUDA error {rc}")


def fill_nv_rows_table_device(rows_ptr: int, scales_ptr: int, rows_per_order: int, row_dim: int, seed: int,
                              stream: int = 0) -> None:
    """Fill a device NVFP4 table stored row by row, u8[2][R][9D/16] (each row's D/2 code
    bytes, then its D/16 block-scale bytes: the contents of fill_nv_table_device), and
    scales f32[2][R]."""
    rc = _synth_lib().ple_synth_fill_nvfp4_rows(ctypes.c_void_p(rows_ptr), ctypes.c_void_p(scales_ptr),
                                                rows_per_order, row_dim, seed, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ple_synth_fill_nvfp4_rows failed with CUDA error {rc}")


def fill_table_device(table_ptr: int, scales_ptr: int, rows_per_order: int, row_dim: int,
                      seed: int, stream: int = 0) -> None:
    """Fill a device table u8[2][R][D] and scales f32[2][R] with the synthetic contents."""
    rc = _synth_lib().ple_synth_fill_table(ctypes.c_void_p(table_ptr), ctypes.c_void_p(scales_ptr),
                                           rows_per_order, row_dim, seed, ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"ple_synth_fill_table failed with CUDA error {rc}")
