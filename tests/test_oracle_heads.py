"""Pins of the oracle's multi-head row layout (reading C-17), CPU only.

The SSD-stream model card ("Qwen3.8 Flash-Next NVFP4 - SSD Stream", section
"技术细节") states 16 table lookups per token of 160-byte FP8 rows. The oracle
reads that as 8 hash heads per order: head j of order n takes sub-table 8n + j
at row fold(k_n ^ j * HEAD_MIX) mod R', and e is the 16 dequantised rows
side by side. Each pin ties the layout to something other than itself: head
0 to the already pinned two-order row IDs, the dependence on the text to the
pages' statements, the concatenation to planted tables and the dequantisation
to torch's float8 decoding; a scalar brute force covers the whole layer.
"""
import math

import numpy as np
import torch

import oracle as O
import ple_inputs as pi

R_HEAD = 4099          # rows per head sub-table (odd, so the row spread is exercised)


def _ids(toks, offsets=None, hist=None, rows=R_HEAD):
    toks = np.asarray(toks)
    offsets = [0, len(toks)] if offsets is None else offsets
    return O.ngram_ids_heads(toks, offsets, rows, hist)


def test_head_zero_is_the_two_order_row():
    """Head 0 of each order mixes in 0, so it is the C-4 row of that order."""
    rng = np.random.default_rng(1)
    toks = rng.integers(0, 248_320, 300)
    offs = [0, 1, 2, 150, 300]
    heads = O.ngram_ids_heads(toks, offs, R_HEAD)
    pairs = O.ngram_ids(toks, offs, R_HEAD)
    assert heads.shape == (300, 16)
    assert np.array_equal(heads[:, 0], pairs[:, 0])
    assert np.array_equal(heads[:, 8], pairs[:, 1])
    # the other heads are different rows of the same context
    assert (heads[:, 1:8] != heads[:, :1]).mean() > 0.99
    assert (heads[:, 9:] != heads[:, 8:9]).mean() > 0.99


def test_heads_dependence_structure():
    """Bigram heads follow (t, t-1) only; trigram heads (t, t-1, t-2) only."""
    base = [11, 22, 33, 44, 55]
    ref = _ids(base)
    for changed, bigram_changes, trigram_changes in [(4, True, True), (3, True, True),
                                                     (2, False, True), (1, False, False)]:
        toks = list(base)
        toks[changed] += 1000
        got = _ids(toks)
        assert np.all((got[4, :8] != ref[4, :8]) == bigram_changes), changed
        assert np.all((got[4, 8:] != ref[4, 8:]) == trigram_changes), changed


def test_heads_identical_contexts_identical_rows():
    toks = [7, 8, 9, 1, 7, 8, 9, 2, 8, 9]
    ids = _ids(toks)
    assert np.array_equal(ids[2], ids[6])          # same (7, 8, 9)
    assert np.array_equal(ids[9, :8], ids[6, :8])  # same bigram (8, 9)
    assert np.all(ids[9, 8:] != ids[6, 8:])        # different t-2


def test_heads_boundaries_and_carried_history():
    packed = _ids([5, 6, 7, 8, 9], offsets=[0, 2, 5])
    assert np.array_equal(packed[:2], _ids([5, 6]))
    assert np.array_equal(packed[2:], _ids([7, 8, 9]))
    toks = [3, 1, 4, 1, 5, 9, 2, 6]
    whole = _ids(toks)
    for cut in range(1, len(toks)):
        prev = ([-1] + toks[:cut])[-2:]
        b = _ids(toks[cut:], hist=np.array([prev]))
        assert np.array_equal(np.concatenate([_ids(toks[:cut]), b]), whole), cut


def test_heads_range_and_spread():
    """Every head's rows lie in [0, R') and spread over it (chi-square)."""
    rng = np.random.default_rng(5)
    toks = rng.integers(0, 248_320, size=12_000)
    R_ = 2048
    ids = _ids(toks, rows=R_)
    assert ids.min() >= 0 and ids.max() < R_
    for h in range(16):
        counts = np.bincount(ids[:, h], minlength=R_)
        chi2 = ((counts - counts.mean()) ** 2 / counts.mean()).sum()
        assert chi2 < R_ + 6 * math.sqrt(2 * R_), h


def _heads_table(seed=3, R_=32, hd=16):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(16, R_, hd)).astype(np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    scales = rng.uniform(0.01, 0.1, size=(16, R_)).astype(np.float32)
    return codes, scales


def test_heads_embed_concatenates_in_head_order():
    """A table whose sub-table h holds one code c_h everywhere (scale 1) gives an e
    whose slice h is e4m3(c_h): catches a wrong head order or slice width."""
    hd, R_ = 16, 8
    cs = np.array([0x38 + h for h in range(16)], np.uint8)        # 1.0, 1.125, ... distinct values
    codes = np.broadcast_to(cs[:, None, None], (16, R_, hd)).copy()
    tab = O.HeadsArrayTable(codes, np.ones((16, R_), np.float32))
    ids = np.arange(16)[None, :].repeat(3, 0) % R_
    e = O.embed(tab, ids)
    assert e.shape == (3, 16 * hd)
    vals = torch.from_numpy(cs).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for h in range(16):
        assert np.all(e[:, h * hd:(h + 1) * hd] == vals[h])


def test_heads_dequantise_matches_torch_float8_times_scale():
    codes, scales = _heads_table()
    tab = O.HeadsArrayTable(codes, scales)
    rng = np.random.default_rng(8)
    ids = rng.integers(0, 32, size=(5, 16))
    e = O.embed(tab, ids)
    f8 = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for i in range(5):
        expect = np.concatenate([f8[h, ids[i, h]] * np.float64(scales[h, ids[i, h]]) for h in range(16)])
        assert np.array_equal(e[i], expect)


def test_synthetic_heads_table_is_the_two_order_table_reshaped():
    """The synthetic multi-head table has the bytes of a [2][8R'][hd] two-order
    table (the device filler writes that shape)."""
    w = pi.workload("heads_tiny")
    ht = w.heads_table()
    pt = pi.SynthTable(w.table_seed, 8 * w.rows_per_order, w.row_dim // 16)
    codes, scales = ht.full()
    pc, ps = pt.full()
    assert np.array_equal(codes.reshape(2, -1, w.row_dim // 16), pc)
    assert np.array_equal(scales.reshape(2, -1), ps)


def _brute_force_heads(tokens, hidden, codes, scales, w_proj, w_gate, conv_w):
    """Scalar loops over one fresh sequence with the multi-head layout."""
    T, H = hidden.shape
    nh, R_, hd = codes.shape
    M = 1 << 64

    def ctx(i):
        return int(tokens[i]) + 1 if i >= 0 else 0

    u = [[0.0] * H for _ in range(T)]
    for t in range(T):
        k2 = (ctx(t) * 0x9E3779B97F4A7C15 % M) ^ (ctx(t - 1) * 0xC2B2AE3D27D4EB4F % M)
        k3 = k2 ^ (ctx(t - 2) * 0x165667B19E3779F9 % M)
        e = []
        for h in range(nh):
            k = (k2 if h < nh // 2 else k3) ^ ((h % (nh // 2)) * 0xFF51AFD7ED558CCD % M)
            r = (k ^ (k >> 32)) % R_
            e += [O.e4m3_decode(codes[h, r, c]) * float(scales[h, r]) for c in range(hd)]
        a = sum(float(w_gate[j]) * float(hidden[t, j]) for j in range(H))
        g = 1.0 / (1.0 + math.exp(-a))
        for j in range(H):
            u[t][j] = g * sum(e[k] * float(w_proj[k, j]) for k in range(len(e)))
    out = np.zeros((T, H))
    for t in range(T):
        for j in range(H):
            y = sum(float(conv_w[j, k]) * u[t - 3 + k][j] for k in range(4) if t - 3 + k >= 0)
            out[t, j] = float(hidden[t, j]) + y
    return out


def test_heads_layer_matches_brute_force():
    w = pi.workload("heads_tiny")
    codes, scales = w.heads_table().full()
    tab = O.HeadsArrayTable(codes, scales)
    W = w.weights()
    rng = np.random.default_rng(4)
    T = 6
    toks = rng.integers(0, w.vocab, T)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    r = O.ple_forward(toks, [0, T], hid, W.w_proj, W.w_gate, W.conv_w, tab, w.rows_per_order)
    assert r["ids"].shape == (T, 16)
    bf = _brute_force_heads(toks, O.bf16_bits_to_f64(hid), codes, scales, O.bf16_bits_to_f64(W.w_proj),
                            O.bf16_bits_to_f64(W.w_gate), W.conv_w)
    assert np.allclose(r["out"], bf, rtol=1e-12, atol=1e-12)


def test_heads_layer_decode_steps_equal_prefill():
    """Decode by single steps with the carried state == one prefill, on the multi-head layout."""
    w = pi.workload("heads_tiny")
    tab = O.HeadsArrayTable(*w.heads_table().full())
    W = w.weights()
    rng = np.random.default_rng(6)
    T = 9
    toks = rng.integers(0, w.vocab, T)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    whole = O.ple_forward(toks, [0, T], hid, W.w_proj, W.w_gate, W.conv_w, tab, w.rows_per_order)
    pre = O.ple_forward(toks[:5], [0, 5], hid[:5], W.w_proj, W.w_gate, W.conv_w, tab, w.rows_per_order)
    hist, conv = pre["hist_out"], pre["conv_out"]
    outs = [pre["out"]]
    for t in range(5, T):
        d = O.ple_decode_step(toks[t:t + 1][None, :], hid[t:t + 1], W.w_proj, W.w_gate, W.conv_w, tab,
                              w.rows_per_order, hist, conv)
        outs.append(d["out"])
        hist, conv = d["hist_out"], d["conv_out"]
    assert np.allclose(np.concatenate(outs), whole["out"], rtol=1e-12, atol=1e-12)
