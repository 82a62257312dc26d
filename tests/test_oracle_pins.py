"""Pins of the CPU oracle against things other than itself (CPU only).

Each pin ties one step of the oracle to a library routine, a closed form, a
special case, an invariant the pages state, or a brute-force evaluation, so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them (``test_oracle_mutations.py`` plants such
mistakes and checks that they are caught).
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import ple_inputs as pi


# ------------------------------------------------------------------ E4M3 decoding (C-5)
def test_e4m3_all_codes_match_torch_float8():
    """All 256 codes: closed form vs torch.float8_e4m3fn decoding (library routine)."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.E4M3_VALUES
    nan_lib = np.isnan(lib)
    assert np.array_equal(nan_lib, np.isnan(ours))
    assert nan_lib.sum() == 2 and nan_lib[0x7F] and nan_lib[0xFF]
    assert np.array_equal(lib[~nan_lib], ours[~nan_lib])


@pytest.mark.parametrize("code,value", [
    (0x7E, 448.0), (0xFE, -448.0), (0x38, 1.0), (0xB8, -1.0), (0x01, 2.0 ** -9),
    (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x00, 0.0), (0x40, 2.0), (0x30, 0.5),
])
def test_e4m3_spot_values(code, value):
    """Values fixed by the OCP FP8 E4M3 format: max 448, min subnormal 2^-9, 1.0 = 0x38."""
    assert O.e4m3_decode(code) == value


def test_e4m3_negative_zero():
    v = O.e4m3_decode(0x80)
    assert v == 0.0 and math.copysign(1.0, v) == -1.0


# ------------------------------------------------------------------ sequence map (C-1)
def test_sequence_map_brute_force():
    offsets = [0, 3, 3, 7, 8]
    seq, pos = O.sequence_map(offsets, 8)
    expect = [(0, 0), (0, 1), (0, 2), (2, 0), (2, 1), (2, 2), (2, 3), (3, 0)]
    assert list(zip(seq.tolist(), pos.tolist())) == expect


# ------------------------------------------------------------------ n-gram IDs (C-2..C-4)
R = 1_000_003


def _ids(tokens, offsets=None, hist=None, rows=R):
    offsets = [0, len(tokens)] if offsets is None else offsets
    return O.ngram_ids(np.array(tokens, dtype=np.int32), offsets, rows, hist)


def test_hash_multiplier_is_the_golden_ratio_constant():
    """P0 is floor(2^64 (sqrt 5 - 1) / 2), the multiplier of Knuth's multiplicative
    hashing, computed here in exact integer arithmetic. P1 and P2 are odd, so each
    product is a bijection of the 64-bit contexts."""
    assert O.P0 == (math.isqrt(5 << 128) - (1 << 64)) // 2
    assert O.P1 % 2 == 1 and O.P2 % 2 == 1


def test_ids_match_the_hash_worked_example():
    """The row IDs of the worked example in ``tests/golden/hash_worked_example.txt``, written
    down from the hash definition in exact integer arithmetic before the oracle existed.
    This pins every constant and step of the hash (all three multipliers, the context offset,
    the fold, the mod) from outside the oracle: a one-digit change to any of them moves some
    row. Positions 2 and 4 share the bigram context (17, 42) and so the bigram row, while
    their trigram rows differ; at the first two positions the trigram key equals the bigram
    key."""
    from tests.test_golden import hash_worked_example
    for rows, toks, expect in hash_worked_example():
        got = [tuple(int(v) for v in r) for r in _ids(toks, rows=rows)]
        assert got == expect, (rows, toks)


def test_ids_dependence_structure():
    """Bigram row depends on (t, t-1) only; trigram row on (t, t-1, t-2) only."""
    base = [11, 22, 33, 44, 55]
    ref = _ids(base)
    for changed, bigram_changes, trigram_changes in [(4, True, True), (3, True, True),
                                                     (2, False, True), (1, False, False)]:
        toks = list(base)
        toks[changed] += 1000
        got = _ids(toks)
        assert (got[4, 0] != ref[4, 0]) == bigram_changes, changed
        assert (got[4, 1] != ref[4, 1]) == trigram_changes, changed


def test_ids_identical_contexts_identical_rows():
    """Identical n-gram contexts give identical rows (pages: rows depend only on the text)."""
    toks = [7, 8, 9, 1, 7, 8, 9, 2, 8, 9]
    ids = _ids(toks)
    assert tuple(ids[2]) == tuple(ids[6])          # same (7,8,9)
    assert ids[9, 0] == ids[6, 0]                  # same bigram (8,9)
    assert ids[9, 1] != ids[6, 1]                  # different t-2 (2 vs 7)


def test_ids_sequence_start_is_boundary():
    """No n-gram crosses a boundary: a token at a sequence start gets the same rows
    as the same token alone; inside, the first two tokens see absent context."""
    packed = _ids([5, 6, 7, 8, 9], offsets=[0, 2, 5])
    assert np.array_equal(packed[:2], _ids([5, 6]))
    assert np.array_equal(packed[2:], _ids([7, 8, 9]))
    assert not np.array_equal(packed[2:], _ids([5, 6, 7, 8, 9])[2:])
    # first token: x_{t-1} = x_{t-2} = 0 so k3 == k2 and, with equal table sizes, equal rows
    one = _ids([123])
    assert one[0, 0] == one[0, 1]
    # second token: x_{t-2} = 0 so again k3 == k2
    two = _ids([123, 456])
    assert two[1, 0] == two[1, 1]
    assert _ids([123, 456, 789])[2, 0] != _ids([123, 456, 789])[2, 1]


def test_ids_carried_history_equals_whole_sequence():
    """Chunked with the last two tokens carried == one whole sequence."""
    toks = [3, 1, 4, 1, 5, 9, 2, 6, 5, 3]
    whole = _ids(toks)
    for cut in range(1, len(toks)):
        a = _ids(toks[:cut])
        prev = ([-1] + toks[:cut])[-2:]
        b = _ids(toks[cut:], hist=np.array([prev]))
        assert np.array_equal(np.concatenate([a, b]), whole), cut


def test_ids_absent_history_is_fresh_sequence():
    toks = [10, 20, 30]
    assert np.array_equal(_ids(toks, hist=np.array([[-1, -1]])), _ids(toks))


def test_ids_range_and_spread():
    """Rows lie in [0, R) and distinct contexts spread over the table (chi-square)."""
    rng = np.random.default_rng(5)
    toks = rng.integers(0, 248_320, size=20_000)
    ids = _ids(toks, rows=4096)
    assert ids.min() >= 0 and ids.max() < 4096
    for n in range(2):
        counts = np.bincount(ids[:, n], minlength=4096)
        chi2 = ((counts - counts.mean()) ** 2 / counts.mean()).sum()
        assert chi2 < 4096 + 6 * math.sqrt(2 * 4096)


def test_ids_rows_per_order_differ():
    ids = O.ngram_ids(np.array([1, 2, 3]), [0, 3], (7, 1_000_003))
    assert ids[:, 0].max() < 7


def test_ids_independent_of_hidden():
    """Row IDs depend only on tokens and boundaries: the forward pass returns the
    same ids for any hidden state."""
    w = pi.workload("tiny")
    tab = O.ArrayTable(*w.table().full())
    W = w.weights()
    toks, offs, hid = pi.tiny_batch(w)
    r1 = O.ple_forward(toks[:32], [0, 32], hid[:32], W.w_proj, W.w_gate, W.conv_w, tab, 4096)
    hid2 = pi.hidden_bf16(np.random.default_rng(9), 32, w.hidden)
    r2 = O.ple_forward(toks[:32], [0, 32], hid2, W.w_proj, W.w_gate, W.conv_w, tab, 4096)
    assert np.array_equal(r1["ids"], r2["ids"])
    assert not np.array_equal(r1["out"], r2["out"])


# ------------------------------------------------------------------ dequant and order sum
def _small_table(seed=3, R_=64, D=16):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(2, R_, D)).astype(np.uint8)
    codes[codes == 0x7F] = 0x7E
    codes[codes == 0xFF] = 0xFE
    scales = rng.uniform(0.01, 0.1, size=(2, R_)).astype(np.float32)
    return codes, scales


def test_dequantise_matches_torch_float8_times_scale():
    codes, scales = _small_table()
    deq = O.dequantise(codes[0], scales[0])
    lib = torch.from_numpy(codes[0]).view(torch.float8_e4m3fn).to(torch.float64) * \
        torch.from_numpy(scales[0]).to(torch.float64)[:, None]
    assert np.array_equal(deq, lib.numpy())


def test_embed_sums_orders():
    codes, scales = _small_table()
    tab = O.ArrayTable(codes, scales)
    ids = np.array([[1, 2], [5, 5], [63, 0]])
    e = O.embed(tab, ids)
    f8 = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for i, (r0, r1) in enumerate(ids):
        expect = f8[0, r0] * np.float64(scales[0, r0]) + f8[1, r1] * np.float64(scales[1, r1])
        assert np.array_equal(e[i], expect)
    # zero trigram scales: e is the bigram row alone
    s2 = scales.copy()
    s2[1] = 0
    assert np.array_equal(O.embed(O.ArrayTable(codes, s2), ids), O.dequantise(codes[0][ids[:, 0]], scales[0][ids[:, 0]]))


# ------------------------------------------------------------------ projection
def test_projection_one_hot_picks_weight_row():
    rng = np.random.default_rng(1)
    W = rng.standard_normal((16, 24))
    e = np.zeros((3, 16))
    e[0, 0] = 1.0
    e[1, 15] = 1.0
    e[2, 7] = -2.0
    v = O.project(e, W)
    assert np.array_equal(v[0], W[0]) and np.array_equal(v[1], W[15]) and np.array_equal(v[2], -2 * W[7])


# ------------------------------------------------------------------ gate (C-8)
def test_gate_zero_weight_is_one_half():
    h = np.random.default_rng(2).standard_normal((5, 8))
    assert np.all(O.gate(h, np.zeros(8)) == 0.5)


def test_gate_sign():
    h = np.ones((1, 4))
    assert O.gate(h, np.full(4, 10.0))[0] > 0.999999
    assert O.gate(h, np.full(4, -10.0))[0] < 1e-6


# ------------------------------------------------------------------ short conv (C-9)
def test_short_conv_matches_numpy_convolve():
    """Causal width-4 conv == numpy.convolve per channel (library routine), zero history."""
    rng = np.random.default_rng(4)
    L, H = 11, 5
    u = rng.standard_normal((L, H))
    cw = rng.standard_normal((H, 4))
    y = O.short_conv(np.concatenate([np.zeros((3, H)), u]), cw)
    for j in range(H):
        # y_t = sum_k cw[k] u_{t-3+k} = sum_m cw[3-m] u_{t-m}  (m = lag)
        ref = np.convolve(u[:, j], cw[j, ::-1], mode="full")[:L]
        assert np.allclose(y[:, j], ref, rtol=0, atol=1e-12)


def test_short_conv_delta_is_identity_and_impulse_response():
    H = 3
    cw_delta = np.tile([0.0, 0.0, 0.0, 1.0], (H, 1))
    u = np.random.default_rng(6).standard_normal((9, H))
    assert np.array_equal(O.short_conv(np.concatenate([np.zeros((3, H)), u]), cw_delta), u)
    cw = np.array([[1.0, 2.0, 3.0, 4.0]] * H)
    imp = np.zeros((3 + 6, H))
    imp[3 + 1] = 1.0                      # impulse at t = 1
    y = O.short_conv(imp, cw)
    assert y[:, 0].tolist() == [0, 4, 3, 2, 1, 0]


# ------------------------------------------------------------------ whole layer
def _tiny_forward(toks, offs, hid, table=None, w=None, **kw):
    w = w or pi.workload("tiny")
    W = w.weights()
    table = table or O.ArrayTable(*w.table().full())
    return O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, table, w.rows_per_order, **kw)


def _brute_force_layer(tokens, hidden, codes, scales, w_proj, w_gate, conv_w):
    """Scalar loops over one fresh sequence: every output element from its definition."""
    T, H = hidden.shape
    D = w_proj.shape[0]
    R_ = codes.shape[1]
    M = 1 << 64

    def ctx(i):
        return int(tokens[i]) + 1 if i >= 0 else 0

    u = [[0.0] * H for _ in range(T)]
    for t in range(T):
        k2 = (ctx(t) * 0x9E3779B97F4A7C15 % M) ^ (ctx(t - 1) * 0xC2B2AE3D27D4EB4F % M)
        k3 = k2 ^ (ctx(t - 2) * 0x165667B19E3779F9 % M)
        r2 = (k2 ^ (k2 >> 32)) % R_
        r3 = (k3 ^ (k3 >> 32)) % R_
        e = [O.e4m3_decode(codes[0, r2, k]) * float(scales[0, r2]) +
             O.e4m3_decode(codes[1, r3, k]) * float(scales[1, r3]) for k in range(D)]
        a = sum(float(w_gate[j]) * float(hidden[t, j]) for j in range(H))
        g = 1.0 / (1.0 + math.exp(-a))
        for j in range(H):
            u[t][j] = g * sum(e[k] * float(w_proj[k, j]) for k in range(D))
    out = np.zeros((T, H))
    for t in range(T):
        for j in range(H):
            y = sum(float(conv_w[j, k]) * u[t - 3 + k][j] for k in range(4) if t - 3 + k >= 0)
            out[t, j] = float(hidden[t, j]) + y
    return out


def test_layer_matches_brute_force_tiny():
    w = pi.workload("tiny")
    codes, scales = w.table().full()
    W = w.weights()
    toks, offs, hid = pi.tiny_batch(w)
    T = 7
    r = _tiny_forward(toks[:T], [0, T], hid[:T])
    bf = _brute_force_layer(toks[:T], O.bf16_bits_to_f64(hid[:T]), codes, scales,
                            O.bf16_bits_to_f64(W.w_proj), O.bf16_bits_to_f64(W.w_gate), W.conv_w)
    assert np.allclose(r["out"], bf, rtol=1e-12, atol=1e-12)


def test_layer_packed_equals_separate():
    w = pi.workload("tiny")
    toks, _, hid = pi.tiny_batch(w)
    offs = [0, 10, 11, 40, 64]
    packed = _tiny_forward(toks[:64], offs, hid[:64])["out"]
    for s in range(4):
        a, b = offs[s], offs[s + 1]
        alone = _tiny_forward(toks[a:b], [0, b - a], hid[a:b])["out"]
        assert np.array_equal(packed[a:b], alone)


def test_layer_chunked_equals_whole():
    w = pi.workload("tiny")
    toks, _, hid = pi.tiny_batch(w)
    T = 50
    whole = _tiny_forward(toks[:T], [0, T], hid[:T])
    hist, conv = None, None
    outs = []
    for a, b in [(0, 1), (1, 3), (3, 20), (20, 50)]:
        r = _tiny_forward(toks[a:b], [0, b - a], hid[a:b], hist=hist, conv_state=conv)
        outs.append(r["out"])
        hist, conv = r["hist_out"], r["conv_out"]
    assert np.allclose(np.concatenate(outs), whole["out"], rtol=0, atol=1e-12)
    assert np.array_equal(hist, whole["hist_out"])
    assert np.allclose(conv, whole["conv_out"], rtol=0, atol=1e-12)


def test_layer_decode_steps_equal_prefill():
    w = pi.workload("tiny")
    W = w.weights()
    table = O.ArrayTable(*w.table().full())
    toks, _, hid = pi.tiny_batch(w)
    T = 12
    whole = _tiny_forward(toks[:T], [0, T], hid[:T])
    hist = np.array([[-1, -1]])
    conv = np.zeros((1, 3, w.hidden))
    outs = []
    for t in range(T):
        r = O.ple_decode_step(toks[t:t + 1].reshape(1, 1), hid[t:t + 1], W.w_proj, W.w_gate, W.conv_w,
                              table, w.rows_per_order, hist, conv)
        outs.append(r["out"])
        hist, conv = r["hist_out"], r["conv_out"]
    assert np.allclose(np.concatenate(outs), whole["out"], rtol=0, atol=1e-12)


def test_decode_commit_prefix_only():
    """The state after a step with n_commit = c equals the state after the first c tokens."""
    w = pi.workload("tiny")
    W = w.weights()
    table = O.ArrayTable(*w.table().full())
    toks, _, hid = pi.tiny_batch(w)
    hist0 = np.array([[4, 9]])
    conv0 = np.random.default_rng(8).standard_normal((1, 3, w.hidden))
    for c in (1, 2, 3):
        r = O.ple_decode_step(toks[:3].reshape(1, 3), hid[:3], W.w_proj, W.w_gate, W.conv_w, table,
                              w.rows_per_order, hist0, conv0, n_commit=[c])
        ref = O.ple_decode_step(toks[:c].reshape(1, c), hid[:c], W.w_proj, W.w_gate, W.conv_w, table,
                                w.rows_per_order, hist0, conv0)
        assert np.array_equal(r["hist_out"], ref["hist_out"])
        assert np.allclose(r["conv_out"], ref["conv_out"], rtol=0, atol=1e-12)
        assert np.allclose(r["out"][:c], ref["out"], rtol=0, atol=1e-12)


def test_zero_gate_returns_hidden():
    """Zero gate: h_t = q and w_gate = -8 q (bf16-exact) drive sigmoid to 0, so out == h."""
    w = pi.workload("tiny")
    rng = np.random.default_rng(12)
    qv = pi.f32_to_bf16_bits(rng.standard_normal(w.hidden).astype(np.float32))
    qf = O.bf16_bits_to_f64(qv)
    wg = pi.f32_to_bf16_bits((-8.0 * qf).astype(np.float32))
    assert np.array_equal(O.bf16_bits_to_f64(wg), -8.0 * qf)
    W = w.weights()
    toks, offs, _ = pi.tiny_batch(w)
    hid = np.tile(qv, (16, 1))
    table = O.ArrayTable(*w.table().full())
    r = O.ple_forward(toks[:16], [0, 16], hid, W.w_proj, wg, W.conv_w, table, w.rows_per_order)
    assert np.array_equal(O.to_f32(r["out"]), O.to_f32(O.bf16_bits_to_f64(hid)))
    assert np.array_equal(O.to_bf16_bits(r["out"]), hid)


def test_delta_conv_gives_gated_projection():
    """Delta conv kernel: out = h + g * (e W) token by token."""
    w = pi.workload("tiny")
    W = w.weights()
    table = O.ArrayTable(*w.table().full())
    toks, offs, hid = pi.tiny_batch(w)
    cw = np.tile(np.array([0, 0, 0, 1], np.float32), (w.hidden, 1))
    r = O.ple_forward(toks[:20], [0, 20], hid[:20], W.w_proj, W.w_gate, cw, table, w.rows_per_order)
    h = O.bf16_bits_to_f64(hid[:20])
    v = O.project(O.embed(table, r["ids"]), O.bf16_bits_to_f64(W.w_proj))
    g = O.gate(h, O.bf16_bits_to_f64(W.w_gate))
    assert np.allclose(r["out"], h + g[:, None] * v, rtol=0, atol=1e-12)


def test_sampled_outputs_equal_full_run():
    w = pi.workload("tiny")
    toks, _, hid = pi.tiny_batch(w)
    offs = [0, 2, 100, 256]
    full = _tiny_forward(toks, offs, hid)["out"]
    sample = np.array([0, 1, 2, 3, 4, 99, 100, 101, 102, 255])
    part = _tiny_forward(toks, offs, hid, sample=sample)["out"]
    assert np.array_equal(part, full[sample])


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1e-3], dtype=np.float64)
    lib = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.to_bf16_bits(x), lib)
