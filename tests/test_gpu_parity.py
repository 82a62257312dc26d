"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on B200.

Row IDs are compared bit for bit; floats (fp32 output) within max |err| 2e-2
and relative L2 1e-3; the bf16 output must equal the round-to-nearest-even of
the same call's fp32 output (so it lies within the float tolerance plus half a
bf16 ulp of the oracle).
Full-scale workloads are compared on sampled outputs the oracle computes
one by one, plus the carried state.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import (MAX_ABS, REL_L2, assert_bf16_close, assert_close, full_layer,  # noqa: F401
                              mid_layer, tiny_layer)

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------- helpers
def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_bf16(bits):
    from ple_inputs.device import bf16_tensor
    return bf16_tensor(bits)


def to_bits(t):
    from ple_inputs.device import bf16_bits
    return bf16_bits(t)


def gpu_ids(L, tokens, offsets, hist=None):
    T = len(tokens)
    ids = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    ple.ple_ngram_ids(L.handle, dev_i32(tokens), T, dev_i32(offsets), len(offsets) - 1,
                      None if hist is None else dev_i32(hist), ids)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    return ids.cpu().numpy()


def gpu_forward(L, tokens, offsets, hidden_bits, out_dtype=1, state=None, path=0):
    """Runs ple_forward; returns (out as float64 or bf16 bits, new state or None)."""
    ple.ple_set_forward_path(L.handle, path)
    T = len(tokens)
    H = L.w.hidden
    hid = dev_bf16(hidden_bits)
    out = torch.empty(T, H, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    st = None
    if state is not None:
        hist, conv = state
        st = (dev_i32(hist), torch.from_numpy(np.ascontiguousarray(conv, np.float32)).cuda())
    ple.ple_forward(L.handle, dev_i32(tokens), T, dev_i32(offsets), len(offsets) - 1, hid, out, out_dtype, st)
    torch.cuda.synchronize()
    ple.ple_set_forward_path(L.handle, 0)
    assert ple.ple_get_error(L.handle) == 0
    res = out.cpu().numpy().astype(np.float64) if out_dtype == 1 else to_bits(out)
    new_state = None if st is None else (st[0].cpu().numpy(), st[1].cpu().numpy())
    return res, new_state


def oracle_forward(L, tokens, offsets, hidden_bits, hist=None, conv=None, sample=None, weights=None):
    W = weights or L.host_weights
    return O.ple_forward(tokens, offsets, hidden_bits, W.w_proj, W.w_gate, W.conv_w, L.host_table,
                         L.w.rows_per_order, hist=hist, conv_state=conv, sample=sample)


def check_state(new_state, ref):
    hist, conv = new_state
    assert np.array_equal(hist, ref["hist_out"])
    assert_close(conv, ref["conv_out"], "conv state")


# ----------------------------------------------------------------------------- inputs
def test_device_table_matches_host_generator_tiny(tiny_layer):
    codes, scales = tiny_layer.w.table().full()
    assert np.array_equal(tiny_layer.table.cpu().numpy().reshape(codes.shape), codes)
    assert np.array_equal(tiny_layer.scales.cpu().numpy().reshape(scales.shape), scales)


def test_device_table_matches_host_generator_full(full_layer):
    w = full_layer.w
    rng = np.random.default_rng(0)
    rows = np.concatenate([[0, 1, w.rows_per_order - 1], rng.integers(0, w.rows_per_order, 61)])
    tab = full_layer.table.view(2, w.rows_per_order, w.row_dim)
    sc = full_layer.scales.view(2, w.rows_per_order)
    idx = torch.from_numpy(rows).cuda()
    for n in range(2):
        assert np.array_equal(tab[n][idx].cpu().numpy(), w.table().codes(n, rows))
        assert np.array_equal(sc[n][idx].cpu().numpy(), w.table().scales(n, rows))


# ----------------------------------------------------------------------------- row IDs
def test_ids_tiny(tiny_layer):
    toks, offs, _ = pi.tiny_batch(tiny_layer.w)
    assert np.array_equal(gpu_ids(tiny_layer, toks, offs), O.ngram_ids(toks, offs, 4096))


def test_ids_boundaries_and_history(tiny_layer):
    rng = np.random.default_rng(1)
    toks = rng.integers(0, 1000, 40).astype(np.int32)
    offs = np.array([0, 1, 1, 3, 3, 3, 20, 40], dtype=np.int32)      # empty, length-1 and length-2 sequences
    hist = rng.integers(-1, 1000, (7, 2)).astype(np.int32)
    hist[2] = [-1, -1]
    hist[3] = [-1, 5]
    for h in (None, hist):
        assert np.array_equal(gpu_ids(tiny_layer, toks, offs, h), O.ngram_ids(toks, offs, 4096, h))


@pytest.mark.parametrize("name", ["prefill", "long", "decode", "mtp"])
def test_ids_full_scale_workloads(full_layer, name):
    w = pi.workload(name)
    R = w.rows_per_order
    if name == "prefill":
        toks, offs, _ = pi.prefill_batch(w)
        hist = None
    elif name == "long":
        toks, _ = next(pi.long_chunks(w, n_chunks=1))
        offs = np.array([0, len(toks)])
        hist = np.array([[123, 4567]])
    elif name == "decode":
        t2, _, hist, _ = pi.decode_batch(w)
        toks = t2.reshape(-1)
        offs = np.arange(t2.shape[0] + 1) * t2.shape[1]
    else:
        s = pi.mtp_session(w, steps=1)
        t2 = s["steps"][0][0]
        toks = t2.reshape(-1)
        offs = np.arange(t2.shape[0] + 1) * t2.shape[1]
        hist = s["prompts"][:, -2:]
    assert np.array_equal(gpu_ids(full_layer, toks, offs, hist), O.ngram_ids(toks, offs, R, hist))


def test_ids_hash_worked_example(tiny_layer, full_layer):  # noqa: F811
    """The worked example of the hash (``tests/golden/hash_worked_example.txt``, written down
    from the definition before any implementation) through the library's own copy of the
    constants: ple_ngram_ids on tables of 4,096 and of 10,000,048 rows per order."""
    from tests.test_golden import hash_worked_example
    layers = {4096: tiny_layer, 10_000_048: full_layer}
    for rows, toks, expect in hash_worked_example():
        L = layers[rows]
        assert L.w.rows_per_order == rows
        got = gpu_ids(L, np.array(toks, np.int32), [0, len(toks)])
        assert [tuple(int(v) for v in r) for r in got] == expect, (rows, toks)


def test_decode_hash_worked_example(tiny_layer):
    """The decode kernel hashes with its own code: one sequence of the worked example's tokens
    with no history, as a single 1 x 5 decode step, must gather the worked example's rows, so it
    matches the oracle run on those literal row IDs."""
    from tests.test_golden import hash_worked_example
    rows, toks, expect = hash_worked_example()[0]
    assert rows == tiny_layer.w.rows_per_order
    w = tiny_layer.w
    hid = pi.hidden_bf16(np.random.default_rng(11), len(toks), w.hidden)
    tk = np.array([toks], np.int32)
    out, _, _ = gpu_decode(tiny_layer, tk, hid, np.full((1, 2), -1, np.int32), np.zeros((1, 3, w.hidden), np.float32))
    W = tiny_layer.host_weights
    e = O.embed(tiny_layer.host_table, np.array(expect, np.int64))
    v = O.project(e, O.bf16_bits_to_f64(W.w_proj))
    g = O.gate(O.bf16_bits_to_f64(hid), O.bf16_bits_to_f64(W.w_gate))
    u = g[:, None] * v
    u_hist = np.concatenate([np.zeros((3, w.hidden)), u])
    y = O.short_conv(u_hist, W.conv_w)
    assert_close(out, O.bf16_bits_to_f64(hid) + y, "decode step on the worked example")


# ----------------------------------------------------------------------------- gather
def _gather(L, ids):
    T = ids.shape[0]
    e = torch.empty(T, L.w.row_dim, dtype=torch.float16, device="cuda")
    ple.ple_gather_rows(L.handle, dev_i32(ids), T, e)
    torch.cuda.synchronize()
    return e.cpu().numpy()


def _check_fp16_rounding(e_gpu, e_ref):
    ref16 = e_ref.astype(np.float16)
    a = e_gpu.view(np.uint16).astype(np.int32)
    b = ref16.view(np.uint16).astype(np.int32)
    ka = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    kb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    ulp = np.abs(ka - kb)
    assert ulp.max() <= 1, ulp.max()
    assert np.mean(ulp) < 1e-3


def test_gather_tiny_all_rows(tiny_layer):
    R = tiny_layer.w.rows_per_order
    ids = np.stack([np.arange(R), (np.arange(R) * 7919) % R], axis=1)
    _check_fp16_rounding(_gather(tiny_layer, ids), O.embed(tiny_layer.host_table, ids))


def test_gather_every_code_and_scale_kind(tiny_layer):
    """Every E4M3 code (NaN codes 0x7F / 0xFF included) against every scale kind
    the dequantisation distinguishes: ordinary, >= 2^7, subnormal, -0, NaN. The
    first 256 rows of each order are overwritten and restored afterwards."""
    L = tiny_layer
    R, D = L.w.rows_per_order, L.w.row_dim
    n = 256
    k = np.arange(D)
    codes = np.empty((2, n, D), np.uint8)
    for i in range(n):
        codes[0, i] = (i * D + k) % 256
        codes[1, i] = (i * D + 5 * k + 17) % 256
    kinds = np.array([0.0123, -3.5, 200.0, 127.9, 128.0, 1e-40, -0.0, np.nan, 2.0 ** -20, 65504 / 448,
                      -1e-3, 7.25], np.float32)
    scales = np.stack([kinds[np.arange(n) % len(kinds)], kinds[(np.arange(n) * 5 + 3) % len(kinds)]])
    tab = L.table.view(2, R, D)
    sc = L.scales.view(2, R)
    saved = (tab[:, :n].clone(), sc[:, :n].clone())
    try:
        tab[:, :n] = torch.from_numpy(codes).cuda()
        sc[:, :n] = torch.from_numpy(scales).cuda()
        t = np.arange(2048)
        ids = np.stack([t % n, (t * 37 + t // n) % n], axis=1)
        got = _gather(L, ids)
    finally:
        tab[:, :n] = saved[0]
        sc[:, :n] = saved[1]
        torch.cuda.synchronize()
    with np.errstate(invalid="ignore", over="ignore"):
        ref = O.embed(O.ArrayTable(codes, scales), ids).astype(np.float16)
    nan = np.isnan(ref)
    assert nan.any() and np.array_equal(np.isnan(got), nan)
    a = got[~nan].view(np.uint16).astype(np.int32)
    b = ref[~nan].view(np.uint16).astype(np.int32)
    ka = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    kb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    assert np.abs(ka - kb).max() <= 1


def test_gather_full_sample(full_layer):
    rng = np.random.default_rng(2)
    R = full_layer.w.rows_per_order
    ids = np.stack([rng.integers(0, R, 512), rng.integers(0, R, 512)], axis=1)
    ids[:4] = [[0, 0], [R - 1, R - 1], [0, R - 1], [R - 1, 0]]
    _check_fp16_rounding(_gather(full_layer, ids), O.embed(full_layer.host_table, ids))


# ----------------------------------------------------------------------------- forward, small
@pytest.mark.parametrize("path", [1, 2])
def test_forward_tiny(tiny_layer, path):
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    ref = oracle_forward(tiny_layer, toks, offs, hid)
    out32, _ = gpu_forward(tiny_layer, toks, offs, hid, 1, path=path)
    assert_close(out32, ref["out"], f"tiny path {path}")
    out16, _ = gpu_forward(tiny_layer, toks, offs, hid, 0, path=path)
    assert np.array_equal(out16, O.to_bf16_bits(out32))          # bf16 = RNE of the same fp32 result
    assert_bf16_close(out16, ref["out"])


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("lengths", [[1], [2], [3], [1, 1, 1], [253, 1, 2], [254], [256], [506, 1],
                                     [100, 0, 0, 157], [1000, 3, 30, 7, 1]])
def test_forward_ragged(tiny_layer, path, lengths):
    w = tiny_layer.w
    rng = np.random.default_rng(sum(lengths) + 7 * len(lengths))
    T = sum(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    ref = oracle_forward(tiny_layer, toks, offs, hid)
    out, _ = gpu_forward(tiny_layer, toks, offs, hid, 1, path=path)
    assert_close(out, ref["out"], f"lengths {lengths} path {path}")


@pytest.mark.parametrize("path", [1, 2])
def test_forward_state_tiny(tiny_layer, path):
    """Carried state: chunks of one sequence with state == the whole sequence; state
    in and out matches the oracle; empty sequences leave their state unchanged."""
    w = tiny_layer.w
    toks, _, hid = pi.tiny_batch(w)
    T = 200
    whole = oracle_forward(tiny_layer, toks[:T], [0, T], hid[:T])
    hist = np.array([[-1, -1]], np.int32)
    conv = np.zeros((1, 3, w.hidden), np.float32)
    outs = []
    for a, b in [(0, 1), (1, 2), (2, 40), (40, 41), (41, 200)]:
        out, (hist, conv) = gpu_forward(tiny_layer, toks[a:b], [0, b - a], hid[a:b], 1, state=(hist, conv), path=path)
        outs.append(out)
    assert_close(np.concatenate(outs), whole["out"], "chunked")
    assert np.array_equal(hist, whole["hist_out"])
    assert_close(conv, whole["conv_out"], "end state")
    # several sequences with arbitrary carried state, one of them empty
    rng = np.random.default_rng(3)
    offs = np.array([0, 50, 50, 52, 120], np.int32)
    hist0 = rng.integers(-1, w.vocab, (4, 2)).astype(np.int32)
    conv0 = rng.standard_normal((4, 3, w.hidden)).astype(np.float32)
    ref = oracle_forward(tiny_layer, toks[:120], offs, hid[:120], hist=hist0, conv=conv0)
    out, st = gpu_forward(tiny_layer, toks[:120], offs, hid[:120], 1, state=(hist0, conv0), path=path)
    assert_close(out, ref["out"], "multi-sequence state")
    check_state(st, ref)
    assert np.array_equal(st[1][1], conv0[1]) and np.array_equal(st[0][1], hist0[1])


def test_forward_paths_agree(tiny_layer):
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    a, _ = gpu_forward(tiny_layer, toks, offs, hid, 1, path=1)
    b, _ = gpu_forward(tiny_layer, toks, offs, hid, 1, path=2)
    assert np.abs(a - b).max() < 1e-4


def test_forward_deterministic(tiny_layer):
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    a, _ = gpu_forward(tiny_layer, toks, offs, hid, 1)
    b, _ = gpu_forward(tiny_layer, toks, offs, hid, 1)
    assert np.array_equal(a, b)


def test_forward_empty_is_noop(tiny_layer):
    out = torch.full((4, tiny_layer.w.hidden), 7.0, device="cuda")
    hid = torch.zeros(4, tiny_layer.w.hidden, dtype=torch.bfloat16, device="cuda")
    offs = dev_i32([0, 0])
    ple.ple_forward(tiny_layer.handle, dev_i32([1]), 0, offs, 1, hid, out, 1)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_forward_max_tokens(tiny_layer):
    w = tiny_layer.w
    T = tiny_layer.config.max_tokens
    rng = np.random.default_rng(11)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.array([0, 700, T], np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    ref = oracle_forward(tiny_layer, toks, offs, hid)
    for path in (0, 1, 2):
        out, _ = gpu_forward(tiny_layer, toks, offs, hid, 1, path=path)
        assert_close(out, ref["out"], f"max tokens path {path}")


# ----------------------------------------------------------------------------- invariants
def _custom_layer(tiny_layer, weights):
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(tiny_layer.w, max_tokens=512, max_seqs=8, weights=weights)
    L.host_table = tiny_layer.host_table
    return L


def test_zero_gate_returns_hidden_in_place(tiny_layer):
    """h_t = q, w_gate = -8 q: the gate is exactly 0, so the in-place bf16 output is h."""
    w = tiny_layer.w
    rng = np.random.default_rng(12)
    qv = pi.f32_to_bf16_bits(rng.standard_normal(w.hidden).astype(np.float32))
    wg = pi.f32_to_bf16_bits((-8.0 * O.bf16_bits_to_f64(qv)).astype(np.float32))
    base = w.weights()
    L = _custom_layer(tiny_layer, pi.Weights(base.w_proj, wg, base.conv_w))
    try:
        toks, offs, _ = pi.tiny_batch(w)
        hid_bits = np.tile(qv, (len(toks), 1))
        for path in (1, 2):
            ple.ple_set_forward_path(L.handle, path)
            hid = dev_bf16(hid_bits)
            ple.ple_forward(L.handle, dev_i32(toks), len(toks), dev_i32(offs), 1, hid, hid, 0)
            torch.cuda.synchronize()
            assert np.array_equal(to_bits(hid), hid_bits)
    finally:
        L.close()


def test_delta_conv_is_identity(tiny_layer):
    """conv taps (0,0,0,1): out = h + g * (e W) token by token."""
    w = tiny_layer.w
    base = w.weights()
    cw = np.tile(np.array([0, 0, 0, 1], np.float32), (w.hidden, 1))
    W = pi.Weights(base.w_proj, base.w_gate, cw)
    L = _custom_layer(tiny_layer, W)
    try:
        toks, offs, hid = pi.tiny_batch(w)
        h = O.bf16_bits_to_f64(hid)
        ids = O.ngram_ids(toks, offs, w.rows_per_order)
        v = O.project(O.embed(L.host_table, ids), O.bf16_bits_to_f64(W.w_proj))
        g = O.gate(h, O.bf16_bits_to_f64(W.w_gate))
        for path in (1, 2):
            out, _ = gpu_forward(L, toks, offs, hid, 1, path=path)
            assert_close(out, h + g[:, None] * v, "delta conv")
    finally:
        L.close()


def test_packed_equals_separate(tiny_layer):
    w = tiny_layer.w
    rng = np.random.default_rng(13)
    lengths = [37, 1, 300, 2, 90]
    T = sum(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    packed, _ = gpu_forward(tiny_layer, toks, offs, hid, 1)
    for s in range(len(lengths)):
        a, b = offs[s], offs[s + 1]
        alone, _ = gpu_forward(tiny_layer, toks[a:b], [0, b - a], hid[a:b], 1)
        assert np.abs(alone - packed[a:b]).max() < 1e-4


def test_ids_independent_of_hidden(tiny_layer):
    """Same tokens, different hidden states: identical rows (IDs need no hidden state)."""
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    a = gpu_ids(tiny_layer, toks, offs)
    gpu_forward(tiny_layer, toks, offs, hid, 1)
    b = gpu_ids(tiny_layer, toks, offs)
    assert np.array_equal(a, b)


# ----------------------------------------------------------------------------- decode
def gpu_decode(L, tokens, hidden_bits, hist, conv, n_commit=None, out_dtype=1):
    B, q = tokens.shape
    out = torch.empty(B * q, L.w.hidden, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    hs = dev_i32(hist)
    cs = torch.from_numpy(np.ascontiguousarray(conv, np.float32)).cuda()
    ple.ple_decode_step(L.handle, dev_i32(tokens), B, q, dev_bf16(hidden_bits), out, out_dtype, hs, cs,
                        None if n_commit is None else dev_i32(n_commit))
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    res = out.cpu().numpy().astype(np.float64) if out_dtype == 1 else to_bits(out)
    return res, hs.cpu().numpy(), cs.cpu().numpy()


def test_decode_steps_equal_prefill_tiny(tiny_layer):
    w = tiny_layer.w
    toks, _, hid = pi.tiny_batch(w)
    T = 24
    whole = oracle_forward(tiny_layer, toks[:T], [0, T], hid[:T])
    hist = np.array([[-1, -1]], np.int32)
    conv = np.zeros((1, 3, w.hidden), np.float32)
    outs = []
    for t in range(T):
        out, hist, conv = gpu_decode(tiny_layer, toks[t:t + 1].reshape(1, 1), hid[t:t + 1], hist, conv)
        outs.append(out)
    assert_close(np.concatenate(outs), whole["out"], "decode by steps")
    assert np.array_equal(hist, whole["hist_out"])


def test_decode_commit_tiny(tiny_layer):
    w = tiny_layer.w
    rng = np.random.default_rng(14)
    B, q = 5, 3
    toks = rng.integers(0, w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, w.hidden)
    hist = rng.integers(-1, w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, w.hidden)).astype(np.float32)
    nc = np.array([1, 2, 3, 1, 3], np.int32)
    W = w.weights()
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, tiny_layer.host_table, w.rows_per_order,
                            hist, conv, n_commit=nc)
    out, h2, c2 = gpu_decode(tiny_layer, toks, hid, hist, conv, nc)
    assert_close(out, ref["out"], "decode outputs")
    assert np.array_equal(h2, ref["hist_out"])
    assert_close(c2, ref["conv_out"], "decode state")


def test_decode_full(full_layer):
    w = pi.workload("decode")
    toks, hid, hist, conv = pi.decode_batch(w)
    W = full_layer.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, full_layer.host_table, w.rows_per_order,
                            hist, conv)
    out, h2, c2 = gpu_decode(full_layer, toks, hid, hist, conv)
    assert_close(out, ref["out"], "full decode")
    assert np.array_equal(h2, ref["hist_out"])
    assert_close(c2, ref["conv_out"], "full decode state")
    out16, _, _ = gpu_decode(full_layer, toks, hid, hist, conv, out_dtype=0)
    assert np.array_equal(out16, O.to_bf16_bits(out))


def test_mtp_steps_full(full_layer):
    """MTP-style batch: 64 sequences x 3 tokens, shared prefixes, n_commit in 1..3."""
    w = pi.workload("mtp")
    s = pi.mtp_session(w, steps=3, prefix=64)
    W = full_layer.host_weights
    B, P = s["prompts"].shape
    toks = s["prompts"].reshape(-1)
    offs = np.arange(B + 1) * P
    hist0 = np.full((B, 2), -1, np.int32)
    conv0 = np.zeros((B, 3, w.hidden), np.float32)
    _, (hist, conv) = gpu_forward(full_layer, toks, offs, s["prompt_hidden"][:B * P], 1, state=(hist0, conv0))
    ref_p = oracle_forward(full_layer, toks, offs, s["prompt_hidden"][:B * P], hist=hist0, conv=conv0,
                           sample=np.array([0, P - 1, B * P - 1]))
    assert np.array_equal(hist, ref_p["hist_out"])
    assert_close(conv, ref_p["conv_out"], "prompt state")
    for tk, hd, nc in s["steps"]:
        ref = O.ple_decode_step(tk, hd, W.w_proj, W.w_gate, W.conv_w, full_layer.host_table, w.rows_per_order,
                                hist, conv, n_commit=nc)
        out, hist, conv = gpu_decode(full_layer, tk, hd, hist, conv, nc)
        assert_close(out, ref["out"], "mtp step")
        assert np.array_equal(hist, ref["hist_out"])
        assert_close(conv, ref["conv_out"], "mtp state")
        # duplicated requests stay identical
        assert np.array_equal(out[:3], out[3:6])


# ----------------------------------------------------------------------------- full-scale forward
def _sample(T, offs, n, seed):
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, n, replace=False).tolist())
    for o in offs:
        for d in (-3, -2, -1, 0, 1, 2, 3):
            if 0 <= o + d < T:
                s.add(int(o + d))
    for k in range(1, T // 253 + 1):          # fused tile edges
        for d in (-1, 0, 1, 2, 3):
            if 0 <= 253 * k + d < T and len(s) < n + 400:
                s.add(253 * k + d)
    return np.array(sorted(s))


def test_prefill_full_sampled(full_layer):
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w)
    T = len(toks)
    out, _ = gpu_forward(full_layer, toks, offs, hid, 1)
    sample = _sample(T, offs, 1500, 21)
    ref = oracle_forward(full_layer, toks, offs, hid, sample=sample)
    assert_close(out[sample], ref["out"], "prefill")
    out16, _ = gpu_forward(full_layer, toks, offs, hid, 0)
    assert np.array_equal(out16, O.to_bf16_bits(out))


def test_prefill_full_in_place_bf16(full_layer):
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w, variant=1, lengths=[4096])
    T = len(toks)
    ref16, _ = gpu_forward(full_layer, toks, offs, hid, 0)
    h = dev_bf16(hid)
    ple.ple_forward(full_layer.handle, dev_i32(toks), T, dev_i32(offs), 1, h, h, 0)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(h), ref16)


def test_long_context_chunks_full(full_layer):
    """Two 16,384-token chunks of one sequence with the state carried across."""
    w = pi.workload("long")
    chunks = list(pi.long_chunks(w, n_chunks=2))
    hist = np.array([[-1, -1]], np.int32)
    conv = np.zeros((1, 3, w.hidden), np.float32)
    ohist, oconv = None, None
    for i, (tk, hd) in enumerate(chunks):
        offs = np.array([0, len(tk)])
        out, (hist, conv) = gpu_forward(full_layer, tk, offs, hd, 1, state=(hist, conv))
        sample = _sample(len(tk), offs, 600, 30 + i)
        ref = oracle_forward(full_layer, tk, offs, hd, hist=ohist, conv=oconv, sample=sample)
        assert_close(out[sample], ref["out"], f"chunk {i}")
        assert np.array_equal(hist, ref["hist_out"])
        assert_close(conv, ref["conv_out"], f"chunk {i} state")
        ohist, oconv = ref["hist_out"], ref["conv_out"]


# ----------------------------------------------------------------------------- errors and controls
def test_device_range_errors(tiny_layer):
    w = tiny_layer.w
    hid = dev_bf16(pi.hidden_bf16(np.random.default_rng(0), 8, w.hidden))
    out = torch.empty(8, w.hidden, device="cuda")
    h = tiny_layer.handle
    ple.ple_forward(h, dev_i32([1, 2, 3, w.vocab, 5, 6, 7, 8]), 8, dev_i32([0, 8]), 1, hid, out, 1)
    assert ple.ple_get_error(h) == 4
    ple.ple_forward(h, dev_i32([1, 2, 3, -1, 5, 6, 7, 8]), 8, dev_i32([0, 8]), 1, hid, out, 1)
    assert ple.ple_get_error(h) == 4
    ple.ple_forward(h, dev_i32(range(8)), 8, dev_i32([0, 6, 3, 8]), 3, hid, out, 1)   # not monotone
    assert ple.ple_get_error(h) == 4
    ple.ple_forward(h, dev_i32(range(8)), 8, dev_i32([0, 7]), 1, hid, out, 1)        # does not end at T
    assert ple.ple_get_error(h) == 4
    ple.ple_forward(h, dev_i32(range(8)), 8, dev_i32([0, 8]), 1, hid, out, 1)
    assert ple.ple_get_error(h) == 0
    hs = dev_i32([[1, 2]] * 4)
    cs = torch.zeros(4, 3, w.hidden, device="cuda")
    ple.ple_decode_step(h, dev_i32(range(8)), 4, 2, hid, out, 1, hs, cs, dev_i32([1, 0, 2, 3]))
    assert ple.ple_get_error(h) == 4


def test_host_argument_errors(tiny_layer):
    w = tiny_layer.w
    h = tiny_layer.handle
    hid = torch.zeros(8, w.hidden, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(8, w.hidden, device="cuda")
    tk, of = dev_i32(range(8)), dev_i32([0, 8])
    n0 = ple.ple_launch_count(h)
    cases = [
        (lambda: ple.ple_forward(h, tk, -1, of, 1, hid, out, 1), 1),
        (lambda: ple.ple_forward(h, tk, 8, of, 1, hid, out, 7), 1),
        (lambda: ple.ple_forward(h, tk, 8, of, 0, hid, out, 1), 2),
        (lambda: ple.ple_forward(h, tk, tiny_layer.config.max_tokens + 1, of, 1, hid, out, 1), 2),
        (lambda: ple.ple_forward(h, tk, 8, of, tiny_layer.config.max_seqs + 1, hid, out, 1), 2),
        (lambda: ple.ple_forward(h, None, 8, of, 1, hid, out, 1), 1),
        (lambda: ple.ple_forward(h, tk, 8, of, 1, hid, hid, 1), 1),                  # in place needs bf16
        (lambda: ple.ple_forward(h, tk, 8, of, 1, hid.data_ptr() + 2, out, 1), 3),   # misaligned
        (lambda: ple.ple_decode_step(h, tk, 0, 1, hid, out, 1, tk, out, None), 2),
        (lambda: ple.ple_decode_step(h, tk, 8, 1, hid, out, 1, None, out, None), 1),
        (lambda: ple.ple_gather_rows(h, None, 4, out), 1),
    ]
    for fn, code in cases:
        with pytest.raises(ple.PleError) as ei:
            fn()
        assert ei.value.code == code
    assert ple.ple_launch_count(h) == n0           # nothing was launched
    assert ple.ple_get_error(h) == 0


def test_create_rejects_out_of_range_weights(tiny_layer):
    w = tiny_layer.w
    base = w.weights()
    wp = base.w_proj.copy()
    wp[3, 5] = pi.f32_to_bf16_bits(np.array([1e5], np.float32))[0]
    from ple_inputs.device import DeviceLayer
    with pytest.raises(ple.PleError) as ei:
        DeviceLayer(w, max_tokens=64, max_seqs=2, weights=pi.Weights(wp, base.w_gate, base.conv_w))
    assert ei.value.code == 8


def test_stage_timing_and_launch_count(tiny_layer):
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    h = tiny_layer.handle
    ple.ple_set_profiling(h, True)
    ple.ple_get_stage_times(h)
    n0 = ple.ple_launch_count(h)
    gpu_forward(tiny_layer, toks, offs, hid, 1, path=1)
    gpu_forward(tiny_layer, toks, offs, hid, 1, path=2)
    st = ple.ple_get_stage_times(h)
    ple.ple_set_profiling(h, False)
    # each forward: one embed kernel (ids, gate, gather) and the projection; split-K adds the combine
    assert ple.ple_launch_count(h) - n0 == 5
    assert st["prepare"][1] == 2 and st["gather"][1] == 0 and st["gemm"][1] == 2 and st["combine"][1] == 1
    assert all(v[0] > 0 for k, v in st.items() if v[1])


# ----------------------------------------------------------------------------- SM-pair tiles (hidden 256)
def _mid_batch(lengths, seed):
    from tests.gpu_common import MID
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    toks = rng.integers(0, MID.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, MID.hidden)
    return toks, offs, hid


@pytest.mark.parametrize("path", [1, 3, 2])
@pytest.mark.parametrize("lengths", [[1000], [1, 2, 3, 600, 0, 400], [253], [254, 253, 1], [4096]])
def test_forward_mid_paths(mid_layer, path, lengths):
    toks, offs, hid = _mid_batch(lengths, sum(lengths) + len(lengths))
    ref = oracle_forward(mid_layer, toks, offs, hid)
    out, _ = gpu_forward(mid_layer, toks, offs, hid, 1, path=path)
    assert_close(out, ref["out"], f"mid {lengths} path {path}")
    out16, _ = gpu_forward(mid_layer, toks, offs, hid, 0, path=path)
    assert np.array_equal(out16, O.to_bf16_bits(out))
    assert_bf16_close(out16, ref["out"])


@pytest.mark.parametrize("path", [1, 3])
def test_forward_mid_state(mid_layer, path):
    toks, _, hid = _mid_batch([900], 5)
    rng = np.random.default_rng(6)
    offs = np.array([0, 300, 301, 301, 900], np.int32)
    hist0 = rng.integers(-1, 5000, (4, 2)).astype(np.int32)
    conv0 = rng.standard_normal((4, 3, 256)).astype(np.float32)
    ref = oracle_forward(mid_layer, toks, offs, hid, hist=hist0, conv=conv0)
    out, st = gpu_forward(mid_layer, toks, offs, hid, 1, state=(hist0, conv0), path=path)
    assert_close(out, ref["out"], "mid state")
    check_state(st, ref)


def test_forward_mid_pair_equals_single(mid_layer):
    toks, offs, hid = _mid_batch([700, 300], 9)
    a, _ = gpu_forward(mid_layer, toks, offs, hid, 1, path=1)
    b, _ = gpu_forward(mid_layer, toks, offs, hid, 1, path=3)
    assert np.abs(a - b).max() < 1e-4


def test_forward_mid_in_place(mid_layer):
    toks, offs, hid = _mid_batch([2000, 96], 10)
    ref16, _ = gpu_forward(mid_layer, toks, offs, hid, 0, path=1)
    h = dev_bf16(hid)
    ple.ple_set_forward_path(mid_layer.handle, 1)
    ple.ple_forward(mid_layer.handle, dev_i32(toks), len(toks), dev_i32(offs), 2, h, h, 0)
    torch.cuda.synchronize()
    ple.ple_set_forward_path(mid_layer.handle, 0)
    assert np.array_equal(to_bits(h), ref16)


def test_decode_mid_in_place(mid_layer):
    """out == hidden: the tokens kernel computes the gates before the projection
    writes anything, and each CTA of the projection reads hidden only at its own
    channels, so an in-place step equals the out-of-place step bit for bit (on
    the channel-split kernel and on the split-K path alike)."""
    from tests.gpu_common import MID
    B, q = 8, 1
    rng = np.random.default_rng(77)
    toks = rng.integers(0, MID.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, MID.hidden)
    hist = rng.integers(-1, MID.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, MID.hidden)).astype(np.float32)
    W = mid_layer.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, mid_layer.host_table, MID.rows_per_order,
                            hist, conv)
    for path in (0, 2):
        ple.ple_set_forward_path(mid_layer.handle, path)
        try:
            apart, h_a, c_a = gpu_decode(mid_layer, toks, hid, hist, conv, out_dtype=0)      # bf16 bits
            h = dev_bf16(hid)
            hs = dev_i32(hist)
            cs = torch.from_numpy(np.ascontiguousarray(conv, np.float32)).cuda()
            ple.ple_decode_step(mid_layer.handle, dev_i32(toks), B, q, h, h, 0, hs, cs)
            torch.cuda.synchronize()
        finally:
            ple.ple_set_forward_path(mid_layer.handle, 0)
        assert ple.ple_get_error(mid_layer.handle) == 0
        assert np.array_equal(to_bits(h), apart), path
        assert np.array_equal(hs.cpu().numpy(), h_a)
        assert np.array_equal(cs.cpu().numpy(), c_a)
        assert_bf16_close(apart, ref["out"])


# ----------------------------------------------------------------------------- decode: channel-split projection
@pytest.mark.parametrize("shape", [(1, 1), (8, 1), (5, 3), (16, 1), (2, 8), (6, 3), (3, 7)])
def test_decode_paths_tiny(tiny_layer, shape):
    """B * q <= 16 runs the channel-split projection kernel, larger steps the split-K
    path; both match the oracle and each other (path 2 forces split-K)."""
    w = tiny_layer.w
    B, q = shape
    rng = np.random.default_rng(B * 100 + q)
    toks = rng.integers(0, w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, w.hidden)
    hist = rng.integers(-1, w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, w.hidden)).astype(np.float32)
    nc = rng.integers(1, q + 1, B).astype(np.int32)
    W = w.weights()
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, tiny_layer.host_table, w.rows_per_order,
                            hist, conv, n_commit=nc)
    outs = []
    for path in (0, 2):
        ple.ple_set_forward_path(tiny_layer.handle, path)
        out, h2, c2 = gpu_decode(tiny_layer, toks, hid, hist, conv, nc)
        ple.ple_set_forward_path(tiny_layer.handle, 0)
        assert_close(out, ref["out"], f"decode {shape} path {path}")
        assert np.array_equal(h2, ref["hist_out"])
        assert_close(c2, ref["conv_out"], f"decode state {shape} path {path}")
        outs.append(out)
    # steps of up to 8 tokens multiply the two orders' exact codes and scale after the
    # products, the split-K path the fp16-rounded sum of the orders: equal within the
    # tolerance, not bit for bit
    assert_close(outs[0], outs[1], f"decode {shape}: channel-split against split-K")


@pytest.mark.parametrize("shape", [(8, 1), (4, 3), (16, 1)])
def test_decode_single_kernel_mid(mid_layer, shape):
    from tests.gpu_common import MID
    B, q = shape
    rng = np.random.default_rng(B * 7 + q)
    toks = rng.integers(0, MID.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, MID.hidden)
    hist = rng.integers(-1, MID.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, MID.hidden)).astype(np.float32)
    W = mid_layer.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, mid_layer.host_table, MID.rows_per_order,
                            hist, conv)
    out, h2, c2 = gpu_decode(mid_layer, toks, hid, hist, conv)
    assert_close(out, ref["out"], f"mid decode {shape}")
    assert np.array_equal(h2, ref["hist_out"])
    assert_close(c2, ref["conv_out"], "mid decode state")
    out16, _, _ = gpu_decode(mid_layer, toks, hid, hist, conv, out_dtype=0)
    assert np.array_equal(out16, O.to_bf16_bits(out))
