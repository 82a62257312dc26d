"""Whole full-scale sessions, in the launch configuration the benchmark times,
checked against the oracle on samples.

The layer remembers only the last two tokens of a sequence and the gated rows
u of its last three positions, and u of a position depends only on that
position's token, its two predecessors and its hidden row. So the oracle can
rebuild the carried state at any point of a long session from a few tokens,
and check sampled outputs anywhere in it:

* long context: all 16 chunks of 16,384 tokens of one 262,144-token sequence,
  with the state carried from chunk to chunk by the library;
* MTP: 64 sequences x 3 tokens for 100 steps after 512-token prompts, 19 of
  them duplicated requests, the state advancing by each step's n_commit.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import assert_close, full_layer  # noqa: F401
from tests.test_gpu_parity import gpu_decode, gpu_forward, oracle_forward

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu


def test_long_context_all_chunks_full(full_layer):  # noqa: F811
    w = pi.workload("long")
    hist = np.array([[-1, -1]], np.int32)
    conv = np.zeros((1, 3, w.hidden), np.float32)
    ohist = oconv = None
    rng = np.random.default_rng(77)
    n = 0
    for c, (tk, hd) in enumerate(pi.long_chunks(w)):
        L = len(tk)
        offs = np.array([0, L])
        out, (hist, conv) = gpu_forward(full_layer, tk, offs, hd, 1, state=(hist, conv))
        # the first positions read the carried state; the rest are spread over the chunk
        sample = np.unique(np.concatenate([[0, 1, 2, 3, L - 1], rng.choice(L, 24, replace=False)]))
        ref = oracle_forward(full_layer, tk, offs, hd, hist=ohist, conv=oconv, sample=sample)
        assert_close(out[sample], ref["out"], f"long-context chunk {c}")
        assert np.array_equal(hist, ref["hist_out"]), c
        assert_close(conv, ref["conv_out"], f"state after chunk {c}")
        ohist, oconv = ref["hist_out"], ref["conv_out"]
        n += 1
    assert n == 16


def _state_after(tokens, hidden_rows, W, table, rows, H):
    """(hist [2], conv [3][H]) after a committed history whose last tokens and their
    hidden rows are given (the oracle's own computation of u for the last three)."""
    toks = list(tokens)
    hist = ([-1, -1] + toks)[-2:]
    conv = np.zeros((3, H))
    k = min(3, len(toks))
    if k:
        win_t = np.array(toks[-k:])
        win_h = np.asarray(hidden_rows[-k:])
        before = ([-1, -1] + toks[:-k])[-2:]
        r = O.ple_forward(win_t, [0, k], win_h, W.w_proj, W.w_gate, W.conv_w, table, rows,
                          hist=np.array([before]), conv_state=np.zeros((1, 3, H)), sample=np.array([], np.int64))
        conv = r["conv_out"][0]
    return np.array(hist, np.int64), conv


def test_mtp_full_session_sampled(full_layer):  # noqa: F811
    w = pi.workload("mtp")
    s = pi.mtp_session(w)
    W = full_layer.host_weights
    table = full_layer.host_table
    R, H = w.rows_per_order, w.hidden
    B, P = s["prompts"].shape
    q = w.extra["q"]
    hist = np.full((B, 2), -1, np.int32)
    conv = np.zeros((B, 3, H), np.float32)
    half = B // 2
    for b0 in (0, half):                       # the prompts in two packed batches, as the benchmark runs them
        toks = s["prompts"][b0:b0 + half].reshape(-1)
        offs = np.arange(half + 1) * P
        _, (h2, c2) = gpu_forward(full_layer, toks, offs, s["prompt_hidden"][b0 * P:(b0 + half) * P], 1,
                                  state=(hist[b0:b0 + half], conv[b0:b0 + half]))
        hist[b0:b0 + half], conv[b0:b0 + half] = h2, c2
    # each sequence's committed history: the last few tokens and their hidden rows
    hist_tok = [list(s["prompts"][b][-5:]) for b in range(B)]
    hist_hid = [list(s["prompt_hidden"][b * P + P - 5:b * P + P]) for b in range(B)]
    sel = [0, 5, 18, 19, 40, 63]               # duplicated requests (0, 5, 18) and independent ones
    checked = 0
    for k, (tk, hd, nc) in enumerate(s["steps"]):
        if k in (0, 1, 37, 99):
            states = [_state_after(hist_tok[b], hist_hid[b], W, table, R, H) for b in sel]
            hist_o = np.stack([st[0] for st in states])
            conv_o = np.stack([st[1] for st in states])
            rows = np.concatenate([np.arange(b * q, (b + 1) * q) for b in sel])
            ref = O.ple_decode_step(tk[sel], hd[rows], W.w_proj, W.w_gate, W.conv_w, table, R, hist_o, conv_o,
                                    n_commit=nc[sel])
        out, hist, conv = gpu_decode(full_layer, tk, hd, hist, conv, nc)
        if k in (0, 1, 37, 99):
            assert_close(out[rows], ref["out"], f"mtp step {k}")
            assert np.array_equal(hist[sel], ref["hist_out"]), k
            assert_close(conv[sel], ref["conv_out"], f"mtp state after step {k}")
            checked += 1
        assert np.array_equal(out[:q], out[5 * q:6 * q])   # duplicated requests stay identical
        for b in range(B):
            hist_tok[b] = (hist_tok[b] + list(tk[b][:nc[b]]))[-5:]
            hist_hid[b] = (hist_hid[b] + list(hd[b * q:b * q + nc[b]]))[-5:]
    assert checked == 4
