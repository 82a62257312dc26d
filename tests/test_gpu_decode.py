"""Decode steps through the C ABI: the two-call form (ple_decode_prepare, then
ple_decode_step_prepared) against ple_decode_step and the CPU oracle, steps in
place, the run-to-run determinism of a step's bits, and the host-side errors of
the two-call form.

The two-call form is the decode side of the pages' split between the lookup,
which needs only the tokens, and the merge, which needs the hidden states (DGX
Spark report, section "n-gram embedding 是一条附加的条件记忆路径"). Its result
must equal ple_decode_step's bit for bit: both compute each token's gate with
the same warp reduction, whichever kernel runs it.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import MID, assert_close, full_layer, mid_layer, tiny_layer  # noqa: F401

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _inputs(w, B, q, seed):
    rng = np.random.default_rng(seed)
    toks = rng.integers(0, w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, w.hidden)
    hist = rng.integers(-1, w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, w.hidden)).astype(np.float32)
    nc = rng.integers(1, q + 1, B).astype(np.int32)
    return toks, hid, hist, conv, nc


def _run(L, toks, hid, hist, conv, nc, prepared, out_dtype=1, in_place=False):
    """One decode step; returns (out as float64 or bf16 bits, hist, conv)."""
    from ple_inputs.device import bf16_bits, bf16_tensor
    B, q = toks.shape
    H = L.w.hidden
    tk, hs = _i32(toks), _i32(hist)
    cs = torch.from_numpy(np.ascontiguousarray(conv)).cuda()
    h = bf16_tensor(hid)
    out = h if in_place else torch.empty(B * q, H, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16,
                                         device="cuda")
    n = None if nc is None else _i32(nc)
    if prepared:
        ple.ple_decode_prepare(L.handle, tk, B, q, hs)
        ple.ple_decode_step_prepared(L.handle, h, out, out_dtype, hs, cs, n)
    else:
        ple.ple_decode_step(L.handle, tk, B, q, h, out, out_dtype, hs, cs, n)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    res = out.cpu().numpy().astype(np.float64) if out_dtype == 1 else bf16_bits(out)
    return res, hs.cpu().numpy(), cs.cpu().numpy()


def _oracle(L, toks, hid, hist, conv, nc):
    W = L.host_weights
    return O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, L.w.rows_per_order, hist, conv,
                             n_commit=nc)


def _check(L, shape, seed, path=0):
    toks, hid, hist, conv, nc = _inputs(L.w, *shape, seed)
    ref = _oracle(L, toks, hid, hist, conv, nc)
    ple.ple_set_forward_path(L.handle, path)
    try:
        a = _run(L, toks, hid, hist, conv, nc, prepared=False)
        b = _run(L, toks, hid, hist, conv, nc, prepared=True)
        a16 = _run(L, toks, hid, hist, conv, nc, prepared=False, out_dtype=0)
        b16 = _run(L, toks, hid, hist, conv, nc, prepared=True, out_dtype=0)
        c16 = _run(L, toks, hid, hist, conv, nc, prepared=True, out_dtype=0, in_place=True)
    finally:
        ple.ple_set_forward_path(L.handle, 0)
    assert_close(a[0], ref["out"], f"decode {shape}")
    assert np.array_equal(a[1], ref["hist_out"])
    assert_close(a[2], ref["conv_out"], f"decode state {shape}")
    for x in (b, a16, b16, c16):
        assert np.array_equal(x[1], a[1]) and np.array_equal(x[2], a[2])
    assert np.array_equal(b[0], a[0])
    assert np.array_equal(b16[0], a16[0]) and np.array_equal(c16[0], a16[0])
    assert np.array_equal(a16[0], O.to_bf16_bits(a[0]))


@pytest.mark.parametrize("shape", [(1, 1), (8, 1), (5, 3), (16, 1), (2, 8), (6, 3), (24, 3)])
def test_decode_prepared_tiny(tiny_layer, shape):
    _check(tiny_layer, shape, seed=shape[0] * 10 + shape[1])


@pytest.mark.parametrize("shape,path", [((8, 1), 0), ((4, 3), 0), ((16, 1), 0), ((8, 1), 2), ((64, 3), 0),
                                        ((6, 3), 0), ((64, 4), 0), ((32, 9), 0), ((64, 3), 2)])
def test_decode_prepared_mid(mid_layer, shape, path):
    """Steps of up to 16 tokens run the channel-split kernel, 17 to 256 tokens the
    split-K kernel with in-kernel sums (256 = its largest N, with fewer stages), more
    than 256 the split-K projection and combine kernel, as does path 2 for any size."""
    _check(mid_layer, shape, seed=shape[0] * 7 + shape[1] + path, path=path)


def test_decode_prepared_full(full_layer):  # noqa: F811
    """The full-scale 8 x 1 decode workload, and a 64 x 3 MTP-style step with n_commit."""
    w = pi.workload("decode")
    toks, hid, hist, conv = pi.decode_batch(w)
    ref = _oracle(full_layer, toks, hid, hist, conv, None)
    a = _run(full_layer, toks, hid, hist, conv, None, prepared=False)
    b = _run(full_layer, toks, hid, hist, conv, None, prepared=True)
    assert_close(a[0], ref["out"], "full decode")
    assert np.array_equal(a[1], ref["hist_out"])
    assert_close(a[2], ref["conv_out"], "full decode state")
    assert np.array_equal(b[0], a[0]) and np.array_equal(b[1], a[1]) and np.array_equal(b[2], a[2])
    toks, hid, hist, conv, nc = _inputs(w, 64, 3, 99)
    sample = np.arange(0, 192, 7)
    a = _run(full_layer, toks, hid, hist, conv, nc, prepared=False)
    b = _run(full_layer, toks, hid, hist, conv, nc, prepared=True)
    assert np.array_equal(b[0], a[0]) and np.array_equal(b[1], a[1]) and np.array_equal(b[2], a[2])
    # the oracle on a sample of the sequences (a step's sequences are independent)
    seqs = np.unique(sample // 3)
    ref = _oracle(full_layer, toks[seqs], hid.reshape(64, 3, -1)[seqs].reshape(-1, w.hidden), hist[seqs], conv[seqs],
                  nc[seqs])
    rows = (seqs[:, None] * 3 + np.arange(3)[None, :]).reshape(-1)
    assert_close(a[0][rows], ref["out"], "full MTP step")
    assert np.array_equal(a[1][seqs], ref["hist_out"])
    assert_close(a[2][seqs], ref["conv_out"], "full MTP state")


@pytest.mark.parametrize("shape", [(1, 1), (3, 1), (1, 3), (64, 3)])
def test_decode_step_bits_repeat(full_layer, shape):  # noqa: F811
    """Every sum in a decode step is taken in a fixed order: 50 runs of the same step
    (full scale, where one token's gate spans many lanes and warps) give the same bits."""
    toks, hid, hist, conv, nc = _inputs(full_layer.w, *shape, 5)
    first = _run(full_layer, toks, hid, hist, conv, nc, prepared=False)
    for _ in range(49):
        again = _run(full_layer, toks, hid, hist, conv, nc, prepared=False)
        assert np.array_equal(again[0], first[0])
        assert np.array_equal(again[2], first[2])


@pytest.mark.parametrize("shape", [(4, 1), (2, 3), (12, 1)])
def test_decode_prepared_route_fixed_at_prepare(mid_layer, shape):
    """ple_decode_prepare chooses the form of the rows it leaves (exact codes and
    row scales for steps of up to 8 tokens, else dequantised rows) with the path in
    force then: a path change before ple_decode_step_prepared leaves the step as
    it was prepared, equal bit for bit to ple_decode_step under the first path."""
    from ple_inputs.device import bf16_tensor
    L = mid_layer
    B, q = shape
    toks, hid, hist, conv, nc = _inputs(L.w, B, q, 11 + B)
    ref = _run(L, toks, hid, hist, conv, nc, prepared=False)
    tk, hs = _i32(toks), _i32(hist)
    cs = torch.from_numpy(np.ascontiguousarray(conv)).cuda()
    out = torch.empty(B * q, L.w.hidden, dtype=torch.float32, device="cuda")
    ple.ple_decode_prepare(L.handle, tk, B, q, hs)
    ple.ple_set_forward_path(L.handle, 2)
    try:
        ple.ple_decode_step_prepared(L.handle, bf16_tensor(hid), out, 1, hs, cs, _i32(nc))
    finally:
        ple.ple_set_forward_path(L.handle, 0)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref[0])
    assert np.array_equal(hs.cpu().numpy(), ref[1]) and np.array_equal(cs.cpu().numpy(), ref[2])


def test_decode_prepared_errors(tiny_layer):
    L = tiny_layer
    w = L.w
    toks, hid, hist, conv, nc = _inputs(w, 2, 1, 3)
    from ple_inputs.device import bf16_tensor
    tk, hs = _i32(toks), _i32(hist)
    cs = torch.from_numpy(conv).cuda()
    h = bf16_tensor(hid)
    out = torch.empty(2, w.hidden, dtype=torch.float32, device="cuda")
    # nothing prepared
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_step_prepared(L.handle, h, out, 1, hs, cs)
    assert ei.value.code == 1
    # another history buffer than the one the rows were computed from
    ple.ple_decode_prepare(L.handle, tk, 2, 1, hs)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_step_prepared(L.handle, h, out, 1, _i32(hist), cs)
    assert ei.value.code == 1
    # a prepared step is consumed by its step
    ple.ple_decode_step_prepared(L.handle, h, out, 1, hs, cs)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_step_prepared(L.handle, h, out, 1, hs, cs)
    assert ei.value.code == 1
    # a forward in between discards it
    ple.ple_decode_prepare(L.handle, tk, 2, 1, hs)
    ple.ple_forward(L.handle, tk, 2, _i32([0, 2]), 1, h, out, 1)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_step_prepared(L.handle, h, out, 1, hs, cs)
    assert ei.value.code == 1
    # shapes and pointers are checked before anything runs
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_prepare(L.handle, tk, 0, 1, hs)
    assert ei.value.code == 2
    with pytest.raises(ple.PleError) as ei:
        ple.ple_decode_prepare(L.handle, tk, 2, 1, None)
    assert ei.value.code == 1
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
