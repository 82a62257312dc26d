"""ple_prepare + ple_forward_prepared against ple_forward, through the C ABI.

The two-call form computes the same layer with the gate moved to a kernel of
its own; the tests require the outputs and the state to equal ple_forward's
bit for bit, on every projection path, across two streams, and check the
host-side errors for a missing or mismatched prepared batch.
"""
import numpy as np
import pytest

import ple_inputs as pi

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

from tests.gpu_common import MID, full_layer, mid_layer, tiny_layer  # noqa: E402,F401
from tests.test_gpu_parity import dev_bf16, dev_i32, gpu_forward, to_bits  # noqa: E402

pytestmark = pytest.mark.gpu


def _prepared(L, tokens, offsets, hidden_bits, out_dtype=1, state=None, path=0, stream=None):
    ple.ple_set_forward_path(L.handle, path)
    T, S, H = len(tokens), len(offsets) - 1, L.w.hidden
    hid = dev_bf16(hidden_bits)
    out = torch.empty(T, H, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    st = None
    if state is not None:
        st = (dev_i32(state[0]), torch.from_numpy(np.ascontiguousarray(state[1], np.float32)).cuda())
    tk, of = dev_i32(tokens), dev_i32(offsets)
    torch.cuda.synchronize()
    if stream is None:
        ple.ple_prepare(L.handle, tk, T, of, S, None if st is None else st[0])
        ple.ple_forward_prepared(L.handle, hid, out, out_dtype, st)
    else:
        side, main = stream
        with torch.cuda.stream(side):
            ple.ple_prepare(L.handle, tk, T, of, S, None if st is None else st[0], side)
            ev = torch.cuda.Event()
            ev.record(side)
        main.wait_event(ev)
        with torch.cuda.stream(main):
            ple.ple_forward_prepared(L.handle, hid, out, out_dtype, st, main)
    torch.cuda.synchronize()
    ple.ple_set_forward_path(L.handle, 0)
    assert ple.ple_get_error(L.handle) == 0
    res = out.cpu().numpy() if out_dtype == 1 else to_bits(out)
    return res, None if st is None else (st[0].cpu().numpy(), st[1].cpu().numpy())


def _f32bits(x):
    """fp32 bit patterns of an fp32-valued array (float64 copies convert back exactly)."""
    return np.asarray(x, np.float32).view(np.uint32)


def _state(rng, S, H, vocab):
    return rng.integers(-1, vocab, (S, 2)).astype(np.int32), rng.standard_normal((S, 3, H)).astype(np.float32)


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("with_state", [False, True])
def test_prepared_equals_forward_tiny(tiny_layer, path, with_state):
    w = tiny_layer.w
    rng = np.random.default_rng(path + 10 * with_state)
    lengths = [300, 1, 2, 700]
    T = sum(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    state = _state(rng, len(lengths), w.hidden, w.vocab) if with_state else None
    for dt in (1, 0):
        ref, ref_st = gpu_forward(tiny_layer, toks, offs, hid, dt, state=state, path=path)
        got, got_st = _prepared(tiny_layer, toks, offs, hid, dt, state=state, path=path)
        assert np.array_equal(_f32bits(got), _f32bits(ref)) if dt == 1 else np.array_equal(got, ref)
        if with_state:
            assert np.array_equal(got_st[0], ref_st[0])
            assert np.array_equal(_f32bits(got_st[1]), _f32bits(ref_st[1]))


@pytest.mark.parametrize("path", [1, 3, 2])
def test_prepared_equals_forward_mid_with_state(mid_layer, path):
    rng = np.random.default_rng(70 + path)
    lengths = [1000, 3, 600, 253]
    T = sum(lengths)
    toks = rng.integers(0, MID.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, MID.hidden)
    state = _state(rng, len(lengths), MID.hidden, MID.vocab)
    ref, ref_st = gpu_forward(mid_layer, toks, offs, hid, 1, state=state, path=path)
    got, got_st = _prepared(mid_layer, toks, offs, hid, 1, state=state, path=path)
    assert np.array_equal(_f32bits(got), _f32bits(ref))
    assert np.array_equal(got_st[0], ref_st[0])
    assert np.array_equal(_f32bits(got_st[1]), _f32bits(ref_st[1]))


def test_prepared_on_a_side_stream(tiny_layer):
    w = tiny_layer.w
    toks, offs, hid = pi.tiny_batch(w)
    ref, _ = gpu_forward(tiny_layer, toks, offs, hid, 1)
    side, main = torch.cuda.Stream(), torch.cuda.Stream()
    got, _ = _prepared(tiny_layer, toks, offs, hid, 1, stream=(side, main))
    assert np.array_equal(_f32bits(got), _f32bits(ref))


def test_prepared_batch_reused_with_other_hidden(tiny_layer):
    w = tiny_layer.w
    rng = np.random.default_rng(3)
    toks = rng.integers(0, w.vocab, 500).astype(np.int32)
    offs = np.array([0, 500], np.int32)
    h1, h2 = pi.hidden_bf16(rng, 500, w.hidden), pi.hidden_bf16(rng, 500, w.hidden)
    ref2, _ = gpu_forward(tiny_layer, toks, offs, h2, 1)
    ple.ple_prepare(tiny_layer.handle, dev_i32(toks), 500, dev_i32(offs), 1)
    outs = []
    for hb in (h1, h2):
        out = torch.empty(500, w.hidden, dtype=torch.float32, device="cuda")
        ple.ple_forward_prepared(tiny_layer.handle, dev_bf16(hb), out, 1)
        torch.cuda.synchronize()
        outs.append(out.cpu().numpy())
    assert np.array_equal(_f32bits(outs[1]), _f32bits(ref2))
    assert not np.array_equal(outs[0], outs[1])


def test_prepared_host_errors(tiny_layer):
    w = tiny_layer.w
    h = tiny_layer.handle
    toks, offs, hid = pi.tiny_batch(w)
    T = len(toks)
    out = torch.empty(T, w.hidden, dtype=torch.float32, device="cuda")
    hd = dev_bf16(hid)
    # a ple_forward discards the prepared batch
    gpu_forward(tiny_layer, toks, offs, hid, 1)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_forward_prepared(h, hd, out, 1)
    assert ei.value.code == 1
    # state given without a prepared history, and the reverse
    ple.ple_prepare(h, dev_i32(toks), T, dev_i32(offs), len(offs) - 1)
    conv = torch.zeros(1, 3, w.hidden, dtype=torch.float32, device="cuda")
    hist = dev_i32(np.full((1, 2), -1, np.int32))
    with pytest.raises(ple.PleError) as ei:
        ple.ple_forward_prepared(h, hd, out, 1, (hist, conv))
    assert ei.value.code == 1
    ple.ple_prepare(h, dev_i32(toks), T, dev_i32(offs), len(offs) - 1, hist)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_forward_prepared(h, hd, out, 1)
    assert ei.value.code == 1
    # a decode step discards it too
    ple.ple_prepare(h, dev_i32(toks), T, dev_i32(offs), len(offs) - 1)
    ple.ple_decode_step(h, dev_i32(toks[:2].reshape(2, 1)), 2, 1, dev_bf16(hid[:2]),
                        torch.empty(2, w.hidden, dtype=torch.float32, device="cuda"), 1,
                        dev_i32(np.full((2, 2), -1, np.int32)),
                        torch.zeros(2, 3, w.hidden, dtype=torch.float32, device="cuda"))
    with pytest.raises(ple.PleError):
        ple.ple_forward_prepared(h, hd, out, 1)
    torch.cuda.synchronize()
    assert ple.ple_get_error(h) == 0


def test_prepared_equals_forward_full(full_layer):
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w)
    ref, _ = gpu_forward(full_layer, toks, offs, hid, 0)
    got, _ = _prepared(full_layer, toks, offs, hid, 0)
    assert np.array_equal(got, ref)


def test_two_launch_embed_ragged_state_full(full_layer):
    """Batches of 4,096 tokens or more take the two-launch embed: an IDs kernel,
    then gate blocks and gather blocks. A ragged batch of 5,001 tokens (the last
    gate block holds one token, the last gather block is partial) with empty
    sequences and carried history and conv state, on samples against the
    oracle; the two-call form of the same batch, whose embed grid has no gate
    blocks, gives the same bits and the same state."""
    from tests.gpu_common import assert_close
    from tests.test_gpu_parity import _sample, check_state, oracle_forward
    w = pi.workload("prefill")
    lengths = [1, 0, 2, 2500, 0, 2495, 3]
    rng = np.random.default_rng(91)
    T, S = sum(lengths), len(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    hist0 = rng.integers(-1, w.vocab, (S, 2)).astype(np.int32)
    hist0[1] = [-1, -1]
    conv0 = rng.standard_normal((S, 3, w.hidden)).astype(np.float32)
    out, st = gpu_forward(full_layer, toks, offs, hid, 1, state=(hist0, conv0))
    sample = _sample(T, offs, 300, 92)
    ref = oracle_forward(full_layer, toks, offs, hid, hist=hist0, conv=conv0, sample=sample)
    assert_close(out[sample], ref["out"], "ragged 5,001-token prefill with state")
    check_state(st, ref)
    got, got_st = _prepared(full_layer, toks, offs, hid, 1, state=(hist0, conv0))
    assert np.array_equal(_f32bits(got), _f32bits(out))
    assert np.array_equal(got_st[0], st[0])
    assert np.array_equal(_f32bits(got_st[1]), _f32bits(st[1]))


# ----------------------------------------------------------------------------- two prepare slots
@pytest.fixture(scope="module")
def mid_two_slots():
    from ple_inputs.device import DeviceLayer
    import oracle as O
    L = DeviceLayer(MID, max_tokens=4096, max_seqs=64, prepare_slots=2)
    codes, scales = MID.table().full()
    L.host_table = O.ArrayTable(codes, scales)
    yield L
    L.close()


def test_two_slots_in_flight(mid_two_slots):
    """A stream of batches with two in flight: batch i + 1 is prepared into the other
    slot on a side stream while batch i is projected on the main stream, the state
    carried from batch to batch. Every output and the final state equal ple_forward's
    run of the same batches one after the other, bit for bit."""
    L = mid_two_slots
    rng = np.random.default_rng(404)
    H = MID.hidden
    batches = []
    for lengths in ([300, 1, 2000], [5, 700, 12], [1500, 3, 1], [64, 64, 64], [1, 1, 900]):
        T = sum(lengths)
        batches.append((rng.integers(0, MID.vocab, T).astype(np.int32),
                        np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32), pi.hidden_bf16(rng, T, H)))
    hist0, conv0 = _state(rng, 3, H, MID.vocab)

    # one call per batch
    hs, cs = dev_i32(hist0), torch.from_numpy(conv0).cuda()
    ref = []
    for tk, of, hd in batches:
        out = torch.empty(len(tk), H, dtype=torch.bfloat16, device="cuda")
        ple.ple_forward(L.handle, dev_i32(tk), len(tk), dev_i32(of), 3, dev_bf16(hd), out, 0, (hs, cs))
        ref.append(out)
    torch.cuda.synchronize()
    ref_state = (hs.cpu().numpy(), cs.cpu().numpy())

    # two slots: the prepare of batch i + 1 reads the history that the projection of
    # batch i writes, so the side stream waits for it; rows then overlap the projection
    hs2, cs2 = dev_i32(hist0), torch.from_numpy(conv0).cuda()
    side, main = torch.cuda.Stream(), torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    main.wait_stream(torch.cuda.current_stream())
    dev = [(dev_i32(tk), dev_i32(of), dev_bf16(hd)) for tk, of, hd in batches]
    torch.cuda.synchronize()
    outs = [torch.empty(len(tk), H, dtype=torch.bfloat16, device="cuda") for tk, _, _ in batches]
    prepared = [torch.cuda.Event() for _ in batches]
    done = [torch.cuda.Event() for _ in batches]
    hist_ready = torch.cuda.Event()
    hist_ready.record(main)
    for i, (tk, of, hd) in enumerate(dev):
        slot = i % 2
        with torch.cuda.stream(side):
            side.wait_event(hist_ready)
            if i >= 2:
                side.wait_event(done[i - 2])            # the slot's previous batch is projected
            ple.ple_prepare_slot(L.handle, slot, tk, len(batches[i][0]), of, 3, hs2, side)
            prepared[i].record(side)
        with torch.cuda.stream(main):
            main.wait_event(prepared[i])
            ple.ple_forward_prepared_slot(L.handle, slot, hd, outs[i], 0, (hs2, cs2), main)
            done[i].record(main)
            hist_ready = torch.cuda.Event()
            hist_ready.record(main)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    for i in range(len(batches)):
        assert torch.equal(outs[i], ref[i]), i
    assert np.array_equal(hs2.cpu().numpy(), ref_state[0])
    assert np.array_equal(cs2.cpu().numpy(), ref_state[1])


def test_slot_one_needs_two_slots(tiny_layer):
    toks, offs, hid = pi.tiny_batch(tiny_layer.w)
    with pytest.raises(ple.PleError) as ei:
        ple.ple_prepare_slot(tiny_layer.handle, 1, dev_i32(toks), len(toks), dev_i32(offs), 1)
    assert ei.value.code == 1
    with pytest.raises(ple.PleError) as ei:
        ple.ple_prepare_slot(tiny_layer.handle, 2, dev_i32(toks), len(toks), dev_i32(offs), 1)
    assert ei.value.code == 1
    out = torch.empty(len(toks), tiny_layer.w.hidden, dtype=torch.float32, device="cuda")
    with pytest.raises(ple.PleError) as ei:
        ple.ple_forward_prepared_slot(tiny_layer.handle, 1, dev_bf16(hid), out, 1)
    assert ei.value.code == 1


def test_slot_batch_survives_forward(mid_two_slots):
    """ple_forward uses slot 0's scratch: a batch prepared in slot 1 stays valid."""
    L = mid_two_slots
    rng = np.random.default_rng(9)
    T = 700
    toks = rng.integers(0, MID.vocab, T).astype(np.int32)
    offs = np.array([0, 200, T], np.int32)
    hid = pi.hidden_bf16(rng, T, MID.hidden)
    ref, _ = gpu_forward(L, toks, offs, hid, 0)
    ple.ple_prepare_slot(L.handle, 1, dev_i32(toks), T, dev_i32(offs), 2)
    other = rng.integers(0, MID.vocab, 300).astype(np.int32)
    gpu_forward(L, other, np.array([0, 300], np.int32), pi.hidden_bf16(rng, 300, MID.hidden), 0)
    out = torch.empty(T, MID.hidden, dtype=torch.bfloat16, device="cuda")
    ple.ple_forward_prepared_slot(L.handle, 1, dev_bf16(hid), out, 0)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    assert np.array_equal(to_bits(out), ref)
