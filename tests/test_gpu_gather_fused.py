"""The gather-fused projection (forward path 4) on B200, through the C ABI.

In this form the projection kernel reads the two FP8 table rows of every
token itself and dequantises them straight into its shared-memory operand
tiles; the rows never pass through HBM as fp16. It must agree with the CPU
oracle within the float tolerance, and with the two-kernel form (path 1: the
embed kernel writes the fp16 rows, the projection loads them by TMA) bit for
bit, since both dequantise through the same function and feed the tensor
cores the same operands in the same order.

Layers: hidden 256 with 128-wide rows (two K-stages per tile, so the loads run
one stage ahead), hidden 256 with 256-wide rows (four K-stages, the deep
pipeline the full-scale layer uses), and the full-scale prefill and
long-context workloads.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import MID, assert_bf16_close, assert_close, full_layer, mid_layer  # noqa: F401

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu

WIDE = pi.Workload("wide", 5000, 8192, 256, 256, table_seed=11, seed=11)


@pytest.fixture(scope="module")
def wide_layer():
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(WIDE, max_tokens=4096, max_seqs=64)
    codes, scales = WIDE.table().full()
    L.host_table = O.ArrayTable(codes, scales)
    yield L
    L.close()


@pytest.fixture(params=["mid", "wide"])
def layer(request, mid_layer, wide_layer):  # noqa: F811
    return mid_layer if request.param == "mid" else wide_layer


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def forward(L, toks, offs, hid_bits, out_dtype, path, state=None, in_place=False):
    """ple_forward on path `path`; returns the device output and the device state."""
    from ple_inputs.device import bf16_tensor
    T, H = len(toks), L.w.hidden
    hid = bf16_tensor(hid_bits)
    if in_place:
        out = hid
    else:
        out = torch.empty(T, H, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    st = None
    if state is not None:
        st = (dev_i32(state[0]), torch.from_numpy(np.ascontiguousarray(state[1], np.float32)).cuda())
    ple.ple_set_forward_path(L.handle, path)
    try:
        ple.ple_forward(L.handle, dev_i32(toks), T, dev_i32(offs), len(offs) - 1, hid, out, out_dtype, st)
        torch.cuda.synchronize()
    finally:
        ple.ple_set_forward_path(L.handle, 0)
    assert ple.ple_get_error(L.handle) == 0
    return out, st


def batch(w, lengths, seed):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return toks, offs, pi.hidden_bf16(rng, T, w.hidden)


def oracle(L, toks, offs, hid, hist=None, conv=None, sample=None):
    W = L.host_weights
    return O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, L.w.rows_per_order,
                         hist=hist, conv_state=conv, sample=sample)


def bits(t):
    from ple_inputs.device import bf16_bits
    return bf16_bits(t)


# tile edges: a fused tile outputs 253 tokens; ragged tails, empty and short sequences
@pytest.mark.parametrize("lengths", [[1000], [1, 2, 3, 600, 0, 400], [253], [254, 253, 1], [3000, 1096]])
def test_gather_fused_matches_oracle_and_two_kernel_form(layer, lengths):
    toks, offs, hid = batch(layer.w, lengths, 100 + sum(lengths) + len(lengths))
    ref = oracle(layer, toks, offs, hid)
    out4, _ = forward(layer, toks, offs, hid, 1, path=4)
    got = out4.cpu().numpy().astype(np.float64)
    assert_close(got, ref["out"], f"gather-fused {lengths}")
    out1, _ = forward(layer, toks, offs, hid, 1, path=1)
    assert torch.equal(out4, out1)
    out16, _ = forward(layer, toks, offs, hid, 0, path=4)
    assert np.array_equal(bits(out16), O.to_bf16_bits(got))
    assert_bf16_close(bits(out16), ref["out"])


def test_gather_fused_carried_state(layer):
    toks, _, hid = batch(layer.w, [900], 5)
    rng = np.random.default_rng(6)
    offs = np.array([0, 300, 301, 301, 900], np.int32)
    hist0 = rng.integers(-1, layer.w.vocab, (4, 2)).astype(np.int32)
    conv0 = rng.standard_normal((4, 3, layer.w.hidden)).astype(np.float32)
    ref = oracle(layer, toks, offs, hid, hist=hist0, conv=conv0)
    out4, st4 = forward(layer, toks, offs, hid, 1, path=4, state=(hist0, conv0))
    assert_close(out4.cpu().numpy(), ref["out"], "gather-fused with state")
    assert np.array_equal(st4[0].cpu().numpy(), ref["hist_out"])
    assert_close(st4[1].cpu().numpy(), ref["conv_out"], "conv state")
    out1, st1 = forward(layer, toks, offs, hid, 1, path=1, state=(hist0, conv0))
    assert torch.equal(out4, out1)
    assert torch.equal(st4[0], st1[0]) and torch.equal(st4[1], st1[1])


def test_gather_fused_in_place(mid_layer):  # noqa: F811
    toks, offs, hid = batch(MID, [2000, 96], 10)
    ref16, _ = forward(mid_layer, toks, offs, hid, 0, path=4)
    h, _ = forward(mid_layer, toks, offs, hid, 0, path=4, in_place=True)
    assert torch.equal(h, ref16)


def test_gather_fused_two_launches(wide_layer):
    toks, offs, hid = batch(WIDE, [1500], 12)
    L = wide_layer
    ple.ple_get_stage_times(L.handle)                  # reset the counters
    ple.ple_set_profiling(L.handle, True)
    n0 = ple.ple_launch_count(L.handle)
    forward(L, toks, offs, hid, 1, path=4)
    ple.ple_set_profiling(L.handle, False)
    assert ple.ple_launch_count(L.handle) - n0 == 2   # IDs + gate, then the projection
    st = ple.ple_get_stage_times(L.handle)
    assert st["prepare"][1] == 1 and st["gemm"][1] == 1 and st["combine"][1] == 0


def test_gather_fused_nvfp4_table_takes_two_kernel_form():
    """Path 4 applies to E4M3 tables; an NVFP4 handle keeps the two-kernel form."""
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(MID, max_tokens=2048, max_seqs=8, table_format=ple.PLE_TABLE_NVFP4)
    try:
        toks, offs, hid = batch(MID, [700, 300], 13)
        a, _ = forward(L, toks, offs, hid, 1, path=4)
        b, _ = forward(L, toks, offs, hid, 1, path=1)
        assert torch.equal(a, b)
    finally:
        L.close()


# ----------------------------------------------------------------------------- full scale
def _sample(T, offs, n, seed):
    rng = np.random.default_rng(seed)
    s = set(rng.choice(T, n, replace=False).tolist())
    for o in offs:
        s.update(int(o + d) for d in range(-3, 4) if 0 <= o + d < T)
    for k in range(1, T // 253 + 1):
        s.update(253 * k + d for d in (-1, 0, 1, 2, 3) if 0 <= 253 * k + d < T)
    return np.array(sorted(s))


def test_gather_fused_full_prefill(full_layer):  # noqa: F811
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w)
    out4, _ = forward(full_layer, toks, offs, hid, 1, path=4)
    out1, _ = forward(full_layer, toks, offs, hid, 1, path=1)
    assert torch.equal(out4, out1)
    sample = _sample(len(toks), offs, 1000, 41)
    ref = oracle(full_layer, toks, offs, hid, sample=sample)
    assert_close(out4.cpu().numpy()[sample], ref["out"], "full prefill, gather-fused")
    out16, _ = forward(full_layer, toks, offs, hid, 0, path=4)
    assert np.array_equal(bits(out16), O.to_bf16_bits(out4.cpu().numpy()))


def test_gather_fused_full_long_chunks(full_layer):  # noqa: F811
    """Two 16,384-token chunks of one sequence with the state carried across,
    on both forms: outputs and states agree bit for bit, and with the oracle."""
    w = pi.workload("long")
    chunks = list(pi.long_chunks(w, n_chunks=2))
    st4 = st1 = (np.array([[-1, -1]], np.int32), np.zeros((1, 3, w.hidden), np.float32))
    ohist = oconv = None
    for i, (tk, hd) in enumerate(chunks):
        offs = np.array([0, len(tk)])
        o4, s4 = forward(full_layer, tk, offs, hd, 1, path=4, state=st4)
        o1, s1 = forward(full_layer, tk, offs, hd, 1, path=1, state=st1)
        assert torch.equal(o4, o1)
        assert torch.equal(s4[0], s1[0]) and torch.equal(s4[1], s1[1])
        sample = _sample(len(tk), offs, 400, 50 + i)
        ref = oracle(full_layer, tk, offs, hd, hist=ohist, conv=oconv, sample=sample)
        assert_close(o4.cpu().numpy()[sample], ref["out"], f"chunk {i}")
        assert np.array_equal(s4[0].cpu().numpy(), ref["hist_out"])
        ohist, oconv = ref["hist_out"], ref["conv_out"]
        st4 = (s4[0].cpu().numpy(), s4[1].cpu().numpy())
        st1 = (s1[0].cpu().numpy(), s1[1].cpu().numpy())
