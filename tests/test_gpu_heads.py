"""The multi-head row layout (PLE_TABLE_E4M3_HEADS) on B200, through the C ABI.

16 lookups of 160-byte rows per token, as the SSD-stream model card states:
8 hash heads per order, each a sub-table of its own; e is the 16 dequantised
rows side by side. Row IDs must match the oracle bit for bit; rows within one
fp16 ulp; the layer within the float tolerance, on a small layer (16 heads of
16 codes) and on the full-scale table (16 x 20,000,096 rows of 160 codes).
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import assert_bf16_close, assert_close, release_device_memory

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu

HT = pi.workload("heads_tiny")


@pytest.fixture(scope="module")
def heads_layer():
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(HT, max_tokens=4096, max_seqs=64, table_format=ple.PLE_TABLE_E4M3_HEADS)
    L.host_table = O.HeadsArrayTable(*HT.heads_table().full())
    yield L
    L.close()


@pytest.fixture(scope="module")
def heads_full_layer():
    from ple_inputs.device import DeviceLayer
    w = pi.workload("heads_full")
    free, _ = torch.cuda.mem_get_info()
    if free < w.rows_per_order * w.row_dim + (8 << 30):
        pytest.skip(f"needs {w.rows_per_order * w.row_dim / 1e9:.0f} GB for the table, {free / 1e9:.0f} GB free")
    L = DeviceLayer(w, max_tokens=16384, max_seqs=64, table_format=ple.PLE_TABLE_E4M3_HEADS)
    L.host_table = w.heads_table()
    yield L
    release_device_memory(L)


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def gpu_ids(L, toks, offs, hist=None):
    T = len(toks)
    ids = torch.empty(T, 16, dtype=torch.int32, device="cuda")
    ple.ple_ngram_ids(L.handle, dev_i32(toks), T, dev_i32(offs), len(offs) - 1,
                      None if hist is None else dev_i32(hist), ids)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    return ids.cpu().numpy()


def gpu_forward(L, toks, offs, hid, out_dtype=1, state=None, path=0):
    from ple_inputs.device import bf16_tensor
    T = len(toks)
    out = torch.empty(T, L.w.hidden, dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    st = None
    if state is not None:
        st = (dev_i32(state[0]), torch.from_numpy(np.ascontiguousarray(state[1], np.float32)).cuda())
    ple.ple_set_forward_path(L.handle, path)
    try:
        ple.ple_forward(L.handle, dev_i32(toks), T, dev_i32(offs), len(offs) - 1, bf16_tensor(hid), out, out_dtype, st)
        torch.cuda.synchronize()
    finally:
        ple.ple_set_forward_path(L.handle, 0)
    assert ple.ple_get_error(L.handle) == 0
    return out, st


def oracle(L, toks, offs, hid, hist=None, conv=None, sample=None):
    W = L.host_weights
    return O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, L.w.rows_per_order,
                         hist=hist, conv_state=conv, sample=sample)


def batch(w, lengths, seed):
    rng = np.random.default_rng(seed)
    T = sum(lengths)
    return (rng.integers(0, w.vocab, T).astype(np.int32), np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32),
            pi.hidden_bf16(rng, T, w.hidden))


def fp16_ulps(a16, ref):
    a = a16.view(np.uint16).astype(np.int32)
    b = ref.astype(np.float16).view(np.uint16).astype(np.int32)
    ka = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    kb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(ka - kb)


# ----------------------------------------------------------------------------- small layer
def test_heads_device_table_matches_host_generator(heads_layer):
    hd = HT.row_dim // 16
    codes = heads_layer.table.view(16, HT.rows_per_order, hd).cpu().numpy()
    scales = heads_layer.scales.view(16, HT.rows_per_order).cpu().numpy()
    hc, hs = HT.heads_table().full()
    assert np.array_equal(codes, hc) and np.array_equal(scales, hs)


def test_heads_ids_bit_exact(heads_layer):
    rng = np.random.default_rng(1)
    toks = rng.integers(0, HT.vocab, 300).astype(np.int32)
    offs = np.array([0, 1, 1, 3, 3, 150, 300], np.int32)       # empty, length-1 and length-2 sequences
    hist = rng.integers(-1, HT.vocab, (6, 2)).astype(np.int32)
    hist[2] = [-1, -1]
    for h in (None, hist):
        assert np.array_equal(gpu_ids(heads_layer, toks, offs, h),
                              O.ngram_ids_heads(toks, offs, HT.rows_per_order, h))


def test_heads_gather_every_row(heads_layer):
    R_ = HT.rows_per_order
    ids = np.stack([(np.arange(R_) * (2 * h + 1)) % R_ for h in range(16)], axis=1).astype(np.int32)
    e = torch.empty(R_, HT.row_dim, dtype=torch.float16, device="cuda")
    ple.ple_gather_rows(heads_layer.handle, dev_i32(ids), R_, e)
    torch.cuda.synchronize()
    ulp = fp16_ulps(e.cpu().numpy(), O.embed(heads_layer.host_table, ids))
    assert ulp.max() <= 1


@pytest.mark.parametrize("lengths", [[1000], [1, 2, 3, 600, 0, 400], [253], [254, 253, 1], [4096]])
@pytest.mark.parametrize("path", [0, 2])
def test_heads_forward(heads_layer, lengths, path):
    toks, offs, hid = batch(HT, lengths, sum(lengths) + len(lengths))
    ref = oracle(heads_layer, toks, offs, hid)
    out, _ = gpu_forward(heads_layer, toks, offs, hid, 1, path=path)
    got = out.cpu().numpy().astype(np.float64)
    assert_close(got, ref["out"], f"heads {lengths} path {path}")
    out16, _ = gpu_forward(heads_layer, toks, offs, hid, 0, path=path)
    from ple_inputs.device import bf16_bits
    assert np.array_equal(bf16_bits(out16), O.to_bf16_bits(got))
    assert_bf16_close(bf16_bits(out16), ref["out"])


def test_heads_forward_carried_state(heads_layer):
    toks, _, hid = batch(HT, [900], 5)
    rng = np.random.default_rng(6)
    offs = np.array([0, 300, 301, 301, 900], np.int32)
    hist0 = rng.integers(-1, HT.vocab, (4, 2)).astype(np.int32)
    conv0 = rng.standard_normal((4, 3, HT.hidden)).astype(np.float32)
    ref = oracle(heads_layer, toks, offs, hid, hist=hist0, conv=conv0)
    out, st = gpu_forward(heads_layer, toks, offs, hid, 1, state=(hist0, conv0))
    assert_close(out.cpu().numpy(), ref["out"], "heads with state")
    assert np.array_equal(st[0].cpu().numpy(), ref["hist_out"])
    assert_close(st[1].cpu().numpy(), ref["conv_out"], "heads conv state")


def test_heads_prepared_equals_forward(heads_layer):
    from ple_inputs.device import bf16_tensor
    toks, offs, hid = batch(HT, [700, 300], 9)
    ref, _ = gpu_forward(heads_layer, toks, offs, hid, 1)
    out = torch.empty_like(ref)
    L = heads_layer
    ple.ple_prepare(L.handle, dev_i32(toks), len(toks), dev_i32(offs), 2)
    ple.ple_forward_prepared(L.handle, bf16_tensor(hid), out, 1)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    assert torch.equal(out, ref)


@pytest.mark.parametrize("B,q", [(8, 1), (4, 3), (64, 3)])
def test_heads_decode_step(heads_layer, B, q):
    rng = np.random.default_rng(B * 10 + q)
    toks = rng.integers(0, HT.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, HT.hidden)
    hist = rng.integers(-1, HT.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, HT.hidden)).astype(np.float32)
    n_commit = rng.integers(1, q + 1, B).astype(np.int32)
    from ple_inputs.device import bf16_tensor
    out = torch.empty(B * q, HT.hidden, dtype=torch.float32, device="cuda")
    hs, cs = dev_i32(hist), torch.from_numpy(conv).cuda()
    ple.ple_decode_step(heads_layer.handle, dev_i32(toks), B, q, bf16_tensor(hid), out, 1, hs, cs, dev_i32(n_commit))
    torch.cuda.synchronize()
    assert ple.ple_get_error(heads_layer.handle) == 0
    W = heads_layer.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, heads_layer.host_table, HT.rows_per_order,
                            hist, conv, n_commit)
    assert_close(out.cpu().numpy(), ref["out"], f"heads decode {B}x{q}")
    assert np.array_equal(hs.cpu().numpy(), ref["hist_out"])
    assert_close(cs.cpu().numpy(), ref["conv_out"], "heads decode state")


# ----------------------------------------------------------------------------- full scale
def test_heads_full_ids_and_prefill(heads_full_layer):
    L = heads_full_layer
    w = L.w
    toks, offs, hid = pi.prefill_batch(pi.workload("prefill"))
    assert np.array_equal(gpu_ids(L, toks, offs), O.ngram_ids_heads(toks, offs, w.rows_per_order))
    out, _ = gpu_forward(L, toks, offs, hid, 1)
    rng = np.random.default_rng(44)
    sample = np.unique(np.concatenate([rng.choice(len(toks), 400, replace=False), offs[:-1], offs[1:] - 1,
                                       np.arange(250, 260)]))
    ref = oracle(L, toks, offs, hid, sample=sample)
    assert_close(out.cpu().numpy()[sample], ref["out"], "full-scale heads prefill")


def test_heads_full_decode(heads_full_layer):
    L = heads_full_layer
    w = L.w
    rng = np.random.default_rng(45)
    B, q = 8, 1
    toks = rng.integers(0, w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B, w.hidden)
    hist = rng.integers(0, w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, w.hidden)).astype(np.float32)
    from ple_inputs.device import bf16_tensor
    out = torch.empty(B, w.hidden, dtype=torch.float32, device="cuda")
    hs, cs = dev_i32(hist), torch.from_numpy(conv).cuda()
    ple.ple_decode_step(L.handle, dev_i32(toks), B, q, bf16_tensor(hid), out, 1, hs, cs, None)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    W = L.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, w.rows_per_order, hist, conv)
    assert_close(out.cpu().numpy(), ref["out"], "full-scale heads decode")
    assert np.array_equal(hs.cpu().numpy(), ref["hist_out"])
