"""ple_embed_static: the row lookup for callers that cannot allocate device memory.

Engines whose caching allocator owns the whole device budget, and runtimes
that forbid device allocation after start-up, cannot call cudaMalloc (or
ple_create, which allocates) when they run the layer. ple_embed_static
serves them: it computes the n-gram row IDs into a fixed array inside the
library and gathers the dequantised rows into the caller's buffer.

This test checks it through the C ABI against the handle-based entry points
(ple_ngram_ids followed by ple_gather_rows) on two calls in a row, the second
one smaller than the first, so that contents the fixed array keeps from the
earlier call cannot leak into a later result; against the CPU oracle (the
n-gram row IDs, then the dequantised rows, within one fp16 ulp) with unequal
sub-table sizes and carried history; and that a call allocates no device
memory. The file's name makes pytest collect it last.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _reference_embed(layer, tokens, offsets, hist):
    """The existing path: row IDs through a handle, then the gather stage."""
    T = len(tokens)
    ids = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    ple.ple_ngram_ids(layer.handle, _i32(tokens), T, _i32(offsets), len(offsets) - 1,
                      None if hist is None else _i32(hist), ids)
    e = torch.empty(T, layer.w.row_dim, dtype=torch.float16, device="cuda")
    ple.ple_gather_rows(layer.handle, ids, T, e)
    torch.cuda.synchronize()
    assert ple.ple_get_error(layer.handle) == 0
    return e.cpu().numpy()


def _static_embed(layer, tokens, offsets, hist):
    w = layer.w
    T = len(tokens)
    e = torch.full((T, w.row_dim), float("nan"), dtype=torch.float16, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ple.ple_embed_static(_i32(tokens), T, _i32(offsets), len(offsets) - 1, None if hist is None else _i32(hist),
                         layer.table, layer.scales, w.rows_per_order, w.rows_per_order, w.row_dim, w.vocab, e,
                         status)
    torch.cuda.synchronize()
    return e.cpu().numpy(), int(status.item())


def test_embed_static_matches_handle_path_on_consecutive_calls():
    from ple_inputs.device import DeviceLayer
    w = pi.workload("tiny")
    layer = DeviceLayer(w, max_tokens=2048, max_seqs=16)
    try:
        rng = np.random.default_rng(2024)
        calls = [
            (rng.integers(0, w.vocab, 1500), [0, 700, 701, 701, 1500], rng.integers(-1, w.vocab, (4, 2))),
            (rng.integers(0, w.vocab, 37), [0, 2, 37], None),
        ]
        for tokens, offsets, hist in calls:
            got, status = _static_embed(layer, tokens, offsets, hist)
            ref = _reference_embed(layer, tokens, offsets, hist)
            assert status == 0
            # same kernels and the same inputs: the rows must agree bit for bit
            assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
    finally:
        layer.close()


def test_embed_static_rejects_too_many_tokens():
    w = pi.workload("tiny")
    T = ple.PLE_STATIC_MAX_TOKENS + 1
    with pytest.raises(ValueError):
        ple.ple_embed_static(0, T, 0, 1, None, 0, 0, w.rows_per_order, w.rows_per_order, w.row_dim, w.vocab, 0)
    # the C entry point itself refuses the size before touching any pointer
    code = ple.lib().ple_embed_static(None, T, None, 1, None, None, None, w.rows_per_order, w.rows_per_order,
                                      w.row_dim, w.vocab, None, None, None)
    assert code == 2


def test_embed_static_reports_range_errors():
    from ple_inputs.device import DeviceLayer
    w = pi.workload("tiny")
    layer = DeviceLayer(w, max_tokens=64, max_seqs=2)
    try:
        _, status = _static_embed(layer, np.array([1, 2, w.vocab, 3]), [0, 4], None)
        assert status == 4
        _, status = _static_embed(layer, np.array([1, 2, 3]), [0, 3], None)
        assert status == 0                      # the status word is cleared by each call
    finally:
        layer.close()


def _static_call(tokens, offsets, hist, table, scales, rows0, rows1, row_dim, vocab, e, status):
    ple.ple_embed_static(_i32(tokens), len(tokens), _i32(offsets), len(offsets) - 1,
                         None if hist is None else _i32(hist), table, scales, rows0, rows1, row_dim, vocab, e, status)


def test_embed_static_matches_oracle_unequal_sub_tables():
    """Rows within one fp16 ulp of the oracle's e = deq(bigram row) + deq(trigram row), with
    sub-tables of 3,001 and 4,000 rows laid back to back in one buffer (order 1 starts at row
    3,001) and carried history, on two calls in a row."""
    w = pi.workload("tiny")
    D = w.row_dim
    codes, scales = w.table().full()                  # [2][4096][D], [2][4096]
    flat_codes = codes.reshape(-1, D)
    flat_scales = scales.reshape(-1)
    rows0, rows1 = 3001, 4000
    host = O.ArrayTable([flat_codes[:rows0], flat_codes[rows0:rows0 + rows1]],
                        [flat_scales[:rows0], flat_scales[rows0:rows0 + rows1]])
    table = torch.from_numpy(np.ascontiguousarray(flat_codes)).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(flat_scales)).cuda()
    rng = np.random.default_rng(77)
    calls = [
        (rng.integers(0, w.vocab, 900), [0, 1, 1, 2, 450, 900],
         np.array([[-1, -1], [5, 6], [-1, 9], [7, 8], [100, 200]])),
        (rng.integers(0, w.vocab, 64), [0, 64], np.array([[12, 13]])),
    ]
    for tokens, offsets, hist in calls:
        T = len(tokens)
        e = torch.full((T, D), float("nan"), dtype=torch.float16, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        _static_call(tokens, offsets, hist, table, sc, rows0, rows1, D, w.vocab, e, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        ids = O.ngram_ids(np.asarray(tokens, np.int32), offsets, (rows0, rows1), hist)
        ref16 = O.embed(host, ids).astype(np.float16)
        a = e.cpu().numpy().view(np.uint16).astype(np.int32)
        b = ref16.view(np.uint16).astype(np.int32)
        ulp = np.abs(np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF) - np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF))
        assert ulp.max() <= 1, ulp.max()


def test_embed_static_allocates_nothing():
    """After a first call on the device, a call changes neither the device's free memory nor
    torch's allocated bytes: its only scratch is the library's fixed array."""
    w = pi.workload("tiny")
    codes, scales = w.table().full()
    table = torch.from_numpy(np.ascontiguousarray(codes.reshape(-1))).cuda()
    sc = torch.from_numpy(np.ascontiguousarray(scales.reshape(-1))).cuda()
    rng = np.random.default_rng(5)
    tokens = _i32(rng.integers(0, w.vocab, 4096))
    offsets = _i32([0, 1000, 4096])
    e = torch.empty(4096, w.row_dim, dtype=torch.float16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    R = w.rows_per_order

    def call():
        ple.ple_embed_static(tokens, 4096, offsets, 2, None, table, sc, R, R, w.row_dim, w.vocab, e, status)

    call()
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0
    assert int(status.item()) == 0


def test_embed_static_empty_batch_writes_status():
    """T == 0 launches no lookup but still reports PLE_OK in the caller's status word."""
    w = pi.workload("tiny")
    status = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    offsets = _i32([0, 0])
    R = w.rows_per_order
    ple.ple_embed_static(0, 0, offsets, 1, None, 0, 0, R, R, w.row_dim, w.vocab, 0, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_embed_static_rejects_oversize_rows():
    w = pi.workload("tiny")
    code = ple.lib().ple_embed_static(None, 4, None, 1, None, None, None, w.rows_per_order, w.rows_per_order,
                                      65536 + 16, w.vocab, None, None, None)
    assert code == 8
