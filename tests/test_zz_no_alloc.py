"""ple_embed_static: the row lookup for callers that cannot allocate device memory.

Engines whose caching allocator owns the whole device budget, and runtimes
that forbid device allocation after start-up, cannot call cudaMalloc (or
ple_create, which allocates) when they run the layer. ple_embed_static
serves them: it computes the n-gram row IDs into a fixed array inside the
library and gathers the dequantised rows into the caller's buffer.

This test checks it through the C ABI against the handle-based entry points
(ple_ngram_ids followed by ple_gather_rows) on two calls in a row, the second
one smaller than the first, so that contents the fixed array keeps from the
earlier call cannot leak into a later result. The file's name makes pytest
collect it last.
"""
import numpy as np
import pytest

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
