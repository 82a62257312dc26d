"""GPU parity of the NVFP4 table variant against the oracle, in both layouts.

Every call goes through the C ABI. The table is the synthetic NVFP4 table of
``ple_inputs`` (packed E2M1 codes, E4M3 block scales, per-row fp32 scales),
stored either in two arrays (PLE_TABLE_NVFP4) or row by row with each row's
block scales after its codes (PLE_TABLE_NVFP4_ROWS, which needs row_dim % 256
== 0: its small workloads are the tiny and mid ones at row_dim 256). The
oracle reads the same contents through ``oracle.Nvfp4ArrayTable`` or the host
generator, whatever the layout.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

from tests.gpu_common import MID, assert_bf16_close, assert_close, release_device_memory  # noqa: E402
from tests.test_gpu_parity import _sample, dev_bf16, dev_i32, gpu_decode, gpu_forward, to_bits  # noqa: E402

pytestmark = pytest.mark.gpu


LAYOUTS = [ple.PLE_TABLE_NVFP4, ple.PLE_TABLE_NVFP4_ROWS]
LAYOUT_IDS = ["arrays", "rows"]


def _wide(w, name):
    """The workload at row_dim 256 (the row layout's smallest row width)."""
    return pi.Workload(name, w.vocab, w.rows_per_order, 256, w.hidden, w.table_seed, w.seed, w.extra)


def _layer(w, max_tokens, max_seqs, fmt):
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(w, max_tokens=max_tokens, max_seqs=max_seqs, table_format=fmt)
    L.rows_layout = fmt == ple.PLE_TABLE_NVFP4_ROWS
    return L


def _code_views(L):
    """Torch views [2][R][D/2] of the device codes and [2][R][D/16] of the block scales."""
    R, D = L.w.rows_per_order, L.w.row_dim
    if L.rows_layout:
        t = L.table.view(2, R, D // 2 + D // 16)
        return t[:, :, :D // 2], t[:, :, D // 2:]
    return L.table.view(2, R, D // 2), L.block_scales.view(2, R, D // 16)


@pytest.fixture(scope="module", params=LAYOUTS, ids=LAYOUT_IDS)
def nv_tiny(request):
    w = pi.workload("tiny")
    if request.param == ple.PLE_TABLE_NVFP4_ROWS:
        w = _wide(w, "tiny256")
    L = _layer(w, 4608, 64, request.param)
    L.host_table = O.Nvfp4ArrayTable(*pi.SynthNvTable(w.table_seed, w.rows_per_order, w.row_dim).full())
    yield L
    L.close()


@pytest.fixture(scope="module", params=LAYOUTS, ids=LAYOUT_IDS)
def nv_mid(request):
    w = MID if request.param == ple.PLE_TABLE_NVFP4 else _wide(MID, "mid256")
    L = _layer(w, 4096, 64, request.param)
    L.host_table = O.Nvfp4ArrayTable(*pi.SynthNvTable(w.table_seed, w.rows_per_order, w.row_dim).full())
    yield L
    L.close()


@pytest.fixture(scope="module", params=LAYOUTS, ids=LAYOUT_IDS)
def nv_full(request):
    w = pi.workload("prefill")
    need = 2 * w.rows_per_order * (w.row_dim // 2 + w.row_dim // 16)
    free, _ = torch.cuda.mem_get_info()
    if free < need + (8 << 30):
        pytest.skip(f"needs {need / 1e9:.0f} GB for the NVFP4 table, {free / 1e9:.0f} GB free")
    L = _layer(w, 16384, 64, request.param)
    L.host_table = pi.SynthNvTable(w.table_seed, w.rows_per_order, w.row_dim)
    yield L
    release_device_memory(L)


def _gather(L, ids):
    T = ids.shape[0]
    e = torch.empty(T, L.w.row_dim, dtype=torch.float16, device="cuda")
    ple.ple_gather_rows(L.handle, dev_i32(ids), T, e)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    return e.cpu().numpy()


def _ulp(a16, b16):
    a = a16.view(np.uint16).astype(np.int32)
    b = b16.view(np.uint16).astype(np.int32)
    ka = np.where(a & 0x8000, -(a & 0x7FFF), a & 0x7FFF)
    kb = np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(ka - kb)


def test_nv_device_table_matches_host_generator(nv_tiny):
    w = nv_tiny.w
    syn = pi.SynthNvTable(w.table_seed, w.rows_per_order, w.row_dim)
    codes, blocks, scales = syn.full()
    if nv_tiny.rows_layout:
        r = np.arange(w.rows_per_order)
        packed = np.stack([syn.packed_rows(0, r), syn.packed_rows(1, r)])
        assert np.array_equal(nv_tiny.table.cpu().numpy(), packed.ravel())
    else:
        assert np.array_equal(nv_tiny.table.cpu().numpy(), codes.ravel())
        assert np.array_equal(nv_tiny.block_scales.cpu().numpy(), blocks.ravel())
    c, b = _code_views(nv_tiny)
    assert np.array_equal(c.cpu().numpy(), codes) and np.array_equal(b.cpu().numpy(), blocks)
    assert np.array_equal(nv_tiny.scales.cpu().numpy(), scales.ravel())


def test_nv_gather_tiny_all_rows(nv_tiny):
    R = nv_tiny.w.rows_per_order
    ids = np.stack([np.arange(R), (np.arange(R) * 7919) % R], axis=1)[:2048]
    got = _gather(nv_tiny, ids)
    ref = O.embed(nv_tiny.host_table, ids).astype(np.float16)
    assert _ulp(got, ref).max() <= 1


def test_nv_gather_every_code_and_block_scale(nv_tiny):
    """Every code byte (both nibbles, every position) against block scales of every
    kind: ordinary, subnormal E4M3, 448, zero and NaN (0x7F). The first 256 rows of
    each order are overwritten and restored afterwards."""
    L = nv_tiny
    R, D = L.w.rows_per_order, L.w.row_dim
    n = 256
    k = np.arange(D // 2)
    codes = np.empty((2, n, D // 2), np.uint8)
    for i in range(n):
        codes[0, i] = (i * 7 + k) % 256
        codes[1, i] = (i * 3 + 5 * k + 11) % 256
    kinds = np.array([0x38, 0x30, 0x01, 0x07, 0x7E, 0x00, 0x7F, 0xB8, 0x3F, 0x44], np.uint8)
    blocks = np.empty((2, n, D // 16), np.uint8)
    for i in range(n):
        blocks[0, i] = kinds[(i + np.arange(D // 16)) % len(kinds)]
        blocks[1, i] = kinds[(3 * i + 2 * np.arange(D // 16) + 1) % len(kinds)]
    scales = np.stack([np.linspace(0.01, 0.2, n), np.linspace(0.3, 0.02, n)]).astype(np.float32)
    tab, blk = _code_views(L)
    sc = L.scales.view(2, R)
    saved = (tab[:, :n].clone(), blk[:, :n].clone(), sc[:, :n].clone())
    try:
        tab[:, :n] = torch.from_numpy(codes).cuda()
        blk[:, :n] = torch.from_numpy(blocks).cuda()
        sc[:, :n] = torch.from_numpy(scales).cuda()
        t = np.arange(2048)
        ids = np.stack([t % n, (t * 37 + t // n) % n], axis=1)
        got = _gather(L, ids)
    finally:
        tab[:, :n], blk[:, :n], sc[:, :n] = saved
        torch.cuda.synchronize()
    with np.errstate(invalid="ignore", over="ignore"):
        exact = O.embed(O.Nvfp4ArrayTable(codes, blocks, scales), ids)
        # the same table with every sign bit cleared: the sum of the two terms' magnitudes
        mag = O.embed(O.Nvfp4ArrayTable(codes & 0x77, blocks & 0x7F, np.abs(scales)), ids)
    ref = exact.astype(np.float16)
    nan = np.isnan(ref)
    assert nan.any() and np.array_equal(np.isnan(got), nan)
    # e is computed in fp32 and rounded to fp16: within one fp16 ulp, except where
    # the two orders' terms cancel, there within the fp32 rounding of the terms
    # (2^-23 of their magnitudes) plus an fp16 ulp
    ulp = _ulp(got[~nan], ref[~nan])
    err = np.abs(got[~nan].astype(np.float64) - exact[~nan])
    lim = 2.0 ** -23 * mag[~nan] + np.abs(np.spacing(ref[~nan]))
    assert np.all((ulp <= 1) | (err <= lim))
    assert np.mean(ulp > 1) < 1e-4


@pytest.mark.parametrize("path", [0, 1, 2])
def test_nv_forward_tiny(nv_tiny, path):
    toks, offs, hid = pi.tiny_batch(nv_tiny.w)
    ref = O.ple_forward(toks, offs, hid, nv_tiny.host_weights.w_proj, nv_tiny.host_weights.w_gate,
                        nv_tiny.host_weights.conv_w, nv_tiny.host_table, nv_tiny.w.rows_per_order)
    out, _ = gpu_forward(nv_tiny, toks, offs, hid, 1, path=path)
    assert_close(out, ref["out"], f"nvfp4 tiny path {path}")
    out16, _ = gpu_forward(nv_tiny, toks, offs, hid, 0, path=path)
    assert np.array_equal(out16, O.to_bf16_bits(out))


@pytest.mark.parametrize("path", [1, 2, 3])
def test_nv_forward_mid_with_state(nv_mid, path):
    rng = np.random.default_rng(31 + path)
    lengths = [700, 1, 2, 253, 1100]
    T = sum(lengths)
    toks = rng.integers(0, MID.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, MID.hidden)
    S = len(lengths)
    hist = rng.integers(-1, MID.vocab, (S, 2)).astype(np.int32)
    conv = rng.standard_normal((S, 3, MID.hidden)).astype(np.float32)
    W = nv_mid.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, nv_mid.host_table, MID.rows_per_order,
                        hist=hist, conv_state=conv)
    out, st = gpu_forward(nv_mid, toks, offs, hid, 1, state=(hist, conv), path=path)
    assert_close(out, ref["out"], f"nvfp4 mid path {path}")
    assert np.array_equal(st[0], ref["hist_out"])
    assert_close(st[1], ref["conv_out"], "nvfp4 mid state")


@pytest.mark.parametrize("lengths", [[4000, 90, 6], [1, 4200, 0, 17]])
def test_nv_bulk_embed_batches(nv_tiny, lengths):
    """Batches of 4,096 tokens or more take the bulk-copy embed (every NVFP4 row
    in one copy in the row layout, two in the array layout): every output
    against the oracle, with carried state."""
    w = nv_tiny.w
    rng = np.random.default_rng(sum(lengths))
    T, S = sum(lengths), len(lengths)
    toks = rng.integers(0, w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, w.hidden)
    hist = rng.integers(-1, w.vocab, (S, 2)).astype(np.int32)
    conv = rng.standard_normal((S, 3, w.hidden)).astype(np.float32)
    W = nv_tiny.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, nv_tiny.host_table, w.rows_per_order,
                        hist=hist, conv_state=conv)
    out, st = gpu_forward(nv_tiny, toks, offs, hid, 1, state=(hist, conv))
    assert_close(out, ref["out"], f"nvfp4 bulk embed {lengths}")
    assert np.array_equal(st[0], ref["hist_out"])
    assert_close(st[1], ref["conv_out"], "nvfp4 bulk embed state")


@pytest.mark.parametrize("shape", [(1, 1), (8, 1), (5, 3), (16, 1), (6, 3)])
def test_nv_decode_paths_tiny(nv_tiny, shape):
    w = nv_tiny.w
    B, q = shape
    rng = np.random.default_rng(B * 10 + q)
    toks = rng.integers(0, w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, w.hidden)
    hist = rng.integers(-1, w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, w.hidden)).astype(np.float32)
    nc = rng.integers(1, q + 1, B).astype(np.int32)
    W = nv_tiny.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, nv_tiny.host_table, w.rows_per_order,
                            hist, conv, n_commit=nc)
    for path in (0, 2):
        ple.ple_set_forward_path(nv_tiny.handle, path)
        out, h2, c2 = gpu_decode(nv_tiny, toks, hid, hist, conv, nc)
        ple.ple_set_forward_path(nv_tiny.handle, 0)
        assert_close(out, ref["out"], f"nvfp4 decode {shape} path {path}")
        assert np.array_equal(h2, ref["hist_out"])
        assert_close(c2, ref["conv_out"], f"nvfp4 decode state {shape}")


def test_nv_gather_full_sample(nv_full):
    rng = np.random.default_rng(12)
    R = nv_full.w.rows_per_order
    ids = np.stack([rng.integers(0, R, 512), rng.integers(0, R, 512)], axis=1)
    ids[:4] = [[0, 0], [R - 1, R - 1], [0, R - 1], [R - 1, 0]]
    got = _gather(nv_full, ids)
    ref = O.embed(nv_full.host_table, ids).astype(np.float16)
    assert _ulp(got, ref).max() <= 1


def test_nv_prefill_full_sampled(nv_full):
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w)
    T = len(toks)
    out, _ = gpu_forward(nv_full, toks, offs, hid, 1)
    sample = _sample(T, offs, 600, 23)
    W = nv_full.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, nv_full.host_table, w.rows_per_order,
                        sample=sample)
    assert_close(out[sample], ref["out"], "nvfp4 prefill")


def test_nv_decode_full(nv_full):
    w = pi.workload("decode")
    toks, hid, hist, conv = pi.decode_batch(w)
    W = nv_full.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, nv_full.host_table, w.rows_per_order,
                            hist, conv)
    out, h2, c2 = gpu_decode(nv_full, toks, hid, hist, conv)
    assert_close(out, ref["out"], "nvfp4 full decode")
    assert np.array_equal(h2, ref["hist_out"])
    out16, _, _ = gpu_decode(nv_full, toks, hid, hist, conv, out_dtype=0)
    assert_bf16_close(out16, ref["out"])
