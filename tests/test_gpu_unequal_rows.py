"""Sub-tables of different sizes (rows[0] != rows[1]) through the C ABI.

The layout puts row r of sub-table n at (n * rows[0] + r): order 1 starts after
all of order 0's rows. Every other test uses equal sub-tables, so this file is
the one that would catch an offset or modulus taken from the wrong order.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

from tests.gpu_common import assert_close  # noqa: E402
from tests.test_gpu_parity import dev_i32, gpu_decode, gpu_forward  # noqa: E402

pytestmark = pytest.mark.gpu

R0, R1 = 3000, 5003


class _Layer:
    """A handle over hand-made sub-tables of R0 and R1 rows (E4M3, NVFP4 in two
    arrays, or NVFP4 row by row at row_dim 256)."""

    def __init__(self, fmt):
        from ple_inputs.device import bf16_tensor
        w = pi.workload("tiny")
        if fmt == ple.PLE_TABLE_NVFP4_ROWS:
            w = pi.Workload("tiny256", w.vocab, w.rows_per_order, 256, w.hidden, w.table_seed, w.seed, w.extra)
        self.w = w
        D, H = w.row_dim, w.hidden
        rng = np.random.default_rng(41 + fmt)
        scales = rng.uniform(0.01, 0.1, R0 + R1).astype(np.float32)
        if fmt in (ple.PLE_TABLE_NVFP4, ple.PLE_TABLE_NVFP4_ROWS):
            codes = rng.integers(0, 256, (R0 + R1, D // 2)).astype(np.uint8)
            blocks = rng.integers(0x30, 0x40, (R0 + R1, D // 16)).astype(np.uint8)
            self.host_table = O.Nvfp4ArrayTable([codes[:R0], codes[R0:]], [blocks[:R0], blocks[R0:]],
                                                [scales[:R0], scales[R0:]])
            if fmt == ple.PLE_TABLE_NVFP4_ROWS:             # each row's block scales after its codes
                codes = np.concatenate([codes, blocks], axis=1)
                self.block_scales = None
            else:
                self.block_scales = torch.from_numpy(blocks.ravel()).cuda()
        else:
            codes = rng.integers(0, 256, (R0 + R1, D)).astype(np.uint8)
            codes[(codes & 0x7F) == 0x7F] = 0x42                # finite codes only
            self.host_table = O.ArrayTable([codes[:R0], codes[R0:]], [scales[:R0], scales[R0:]])
            self.block_scales = None
        self.table = torch.from_numpy(codes.ravel()).cuda()
        self.scales = torch.from_numpy(scales).cuda()
        self.host_weights = w.weights()
        self.w_proj = bf16_tensor(self.host_weights.w_proj)
        self.w_gate = bf16_tensor(self.host_weights.w_gate)
        self.conv_w = torch.from_numpy(np.ascontiguousarray(self.host_weights.conv_w, np.float32)).cuda()
        cfg = ple.PleConfig()
        cfg.vocab, cfg.hidden, cfg.row_dim = w.vocab, H, D
        cfg.max_tokens, cfg.max_seqs, cfg.table_format = 2048, 64, fmt
        cfg.rows[0], cfg.rows[1] = R0, R1
        pw = ple.PleWeights(self.table.data_ptr(), self.scales.data_ptr(), self.w_proj.data_ptr(),
                            self.w_gate.data_ptr(), self.conv_w.data_ptr(),
                            None if self.block_scales is None else self.block_scales.data_ptr())
        self.handle = ple.ple_create(cfg, pw)

    def close(self):
        ple.ple_destroy(self.handle)


@pytest.fixture(scope="module", params=[0, 1, 3], ids=["e4m3", "nvfp4", "nvfp4_rows"])
def layer(request):
    L = _Layer(request.param)
    yield L
    L.close()


def test_unequal_rows_ids_and_gather(layer):
    rng = np.random.default_rng(5)
    toks = rng.integers(0, layer.w.vocab, 700).astype(np.int32)
    offs = np.array([0, 300, 301, 700], np.int32)
    ids = torch.empty(700, 2, dtype=torch.int32, device="cuda")
    ple.ple_ngram_ids(layer.handle, dev_i32(toks), 700, dev_i32(offs), 3, None, ids)
    torch.cuda.synchronize()
    got = ids.cpu().numpy()
    assert np.array_equal(got, O.ngram_ids(toks, offs, (R0, R1)))
    assert got[:, 0].max() < R0 and got[:, 1].max() < R1 and got[:, 1].max() >= R0
    # the rows past R0 in order 1 and the last row of each order
    probe = np.array([[R0 - 1, R1 - 1], [0, R0], [R0 - 1, R0 + 7], [5, 0]], np.int32)
    e = torch.empty(len(probe), layer.w.row_dim, dtype=torch.float16, device="cuda")
    ple.ple_gather_rows(layer.handle, dev_i32(probe), len(probe), e)
    torch.cuda.synchronize()
    assert ple.ple_get_error(layer.handle) == 0
    ref = O.embed(layer.host_table, probe).astype(np.float16)
    diff = np.abs(e.cpu().numpy().view(np.uint16).astype(np.int32) - ref.view(np.uint16).astype(np.int32))
    assert diff.max() <= 1


@pytest.mark.parametrize("path", [1, 2])
def test_unequal_rows_forward(layer, path):
    rng = np.random.default_rng(6 + path)
    lengths = [400, 2, 650]
    T = sum(lengths)
    toks = rng.integers(0, layer.w.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, layer.w.hidden)
    W = layer.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, layer.host_table, (R0, R1))
    out, _ = gpu_forward(layer, toks, offs, hid, 1, path=path)
    assert_close(out, ref["out"], f"unequal rows path {path}")


@pytest.mark.parametrize("shape", [(8, 1), (4, 3), (12, 2)])
def test_unequal_rows_decode(layer, shape):
    B, q = shape
    rng = np.random.default_rng(B + 10 * q)
    toks = rng.integers(0, layer.w.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, layer.w.hidden)
    hist = rng.integers(-1, layer.w.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, layer.w.hidden)).astype(np.float32)
    W = layer.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, layer.host_table, (R0, R1), hist, conv)
    for path in (0, 2):
        ple.ple_set_forward_path(layer.handle, path)
        out, h2, c2 = gpu_decode(layer, toks, hid, hist, conv)
        ple.ple_set_forward_path(layer.handle, 0)
        assert_close(out, ref["out"], f"unequal rows decode {shape} path {path}")
        assert np.array_equal(h2, ref["hist_out"])
