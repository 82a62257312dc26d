"""Row widths with an odd number of 64-code K-blocks, on B200 through the C ABI.

The SM-pair projection and the MTP-size decode kernel fetch both operands two
K-blocks per TMA copy (3-D boxes {64, rows, 2}). With 192-wide rows (three
K-blocks) the last box of a tile reaches one K-block past the tensor: TMA fills
it with zeros and counts its bytes, and the kernels do not multiply it. In the
MTP kernel's K-splits of one K-block each, every box also carries the next
split's K-block, which its split leaves out. Both must agree with the CPU
oracle within the float tolerance.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import assert_close

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu

ODD = pi.Workload("odd", 4000, 6000, 192, 256, table_seed=13, seed=13)


@pytest.fixture(scope="module")
def odd_layer():
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(ODD, max_tokens=4096, max_seqs=64)
    codes, scales = ODD.table().full()
    L.host_table = O.ArrayTable(codes, scales)
    yield L
    L.close()


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("lengths,path", [([1000], 1), ([1, 600, 0, 253], 1), ([700, 60], 0)])
def test_forward_odd_kblocks(odd_layer, lengths, path):
    from ple_inputs.device import bf16_tensor
    L = odd_layer
    rng = np.random.default_rng(sum(lengths) + path)
    T = sum(lengths)
    toks = rng.integers(0, ODD.vocab, T).astype(np.int32)
    offs = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    hid = pi.hidden_bf16(rng, T, ODD.hidden)
    W = L.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, ODD.rows_per_order)
    out = torch.empty(T, ODD.hidden, dtype=torch.float32, device="cuda")
    ple.ple_set_forward_path(L.handle, path)
    try:
        ple.ple_forward(L.handle, _i32(toks), T, _i32(offs), len(lengths), bf16_tensor(hid), out, 1)
        torch.cuda.synchronize()
    finally:
        ple.ple_set_forward_path(L.handle, 0)
    assert ple.ple_get_error(L.handle) == 0
    assert_close(out.cpu().numpy().astype(np.float64), ref["out"], f"odd K-blocks {lengths} path {path}")


@pytest.mark.parametrize("B,q", [(64, 3), (20, 2)])
def test_mtp_step_odd_kblocks(odd_layer, B, q):
    from ple_inputs.device import bf16_tensor
    L = odd_layer
    rng = np.random.default_rng(B * 10 + q)
    toks = rng.integers(0, ODD.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, ODD.hidden)
    hist = rng.integers(-1, ODD.vocab, (B, 2)).astype(np.int32)
    conv = rng.standard_normal((B, 3, ODD.hidden)).astype(np.float32)
    nc = rng.integers(1, q + 1, B).astype(np.int32)
    W = L.host_weights
    ref = O.ple_decode_step(toks, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, ODD.rows_per_order, hist, conv,
                            n_commit=nc)
    hs, cs = _i32(hist), torch.from_numpy(conv).cuda()
    out = torch.empty(B * q, ODD.hidden, dtype=torch.float32, device="cuda")
    ple.ple_decode_step(L.handle, _i32(toks), B, q, bf16_tensor(hid), out, 1, hs, cs, _i32(nc))
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    assert_close(out.cpu().numpy().astype(np.float64), ref["out"], f"MTP {B}x{q} odd K-blocks")
    assert np.array_equal(hs.cpu().numpy(), ref["hist_out"])
    assert_close(cs.cpu().numpy(), ref["conv_out"], "MTP state odd K-blocks")
