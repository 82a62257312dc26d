"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's kernels is bounded; when one runs out, the
kernel records PLE_ERR_TIMEOUT in the handle's sticky status and returns. This
test makes such a wait run out on purpose (ple_wait_selftest: an mbarrier that
nothing completes, a limit of about a millisecond) and checks that the status
reports it, that reading the status clears it, and that the CUDA context stays
usable: the layer still matches the oracle afterwards.
"""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi
from tests.gpu_common import assert_close, tiny_layer  # noqa: F401

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu

PLE_ERR_TIMEOUT = 7


def test_bounded_wait_reports_timeout_and_context_survives(tiny_layer):  # noqa: F811
    L = tiny_layer
    h = L.handle
    assert ple.ple_get_error(h) == 0
    ple.ple_wait_selftest(h, 2_000_000)
    assert ple.ple_get_error(h) == PLE_ERR_TIMEOUT
    assert ple.ple_get_error(h) == 0                  # the read clears the sticky status
    w = L.w
    toks, offs, hid = pi.tiny_batch(w)
    from ple_inputs.device import bf16_tensor
    out = torch.empty(len(toks), w.hidden, dtype=torch.float32, device="cuda")
    ple.ple_forward(h, torch.from_numpy(toks).cuda(), len(toks), torch.from_numpy(offs).cuda(), 1, bf16_tensor(hid),
                    out, ple.PLE_OUT_F32)
    torch.cuda.synchronize()
    assert ple.ple_get_error(h) == 0
    W = L.host_weights
    ref = O.ple_forward(toks, offs, hid, W.w_proj, W.w_gate, W.conv_w, L.host_table, w.rows_per_order)
    assert_close(out.cpu().numpy(), ref["out"], "forward after a timed-out wait")


def test_selftest_argument_checks(tiny_layer):  # noqa: F811
    lib = ple.lib()
    assert lib.ple_wait_selftest(None, 1000, None) == 1
    assert lib.ple_wait_selftest(tiny_layer.handle, 0, None) == 1
    assert lib.ple_wait_selftest(tiny_layer.handle, 3_000_000_000, None) == 1
