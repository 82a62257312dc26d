"""The layer captured in CUDA graphs (the pages' engines replay decode steps from
graphs) replays to the same bits as eager launches.

Every call is stream-ordered and does its host work (argument checks, tensor
maps, launch planning) at capture time; the kernels keep no state between
launches that a replay could see stale. The forms captured: a decode step
(the tokens kernel, then the channel-split projection under programmatic
dependent launch), an MTP-style decode step on the split-K path, prefills on
SM-pair and single-SM tiles (of 4,096 tokens too, whose embed is two launches)
and a small forward on the split-K path (projection then combine).
"""
import numpy as np
import pytest

import ple_inputs as pi
from tests.gpu_common import MID, mid_layer  # noqa: F401

torch = pytest.importorskip("torch")
ple = pytest.importorskip("gram_embedding_lookup_b200")

pytestmark = pytest.mark.gpu


def _i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def test_decode_step_graph_replay_matches_eager(mid_layer):  # noqa: F811
    from ple_inputs.device import bf16_tensor
    L = mid_layer
    B, q, steps = 8, 1, 5
    rng = np.random.default_rng(31)
    toks = [rng.integers(0, MID.vocab, (B, q)).astype(np.int32) for _ in range(steps)]
    hids = [pi.hidden_bf16(rng, B * q, MID.hidden) for _ in range(steps)]
    hist0 = rng.integers(0, MID.vocab, (B, 2)).astype(np.int32)
    conv0 = rng.standard_normal((B, 3, MID.hidden)).astype(np.float32)

    # eager
    hs, cs = _i32(hist0), torch.from_numpy(conv0).cuda()
    outs = []
    for k in range(steps):
        out = torch.empty(B * q, MID.hidden, dtype=torch.float32, device="cuda")
        ple.ple_decode_step(L.handle, _i32(toks[k]), B, q, bf16_tensor(hids[k]), out, 1, hs, cs, None)
        outs.append(out)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0

    # one captured step on static buffers, replayed per step after refilling the inputs
    s_tok = _i32(toks[0])
    s_hid = bf16_tensor(hids[0])
    s_out = torch.empty(B * q, MID.hidden, dtype=torch.float32, device="cuda")
    s_hs, s_cs = _i32(hist0), torch.from_numpy(conv0).cuda()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):                     # warm-up launch outside the capture
        ple.ple_decode_step(L.handle, s_tok, B, q, s_hid, s_out, 1, _i32(hist0), torch.from_numpy(conv0).cuda(), None,
                            stream.cuda_stream)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        ple.ple_decode_step(L.handle, s_tok, B, q, s_hid, s_out, 1, s_hs, s_cs, None,
                            torch.cuda.current_stream().cuda_stream)
    s_hs.copy_(_i32(hist0))
    s_cs.copy_(torch.from_numpy(conv0).cuda())
    for k in range(steps):
        s_tok.copy_(_i32(toks[k]))
        s_hid.copy_(bf16_tensor(hids[k]))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(s_out, outs[k]), k
    assert torch.equal(s_hs, hs) and torch.equal(s_cs, cs)
    assert ple.ple_get_error(L.handle) == 0
    del graph


@pytest.mark.parametrize("lengths,path", [([1500, 700, 1], 1), ([40, 3, 5], 2), ([4000, 90, 6], 1), ([4000, 0, 96], 3)])
def test_forward_graph_replay_matches_eager(mid_layer, lengths, path):  # noqa: F811
    """4,096-token batches take the two-launch embed (row IDs, then the bulk-copy
    pipeline as its programmatic dependent) ahead of the projection."""
    from ple_inputs.device import bf16_tensor
    L = mid_layer
    rng = np.random.default_rng(sum(lengths))
    T = sum(lengths)
    toks = _i32(rng.integers(0, MID.vocab, T))
    offs = _i32(np.concatenate([[0], np.cumsum(lengths)]))
    hid = bf16_tensor(pi.hidden_bf16(rng, T, MID.hidden))
    S = len(lengths)
    ple.ple_set_forward_path(L.handle, path)
    try:
        ref = torch.empty(T, MID.hidden, dtype=torch.bfloat16, device="cuda")
        ple.ple_forward(L.handle, toks, T, offs, S, hid, ref, 0)
        torch.cuda.synchronize()
        out = torch.full_like(ref, float("nan"))
        stream = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            ple.ple_forward(L.handle, toks, T, offs, S, hid, out, 0, None, torch.cuda.current_stream().cuda_stream)
        for _ in range(3):
            out.fill_(float("nan"))
            graph.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, ref)
        assert ple.ple_get_error(L.handle) == 0
        del graph
    finally:
        ple.ple_set_forward_path(L.handle, 0)


@pytest.mark.parametrize("path,kernels", [(0, 2), (2, 3)])
def test_split_decode_step_graph_replay_matches_eager(mid_layer, path, kernels):  # noqa: F811
    """A decode step of more than 16 tokens (an MTP-style step with n_commit): the
    tokens kernel, then the split-K projection with its sums, gate, conv and state
    in one kernel (automatic path), or the split-K projection and a combine kernel
    (path 2), chained by programmatic dependent launch. Captured once, it replays
    to the same bits."""
    from ple_inputs.device import bf16_tensor
    L = mid_layer
    ple.ple_set_forward_path(L.handle, path)
    try:
        _split_decode_graph(L, kernels)
    finally:
        ple.ple_set_forward_path(L.handle, 0)


def _split_decode_graph(L, kernels):
    from ple_inputs.device import bf16_tensor
    B, q = 24, 3
    rng = np.random.default_rng(32)
    tok = rng.integers(0, MID.vocab, (B, q)).astype(np.int32)
    hid = pi.hidden_bf16(rng, B * q, MID.hidden)
    hist0 = rng.integers(0, MID.vocab, (B, 2)).astype(np.int32)
    conv0 = rng.standard_normal((B, 3, MID.hidden)).astype(np.float32)
    nc = _i32(rng.integers(1, q + 1, B))
    hs, cs = _i32(hist0), torch.from_numpy(conv0).cuda()
    ref = torch.empty(B * q, MID.hidden, dtype=torch.float32, device="cuda")
    n0 = ple.ple_launch_count(L.handle)
    ple.ple_decode_step(L.handle, _i32(tok), B, q, bf16_tensor(hid), ref, 1, hs, cs, nc)
    torch.cuda.synchronize()
    assert ple.ple_get_error(L.handle) == 0
    assert ple.ple_launch_count(L.handle) - n0 == kernels
    s_tok, s_hid = _i32(tok), bf16_tensor(hid)
    s_hs, s_cs = _i32(hist0), torch.from_numpy(conv0).cuda()
    out = torch.empty_like(ref)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        ple.ple_decode_step(L.handle, s_tok, B, q, s_hid, out, 1, s_hs, s_cs, nc, torch.cuda.current_stream().cuda_stream)
    s_hs.copy_(_i32(hist0))
    s_cs.copy_(torch.from_numpy(conv0).cuda())
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(s_hs, hs) and torch.equal(s_cs, cs)
    assert ple.ple_get_error(L.handle) == 0
    del graph
