"""Pins of the oracle's NVFP4 table variant (C-16), on the CPU.

The capacity variant of the pages stores the table in NVFP4: about 26.82 GiB
against 95.37 GiB in BF16 (deletoe.com page, section "第三条路：把 PLE 也量化，
能塞下，但不够快"; DGX Spark report, section "运行时内存占用"). Codes are FP4
E2M1, two per byte with the low nibble first, with one E4M3 scale per 16 codes
and the per-row fp32 scale of the FP8 table kept as the outer factor.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
import ple_inputs as pi

# FP4 E2M1 magnitudes as tabulated in the OCP Microscaling Formats (MX)
# specification v1.0, for codes 0..7; codes 8..15 are their negatives.
OCP_E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_all_codes_match_ocp_table():
    for c in range(16):
        mag = OCP_E2M1[c & 7]
        v = O.e2m1_decode(c)
        assert v == (-mag if c & 8 else mag)
        assert math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0)
    assert np.array_equal(O.E2M1_VALUES, [O.e2m1_decode(c) for c in range(16)])


def _e2m1_as_e4m3_byte(c: int) -> int:
    """The E4M3 encoding of E2M1 code c (every E2M1 value is exact in E4M3)."""
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    if e == 0:
        mag = 0x30 if m else 0x00          # 0.5 = 2^-1 (exponent field 6); 0
    else:
        mag = ((e + 6) << 3) | (m << 2)    # (1 + m/2) 2^(e-1): exponent field e-1+7
    return (s << 7) | mag


def test_e2m1_matches_torch_float8_through_exact_reencoding():
    b = torch.tensor([_e2m1_as_e4m3_byte(c) for c in range(16)], dtype=torch.uint8)
    lib = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(lib, O.E2M1_VALUES)
    assert np.array_equal(np.signbit(lib), np.signbit(O.E2M1_VALUES))


def test_unpack_low_nibble_first():
    codes = O.unpack_fp4(np.array([[0x21, 0xF8, 0x07]], np.uint8))
    assert codes.tolist() == [[1, 2, 8, 15, 7, 0]]
    assert O.E2M1_VALUES[codes[0]].tolist()[:4] == [0.5, 1.0, -0.0, -6.0]


def _small_nv_table(rng, R=16, D=64):
    codes = rng.integers(0, 256, size=(2, R, D // 2)).astype(np.uint8)
    blocks = rng.integers(0x28, 0x48, size=(2, R, D // 16)).astype(np.uint8)
    scales = rng.uniform(0.01, 0.1, size=(2, R)).astype(np.float32)
    return codes, blocks, scales


def test_block_scale_covers_sixteen_elements():
    rng = np.random.default_rng(3)
    codes, blocks, scales = _small_nv_table(rng)
    base = O.dequantise_nvfp4(codes[0], blocks[0], scales[0])
    for j in range(4):
        b2 = blocks[0].copy()
        b2[5, j] = 0x00                    # E4M3 zero: this block of row 5 only
        d = O.dequantise_nvfp4(codes[0], b2, scales[0])
        assert np.all(d[5, 16 * j:16 * j + 16] == 0)
        keep = np.ones_like(d, dtype=bool)
        keep[5, 16 * j:16 * j + 16] = False
        assert np.array_equal(d[keep], base[keep])


def test_dequantise_nvfp4_brute_force():
    rng = np.random.default_rng(4)
    codes, blocks, scales = _small_nv_table(rng, R=6, D=64)
    f8 = torch.from_numpy(blocks[0]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.dequantise_nvfp4(codes[0], blocks[0], scales[0])
    for r in range(codes.shape[1]):
        for k in range(64):
            byte = int(codes[0, r, k // 2])
            c = (byte >> (4 * (k % 2))) & 0xF
            mag = OCP_E2M1[c & 7]
            v = (-mag if c & 8 else mag) * f8[r, k // 16] * float(scales[0, r])
            assert got[r, k] == v


def test_embed_nvfp4_sums_orders():
    rng = np.random.default_rng(5)
    codes, blocks, scales = _small_nv_table(rng)
    tab = O.Nvfp4ArrayTable(codes, blocks, scales)
    ids = np.array([[1, 2], [5, 5], [15, 0]])
    e = O.embed(tab, ids)
    for i, (r0, r1) in enumerate(ids):
        expect = O.dequantise_nvfp4(codes[0][[r0]], blocks[0][[r0]], scales[0][[r0]])[0] + \
            O.dequantise_nvfp4(codes[1][[r1]], blocks[1][[r1]], scales[1][[r1]])[0]
        assert np.array_equal(e[i], expect)


def _brute_force_layer_nv(tokens, hidden, codes, blocks, scales, w_proj, w_gate, conv_w):
    """Scalar loops over one fresh sequence with an NVFP4 table."""
    T, H = hidden.shape
    D = w_proj.shape[0]
    R_ = codes.shape[1]
    M = 1 << 64
    f8 = torch.from_numpy(blocks).view(torch.float8_e4m3fn).to(torch.float64).numpy()

    def ctx(i):
        return int(tokens[i]) + 1 if i >= 0 else 0

    def elem(n, r, k):
        c = (int(codes[n, r, k // 2]) >> (4 * (k % 2))) & 0xF
        mag = OCP_E2M1[c & 7]
        return (-mag if c & 8 else mag) * f8[n, r, k // 16] * float(scales[n, r])

    u = [[0.0] * H for _ in range(T)]
    for t in range(T):
        k2 = (ctx(t) * 0x9E3779B97F4A7C15 % M) ^ (ctx(t - 1) * 0xC2B2AE3D27D4EB4F % M)
        k3 = k2 ^ (ctx(t - 2) * 0x165667B19E3779F9 % M)
        r2 = (k2 ^ (k2 >> 32)) % R_
        r3 = (k3 ^ (k3 >> 32)) % R_
        e = [elem(0, r2, k) + elem(1, r3, k) for k in range(D)]
        a = sum(float(w_gate[j]) * float(hidden[t, j]) for j in range(H))
        g = 1.0 / (1.0 + math.exp(-a))
        for j in range(H):
            u[t][j] = g * sum(e[k] * float(w_proj[k, j]) for k in range(D))
    out = np.zeros((T, H))
    for t in range(T):
        for j in range(H):
            y = sum(float(conv_w[j, k]) * u[t - 3 + k][j] for k in range(4) if t - 3 + k >= 0)
            out[t, j] = float(hidden[t, j]) + y
    return out


def test_layer_with_nvfp4_table_matches_brute_force_tiny():
    w = pi.workload("tiny")
    codes, blocks, scales = pi.SynthNvTable(w.table_seed, w.rows_per_order, w.row_dim).full()
    W = w.weights()
    toks, offs, hid = pi.tiny_batch(w)
    T = 6
    r = O.ple_forward(toks[:T], [0, T], hid[:T], W.w_proj, W.w_gate, W.conv_w,
                      O.Nvfp4ArrayTable(codes, blocks, scales), w.rows_per_order)
    bf = _brute_force_layer_nv(toks[:T], O.bf16_bits_to_f64(hid[:T]), codes, blocks, scales,
                               O.bf16_bits_to_f64(W.w_proj), O.bf16_bits_to_f64(W.w_gate), W.conv_w)
    assert np.allclose(r["out"], bf, rtol=1e-12, atol=1e-12)


def test_synthetic_nv_table_draws():
    t = pi.SynthNvTable(7, 512, 128)
    c = t.codes(1, np.arange(512))
    nib = np.concatenate([c & 15, c >> 4]).ravel()
    counts = np.bincount(nib, minlength=16)
    assert counts.min() > 0.9 * counts.mean() and counts.max() < 1.1 * counts.mean()
    b = t.block_scales(0, np.arange(512))
    assert b.min() == 0x30 and b.max() == 0x3F
    # rows are independent of the other sub-table and reproducible
    assert np.array_equal(t.codes(1, [5]), pi.nv_table_codes(7, 512, 128, 1, [5]))
    assert not np.array_equal(t.codes(0, [5]), t.codes(1, [5]))


@pytest.mark.parametrize("bad", ["high_nibble_first", "block_of_eight", "no_block_scale"])
def test_nvfp4_mutations_are_caught(monkeypatch, bad):
    import oracle.ple_oracle as OP
    orig_unpack, orig_deq = OP.unpack_fp4, OP.dequantise_nvfp4

    if bad == "high_nibble_first":
        def unpack(p):
            c = orig_unpack(p)
            c[..., 0::2], c[..., 1::2] = c[..., 1::2].copy(), c[..., 0::2].copy()
            return c
        monkeypatch.setattr(OP, "unpack_fp4", unpack)
        monkeypatch.setattr(O, "unpack_fp4", unpack)
    else:
        def deq(packed, blocks, scales):
            codes = OP.unpack_fp4(packed)
            b = OP.E4M3_VALUES[np.asarray(blocks, np.uint8)]
            if bad == "block_of_eight":
                per = np.repeat(b, 8, axis=-1)
                per = np.concatenate([per, per], axis=-1)[..., :codes.shape[-1]]
            else:
                per = np.ones(codes.shape)
            return OP.E2M1_VALUES[codes] * per * np.asarray(scales, np.float64)[:, None]
        monkeypatch.setattr(OP, "dequantise_nvfp4", deq)
        monkeypatch.setattr(O, "dequantise_nvfp4", deq)
    caught = 0
    for pin in (test_unpack_low_nibble_first, test_block_scale_covers_sixteen_elements,
                test_dequantise_nvfp4_brute_force, test_layer_with_nvfp4_table_matches_brute_force_tiny):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1
    monkeypatch.setattr(OP, "unpack_fp4", orig_unpack)
    monkeypatch.setattr(OP, "dequantise_nvfp4", orig_deq)
