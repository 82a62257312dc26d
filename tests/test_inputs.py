"""The seeded input generators (CPU)."""
import numpy as np

import ple_inputs as pi


def test_splitmix64_published_sequence():
    """splitmix64 seeded with 1234567: the first five outputs of the published generator."""
    idx = np.arange(5, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(1234567) + (idx + np.uint64(1)) * np.uint64(pi.GAMMA)
    assert pi._mix(z).tolist() == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                                   4593380528125082431, 16408922859458223821]


def test_table_codes_finite_and_uniform():
    t = pi.SynthTable(seed=0, rows_per_order=4096, row_dim=64)
    codes, scales = t.full()
    assert codes.dtype == np.uint8 and codes.shape == (2, 4096, 64)
    counts = np.bincount(codes.reshape(-1), minlength=256)
    assert counts[0x7F] == 0 and counts[0xFF] == 0
    finite = np.delete(counts, [0x7F, 0xFF])
    expect = codes.size / 254
    chi2 = ((finite - expect) ** 2 / expect).sum()
    assert chi2 < 253 + 6 * np.sqrt(2 * 253)
    assert scales.dtype == np.float32 and scales.min() >= 0.01 and scales.max() < 0.1


def test_table_rows_on_demand_match_full():
    t = pi.SynthTable(seed=5, rows_per_order=300, row_dim=32)
    codes, scales = t.full()
    rows = np.array([0, 299, 17, 17])
    assert np.array_equal(t.codes(1, rows), codes[1][rows])
    assert np.array_equal(t.scales(0, rows), scales[0][rows])


def test_bf16_inputs_round_nearest_even():
    import torch
    x = np.random.default_rng(0).standard_normal(1000).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(pi.f32_to_bf16_bits(x), lib)


def test_workload_shapes():
    w = pi.workload("prefill")
    toks, offs, hid = pi.prefill_batch(w)
    assert offs.tolist() == [0, 1000, 4384, 8384, 16384]
    assert toks.shape == (16384,) and hid.shape == (16384, 2560)
    assert toks.min() >= 0 and toks.max() < 248_320
    assert w.table_bytes == 51_200_245_760
    d = pi.workload("decode")
    tk, h, hist, conv = pi.decode_batch(d)
    assert tk.shape == (8, 1) and hist.shape == (8, 2) and conv.shape == (8, 3, 2560)


def test_zipf_is_heavy_tailed():
    rng = np.random.default_rng(3)
    t = pi.tokens_zipf(rng, 100_000, 248_320)
    top = np.mean(t == 0)
    expect = 1.0 / np.sum(np.arange(1, 248_321, dtype=np.float64) ** -1.1)   # P(rank 1) ~ 0.130
    assert abs(top - expect) < 5 * np.sqrt(expect * (1 - expect) / t.size)


def test_mtp_session_structure():
    w = pi.workload("mtp")
    s = pi.mtp_session(w, steps=5)
    assert s["prompts"].shape == (64, 512)
    assert np.all(s["prompts"][:19] == s["prompts"][0])
    for toks, hid, nc in s["steps"]:
        assert toks.shape == (64, 3) and hid.shape == (192, 2560)
        assert np.all(toks[:19] == toks[0]) and nc.min() >= 1 and nc.max() <= 3


def test_nv_packed_rows_layout():
    """The row layout of the NVFP4 table: row r is its D/2 code bytes, then its D/16
    block-scale bytes (9D/16 bytes), the same contents as the two-array layout."""
    t = pi.SynthNvTable(seed=3, rows_per_order=64, row_dim=256)
    rows = np.array([0, 63, 5, 5])
    p = t.packed_rows(1, rows)
    assert p.dtype == np.uint8 and p.shape == (4, 256 // 2 + 256 // 16)
    assert np.array_equal(p[:, :128], t.codes(1, rows))
    assert np.array_equal(p[:, 128:], t.block_scales(1, rows))
    assert not np.array_equal(t.packed_rows(0, rows), p)
