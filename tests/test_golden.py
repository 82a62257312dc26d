"""The pages' printed figures against the table geometry and row layouts that
the oracle and the synthetic inputs use (CPU only).

The figures live in ``tests/golden/page_figures.txt``, each with the page and
section it comes from. They fix the table's size in bytes (two orders of
10,000,048 rows of 2560 E4M3 codes, or 16 heads of 160-byte rows), its size
in BF16 and in NVFP4 (which pins the NVFP4 layout at 4.5 bits per element:
packed codes plus one E4M3 block scale per 16 elements), and the model's
hidden size and vocabulary.
"""
import os

import numpy as np

import oracle as O
import ple_inputs as pi

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "page_figures.txt")
HASH_EXAMPLE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hash_worked_example.txt")


def hash_worked_example():
    """The worked example of the n-gram hash: [(rows, tokens, [(bigram row, trigram row), ...]), ...]
    for one sequence each with no carried history (``tests/golden/hash_worked_example.txt``)."""
    cases = []
    with open(HASH_EXAMPLE, encoding="utf-8") as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            rows, toks, ids = (part.split() for part in line.split("|"))
            pairs = [tuple(int(v) for v in pair.split(",")) for pair in ids]
            cases.append((int(rows[0]), [int(t) for t in toks], pairs))
    return cases


def _figures():
    out = {}
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            head, cite = line.split("|", 1)
            name, value = head.split()
            assert cite.strip(), f"{name} has no citation"
            out[name] = float(value) if "." in value else int(value)
    return out


F = _figures()


def test_fixture_lists_every_figure():
    assert set(F) == {"ple_table_bytes", "ple_table_bytes_card", "ple_table_gib", "ple_table_bf16_gib",
                      "ple_table_nvfp4_gib", "lookups_per_token", "fp8_row_bytes", "hidden", "vocab"}


def test_two_order_table_bytes():
    w = pi.workload("prefill")
    # the oracle reads one code byte per element of a row
    codes = np.full((1, w.row_dim), 0x38, np.uint8)
    assert O.dequantise(codes, np.ones(1, np.float32)).shape == (1, w.row_dim)
    assert 2 * w.rows_per_order * codes.shape[1] == F["ple_table_bytes"] == F["ple_table_bytes_card"]
    assert round(F["ple_table_bytes"] / 2 ** 30, 2) == F["ple_table_gib"]


def test_multi_head_table_geometry():
    w = pi.workload("heads_full")
    heads = 2 * O.HEADS_PER_ORDER
    assert heads == F["lookups_per_token"]
    assert w.row_dim // heads == F["fp8_row_bytes"]
    assert heads * w.rows_per_order * (w.row_dim // heads) == F["ple_table_bytes"]


def test_bf16_and_nvfp4_table_sizes():
    w = pi.workload("prefill")
    R, D = w.rows_per_order, w.row_dim
    assert round(2 * R * D * 2 / 2 ** 30, 2) == F["ple_table_bf16_gib"]
    # the NVFP4 layout the oracle reads: D/2 bytes of packed codes, D/16 block-scale bytes per row
    packed = np.zeros((1, D // 2), np.uint8)
    blocks = np.full((1, D // 16), 0x38, np.uint8)
    assert O.dequantise_nvfp4(packed, blocks, np.ones(1, np.float32)).shape == (1, D)
    assert round(2 * R * (packed.shape[1] + blocks.shape[1]) / 2 ** 30, 2) == F["ple_table_nvfp4_gib"]


def test_model_dimensions():
    w = pi.workload("prefill")
    assert w.hidden == F["hidden"]
    assert w.vocab == F["vocab"]


def test_hash_worked_example_fixture_shape():
    cases = hash_worked_example()
    assert [(r, len(t)) for r, t, _ in cases] == [(4096, 5), (10_000_048, 5), (10_000_048, 3)]
    for rows, toks, ids in cases:
        assert len(ids) == len(toks)
        assert all(0 <= a < rows and 0 <= b < rows for a, b in ids)
