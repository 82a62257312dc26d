"""The C-ABI libraries load and export every declared symbol (CPU only: no kernels run)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header: str):
    with open(os.path.join(ROOT, "include", header)) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ple_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def libple():
    import gram_embedding_lookup_b200 as ple
    if not os.path.exists(ple.LIB_PATH):
        from gram_embedding_lookup_b200.build import build
        build()
    return ple.lib()


def test_header_declares_the_boundary():
    names = _declared("ple.h")
    for n in ["ple_create", "ple_destroy", "ple_ngram_ids", "ple_gather_rows", "ple_forward", "ple_decode_step",
              "ple_get_error", "ple_status_string"]:
        assert n in names


def test_every_declared_symbol_is_exported(libple):
    for header in os.listdir(os.path.join(ROOT, "include")):
        if header.endswith(".h"):
            for name in _declared(header):
                assert hasattr(libple, name), f"{name} ({header}) not exported"


def test_synth_library_exports():
    import ple_inputs
    lib = ple_inputs._synth_lib()
    assert hasattr(lib, "ple_synth_fill_table") and hasattr(lib, "ple_synth_stream_base")


def test_synth_stream_base_matches_host():
    import ple_inputs
    lib = ple_inputs._synth_lib()
    for seed, tag in [(0, 1), (1, 2), (12345, 1), (2**63 + 5, 2)]:
        assert lib.ple_synth_stream_base(seed, tag) == ple_inputs.stream_base(seed, tag)


def test_status_strings(libple):
    import gram_embedding_lookup_b200 as ple
    for code in range(9):
        assert ple.ple_status_string(code) not in ("", "unknown status")
    assert ple.ple_status_string(99) == "unknown status"


def test_null_arguments_rejected_on_host(libple):
    """Argument errors are returned before anything touches the device."""
    import gram_embedding_lookup_b200 as ple
    out = ctypes.c_void_p()
    assert libple.ple_create(None, None, None, ctypes.byref(out)) == 1
    cfg = ple.PleConfig(vocab=10, hidden=100, row_dim=64, max_tokens=4, max_seqs=1)
    wts = ple.PleWeights(16, 16, 16, 16, 16)
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 8  # hidden % 128
    cfg.hidden = 128
    cfg.rows[0] = 0
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 1
    cfg.rows[0] = cfg.rows[1] = 16
    wts.table = 17
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 3  # misaligned
    wts.table = 16
    cfg.table_format = 4                          # no such format
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 1
    cfg.table_format = ple.PLE_TABLE_E4M3_HEADS   # 16 head rows need row_dim % 256 == 0 ...
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 8
    cfg.row_dim = 256
    cfg.rows[1] = 17                              # ... and equal rows per head sub-table
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 1
    cfg.row_dim, cfg.rows[1] = 64, 16
    cfg.table_format = ple.PLE_TABLE_NVFP4        # NVFP4 needs block scales
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 1
    wts.block_scales = 24                         # ... 16-byte aligned
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 3
    cfg.table_format = ple.PLE_TABLE_NVFP4_ROWS   # rows of row_dim * 9/16 bytes need row_dim % 256 == 0 ...
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 8
    cfg.row_dim = 256                             # ... and keep the block scales in the rows
    assert libple.ple_create(ctypes.byref(cfg), ctypes.byref(wts), None, ctypes.byref(out)) == 1
    assert libple.ple_destroy(None) == 1
    assert libple.ple_forward(None, None, 0, None, 1, None, None, 0, None, None) == 1
    assert libple.ple_decode_step(None, None, 1, 1, None, None, 0, None, None, None, None) == 1
    assert libple.ple_ngram_ids(None, None, 0, None, 1, None, None, None) == 1
    assert libple.ple_gather_rows(None, None, 0, None, None) == 1
    assert libple.ple_get_error(None) == 1
    assert libple.ple_launch_count(None) == -1
    assert libple.ple_wait_selftest(None, 1000, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import gram_embedding_lookup_b200 as ple
    monkeypatch.setattr(ple, "_LIB", None)
    monkeypatch.setattr(ple, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        ple.lib()
