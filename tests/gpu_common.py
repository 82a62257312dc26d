"""Shared fixtures and comparison helpers for the GPU parity tests."""
import numpy as np
import pytest

import oracle as O
import ple_inputs as pi

# Float tolerance of the layer's fp32 output against the float64 oracle.
MAX_ABS = 2e-2
REL_L2 = 1e-3


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    d = got - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / denom) if denom > 0 else float(np.linalg.norm(d))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max abs {max_abs:.3e}, rel L2 {rel:.3e}"
    return max_abs, rel


def assert_bf16_close(bits: np.ndarray, ref: np.ndarray):
    """bf16 output vs the float64 oracle: within the fp32 tolerance plus the bf16
    rounding error (half an ulp, at most 2^-8 of the magnitude)."""
    got = O.bf16_bits_to_f64(bits)
    bound = MAX_ABS + np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= bound)


def bf16_to_f64(bits):
    return O.bf16_bits_to_f64(bits)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """|a - b| in units in the last place of bf16 (sign-magnitude ordering)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(key(a_bits) - key(b_bits))


@pytest.fixture(scope="session")
def tiny_layer():
    import torch  # noqa: F401
    from ple_inputs.device import DeviceLayer
    w = pi.workload("tiny")
    L = DeviceLayer(w, max_tokens=2048, max_seqs=64)
    codes, scales = w.table().full()
    L.host_table = O.ArrayTable(codes, scales)
    yield L
    L.close()


_SHARED = {}


def release_device_memory(layer):
    """Close a layer, drop its device tensors and return the cached blocks to the
    driver, so that the next module's full-scale table finds the memory free."""
    import gc
    import torch
    layer.close()
    for name in ("table", "scales", "block_scales", "w_proj", "w_gate", "conv_w"):
        if hasattr(layer, name):
            setattr(layer, name, None)
    gc.collect()
    torch.cuda.empty_cache()


@pytest.fixture(scope="session")
def full_layer():
    """The full-scale table (51.2 GB) and weights, created once per test process.
    Every test module imports this fixture, and pytest would otherwise build one
    instance per importing module."""
    import torch
    from ple_inputs.device import DeviceLayer
    if "full" not in _SHARED:
        w = pi.workload("prefill")
        free, _ = torch.cuda.mem_get_info()
        if free < w.table_bytes + (8 << 30):
            pytest.skip(f"needs {w.table_bytes / 1e9:.0f} GB for the full table, {free / 1e9:.0f} GB free")
        L = DeviceLayer(w, max_tokens=16384, max_seqs=64)
        L.host_table = w.table()
        _SHARED["full"] = L
    return _SHARED["full"]


MID = pi.Workload("mid", 5000, 8192, 128, 256, table_seed=7, seed=7)


@pytest.fixture(scope="session")
def mid_layer():
    """hidden 256: the fused path runs on SM-pair tiles (path 1) or single-SM tiles (path 3)."""
    import torch  # noqa: F401
    from ple_inputs.device import DeviceLayer
    L = DeviceLayer(MID, max_tokens=4096, max_seqs=64)
    codes, scales = MID.table().full()
    L.host_table = O.ArrayTable(codes, scales)
    yield L
    L.close()
