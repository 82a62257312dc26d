"""Plant plausible mistakes in the CPU oracle and check that a pin catches each.

Every mutation is applied to the oracle on the CPU (monkeypatch) and removed
after the test; the GPU path is not involved.
"""
import numpy as np
import pytest

import oracle as O
import oracle.ple_oracle as OP
import tests.test_oracle_pins as pins


def _fails(fn):
    try:
        fn()
    except (AssertionError, ValueError, IndexError):
        return True
    return False


def _patch(monkeypatch, name, fn):
    monkeypatch.setattr(OP, name, fn)
    monkeypatch.setattr(O, name, fn)


def test_reversed_conv_taps_caught(monkeypatch):
    def bad(u_hist, conv_w):
        return OP.__dict__["_orig_short_conv"](u_hist, np.asarray(conv_w)[:, ::-1])
    monkeypatch.setitem(OP.__dict__, "_orig_short_conv", OP.short_conv)
    _patch(monkeypatch, "short_conv", bad)
    assert _fails(pins.test_short_conv_matches_numpy_convolve)
    assert _fails(pins.test_short_conv_delta_is_identity_and_impulse_response)


def test_gate_sign_flip_caught(monkeypatch):
    orig = OP.gate
    _patch(monkeypatch, "gate", lambda h, w: orig(h, -np.asarray(w, np.float64)))
    assert _fails(pins.test_gate_sign)
    assert _fails(pins.test_zero_gate_returns_hidden)


def test_dropped_trigram_term_caught(monkeypatch):
    def bad(x0, x1, x2):
        k2, _ = OP.__dict__["_orig_keys"](x0, x1, x2)
        return k2, k2
    monkeypatch.setitem(OP.__dict__, "_orig_keys", OP.ngram_keys)
    _patch(monkeypatch, "ngram_keys", bad)
    assert _fails(pins.test_ids_dependence_structure)


def test_swapped_context_index_caught(monkeypatch):
    orig = OP.ngram_contexts

    def bad(tokens, offsets, hist=None):
        x0, x1, x2 = orig(tokens, offsets, hist)
        return x0, x2, x1
    _patch(monkeypatch, "ngram_contexts", bad)
    assert _fails(pins.test_ids_dependence_structure)


def test_dropped_bigram_context_caught(monkeypatch):
    def bad(x0, x1, x2):
        return OP.__dict__["_orig_keys"](x0, 0, x2)
    monkeypatch.setitem(OP.__dict__, "_orig_keys", OP.ngram_keys)
    _patch(monkeypatch, "ngram_keys", bad)
    assert _fails(pins.test_ids_dependence_structure)


def test_swapped_history_slots_caught(monkeypatch):
    orig = OP.ngram_contexts

    def bad(tokens, offsets, hist=None):
        h = None if hist is None else np.asarray(hist)[:, ::-1]
        return orig(tokens, offsets, h)
    _patch(monkeypatch, "ngram_contexts", bad)
    assert _fails(pins.test_ids_carried_history_equals_whole_sequence)


def test_transposed_projection_caught(monkeypatch):
    _patch(monkeypatch, "project", lambda e, w: np.asarray(e, np.float64) @ np.asarray(w, np.float64).T)
    assert _fails(pins.test_projection_one_hot_picks_weight_row)


def test_missing_order_sum_caught(monkeypatch):
    def bad(table, ids):
        ids = np.asarray(ids, dtype=np.int64)
        return OP.dequantise(table.codes(0, ids[:, 0]), table.scales(0, ids[:, 0]))
    _patch(monkeypatch, "embed", bad)
    assert _fails(pins.test_embed_sums_orders)


def test_wrong_subnormal_decode_caught(monkeypatch):
    table = O.E4M3_VALUES.copy()
    table[1:8] *= 2.0            # subnormals scaled like normals (a classic slip)
    monkeypatch.setattr(OP, "E4M3_VALUES", table)
    monkeypatch.setattr(O, "E4M3_VALUES", table)
    assert _fails(pins.test_e4m3_all_codes_match_torch_float8)


@pytest.mark.parametrize("shift", [31, 33])
def test_wrong_fold_shift_caught_by_brute_force(monkeypatch, shift):
    _patch(monkeypatch, "fold", lambda k: k ^ (k >> shift))
    assert _fails(pins.test_layer_matches_brute_force_tiny)


# ------------------------------------------------------------------ multi-head layout (C-17)
import tests.test_oracle_heads as heads_pins  # noqa: E402


def _bad_heads(mix_of_head, key_of_head):
    def bad(tokens, offsets, rows_per_head, hist=None, heads=OP.HEADS_PER_ORDER):
        x0, x1, x2 = OP.ngram_contexts(tokens, offsets, hist)
        ids = np.zeros((len(x0), 2 * heads), dtype=np.int64)
        for t in range(len(x0)):
            keys = OP.ngram_keys(x0[t], x1[t], x2[t])
            for n in range(2):
                for j in range(heads):
                    k = keys[key_of_head(n)] ^ (mix_of_head(j) * OP.HEAD_MIX & OP._MASK64)
                    ids[t, n * heads + j] = OP.fold(k) % int(rows_per_head)
        return ids
    return bad


def test_heads_trigram_from_bigram_key_caught(monkeypatch):
    _patch(monkeypatch, "ngram_ids_heads", _bad_heads(lambda j: j, lambda n: 0))
    assert _fails(heads_pins.test_heads_dependence_structure)


def test_heads_mix_offset_caught(monkeypatch):
    _patch(monkeypatch, "ngram_ids_heads", _bad_heads(lambda j: j + 1, lambda n: n))
    assert _fails(heads_pins.test_head_zero_is_the_two_order_row)


def test_heads_without_mix_caught(monkeypatch):
    _patch(monkeypatch, "ngram_ids_heads", _bad_heads(lambda j: 0, lambda n: n))
    assert _fails(heads_pins.test_head_zero_is_the_two_order_row)


def test_heads_reversed_concatenation_caught(monkeypatch):
    orig = OP.embed

    def bad(table, ids):
        e = orig(table, ids)
        if getattr(table, "format", "") != "heads":
            return e
        n = np.asarray(ids).shape[1]
        return np.concatenate(np.split(e, n, axis=1)[::-1], axis=1)
    _patch(monkeypatch, "embed", bad)
    assert _fails(heads_pins.test_heads_embed_concatenates_in_head_order)
    assert _fails(heads_pins.test_heads_layer_matches_brute_force)


@pytest.mark.parametrize("bad", [0x9E3779B9, 0x9E3779B97F4A7C13, 0x9E3779B97F4A7C17])
def test_mistyped_hash_multiplier_caught(monkeypatch, bad):
    """The 32-bit golden-ratio constant, or the 64-bit one off in its last digit:
    the structural ID pins still hold for either, the closed-form pin does not."""
    monkeypatch.setattr(OP, "P0", bad)
    monkeypatch.setattr(O, "P0", bad)
    assert _fails(pins.test_hash_multiplier_is_the_golden_ratio_constant)


@pytest.mark.parametrize("name,delta", [("P0", 1 << 8), ("P1", 1 << 36), ("P2", 1 << 4), ("P1", 0x30 << 56)])
def test_one_digit_hash_constant_change_caught(monkeypatch, name, delta):
    """Changing one hex digit of a hash multiplier (kept odd) moves some worked-example row."""
    monkeypatch.setattr(OP, name, getattr(OP, name) ^ delta)
    assert getattr(OP, name) % 2 == 1
    assert _fails(pins.test_ids_match_the_hash_worked_example)


def test_context_offset_dropped_caught(monkeypatch):
    """Contexts without the +1 (token 0 indistinguishable from an absent position)."""
    monkeypatch.setattr(OP, "_context_value", lambda token: int(token) & 0xFFFFFFFF)
    assert _fails(pins.test_ids_match_the_hash_worked_example)
