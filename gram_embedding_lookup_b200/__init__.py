"""Python binding of libple, the B200 n-gram embedding (PLE) layer.

A thin ctypes layer over the C ABI declared in ``include/ple.h``: the functions
below carry the same names and arguments as the C entry points and only
marshal arguments (device pointers may be given as ints or as torch tensors,
whose ``data_ptr()`` is used; streams as ints or ``torch.cuda.Stream``).
Every step of the layer runs in the library's CUDA kernels. If ``libple.so``
has not been built, importing works but every call raises ``RuntimeError``.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "PleError", "PleConfig", "PleWeights", "PleState", "lib", "ple_create", "ple_destroy",
    "ple_ngram_ids", "ple_gather_rows", "ple_forward", "ple_prepare", "ple_forward_prepared", "ple_decode_step",
    "ple_decode_prepare", "ple_decode_step_prepared", "ple_prepare_slot", "ple_forward_prepared_slot",
    "ple_get_error",
    "ple_status_string", "ple_set_profiling", "ple_get_stage_times", "ple_set_forward_path",
    "ple_launch_count", "ple_wait_selftest", "ple_embed_static", "PLE_STATIC_MAX_TOKENS", "PLE_OUT_BF16", "PLE_OUT_F32",
    "PLE_TABLE_E4M3", "PLE_TABLE_NVFP4", "PLE_TABLE_E4M3_HEADS", "PLE_TABLE_NVFP4_ROWS", "STATUS",
    "STAGES", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libple.so")

PLE_OUT_BF16 = 0
PLE_OUT_F32 = 1
PLE_TABLE_E4M3 = 0
PLE_TABLE_NVFP4 = 1
PLE_TABLE_E4M3_HEADS = 2   # 16 hash-head sub-tables of row_dim / 16 codes; row IDs [T][16]
PLE_TABLE_NVFP4_ROWS = 3   # the NVFP4 table with each row's block scales after its codes
PLE_STATIC_MAX_TOKENS = 16384   # the fixed row-ID array of ple_embed_static
STATUS = {0: "PLE_OK", 1: "PLE_ERR_INVALID_ARG", 2: "PLE_ERR_SHAPE", 3: "PLE_ERR_ALIGN", 4: "PLE_ERR_RANGE",
          5: "PLE_ERR_OOM", 6: "PLE_ERR_CUDA", 7: "PLE_ERR_TIMEOUT", 8: "PLE_ERR_UNSUPPORTED"}
STAGES = ("prepare", "gather", "gemm", "combine")


class PleError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{what}: {self.name} ({ple_status_string(code)})")


class PleConfig(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int32), ("hidden", ctypes.c_int32), ("row_dim", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("max_seqs", ctypes.c_int32), ("table_format", ctypes.c_int32),
                ("prepare_slots", ctypes.c_int32), ("rows", ctypes.c_int64 * 2)]


class PleWeights(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("w_proj", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p), ("conv_w", ctypes.c_void_p), ("block_scales", ctypes.c_void_p)]


class PleState(ctypes.Structure):
    _fields_ = [("hist", ctypes.c_void_p), ("conv", ctypes.c_void_p)]


_LIB = None
_VP = ctypes.c_void_p
_I32 = ctypes.c_int32


def lib() -> ctypes.CDLL:
    """The loaded libple.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m gram_embedding_lookup_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "ple_create": ([ctypes.POINTER(PleConfig), ctypes.POINTER(PleWeights), _VP, ctypes.POINTER(_VP)], _I32),
            "ple_destroy": ([_VP], _I32),
            "ple_ngram_ids": ([_VP, _VP, _I32, _VP, _I32, _VP, _VP, _VP], _I32),
            "ple_gather_rows": ([_VP, _VP, _I32, _VP, _VP], _I32),
            "ple_forward": ([_VP, _VP, _I32, _VP, _I32, _VP, _VP, _I32, ctypes.POINTER(PleState), _VP], _I32),
            "ple_decode_step": ([_VP, _VP, _I32, _I32, _VP, _VP, _I32, _VP, _VP, _VP, _VP], _I32),
            "ple_prepare": ([_VP, _VP, _I32, _VP, _I32, _VP, _VP], _I32),
            "ple_forward_prepared": ([_VP, _VP, _VP, _I32, ctypes.POINTER(PleState), _VP], _I32),
            "ple_decode_prepare": ([_VP, _VP, _I32, _I32, _VP, _VP], _I32),
            "ple_prepare_slot": ([_VP, _I32, _VP, _I32, _VP, _I32, _VP, _VP], _I32),
            "ple_forward_prepared_slot": ([_VP, _I32, _VP, _VP, _I32, ctypes.POINTER(PleState), _VP], _I32),
            "ple_decode_step_prepared": ([_VP, _VP, _VP, _I32, _VP, _VP, _VP, _VP], _I32),
            "ple_get_error": ([_VP], _I32),
            "ple_status_string": ([_I32], ctypes.c_char_p),
            "ple_set_profiling": ([_VP, _I32], _I32),
            "ple_get_stage_times": ([_VP, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int64)], _I32),
            "ple_set_forward_path": ([_VP, _I32], _I32),
            "ple_launch_count": ([_VP], ctypes.c_int64),
            "ple_wait_selftest": ([_VP, ctypes.c_int64, _VP], _I32),
            "ple_embed_static": ([_VP, _I32, _VP, _I32, _VP, _VP, _VP, ctypes.c_int64, ctypes.c_int64, _I32, _I32,
                                  _VP, _VP, _VP], _I32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x or None
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "cuda_stream"):
        return x.cuda_stream or None
    raise TypeError(f"cannot pass {type(x)} as a device pointer")


def _stream(s) -> int | None:
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream or None
    return int(s) or None


def _check(code: int, what: str) -> None:
    if code != 0:
        raise PleError(code, what)


def ple_status_string(code: int) -> str:
    try:
        return lib().ple_status_string(code).decode()
    except RuntimeError:
        return STATUS.get(code, "unknown")


def ple_create(config: PleConfig, weights: PleWeights, stream=None) -> int:
    h = _VP()
    _check(lib().ple_create(ctypes.byref(config), ctypes.byref(weights), _stream(stream), ctypes.byref(h)),
           "ple_create")
    return h.value


def ple_destroy(handle: int) -> None:
    _check(lib().ple_destroy(handle), "ple_destroy")


def ple_ngram_ids(handle, tokens, T, offsets, S, hist, ids, stream=None) -> None:
    _check(lib().ple_ngram_ids(handle, _ptr(tokens), T, _ptr(offsets), S, _ptr(hist), _ptr(ids), _stream(stream)),
           "ple_ngram_ids")


def ple_gather_rows(handle, ids, T, e_out, stream=None) -> None:
    _check(lib().ple_gather_rows(handle, _ptr(ids), T, _ptr(e_out), _stream(stream)), "ple_gather_rows")


def ple_forward(handle, tokens, T, offsets, S, hidden, out, out_dtype, state=None, stream=None) -> None:
    st = None
    if state is not None:
        hist, conv = state
        st = ctypes.byref(PleState(_ptr(hist), _ptr(conv)))
    _check(lib().ple_forward(handle, _ptr(tokens), T, _ptr(offsets), S, _ptr(hidden), _ptr(out), out_dtype, st,
                             _stream(stream)), "ple_forward")


def ple_prepare(handle, tokens, T, offsets, S, hist=None, stream=None) -> None:
    _check(lib().ple_prepare(handle, _ptr(tokens), T, _ptr(offsets), S, _ptr(hist), _stream(stream)), "ple_prepare")


def ple_forward_prepared(handle, hidden, out, out_dtype, state=None, stream=None) -> None:
    st = None
    if state is not None:
        hist, conv = state
        st = ctypes.byref(PleState(_ptr(hist), _ptr(conv)))
    _check(lib().ple_forward_prepared(handle, _ptr(hidden), _ptr(out), out_dtype, st, _stream(stream)),
           "ple_forward_prepared")


def ple_decode_step(handle, tokens, B, q, hidden, out, out_dtype, hist, conv_state, n_commit=None,
                    stream=None) -> None:
    _check(lib().ple_decode_step(handle, _ptr(tokens), B, q, _ptr(hidden), _ptr(out), out_dtype, _ptr(hist),
                                 _ptr(conv_state), _ptr(n_commit), _stream(stream)), "ple_decode_step")


def ple_prepare_slot(handle, slot, tokens, T, offsets, S, hist=None, stream=None) -> None:
    _check(lib().ple_prepare_slot(handle, slot, _ptr(tokens), T, _ptr(offsets), S, _ptr(hist), _stream(stream)),
           "ple_prepare_slot")


def ple_forward_prepared_slot(handle, slot, hidden, out, out_dtype, state=None, stream=None) -> None:
    st = None
    if state is not None:
        hist, conv = state
        st = ctypes.byref(PleState(_ptr(hist), _ptr(conv)))
    _check(lib().ple_forward_prepared_slot(handle, slot, _ptr(hidden), _ptr(out), out_dtype, st, _stream(stream)),
           "ple_forward_prepared_slot")


def ple_decode_prepare(handle, tokens, B, q, hist, stream=None) -> None:
    _check(lib().ple_decode_prepare(handle, _ptr(tokens), B, q, _ptr(hist), _stream(stream)), "ple_decode_prepare")


def ple_decode_step_prepared(handle, hidden, out, out_dtype, hist, conv_state, n_commit=None, stream=None) -> None:
    _check(lib().ple_decode_step_prepared(handle, _ptr(hidden), _ptr(out), out_dtype, _ptr(hist), _ptr(conv_state),
                                          _ptr(n_commit), _stream(stream)), "ple_decode_step_prepared")


def ple_get_error(handle) -> int:
    """The sticky device status (0 = ok), cleared by the call."""
    return lib().ple_get_error(handle)


def ple_set_profiling(handle, enable: bool) -> None:
    _check(lib().ple_set_profiling(handle, 1 if enable else 0), "ple_set_profiling")


def ple_get_stage_times(handle):
    """{stage: (milliseconds, launches)} since the previous call."""
    ms = (ctypes.c_float * 4)()
    n = (ctypes.c_int64 * 4)()
    _check(lib().ple_get_stage_times(handle, ms, n), "ple_get_stage_times")
    return {STAGES[i]: (float(ms[i]), int(n[i])) for i in range(4)}


def ple_set_forward_path(handle, path: int) -> None:
    _check(lib().ple_set_forward_path(handle, path), "ple_set_forward_path")


def ple_launch_count(handle) -> int:
    return int(lib().ple_launch_count(handle))


def ple_wait_selftest(handle, limit_cycles: int, stream=None) -> None:
    """Run one bounded device wait that nothing completes (see include/ple.h); the
    handle's status then reads PLE_ERR_TIMEOUT."""
    _check(lib().ple_wait_selftest(handle, int(limit_cycles), _stream(stream)), "ple_wait_selftest")


def ple_embed_static(tokens, T, offsets, S, hist, table, scales, rows0, rows1, row_dim, vocab, e_out,
                     status_out=None, stream=None) -> None:
    """N-gram row IDs and row gather into e_out (fp16 [T][row_dim]) without any
    device allocation, for callers that cannot allocate: the row IDs go to a
    fixed array in the library (at most PLE_STATIC_MAX_TOKENS tokens per call,
    one call at a time per device; see include/ple.h)."""
    if T > PLE_STATIC_MAX_TOKENS:
        raise ValueError(f"ple_embed_static takes at most {PLE_STATIC_MAX_TOKENS} tokens per call, got {T}")
    _check(lib().ple_embed_static(_ptr(tokens), T, _ptr(offsets), S, _ptr(hist), _ptr(table), _ptr(scales),
                                  rows0, rows1, row_dim, vocab, _ptr(e_out), _ptr(status_out), _stream(stream)),
           "ple_embed_static")
