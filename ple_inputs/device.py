"""Device-resident synthetic inputs for the GPU tests and the benchmark.

Allocates the synthetic table, scales and weights of a workload in device
memory (torch is used only to allocate and to copy), fills the table with the
device generator, and creates a libple handle over them. Nothing here computes
any part of the layer.
"""
from __future__ import annotations

import numpy as np
import torch

import gram_embedding_lookup_b200 as ple
from . import Workload, fill_nv_rows_table_device, fill_nv_table_device, fill_table_device


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns (uint16 ndarray) -> torch.bfloat16 tensor on `device`."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class DeviceLayer:
    """A workload's table and weights on the current device, plus a libple handle.

    table_format ple.PLE_TABLE_NVFP4 builds the synthetic NVFP4 table instead
    (packed codes in ``table``, E4M3 block scales in ``block_scales``);
    ple.PLE_TABLE_NVFP4_ROWS the same contents row by row in ``table`` (each
    row's codes, then its block scales);
    ple.PLE_TABLE_E4M3_HEADS builds the multi-head table (16 sub-tables of
    rows_per_order rows of row_dim / 16 codes)."""

    def __init__(self, w: Workload, max_tokens: int, max_seqs: int, weights=None, stream=None,
                 table_format: int = 0, prepare_slots: int = 1):
        self.w = w
        self.table_format = table_format
        R, D, H = w.rows_per_order, w.row_dim, w.hidden
        s = torch.cuda.current_stream() if stream is None else stream
        heads = table_format == ple.PLE_TABLE_E4M3_HEADS
        self.scales = torch.empty((16 if heads else 2) * R, dtype=torch.float32, device="cuda")
        if heads:
            # 16 sub-tables of R rows x D/16 codes: the bytes of a [2][8R][D/16] table
            self.table = torch.empty(R * D, dtype=torch.uint8, device="cuda")
            self.block_scales = None
            fill_table_device(self.table.data_ptr(), self.scales.data_ptr(), 8 * R, D // 16, w.table_seed,
                              s.cuda_stream)
        elif table_format == ple.PLE_TABLE_NVFP4:
            self.table = torch.empty(2 * R * D // 2, dtype=torch.uint8, device="cuda")
            self.block_scales = torch.empty(2 * R * D // 16, dtype=torch.uint8, device="cuda")
            fill_nv_table_device(self.table.data_ptr(), self.block_scales.data_ptr(), self.scales.data_ptr(), R, D,
                                 w.table_seed, s.cuda_stream)
        elif table_format == ple.PLE_TABLE_NVFP4_ROWS:
            self.table = torch.empty(2 * R * (D // 2 + D // 16), dtype=torch.uint8, device="cuda")
            self.block_scales = None
            fill_nv_rows_table_device(self.table.data_ptr(), self.scales.data_ptr(), R, D, w.table_seed,
                                      s.cuda_stream)
        else:
            self.table = torch.empty(2 * R * D, dtype=torch.uint8, device="cuda")
            self.block_scales = None
            fill_table_device(self.table.data_ptr(), self.scales.data_ptr(), R, D, w.table_seed, s.cuda_stream)
        self.host_weights = weights if weights is not None else w.weights()
        self.w_proj = bf16_tensor(self.host_weights.w_proj)
        self.w_gate = bf16_tensor(self.host_weights.w_gate)
        self.conv_w = torch.from_numpy(np.ascontiguousarray(self.host_weights.conv_w, np.float32)).cuda()
        cfg = ple.PleConfig()
        cfg.vocab, cfg.hidden, cfg.row_dim = w.vocab, H, D
        cfg.max_tokens, cfg.max_seqs, cfg.table_format = max_tokens, max_seqs, table_format
        cfg.prepare_slots = prepare_slots
        cfg.rows[0] = R
        cfg.rows[1] = R
        self.config = cfg
        pw = ple.PleWeights(self.table.data_ptr(), self.scales.data_ptr(), self.w_proj.data_ptr(),
                            self.w_gate.data_ptr(), self.conv_w.data_ptr(),
                            self.block_scales.data_ptr() if self.block_scales is not None else None)
        self.weights = pw
        self.handle = ple.ple_create(cfg, pw, s.cuda_stream)

    def close(self):
        if self.handle:
            ple.ple_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
