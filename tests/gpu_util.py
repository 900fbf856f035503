"""Helpers shared by the GPU parity tests: host<->device bf16 bits, oracle comparisons."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from tests.msa_check import compare_selection_row, log_ties, sel_sorted_ok_rows


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def check_selection(gpu_sel, ora_sel, kth, q_idx_rows, pooled_g, t, label="unlabelled"):
    """Compare the selections of rows of one group under the near-tie rule; logs the counts
    under `label` and returns (n_near, n_cancel). Asserts that every GPU row is a valid,
    ascending, -1 padded set and that every difference is an allowed near-tie."""
    gpu_sel = np.asarray(gpu_sel)
    ora_sel = np.asarray(ora_sel)
    assert sel_sorted_ok_rows(gpu_sel).all(), "GPU selection rows not ascending / -1 padded"
    differ = np.nonzero((gpu_sel != ora_sel).any(axis=1))[0]
    near = cancel = 0
    bad = []
    for r in differ:
        c = int(t[r]) // 128
        s = oracle.block_scores(q_idx_rows[r], pooled_g, c)
        absscale = (np.abs(f32(q_idx_rows[r]).astype(np.float64)[None, :] * pooled_g[:c]).sum(1) / 8.0
                    if c else None)
        ok, n1, n2 = compare_selection_row(gpu_sel[r], ora_sel[r], s, kth[r], absscale)
        if not ok:
            bad.append((int(t[r]), list(gpu_sel[r]), list(ora_sel[r])))
        near += n1
        cancel += n2
    log_ties(label, len(t), len(differ), near, cancel)
    assert not bad, f"{len(bad)} selection mismatches beyond near-ties, first: {bad[:3]}"
    return near, cancel
