"""Helpers shared by the GPU parity tests: moving synthetic inputs to the
device and comparing the CUDA path with the oracle under the stated tolerances.

Tolerances (from the method's parity contract):
  counts, slices, warped depth  bit-exact
  selected blocks               bit-exact except rows whose differing blocks
                                all sit within TIE_TOL of the oracle's
                                selection threshold (counted and reported)
  attention output (bf16 in)    max-abs <= 2e-2 and mean-abs <= 2e-3
"""
from __future__ import annotations

import numpy as np
import torch

TIE_TOL = 1e-4
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def compare_selection(gpu_idx: np.ndarray, oracle_idx: np.ndarray, s_mod: np.ndarray, m: int,
                      tol: float = TIE_TOL) -> int:
    """Returns the number of rows that differ only at near-ties; raises on any
    other difference. Arrays are [..., topk] with matching leading shape;
    s_mod [..., n_past] holds the oracle's modulated scores."""
    g = gpu_idx.reshape(-1, gpu_idx.shape[-1])
    o = oracle_idx.reshape(-1, oracle_idx.shape[-1])
    s = s_mod.reshape(-1, s_mod.shape[-1])
    n_past = s.shape[1]
    k_past = g.shape[1] - m
    ties = 0
    for r in range(g.shape[0]):
        row = g[r]
        assert (np.diff(row) > 0).all(), f"row {r}: indices not strictly ascending"
        assert row[k_past:].tolist() == list(range(n_past, n_past + m)), f"row {r}: current chunk"
        if np.array_equal(row, o[r]):
            continue
        theta = np.sort(s[r])[::-1][k_past - 1]
        diff = set(row.tolist()) ^ set(o[r].tolist())
        bad = [kb for kb in diff if abs(s[r][kb] - theta) >= tol]
        assert not bad, f"row {r}: blocks {bad[:8]} differ beyond the tie tolerance"
        ties += 1
    return ties


def compare_attention(o_gpu: torch.Tensor, o_ref: np.ndarray, what: str = "O"):
    got = o_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - o_ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: max-abs {mx:.3g} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean-abs {mean:.3g} > {O_MEAN_ABS}"
    return mx, mean
