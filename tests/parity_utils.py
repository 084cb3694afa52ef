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

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from oracle import velox_oracle as vo

TIE_TOL = 1e-4
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3

# every selection comparison of the session: (label, near-tie rows, rows compared);
# every attention comparison: (label, rows, worst max-abs, worst mean-abs). Both
# are printed in the terminal summary by conftest.py
TIE_LOG: list = []
ATTN_LOG: list = []


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def tie_bound(rows: int) -> int:
    """Largest near-tie count accepted without question: a few rows, or 1 % of
    them. The rule itself allows any number of near-tie rows; a count above this
    would mean the kernel's scores drift from the oracle's systematically."""
    return max(3, rows // 100)


def compare_selection(gpu_idx: np.ndarray, oracle_idx: np.ndarray, s_mod: np.ndarray, m: int,
                      tol: float = TIE_TOL, label: str | None = None) -> int:
    """Returns the number of rows that differ only at near-ties; raises on any
    other difference. Arrays are [..., topk] with matching leading shape;
    s_mod [..., n_past] holds the oracle's modulated scores. With a label the
    count is logged for the session's tie report."""
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
    if label is not None:
        TIE_LOG.append((label, ties, g.shape[0]))
    return ties


def compare_attention(o_gpu: torch.Tensor, o_ref: np.ndarray, what: str = "O"):
    got = o_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - o_ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: max-abs {mx:.3g} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: mean-abs {mean:.3g} > {O_MEAN_ABS}"
    return mx, mean


def oracle_route_per_head(q: np.ndarray, k: np.ndarray, counts, alpha: float, topk: int, T: int,
                          workers: int = 4):
    """The oracle's routing of every head of q [B,H,Nq,d] / k [B,H,Nk,d], one
    head at a time (a head's float64 keys are 231 MB at 48 past chunks), on a
    few host threads. Returns (idx [B,H,m,topk], s' [B,H,m,n_past])."""
    H = q.shape[1]

    def one(h):
        return vo.route_topk(q[:, h:h + 1], k[:, h:h + 1], counts, alpha, topk, T)

    with ThreadPoolExecutor(max(1, min(workers, H))) as ex:
        res = list(ex.map(one, range(H)))
    return (np.concatenate([r[0] for r in res], axis=1),
            np.concatenate([r[1] for r in res], axis=1))


def attention_rows_vs_oracle(vx, q: np.ndarray, k: np.ndarray, v: np.ndarray, idx: np.ndarray,
                             T: int, rows, label: str, lse_tol: float = 1e-3, workers: int = 8):
    """Runs the CUDA attention on q/k/v (bf16 bit patterns, [B,H,N,d]) with the
    selection idx -- normally the oracle's own, so that rows where the two
    selections differ at a near-tie are still checked -- and compares the
    listed (b, h, qb) query blocks with the oracle's, element by element.
    Returns the worst (max-abs, mean-abs) over the rows."""
    o, lse = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(idx), T)
    o_h = o.float().cpu().numpy().astype(np.float64)
    lse_h = lse.cpu().numpy()

    def one(r):
        return r, vo.sparse_attention(q, k, v, idx, T, rows=[r])[tuple(r)]

    with ThreadPoolExecutor(max(1, min(workers, len(rows)))) as ex:
        ref = list(ex.map(one, rows))
    worst_max = worst_mean = 0.0
    for (b, h, qb), (o_ref, lse_ref) in ref:
        sl = slice(qb * T, (qb + 1) * T)
        err = np.abs(o_h[b, h, sl] - o_ref)
        assert np.isfinite(o_h[b, h, sl]).all(), f"{label} row {(b, h, qb)}: non-finite output"
        mx, mean = float(err.max()), float(err.mean())
        assert mx <= O_MAX_ABS, f"{label} row {(b, h, qb)}: max-abs {mx:.3g} > {O_MAX_ABS}"
        assert mean <= O_MEAN_ABS, f"{label} row {(b, h, qb)}: mean-abs {mean:.3g} > {O_MEAN_ABS}"
        le = float(np.abs(lse_h[b, h, sl] - lse_ref).max())
        assert le < lse_tol, f"{label} row {(b, h, qb)}: lse error {le:.3g}"
        worst_max, worst_mean = max(worst_max, mx), max(worst_mean, mean)
    ATTN_LOG.append((label, len(rows), worst_max, worst_mean))
    return worst_max, worst_mean
