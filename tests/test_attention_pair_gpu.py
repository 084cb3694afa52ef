"""The CTA-pair attention kernel (d = T = 128; two SMs per tensor-core MMA, the
two query blocks of a stage walking the union of their routed lists with a
per-block mask) on routed lists, forced through the test entry point: the
library sends routed lists to the single-SM two-block kernel and dense walks to
this one. Element by element against the oracle: adjacent blocks with shared
lists (the union path), repeated and out-of-range indices (the concatenation
path, out-of-range flagged and read as block 0), more than 8192 key blocks
(concatenation), odd query-block counts (a cluster with missing blocks)."""
import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo
from tests.parity_utils import attention_rows_vs_oracle, compare_attention, dev, oracle_route_per_head

pytestmark = pytest.mark.gpu


def _pair(vx, q, k, v, idx, status=None):
    B, H, Nq, _ = q.shape
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if status is None else status
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
    o = vx.sparse_attn_fwd_test(q, k, v, idx, 128, st, 2.0, vx.VELOX_TEST_FORCE_PAIR, lse=lse)
    torch.cuda.synchronize()
    return o, lse, int(st.item())


class _ForcedPair:
    """Stands in for the binding in attention_rows_vs_oracle: the same call
    through the test entry point with the pair kernel forced."""

    def __init__(self, vx):
        self.vx = vx

    def sparse_attn_fwd(self, q, k, v, idx, T):
        o, lse, st = _pair(self.vx, q, k, v, idx)
        assert st == 0
        return o, lse


def test_pair_kernel_routed_lists_match_the_oracle():
    from geometry_routed_block_b200 import velox as vx
    heads = (1, 22)
    c = synth.make_case(4, P=8, heads=heads)
    s = c.shape
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    q, k, v = c.q[0], c.k[0], c.v[0]
    want, _ = oracle_route_per_head(q, k, counts, s.alpha, s.topk, s.T)
    rows = [(0, i, qb) for i in range(2) for qb in range(s.m)]
    attention_rows_vs_oracle(_ForcedPair(vx), q, k, v, want, s.T, rows,
                             label=f"CTA-pair kernel, workload 4 P = 8, heads {heads}")
    # the library's default kernel for these lists gives the same result
    o_pair, _, _ = _pair(vx, dev(q), dev(k), dev(v), dev(want))
    o_def, _ = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(want), s.T)
    compare_attention(o_pair, o_def.float().cpu().numpy().astype(np.float64), "pair vs default")


@pytest.mark.parametrize("m,nkb,topk,kind", [(3, 11, 5, "repeats"), (5, 20, 7, "sorted"),
                                             (6, 40, 9, "shuffled"), (2, 8200, 7, "sorted")])
def test_pair_kernel_list_shapes(m, nkb, topk, kind):
    from geometry_routed_block_b200 import velox as vx
    rng = np.random.default_rng(m * 100 + nkb)
    T, d, B, H = 128, 128, 1 if nkb > 1000 else 2, 1 if nkb > 1000 else 3
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    q, kk, vv = f(B, H, m * T, d), f(B, H, nkb * T, d), f(B, H, nkb * T, d)
    rows = []
    for _ in range(B * H * m):
        if kind == "repeats":
            rows.append(rng.integers(0, nkb, topk))
        else:
            r = rng.choice(nkb, topk, replace=False)
            rows.append(np.sort(r) if kind == "sorted" else r)
    idx = np.stack(rows).reshape(B, H, m, topk).astype(np.int32)
    if kind == "repeats":
        idx[0, 0, 0] = [3, 3, 3, 7, 0]
    o, lse, st = _pair(vx, dev(q), dev(kk), dev(vv), dev(idx))
    assert st == 0
    o_ref, lse_ref = vo.sparse_attention(q, kk, vv, idx, T)
    compare_attention(o, o_ref, f"pair kernel, {kind} lists, m = {m}, {nkb} key blocks")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 1e-3


def test_pair_kernel_flags_bad_indices():
    from geometry_routed_block_b200 import velox as vx
    rng = np.random.default_rng(11)
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    q, k, v = f(1, 1, 256, 128), f(1, 1, 1024, 128), f(1, 1, 1024, 128)
    idx = np.array([[[[0, 1, -5], [2, 8, 3]]]], dtype=np.int32)  # -5 and 8 are out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _, st = _pair(vx, dev(q), dev(k), dev(v), dev(idx), status)
    assert st & vx.VELOX_STATUS_BAD_INDEX
    fixed = np.array([[[[0, 1, 0], [2, 0, 3]]]], dtype=np.int32)  # replaced by block 0
    o_ref, _ = vo.sparse_attention(q, k, v, fixed, 128)
    compare_attention(o, o_ref, "pair kernel, bad-index replacement")
