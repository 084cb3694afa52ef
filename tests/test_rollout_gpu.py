"""GPU parity of the chunk-by-chunk rollout state (geometry_routed_block_b200.rollout):
a KV cache with room for more chunks than the current one, the pooled-key cache
appended per finished chunk, slices rebuilt per chunk, and both geometry
schedules, against the oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo
from tests.parity_utils import compare_selection, dev

pytestmark = pytest.mark.gpu

N0, CAP = 8, 11  # chunks 8 and 9 are generated; the KV cache holds 11 chunks


@pytest.fixture(scope="module")
def case():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return synth.make_case(4, P=CAP - 1, heads=(0, 7))  # Nk = 11 chunks, 2 heads


def run(case, schedule):
    from geometry_routed_block_b200.rollout import Rollout
    from geometry_routed_block_b200 import velox as vx
    c, s = case, case.shape
    q, k, v = dev(c.q[0]), dev(c.k[0]), dev(c.v[0])
    cams = dev(np.concatenate([c.past_cams[0], c.cur_cam], 0))  # 11 cameras
    final = dev(np.concatenate([c.past_depth[0], c.cur_depth], 0))
    topk_of = lambda n: synth.topk_for(n, s.m)
    R = Rollout([k], B=1, H=q.shape[1], d=s.d, T=s.T, F=s.F, Hp=s.Hp, Wp=s.Wp, capacity=CAP,
                cams=cams, poses=dev(c.past_poses[0]), intr=dev(c.past_intr[0]), alpha=s.alpha,
                topk_of=topk_of, schedule=schedule)
    R.prefill(N0, final[:N0])
    idx, out = {}, {}
    for n in (N0, N0 + 1):
        R.begin_chunk(n)
        for _ in range(2):  # two denoising steps
            i = R.route(0, q)
            o, _ = R.attend(0, q, v, i)
        idx[n], out[n] = i.clone(), o.clone()
        R.end_chunk(n, final[n])
    torch.cuda.synchronize()
    return R, idx, out, (q, k, v)


def oracle_counts(case, n, slot_depth):
    """Counts of chunk n from depth slots 0..n-1 (`slot_depth` [n,Hp,Wp])."""
    c, s = case, case.shape
    cams = np.concatenate([c.past_cams[0], c.cur_cam], 0)
    cur = vo.depth_multiwarp(slot_depth, cams[:n], cams[n], 0.01)
    sl = vo.slices_build(slot_depth, c.past_poses[0][:n], c.past_intr[0][:n])
    return vo.block_overlap(cur[None], cams[n:n + 1], sl[None], s.F, s.T), cur


@pytest.mark.parametrize("schedule", ["boundary", "pipelined"])
def test_rollout_geometry_routing_attention(case, schedule):
    from geometry_routed_block_b200 import velox as vx
    c, s = case, case.shape
    R, idx, out, (q, k, v) = run(case, schedule)
    final = np.concatenate([c.past_depth[0], c.cur_depth], 0)
    # slices of the finished chunks from their final depth, rebuilt one by one
    want_sl = vo.slices_build(final[:N0 + 1], c.past_poses[0][:N0 + 1], c.past_intr[0][:N0 + 1])
    assert np.array_equal(R.slices[:N0 + 1].cpu().numpy(), want_sl)
    for n in (N0, N0 + 1):
        slots = final[:n].copy()
        if schedule == "pipelined" and n > N0:
            # built during chunk n-1: chunk n-1's slot held its own warped depth
            _, est = oracle_counts(case, n - 1, final[:n - 1])
            slots[n - 1] = est
        counts, _ = oracle_counts(case, n, slots)
        assert np.array_equal(R.counts[n].cpu().numpy(), counts), (schedule, n)
        # routing from the pooled-key cache over the capacity-sized KV cache ==
        # the oracle on a KV cache that ends at chunk n
        kn = c.k[0][:, :, : (n + 1) * s.Nq]
        want, s_mod = vo.route_topk(c.q[0], kn, counts, s.alpha, synth.topk_for(n, s.m), s.T)
        ties = compare_selection(idx[n].cpu().numpy(), want, s_mod, s.m,
                                 label=f"rollout ({schedule} geometry), chunk {n}, cached routing")
        assert ties <= 2
        # attention over the capacity-sized cache == attention over a cache that
        # ends at chunk n (the same kernel walk, bit for bit)
        kc = k[:, :, : (n + 1) * s.Nq].contiguous()
        vc = v[:, :, : (n + 1) * s.Nq].contiguous()
        o_ref, _ = vx.sparse_attn_fwd(q, kc, vc, idx[n], s.T, want_lse=False)
        assert torch.equal(out[n], o_ref)
