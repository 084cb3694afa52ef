"""Pins for the fp64 CPU oracle: each function is checked against something
other than itself -- hand-worked examples (tests/golden/), closed forms, special
cases that reduce to a textbook or library routine, brute force on tiny inputs
and invariants of the method. CPU only."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def read_fixture(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or "|" not in line:
                continue
            key, vals = line.split("|")
            rows[key.strip()] = [float(x) for x in vals.split()]
    return rows


# ----------------------------------------------------------------------------
# input widening
# ----------------------------------------------------------------------------

def test_widen_bf16_bit_patterns():
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0000, 0x4049], dtype=np.uint16)
    assert vo.widen(bits).tolist() == [1.0, -2.0, 0.25, 0.0, 3.140625]


def test_synth_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -3.0 - 2 ** -9], dtype=np.float32)
    got = vo.widen(synth.f32_to_bf16_bits(x))
    assert got.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -3.0]


# ----------------------------------------------------------------------------
# slices
# ----------------------------------------------------------------------------

def test_slices_build_closed_form():
    d = np.array([[[3.0, np.nan, 0.0], [np.inf, 7.5, -1.0]],
                  [[np.nan, np.nan, np.nan], [0.0, -2.0, np.inf]],
                  [[4.25, 4.25, 4.25], [4.25, 4.25, 4.25]]], dtype=np.float32)
    poses = np.arange(36, dtype=np.float32).reshape(3, 12)
    intr = np.arange(100, 112, dtype=np.float32).reshape(3, 4)
    s = vo.slices_build(d, poses, intr)
    assert s.dtype == np.float32 and s.shape == (3, 18)
    assert s[0, 16] == 3.0 and s[0, 17] == 7.5
    assert s[1, 16] == np.inf and s[1, 17] == -np.inf
    assert s[2, 16] == 4.25 and s[2, 17] == 4.25
    assert (s[:, :12] == poses).all() and (s[:, 12:16] == intr).all()


# ----------------------------------------------------------------------------
# overlap counts
# ----------------------------------------------------------------------------

def test_overlap_hand_worked_example():
    g = read_fixture("overlap_worked.txt")
    Hp, Wp, F, T = (int(x) for x in g["Hp Wp F T"])
    depth = np.array(g["cur_depth"], dtype=np.float32).reshape(1, Hp, Wp)
    cur = np.array(g["cur_cam"], dtype=np.float32)[None]
    sl = np.stack([np.array(g[k], dtype=np.float32) for k in ("slice_A", "slice_B", "slice_C")])[None]
    counts = vo.block_overlap(depth, cur, sl, F, T)
    assert counts[0, 0].tolist() == [int(x) for x in g["counts_block0"]]
    assert counts[0, 1].tolist() == [int(x) for x in g["counts_block1"]]


def _cfg2_geometry():
    return synth.geometry_only(2)


def test_overlap_identical_pose_is_full():
    c = _cfg2_geometry()
    s = c.shape
    z = c.cur_depth[0]
    rec = c.cur_cam[0].copy()
    rec[16], rec[17] = z.min() - 1.0, z.max() + 1.0
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, rec[None, None], s.F, s.T)
    assert (counts == s.T).all()


def test_overlap_rotated_pose_identity_in_world():
    # Same camera, but the current pose is a genuine rotation + translation (not
    # symmetric), so a transposed R in either direction breaks the identity.
    intr = synth.intrinsics(16, 24, 70.0)
    pose = synth.pose_looking((0.3, 1.2, -0.7), (0.8, -0.2, 0.55))
    cam = synth.camera_record(pose, intr, 0.5, 20.0)
    depth = np.random.default_rng(0).uniform(1.0, 10.0, (1, 16, 24)).astype(np.float32)
    counts = vo.block_overlap(depth, cam[None], cam[None, None], 1, 64)
    assert (counts == 64).all()
    # shrink the interval so only depths in [2, 5] count
    cam2 = cam.copy()
    cam2[16], cam2[17] = 2.0, 5.0
    counts = vo.block_overlap(depth, cam[None], cam2[None, None], 1, 64)
    want = ((depth[0] >= 2.0) & (depth[0] <= 5.0)).reshape(-1, 64).sum(1)
    assert counts[0, :, 0].tolist() == want.tolist()


def test_overlap_away_is_zero():
    c = _cfg2_geometry()
    s = c.shape
    R = c.cur_cam[0, :9].astype(np.float64).reshape(3, 3)
    t = c.cur_cam[0, 9:12].astype(np.float64)
    C = -R.T @ t
    fwd = R[2]
    pose = synth.pose_looking(C, -fwd)  # yawed 180 degrees, same centre
    rec = synth.camera_record(pose, c.cur_cam[0, 12:16], 0.0, 1e9)
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, rec[None, None], s.F, s.T)
    assert (counts == 0).all()


def test_overlap_invalid_depth_counts_outside():
    c = _cfg2_geometry()
    s = c.shape
    rec = c.cur_cam[0].copy()
    rec[16], rec[17] = 0.0, 1e9
    for bad in (np.nan, 0.0, -3.0, np.inf):
        d = np.full_like(c.cur_depth, bad)
        counts = vo.block_overlap(d, c.cur_cam, rec[None, None], s.F, s.T)
        assert (counts == 0).all()


def _frustum_planes_count(depth, cur_rec, sl_rec, T):
    """Second formulation: world points as camera centre + z * world ray, and
    membership by the six half-spaces of the slice's frustum built from its
    corner rays (plus the depth interval along the viewing axis)."""
    Hp, Wp = depth.shape
    R = cur_rec[:9].astype(np.float64).reshape(3, 3)
    t = cur_rec[9:12].astype(np.float64)
    fx, fy, cx, cy = cur_rec[12:16].astype(np.float64)
    C = -R.T @ t
    rr, cc = np.meshgrid(np.arange(Hp) + 0.5, np.arange(Wp) + 0.5, indexing="ij")
    rays = np.stack([(cc - cx) / fx, (rr - cy) / fy, np.ones_like(cc)], -1).reshape(-1, 3)
    z = depth.reshape(-1).astype(np.float64)
    pts = C[None] + z[:, None] * (rays @ R)
    Rj = sl_rec[:9].astype(np.float64).reshape(3, 3)
    tj = sl_rec[9:12].astype(np.float64)
    fxj, fyj, cxj, cyj, near, far = sl_rec[12:18].astype(np.float64)
    Cj = -Rj.T @ tj
    corners = [(0.0, 0.0), (Wp, 0.0), (Wp, Hp), (0.0, Hp)]
    dirs = [Rj.T @ np.array([(u - cxj) / fxj, (v - cyj) / fyj, 1.0]) for u, v in corners]
    axis = Rj[2]
    rel = pts - Cj[None]
    depth_j = rel @ axis
    ok = (depth_j >= near) & (depth_j <= far) & (depth_j > 0)
    margin = np.minimum(np.abs(depth_j - near), np.abs(depth_j - far))
    for i in range(4):
        n = np.cross(dirs[i], dirs[(i + 1) % 4])
        if n @ axis < 0:
            n = -n
        dist = rel @ n / np.linalg.norm(n)
        inclusive = i in (0, 3)  # top edge (v=0) and left edge (u=0) are inclusive
        ok &= (dist >= 0) if inclusive else (dist > 0)
        margin = np.minimum(margin, np.abs(dist))
    ok &= np.isfinite(z) & (z > 0)
    near_boundary = margin < 1e-9 * np.maximum(1.0, np.abs(depth_j))
    return ok.reshape(-1, T).sum(1), int(near_boundary.sum())


def test_overlap_matches_frustum_halfspaces_workload1():
    c = synth.make_case(1)
    s = c.shape
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    assert counts.sum() > 0 and (counts < s.T).any()
    for j in range(s.P):
        want, amb = _frustum_planes_count(c.cur_depth[0], c.cur_cam[0], c.past_cams[0, j], s.T)
        assert amb == 0
        assert counts[0, :, j].tolist() == want.tolist()


def test_overlap_matches_frustum_halfspaces_walk():
    c = _cfg2_geometry()
    s = c.shape
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    assert counts.sum() > 0
    tot_amb = 0
    for j in range(s.P):
        want, amb = _frustum_planes_count(c.cur_depth[0], c.cur_cam[0], sl[j], s.T)
        tot_amb += amb
        if amb == 0:
            # the F frames of a chunk share one depth map, so per-frame counts repeat
            assert counts[0, :, j].tolist() == np.tile(want, s.F).tolist()
    assert tot_amb <= 4 * s.T


# ----------------------------------------------------------------------------
# pooling, scores, modulation, selection
# ----------------------------------------------------------------------------

def test_pool_closed_forms():
    x = np.full((1, 1, 256, 4), 0.75, dtype=np.float32)
    assert (vo.pool_blocks(x, 64) == 0.75).all()
    ramp = np.arange(256, dtype=np.float32)[None, None, :, None] * np.ones(4, np.float32)
    p = vo.pool_blocks(ramp, 64)[0, 0, :, 0]
    assert p.tolist() == [31.5, 95.5, 159.5, 223.5]


def test_scores_hand_example():
    # d = 4, T = 2, Nq = 2 (m = 1), one past chunk of 1 block + current chunk.
    q = np.zeros((1, 1, 2, 4), np.float32)
    q[..., 0] = 1.0
    q[..., 1] = 3.0  # qbar = (1, 3, 0, 0)
    k = np.zeros((1, 1, 4, 4), np.float32)
    k[0, 0, 0] = [2.0, 1.0, 5.0, 0.0]
    k[0, 0, 1] = [2.0, -1.0, -5.0, 8.0]  # kbar = (2, 0, 0, 4) -> s = 2 / sqrt(4) = 1
    k[0, 0, 2:] = 100.0  # current chunk: never scored
    s = vo.block_scores(q, k, 2)
    assert s.shape == (1, 1, 1, 1) and s[0, 0, 0, 0] == 1.0


def test_modulation_rules():
    rng = np.random.default_rng(5)
    B, H, m, P = 1, 3, 4, 5
    s = rng.standard_normal((B, H, m, P * m))
    counts = rng.integers(0, 65, size=(B, m, P)).astype(np.int32)
    counts[0, 2] = 0  # query block 2 is uncovered
    out = vo.modulate(s, counts, 2.0, 64)
    assert np.array_equal(out[0, :, 2], s[0, :, 2])  # exactly no bias
    for qb in (0, 1, 3):
        for kb in range(P * m):
            assert out[0, 1, qb, kb] == s[0, 1, qb, kb] + 2.0 * counts[0, qb, kb // m] / 64
    assert np.array_equal(vo.modulate(s, counts, 0.0, 64), s)
    assert np.array_equal(vo.modulate(s, None, 2.0, 64), s)


def _brute_select(row, k_past, n_past):
    best, best_key = None, None
    for sub in itertools.combinations(range(n_past), k_past):
        tot = math.fsum(row[list(sub)])
        key = (-tot, sub)
        if best_key is None or key < best_key:
            best_key, best = key, sub
    return list(best)


def test_selection_matches_bruteforce_workload1():
    c = synth.make_case(1)
    s = c.shape
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    s_mod = vo.modulate(vo.block_scores(c.q[0], c.k[0], s.T), counts, s.alpha, s.T)
    n_past = s.P * s.m
    for k_past in range(0, n_past + 1):
        idx = vo.select_topk(s_mod, s.m + k_past, s.m)
        for h in range(s.H):
            for qb in range(s.m):
                want = _brute_select(s_mod[0, h, qb], k_past, n_past) + list(range(n_past, n_past + s.m))
                assert idx[0, h, qb].tolist() == want


def test_selection_tie_break_prefers_smaller_index():
    row = np.array([0.5, 2.0, 1.0, 2.0, 1.0, 1.0, -3.0, 2.0])
    s_mod = row[None, None, None, :]
    idx = vo.select_topk(s_mod, 2 + 4, 2)  # m = 2 current blocks, 4 past
    assert idx[0, 0, 0].tolist() == [1, 2, 3, 7, 8, 9]
    for k_past in range(0, 9):
        got = vo.select_topk(s_mod, 2 + k_past, 2)[0, 0, 0, :k_past].tolist()
        assert got == _brute_select(row, k_past, 8)


def test_selection_rejects_bad_topk():
    with pytest.raises(ValueError):
        vo.select_topk(np.zeros((1, 1, 2, 6)), 1, 2)
    with pytest.raises(ValueError):
        vo.select_topk(np.zeros((1, 1, 2, 6)), 9, 2)


def test_alpha_zero_equals_native_routing():
    c = synth.make_case(1)
    s = c.shape
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    i0, s0 = vo.route_topk(c.q[0], c.k[0], counts, 0.0, s.topk, s.T)
    i1, s1 = vo.route_topk(c.q[0], c.k[0], None, 0.0, s.topk, s.T)
    assert np.array_equal(i0, i1) and np.array_equal(s0, s1)


def test_routing_permutation_invariance():
    c = synth.make_case(1)
    s = c.shape
    perm = np.array([2, 0, 3, 1])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    idx, _ = vo.route_topk(c.q[0], c.k[0], counts, s.alpha, s.topk, s.T)
    kk = c.k[0].reshape(s.B, s.H, s.P + 1, s.Nq, s.d).copy()
    kk[:, :, : s.P] = kk[:, :, perm]
    counts_p = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams[:, perm], s.F, s.T)
    assert np.array_equal(counts_p, counts[:, :, perm])
    idx_p, _ = vo.route_topk(c.q[0], kk.reshape(c.k[0].shape), counts_p, s.alpha, s.topk, s.T)
    inv = np.argsort(perm)  # new chunk position of old chunk c
    n_past = s.P * s.m

    def remap(kb):
        if kb >= n_past:
            return kb
        return inv[kb // s.m] * s.m + kb % s.m

    for h in range(s.H):
        for qb in range(s.m):
            want = sorted(remap(kb) for kb in idx[0, h, qb])
            assert idx_p[0, h, qb].tolist() == want


def test_modulation_changes_selection_workload1():
    c = synth.make_case(1)
    s = c.shape
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    i0, _ = vo.route_topk(c.q[0], c.k[0], counts, 0.0, s.topk, s.T)
    i2, _ = vo.route_topk(c.q[0], c.k[0], counts, 50.0, s.topk, s.T)
    assert not np.array_equal(i0, i2)


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def test_dense_attention_equals_sdpa():
    c = synth.make_case(1)
    s = c.shape
    O, lse = vo.sparse_attention(c.q[0], c.k[0], c.v[0], None, s.T)
    q = torch.from_numpy(c.q[0].astype(np.float64))
    k = torch.from_numpy(c.k[0].astype(np.float64))
    v = torch.from_numpy(c.v[0].astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    assert np.abs(O - ref.numpy()).max() < 1e-12
    ref_lse = torch.logsumexp((q @ k.transpose(-1, -2)) / math.sqrt(s.d), dim=-1)
    assert np.abs(lse - ref_lse.numpy()).max() < 1e-12


def test_dense_attention_equals_sdpa_bf16_inputs():
    rng = np.random.default_rng(3)
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 2, 256, 128), dtype=np.float32))
    k = synth.f32_to_bf16_bits(rng.standard_normal((1, 2, 768, 128), dtype=np.float32))
    v = synth.f32_to_bf16_bits(rng.standard_normal((1, 2, 768, 128), dtype=np.float32))
    O, _ = vo.sparse_attention(q, k, v, None, 128)
    tq, tk, tv = (torch.from_numpy(synth.bf16_bits_to_f64(x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    assert np.abs(O - ref.numpy()).max() < 1e-12


def test_sparse_attention_equals_masked_dense():
    c = synth.make_case(1)
    s = c.shape
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, c.past_cams, s.F, s.T)
    idx, _ = vo.route_topk(c.q[0], c.k[0], counts, s.alpha, s.topk, s.T)
    O, lse = vo.sparse_attention(c.q[0], c.k[0], c.v[0], idx, s.T)
    q = torch.from_numpy(c.q[0].astype(np.float64))
    k = torch.from_numpy(c.k[0].astype(np.float64))
    v = torch.from_numpy(c.v[0].astype(np.float64))
    mask = torch.full((s.B, s.H, s.Nq, s.Nk), float("-inf"), dtype=torch.float64)
    for b in range(s.B):
        for h in range(s.H):
            for qb in range(s.m):
                for kb in idx[b, h, qb]:
                    mask[b, h, qb * s.T:(qb + 1) * s.T, kb * s.T:(kb + 1) * s.T] = 0.0
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    assert np.abs(O - ref.numpy()).max() < 1e-12
    # convexity: every output lies within the selected values' range
    for h in range(s.H):
        for qb in range(s.m):
            keys = (idx[0, h, qb][:, None] * s.T + np.arange(s.T)).reshape(-1)
            vs = c.v[0][0, h, keys].astype(np.float64)
            o = O[0, h, qb * s.T:(qb + 1) * s.T]
            assert (o <= vs.max(0) + 1e-12).all() and (o >= vs.min(0) - 1e-12).all()
    rows = vo.sparse_attention(c.q[0], c.k[0], c.v[0], idx, s.T, rows=[(0, 1, 2)])
    o, l = rows[(0, 1, 2)]
    assert np.array_equal(o, O[0, 1, 2 * s.T:3 * s.T]) and np.array_equal(l, lse[0, 1, 2 * s.T:3 * s.T])


def test_attention_all_blocks_listed_equals_dense():
    c = synth.make_case(1)
    s = c.shape
    idx = np.broadcast_to(np.arange(s.nKB, dtype=np.int32), (s.B, s.H, s.m, s.nKB))
    O1, l1 = vo.sparse_attention(c.q[0], c.k[0], c.v[0], idx, s.T)
    O0, l0 = vo.sparse_attention(c.q[0], c.k[0], c.v[0], None, s.T)
    assert np.abs(O1 - O0).max() < 1e-13 and np.abs(l1 - l0).max() < 1e-13


# ----------------------------------------------------------------------------
# multiwarp
# ----------------------------------------------------------------------------

def test_multiwarp_hand_worked_example():
    g = read_fixture("multiwarp_worked.txt")
    Hp, Wp, rel = int(g["Hp Wp rel_tol"][0]), int(g["Hp Wp rel_tol"][1]), g["Hp Wp rel_tol"][2]
    cam = np.array(g["cam"], dtype=np.float32)
    d = np.stack([np.array(g["depth_chunk0"], np.float32), np.array(g["depth_chunk1"], np.float32)])
    d = d.reshape(2, Hp, Wp)
    out = vo.depth_multiwarp(d, np.stack([cam, cam]), cam, rel)
    want = np.array(g["expected"], np.float32).reshape(Hp, Wp)
    assert np.array_equal(out, want)
    out1 = vo.depth_multiwarp(d[1:], cam[None], cam, rel)
    want1 = np.array(g["expected_chunk1_only"], np.float32).reshape(Hp, Wp)
    assert np.array_equal(out1, want1, equal_nan=True)


def test_multiwarp_single_chunk_same_pose_reproduces_depth():
    c = _cfg2_geometry()
    d = c.past_depth[0, -1:]
    cam = synth.camera_record(c.past_poses[0, -1], c.past_intr[0, -1])
    out = vo.depth_multiwarp(d, cam[None], cam)
    # float32 R is orthonormal only to ~1e-7, so R R^T differs from I by a few ulp
    assert np.isfinite(out).all()
    assert np.abs(out - d[0]).max() <= 3e-7 * d[0].max()
    # an axis-aligned rotation is exactly orthonormal: the depth comes back bit for bit
    cam_x = cam.copy()
    cam_x[:9] = [0, 0, -1, 0, 1, 0, 1, 0, 0]
    out = vo.depth_multiwarp(d, cam_x[None], cam_x)
    assert np.array_equal(out, d[0])


def test_multiwarp_recency_and_tolerance():
    c = _cfg2_geometry()
    cam = synth.camera_record(c.past_poses[0, -1], c.past_intr[0, -1])
    cam[:9] = [0, 0, -1, 0, 1, 0, 1, 0, 0]  # exactly orthonormal: depths return bit for bit
    base = c.past_depth[0, -1]
    near_later = (base * np.float32(1.005)).astype(np.float32)
    far_later = (base * np.float32(1.02)).astype(np.float32)
    out = vo.depth_multiwarp(np.stack([base, near_later]), np.stack([cam, cam]), cam)
    assert np.array_equal(out, near_later)  # later chunk within 1% wins
    out = vo.depth_multiwarp(np.stack([base, far_later]), np.stack([cam, cam]), cam)
    assert np.array_equal(out, base)  # later chunk 2% behind loses
    out = vo.depth_multiwarp(np.stack([far_later, base]), np.stack([cam, cam]), cam)
    assert np.array_equal(out, base)  # nearer AND later


def test_multiwarp_bruteforce_candidates():
    """Per target pixel, sort every candidate by the rule written as a key:
    (is a winner, chunk, -depth) maximal -> same depth as the oracle."""
    c = synth.geometry_only(3, P=6)
    s = c.shape
    cams = np.stack([synth.camera_record(c.past_poses[0, j], c.past_intr[0, j]) for j in range(6)])
    out = vo.depth_multiwarp(c.past_depth[0], cams, c.cur_cam[0])
    tgt, ch, zs = vo.multiwarp_candidates(c.past_depth[0], cams, c.cur_cam[0])
    want = np.full(s.Hp * s.Wp, np.nan, np.float32)
    fac = 1.0 + float(np.float32(0.01))
    for p in np.unique(tgt):
        sel = tgt == p
        zz, jj = zs[sel], ch[sel]
        win = zz <= zz.min() * fac
        keys = sorted(zip(win, jj, -zz))
        want[p] = np.float32(-keys[-1][2])
    assert np.array_equal(out.reshape(-1), want, equal_nan=True)
    assert np.isfinite(out).mean() > 0.3


def test_multiwarp_holes_are_nan():
    c = _cfg2_geometry()
    cam = synth.camera_record(c.past_poses[0, -1], c.past_intr[0, -1])
    d = np.full((1,) + c.past_depth.shape[2:], np.nan, np.float32)
    out = vo.depth_multiwarp(d, cam[None], cam)
    assert np.isnan(out).all()
