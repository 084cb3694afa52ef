"""GPU parity: the CUDA path (through the C ABI binding) against the fp64 CPU
oracle on the same seeded inputs. Needs a B200 and the built libvelox.so."""
import math

import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo
from tests.parity_utils import (TIE_LOG, attention_rows_vs_oracle, compare_attention,
                                compare_selection, dev, host_bits, oracle_route_per_head,
                                tie_bound)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vx():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from geometry_routed_block_b200 import velox
    return velox


def cams_of(case):
    return dev(case.past_cams), dev(case.cur_cam)


# ---------------------------------------------------------------- workload 1 (tiny, fp32)

@pytest.fixture(scope="module")
def tiny():
    return synth.make_case(1)


def test_tiny_overlap_counts_exact(vx, tiny):
    s = tiny.shape
    past, cur = cams_of(tiny)
    counts = vx.block_overlap(dev(tiny.cur_depth), cur, past, s.F, s.T)
    want = vo.block_overlap(tiny.cur_depth, tiny.cur_cam, tiny.past_cams, s.F, s.T)
    assert np.array_equal(counts.cpu().numpy(), want)
    assert want.sum() > 0


def test_tiny_routing_matches_oracle(vx, tiny):
    s = tiny.shape
    counts = vo.block_overlap(tiny.cur_depth, tiny.cur_cam, tiny.past_cams, s.F, s.T)
    q, k = dev(tiny.q[0]), dev(tiny.k[0])
    for alpha, topk in ((2.0, 6), (0.0, 6), (2.0, 4), (2.0, 20), (50.0, 11)):
        idx = vx.route_topk(q, k, dev(counts), alpha, topk, s.T)
        want, s_mod = vo.route_topk(tiny.q[0], tiny.k[0], counts, alpha, topk, s.T)
        compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                          label=f"workload 1, alpha {alpha:g}, k {topk}")
    a0 = vx.route_topk(q, k, dev(counts), 0.0, 6, s.T)
    nat = vx.route_topk(q, k, None, 2.0, 6, s.T)
    assert torch.equal(a0, nat)  # alpha = 0 is the native routing, bit for bit


def test_tiny_cast_matches_host_rounding(vx, tiny):
    got = host_bits(vx.cast_bf16(dev(tiny.q[0])))
    assert np.array_equal(got, synth.f32_to_bf16_bits(tiny.q[0]))


def test_tiny_attention_sparse_and_dense(vx, tiny):
    s = tiny.shape
    counts = vo.block_overlap(tiny.cur_depth, tiny.cur_cam, tiny.past_cams, s.F, s.T)
    idx, _ = vo.route_topk(tiny.q[0], tiny.k[0], counts, s.alpha, s.topk, s.T)
    qb, kb, vb = (synth.f32_to_bf16_bits(x[0]) for x in (tiny.q, tiny.k, tiny.v))
    q, k, v = (vx.cast_bf16(dev(x[0])) for x in (tiny.q, tiny.k, tiny.v))
    o, lse = vx.sparse_attn_fwd(q, k, v, dev(idx), s.T)
    o_ref, lse_ref = vo.sparse_attention(qb, kb, vb, idx, s.T)
    compare_attention(o, o_ref, "tiny sparse")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 1e-3
    o, lse = vx.sparse_attn_fwd(q, k, v, None, s.T)
    o_ref, lse_ref = vo.sparse_attention(qb, kb, vb, None, s.T)
    compare_attention(o, o_ref, "tiny dense")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 1e-3


# ---------------------------------------------------------------- workload 2 (dense parity)

@pytest.fixture(scope="module")
def walk():
    return synth.make_case(2)


def test_walk_slices_and_counts_exact(vx, walk):
    s = walk.shape
    sl = vx.slices_build(dev(walk.past_depth[0]), dev(walk.past_poses[0]), dev(walk.past_intr[0]))
    want_sl = vo.slices_build(walk.past_depth[0], walk.past_poses[0], walk.past_intr[0])
    assert np.array_equal(sl.cpu().numpy(), want_sl)
    counts = vx.block_overlap(dev(walk.cur_depth), dev(walk.cur_cam), sl[None], s.F, s.T)
    want = vo.block_overlap(walk.cur_depth, walk.cur_cam, want_sl[None], s.F, s.T)
    assert np.array_equal(counts.cpu().numpy(), want)
    assert want.sum() > 0 and (want < s.T).any()


def test_walk_dense_attention_rows(vx, walk):
    s = walk.shape
    q, k, v = dev(walk.q[0]), dev(walk.k[0]), dev(walk.v[0])
    rows = [(0, h, qb) for h in (0, 5, 11) for qb in (0, 17, 35)]
    ref = vo.sparse_attention(walk.q[0], walk.k[0], walk.v[0], None, s.T, rows=rows)
    o, lse = vx.sparse_attn_fwd(q, k, v, None, s.T)
    # top-k = every block, listed explicitly, is the same computation (on the
    # two-block kernel; the dense walk runs on the CTA-pair kernel, which takes
    # a quarter of its exponentials on the FMA pipe, so the two agree to a few
    # bf16 units in the last place rather than bit for bit)
    all_idx = torch.arange(s.nKB, dtype=torch.int32, device="cuda").expand(s.B, s.H, s.m, s.nKB)
    o2, _ = vx.sparse_attn_fwd(q, k, v, all_idx.contiguous(), s.T)
    for (b, h, qb), (o_ref, lse_ref) in ref.items():
        sl = slice(qb * s.T, (qb + 1) * s.T)
        compare_attention(o[b, h, sl], o_ref, f"dense row {(b, h, qb)}")
        compare_attention(o2[b, h, sl], o_ref, f"all-listed row {(b, h, qb)}")
        assert np.abs(lse[b, h, sl].cpu().numpy() - lse_ref).max() < 1e-3
    assert float((o.float() - o2.float()).abs().max()) <= 4e-3


def test_walk_routing_alpha0_and_geometry(vx, walk):
    s = walk.shape
    sl = vo.slices_build(walk.past_depth[0], walk.past_poses[0], walk.past_intr[0])
    counts = vo.block_overlap(walk.cur_depth, walk.cur_cam, sl[None], s.F, s.T)
    q, k = dev(walk.q[0]), dev(walk.k[0])
    topk = 65
    total_ties = 0
    for alpha, cnt in ((0.0, counts), (2.0, counts), (2.0, None)):
        idx = vx.route_topk(q, k, None if cnt is None else dev(cnt), alpha, topk, s.T)
        want, s_mod = vo.route_topk(walk.q[0], walk.k[0], cnt, alpha, topk, s.T)
        geo = "no geometry" if cnt is None else f"alpha {alpha:g}"
        total_ties += compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                                        label=f"workload 2, {geo}, k {topk}, all 12 heads")
    assert total_ties <= tie_bound(3 * s.H * s.m)


def test_walk_routed_attention(vx, walk):
    s = walk.shape
    sl = vo.slices_build(walk.past_depth[0], walk.past_poses[0], walk.past_intr[0])
    counts = vo.block_overlap(walk.cur_depth, walk.cur_cam, sl[None], s.F, s.T)
    idx, _ = vo.route_topk(walk.q[0], walk.k[0], counts, s.alpha, 65, s.T)
    rows = [(0, h, qb) for h in (1, 7) for qb in (0, 9, 35)]
    ref = vo.sparse_attention(walk.q[0], walk.k[0], walk.v[0], idx, s.T, rows=rows)
    o, _ = vx.sparse_attn_fwd(dev(walk.q[0]), dev(walk.k[0]), dev(walk.v[0]), dev(idx), s.T)
    for (b, h, qb), (o_ref, _) in ref.items():
        compare_attention(o[b, h, qb * s.T:(qb + 1) * s.T], o_ref, f"routed row {(b, h, qb)}")


# ---------------------------------------------------------------- kernel variants and edges

def _random_qkv(rng, B, H, Nq, Nk, d):
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    return f(B, H, Nq, d), f(B, H, Nk, d), f(B, H, Nk, d)


@pytest.mark.parametrize("T,d", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_attention_variants_with_duplicates_and_ragged_tiles(vx, T, d):
    rng = np.random.default_rng(T * 1000 + d)
    B, H = 2, 3
    Nq = 3 * T          # three query blocks: for T=64 the last 128-row tile is half outside
    Nk = 11 * T
    q, k, v = _random_qkv(rng, B, H, Nq, Nk, d)
    m, nkb = Nq // T, Nk // T
    topk = 5
    idx = rng.integers(0, nkb, size=(B, H, m, topk)).astype(np.int32)
    idx[0, 0, 0] = [3, 3, 3, 7, 0]   # a block listed several times counts several times
    o, lse = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(idx), T)
    o_ref, lse_ref = vo.sparse_attention(q, k, v, idx, T)
    compare_attention(o, o_ref, f"T={T} d={d}")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 1e-3
    o, _ = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), None, T)
    o_ref, _ = vo.sparse_attention(q, k, v, None, T)
    compare_attention(o, o_ref, f"dense T={T} d={d}")


def test_attention_large_logits_rescale(vx):
    # scores that grow along the walk force the running max (and O) to be rescaled
    rng = np.random.default_rng(7)
    T, d, B, H = 128, 128, 1, 2
    Nq, Nk = 256, 2048
    qf = rng.standard_normal((B, H, Nq, d), dtype=np.float32)
    kf = rng.standard_normal((B, H, Nk, d), dtype=np.float32)
    ramp = np.linspace(0.2, 6.0, Nk, dtype=np.float32)[None, None, :, None]
    kf = kf * ramp + ramp * qf.mean(axis=2, keepdims=True)
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, H, Nk, d), dtype=np.float32))
    o, lse = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), None, T)
    o_ref, lse_ref = vo.sparse_attention(q, k, v, None, T)
    compare_attention(o, o_ref, "rescale")
    assert np.abs(lse.cpu().numpy() - lse_ref).max() < 2e-3


def test_route_topk_extremes(vx, walk):
    s = walk.shape
    q, k = dev(walk.q[0]), dev(walk.k[0])
    only_cur = vx.route_topk(q, k, None, 0.0, s.m, s.T).cpu().numpy()
    assert (only_cur == np.arange(s.nKB - s.m, s.nKB)).all()
    everything = vx.route_topk(q, k, None, 0.0, s.nKB, s.T).cpu().numpy()
    assert (everything == np.arange(s.nKB)).all()


def test_bad_indices_are_flagged_not_faulting(vx):
    rng = np.random.default_rng(11)
    T, d = 128, 128
    q, k, v = _random_qkv(rng, 1, 1, 256, 1024, d)
    idx = np.array([[[[0, 1, -5], [2, 8, 3]]]], dtype=np.int32)  # -5 and 8 are out of range
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(idx), T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & vx.VELOX_STATUS_BAD_INDEX
    assert torch.isfinite(o.float()).all()
    fixed = np.array([[[[0, 1, 0], [2, 0, 3]]]], dtype=np.int32)  # replaced by block 0
    o_ref, _ = vo.sparse_attention(q, k, v, fixed, T)
    compare_attention(o, o_ref, "bad-index replacement")
    status.zero_()
    vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(fixed), T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


# ---------------------------------------------------------------- multiwarp

def test_multiwarp_hand_example(vx):
    from tests.test_oracle_pins import read_fixture
    g = read_fixture("multiwarp_worked.txt")
    Hp, Wp, rel = int(g["Hp Wp rel_tol"][0]), int(g["Hp Wp rel_tol"][1]), g["Hp Wp rel_tol"][2]
    cam = np.array(g["cam"], dtype=np.float32)
    d = np.stack([np.array(g["depth_chunk0"], np.float32),
                  np.array(g["depth_chunk1"], np.float32)]).reshape(2, Hp, Wp)
    out = vx.depth_multiwarp(dev(d), dev(np.stack([cam, cam])), dev(cam), rel)
    assert np.array_equal(out.cpu().numpy(), np.array(g["expected"], np.float32).reshape(Hp, Wp))


def test_multiwarp_pipeline_geometry_exact(vx):
    c = synth.geometry_only(5)
    s = c.shape
    cams = np.stack([synth.camera_record(c.past_poses[0, j], c.past_intr[0, j]) for j in range(s.P)])
    got = vx.depth_multiwarp(dev(c.past_depth[0]), dev(cams), dev(c.cur_cam[0]), 0.01).cpu().numpy()
    want = vo.depth_multiwarp(c.past_depth[0], cams, c.cur_cam[0], 0.01)
    assert np.array_equal(got, want, equal_nan=True)
    assert np.isfinite(want).mean() > 0.5
    # the warped depth then feeds the overlap counts
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vx.block_overlap(dev(want[None]), dev(c.cur_cam), dev(sl[None]), s.F, s.T)
    assert np.array_equal(counts.cpu().numpy(), vo.block_overlap(want[None], c.cur_cam, sl[None], s.F, s.T))


# ---------------------------------------------------------------- chunk-48 headline, full size

@pytest.fixture(scope="module")
def headline():
    return synth.make_case(3)


def test_headline_geometry_exact(vx, headline):
    c = headline
    s = c.shape
    sl = vx.slices_build(dev(c.past_depth[0]), dev(c.past_poses[0]), dev(c.past_intr[0]))
    want_sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    assert np.array_equal(sl.cpu().numpy(), want_sl)
    counts = vx.block_overlap(dev(c.cur_depth), dev(c.cur_cam), sl[None], s.F, s.T)
    assert np.array_equal(counts.cpu().numpy(),
                          vo.block_overlap(c.cur_depth, c.cur_cam, want_sl[None], s.F, s.T))


def test_headline_routing_all_heads(vx, headline):
    """Workload 3 at full size (Nk = 225,792, 1,764 key blocks, k = 353): the
    selection of every one of the 24 heads x 36 query blocks against the oracle."""
    c = headline
    s = c.shape
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    idx = vx.route_topk(dev(c.q[0]), dev(c.k[0]), dev(counts), s.alpha, s.topk, s.T)
    want, s_mod = oracle_route_per_head(c.q[0], c.k[0], counts, s.alpha, s.topk, s.T)
    got = idx.cpu().numpy()
    assert got.shape == want.shape == (1, s.H, s.m, s.topk)
    ties = compare_selection(got, want, s_mod, s.m, label="workload 3 (chunk 48), all 24 heads")
    assert ties <= tie_bound(s.H * s.m)


def test_headline_attention_four_heads_every_query_block(vx, headline):
    """Workload 3 at full size: attention of 4 heads x all 36 query blocks on
    the oracle's own selection (353 key blocks per query block), element by
    element against the oracle."""
    c = headline
    s = c.shape
    heads = [0, 7, 13, 23]
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    q, k, v = (np.ascontiguousarray(x[0][:, heads]) for x in (c.q, c.k, c.v))
    want, _ = oracle_route_per_head(q, k, counts, s.alpha, s.topk, s.T)
    rows = [(0, i, qb) for i in range(len(heads)) for qb in range(s.m)]
    attention_rows_vs_oracle(vx, q, k, v, want, s.T, rows,
                             label=f"workload 3 (chunk 48), heads {heads}, every query block")


@pytest.mark.parametrize("P", [8, 16, 24, 32, 96])
def test_rollout_sweep_geometry_routing_attention(vx, P):
    """Workload 4 at P past chunks (k = 20 % of the key blocks): slices and
    counts bit-exact, the selection of two heads against the oracle, and
    attention rows of both heads on the oracle's selection."""
    heads = (0, 11) if P == 96 else (1, 22)
    c = synth.make_case(4, P=P, heads=heads)
    s = c.shape
    sl = vx.slices_build(dev(c.past_depth[0]), dev(c.past_poses[0]), dev(c.past_intr[0]))
    want_sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    assert np.array_equal(sl.cpu().numpy(), want_sl)
    counts = vx.block_overlap(dev(c.cur_depth), dev(c.cur_cam), sl[None], s.F, s.T)
    want_counts = vo.block_overlap(c.cur_depth, c.cur_cam, want_sl[None], s.F, s.T)
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    q, k, v = c.q[0], c.k[0], c.v[0]
    idx = vx.route_topk(dev(q), dev(k), counts, s.alpha, s.topk, s.T)
    want, s_mod = oracle_route_per_head(q, k, want_counts, s.alpha, s.topk, s.T)
    ties = compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                             label=f"workload 4, P = {P} (k {s.topk} of {s.nKB}), heads {heads}")
    assert ties <= tie_bound(2 * s.m)
    rows = [(0, i, qb) for i in range(2) for qb in (0, 5, 12, 17, 23, 30, 35)]
    attention_rows_vs_oracle(vx, q, k, v, want, s.T, rows,
                             label=f"workload 4, P = {P}, heads {heads}")


def test_rollout_p224_largest_size_geometry_routing_attention(vx):
    """224 past chunks: 8,100 key blocks (the router's limit is 8,192), 8,064
    past candidates per row (the radix selection path), 1,620 kept blocks."""
    c = synth.make_case(4, P=224, heads=(5,))
    s = c.shape
    assert s.nKB == 8100 and s.topk == 1620
    sl = vx.slices_build(dev(c.past_depth[0]), dev(c.past_poses[0]), dev(c.past_intr[0]))
    want_sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    assert np.array_equal(sl.cpu().numpy(), want_sl)
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, want_sl[None], s.F, s.T)
    got_counts = vx.block_overlap(dev(c.cur_depth), dev(c.cur_cam), sl[None], s.F, s.T)
    assert np.array_equal(got_counts.cpu().numpy(), counts)
    q, k, v = dev(c.q[0]), dev(c.k[0]), dev(c.v[0])
    idx = vx.route_topk(q, k, got_counts, s.alpha, s.topk, s.T)
    want, s_mod = vo.route_topk(c.q[0], c.k[0], counts, s.alpha, s.topk, s.T)
    ties = compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                             label="workload 4, P = 224 (8,064 candidates per row), head 5")
    assert ties <= tie_bound(s.m)
    o, lse = vx.sparse_attn_fwd(q, k, v, dev(want), s.T)
    ref = vo.sparse_attention(c.q[0], c.k[0], c.v[0], want, s.T, rows=[(0, 0, 0), (0, 0, 35)])
    for (b, h, qb), (o_ref, lse_ref) in ref.items():
        sl_ = slice(qb * s.T, (qb + 1) * s.T)
        compare_attention(o[b, h, sl_], o_ref, f"P=224 row {(b, h, qb)}")
        assert np.abs(lse[b, h, sl_].cpu().numpy() - lse_ref).max() < 1e-3


@pytest.mark.parametrize("n_past", [255, 256, 257, 512, 513, 1024, 1025, 2048, 2049, 4096, 4097])
def test_selection_sizes_cover_every_kernel_variant(vx, n_past):
    """One query block (T = d = 64, two heads, fp32 routing) against n_past past
    blocks of one block per chunk: every selection variant (one CTA per row with
    1 to 16 keys per thread, the radix selection beyond 4096), the modulation,
    and k_past from 1 to n_past - 1."""
    rng = np.random.default_rng(n_past)
    T, d, B, H, m = 64, 64, 1, 2, 1
    q = rng.standard_normal((B, H, m * T, d), dtype=np.float32)
    k = rng.standard_normal((B, H, (n_past + m) * T, d), dtype=np.float32)
    counts = rng.integers(0, T + 1, size=(B, m, n_past)).astype(np.int32)
    counts[..., rng.random(n_past) < 0.3] = 0
    ties = rows = 0
    for k_past in (1, n_past // 3, n_past - 1):
        got = vx.route_topk(dev(q), dev(k), dev(counts), 2.0, k_past + m, T).cpu().numpy()
        want, s_mod = vo.route_topk(q, k, counts, 2.0, k_past + m, T)
        t = compare_selection(got, want, s_mod, m)
        assert t <= 1, (n_past, k_past)
        ties, rows = ties + t, rows + B * H * m
    TIE_LOG.append((f"selection kernel variant, {n_past} candidates, k_past 1 / n/3 / n-1",
                    ties, rows))


def test_overlap_stress_grid_exact(vx):
    """A 256 x 384 grid (768 query blocks of 128 one-frame tokens) against 96
    slices: counts bit-exact against the oracle for both scenes."""
    g = synth.stress_geometry(2, 96, 256, 384, seed=77)
    B, P = 2, 96
    sl = vo.slices_build(g["past_depth"].reshape(B * P, 32, 48), g["past_poses"].reshape(B * P, 12),
                         g["past_intr"].reshape(B * P, 4)).reshape(B, P, 18)
    got = vx.block_overlap(dev(g["cur_depth"]), dev(g["cur_cam"]), dev(sl), 1, 128).cpu().numpy()
    want = vo.block_overlap(g["cur_depth"], g["cur_cam"], sl, 1, 128)
    assert np.array_equal(got, want)
    assert (want.sum(-1) > 0).mean() > 0.5


def test_overlap_exact_on_slice_boundaries(vx):
    """Points that land on a slice's bounds up to float64 rounding: past cameras
    with the current pose, depth intervals whose ends are depths of the map, and
    principal points shifted by half a pixel so that pixel centres project onto
    u = 0, u = W, v = 0 or v = H. The kernel decides every point in float64, in
    the oracle's operation order with no fused multiply-add, so the counts
    match the oracle exactly even there."""
    rng = np.random.default_rng(5)
    Hp, Wp, T, F = 16, 24, 64, 1
    pose = synth.pose_looking((0.3, 1.2, -0.7), (0.2, -0.1, 1.0))
    intr = synth.intrinsics(Hp, Wp, 60.0)
    depth = rng.uniform(1.0, 9.0, (1, Hp, Wp)).astype(np.float32)
    depth[0, 3, 5] = np.float32(2.0)
    depth[0, 7, 9] = np.float32(6.5)
    cur = synth.camera_record(pose, intr)[None]
    z = depth[0].ravel()
    cams = []
    for zn, zf in ((2.0, 6.5), (float(np.sort(z)[10]), float(np.sort(z)[-10])), (0.0, 100.0)):
        for dcx, dcy in ((0.0, 0.0), (-0.5, 0.0), (0.5, 0.0), (0.0, -0.5), (0.0, 0.5)):
            k = intr.copy()
            k[2] += dcx
            k[3] += dcy
            cams.append(synth.camera_record(pose, k, zn, zf))
    sl = np.stack(cams)[None]
    got = vx.block_overlap(dev(depth), dev(cur), dev(sl), F, T).cpu().numpy()
    want = vo.block_overlap(depth, cur, sl, F, T)
    assert np.array_equal(got, want)
    assert 0 < want.sum() < want.size * T


def test_route_exact_ties_break_to_the_smaller_index(vx):
    # past chunks 0-2 are copies, and so are 3-5: their pooled scores tie exactly
    # (in fp32 on the device and in fp64 in the oracle), so the selection is
    # fixed by the tie-break alone
    rng = np.random.default_rng(21)
    T, d, B, H, m = 64, 64, 1, 2, 2
    Nq = m * T
    q = rng.standard_normal((B, H, Nq, d), dtype=np.float32)
    base = rng.standard_normal((2, B, H, Nq, d), dtype=np.float32)
    cur = rng.standard_normal((B, H, Nq, d), dtype=np.float32)
    k = np.concatenate([base[0]] * 3 + [base[1]] * 3 + [cur], axis=2)
    for dtype in ("f32", "bf16"):
        qq, kk = (q, k) if dtype == "f32" else (synth.f32_to_bf16_bits(q), synth.f32_to_bf16_bits(k))
        for topk in (m + 1, m + 2, m + 5, m + 7, m + 11):
            got = vx.route_topk(dev(qq), dev(kk), None, 0.0, topk, T).cpu().numpy()
            want, _ = vo.route_topk(qq, kk, None, 0.0, topk, T)
            assert np.array_equal(got, want), (dtype, topk)


def test_pipeline_async_geometry_matches_serial_and_oracle(vx):
    """Multiwarp -> slices -> overlap on a side stream while the keys are
    pooled; the selection waits for the counts through an event. Same result as
    running everything on one stream, and as the oracle (sampled heads)."""
    c = synth.make_case(5, layers=1)
    s = c.shape
    cams = np.stack([synth.camera_record(c.past_poses[0, j], c.past_intr[0, j]) for j in range(s.P)])
    q, k = dev(c.q[0]), dev(c.k[0])
    pd, poses, intr = dev(c.past_depth[0]), dev(c.past_poses[0]), dev(c.past_intr[0])
    cur = dev(c.cur_cam)

    def geometry(stream=None):
        depth = vx.depth_multiwarp(pd, dev(cams), cur[0], 0.01, stream=stream)
        sl = vx.slices_build(pd, poses, intr, stream=stream)
        return vx.block_overlap(depth[None], cur, sl[None], s.F, s.T, stream=stream)

    serial_counts = geometry()
    serial = vx.route_topk(q, k, serial_counts, s.alpha, s.topk, s.T)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    ev0, ev = torch.cuda.Event(), torch.cuda.Event()
    ev0.record(main)
    side.wait_event(ev0)
    async_counts = geometry(stream=side)
    ev.record(side)
    async_idx = vx.route_topk(q, k, async_counts, s.alpha, s.topk, s.T, counts_ready=ev)
    torch.cuda.synchronize()
    assert torch.equal(serial_counts, async_counts) and torch.equal(serial, async_idx)
    depth = vo.depth_multiwarp(c.past_depth[0], cams, c.cur_cam[0], 0.01)
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(depth[None], c.cur_cam, sl[None], s.F, s.T)
    assert np.array_equal(async_counts.cpu().numpy(), counts)
    heads = [2, 17]
    want, s_mod = vo.route_topk(c.q[0][:, heads], c.k[0][:, heads], counts, s.alpha, s.topk, s.T)
    ties = compare_selection(async_idx[:, heads].cpu().numpy(), want, s_mod, s.m,
                             label=f"workload 5 layer 0, async geometry, heads {heads}")
    assert ties <= tie_bound(2 * s.m)


def test_pipeline_layers_0_15_29_routing_and_attention():
    """Workload 5 (30 layers at chunk 48, current depth from the multiwarp of
    the 48 past depth maps): geometry exact on the GPU, then for layers 0, 15
    and 29 the selection of two heads against the oracle and attention of both
    heads' 36 query blocks on the oracle's selection. Layers are drawn on the
    host with one generator per (layer, head), workload 3's structure."""
    from geometry_routed_block_b200 import velox as vx
    layers, heads = (0, 15, 29), (3, 19)
    c = synth.make_case(5, layers=30, heads=heads, layer_ids=layers)
    s = c.shape
    cams = np.stack([synth.camera_record(c.past_poses[0, j], c.past_intr[0, j]) for j in range(s.P)])
    pd = dev(c.past_depth[0])
    depth = vx.depth_multiwarp(pd, dev(cams), dev(c.cur_cam[0]), 0.01)
    sl = vx.slices_build(pd, dev(c.past_poses[0]), dev(c.past_intr[0]))
    counts = vx.block_overlap(depth[None], dev(c.cur_cam), sl[None], s.F, s.T)
    want_depth = vo.depth_multiwarp(c.past_depth[0], cams, c.cur_cam[0], 0.01)
    want_sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    want_counts = vo.block_overlap(want_depth[None], c.cur_cam, want_sl[None], s.F, s.T)
    assert np.array_equal(depth.cpu().numpy(), want_depth, equal_nan=True)
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    for li, l in enumerate(layers):
        q, k, v = c.q[li], c.k[li], c.v[li]
        idx = vx.route_topk(dev(q), dev(k), counts, s.alpha, s.topk, s.T)
        want, s_mod = oracle_route_per_head(q, k, want_counts, s.alpha, s.topk, s.T)
        ties = compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                                 label=f"workload 5, layer {l}, heads {heads}")
        assert ties <= tie_bound(2 * s.m)
        rows = [(0, i, qb) for i in range(2) for qb in range(s.m)]
        attention_rows_vs_oracle(vx, q, k, v, want, s.T, rows,
                                 label=f"workload 5, layer {l}, heads {heads}, every query block")


# ---------------------------------------------------------------- pooled-key cache

@pytest.mark.parametrize("cfg", [1, 2])
def test_kbar_cache_matches_oracle_pooling(vx, cfg):
    c = synth.make_case(cfg)
    s = c.shape
    k = dev(c.k[0])
    kbar = vx.kbar_cache(s.B, s.H, s.P, s.Nq, s.d, s.T)
    for j in range(s.P):
        vx.kbar_append(k, s.Nq, s.T, j, kbar)
    want = vo.pool_blocks(c.k[0][:, :, : s.P * s.Nq], s.T)
    got = kbar.cpu().numpy().astype(np.float64)
    assert np.abs(got - want).max() <= 1e-6 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("cfg", [1, 3])
def test_cached_routing_equals_streaming_routing(vx, cfg):
    c = synth.make_case(cfg)
    s = c.shape
    q, k = dev(c.q[0]), dev(c.k[0])
    if cfg == 1:
        counts = vx.block_overlap(dev(c.cur_depth), dev(c.cur_cam), dev(c.past_cams), s.F, s.T)
    else:
        sl = vx.slices_build(dev(c.past_depth[0]), dev(c.past_poses[0]), dev(c.past_intr[0]))
        counts = vx.block_overlap(dev(c.cur_depth), dev(c.cur_cam), sl[None], s.F, s.T)
    kbar = vx.kbar_cache(s.B, s.H, s.P + 3, s.Nq, s.d, s.T)  # spare capacity
    for j in range(s.P):
        vx.kbar_append(k, s.Nq, s.T, j, kbar)
    for alpha in (0.0, s.alpha):
        want = vx.route_topk(q, k, counts, alpha, s.topk, s.T)
        got = vx.route_topk_cached(q, kbar, s.P, counts, alpha, s.topk, s.T)
        assert torch.equal(got, want)
    # no past chunk yet: only the current chunk's blocks
    only = vx.route_topk_cached(q, kbar, 0, None, s.alpha, s.m, s.T).cpu().numpy()
    assert (only == np.arange(s.m)).all()


# ---------------------------------------------------------------- 64-token blocks

@pytest.mark.parametrize("d", [128, 64])
def test_t64_routed_attention_pairs_blocks(vx, d):
    """64-token blocks (workload 4's generator at P = 8 with T = 64): the kernel
    packs two adjacent query blocks into one 128-row tile that walks the union
    of their routed lists; every query block of two heads against the oracle,
    on the oracle's selection, and the GPU selection against the oracle's."""
    heads = (2, 19)
    c = synth.make_case(4, P=8, heads=heads, T=64, d=d)
    s = c.shape
    assert s.T == 64 and s.m == 72
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    q, k, v = c.q[0], c.k[0], c.v[0]
    want, s_mod = oracle_route_per_head(q, k, counts, s.alpha, s.topk, s.T)
    idx = vx.route_topk(dev(q), dev(k), dev(counts), s.alpha, s.topk, s.T)
    ties = compare_selection(idx.cpu().numpy(), want, s_mod, s.m,
                             label=f"workload 4, P = 8, T = 64, d = {d}, heads {heads}")
    assert ties <= tie_bound(2 * s.m)
    rows = [(0, i, qb) for i in range(2) for qb in range(s.m)]
    attention_rows_vs_oracle(vx, q, k, v, want, s.T, rows,
                             label=f"workload 4, P = 8, T = 64, d = {d} (paired query blocks)")


@pytest.mark.parametrize("T,d", [(64, 128), (64, 64), (128, 64)])
def test_other_tile_shapes_at_chunk_48(vx, T, d):
    """The other block sizes and head dims at the headline's 48 past chunks
    (workload 4's generator with T and d set: the shapes of the bench line's
    tile_shapes record): routing of two heads against the oracle, and
    attention on 12 query blocks spread over each head on the oracle's
    selection (64-token blocks: the two-tile kernel and the split scoring)."""
    heads = (4, 21)
    c = synth.make_case(4, P=48, heads=heads, T=T, d=d)
    s = c.shape
    sl = vo.slices_build(c.past_depth[0], c.past_poses[0], c.past_intr[0])
    counts = vo.block_overlap(c.cur_depth, c.cur_cam, sl[None], s.F, s.T)
    q, k, v = c.q[0], c.k[0], c.v[0]
    want, s_mod = oracle_route_per_head(q, k, counts, s.alpha, s.topk, s.T)
    idx = vx.route_topk(dev(q), dev(k), dev(counts), s.alpha, s.topk, s.T)
    label = f"chunk 48, T = {T}, d = {d}, heads {heads}"
    ties = compare_selection(idx.cpu().numpy(), want, s_mod, s.m, label=label)
    assert ties <= tie_bound(2 * s.m)
    step = max(1, s.m // 12)
    rows = [(0, i, qb) for i in range(2) for qb in range(0, s.m, step)][:24]
    attention_rows_vs_oracle(vx, q, k, v, want, s.T, rows, label=label)


def test_t64_routing_takes_exactly_its_workspace(vx):
    """64-token routing keeps the pooled past keys in the workspace: the size
    the library reports is enough (same selection as with room to spare) and
    256 bytes less is refused."""
    rng = np.random.default_rng(6464)
    B, H, T, d, m, P = 1, 2, 64, 128, 6, 5
    q, k, _ = _random_qkv(rng, B, H, m * T, (P + 1) * m * T, d)
    q, k = dev(q), dev(k)
    topk = 13
    n = vx.lib.velox_route_topk_workspace_size(B, H, m * T, (P + 1) * m * T, d, T)
    big = torch.empty(n + 4096, dtype=torch.uint8, device="cuda")
    exact = torch.empty(n, dtype=torch.uint8, device="cuda")
    want = vx.route_topk(q, k, None, 0.0, topk, T, ws=big)
    got = vx.route_topk(q, k, None, 0.0, topk, T, ws=exact)
    assert torch.equal(got, want)
    with pytest.raises(vx.VeloxError):
        vx.route_topk(q, k, None, 0.0, topk, T, ws=exact[: n - 256])


def test_t64_long_lists_fall_back_to_one_block_per_tile(vx):
    """A routed list longer than two of them fit in the tile's walk (4,096
    blocks): one 64-token block per tile, still exact against the oracle."""
    rng = np.random.default_rng(64)
    T, d, B, H, m, nkb, topk = 64, 128, 1, 1, 3, 4500, 4200
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    q, k, v = f(B, H, m * T, d), f(B, H, nkb * T, d), f(B, H, nkb * T, d)
    idx = np.stack([np.sort(rng.choice(nkb, topk, replace=False)) for _ in range(m)])
    idx = idx.reshape(B, H, m, topk).astype(np.int32)
    o, lse = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(idx), T)
    ref = vo.sparse_attention(q, k, v, idx, T, rows=[(0, 0, qb) for qb in range(m)])
    for (b, h, qb), (o_ref, lse_ref) in ref.items():
        sl_ = slice(qb * T, (qb + 1) * T)
        compare_attention(o[b, h, sl_], o_ref, f"T = 64, 4,200-block list, row {qb}")
        assert np.abs(lse[b, h, sl_].cpu().numpy() - lse_ref).max() < 1e-3
