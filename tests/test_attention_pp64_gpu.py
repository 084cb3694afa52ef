"""The two-tile attention kernel for 64-token blocks (head dim 128): a CTA owns
four query blocks as two 128-row tiles, each tile walking the union of its two
blocks' routed lists, two walk entries per 128-key tile. (With head dim 64 the
library keeps the one-tile kernel, which pairs two blocks per tile; the same
cases run on it.) Element by element against the oracle on what is particular
to the two-tile kernel: CTAs with one to four query
blocks, adjacent blocks with disjoint lists (one block's rows see masked
entries before its first listed one), identical lists, repeated blocks (the
concatenated walk), odd walk lengths (a half tile no block listed), tiles whose
walks differ in length, dense walks over an odd number of key blocks, large
logits (rescaling), out-of-range indices; and the limits past which the
library sends 64-token blocks to the one-tile kernel (lists of more than 2,048
blocks, more than 16,384 key blocks)."""
import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo
from tests.parity_utils import compare_attention, dev

pytestmark = pytest.mark.gpu

T, D = 64, 128
DIMS = pytest.mark.parametrize("d", [128, 64])


@pytest.fixture(scope="module")
def vx():
    from geometry_routed_block_b200 import velox
    return velox


def _qkv(rng, B, H, m, nkb, d=D):
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    return f(B, H, m * T, d), f(B, H, nkb * T, d), f(B, H, nkb * T, d)


def _check(vx, q, k, v, idx, label, rows=None, lse_tol=1e-3):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), None if idx is None else dev(idx), T,
                                status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, label
    ref = vo.sparse_attention(q, k, v, idx, T, rows=rows)
    if rows is None:
        o_ref, lse_ref = ref
        compare_attention(o, o_ref, label)
        assert np.abs(lse.cpu().numpy() - lse_ref).max() < lse_tol, label
        return
    for (b, h, qb), (o_ref, lse_ref) in ref.items():
        sl = slice(qb * T, (qb + 1) * T)
        compare_attention(o[b, h, sl], o_ref, f"{label}, row {(b, h, qb)}")
        assert np.abs(lse[b, h, sl].cpu().numpy() - lse_ref).max() < lse_tol, label


@DIMS
@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 6, 7, 9])
def test_ragged_ctas_random_lists(vx, m, d):
    rng = np.random.default_rng(640 + m + d)
    B, H, nkb, topk = 2, 3, 23, 6
    q, k, v = _qkv(rng, B, H, m, nkb, d)
    idx = np.stack([rng.choice(nkb, topk, replace=False) for _ in range(B * H * m)])
    _check(vx, q, k, v, idx.reshape(B, H, m, topk).astype(np.int32),
           f"m = {m}, d = {d}, shuffled lists")


@DIMS
@pytest.mark.parametrize("kind", ["disjoint", "identical", "repeats", "nested"])
def test_list_structures(vx, kind, d):
    rng = np.random.default_rng({"disjoint": 1, "identical": 2, "repeats": 3, "nested": 4}[kind])
    B, H, m, nkb, topk = 1, 2, 8, 40, 9
    q, k, v = _qkv(rng, B, H, m, nkb, d)
    idx = np.empty((B, H, m, topk), dtype=np.int32)
    for h in range(H):
        for qb in range(m):
            if kind == "disjoint":
                # even blocks list the upper key blocks, odd ones the lower: in
                # each tile the walk's first entries belong to one block only
                base = 30 if qb % 2 == 0 else 0
                idx[0, h, qb] = rng.permutation(np.arange(base, base + topk))
            elif kind == "identical":
                idx[0, h, qb] = np.sort(rng.choice(nkb, topk, replace=False)) if qb % 2 == 0 \
                    else idx[0, h, qb - 1]
            elif kind == "repeats":
                idx[0, h, qb] = rng.integers(0, 5, size=topk)
            else:
                # the odd block shares all but `extra` of the even block's list:
                # tile A's walk is the longer in the first CTA, tile B's in the
                # second (one tile runs on alone at the end)
                if qb % 2 == 0:
                    idx[0, h, qb] = rng.choice(nkb, topk, replace=False)
                else:
                    extra = 3 if qb in (1, 7) else 0
                    sub = rng.choice(idx[0, h, qb - 1], topk - extra, replace=False)
                    pad = rng.choice(np.setdiff1d(np.arange(nkb), idx[0, h, qb - 1]),
                                     topk - len(sub), replace=False)
                    idx[0, h, qb] = np.concatenate([sub, pad])
    _check(vx, q, k, v, idx, f"{kind} lists, d = {d}")


@DIMS
@pytest.mark.parametrize("nkb", [1, 2, 11, 64])
def test_dense_walks(vx, nkb, d):
    rng = np.random.default_rng(6400 + nkb + d)
    q, k, v = _qkv(rng, 1, 2, 6, nkb, d)
    _check(vx, q, k, v, None, f"dense over {nkb} key blocks, d = {d}")


@DIMS
def test_large_logits_rescale(vx, d):
    rng = np.random.default_rng(6464 + d)
    B, H, m, nkb = 1, 2, 6, 40
    qf = rng.standard_normal((B, H, m * T, d), dtype=np.float32)
    kf = rng.standard_normal((B, H, nkb * T, d), dtype=np.float32)
    ramp = np.linspace(0.2, 6.0, nkb * T, dtype=np.float32)[None, None, :, None]
    kf = kf * ramp + ramp * qf.mean(axis=2, keepdims=True)
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    v = synth.f32_to_bf16_bits(rng.standard_normal((B, H, nkb * T, d), dtype=np.float32))
    idx = np.stack([np.sort(rng.choice(nkb, 17, replace=False)) for _ in range(B * H * m)])
    _check(vx, q, k, v, idx.reshape(B, H, m, 17).astype(np.int32), "rescale, routed",
           lse_tol=2e-3)
    _check(vx, q, k, v, None, "rescale, dense", lse_tol=2e-3)


@DIMS
def test_bad_indices_flagged(vx, d):
    rng = np.random.default_rng(646 + d)
    q, k, v = _qkv(rng, 1, 1, 5, 16, d)
    idx = np.array([[[[0, 1, -5], [2, 16, 3], [4, 5, 6], [7, 8, 99], [1, 2, 3]]]], dtype=np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, _ = vx.sparse_attn_fwd(dev(q), dev(k), dev(v), dev(idx), T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & vx.VELOX_STATUS_BAD_INDEX
    fixed = np.where((idx < 0) | (idx >= 16), 0, idx).astype(np.int32)
    o_ref, _ = vo.sparse_attention(q, k, v, fixed, T)
    compare_attention(o, o_ref, "bad-index replacement, 64-token blocks")


def test_lists_longer_than_the_walk_take_the_one_tile_kernel(vx):
    """2,500 blocks per list: two lists no longer fit this kernel's walk; the
    one-tile kernel (which pairs lists of up to 4,096) serves them."""
    rng = np.random.default_rng(2500)
    m, nkb, topk = 3, 3000, 2500
    q, k, v = _qkv(rng, 1, 1, m, nkb)
    idx = np.stack([rng.choice(nkb, topk, replace=False) for _ in range(m)])
    _check(vx, q, k, v, idx.reshape(1, 1, m, topk).astype(np.int32), "2,500-block lists")


def test_more_key_blocks_than_a_walk_entry_holds(vx):
    """16,500 key blocks (past the 14-bit entry): the one-tile kernel."""
    rng = np.random.default_rng(16500)
    m, nkb, topk = 3, 16500, 7
    idx = np.stack([rng.choice(nkb, topk, replace=False) for _ in range(m)])
    idx[0, :2] = [16499, 16384]
    # random keys and values in the listed blocks only (the rest stay zero)
    q, kl, vl = _qkv(rng, 1, 1, m, m * topk)
    k = np.zeros((1, 1, nkb * T, D), dtype=np.uint16)
    v = np.zeros_like(k)
    for j, kb in enumerate(idx.reshape(-1)):
        k[0, 0, kb * T:(kb + 1) * T] = kl[0, 0, j * T:(j + 1) * T]
        v[0, 0, kb * T:(kb + 1) * T] = vl[0, 0, j * T:(j + 1) * T]
    _check(vx, q, k, v, idx.reshape(1, 1, m, topk).astype(np.int32), "16,500 key blocks")
