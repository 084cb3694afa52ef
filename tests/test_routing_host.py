"""Host-side invariants of the routing kernels (CPU).

The selection kernel maps a past key block kb to its chunk kb // m as
trunc((kb + 1/2) * fp32(1/m)) in float32 (round-to-nearest multiply): the
quotient sits at least 1/(2m) from an integer, so the truncation is exact for
every block count the library accepts (Nk / T <= 8192)."""
import numpy as np


def test_reciprocal_chunk_division_is_exact():
    kb_all = np.arange(8192, dtype=np.int64)
    kbf = kb_all.astype(np.float32) + np.float32(0.5)
    for m in range(1, 8193):
        inv = np.float32(1.0) / np.float32(m)
        got = np.trunc((kbf * inv).astype(np.float32)).astype(np.int64)
        assert np.array_equal(got, kb_all // m), m


def test_selection_change_metric():
    import bench
    n_past = 10
    # two rows, k = 4 with 2 current blocks (indices >= n_past) each
    ref = np.array([[1, 2, 10, 11], [0, 5, 10, 11]])
    same = bench.selection_change(ref, ref.copy(), n_past)
    assert same == {"jaccard": 1.0, "recall": 1.0, "rows_identical": 1.0}
    got = np.array([[1, 3, 10, 11], [0, 5, 10, 11]])
    r = bench.selection_change(ref, got, n_past)
    # row 0: {1,2} vs {1,3} -> J = 1/3, recall 1/2; row 1 identical
    assert abs(r["jaccard"] - round((1 / 3 + 1) / 2, 4)) < 1e-12
    assert r["recall"] == 0.75 and r["rows_identical"] == 0.5
    disjoint = bench.selection_change(ref, np.array([[3, 4, 10, 11], [1, 2, 10, 11]]), n_past)
    assert disjoint == {"jaccard": 0.0, "recall": 0.0, "rows_identical": 0.0}


def test_perturb_depth_model():
    from geometry_routed_block_b200 import synth
    rng = np.random.default_rng(3)
    d = rng.uniform(1, 10, (4, 8, 8)).astype(np.float32)
    d[0, 0, 0] = np.nan
    assert np.array_equal(synth.perturb_depth(d, rng), d, equal_nan=True)
    # a power-of-two scale is exact in float32
    assert np.array_equal(synth.perturb_depth(d, rng, scale=2.0), d * 2, equal_nan=True)
    h = synth.perturb_depth(d, np.random.default_rng(4), hole_frac=0.5)
    frac = np.isnan(h).mean()
    assert 0.35 < frac < 0.65 and np.isnan(h[0, 0, 0])
    n = synth.perturb_depth(d, np.random.default_rng(5), noise_sd=0.05)
    rel = np.abs(n / d - 1)[np.isfinite(d)]
    assert 0.02 < rel.mean() < 0.06 and np.isnan(n[0, 0, 0])
