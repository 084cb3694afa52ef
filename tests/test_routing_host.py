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
