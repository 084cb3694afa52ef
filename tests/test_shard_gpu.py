"""The head-sharded multi-GPU mode on one GPU: a rank that holds only its share
of the heads (geometry replicated) must produce exactly the counts, selection,
output and LSE of those heads in the full-head run -- routing and attention of
head h read only head h's Q/K/V -- so that the all-gather of the shares is the
full-head result. Runs bench.Workload, the step the benchmark times."""
import os
import sys

import pytest
import torch

from geometry_routed_block_b200 import synth

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world,rank", [(4, 1), (8, 7)])
def test_head_share_equals_slice_of_full_head_run(world, rank):
    sys.path.insert(0, ROOT)
    import bench
    device = torch.device("cuda", 0)
    full = synth.make_case(4, P=8)
    h0, h1 = bench.head_range(full.shape.H, world, rank)
    part = synth.make_case(4, P=8, heads=tuple(range(h0, h1)))
    wf, wp = bench.Workload(full, device), bench.Workload(part, device)
    # the share's output goes straight into its slice of a gathered buffer, as in
    # the benchmark (at world size 1 the gather is the identity)
    o_all = torch.empty((1,) + tuple(wp.o.shape[1:]), dtype=wp.o.dtype, device=device)
    wp.o = o_all[0:1]
    for w in (wf, wp):
        w.step()
    torch.cuda.synchronize()
    assert torch.equal(wp.counts, wf.counts)
    assert torch.equal(wp.idx, wf.idx[:, h0:h1])
    assert torch.equal(wp.o, wf.o[:, h0:h1])
    assert torch.equal(wp.lse, wf.lse[:, h0:h1])
    assert torch.equal(bench.gather_heads(o_all, wp.o, 1), wf.o[:, h0:h1])
    assert int(wf.status.item()) == 0 and int(wp.status.item()) == 0
