"""The attention kernels' bounded waits, made to run out on purpose without a
fault: through the test entry point, the tensor-core issuer issues nothing, so
no MMA completion ever arrives and every wait on one expires after a short
limit. The kernel must then report VELOX_STATUS_TIMEOUT in the status word,
drain the copies it started and return; the device stays usable, and a normal
call right after gives the oracle's output with a clean status."""
import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth
from oracle import velox_oracle as vo
from tests.parity_utils import compare_attention, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,d", [(128, 128), (64, 128)])
def test_expired_waits_report_timeout_and_leave_the_device_usable(T, d):
    from geometry_routed_block_b200 import velox as vx
    rng = np.random.default_rng(T + d)
    B, H, Nq, Nk = 1, 2, 4 * T, 12 * T
    f = lambda *sh: synth.f32_to_bf16_bits(rng.standard_normal(sh, dtype=np.float32))
    q, k, v = f(B, H, Nq, d), f(B, H, Nk, d), f(B, H, Nk, d)
    m = Nq // T
    idx = np.sort(rng.choice(Nk // T, size=(B, H, m, 5), replace=True), axis=-1).astype(np.int32)
    qd, kd, vd, idd = dev(q), dev(k), dev(v), dev(idx)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # 8 CTAs (T = 128: two query blocks each; T = 64: one each), 50 ms limit
    vx.sparse_attn_fwd_test(qd, kd, vd, idd, T, status, 0.05, vx.VELOX_TEST_SKIP_MMA)
    torch.cuda.synchronize()
    assert int(status.item()) & vx.VELOX_STATUS_TIMEOUT
    assert not int(status.item()) & vx.VELOX_STATUS_BAD_INDEX
    # the context is intact: normal calls (test entry point without the hook,
    # and the product entry point) give the oracle's result with a clean status
    status.zero_()
    o1 = vx.sparse_attn_fwd_test(qd, kd, vd, idd, T, status, 2.0, 0)
    o2, _ = vx.sparse_attn_fwd(qd, kd, vd, idd, T, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o_ref, _ = vo.sparse_attention(q, k, v, idx, T)
    compare_attention(o1, o_ref, "after timeout (test entry point)")
    compare_attention(o2, o_ref, "after timeout")
    assert torch.equal(o1, o2)


def test_test_entry_point_rejects_bad_limits_and_flags():
    from geometry_routed_block_b200 import velox as vx
    x = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for limit, flags in ((0.0, 0), (20.0, 0), (1.0, 4)):
        with pytest.raises(vx.VeloxError):
            vx.sparse_attn_fwd_test(x, x, x, None, 128, status, limit, flags)
