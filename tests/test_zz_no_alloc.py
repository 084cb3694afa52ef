"""velox_depth_multiwarp_noalloc: the multiwarp for callers that cannot allocate
device memory (a plugin that is handed only its input and output buffers, a
latency-critical loop that must not call cudaMalloc). Its scratch is a fixed
array inside the library, so the test checks, through the C ABI, that two
calls in a row -- on different inputs, so the second starts from the first
one's leftovers -- give exactly the depth of the workspace entry point
(depth is compared bit for bit, NaN holes included), including a grid of
exactly the limit (256 x 256, where the scratch layout fills the array), and
that grids above the limit are refused without a launch.

Collected last (file name) so that a failure here does not hide the others."""
import ctypes

import numpy as np
import pytest
import torch

from geometry_routed_block_b200 import synth

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _inputs(cfg, seed):
    c = synth.geometry_only(cfg, seed=seed)
    s = c.shape
    cams = np.stack([synth.camera_record(c.past_poses[0, j], c.past_intr[0, j]) for j in range(s.P)])
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return to(c.past_depth[0]), to(cams), to(c.cur_cam[0]), s


def test_noalloc_multiwarp_matches_workspace_entry_point():
    assert torch.cuda.is_available()
    from geometry_routed_block_b200 import velox as vx
    lib = vx.lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # two calls in a row on different scenes (48 past chunks each, 32 x 48 grid)
    for cfg, seed in ((5, 1005), (5, 2024)):
        pd, cams, cur, s = _inputs(cfg, seed)
        want = vx.depth_multiwarp(pd, cams, cur, 0.01)
        got = torch.full((s.Hp, s.Wp), -7.0, dtype=torch.float32, device="cuda")
        rc = lib.velox_depth_multiwarp_noalloc(_ptr(pd), _ptr(cams), _ptr(cur), s.P, s.Hp, s.Wp,
                                               0.01, _ptr(got), stream)
        assert rc == 0, vx.strerror(rc)
        torch.cuda.synchronize()
        g, w = got.cpu().numpy(), want.cpu().numpy()
        assert np.array_equal(g, w, equal_nan=True)
        assert np.isfinite(w).mean() > 0.5


def _room_at(Hp, Wp, P, seed):
    """P past depth maps of a synthetic room along the camera loop, cast at
    Hp x Wp, with their cameras and the current camera (chunk P)."""
    scene = synth.room_scene(np.random.default_rng(seed))
    intr = synth.intrinsics(Hp, Wp, 60.0)
    poses = [synth.loop_pose(n)[0] for n in range(P + 1)]
    past = np.stack([synth.render_depth(scene, poses[j], intr, Hp, Wp) for j in range(P)])
    cams = np.stack([synth.camera_record(poses[j], intr) for j in range(P)])
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return to(past), to(cams), to(synth.camera_record(poses[P], intr))


def test_noalloc_multiwarp_at_the_pixel_limit():
    from geometry_routed_block_b200 import velox as vx
    lib = vx.lib
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    Hp = Wp = 256
    assert Hp * Wp == 65536  # VELOX_MULTIWARP_NOALLOC_MAX_PIXELS
    pd, cams, cur = _room_at(Hp, Wp, 6, 31)
    want = vx.depth_multiwarp(pd, cams, cur, 0.01)
    for _ in range(2):
        got = torch.full((Hp, Wp), -7.0, dtype=torch.float32, device="cuda")
        rc = lib.velox_depth_multiwarp_noalloc(_ptr(pd), _ptr(cams), _ptr(cur), 6, Hp, Wp, 0.01,
                                               _ptr(got), stream)
        assert rc == 0, vx.strerror(rc)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy(), want.cpu().numpy(), equal_nan=True)
    # a forward splat of six maps at this resolution leaves holes; enough pixels
    # are covered that the comparison is not trivial
    assert torch.isfinite(want).float().mean().item() > 0.3


def test_noalloc_multiwarp_rejects_grids_above_the_limit():
    from geometry_routed_block_b200 import velox as vx
    lib = vx.lib
    limit = 65536
    pd = torch.zeros((1, 257, 256), dtype=torch.float32, device="cuda")
    cam = torch.zeros(18, dtype=torch.float32, device="cuda")
    out = torch.full((257, 256), 3.25, dtype=torch.float32, device="cuda")
    rc = lib.velox_depth_multiwarp_noalloc(_ptr(pd), _ptr(cam), _ptr(cam), 1, 257, 256, 0.01,
                                           _ptr(out), None)
    torch.cuda.synchronize()
    assert rc == vx.VELOX_EINVAL and 257 * 256 > limit
    assert bool((out == 3.25).all())  # nothing was launched: the output is untouched
