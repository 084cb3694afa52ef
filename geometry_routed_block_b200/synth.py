"""Seeded synthetic inputs for the Velox routed-attention path.

This module builds scenes, camera trajectories, depth maps and Q/K/V tensors. It
is the one piece shared by the CPU oracle's tests and the CUDA path: it holds
none of the method's arithmetic (no overlap counting, pooling, scoring,
selection, attention or depth warping). Depth maps come from an analytic ray
cast of the synthetic scene; that is scene rendering, not a step of the method.

Camera records are float32[18]:  R (row-major 3x3, world->camera, OpenCV axes:
x right, y down, z forward), t[3] (x_c = R x_w + t), fx, fy, cx, cy (latent-grid
pixel units), znear, zfar (depth interval; 0 for cameras that carry none).

bf16 tensors are carried as uint16 numpy arrays holding the bf16 bit pattern
(round-to-nearest-even from float32).

Workloads (sizes from the method's headline chunk-48 setting and its neighbours):
  1  tiny: B1 H2 d64 T64, 16x16 grid, 1 frame, 4 past chunks, fp32 Q/K/V
  2  dense-parity: B1 H12 d128 T128, 3x32x48 tokens, 8 past chunks, bf16
  3  chunk-48 headline: B1 H24 d128 T128, 3x32x48 tokens, 48 past chunks, bf16
  4  rollout sweep: workload 3 at 8/16/24/32/48/96 past chunks
  5  per-step pipeline: workload 3 with 30 layers and warped current depth
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

CAM_FLOATS = 18


@dataclass
class Shape:
    B: int
    H: int
    d: int
    T: int
    F: int
    Hp: int
    Wp: int
    P: int
    topk: int
    alpha: float
    fov_deg: float = 60.0
    layers: int = 1
    dtype: str = "bf16"

    @property
    def Nq(self) -> int:
        return self.F * self.Hp * self.Wp

    @property
    def m(self) -> int:
        return self.Nq // self.T

    @property
    def Nk(self) -> int:
        return (self.P + 1) * self.Nq

    @property
    def nKB(self) -> int:
        return self.Nk // self.T


def topk_for(P: int, m: int = 36, frac: float = 0.2) -> int:
    """About 20% of all key blocks, current chunk included."""
    return int(round(frac * (P + 1) * m))


SHAPES = {
    1: Shape(B=1, H=2, d=64, T=64, F=1, Hp=16, Wp=16, P=4, topk=6, alpha=2.0, dtype="f32"),
    2: Shape(B=1, H=12, d=128, T=128, F=3, Hp=32, Wp=48, P=8, topk=324, alpha=2.0),
    3: Shape(B=1, H=24, d=128, T=128, F=3, Hp=32, Wp=48, P=48, topk=353, alpha=2.0),
    5: Shape(B=1, H=24, d=128, T=128, F=3, Hp=32, Wp=48, P=48, topk=353, alpha=2.0, layers=30),
}
SWEEP_P = (8, 16, 24, 32, 48, 96)


def shape_for(cfg: int, P: int | None = None, H: int | None = None,
              layers: int | None = None, T: int | None = None, d: int | None = None) -> Shape:
    if cfg == 4:
        base = SHAPES[3]
        P = 48 if P is None else P
        T = base.T if T is None else T
        d = base.d if d is None else d
        m = base.F * base.Hp * base.Wp // T
        s = Shape(**{**base.__dict__, "P": P, "T": T, "d": d, "topk": topk_for(P, m)})
    else:
        s = Shape(**SHAPES[cfg].__dict__)
        if P is not None and P != s.P:
            s.P = P
            s.topk = min(s.topk, s.nKB) if cfg in (1, 2) else topk_for(P, s.m)
    if H is not None:
        s.H = H
    if layers is not None:
        s.layers = layers
    return s


# ----------------------------------------------------------------------------
# bf16 helpers (input encoding only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 -> bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    out = ((u + np.uint32(0x7FFF) + r) >> np.uint32(16)).astype(np.uint16)
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# cameras and scenes
# ----------------------------------------------------------------------------

def intrinsics(Hp: int, Wp: int, fov_deg: float) -> np.ndarray:
    """Pinhole intrinsics for a horizontal field of view, principal point at
    the grid centre, square pixels. Evaluated on the host in double and
    stored as float32, so no transcendental runs on either side of the path."""
    fx = (Wp / 2.0) / math.tan(math.radians(fov_deg) / 2.0)
    return np.array([fx, fx, Wp / 2.0, Hp / 2.0], dtype=np.float32)


def pose_looking(pos, forward) -> np.ndarray:
    """World->camera [R|t] (float32[12]) for a camera at `pos` looking along
    `forward`, world up = +y, OpenCV camera axes (y down)."""
    pos = np.asarray(pos, dtype=np.float64)
    z = np.asarray(forward, dtype=np.float64)
    z = z / np.linalg.norm(z)
    down = np.array([0.0, -1.0, 0.0])
    x = np.cross(down, z)
    x = x / np.linalg.norm(x)
    y = np.cross(z, x)
    R = np.stack([x, y, z])
    t = -R @ pos
    return np.concatenate([R.reshape(-1), t]).astype(np.float32)


def camera_record(pose12: np.ndarray, intr4: np.ndarray, znear: float = 0.0,
                  zfar: float = 0.0) -> np.ndarray:
    rec = np.zeros(CAM_FLOATS, dtype=np.float32)
    rec[:12] = pose12
    rec[12:16] = intr4
    rec[16] = znear
    rec[17] = zfar
    return rec


@dataclass
class Scene:
    boxes: list = field(default_factory=list)   # (lo[3], hi[3])
    room: tuple | None = None                    # (lo[3], hi[3]) interior
    ground: bool = False
    miss_depth: float = 50.0


def _ray_box(o, w, lo, hi):
    """Slab test, vectorised over rays. Returns entry distance (inf on miss)."""
    with np.errstate(divide="ignore", invalid="ignore"):
        inv = 1.0 / w
        t1 = (lo[None, :] - o[None, :]) * inv
        t2 = (hi[None, :] - o[None, :]) * inv
    tmin = np.nanmax(np.minimum(t1, t2), axis=1)
    tmax = np.nanmin(np.maximum(t1, t2), axis=1)
    hit = (tmax >= tmin) & (tmin > 1e-6)
    return np.where(hit, tmin, np.inf)


def _ray_room(o, w, lo, hi):
    """Exit distance of rays starting inside an axis-aligned room."""
    with np.errstate(divide="ignore", invalid="ignore"):
        tp = np.where(w > 0, (hi[None, :] - o[None, :]) / w, np.inf)
        tn = np.where(w < 0, (lo[None, :] - o[None, :]) / w, np.inf)
    return np.minimum(tp, tn).min(axis=1)


def render_depth(scene: Scene, pose12: np.ndarray, intr4: np.ndarray, Hp: int,
                 Wp: int) -> np.ndarray:
    """z-depth of the first surface hit through every pixel centre (float32)."""
    R = pose12[:9].astype(np.float64).reshape(3, 3)
    t = pose12[9:12].astype(np.float64)
    fx, fy, cx, cy = (float(v) for v in intr4)
    o = -R.T @ t
    rr, cc = np.meshgrid(np.arange(Hp) + 0.5, np.arange(Wp) + 0.5, indexing="ij")
    dc = np.stack([(cc - cx) / fx, (rr - cy) / fy, np.ones_like(cc)], axis=-1).reshape(-1, 3)
    w = dc @ R  # rows: R^T d_c; a unit step of the ray parameter is one unit of camera z
    best = np.full(w.shape[0], np.inf)
    for lo, hi in scene.boxes:
        best = np.minimum(best, _ray_box(o, w, np.asarray(lo, float), np.asarray(hi, float)))
    if scene.room is not None:
        best = np.minimum(best, _ray_room(o, w, np.asarray(scene.room[0], float),
                                          np.asarray(scene.room[1], float)))
    if scene.ground:
        with np.errstate(divide="ignore", invalid="ignore"):
            tg = np.where(w[:, 1] < 0, -o[1] / w[:, 1], np.inf)
        best = np.minimum(best, tg)
    best = np.minimum(best, scene.miss_depth)
    return best.reshape(Hp, Wp).astype(np.float32)


def room_scene(rng: np.random.Generator) -> Scene:
    """12 x 12 x 4 room with 8 boxes, kept clear of the radius-3 camera loop."""
    boxes = []
    for _ in range(3):  # central boxes
        c = rng.uniform(-1.1, 1.1, size=2)
        hx, hz = rng.uniform(0.2, 0.5, size=2)
        h = rng.uniform(0.6, 2.5)
        boxes.append(((c[0] - hx, 0.0, c[1] - hz), (c[0] + hx, h, c[1] + hz)))
    for _ in range(5):  # boxes against the walls
        ang = rng.uniform(0, 2 * math.pi)
        r = rng.uniform(4.6, 5.2)
        c = (r * math.cos(ang), r * math.sin(ang))
        hx, hz = rng.uniform(0.3, 0.7, size=2)
        h = rng.uniform(0.5, 3.0)
        boxes.append(((max(c[0] - hx, -5.95), 0.0, max(c[1] - hz, -5.95)),
                      (min(c[0] + hx, 5.95), h, min(c[1] + hz, 5.95))))
    return Scene(boxes=boxes, room=((-6.0, 0.0, -6.0), (6.0, 4.0, 6.0)))


def ground_scene(rng: np.random.Generator) -> Scene:
    """Ground plane y = 0 plus 6 boxes around a forward walk along +z."""
    boxes = []
    for i in range(6):
        side = -1 if i % 2 == 0 else 1
        cz = rng.uniform(2.0, 14.0)
        cx = side * rng.uniform(1.8, 4.5)
        hx, hz = rng.uniform(0.4, 1.0, size=2)
        h = rng.uniform(0.8, 3.5)
        boxes.append(((cx - hx, 0.0, cz - hz), (cx + hx, h, cz + hz)))
    return Scene(boxes=boxes, ground=True, miss_depth=50.0)


def loop_pose(n: int, radius: float = 3.0, period: int = 16, height: float = 1.5):
    """Camera n on a circle of `radius`, 360/period degrees per chunk, facing the tangent."""
    th = 2 * math.pi * (n % period) / period
    pos = (radius * math.cos(th), height, radius * math.sin(th))
    fwd = (-math.sin(th), 0.0, math.cos(th))
    return pose_looking(pos, fwd), math.degrees(th) % 360.0


def walk_poses(n_total: int, rng: np.random.Generator, height: float = 1.5):
    poses, yaws = [], []
    pos = np.array([0.0, height, 0.0])
    yaw = 0.0
    for _ in range(n_total):
        fwd = (math.sin(math.radians(yaw)), 0.0, math.cos(math.radians(yaw)))
        poses.append(pose_looking(pos, fwd))
        yaws.append(yaw)
        pos = pos + np.array([fwd[0], 0.0, fwd[2]])
        yaw += rng.uniform(-10.0, 10.0)
    return poses, yaws


def view_overlap_proxy(yaw_a: float, yaw_b: float, fov_deg: float) -> float:
    """Scene-level ground truth used only to shape synthetic K: the fraction of
    the horizontal field of view two cameras share when their yaws differ by
    the wrapped angle between them (1 at equal yaw, 0 beyond one field of view)."""
    dy = abs((yaw_a - yaw_b + 180.0) % 360.0 - 180.0)
    return max(0.0, 1.0 - dy / fov_deg)


# ----------------------------------------------------------------------------
# cases
# ----------------------------------------------------------------------------

@dataclass
class Case:
    cfg: int
    shape: Shape
    seed: int
    q: np.ndarray            # [L,B,H,Nq,d] uint16 (bf16) or float32
    k: np.ndarray            # [L,B,H,Nk,d]
    v: np.ndarray            # [L,B,H,Nk,d]
    cur_depth: np.ndarray    # [B,Hp,Wp] float32 (ground truth for the current camera)
    cur_cam: np.ndarray      # [B,18] float32
    past_depth: np.ndarray | None   # [B,P,Hp,Wp] float32
    past_poses: np.ndarray | None   # [B,P,12]
    past_intr: np.ndarray | None    # [B,P,4]
    past_cams: np.ndarray           # [B,P,18] (znear/zfar set only where given directly)
    slices_given: bool              # True: znear/zfar of past_cams are inputs (workload 1)
    meta: dict = field(default_factory=dict)


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _tiny(seed: int) -> Case:
    s = SHAPES[1]
    rng = np.random.default_rng(seed)
    intr = intrinsics(s.Hp, s.Wp, s.fov_deg)
    past = []
    for j in range(s.P):
        th = math.radians(15.0 * j)
        pos = (2.0 * math.sin(th), 0.0, 2.0 * math.cos(th))
        pose = pose_looking(pos, (-pos[0], 0.0, -pos[2]))
        lo, hi = np.sort(rng.uniform(1.0, 10.0, size=2))
        past.append(camera_record(pose, intr, lo, hi))
    th = math.radians(60.0)
    pos = (2.0 * math.sin(th), 0.0, 2.0 * math.cos(th))
    cur = camera_record(pose_looking(pos, (-pos[0], 0.0, -pos[2])), intr)
    depth = rng.uniform(1.0, 10.0, size=(s.Hp, s.Wp)).astype(np.float32)
    q = _normal(rng, (1, s.B, s.H, s.Nq, s.d))
    k = _normal(rng, (1, s.B, s.H, s.Nk, s.d))
    v = _normal(rng, (1, s.B, s.H, s.Nk, s.d))
    return Case(cfg=1, shape=s, seed=seed, q=q, k=k, v=v, cur_depth=depth[None],
                cur_cam=cur[None], past_depth=None, past_poses=None, past_intr=None,
                past_cams=np.stack(past)[None], slices_given=True)


def _parallel_heads(fn, jobs):
    """Run per-head generators on a thread pool (numpy releases the GIL)."""
    workers = max(1, min(32, os.cpu_count() or 1, len(jobs)))
    if workers == 1:
        return [fn(*j) for j in jobs]
    with ThreadPoolExecutor(workers) as ex:
        return list(ex.map(lambda j: fn(*j), jobs))


def _walk(seed: int, s: Shape) -> Case:
    rng = np.random.default_rng(seed)
    scene = ground_scene(rng)
    intr = intrinsics(s.Hp, s.Wp, s.fov_deg)
    poses, _ = walk_poses(s.P + 1, rng)
    depths = np.stack([render_depth(scene, p, intr, s.Hp, s.Wp) for p in poses])
    L = s.layers
    q = np.empty((L, s.B, s.H, s.Nq, s.d), np.uint16)
    k = np.empty((L, s.B, s.H, s.Nk, s.d), np.uint16)
    v = np.empty((L, s.B, s.H, s.Nk, s.d), np.uint16)

    def head(l, h):
        hrng = np.random.default_rng([seed, l, h])
        q[l, 0, h] = f32_to_bf16_bits(_normal(hrng, (s.Nq, s.d)))
        off = 0.5 * _normal(hrng, (s.P, 1, s.d))  # one mean offset per past chunk
        kh = _normal(hrng, (s.P + 1, s.Nq, s.d))
        kh[: s.P] += off
        k[l, 0, h] = f32_to_bf16_bits(kh.reshape(s.Nk, s.d))
        v[l, 0, h] = f32_to_bf16_bits(_normal(hrng, (s.Nk, s.d)))

    _parallel_heads(head, [(l, h) for l in range(L) for h in range(s.H)])
    past_poses = np.stack(poses[: s.P])
    past_intr = np.tile(intr, (s.P, 1))
    cams = np.stack([camera_record(p, intr) for p in poses[: s.P]])
    return Case(cfg=2, shape=s, seed=seed, q=q, k=k, v=v, cur_depth=depths[s.P][None],
                cur_cam=camera_record(poses[s.P], intr)[None], past_depth=depths[: s.P][None],
                past_poses=past_poses[None], past_intr=past_intr[None], past_cams=cams[None],
                slices_given=False)


def _loop(cfg: int, seed: int, s: Shape, heads: tuple | None = None,
          layer_ids: tuple | None = None) -> Case:
    """Room scene, looping trajectory (period 16), K of past chunk c shifted
    toward the head's query mean by the view-overlap proxy of chunk c.

    `heads` and `layer_ids` restrict which heads and layers are materialised;
    every (layer, head) has its own generator, so its values do not depend on
    the selection."""
    rng = np.random.default_rng(seed)
    scene = room_scene(rng)
    intr = intrinsics(s.Hp, s.Wp, s.fov_deg)
    poses, yaws = zip(*[loop_pose(n) for n in range(s.P + 1)])
    depths = np.stack([render_depth(scene, p, intr, s.Hp, s.Wp) for p in poses])
    ov = np.array([view_overlap_proxy(yaws[c], yaws[s.P], s.fov_deg) for c in range(s.P)],
                  dtype=np.float32)
    lsel = list(range(s.layers)) if layer_ids is None else list(layer_ids)
    hsel = list(range(s.H)) if heads is None else list(heads)
    q = np.empty((len(lsel), s.B, len(hsel), s.Nq, s.d), np.uint16)
    k = np.empty((len(lsel), s.B, len(hsel), s.Nk, s.d), np.uint16)
    v = np.empty((len(lsel), s.B, len(hsel), s.Nk, s.d), np.uint16)
    mus = {l: 0.5 * _normal(np.random.default_rng([seed, l]), (s.H, s.d)) for l in lsel}

    def head(li, l, i, h):
        hrng = np.random.default_rng([seed, l, h])
        mu = mus[l][h]
        q[li, 0, i] = f32_to_bf16_bits(_normal(hrng, (s.Nq, s.d)) + mu)
        kh = _normal(hrng, (s.P + 1, s.Nq, s.d))
        kh[: s.P] += ov[:, None, None] * mu[None, None, :]
        k[li, 0, i] = f32_to_bf16_bits(kh.reshape(s.Nk, s.d))
        v[li, 0, i] = f32_to_bf16_bits(_normal(hrng, (s.Nk, s.d)))

    _parallel_heads(head, [(li, l, i, h) for li, l in enumerate(lsel) for i, h in enumerate(hsel)])
    past_poses = np.stack(poses[: s.P])
    cams = np.stack([camera_record(p, intr) for p in poses[: s.P]])
    return Case(cfg=cfg, shape=s, seed=seed, q=q, k=k, v=v, cur_depth=depths[s.P][None],
                cur_cam=camera_record(poses[s.P], intr)[None], past_depth=depths[: s.P][None],
                past_poses=past_poses[None], past_intr=np.tile(intr, (s.P, 1))[None],
                past_cams=cams[None], slices_given=False,
                meta={"view_overlap": ov, "heads": hsel, "layers": lsel})


def stress_geometry(B: int, P: int, Hp: int, Wp: int, seed: int, fov_deg: float = 60.0,
                    past_grid: tuple = (32, 48)) -> dict:
    """B independent rooms (workload 3's scene generator, one seed per scene) seen
    along workload 3's camera loop: the current chunk (index P) has a depth map at
    Hp x Wp by ray cast; the P past chunks' depth maps are cast at the coarser
    `past_grid` (they only fix each slice's [min, max]); every camera's intrinsics
    are for the Hp x Wp grid. Returns float32 arrays cur_depth [B,Hp,Wp],
    cur_cam [B,18], past_depth [B,P,h,w], past_poses [B,P,12], past_intr [B,P,4]."""
    intr = intrinsics(Hp, Wp, fov_deg)
    intr_lr = intrinsics(past_grid[0], past_grid[1], fov_deg)
    poses = [loop_pose(n)[0] for n in range(P + 1)]
    out = {"cur_depth": np.empty((B, Hp, Wp), np.float32),
           "cur_cam": np.empty((B, CAM_FLOATS), np.float32),
           "past_depth": np.empty((B, P) + tuple(past_grid), np.float32),
           "past_poses": np.tile(np.stack(poses[:P]), (B, 1, 1)).astype(np.float32),
           "past_intr": np.tile(intr, (B, P, 1)).astype(np.float32)}

    def scene_job(b):
        scene = room_scene(np.random.default_rng([seed, b]))
        out["cur_depth"][b] = render_depth(scene, poses[P], intr, Hp, Wp)
        out["cur_cam"][b] = camera_record(poses[P], intr)
        for j in range(P):
            out["past_depth"][b, j] = render_depth(scene, poses[j], intr_lr, *past_grid)

    with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
        list(ex.map(scene_job, range(B)))
    return out


def perturb_depth(depth: np.ndarray, rng: np.random.Generator, noise_sd: float = 0.0,
                  hole_frac: float = 0.0, scale: float = 1.0) -> np.ndarray:
    """Depth-estimation error model for robustness studies (input generation,
    not a step of the method): a global scale bias, then per-pixel
    multiplicative Gaussian noise z * (1 + noise_sd * N(0,1)), then holes (NaN)
    at a random `hole_frac` of the pixels. Pixels that were invalid stay
    invalid; noise that drives a depth to <= 0 leaves it invalid as well."""
    d = np.asarray(depth, dtype=np.float64) * scale
    if noise_sd > 0:
        d = d * (1.0 + noise_sd * rng.standard_normal(d.shape))
    if hole_frac > 0:
        d[rng.random(d.shape) < hole_frac] = np.nan
    return d.astype(np.float32)


def make_case(cfg: int, seed: int | None = None, P: int | None = None, H: int | None = None,
              layers: int | None = None, heads: tuple | None = None, T: int | None = None,
              d: int | None = None, layer_ids: tuple | None = None) -> Case:
    """Build workload `cfg` (1..5). Default seed is 1000 + cfg. Workload 4 also
    takes another block size T or head dim d. For workloads 3-5, `heads` and
    `layer_ids` materialise only those heads and layers (q/k/v are then
    [len(layer_ids), B, len(heads), N, d])."""
    seed = 1000 + cfg if seed is None else seed
    if cfg == 1:
        return _tiny(seed)
    s = shape_for(cfg, P=P, H=H, layers=layers, T=T, d=d)
    if cfg == 2:
        return _walk(seed, s)
    return _loop(cfg, seed, s, heads=heads, layer_ids=layer_ids)


def geometry_only(cfg: int, seed: int | None = None, P: int | None = None):
    """Cameras and depth maps of workload `cfg` without Q/K/V (cheap)."""
    seed = 1000 + cfg if seed is None else seed
    s = shape_for(cfg, P=P, H=1, layers=1)
    s_small = Shape(**{**s.__dict__, "H": 1, "d": 8})
    if cfg == 1:
        c = _tiny(seed)
        return c
    c = _walk(seed, s_small) if cfg == 2 else _loop(cfg, seed, s_small, heads=())
    c.shape = s
    return c
