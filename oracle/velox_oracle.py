"""CPU oracle for the Velox geometry-routed block-sparse attention path (fp64).

TEST INFRASTRUCTURE ONLY. This module is imported by tests/, by
__graft_entry__.smoke() and by bench.py's cpu_baseline leg, and by nothing on the
product path. It shares no code with the CUDA library: it reads plain numpy
arrays (float32 inputs, bf16 inputs as uint16 bit patterns) and computes every
step in float64 with numpy, one elementwise operation at a time, so that a
reader can check each line against the method.

Sources (pages on the Velox method; they give the structure of the method but
no formula, constant or kernel):
  [DE] "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
       "Tiefenanalyse" -- four steps: (1) every past chunk is a camera-frustum
       slice with a depth interval; (2) the current chunk's depth comes from a
       recency-priority multiwarp of past depth; (3) slice overlap softly
       modulates the block importance the model computes in each layer
       (modulation, not replacement); (4) regions no history covers get no
       geometric bias. Routing granularity = token block = attention tile.
  [KO] "Velox: 공간 메모리로 비디오 월드 모델 추론 가속", sections "배경" (region-level
       context selection over a KV cache that grows per chunk) and "심층 분석"
       (same four steps; the kernel really skips unneeded blocks).

Where the pages are silent the oracle takes the plainest reading:
  * modulation: s' = s + alpha * overlap on covered query blocks, overlap =
    count / T, covered = at least one point of the block inside some past slice;
  * block importance s = mean-pooled Q block . mean-pooled K block / sqrt(d),
    per (batch, head);
  * top-k counts the always-kept current-chunk blocks (k_past = k - m), ties go
    to the smaller key-block index, indices are emitted ascending;
  * depth interval of a past chunk = [min, max] of its valid depth;
  * cameras: world->camera [R|t], OpenCV axes, z-depth, pixel centres at +0.5;
  * multiwarp: nearest-pixel splat (floor of the projected coordinate); per
    target pixel the most recent chunk among candidates within (1 + rel_tol)
    of the nearest depth wins, at its smallest depth; holes are NaN.

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------

def widen(x: np.ndarray) -> np.ndarray:
    """float32 -> float64 exactly; uint16 arrays are bf16 bit patterns."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(F64)
    return np.asarray(x, dtype=np.float32).astype(F64)


class Camera:
    """Camera record float32[18] = R[9] (row-major, world->camera), t[3],
    fx, fy, cx, cy, znear, zfar -- every field widened to float64."""

    def __init__(self, rec: np.ndarray):
        r = np.asarray(rec, dtype=np.float32).astype(F64)
        self.R = r[0:9].reshape(3, 3)
        self.t = r[9:12]
        self.fx, self.fy, self.cx, self.cy = r[12], r[13], r[14], r[15]
        self.znear, self.zfar = r[16], r[17]


def valid_depth(z: np.ndarray) -> np.ndarray:
    """A depth sample is usable when it is finite and positive."""
    return np.isfinite(z) & (z > 0)


# ----------------------------------------------------------------------------
# pinhole geometry ([DE] Tiefenanalyse, steps 1-2)
# ----------------------------------------------------------------------------

def backproject(r: np.ndarray, c: np.ndarray, z: np.ndarray, cam: Camera):
    """Pixel (row r, column c) at z-depth z -> world point, via
    p_c = ((u-cx)/fx*z, (v-cy)/fy*z, z) with u = c+0.5, v = r+0.5, and
    p_w = R^T (p_c - t), each row summed left to right."""
    u = c.astype(F64) + 0.5
    v = r.astype(F64) + 0.5
    xc = ((u - cam.cx) / cam.fx) * z
    yc = ((v - cam.cy) / cam.fy) * z
    zc = z
    dx = xc - cam.t[0]
    dy = yc - cam.t[1]
    dz = zc - cam.t[2]
    R = cam.R
    xw = (R[0, 0] * dx + R[1, 0] * dy) + R[2, 0] * dz
    yw = (R[0, 1] * dx + R[1, 1] * dy) + R[2, 1] * dz
    zw = (R[0, 2] * dx + R[1, 2] * dy) + R[2, 2] * dz
    return xw, yw, zw


def to_camera(xw, yw, zw, cam: Camera):
    """World point -> camera coordinates q = R p_w + t, each row left to right."""
    R, t = cam.R, cam.t
    qx = ((R[0, 0] * xw + R[0, 1] * yw) + R[0, 2] * zw) + t[0]
    qy = ((R[1, 0] * xw + R[1, 1] * yw) + R[1, 2] * zw) + t[1]
    qz = ((R[2, 0] * xw + R[2, 1] * yw) + R[2, 2] * zw) + t[2]
    return qx, qy, qz


def image_coords(qx, qy, qz, cam: Camera):
    """Continuous pixel coordinates u = fx*(qx/qz)+cx, v = fy*(qy/qz)+cy."""
    with np.errstate(divide="ignore", invalid="ignore"):
        uu = cam.fx * (qx / qz) + cam.cx
        vv = cam.fy * (qy / qz) + cam.cy
    return uu, vv


# ----------------------------------------------------------------------------
# step 1: frustum slices with a depth interval
# ----------------------------------------------------------------------------

def slices_build(depth: np.ndarray, poses: np.ndarray, intr: np.ndarray) -> np.ndarray:
    """Past chunk j -> slice record (pose, intrinsics, [near_j, far_j]) with
    near/far = min/max of the chunk's valid depth; no valid pixel -> the
    empty interval [+inf, -inf]. depth [P,Hp,Wp] f32, poses [P,12], intr [P,4]."""
    P = depth.shape[0]
    out = np.zeros((P, 18), dtype=np.float32)
    for j in range(P):
        z = depth[j].reshape(-1)
        ok = valid_depth(z)
        if ok.any():
            near, far = z[ok].min(), z[ok].max()
        else:
            near, far = np.float32(np.inf), np.float32(-np.inf)
        out[j, 0:12] = poses[j]
        out[j, 12:16] = intr[j]
        out[j, 16] = near
        out[j, 17] = far
    return out


# ----------------------------------------------------------------------------
# step 3 (geometry half): per (query block, past slice) overlap counts
# ----------------------------------------------------------------------------

def token_pixels(Nq: int, Hp: int, Wp: int):
    """Token tau of the current chunk -> (frame, row, col) in raster order."""
    tau = np.arange(Nq)
    f = tau // (Hp * Wp)
    rem = tau % (Hp * Wp)
    return f, rem // Wp, rem % Wp


def inside_slice(xw, yw, zw, cam: Camera, Hp: int, Wp: int) -> np.ndarray:
    """A world point is inside slice j when, in camera j, near <= z <= far,
    z > 0 and its projection falls in [0, Wp) x [0, Hp)."""
    qx, qy, qz = to_camera(xw, yw, zw, cam)
    front = qz > 0
    uu, vv = image_coords(qx, qy, qz, cam)
    with np.errstate(invalid="ignore"):
        ok = (qz >= cam.znear) & (qz <= cam.zfar) & front
        ok &= (uu >= 0) & (uu < Wp) & (vv >= 0) & (vv < Hp)
    return ok


def block_overlap(cur_depth: np.ndarray, cur_cam: np.ndarray, slices: np.ndarray,
                  F: int, T: int) -> np.ndarray:
    """counts[b, qb, j] = number of the T points of query block qb (pixel
    centres back-projected with the current depth and camera) that lie inside
    past slice j. Invalid depth (NaN, inf, <= 0) counts as outside.
    cur_depth [B,Hp,Wp] f32, cur_cam [B,18], slices [B,P,18] -> int32 [B,m,P]."""
    B, Hp, Wp = cur_depth.shape
    P = slices.shape[1]
    Nq = F * Hp * Wp
    m = Nq // T
    _, r, c = token_pixels(Nq, Hp, Wp)
    out = np.zeros((B, m, P), dtype=np.int32)
    for b in range(B):
        cam = Camera(cur_cam[b])
        z = cur_depth[b].astype(F64)[r, c]
        ok_z = valid_depth(z)
        zz = np.where(ok_z, z, 1.0)
        xw, yw, zw = backproject(r, c, zz, cam)
        for j in range(P):
            inside = inside_slice(xw, yw, zw, Camera(slices[b, j]), Hp, Wp) & ok_z
            out[b, :, j] = inside.reshape(m, T).sum(axis=1)
    return out


# ----------------------------------------------------------------------------
# step 3 (model half): block importance, modulation, selection
# ----------------------------------------------------------------------------

def pool_blocks(x: np.ndarray, T: int) -> np.ndarray:
    """Mean over each run of T consecutive tokens: [..., N, d] -> [..., N/T, d]."""
    x = widen(x)
    sh = x.shape
    return x.reshape(sh[:-2] + (sh[-2] // T, T, sh[-1])).mean(axis=-2)


def block_scores(q: np.ndarray, k: np.ndarray, T: int) -> np.ndarray:
    """s[b,h,qb,kb] = qbar[qb] . kbar[kb] / sqrt(d) over PAST key blocks only
    (the current chunk's blocks are always kept and never scored).
    q [B,H,Nq,d], k [B,H,Nk,d] -> [B,H,m,P*m]."""
    Nq, d = q.shape[-2], q.shape[-1]
    Nk = k.shape[-2]
    n_past = (Nk - Nq) // T
    qbar = pool_blocks(q, T)
    kbar = pool_blocks(k[..., : n_past * T, :], T)
    s = np.einsum("bhqd,bhkd->bhqk", qbar, kbar)
    return s / np.sqrt(F64(d))


def modulate(s: np.ndarray, counts: np.ndarray | None, alpha: float, T: int) -> np.ndarray:
    """s'[b,h,qb,kb] = s + alpha * counts[b,qb,chunk(kb)] / T on covered query
    blocks (at least one point inside some slice), s' = s elsewhere.
    chunk(kb) = kb // m. counts None means no geometry: s' = s."""
    out = s.copy()
    if counts is None:
        return out
    B, H, m, n_past = s.shape
    chunk = np.arange(n_past) // m
    for b in range(B):
        for qb in range(m):
            if counts[b, qb].sum() > 0:
                overlap = counts[b, qb, chunk].astype(F64) / T
                out[b, :, qb, :] = s[b, :, qb, :] + F64(alpha) * overlap[None, :]
    return out


def select_topk(s_mod: np.ndarray, topk: int, m: int) -> np.ndarray:
    """Per query block: all m current-chunk blocks plus the topk - m past blocks
    with the largest s' (equal s': smaller index first); ascending indices.
    s_mod [B,H,m,n_past] -> int32 [B,H,m,topk]."""
    B, H, mq, n_past = s_mod.shape
    n_kb = n_past + m
    if topk < m or topk > n_kb:
        raise ValueError("topk must lie in [m, number of key blocks]")
    k_past = topk - m
    cur = np.arange(n_past, n_kb)
    out = np.zeros((B, H, mq, topk), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(mq):
                row = s_mod[b, h, qb]
                order = np.lexsort((np.arange(n_past), -row))  # by -s', then index
                chosen = np.sort(order[:k_past])
                out[b, h, qb] = np.concatenate([chosen, cur])
    return out


def route_topk(q, k, counts, alpha: float, topk: int, T: int):
    """Full routing: returns (idx [B,H,m,topk] int32, s' [B,H,m,n_past] fp64)."""
    Nq = q.shape[-2]
    s = block_scores(q, k, T)
    s_mod = modulate(s, counts, alpha, T)
    return select_topk(s_mod, topk, Nq // T), s_mod


# ----------------------------------------------------------------------------
# step 4 (kernel): attention restricted to the routed blocks
# ----------------------------------------------------------------------------

def sparse_attention(q, k, v, idx, T: int, scale: float | None = None, rows=None):
    """For query block qb of (b,h): keys/values = the T-token blocks listed in
    idx[b,h,qb] (all blocks when idx is None); O = softmax(Q K^T * scale) V with
    the softmax taken in fp64 after subtracting the row max; lse = natural log
    of the row's sum of exponentials (of the scaled scores).
    rows: optional list of (b,h,qb) to compute; returns dict {(b,h,qb): (O, lse)}
    when given, else full arrays O [B,H,Nq,d], lse [B,H,Nq]."""
    B, H, Nq, d = q.shape
    Nk = k.shape[-2]
    scale = 1.0 / np.sqrt(F64(d)) if scale is None else F64(scale)
    m = Nq // T
    all_blocks = np.arange(Nk // T)

    def one(b, h, qb):
        blocks = all_blocks if idx is None else np.asarray(idx[b, h, qb])
        keys = (blocks[:, None] * T + np.arange(T)[None, :]).reshape(-1)
        Q = widen(q[b, h, qb * T:(qb + 1) * T])
        K = widen(k[b, h, keys])
        V = widen(v[b, h, keys])
        S = (Q @ K.T) * scale
        mx = S.max(axis=1, keepdims=True)
        p = np.exp(S - mx)
        l = p.sum(axis=1, keepdims=True)
        O = (p @ V) / l
        lse = mx[:, 0] + np.log(l[:, 0])
        return O, lse

    if rows is not None:
        return {tuple(r): one(*r) for r in rows}
    O = np.zeros((B, H, Nq, d), dtype=F64)
    L = np.zeros((B, H, Nq), dtype=F64)
    for b in range(B):
        for h in range(H):
            for qb in range(m):
                o, l = one(b, h, qb)
                O[b, h, qb * T:(qb + 1) * T] = o
                L[b, h, qb * T:(qb + 1) * T] = l
    return O, L


# ----------------------------------------------------------------------------
# step 2: recency-priority multiwarp of past depth into the current view
# ----------------------------------------------------------------------------

def multiwarp_candidates(past_depth, past_cams, cur_cam):
    """Every valid pixel of every past depth map, back-projected with its own
    camera and moved into the current camera. Returns (target pixel index,
    chunk j, depth z in the current camera) for points in front of the camera
    whose projection lands on the grid; target = floor of the projection."""
    P, Hp, Wp = past_depth.shape
    cur = Camera(cur_cam)
    rr, cc = np.meshgrid(np.arange(Hp), np.arange(Wp), indexing="ij")
    rr, cc = rr.reshape(-1), cc.reshape(-1)
    tgt, chunk, zs = [], [], []
    for j in range(P):
        z = past_depth[j].astype(F64).reshape(-1)
        ok = valid_depth(z)
        xw, yw, zw = backproject(rr[ok], cc[ok], z[ok], Camera(past_cams[j]))
        qx, qy, qz = to_camera(xw, yw, zw, cur)
        uu, vv = image_coords(qx, qy, qz, cur)
        with np.errstate(invalid="ignore"):
            keep = (qz > 0) & (uu >= 0) & (uu < Wp) & (vv >= 0) & (vv < Hp)
        tr = np.floor(vv[keep]).astype(np.int64)
        tc = np.floor(uu[keep]).astype(np.int64)
        tgt.append(tr * Wp + tc)
        chunk.append(np.full(tr.shape, j, dtype=np.int64))
        zs.append(qz[keep])
    return np.concatenate(tgt), np.concatenate(chunk), np.concatenate(zs)


def depth_multiwarp(past_depth, past_cams, cur_cam, rel_tol: float = 0.01) -> np.ndarray:
    """Current depth [Hp,Wp] float32: per target pixel, among its candidates,
    z_min = nearest depth; winners = candidates with z <= z_min * (1 + rel_tol)
    (rel_tol widened from float32); the most recent winning chunk (largest j)
    is taken at its smallest depth; no candidate -> NaN."""
    P, Hp, Wp = past_depth.shape
    tgt, chunk, zs = multiwarp_candidates(past_depth, past_cams, cur_cam)
    factor = 1.0 + F64(np.float32(rel_tol))
    out = np.full(Hp * Wp, np.nan, dtype=np.float32)
    per_pixel: dict[int, list] = {}
    for p, j, z in zip(tgt.tolist(), chunk.tolist(), zs.tolist()):
        per_pixel.setdefault(p, []).append((j, z))
    for p, cands in per_pixel.items():
        zmin = min(z for _, z in cands)
        thr = zmin * factor
        jwin = max(j for j, z in cands if z <= thr)
        out[p] = np.float32(min(z for j, z in cands if j == jwin))
    return out.reshape(Hp, Wp)
