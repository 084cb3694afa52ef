"""Chunk-by-chunk rollout state for geometry-routed attention.

A chunked video world model generates one chunk at a time and denoises it in
several steps, each running every layer. Across that loop the routing inputs
change only at chunk boundaries: a finished chunk's keys, depth map and
frustum slice are fixed from then on ("Velox: Raumgedaechtnis beschleunigt
Video-Weltmodelle", section "Tiefenanalyse": each past chunk is a frustum
slice with a depth interval; the current chunk's depth is a recency-priority
warp of past depth; slice construction runs asynchronously to denoising).
`Rollout` keeps that state on the device and orders the library calls:

- a KV cache per layer with room for `capacity` chunks, chunk c in rows
  [c*Nq, (c+1)*Nq) of every head (owned by the caller; attention is given the
  whole capacity, the routed indices never point past the current chunk);
- the pooled-key cache per layer, appended once when a chunk is finished;
- one depth slot and one slice per chunk (a slice is rebuilt when its chunk's
  final depth arrives);
- the geometry of a chunk (multiwarp -> slices -> overlap counts) on a side
  stream.

Two geometry schedules:

- "boundary": chunk n's geometry is built when chunk n starts, from the final
  depth of chunks 0..n-1; only the first selection of the chunk waits for it
  (an event), the key scoring does not.
- "pipelined": chunk n+1's geometry is built while chunk n is denoised, so
  nothing waits at the boundary. Chunk n's final depth does not exist yet at
  that time, so its depth slot holds its own multiwarp estimate (the warped
  depth its routing uses); the final depth replaces it for every later chunk.

Orchestration only: every step runs in libvelox's kernels.
"""
from __future__ import annotations

import torch

from geometry_routed_block_b200 import velox as vx

SCHEDULES = ("boundary", "pipelined")


class Rollout:
    def __init__(self, k_caches, *, B: int, H: int, d: int, T: int, F: int, Hp: int, Wp: int,
                 capacity: int, cams: torch.Tensor, poses: torch.Tensor, intr: torch.Tensor,
                 alpha: float, topk_of, schedule: str = "pipelined", rel_tol: float = 0.01):
        """k_caches: per layer, K [B,H,capacity*Nq,d] (bf16 or f32).
        cams [N,18], poses [N,12], intr [N,4] float32 on the device: every chunk's
        camera (N >= capacity + 1 for the pipelined schedule's last look-ahead).
        topk_of(n): kept key blocks (current chunk included) with n past chunks."""
        if schedule not in SCHEDULES:
            raise ValueError(f"schedule must be one of {SCHEDULES}")
        if B != 1:
            raise ValueError("one camera trajectory per rollout (B = 1)")
        self.k = list(k_caches)
        self.B, self.H, self.d, self.T, self.F, self.Hp, self.Wp = B, H, d, T, F, Hp, Wp
        self.Nq = F * Hp * Wp
        self.m = self.Nq // T
        self.capacity = capacity
        self.cams, self.poses, self.intr = cams, poses, intr
        self.alpha, self.topk_of, self.schedule, self.rel_tol = alpha, topk_of, schedule, rel_tol
        dev = cams.device
        n_geo = cams.shape[0]
        self.depth = torch.full((n_geo, Hp, Wp), float("nan"), dtype=torch.float32, device=dev)
        self.slices = torch.zeros((n_geo, vx.CAM_FLOATS), dtype=torch.float32, device=dev)
        self.cur_depth = torch.full((n_geo, 1, Hp, Wp), float("nan"), dtype=torch.float32,
                                    device=dev)
        self.kbar = [vx.kbar_cache(B, H, capacity, self.Nq, d, T, dev) for _ in self.k]
        self.mw_ws = vx.depth_multiwarp_workspace(Hp, Wp, dev)
        self.ws = vx.route_workspace(B, H, self.Nq, capacity * self.Nq, d, T, dev)
        self.counts = {}
        self.side = torch.cuda.Stream(device=dev)
        self.geo_ready = {}
        self.n = None

    # ------------------------------------------------------------ geometry
    def _counts_buf(self, n: int) -> torch.Tensor:
        if n not in self.counts:
            self.counts[n] = torch.empty((self.B, self.m, n), dtype=torch.int32,
                                         device=self.cams.device)
        return self.counts[n]

    def _slice(self, c: int, stream) -> None:
        vx.slices_build(self.depth[c:c + 1], self.poses[c:c + 1], self.intr[c:c + 1],
                        out=self.slices[c:c + 1], stream=stream)

    def _geometry(self, n: int, stream, rebuild=()) -> torch.cuda.Event:
        """Counts of chunk n against past chunks 0..n-1 from the depth slots as
        they stand; the slices listed in `rebuild` are built first."""
        for c in rebuild:
            self._slice(c, stream)
        vx.depth_multiwarp(self.depth[:n], self.cams[:n], self.cams[n], self.rel_tol,
                           ws=self.mw_ws, out=self.cur_depth[n, 0], stream=stream)
        vx.block_overlap(self.cur_depth[n], self.cams[n:n + 1], self.slices[:n][None], self.F,
                         self.T, out=self._counts_buf(n), stream=stream)
        ev = torch.cuda.Event()
        ev.record(stream)
        return ev

    def prefill(self, n0: int, final_depth: torch.Tensor) -> None:
        """Chunks 0..n0-1 are finished: final_depth [n0,Hp,Wp]; their keys are in
        the KV caches. Pools their keys, builds their slices and, for the
        pipelined schedule, chunk n0's geometry."""
        main = torch.cuda.current_stream()
        self.depth[:n0].copy_(final_depth)
        vx.slices_build(self.depth[:n0], self.poses[:n0], self.intr[:n0], out=self.slices[:n0])
        for layer, k in enumerate(self.k):
            for c in range(n0):
                vx.kbar_append(k, self.Nq, self.T, c, self.kbar[layer])
        self.start(n0)

    def start(self, n0: int) -> None:
        """(Re)starts the rollout at chunk n0, chunks 0..n0-1 final. The
        pipelined schedule builds chunk n0's geometry here, as chunk n0-1's
        look-ahead would have."""
        self.side.wait_stream(torch.cuda.current_stream())
        self.geo_ready = {}
        if self.schedule == "pipelined":
            self.geo_ready[n0] = self._geometry(n0, self.side)
        self.n = None

    def begin_chunk(self, n: int) -> None:
        """Chunk n starts (n past chunks). Enqueues the side-stream geometry."""
        if n + 1 > self.capacity:
            raise ValueError("KV cache capacity exceeded")
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)  # depth slots / slices written on the main stream
        if self.schedule == "boundary":
            self.geo_ready[n] = self._geometry(n, self.side, rebuild=(n - 1,))
        else:
            if n not in self.geo_ready:
                raise RuntimeError(f"chunk {n}'s geometry was not built ahead")
            if n + 1 < self.cams.shape[0]:
                # chunk n-1's slot holds its final depth now; chunk n's slot gets
                # chunk n's own warped depth, the best estimate before it is done
                with torch.cuda.stream(self.side):
                    self.depth[n].copy_(self.cur_depth[n, 0])
                self.geo_ready[n + 1] = self._geometry(n + 1, self.side, rebuild=(n - 1, n))
        self.n = n
        self._first_route = True

    def route(self, layer: int, q: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """Routed key blocks of the current chunk for `layer` (pooled-key cache +
        this chunk's counts). The chunk's first selection waits for its
        geometry; the key scoring before it does not."""
        n = self.n
        ev = self.geo_ready[n] if self._first_route else None
        self._first_route = False
        return vx.route_topk_cached(q, self.kbar[layer], n, self.counts[n], self.alpha,
                                    self.topk_of(n), self.T, ws=self.ws, out=out, counts_ready=ev)

    def attend(self, layer: int, q: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
               out: torch.Tensor | None = None, status: torch.Tensor | None = None):
        """Block-sparse attention of the current chunk over the whole KV cache."""
        return vx.sparse_attn_fwd(q, self.k[layer], v, idx, self.T, out=out, want_lse=False,
                                  status=status)

    def end_chunk(self, n: int, final_depth: torch.Tensor) -> None:
        """Chunk n is finished: its keys (rows of chunk n in every layer's KV
        cache) are pooled into the caches and its final depth [Hp,Wp] is kept."""
        main = torch.cuda.current_stream()
        for layer, k in enumerate(self.k):
            vx.kbar_append(k, self.Nq, self.T, n, self.kbar[layer])
        # the side stream may still read chunk n's slot (its estimate)
        main.wait_stream(self.side)
        self.depth[n].copy_(final_depth)
        self.n = None
