"""ctypes binding of libvelox (include/velox.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch supplies device memory (output and scratch tensors are
allocated here with torch) and the current CUDA stream. Importing this module
fails loudly when libvelox.so has not been built; there is no fallback.

Camera / slice records are float32 tensors whose last dimension is 18, laid out
like velox_slice_t: R (9, row-major, world->camera), t (3), fx, fy, cx, cy,
znear, zfar.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvelox.so")

VELOX_OK = 0
VELOX_EINVAL = -1
VELOX_EUNSUPPORTED = -2
VELOX_ECUDA = -3
VELOX_ETIMEOUT = -4
VELOX_EBOUNDS = -5
VELOX_STATUS_BAD_INDEX = 1
VELOX_STATUS_TIMEOUT = 2
VELOX_TEST_SKIP_MMA = 1
VELOX_TEST_FORCE_PAIR = 2
VELOX_BF16 = 0
VELOX_F32 = 1
CAM_FLOATS = 18

_c_int, _c_size, _vp, _c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float

# name -> (restype, argtypes); mirrors include/velox.h
SIGNATURES = {
    "velox_version": (_c_int, []),
    "velox_strerror": (ctypes.c_char_p, [_c_int]),
    "velox_slices_build": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp]),
    "velox_block_overlap": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                     _vp, _vp]),
    "velox_route_topk_workspace_size": (_c_size, [_c_int] * 6),
    "velox_route_topk": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _vp, _c_float, _c_int, _vp, _vp, _c_size, _vp, _vp]),
    "velox_sparse_attn_fwd": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                       _c_int, _c_int, _c_float, _vp, _vp, _vp, _vp]),
    "velox_sparse_attn_fwd_test": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                            _c_int, _c_int, _c_int, _c_float, _vp, _vp, _vp,
                                            ctypes.c_double, _c_int, _vp]),
    "velox_depth_multiwarp_workspace_size": (_c_size, [_c_int, _c_int]),
    "velox_depth_multiwarp": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_float, _vp, _vp,
                                       _c_size, _vp]),
    "velox_cast_bf16": (_c_int, [_vp, _vp, _c_size, _vp]),
    "velox_depth_multiwarp_noalloc": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_float,
                                               _vp, _vp]),
    "velox_fp64_fma_bench": (_c_int, [_vp, _c_int, _c_int, _c_int, _vp]),
    "velox_kbar_cache_bytes": (_c_size, [_c_int] * 6),
    "velox_kbar_append": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _vp, _c_int, _vp]),
    "velox_route_topk_cached": (_c_int, [_vp, _c_int, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                         _c_int, _c_int, _vp, _c_float, _c_int, _vp, _vp, _c_size,
                                         _vp, _vp]),
}


class VeloxError(RuntimeError):
    def __init__(self, what: str, code: int):
        super().__init__(f"{what} failed: {strerror(code)} ({code})")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libvelox.so not found at {path}; build it with `python -m geometry_routed_block_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load_library()


def strerror(code: int) -> str:
    return lib.velox_strerror(code).decode()


def _check(code: int, what: str) -> None:
    if code != VELOX_OK:
        raise VeloxError(what, code)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libvelox takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libvelox takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream: torch.cuda.Stream | None = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


# ---------------------------------------------------------------- geometry

def slices_build(depth: torch.Tensor, poses: torch.Tensor, intr: torch.Tensor,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """depth [P,Hp,Wp] f32, poses [P,12] f32, intr [P,4] f32 -> slices [P,18] f32."""
    P, Hp, Wp = depth.shape
    for t, n in ((depth, "depth"), (poses, "poses"), (intr, "intr")):
        _expect(t, torch.float32, n)
    if out is None:
        out = torch.empty((P, CAM_FLOATS), dtype=torch.float32, device=depth.device)
    _check(lib.velox_slices_build(_ptr(depth), _ptr(poses), _ptr(intr), P, Hp, Wp, _ptr(out),
                                  _stream(stream)), "velox_slices_build")
    return out


def block_overlap(cur_depth: torch.Tensor, cur_cam: torch.Tensor, slices: torch.Tensor, F: int,
                  T: int, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """cur_depth [B,Hp,Wp] f32, cur_cam [B,18], slices [B,P,18] -> counts [B,m,P] int32."""
    B, Hp, Wp = cur_depth.shape
    P = slices.shape[1]
    m = F * Hp * Wp // T
    for t, n in ((cur_depth, "cur_depth"), (cur_cam, "cur_cam"), (slices, "slices")):
        _expect(t, torch.float32, n)
    if out is None:
        out = torch.empty((B, m, P), dtype=torch.int32, device=cur_depth.device)
    _check(lib.velox_block_overlap(_ptr(cur_depth), _ptr(cur_cam), _ptr(slices), B, P, F, Hp, Wp, T,
                                   _ptr(out), _stream(stream)), "velox_block_overlap")
    return out


def depth_multiwarp_workspace(Hp: int, Wp: int, device="cuda") -> torch.Tensor:
    n = lib.velox_depth_multiwarp_workspace_size(Hp, Wp)
    return torch.empty(n, dtype=torch.uint8, device=device)


def depth_multiwarp(past_depth: torch.Tensor, past_cams: torch.Tensor, cur_cam: torch.Tensor,
                    rel_tol: float = 0.01, ws: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """past_depth [P,Hp,Wp] f32, past_cams [P,18], cur_cam [18] -> current depth [Hp,Wp] f32."""
    P, Hp, Wp = past_depth.shape
    if ws is None:
        ws = depth_multiwarp_workspace(Hp, Wp, past_depth.device)
    if out is None:
        out = torch.empty((Hp, Wp), dtype=torch.float32, device=past_depth.device)
    _check(lib.velox_depth_multiwarp(_ptr(past_depth), _ptr(past_cams), _ptr(cur_cam), P, Hp, Wp,
                                     float(rel_tol), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "velox_depth_multiwarp")
    return out


# ---------------------------------------------------------------- routing

def route_workspace(B: int, H: int, Nq: int, Nk: int, d: int, T: int, device="cuda") -> torch.Tensor:
    n = lib.velox_route_topk_workspace_size(B, H, Nq, Nk, d, T)
    if n == 0:
        raise VeloxError("velox_route_topk_workspace_size", VELOX_EINVAL)
    return torch.empty(n, dtype=torch.uint8, device=device)


def route_topk(q: torch.Tensor, k: torch.Tensor, counts: torch.Tensor | None, alpha: float,
               topk: int, T: int, ws: torch.Tensor | None = None, out: torch.Tensor | None = None,
               counts_ready: torch.cuda.Event | None = None, stream=None) -> torch.Tensor:
    """q [B,H,Nq,d], k [B,H,Nk,d] (bf16 or f32), counts [B,m,P] int32 or None ->
    idx [B,H,m,topk] int32 (ascending key-block indices). With `counts_ready`,
    only the selection kernel waits for that event (the counts' producer may
    still be running on another stream while the keys are pooled)."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    if q.dtype != k.dtype:
        raise TypeError("q and k must share a dtype")
    dtype = {torch.bfloat16: VELOX_BF16, torch.float32: VELOX_F32}.get(q.dtype)
    if dtype is None:
        raise TypeError(f"unsupported dtype {q.dtype}")
    if counts is not None:
        _expect(counts, torch.int32, "counts")
    if ws is None:
        ws = route_workspace(B, H, Nq, Nk, d, T, q.device)
    if out is None:
        out = torch.empty((B, H, Nq // T, topk), dtype=torch.int32, device=q.device)
    ev = ctypes.c_void_p(counts_ready.cuda_event) if counts_ready is not None else None
    _check(lib.velox_route_topk(_ptr(q), _ptr(k), dtype, B, H, Nq, Nk, d, T, _ptr(counts),
                                float(alpha), int(topk), _ptr(out), _ptr(ws), ws.numel(), ev,
                                _stream(stream)), "velox_route_topk")
    return out


# ---------------------------------------------------------------- pooled-key cache

def kbar_cache(B: int, H: int, max_past_chunks: int, Nq: int, d: int, T: int,
               device="cuda") -> torch.Tensor:
    """An empty pooled-key cache [B, H, max_past_chunks * Nq/T, d] float32."""
    if lib.velox_kbar_cache_bytes(B, H, max_past_chunks, Nq, d, T) == 0:
        raise VeloxError("velox_kbar_cache_bytes", VELOX_EINVAL)
    return torch.empty((B, H, max_past_chunks * (Nq // T), d), dtype=torch.float32, device=device)


def kbar_append(k: torch.Tensor, Nq: int, T: int, chunk: int, kbar: torch.Tensor,
                stream=None) -> torch.Tensor:
    """Pools chunk `chunk` of the KV cache k [B,H,Nk,d] into kbar."""
    B, H, Nk, d = k.shape
    dtype = {torch.bfloat16: VELOX_BF16, torch.float32: VELOX_F32}.get(k.dtype)
    if dtype is None:
        raise TypeError(f"unsupported dtype {k.dtype}")
    _expect(kbar, torch.float32, "kbar")
    max_chunks = kbar.shape[2] // (Nq // T)
    _check(lib.velox_kbar_append(_ptr(k), dtype, B, H, Nk, Nq, d, T, int(chunk), _ptr(kbar),
                                 max_chunks, _stream(stream)), "velox_kbar_append")
    return kbar


def route_topk_cached(q: torch.Tensor, kbar: torch.Tensor, P: int, counts: torch.Tensor | None,
                      alpha: float, topk: int, T: int, ws: torch.Tensor | None = None,
                      out: torch.Tensor | None = None, counts_ready: torch.cuda.Event | None = None,
                      stream=None) -> torch.Tensor:
    """route_topk over P past chunks whose pooled keys are in kbar."""
    B, H, Nq, d = q.shape
    dtype = {torch.bfloat16: VELOX_BF16, torch.float32: VELOX_F32}.get(q.dtype)
    if dtype is None:
        raise TypeError(f"unsupported dtype {q.dtype}")
    _expect(kbar, torch.float32, "kbar")
    if counts is not None:
        _expect(counts, torch.int32, "counts")
    max_chunks = kbar.shape[2] // (Nq // T)
    if ws is None:
        ws = route_workspace(B, H, Nq, (P + 1) * Nq, d, T, q.device)
    if out is None:
        out = torch.empty((B, H, Nq // T, topk), dtype=torch.int32, device=q.device)
    ev = ctypes.c_void_p(counts_ready.cuda_event) if counts_ready is not None else None
    _check(lib.velox_route_topk_cached(_ptr(q), dtype, _ptr(kbar), max_chunks, B, H, Nq, int(P), d,
                                       T, _ptr(counts), float(alpha), int(topk), _ptr(out),
                                       _ptr(ws), ws.numel(), ev, _stream(stream)),
           "velox_route_topk_cached")
    return out


# ---------------------------------------------------------------- attention

def sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor | None,
                    T: int, scale: float | None = None, want_lse: bool = True,
                    status: torch.Tensor | None = None, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, stream=None):
    """q [B,H,Nq,d], k/v [B,H,Nk,d] bf16, idx [B,H,m,topk] int32 or None (dense)
    -> (O [B,H,Nq,d] bf16, lse [B,H,Nq] f32 or None)."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _expect(t, torch.bfloat16, n)
    topk = 0
    if idx is not None:
        _expect(idx, torch.int32, "idx")
        topk = idx.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    if not want_lse:
        lse = None
    if status is not None:
        _expect(status, torch.int32, "status")
    _check(lib.velox_sparse_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), topk, B, H, Nq, Nk, d,
                                     T, float(scale), _ptr(out), _ptr(lse), _ptr(status),
                                     _stream(stream)), "velox_sparse_attn_fwd")
    return out, lse


def sparse_attn_fwd_test(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         idx: torch.Tensor | None, T: int, status: torch.Tensor,
                         wait_limit_s: float, flags: int, out: torch.Tensor | None = None,
                         lse: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """sparse_attn_fwd through the test entry point (bounded-wait limit and
    test-hook flags); returns O (unwritten when the waits ran out). An `lse`
    tensor [B,H,Nq] f32, when given, receives the log-sum-exp."""
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _expect(t, torch.bfloat16, n)
    _expect(status, torch.int32, "status")
    topk = 0
    if idx is not None:
        _expect(idx, torch.int32, "idx")
        topk = idx.shape[-1]
    if out is None:
        out = torch.empty_like(q)
    _check(lib.velox_sparse_attn_fwd_test(_ptr(q), _ptr(k), _ptr(v), _ptr(idx), topk, B, H, Nq, Nk,
                                          d, T, float(1.0 / math.sqrt(d)), _ptr(out), _ptr(lse),
                                          _ptr(status), float(wait_limit_s), int(flags),
                                          _stream(stream)), "velox_sparse_attn_fwd_test")
    return out


def fp64_fma_bench(out: torch.Tensor, blocks: int, threads: int, iters: int, stream=None) -> int:
    """Launches the float64 FMA throughput kernel; returns its FLOP count."""
    _expect(out, torch.float64, "out")
    _check(lib.velox_fp64_fma_bench(_ptr(out), int(blocks), int(threads), int(iters),
                                    _stream(stream)), "velox_fp64_fma_bench")
    return 16 * int(blocks) * int(threads) * int(iters)


def cast_bf16(x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """float32 -> bf16 (round to nearest even) on the device."""
    _expect(x, torch.float32, "x")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _check(lib.velox_cast_bf16(_ptr(x), _ptr(out), x.numel(), _stream(stream)), "velox_cast_bf16")
    return out


def depth_multiwarp_noalloc(past_depth: torch.Tensor, past_cams: torch.Tensor,
                            cur_cam: torch.Tensor, rel_tol: float = 0.01,
                            out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """depth_multiwarp with the library's fixed scratch instead of a caller
    workspace (grids up to 65536 pixels; concurrent calls race)."""
    P, Hp, Wp = past_depth.shape
    if out is None:
        out = torch.empty((Hp, Wp), dtype=torch.float32, device=past_depth.device)
    _check(lib.velox_depth_multiwarp_noalloc(_ptr(past_depth), _ptr(past_cams), _ptr(cur_cam), P,
                                             Hp, Wp, float(rel_tol), _ptr(out), _stream(stream)),
           "velox_depth_multiwarp_noalloc")
    return out
