"""The C ABI: libvelox.so builds, loads, exports every function include/velox.h
declares, and rejects bad arguments before launching anything. CPU only: the
rejected calls return before touching the CUDA runtime."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "velox.h")


@pytest.fixture(scope="module")
def lib():
    from geometry_routed_block_b200 import build
    build.build()
    from geometry_routed_block_b200 import velox
    return velox.lib


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VELOX_API\s+[\w\s\*]+?\b(velox_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for want in ("velox_slices_build", "velox_block_overlap", "velox_route_topk",
                 "velox_sparse_attn_fwd", "velox_depth_multiwarp"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol(lib):
    from geometry_routed_block_b200 import velox
    assert set(declared_functions()) <= set(velox.SIGNATURES)


def test_version_and_strerror(lib):
    assert lib.velox_version() >= 100
    assert lib.velox_strerror(0) == b"ok"
    assert lib.velox_strerror(-1) == b"invalid argument"
    assert lib.velox_strerror(12345) == b"unknown error"


FAKE = ctypes.c_void_p(1 << 20)   # non-null, 256-byte aligned; never dereferenced
FAKE_ODD = ctypes.c_void_p((1 << 20) + 2)
NULL = None


def test_route_topk_rejects(lib):
    f = lib.velox_route_topk
    ok = dict(q=FAKE, k=FAKE, dtype=0, B=1, H=2, Nq=256, Nk=1280, d=64, T=64, counts=NULL,
              alpha=2.0, topk=6, idx=FAKE, ws=FAKE, ws_bytes=1 << 30, ready=NULL, stream=NULL)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["q"], a["k"], a["dtype"], a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["T"],
                 a["counts"], a["alpha"], a["topk"], a["idx"], a["ws"], a["ws_bytes"], a["ready"],
                 a["stream"])

    assert call(q=NULL) == -1
    assert call(idx=NULL) == -1
    assert call(dtype=7) == -2
    assert call(T=32) == -2
    assert call(d=96) == -2
    assert call(Nq=200) == -1          # not a multiple of T
    assert call(Nk=1300) == -1         # not a multiple of Nq
    assert call(topk=3) == -1          # fewer than the m = 4 current blocks
    assert call(topk=21) == -1         # more than the 20 key blocks
    assert call(ws_bytes=16) == -1
    assert call(q=FAKE_ODD) == -1      # misaligned
    assert call(alpha=float("nan")) == -1


def test_workspace_holds_pooled_keys_for_64_token_blocks(lib):
    # 64-token blocks pool every past key block into the workspace before
    # scoring: beyond q-bar (B*H*m*d) and the scores (B*H*m*n_past) it holds
    # B*H*n_past*d floats; 128-token blocks score as they pool and need no more
    B, H, d, Nq = 1, 2, 128, 512
    for T, Nk in ((64, 5 * 512), (128, 5 * 512)):
        m, n_past = Nq // T, (Nk - Nq) // T
        base = 4 * B * H * m * (d + n_past)
        size = lib.velox_route_topk_workspace_size(B, H, Nq, Nk, d, T)
        if T == 64:
            assert size >= base + 4 * B * H * n_past * d
        else:
            assert base <= size < base + 4 * B * H * n_past * d


def test_workspace_sizes(lib):
    assert lib.velox_route_topk_workspace_size(1, 2, 256, 1280, 64, 64) > 0
    assert lib.velox_route_topk_workspace_size(1, 2, 250, 1280, 64, 64) == 0
    assert lib.velox_depth_multiwarp_workspace_size(32, 48) >= 32 * 48 * 20
    assert lib.velox_depth_multiwarp_workspace_size(0, 48) == 0


def test_sparse_attn_rejects(lib):
    f = lib.velox_sparse_attn_fwd
    ok = dict(q=FAKE, k=FAKE, v=FAKE, idx=FAKE, topk=6, B=1, H=2, Nq=256, Nk=1280, d=64, T=64,
              scale=0.125, o=FAKE, lse=NULL, status=NULL, stream=NULL)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["q"], a["k"], a["v"], a["idx"], a["topk"], a["B"], a["H"], a["Nq"], a["Nk"],
                 a["d"], a["T"], a["scale"], a["o"], a["lse"], a["status"], a["stream"])

    assert call(v=NULL) == -1
    assert call(o=NULL) == -1
    assert call(T=256) == -2
    assert call(d=32) == -2
    assert call(Nq=100) == -1
    assert call(Nk=1000) == -1
    assert call(topk=0) == -1
    assert call(topk=21) == -1
    assert call(scale=0.0) == -1
    assert call(scale=float("inf")) == -1
    assert call(k=FAKE_ODD) == -1


def test_geometry_rejects(lib):
    assert lib.velox_slices_build(NULL, FAKE, FAKE, 4, 16, 16, FAKE, NULL) == -1
    assert lib.velox_slices_build(FAKE, FAKE, FAKE, 0, 16, 16, FAKE, NULL) == -1
    assert lib.velox_block_overlap(FAKE, FAKE, FAKE, 1, 4, 1, 16, 16, 60, FAKE, NULL) == -1
    assert lib.velox_block_overlap(FAKE, FAKE, FAKE, 1, 4, 1, 16, 15, 64, FAKE, NULL) == -1
    assert lib.velox_block_overlap(FAKE, FAKE, NULL, 1, 4, 1, 16, 16, 64, FAKE, NULL) == -1
    mw = lib.velox_depth_multiwarp
    assert mw(FAKE, FAKE, FAKE, 4, 16, 16, -0.5, FAKE, FAKE, 1 << 20, NULL) == -1
    assert mw(FAKE, FAKE, FAKE, 4, 16, 16, 0.01, FAKE, FAKE, 8, NULL) == -1
    assert mw(FAKE, FAKE, FAKE, 0, 16, 16, 0.01, FAKE, FAKE, 1 << 20, NULL) == -1
    assert lib.velox_cast_bf16(NULL, FAKE, 4, NULL) == -1


def test_fp64_fma_bench_rejects(lib):
    f = lib.velox_fp64_fma_bench
    assert f(NULL, 1, 32, 1, NULL) == -1
    assert f(FAKE, 0, 32, 1, NULL) == -1
    assert f(FAKE, 1, 48, 1, NULL) == -1
    assert f(FAKE, 1, 2048, 1, NULL) == -1
    assert f(FAKE, 1, 32, 0, NULL) == -1
