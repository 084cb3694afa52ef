// C ABI of libvelox: argument validation, then kernel launches on the caller's
// stream. Nothing here allocates, frees or synchronises.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "velox_internal.cuh"

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
inline bool tile_ok(int x) { return x == 64 || x == 128; }

}  // namespace

extern "C" {

int velox_version(void) { return 100; }

const char* velox_strerror(int code) {
    switch (code) {
        case VELOX_OK: return "ok";
        case VELOX_EINVAL: return "invalid argument";
        case VELOX_EUNSUPPORTED: return "unsupported configuration";
        case VELOX_ECUDA: return "CUDA error";
        case VELOX_ETIMEOUT: return "bounded wait expired";
        case VELOX_EBOUNDS: return "index out of range";
        default: return "unknown error";
    }
}

int velox_slices_build(const float* depth, const float* poses, const float* intr, int P, int Hp,
                       int Wp, velox_slice_t* slices, void* stream) {
    if (!depth || !poses || !intr || !slices || P < 1 || Hp < 1 || Wp < 1) return VELOX_EINVAL;
    return velox::slices_launch(depth, poses, intr, P, Hp * Wp, slices, as_stream(stream));
}

int velox_block_overlap(const float* cur_depth, const velox_slice_t* cur_cam,
                        const velox_slice_t* slices, int B, int P, int F, int Hp, int Wp, int T,
                        int32_t* counts, void* stream) {
    if (!cur_depth || !cur_cam || !slices || !counts) return VELOX_EINVAL;
    if (B < 1 || P < 1 || F < 1 || Hp < 1 || Wp < 1 || T < 32 || T > 1024 || (T % 32) != 0)
        return VELOX_EINVAL;
    const long long Nq = static_cast<long long>(F) * Hp * Wp;
    if (Nq % T != 0 || Nq > (1ll << 30)) return VELOX_EINVAL;
    const int m = static_cast<int>(Nq / T);
    return velox::overlap_launch(cur_depth, cur_cam, slices, B, P, Hp, Wp, T, m, counts,
                                 as_stream(stream));
}

size_t velox_route_topk_workspace_size(int B, int H, int Nq, int Nk, int d, int T) {
    if (B < 1 || H < 1 || T < 1 || Nq < T || Nq % T || Nk < Nq || Nk % Nq || d < 1) return 0;
    const int m = Nq / T;
    const int n_past = (Nk - Nq) / T;
    return velox::route_ws_bytes(B, H, m, n_past, d, T);
}

int velox_route_topk(const void* q, const void* k, int dtype, int B, int H, int Nq, int Nk, int d,
                     int T, const int32_t* counts, float alpha, int topk, int32_t* idx, void* ws,
                     size_t ws_bytes, void* counts_ready, void* stream) {
    if (!q || !k || !idx || !ws) return VELOX_EINVAL;
    if (dtype != VELOX_BF16 && dtype != VELOX_F32) return VELOX_EUNSUPPORTED;
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || T < 1) return VELOX_EINVAL;
    if (!tile_ok(T) || !tile_ok(d)) return VELOX_EUNSUPPORTED;
    if (Nq % T || Nk % Nq) return VELOX_EINVAL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(ws, 256) || !aligned(idx, 4))
        return VELOX_EINVAL;
    if (!std::isfinite(alpha)) return VELOX_EINVAL;
    const int m = Nq / T;
    const int n_kb = Nk / T;
    if (topk < m || topk > n_kb) return VELOX_EINVAL;
    const size_t need = velox_route_topk_workspace_size(B, H, Nq, Nk, d, T);
    if (need == 0 || ws_bytes < need) return VELOX_EINVAL;
    if (static_cast<long long>(B) * H * Nk * d >= (1ll << 40)) return VELOX_EINVAL;
    if (Nk / T > 8192) return VELOX_EINVAL;  // key-block index range of the selection

    velox::RouteArgs r{};
    r.B = B;
    r.H = H;
    r.Nq = Nq;
    r.Nk = Nk;
    r.d = d;
    r.T = T;
    r.m = m;
    r.P = Nk / Nq - 1;
    r.n_past = r.P * m;
    r.topk = topk;
    r.counts = r.P > 0 ? counts : nullptr;
    r.alpha = alpha;
    r.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    r.idx = idx;
    const size_t rows = static_cast<size_t>(B) * H * m;
    const size_t qbar_bytes = (rows * d * sizeof(float) + 255) & ~static_cast<size_t>(255);
    r.qbar = static_cast<float*>(ws);
    r.scores = reinterpret_cast<float*>(static_cast<char*>(ws) + qbar_bytes);
    if (velox::route_split_scoring(T, d)) {
        const size_t scores_bytes =
            (rows * static_cast<size_t>(r.n_past) * sizeof(float) + 255) & ~static_cast<size_t>(255);
        r.kbar_ws = reinterpret_cast<float*>(static_cast<char*>(ws) + qbar_bytes + scores_bytes);
    }
    r.counts_ready = static_cast<cudaEvent_t>(counts_ready);
    return velox::route_launch(q, k, dtype, r, as_stream(stream));
}

}  // extern "C"

namespace {

int sparse_attn(const void* q, const void* k, const void* v, const int32_t* idx, int topk, int B,
                int H, int Nq, int Nk, int d, int T, float scale, void* o, float* lse,
                int32_t* status, unsigned long long wait_ns, int skip_mma, int force_pair,
                void* stream) {
    if (!q || !k || !v || !o) return VELOX_EINVAL;
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || T < 1) return VELOX_EINVAL;
    if (!tile_ok(T) || !tile_ok(d)) return VELOX_EUNSUPPORTED;
    if (Nq % T || Nk % T) return VELOX_EINVAL;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
        return VELOX_EINVAL;
    if (!(scale > 0.0f) || !std::isfinite(scale)) return VELOX_EINVAL;
    const long long rows_k = static_cast<long long>(B) * H * Nk;
    if (rows_k >= (1ll << 31) || static_cast<long long>(B) * H * Nq >= (1ll << 31))
        return VELOX_EINVAL;
    const int n_kb = Nk / T;
    if (idx && (topk < 1 || topk > n_kb)) return VELOX_EINVAL;
    if (H > 65535 || B > 65535) return VELOX_EINVAL;

    velox::AttnArgs a{};
    a.idx = idx;
    a.n_sel = idx ? topk : n_kb;
    a.H = H;
    a.Nq = Nq;
    a.Nk = Nk;
    a.T = T;
    a.m = Nq / T;
    a.n_kb = n_kb;
    a.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.status = status;
    a.wait_ns = wait_ns;
    a.skip_mma = skip_mma;
    a.force_pair = force_pair;
    return velox::attn_fwd_launch(q, k, v, a, B, d, as_stream(stream));
}

}  // namespace

extern "C" {

int velox_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                          int topk, int B, int H, int Nq, int Nk, int d, int T, float scale,
                          void* o, float* lse, int32_t* status, void* stream) {
    return sparse_attn(q, k, v, idx, topk, B, H, Nq, Nk, d, T, scale, o, lse, status,
                       velox::WAIT_LIMIT_NS, 0, 0, stream);
}

int velox_sparse_attn_fwd_test(const void* q, const void* k, const void* v, const int32_t* idx,
                               int topk, int B, int H, int Nq, int Nk, int d, int T, float scale,
                               void* o, float* lse, int32_t* status, double wait_limit_s,
                               int flags, void* stream) {
    if (!(wait_limit_s >= 1e-3 && wait_limit_s <= 10.0)) return VELOX_EINVAL;
    if (flags & ~(VELOX_TEST_SKIP_MMA | VELOX_TEST_FORCE_PAIR)) return VELOX_EINVAL;
    return sparse_attn(q, k, v, idx, topk, B, H, Nq, Nk, d, T, scale, o, lse, status,
                       static_cast<unsigned long long>(wait_limit_s * 1e9),
                       (flags & VELOX_TEST_SKIP_MMA) ? 1 : 0,
                       (flags & VELOX_TEST_FORCE_PAIR) ? 1 : 0, stream);
}

size_t velox_kbar_cache_bytes(int B, int H, int max_past_chunks, int Nq, int d, int T) {
    if (B < 1 || H < 1 || max_past_chunks < 1 || T < 1 || Nq < T || Nq % T || d < 1) return 0;
    return static_cast<size_t>(B) * H * max_past_chunks * (Nq / T) * d * sizeof(float);
}

int velox_kbar_append(const void* k, int dtype, int B, int H, int Nk, int Nq, int d, int T, int chunk,
                      float* kbar, int max_past_chunks, void* stream) {
    if (!k || !kbar) return VELOX_EINVAL;
    if (dtype != VELOX_BF16 && dtype != VELOX_F32) return VELOX_EUNSUPPORTED;
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || d < 1 || T < 1 || max_past_chunks < 1)
        return VELOX_EINVAL;
    if (!tile_ok(T) || !tile_ok(d)) return VELOX_EUNSUPPORTED;
    if (Nq % T || Nk % T) return VELOX_EINVAL;
    if (chunk < 0 || chunk >= max_past_chunks || static_cast<long long>(chunk + 1) * Nq > Nk)
        return VELOX_EINVAL;
    if (!aligned(k, 16) || !aligned(kbar, 16)) return VELOX_EINVAL;
    if (static_cast<long long>(B) * H > 65535) return VELOX_EINVAL;
    return velox::kbar_append_launch(k, dtype, B * H, Nk, Nq, d, T, chunk, max_past_chunks * (Nq / T),
                                     kbar, as_stream(stream));
}

int velox_route_topk_cached(const void* q, int dtype, const float* kbar, int max_past_chunks, int B,
                            int H, int Nq, int P, int d, int T, const int32_t* counts, float alpha,
                            int topk, int32_t* idx, void* ws, size_t ws_bytes, void* counts_ready,
                            void* stream) {
    if (!q || !idx || !ws || (P > 0 && !kbar)) return VELOX_EINVAL;
    if (dtype != VELOX_BF16 && dtype != VELOX_F32) return VELOX_EUNSUPPORTED;
    if (B < 1 || H < 1 || Nq < 1 || d < 1 || T < 1 || P < 0 || P > max_past_chunks)
        return VELOX_EINVAL;
    if (!tile_ok(T) || !tile_ok(d)) return VELOX_EUNSUPPORTED;
    if (Nq % T) return VELOX_EINVAL;
    if (!aligned(q, 16) || !aligned(ws, 256) || !aligned(idx, 4) || (kbar && !aligned(kbar, 16)))
        return VELOX_EINVAL;
    if (!std::isfinite(alpha)) return VELOX_EINVAL;
    const long long Nk = static_cast<long long>(P + 1) * Nq;
    if (Nk >= (1ll << 31) || Nk / T > 8192) return VELOX_EINVAL;
    const int m = Nq / T;
    const int n_kb = static_cast<int>(Nk / T);
    if (topk < m || topk > n_kb) return VELOX_EINVAL;
    const size_t need = velox_route_topk_workspace_size(B, H, Nq, static_cast<int>(Nk), d, T);
    if (need == 0 || ws_bytes < need) return VELOX_EINVAL;

    velox::RouteArgs r{};
    r.B = B;
    r.H = H;
    r.Nq = Nq;
    r.Nk = static_cast<int>(Nk);
    r.d = d;
    r.T = T;
    r.m = m;
    r.P = P;
    r.n_past = P * m;
    r.topk = topk;
    r.counts = P > 0 ? counts : nullptr;
    r.alpha = alpha;
    r.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    r.idx = idx;
    const size_t rows = static_cast<size_t>(B) * H * m;
    const size_t qbar_bytes = (rows * d * sizeof(float) + 255) & ~static_cast<size_t>(255);
    r.qbar = static_cast<float*>(ws);
    r.scores = reinterpret_cast<float*>(static_cast<char*>(ws) + qbar_bytes);
    r.counts_ready = static_cast<cudaEvent_t>(counts_ready);
    r.kbar = kbar;
    r.kbar_cap = max_past_chunks * m;
    return velox::route_launch(q, nullptr, dtype, r, as_stream(stream));
}

size_t velox_depth_multiwarp_workspace_size(int Hp, int Wp) {
    if (Hp < 1 || Wp < 1) return 0;
    return velox::multiwarp_ws_bytes(Hp * Wp);
}

int velox_depth_multiwarp(const float* past_depth, const velox_slice_t* past_cams,
                          const velox_slice_t* cur_cam, int P, int Hp, int Wp, float rel_tol,
                          float* cur_depth, void* ws, size_t ws_bytes, void* stream) {
    if (!past_depth || !past_cams || !cur_cam || !cur_depth || !ws) return VELOX_EINVAL;
    if (P < 1 || Hp < 1 || Wp < 1 || !(rel_tol >= 0.0f) || !std::isfinite(rel_tol))
        return VELOX_EINVAL;
    if (static_cast<long long>(P) * Hp * Wp >= (1ll << 31)) return VELOX_EINVAL;
    if (!aligned(ws, 8) || ws_bytes < velox_depth_multiwarp_workspace_size(Hp, Wp))
        return VELOX_EINVAL;
    return velox::multiwarp_launch(past_depth, past_cams, cur_cam, P, Hp, Wp, rel_tol, cur_depth,
                                   ws, as_stream(stream));
}

int velox_fp64_fma_bench(double* out, int blocks, int threads, int iters, void* stream) {
    if (!out || blocks < 1 || threads < 32 || threads > 1024 || (threads % 32) != 0 || iters < 1)
        return VELOX_EINVAL;
    return velox::fp64_fma_launch(out, blocks, threads, iters, as_stream(stream));
}

int velox_cast_bf16(const float* x, uint16_t* y, size_t n, void* stream) {
    if (!x || !y) return VELOX_EINVAL;
    if (n == 0) return VELOX_OK;
    return velox::cast_bf16_launch(x, y, n, as_stream(stream));
}

}  // extern "C"
