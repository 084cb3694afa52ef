// Geometry-modulated block routing for sm_100a (memory-bound).
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse", steps 3 and 4 -- the overlap of a query block's region with
// each past frustum slice softly modulates the block importance the model
// computes itself (modulation, not replacement), and query blocks no history
// covers keep the model's own routing.
//
// Kernels:
//   pool_q      qbar[b,h,qb,:] = mean of the T query rows of block qb (fp32)
//   pool_score  streams the past keys once (16-byte loads): pools each key
//               block, dots it with every qbar of its head and writes the
//               modulated score s' = qbar.kbar / sqrt(d) (+ alpha * count / T
//               on covered query blocks). Eight consecutive key blocks form
//               one work item so each query block's scores leave as one
//               32-byte sector.
//   select      one warp per (b, h, qb): radix select of the (topk - m)
//               largest s' over the past blocks (equal s': smaller index
//               first), then the m current-chunk blocks; ascending indices.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "velox_internal.cuh"

namespace velox {

namespace {

constexpr int POOL_THREADS = 256;
constexpr int KGROUP = 8;  // key blocks per pool_score work item

template <typename TIn>
struct VecTraits;
template <>
struct VecTraits<__nv_bfloat16> {
    static constexpr int VEC = 8;
    __device__ static void add(float* acc, const uint4& u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct VecTraits<float> {
    static constexpr int VEC = 4;
    __device__ static void add(float* acc, const uint4& u) {
        acc[0] += __uint_as_float(u.x);
        acc[1] += __uint_as_float(u.y);
        acc[2] += __uint_as_float(u.z);
        acc[3] += __uint_as_float(u.w);
    }
};

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Mean over T rows of a row-major [T][D] block at `src` into out[0..D) (shared).
// `red` is shared scratch of (256 / (D / VEC)) * D floats. Ends with a barrier.
template <typename TIn, int D, int T>
__device__ __forceinline__ void pool_block(const TIn* __restrict__ src, float* out, float* red) {
    using V = VecTraits<TIn>;
    constexpr int TPR = D / V::VEC;           // threads per row
    constexpr int RPP = POOL_THREADS / TPR;   // rows per pass
    constexpr int PASSES = T / RPP;
    const int t = threadIdx.x;
    const int cg = t % TPR, r0 = t / TPR;
    uint4 buf[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p)
        buf[p] = ldg_stream(src + static_cast<size_t>(r0 + p * RPP) * D + cg * V::VEC);
    float acc[V::VEC];
#pragma unroll
    for (int i = 0; i < V::VEC; ++i) acc[i] = 0.f;
#pragma unroll
    for (int p = 0; p < PASSES; ++p) V::add(acc, buf[p]);
#pragma unroll
    for (int i = 0; i < V::VEC; ++i) red[r0 * D + cg * V::VEC + i] = acc[i];
    __syncthreads();
    if (t < D) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < RPP; ++r) s += red[r * D + t];
        out[t] = s * (1.0f / T);
    }
    __syncthreads();
}

template <typename TIn, int D, int T>
__global__ void __launch_bounds__(POOL_THREADS) pool_q_kernel(const TIn* __restrict__ q, float* qbar) {
    using V = VecTraits<TIn>;
    __shared__ float red[(POOL_THREADS / (D / V::VEC)) * D];
    __shared__ float out[D];
    const size_t blk = blockIdx.x;
    pool_block<TIn, D, T>(q + blk * T * D, out, red);
    if (threadIdx.x < D) qbar[blk * D + threadIdx.x] = out[threadIdx.x];
}

template <typename TIn, int D, int T>
__global__ void __launch_bounds__(POOL_THREADS)
    pool_score_kernel(const TIn* __restrict__ k, const float* __restrict__ qbar, RouteArgs r) {
    using V = VecTraits<TIn>;
    extern __shared__ float dsm[];
    float* q_s = dsm;                                  // [m][D]
    float* kb_s = q_s + r.m * D;                       // [KGROUP][D]
    float* red = kb_s + KGROUP * D;                    // [RPP][D]
    int* cov_s = reinterpret_cast<int*>(red + (POOL_THREADS / (D / V::VEC)) * D);  // [m]

    const int bh = blockIdx.y;
    const int b = bh / r.H;
    const int t = threadIdx.x;
    for (int i = t; i < r.m * D; i += POOL_THREADS) q_s[i] = qbar[static_cast<size_t>(bh) * r.m * D + i];
    const int32_t* cnt = r.counts ? r.counts + static_cast<size_t>(b) * r.m * r.P : nullptr;
    for (int qb = t; qb < r.m; qb += POOL_THREADS) {
        int any = 0;
        if (cnt)
            for (int j = 0; j < r.P; ++j) any |= (cnt[qb * r.P + j] > 0);
        cov_s[qb] = any;
    }
    __syncthreads();

    const TIn* kh = k + static_cast<size_t>(bh) * r.Nk * D;
    const int n_groups = (r.n_past + KGROUP - 1) / KGROUP;
    const int warp = t >> 5, lane = t & 31;
    const float invT = 1.0f / T;
    for (int g = blockIdx.x; g < n_groups; g += gridDim.x) {
        const int kb0 = g * KGROUP;
        const int nk = min(KGROUP, r.n_past - kb0);
        for (int i = 0; i < nk; ++i)
            pool_block<TIn, D, T>(kh + static_cast<size_t>(kb0 + i) * T * D, kb_s + i * D, red);
        // scores: warp w takes query blocks w, w+8, ...; lanes split d
        for (int qb = warp; qb < r.m; qb += POOL_THREADS / 32) {
            float qv[D / 32];
#pragma unroll
            for (int u = 0; u < D / 32; ++u) qv[u] = q_s[qb * D + lane + 32 * u];
            float mine = 0.f;
#pragma unroll
            for (int i = 0; i < KGROUP; ++i) {
                float p = 0.f;
                if (i < nk) {
#pragma unroll
                    for (int u = 0; u < D / 32; ++u) p = fmaf(qv[u], kb_s[i * D + lane + 32 * u], p);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
                if (lane == i) mine = p;
            }
            if (lane < nk) {
                const int kb = kb0 + lane;
                float s = mine * r.inv_sqrt_d;
                if (cov_s[qb]) s = s + r.alpha * static_cast<float>(cnt[qb * r.P + kb / r.m]) * invT;
                r.scores[(static_cast<size_t>(bh) * r.m + qb) * r.n_past + kb] = s;
            }
        }
        __syncthreads();
    }
}

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int SEL_WARPS = 8;

__global__ void __launch_bounds__(SEL_WARPS * 32)
    select_kernel(const float* __restrict__ scores, int rows, int n_past, int m, int k_past, int topk,
                  int32_t* __restrict__ idx) {
    __shared__ uint32_t hist_all[SEL_WARPS][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * SEL_WARPS + warp;
    if (row >= rows) return;
    const float* sc = scores + static_cast<size_t>(row) * n_past;
    int32_t* out = idx + static_cast<size_t>(row) * topk;
    for (int i = lane; i < m; i += 32) out[k_past + i] = n_past + i;
    if (k_past <= 0) return;
    if (k_past >= n_past) {
        for (int i = lane; i < n_past; i += 32) out[i] = i;
        return;
    }
    uint32_t* h = hist_all[warp];
    uint32_t prefix = 0, mask = 0;
    int remaining = k_past;
    const unsigned FULL = 0xffffffffu;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = lane; i < 256; i += 32) h[i] = 0;
        __syncwarp();
        for (int i = lane; i < n_past; i += 32) {
            const uint32_t key = order_key(sc[i]);
            if ((key & mask) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
        }
        __syncwarp();
        int cnt[8], tot = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            cnt[u] = static_cast<int>(h[255 - 8 * lane - u]);
            tot += cnt[u];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += v;
        }
        const int excl = incl - tot;
        const bool mine = excl < remaining && remaining <= incl;
        const unsigned bal = __ballot_sync(FULL, mine);
        const int src = __ffs(bal) - 1;
        int digit = 0, above = 0;
        if (mine) {
            int acc = excl;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (acc + cnt[u] >= remaining) {
                    digit = 255 - 8 * lane - u;
                    above = acc;
                    break;
                }
                acc += cnt[u];
            }
        }
        digit = __shfl_sync(FULL, digit, src);
        above = __shfl_sync(FULL, above, src);
        remaining -= above;
        prefix |= static_cast<uint32_t>(digit) << shift;
        mask |= 0xFFu << shift;
        __syncwarp();
    }
    // prefix is the k_past-th largest key; take every larger key and the first
    // `remaining` equal keys in index order
    const unsigned lt = (1u << lane) - 1u;
    int written = 0, eq_seen = 0;
    for (int base = 0; base < n_past; base += 32) {
        const int i = base + lane;
        const uint32_t key = i < n_past ? order_key(sc[i]) : 0u;
        const bool gt = i < n_past && key > prefix;
        const bool eq = i < n_past && key == prefix;
        const unsigned eqb = __ballot_sync(FULL, eq);
        const bool take = gt || (eq && (eq_seen + __popc(eqb & lt)) < remaining);
        const unsigned tb = __ballot_sync(FULL, take);
        if (take) out[written + __popc(tb & lt)] = i;
        written += __popc(tb);
        eq_seen += __popc(eqb);
    }
}

template <typename TIn, int D, int T>
int route_typed(const TIn* q, const TIn* k, const RouteArgs& r, cudaStream_t st) {
    using V = VecTraits<TIn>;
    const int BH = r.B * r.H;
    pool_q_kernel<TIn, D, T><<<BH * r.m, POOL_THREADS, 0, st>>>(q, r.qbar);
    if (r.n_past > 0) {
        const size_t smem = (static_cast<size_t>(r.m) * D + KGROUP * D +
                             (POOL_THREADS / (D / V::VEC)) * D) * sizeof(float) +
                            static_cast<size_t>(r.m) * sizeof(int);
        auto kern = pool_score_kernel<TIn, D, T>;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return VELOX_ECUDA;
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int n_groups = (r.n_past + KGROUP - 1) / KGROUP;
        // about 4 resident CTAs per SM over all heads
        int gx = (4 * sms + BH - 1) / BH;
        gx = max(1, min(gx, n_groups));
        pool_score_kernel<TIn, D, T><<<dim3(gx, BH), POOL_THREADS, smem, st>>>(k, r.qbar, r);
    }
    const int rows = BH * r.m;
    select_kernel<<<(rows + SEL_WARPS - 1) / SEL_WARPS, SEL_WARPS * 32, 0, st>>>(
        r.scores, rows, r.n_past, r.m, r.topk - r.m, r.topk, r.idx);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

template <typename TIn>
int route_dispatch(const void* q, const void* k, const RouteArgs& r, cudaStream_t st) {
    const TIn* tq = static_cast<const TIn*>(q);
    const TIn* tk = static_cast<const TIn*>(k);
    if (r.d == 128 && r.T == 128) return route_typed<TIn, 128, 128>(tq, tk, r, st);
    if (r.d == 128 && r.T == 64) return route_typed<TIn, 128, 64>(tq, tk, r, st);
    if (r.d == 64 && r.T == 128) return route_typed<TIn, 64, 128>(tq, tk, r, st);
    if (r.d == 64 && r.T == 64) return route_typed<TIn, 64, 64>(tq, tk, r, st);
    return VELOX_EUNSUPPORTED;
}

}  // namespace

size_t route_ws_bytes(int B, int H, int m, int n_past, int d) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t rows = static_cast<size_t>(B) * H * m;
    return up(rows * d * sizeof(float)) + up(rows * static_cast<size_t>(n_past) * sizeof(float));
}

int route_launch(const void* q, const void* k, int dtype, const RouteArgs& r, cudaStream_t st) {
    if (dtype == VELOX_BF16) return route_dispatch<__nv_bfloat16>(q, k, r, st);
    if (dtype == VELOX_F32) return route_dispatch<float>(q, k, r, st);
    return VELOX_EUNSUPPORTED;
}

}  // namespace velox
