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
//               block and dots it with every qbar of its head, writing the
//               block importance s = qbar.kbar / sqrt(d). One warp pools one
//               key block at a time; warps run independently.
//   select      one CTA per (b, h, qb): applies the modulation
//               s' = s + alpha * count / T on covered query blocks, then
//               selects exactly the (topk - m) largest s' over the past blocks
//               (equal s': smaller index first) by four 8-bit radix rounds on
//               order-preserving keys held in registers (one warp per row
//               beyond 4096 blocks), then the m current-chunk blocks;
//               ascending indices.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "velox_internal.cuh"

namespace velox {

namespace {

constexpr int POOL_THREADS = 256;

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
    // the scorer, launched as this grid's dependent, may start at once: it
    // streams its first key blocks and waits for q-bar only when it needs it
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float red[(POOL_THREADS / (D / V::VEC)) * D];
    __shared__ float out[D];
    const size_t blk = blockIdx.x;
    pool_block<TIn, D, T>(q + blk * T * D, out, red);
    if (threadIdx.x < D) qbar[blk * D + threadIdx.x] = out[threadIdx.x];
}

// Loads of one warp's [T][D] block: lane (cg, r0) reads 16-byte column group
// cg of rows r0, r0 + RPW, ...; the first batch is issued by warp_pool_first so
// that a caller can overlap it with other work.
template <typename TIn, int D, int T>
struct WarpPoolShape {
    using V = VecTraits<TIn>;
    static constexpr int TPR = D / V::VEC;
    static constexpr int RPW = 32 / TPR;
    static constexpr int LOADS = T / RPW;
    static constexpr int BATCH = LOADS < 16 ? LOADS : 16;
};

template <typename TIn, int D, int T>
__device__ __forceinline__ void warp_pool_first(const TIn* __restrict__ blk, int lane,
                                                uint4* buf) {
    using S = WarpPoolShape<TIn, D, T>;
    const int cg = lane % S::TPR, r0 = lane / S::TPR;
    const TIn* base = blk + static_cast<size_t>(r0) * D + cg * S::V::VEC;
#pragma unroll
    for (int i = 0; i < S::BATCH; ++i) buf[i] = ldg_stream(base + static_cast<size_t>(i) * S::RPW * D);
}

// One warp pools one [T][D] block: all of a lane's loads in flight at once, in
// batches (the first batch already issued into `first` by warp_pool_first),
// sums in fp32 pairs, then the lanes of a column group reduce by shuffles.
// On return every lane holds the column sums of its group, times 1/T.
template <typename TIn, int D, int T>
__device__ __forceinline__ void warp_pool_rest(const TIn* __restrict__ blk, int lane,
                                               const uint4* first, float* kbar) {
    using V = VecTraits<TIn>;
    using S = WarpPoolShape<TIn, D, T>;
    constexpr int TPR = S::TPR;
    constexpr int RPW = S::RPW;
    constexpr int LOADS = S::LOADS;
    constexpr int BATCH = S::BATCH;
    const int cg = lane % TPR, r0 = lane / TPR;
    const TIn* base = blk + static_cast<size_t>(r0) * D + cg * V::VEC;
    float acc[V::VEC];
#pragma unroll
    for (int i = 0; i < V::VEC; ++i) acc[i] = 0.f;
#pragma unroll
    for (int i = 0; i < BATCH; ++i) V::add(acc, first[i]);
#pragma unroll
    for (int b0 = BATCH; b0 < LOADS; b0 += BATCH) {
        uint4 buf[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i)
            buf[i] = ldg_stream(base + static_cast<size_t>(b0 + i) * RPW * D);
#pragma unroll
        for (int i = 0; i < BATCH; ++i) V::add(acc, buf[i]);
    }
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1) {
#pragma unroll
        for (int i = 0; i < V::VEC; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    }
#pragma unroll
    for (int i = 0; i < V::VEC; ++i) kbar[i] = acc[i] * (1.0f / T);
}

template <typename TIn, int D, int T>
__device__ __forceinline__ void warp_pool(const TIn* __restrict__ blk, int lane, float* kbar) {
    uint4 first[WarpPoolShape<TIn, D, T>::BATCH];
    warp_pool_first<TIn, D, T>(blk, lane, first);
    warp_pool_rest<TIn, D, T>(blk, lane, first, kbar);
}

// CTA = one (b, h) slice of the grid; each warp walks its own past key blocks
// (kb = blockIdx.x * WARPS + warp, strided by the grid), pools one block at a
// time and scores it against every query block of its head straight from
// shared memory. Warps never wait for one another after the q-bar load.
template <typename TIn, int D, int T>
__global__ void __launch_bounds__(POOL_THREADS)
    pool_score_kernel(const TIn* __restrict__ k, const float* __restrict__ qbar, RouteArgs r) {
    using V = VecTraits<TIn>;
    constexpr int TPR = D / V::VEC;
    constexpr int RPW = 32 / TPR;
    constexpr int WARPS = POOL_THREADS / 32;
    extern __shared__ float dsm[];
    float* q_s = dsm;  // [m][D]

    const int bh = blockIdx.y;
    const int t = threadIdx.x;
    const TIn* kh = k + static_cast<size_t>(bh) * r.Nk * D;
    const int warp = t >> 5, lane = t & 31;
    const int cg = lane % TPR, r0 = lane / TPR;
    const int stride = gridDim.x * WARPS;
    int kb = blockIdx.x * WARPS + warp;
    // the first loads of this warp's first key block fly while q-bar is staged
    uint4 first[WarpPoolShape<TIn, D, T>::BATCH];
    if (kb < r.n_past)
        warp_pool_first<TIn, D, T>(kh + static_cast<size_t>(kb) * T * D, lane, first);
    // the selection, launched as this grid's dependent, may be scheduled now:
    // it waits for this grid to finish before it reads a score
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // q-bar comes from the preceding pool_q grid (a no-op without a dependent launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = t; i < r.m * D; i += POOL_THREADS) q_s[i] = qbar[static_cast<size_t>(bh) * r.m * D + i];
    __syncthreads();

    float* srow = r.scores + static_cast<size_t>(bh) * r.m * r.n_past;
    for (bool head = true; kb < r.n_past; kb += stride, head = false) {
        float kv[V::VEC];
        if (head)
            warp_pool_rest<TIn, D, T>(kh + static_cast<size_t>(kb) * T * D, lane, first, kv);
        else
            warp_pool<TIn, D, T>(kh + static_cast<size_t>(kb) * T * D, lane, kv);
        // every lane runs the same number of iterations (full-warp shuffles)
        for (int q0 = 0; q0 < r.m; q0 += RPW) {
            const int qb = q0 + r0;
            const bool valid = qb < r.m;
            float p = 0.f;
            if (valid) {
                const float* qrow = q_s + qb * D + cg * V::VEC;
#pragma unroll
                for (int i = 0; i < V::VEC; ++i) p = fmaf(qrow[i], kv[i], p);
            }
#pragma unroll
            for (int o = 1; o < TPR; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if (valid && cg == 0) srow[static_cast<size_t>(qb) * r.n_past + kb] = p * r.inv_sqrt_d;
        }
    }
}

// Pools the m key blocks of one chunk of every (b, h) into the k-bar cache:
// kbar[bh][chunk * m + i][:] = mean of K rows [chunk * Nq + i * T, + T).
template <typename TIn, int D, int T>
__global__ void __launch_bounds__(POOL_THREADS)
    kbar_append_kernel(const TIn* __restrict__ k, int Nk, int Nq, int m, int chunk, int cap,
                       float* __restrict__ kbar) {
    using V = VecTraits<TIn>;
    constexpr int TPR = D / V::VEC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * (POOL_THREADS / 32) + warp;
    if (i >= m) return;
    const int bh = blockIdx.y;
    const int cg = lane % TPR, r0 = lane / TPR;
    float kv[V::VEC];
    warp_pool<TIn, D, T>(k + (static_cast<size_t>(bh) * Nk + static_cast<size_t>(chunk) * Nq +
                              static_cast<size_t>(i) * T) * D,
                         lane, kv);
    if (r0 == 0) {
        float4* dst = reinterpret_cast<float4*>(
            kbar + (static_cast<size_t>(bh) * cap + static_cast<size_t>(chunk) * m + i) * D +
            cg * V::VEC);
#pragma unroll
        for (int j = 0; j < V::VEC / 4; ++j)
            dst[j] = make_float4(kv[4 * j], kv[4 * j + 1], kv[4 * j + 2], kv[4 * j + 3]);
    }
}

// Scores of the past key blocks from the k-bar cache, each dot product summed
// in exactly the order pool_score_kernel uses (per column group of VEC an FMA
// chain, then the pairwise tree its shuffles form), so cached and streaming
// routing give bit-identical scores. A CTA takes SC_KT cached blocks of one
// head; thread (j, g) scores block j against SC_QA query blocks at a time
// (groups g, g + SC_QG, ...), so one shared-memory read of a key group serves
// SC_QA outputs and the query groups are warp-wide broadcasts. The tree is
// built as the column groups come: a node that is a right child at level L is
// added to the left subtree kept for that level.
constexpr int SC_KT = 32;  // key blocks per CTA
constexpr int SC_QG = 8;   // 256 threads = SC_KT x SC_QG
constexpr int SC_QA = 5;   // query blocks per thread and pass

template <typename TIn, int D>
__global__ void __launch_bounds__(256) score_cached_kernel(const float* __restrict__ qbar, RouteArgs r) {
    using V = VecTraits<TIn>;
    constexpr int VEC = V::VEC;
    constexpr int TPR = D / VEC;  // column groups = lanes of one row in the streaming scorer
    constexpr int LOG = TPR == 8 ? 3 : (TPR == 16 ? 4 : 5);
    static_assert((1 << LOG) == TPR, "column groups must be 8, 16 or 32");
    extern __shared__ float sm[];
    constexpr int KP = D + 4;          // padded row: 16-byte aligned, 128-bit reads conflict-free
    float* q_s = sm;                   // [m][D]
    float* k_s = q_s + r.m * D;        // [SC_KT][KP]
    // the selection, launched as this grid's dependent, may be scheduled now
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int bh = blockIdx.y;
    const int kb0 = blockIdx.x * SC_KT;
    const int nk = min(SC_KT, r.n_past - kb0);
    const int t = threadIdx.x;
    // 16-byte loads, all of a thread's in flight together (D is a multiple of 4)
    const float4* qsrc = reinterpret_cast<const float4*>(qbar + static_cast<size_t>(bh) * r.m * D);
    const float4* ksrc = reinterpret_cast<const float4*>(r.kbar + (static_cast<size_t>(bh) * r.kbar_cap + kb0) * D);
    constexpr int D4 = D / 4;
#pragma unroll 4
    for (int i = t; i < r.m * D4; i += 256) reinterpret_cast<float4*>(q_s)[i] = __ldg(qsrc + i);
#pragma unroll 8
    for (int i = t; i < nk * D4; i += 256)
        *reinterpret_cast<float4*>(k_s + (i / D4) * KP + (i % D4) * 4) = __ldg(ksrc + i);
    __syncthreads();
    const int j = t % SC_KT;
    if (j >= nk) return;  // no barrier follows
    const float4* krow = reinterpret_cast<const float4*>(k_s + j * KP);
    float* scol = r.scores + static_cast<size_t>(bh) * r.m * r.n_past + kb0 + j;
    for (int q0 = (t / SC_KT) * SC_QA; q0 < r.m; q0 += SC_QG * SC_QA) {
        float stk[SC_QA][LOG];  // [a][L]: left subtree pending at level L (L >= 1)
        float root[SC_QA];
#pragma unroll 1
        for (int c = 0; c < TPR / 2; ++c) {  // column groups 2c and 2c + 1: a level-1 node
            float node[SC_QA];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int g = 2 * c + h;
                float kv[VEC];
#pragma unroll
                for (int v4 = 0; v4 < VEC / 4; ++v4) {
                    const float4 b = krow[g * (VEC / 4) + v4];
                    kv[4 * v4] = b.x;
                    kv[4 * v4 + 1] = b.y;
                    kv[4 * v4 + 2] = b.z;
                    kv[4 * v4 + 3] = b.w;
                }
#pragma unroll
                for (int a = 0; a < SC_QA; ++a) {
                    const int qb = min(q0 + a, r.m - 1);  // rows past m are computed and dropped
                    const float4* qr = reinterpret_cast<const float4*>(q_s + qb * D + g * VEC);
                    float p = 0.f;
#pragma unroll
                    for (int v4 = 0; v4 < VEC / 4; ++v4) {
                        const float4 x = qr[v4];
                        p = fmaf(x.x, kv[4 * v4], p);
                        p = fmaf(x.y, kv[4 * v4 + 1], p);
                        p = fmaf(x.z, kv[4 * v4 + 2], p);
                        p = fmaf(x.w, kv[4 * v4 + 3], p);
                    }
                    node[a] = h == 0 ? p : node[a] + p;
                }
            }
            // node c at level 1 is a right child at level L when bit L-1 of c is set
#pragma unroll
            for (int a = 0; a < SC_QA; ++a) {
                float v = node[a];
                bool placed = false;
#pragma unroll
                for (int L = 1; L < LOG; ++L) {
                    if (!placed) {
                        if (((c >> (L - 1)) & 1) == 0) {
                            stk[a][L] = v;
                            placed = true;
                        } else {
                            v = stk[a][L] + v;
                        }
                    }
                }
                if (!placed) root[a] = v;
            }
        }
#pragma unroll
        for (int a = 0; a < SC_QA; ++a)
            if (q0 + a < r.m) scol[static_cast<size_t>(q0 + a) * r.n_past] = root[a] * r.inv_sqrt_d;
    }
}

struct SelArgs {
    const float* scores;  // [rows][n_past] raw block scores
    int rows, n_past, m, H, P, k_past, topk;
    const int32_t* counts;  // [B][m][P] or nullptr
    float alpha, invT;
    int32_t* idx;
};

// Geometric modulation of one row: s' = s + alpha * count[chunk(kb)] / T when
// the query block is covered (some count > 0), s' = s otherwise.
struct RowMod {
    const int32_t* cnt;  // counts[b][qb][*] or nullptr when uncovered / no geometry
    float alpha, invT;
    float inv_m;
    // chunk(kb) = kb / m as floor((kb + 1/2) / m): the quotient sits at least
    // 1/(2m) from an integer and the product is accurate to ~1e-4 for
    // kb < 2^13, so the conversion truncates to the exact integer quotient
    __device__ __forceinline__ float operator()(float sc, int kb) const {
        if (!cnt) return sc;
        const int chunk = __float2int_rz(__fmul_rn(static_cast<float>(kb) + 0.5f, inv_m));
        return sc + alpha * static_cast<float>(__ldg(cnt + chunk)) * invT;
    }
};

// Called by all 32 lanes of a warp: the lanes read the row's counts in
// parallel and a ballot decides whether the query block is covered.
__device__ __forceinline__ RowMod row_mod(const SelArgs& a, int row, int lane) {
    RowMod r{nullptr, a.alpha, a.invT, 1.0f / static_cast<float>(a.m)};
    if (a.counts) {
        const int qb = row % a.m;
        const int b = (row / a.m) / a.H;
        const int32_t* c = a.counts + (static_cast<size_t>(b) * a.m + qb) * a.P;
        bool any = false;
        for (int j = lane; j < a.P; j += 32) any |= __ldg(c + j) > 0;
        if (__any_sync(0xffffffffu, any)) r.cnt = c;
    }
    return r;
}

__device__ __forceinline__ uint32_t order_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int SEL_WARPS = 8;

__global__ void __launch_bounds__(SEL_WARPS * 32) select_kernel(const SelArgs a) {
    __shared__ uint32_t hist_all[SEL_WARPS][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * SEL_WARPS + warp;
    if (row >= a.rows) return;
    // launched as the scorer's dependent: scores (and counts) only after it is done
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int n_past = a.n_past, m = a.m, k_past = a.k_past;
    const float* sc = a.scores + static_cast<size_t>(row) * n_past;
    int32_t* out = a.idx + static_cast<size_t>(row) * a.topk;
    const RowMod mod = row_mod(a, row, lane);
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
            const uint32_t key = order_key(mod(sc[i], i));
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
        const uint32_t key = i < n_past ? order_key(mod(sc[i], i)) : 0u;
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

// One CTA (THREADS threads) per (b, h, qb) row of at most THREADS * CH past
// blocks: thread t keeps the keys of blocks t, t + THREADS, ... in registers.
// The (k_past)-th largest key u is found 8 bits at a time from the top, each
// round a 256-bin histogram of the keys that still match the chosen prefix.
// (Measured at the chunk-48 size: 18.3 us per launch, against 22.6 us for a
// 32-round bitwise bisection with the same emission.)
// Then every warp emits, from a shared-memory copy of its segment of the row,
// the keys above u and the first equal ones in index order, at offsets from a
// prefix over the warps' counts. Padding keys are 0, below every real key.
constexpr int SEL_CTA_THREADS = 256;  // measured against 64 and 128

template <int THREADS, int CH>
__global__ void __launch_bounds__(THREADS) select_cta_kernel(const SelArgs a) {
    constexpr int SEL_CTA_WARPS = THREADS / 32;
    extern __shared__ uint32_t keys_s[];  // [n_past]
    __shared__ int covered;
    __shared__ int seg_cnt[2][SEL_CTA_WARPS];
    const unsigned FULL = 0xffffffffu;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int row = blockIdx.x;
    const int n_past = a.n_past, m = a.m, k_past = a.k_past;
    const float* sc = a.scores + static_cast<size_t>(row) * n_past;
    int32_t* out = a.idx + static_cast<size_t>(row) * a.topk;
    for (int i = t; i < m; i += THREADS) out[k_past + i] = n_past + i;
    if (k_past <= 0) return;  // uniform across the CTA
    if (k_past >= n_past) {
        for (int i = t; i < n_past; i += THREADS) out[i] = i;
        return;
    }
    // launched as the scorer's dependent: scores (and counts) only after it is done
    asm volatile("griddepcontrol.wait;" ::: "memory");
    RowMod mod{nullptr, a.alpha, a.invT, 1.0f / static_cast<float>(a.m)};
    if (warp == 0) {
        const RowMod w = row_mod(a, row, lane);
        if (lane == 0) covered = w.cnt ? 1 : 0;
    }
    __syncthreads();
    if (covered && a.counts) {
        const int qb = row % a.m;
        const int b = (row / a.m) / a.H;
        mod.cnt = a.counts + (static_cast<size_t>(b) * a.m + qb) * a.P;
    }
    uint32_t key[CH];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const int i = c * THREADS + t;
        key[c] = i < n_past ? order_key(mod(__ldg(sc + i), i)) : 0u;
        if (i < n_past) keys_s[i] = key[c];
    }
    uint32_t u;
    {
        // 8-bit digits from the top: per round a 256-bin histogram of the digits
        // of the keys that still match the chosen prefix (equal digits within a
        // warp are added by one atomic), then warp 0 finds the digit that holds
        // the remaining-th largest key by a scan from the top bin down
        __shared__ __align__(16) int hist[256];
        __shared__ int pick[2];
        uint32_t prefix = 0, pmask = 0;
        int remaining = k_past;
#pragma unroll 1
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = t; i < 256; i += THREADS) hist[i] = 0;
            __syncthreads();
#pragma unroll
            for (int c = 0; c < CH; ++c) {
                const int i = c * THREADS + t;
                const bool in = i < n_past && (key[c] & pmask) == prefix;
                const int dg = in ? static_cast<int>((key[c] >> shift) & 255u) : -1;
                const unsigned peers = __match_any_sync(FULL, dg);
                if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[dg], __popc(peers));
            }
            __syncthreads();
            if (warp == 0) {
                // lane L takes bins 255-8L down to 248-8L: 32 contiguous bytes
                const int4 lo = reinterpret_cast<const int4*>(hist)[62 - 2 * lane];
                const int4 hi = reinterpret_cast<const int4*>(hist)[63 - 2 * lane];
                const int cnt[8] = {hi.w, hi.z, hi.y, hi.x, lo.w, lo.z, lo.y, lo.x};
                int tot = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) tot += cnt[q];
                int incl = tot;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(FULL, incl, o);
                    if (lane >= o) incl += v;
                }
                const int excl = incl - tot;
                if (excl < remaining && remaining <= incl) {  // exactly one lane
                    int acc = excl;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (acc + cnt[q] >= remaining) {
                            pick[0] = 255 - 8 * lane - q;
                            pick[1] = acc;
                            break;
                        }
                        acc += cnt[q];
                    }
                }
            }
            __syncthreads();
            remaining -= pick[1];
            prefix |= static_cast<uint32_t>(pick[0]) << shift;
            pmask |= 0xFFu << shift;
            __syncthreads();  // pick and hist are rewritten next round
        }
        u = prefix;
    }
    // emission: warp w owns keys [s0, s1) of the row
    const unsigned lt = (1u << lane) - 1u;
    const int seg = ((n_past + THREADS - 1) / THREADS) * 32;
    const int s0 = min(n_past, warp * seg), s1 = min(n_past, s0 + seg);
    unsigned gt = 0, eq = 0;
    for (int i = s0 + lane; i < s1; i += 32) {
        const uint32_t k = keys_s[i];
        gt += k > u ? 1u : 0u;
        eq += k == u ? 1u : 0u;
    }
    gt = __reduce_add_sync(FULL, gt);
    eq = __reduce_add_sync(FULL, eq);
    if (lane == 0) {
        seg_cnt[0][warp] = static_cast<int>(gt);
        seg_cnt[1][warp] = static_cast<int>(eq);
    }
    __syncthreads();
    int gt_total = 0, gt_before = 0, eq_before = 0;
#pragma unroll
    for (int w = 0; w < SEL_CTA_WARPS; ++w) {
        gt_total += seg_cnt[0][w];
        if (w < warp) {
            gt_before += seg_cnt[0][w];
            eq_before += seg_cnt[1][w];
        }
    }
    const int remaining = k_past - gt_total;  // equal keys taken, smallest indices first
    int written = gt_before + min(eq_before, remaining);
    int eq_seen = eq_before;
    for (int base = s0; base < s1; base += 32) {
        const int i = base + lane;
        const uint32_t k = i < s1 ? keys_s[i] : 0u;
        const bool is_eq = i < s1 && k == u;
        const unsigned eqb = __ballot_sync(FULL, is_eq);
        const bool take = (i < s1 && k > u) || (is_eq && (eq_seen + __popc(eqb & lt)) < remaining);
        const unsigned tb = __ballot_sync(FULL, take);
        if (take) out[written + __popc(tb & lt)] = i;
        written += __popc(tb);
        eq_seen += __popc(eqb);
    }
}

// A kernel launched as the programmatic dependent of the one before it in the
// stream: its CTAs may be scheduled while that grid still runs, and wait for it
// with griddepcontrol.wait before they read what it writes.
template <typename Kern, typename... Args>
cudaError_t launch_dependent(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             const Args&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// the selection, launched as the dependent of the scorer
int select_launch(const SelArgs& a, cudaStream_t st) {
    constexpr int TH = SEL_CTA_THREADS;
    const size_t smem = static_cast<size_t>(a.n_past) * sizeof(uint32_t);
    const dim3 grid(a.rows), block(TH);
    cudaError_t e;
    if (a.n_past <= TH * 1)
        e = launch_dependent(select_cta_kernel<TH, 1>, grid, block, smem, st, a);
    else if (a.n_past <= TH * 2)
        e = launch_dependent(select_cta_kernel<TH, 2>, grid, block, smem, st, a);
    else if (a.n_past <= TH * 4)
        e = launch_dependent(select_cta_kernel<TH, 4>, grid, block, smem, st, a);
    else if (a.n_past <= TH * 8)
        e = launch_dependent(select_cta_kernel<TH, 8>, grid, block, smem, st, a);
    else if (a.n_past <= TH * 16)
        e = launch_dependent(select_cta_kernel<TH, 16>, grid, block, smem, st, a);
    else
        e = launch_dependent(select_kernel, dim3((a.rows + SEL_WARPS - 1) / SEL_WARPS),
                             dim3(SEL_WARPS * 32), 0, st, a);
    return e == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

template <typename TIn, int D, int T>
int route_typed(const TIn* q, const TIn* k, const RouteArgs& r, cudaStream_t st) {
    using V = VecTraits<TIn>;
    const int BH = r.B * r.H;
    RouteArgs rc = r;
    if (!r.kbar && r.kbar_ws && r.n_past > 0) {
        // split scoring: every past key block is pooled first (pure streaming,
        // one warp per block), then scored from the pooled keys like a cache
        kbar_append_kernel<TIn, D, T><<<dim3((r.n_past + POOL_THREADS / 32 - 1) / (POOL_THREADS / 32), BH),
                                        POOL_THREADS, 0, st>>>(k, r.Nk, r.Nq, r.n_past, 0, r.n_past,
                                                               r.kbar_ws);
        rc.kbar = r.kbar_ws;
        rc.kbar_cap = r.n_past;
    }
    pool_q_kernel<TIn, D, T><<<BH * r.m, POOL_THREADS, 0, st>>>(q, r.qbar);
    if (r.n_past > 0) {
        if (rc.kbar) {
            const size_t smem =
                (static_cast<size_t>(r.m) * D + static_cast<size_t>(SC_KT) * (D + 4)) * sizeof(float);
            auto sk = score_cached_kernel<TIn, D>;
            if (smem > 227 * 1024) return VELOX_EUNSUPPORTED;
            if (smem > 48 * 1024 &&
                cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)) != cudaSuccess)
                return VELOX_ECUDA;
            sk<<<dim3((r.n_past + SC_KT - 1) / SC_KT, BH), 256, smem, st>>>(r.qbar, rc);
        } else {
        const size_t smem = static_cast<size_t>(r.m) * D * sizeof(float);
        auto kern = pool_score_kernel<TIn, D, T>;
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return VELOX_ECUDA;
        int dev = 0, sms = 148, occ = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, POOL_THREADS, smem) !=
                cudaSuccess ||
            occ < 1)
            occ = 1;
        // every CTA resident at once, and every warp with the same number of
        // key blocks (the fewest per warp that fit, then the fewest CTAs that
        // give it): the stream of K has no tail of half-busy SMs
        const int warps = POOL_THREADS / 32;
        const int gx_max = max(1, occ * sms / BH);
        const int per_warp = (r.n_past + warps * gx_max - 1) / (warps * gx_max);
        const int gx = max(1, (r.n_past + warps * per_warp - 1) / (warps * per_warp));
        // launched as pool_q's programmatic dependent (see pool_score_kernel)
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(gx, BH);
        cfg.blockDim = dim3(POOL_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, kern, k, static_cast<const float*>(r.qbar), r) != cudaSuccess)
            return VELOX_ECUDA;
        }
    }
    // the counts are read by the selection only: it may wait for them alone
    if (r.counts_ready && cudaStreamWaitEvent(st, r.counts_ready, 0) != cudaSuccess)
        return VELOX_ECUDA;
    SelArgs sa{r.scores, BH * r.m, r.n_past, r.m, r.H, r.P, r.topk - r.m, r.topk,
               r.counts, r.alpha, 1.0f / static_cast<float>(T), r.idx};
    if (select_launch(sa, st) != VELOX_OK) return VELOX_ECUDA;
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

template <typename TIn, int D, int T>
int append_typed(const TIn* k, int BH, int Nk, int Nq, int chunk, int cap, float* kbar,
                 cudaStream_t st) {
    const int m = Nq / T;
    const int warps = POOL_THREADS / 32;
    kbar_append_kernel<TIn, D, T><<<dim3((m + warps - 1) / warps, BH), POOL_THREADS, 0, st>>>(
        k, Nk, Nq, m, chunk, cap, kbar);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

template <typename TIn>
int append_dispatch(const void* k, int BH, int Nk, int Nq, int d, int T, int chunk, int cap,
                    float* kbar, cudaStream_t st) {
    const TIn* tk = static_cast<const TIn*>(k);
    if (d == 128 && T == 128) return append_typed<TIn, 128, 128>(tk, BH, Nk, Nq, chunk, cap, kbar, st);
    if (d == 128 && T == 64) return append_typed<TIn, 128, 64>(tk, BH, Nk, Nq, chunk, cap, kbar, st);
    if (d == 64 && T == 128) return append_typed<TIn, 64, 128>(tk, BH, Nk, Nq, chunk, cap, kbar, st);
    if (d == 64 && T == 64) return append_typed<TIn, 64, 64>(tk, BH, Nk, Nq, chunk, cap, kbar, st);
    return VELOX_EUNSUPPORTED;
}

}  // namespace

int kbar_append_launch(const void* k, int dtype, int BH, int Nk, int Nq, int d, int T, int chunk,
                       int cap, float* kbar, cudaStream_t st) {
    if (dtype == VELOX_BF16)
        return append_dispatch<__nv_bfloat16>(k, BH, Nk, Nq, d, T, chunk, cap, kbar, st);
    if (dtype == VELOX_F32) return append_dispatch<float>(k, BH, Nk, Nq, d, T, chunk, cap, kbar, st);
    return VELOX_EUNSUPPORTED;
}

// With 64-token blocks a key block is half as many bytes and meets twice as
// many query blocks, so pool_score spends four times the time per byte of K
// scoring, with no loads in flight, and streams K at under half of HBM. There
// the scoring is split off: kbar_append pools every past block (one warp per
// block, nothing else to do) and score_cached scores them from shared-memory
// tiles. The split costs the pooled keys' round trip (B*H*n_past*d floats,
// written and read once), so 128-token blocks keep the fused scorer (measured
// at 20 % of the key blocks: T 64 d 128 P 48 467 -> 358 us, P 8 101 -> 79;
// T 64 d 64 P 48 271 -> 207; T 128 d 128 P 48 225 -> 244 had it been split).
bool route_split_scoring(int T, int d) {
    (void)d;
    return T == 64;
}

size_t route_ws_bytes(int B, int H, int m, int n_past, int d, int T) {
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t rows = static_cast<size_t>(B) * H * m;
    size_t bytes = up(rows * d * sizeof(float)) + up(rows * static_cast<size_t>(n_past) * sizeof(float));
    if (route_split_scoring(T, d))
        bytes += up(static_cast<size_t>(B) * H * n_past * d * sizeof(float));
    return bytes;
}

int route_launch(const void* q, const void* k, int dtype, const RouteArgs& r, cudaStream_t st) {
    if (dtype == VELOX_BF16) return route_dispatch<__nv_bfloat16>(q, k, r, st);
    if (dtype == VELOX_F32) return route_dispatch<float>(q, k, r, st);
    return VELOX_EUNSUPPORTED;
}

}  // namespace velox
