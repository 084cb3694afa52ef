// Block-sparse attention forward for sm_100a, two query blocks per CTA
// (head dim 128, 128-token blocks).
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse" -- each query block attends only to the key blocks routed to
// it, at the granularity of the attention tile. Here a CTA owns two adjacent
// query blocks A and B of one (batch, head), each with its own list of key
// blocks, and interleaves them on the tensor core:
//
//   S_A(i) = Q_A K_A(i)^T,  O_B += P_B(i-1) V_B(i-1),  S_B(i) = Q_B K_B(i)^T,
//   O_A += P_A(i) V_A(i),   S_A(i+1) ...
//
// While one block's softmax turns S into P, the tensor core works on the
// other block, so neither the exponentials nor the S -> P -> PV round trip
// leave it idle.
//
// CTA = 12 warps (three warpgroups):
//   warps 0-3   softmax / correction / epilogue of block A (row = TMEM lane)
//   warps 4-7   the same for block B
//   warp 8      TMA producer of the K tiles, in consumption order A0 B0 A1 B1 ...
//               (2-deep ring: one slot per block)
//   warp 9      tcgen05 issuer (one thread)
//   warp 10     TMA producer of the V tiles, same order
//   warp 11     idle
// Shared memory: Q_A, Q_B (32 KB each), K ring (2 x 32 KB), V ring (2 x 32 KB),
// all 128-byte swizzled. Tensor memory (512 columns): S_A, S_B (128 fp32
// columns each; P, as bf16 pairs, overwrites the upper half of S once S has
// been read), O_A, O_B (128 fp32 columns each).
// Ordering: S_t(i+1) overwrites the P_t(i) that O_t += P_t(i) V_t(i) reads;
// the issuing thread issues the P V first, and MMAs from one thread execute
// in issue order. A commit tracks every MMA issued before it, so S_t(i+1)
// complete implies O_t += P_t(i) V_t(i) complete. P V is issued in two halves
// of the keys: the softmax stores the P of keys 64-127 first (their scores are
// still in registers after the row max) and releases them at once, so the
// tensor core works on that half while the softmax computes the other.
#include "attn_common.cuh"

namespace velox {

namespace {

constexpr int PP_THREADS = 384;
constexpr int PP_D = 128;
constexpr int PP_BN = 128;
constexpr int PP_KST = 2;
constexpr int PP_VST = 2;
constexpr int PP_WARP_TMA_K = 8;
constexpr int PP_WARP_MMA = 9;
constexpr int PP_WARP_TMA_V = 10;

struct PPLayout {
    static constexpr int TILE = 128 * 128 * 2;  // a Q, K or V tile: 128 rows x 128 bf16
    static constexpr int OFF_Q = 0;             // Q_A, Q_B
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + PP_KST * TILE;
    static constexpr int OFF_BAR = OFF_V + PP_VST * TILE;
    // q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_full[2],
    // pv_done[2], p_half[2], mma_drain
    static constexpr int NBAR = 1 + 2 * PP_KST + 2 * PP_VST + 9;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
    static_assert(SMEM <= 232448, "shared memory budget");
    static constexpr int TMEM_COLS = 512;      // S_A, S_B, O_A, O_B
    static constexpr int TMEM_O = 256;
    static constexpr int P_OFF = 64;           // P inside S: columns 64..127
};

struct PPBars {
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    __device__ uint32_t k_full(int s) const { return base + 8 * (1 + s); }
    __device__ uint32_t k_empty(int s) const { return base + 8 * (1 + PP_KST + s); }
    __device__ uint32_t v_full(int s) const { return base + 8 * (1 + 2 * PP_KST + s); }
    __device__ uint32_t v_empty(int s) const { return base + 8 * (1 + 2 * PP_KST + PP_VST + s); }
    static constexpr int R = 1 + 2 * PP_KST + 2 * PP_VST;
    __device__ uint32_t s_full(int t) const { return base + 8 * (R + t); }
    __device__ uint32_t p_full(int t) const { return base + 8 * (R + 2 + t); }
    __device__ uint32_t pv_done(int t) const { return base + 8 * (R + 4 + t); }
    __device__ uint32_t p_half(int t) const { return base + 8 * (R + 6 + t); }
    __device__ uint32_t mma_drain() const { return base + 8 * (R + 8); }
};

// exponentials of 64 scores (one half row) in place, sums into sum2. Every
// exponential goes to the ex2 unit here: with two blocks in flight the
// softmax has slack, and moving part of them to the FMA pipe (as the
// single-block kernel does) only adds issue pressure (measured on the chunk-48
// walk: none of the pairs emulated 1,171 TFLOP/s, 3/8 1,152, 4/8 1,091).
__device__ __forceinline__ void exp_half(float* s, float sl2, float m, float2* sum2) {
    const float2 sc2 = make_float2(sl2, sl2);
    const float2 ng2 = make_float2(-m, -m);
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
        float2 x = __ffma2_rn(make_float2(s[i], s[i + 1]), sc2, ng2);
        x.x = ex2_approx(x.x);
        x.y = ex2_approx(x.y);
        s[i] = x.x;
        s[i + 1] = x.y;
        sum2[(i >> 1) & 3] = __fadd2_rn(sum2[(i >> 1) & 3], x);
    }
}

// 64 probabilities -> 32 bf16 pairs in tensor memory at column `t_p`
__device__ __forceinline__ void store_p_half(uint32_t t_p, const float* s) {
    float pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = __uint_as_float(pack_bf16x2(s[2 * i], s[2 * i + 1]));
    tmem_st32(t_p, pk);
}

__global__ void __launch_bounds__(PP_THREADS, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
    using L = PPLayout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qb_a = 2 * blockIdx.x;
    const bool has_b = qb_a + 1 < a.m;
    const int bh = blockIdx.z * a.H + blockIdx.y;
    const int n = a.n_sel;
    const int ntile = has_b ? 2 : 1;

    PPBars bars{sbase + L::OFF_BAR};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bars.q_full(), 1);
        for (int s = 0; s < PP_KST; ++s) {
            mbar_init(bars.k_full(s), 1);
            mbar_init(bars.k_empty(s), 1);
        }
        for (int s = 0; s < PP_VST; ++s) {
            mbar_init(bars.v_full(s), 1);
            mbar_init(bars.v_empty(s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars.s_full(t), 1);
            mbar_init(bars.p_full(t), 4);  // one elected arrive per softmax warp
            mbar_init(bars.p_half(t), 4);
            mbar_init(bars.pv_done(t), 1);
        }
        mbar_init(bars.mma_drain(), 1);
        fence_mbar_init();
    }
    if (warp == PP_WARP_MMA) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == PP_WARP_TMA_K && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == PP_WARP_TMA_K || warp == PP_WARP_TMA_V) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            const bool is_v = warp == PP_WARP_TMA_V;
            const int nst = is_v ? PP_VST : PP_KST;
            const CUtensorMap* tm = is_v ? &tmV : &tmK;
            const uint32_t ring = sbase + (is_v ? L::OFF_V : L::OFF_K);
            auto full = [&](int st) { return is_v ? bars.v_full(st) : bars.k_full(st); };
            auto empty = [&](int st) { return is_v ? bars.v_empty(st) : bars.k_empty(st); };
            if (!is_v) {
                const int qrow = bh * a.Nq + qb_a * PP_BN;
                mbar_arrive_expect_tx(bars.q_full(), ntile * L::TILE);
                for (int t = 0; t < ntile; ++t) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        tma_load_2d(sbase + L::OFF_Q + t * L::TILE + c * (128 * 128), &tmQ,
                                    bars.q_full(), c * 64, qrow + t * PP_BN);
                }
            }
            const int krow0 = bh * a.Nk;
            auto fetch = [&](int t, int i) -> int {
                if (!a.idx) return i;
                const int32_t* row =
                    a.idx + (static_cast<size_t>(bh) * a.m + qb_a + t) * static_cast<size_t>(n);
                int kb = __ldg(row + i);
                if (kb < 0 || kb >= a.n_kb) {
                    if (a.status && !is_v) atomicOr(a.status, VELOX_STATUS_BAD_INDEX);
                    kb = 0;
                }
                return kb;
            };
            const int total = n * ntile;  // loads in order A0 B0 A1 B1 ...
            int issued = 0;
            int kb = fetch(0, 0);
            for (int l = 0; l < total; ++l) {
                const int st = l % nst;
                const int nl = l + 1;
                const int kb_next = nl < total ? fetch(nl % ntile, nl / ntile) : 0;
                if (l >= nst) {
                    // With two blocks each ring holds one tile per block, so a slot
                    // is free once that block's previous S (or P V) is complete:
                    // wait on that completion barrier (it cannot run two phases
                    // ahead: the block's next GEMM needs the tile loaded here). A
                    // single-block CTA has per-slot barriers instead.
                    uint32_t bar, par;
                    if (ntile == 2) {
                        const int pt = l & 1, pi = (l - 2) >> 1;
                        bar = is_v ? bars.pv_done(pt) : bars.s_full(pt);
                        par = static_cast<uint32_t>(pi & 1);
                    } else {
                        bar = empty(st);
                        par = static_cast<uint32_t>(((l / nst) - 1) & 1);
                    }
                    if (!mbar_wait(bar, par, abort_flag, a.wait_ns)) break;
                }
                mbar_arrive_expect_tx(full(st), L::TILE);
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    tma_load_2d(ring + st * L::TILE + c * (128 * 128), tm, full(st), c * 64,
                                krow0 + kb * PP_BN);
                issued = l + 1;
                kb = kb_next;
            }
            // copies still in flight (only possible after an abort) land before exit
            if (!is_v) drain_wait(bars.q_full(), 0);
            for (int l = issued - 1; l >= 0 && l >= issued - nst; --l)
                drain_wait(full(l % nst), (l / nst) & 1);
        }
    } else if (warp == PP_WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // (with the skip_mma test hook it issues nothing: every wait on an MMA
        // completion then runs out, and the kernel reports the timeout)
        if (lane == 0 && !a.skip_mma) {
            constexpr uint32_t ID_S = idesc_bf16_f32(128, PP_BN, false, false);
            constexpr uint32_t ID_PV = idesc_bf16_f32(128, PP_D, false, true);
            bool ok = mbar_wait(bars.q_full(), 0, abort_flag, a.wait_ns);
            tc_fence_after();
            int kl = 0, vl = 0;
            auto issue_s = [&](int t) -> bool {
                const int st = kl % PP_KST;
                if (!mbar_wait(bars.k_full(st), (kl / PP_KST) & 1, abort_flag, a.wait_ns))
                    return false;
                tc_fence_after();
                const uint32_t d = tmem + t * 128;
#pragma unroll
                for (int kk = 0; kk < PP_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sbase + L::OFF_Q + t * L::TILE + off, 16);
                    const uint64_t bd = smem_desc_sw128(sbase + L::OFF_K + st * L::TILE + off, 16);
                    mma_bf16_ss(d, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                }
                if (!has_b) mma_commit(bars.k_empty(st));
                mma_commit(bars.s_full(t));
                ++kl;
                return true;
            };
            // O_t += P_t(i) V_t(i) in two halves of the keys: keys 64-127 as soon as
            // the softmax has stored their P (p_half), keys 0-63 once all of P is
            // stored (p_full), so the tensor core starts on P V while the softmax
            // still computes the rest of P
            auto issue_pv = [&](int t, int i) -> bool {
                const int st = vl % PP_VST;
                if (!mbar_wait(bars.v_full(st), (vl / PP_VST) & 1, abort_flag, a.wait_ns))
                    return false;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t bar = h == 0 ? bars.p_half(t) : bars.p_full(t);
                    if (!mbar_wait(bar, i & 1, abort_flag, a.wait_ns)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < PP_BN / 32; ++j) {
                        const int kk = (h == 0 ? PP_BN / 32 : 0) + j;
                        const uint32_t at = tmem + t * 128 + L::P_OFF + kk * 8;
                        const uint64_t bd = smem_desc_sw128(
                            sbase + L::OFF_V + st * L::TILE + kk * (16 * 128), PP_BN * 128);
                        mma_bf16_ts(tmem + L::TMEM_O + t * 128, at, bd, ID_PV,
                                    (i > 0 || h > 0 || j > 0) ? 1u : 0u);
                    }
                }
                if (!has_b) mma_commit(bars.v_empty(st));
                mma_commit(bars.pv_done(t));
                ++vl;
                return true;
            };
            for (int i = 0; ok && i < n; ++i) {
                if (!issue_s(0)) break;
                if (has_b && i > 0 && !issue_pv(1, i - 1)) break;
                if (has_b && !issue_s(1)) break;
                if (!issue_pv(0, i)) break;
                if (has_b && i == n - 1) issue_pv(1, i);
            }
            // every MMA issued above has completed before this thread leaves (on
            // an abort, too), so none is in flight when tensor memory is freed
            mma_commit(bars.mma_drain());
            drain_wait(bars.mma_drain(), 0);
        }
    } else if (warp < 8 && (warp < 4 || has_b)) {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp >> 2;  // 0 = block A, 1 = block B
        const int qb = qb_a + t;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + t * 128;
        const uint32_t t_o = tmem + lane_base + L::TMEM_O + t * 128;
        const float sl2 = a.scale_log2;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            if (!warp_wait(bars.s_full(t), i & 1, abort_flag, a.wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // pass 1: row max over the two halves of S (columns 0-63, then 64-127)
            float s[64];
            float acc[8];
            tmem_ld32(t_s, s);
            tmem_ld32(t_s + 32, s + 32);
            tmem_wait_ld();
            reg_fence32(s);
            reg_fence32(s + 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = s[k];
            max_range<8, 64>(s, acc);
            tmem_ld32(t_s + 64, s);
            tmem_ld32(t_s + 96, s + 32);
            tmem_wait_ld();
            reg_fence32(s);
            reg_fence32(s + 32);
            max_range<0, 64>(s, acc);
            float mx = max3f(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], acc[5]),
                             fmaxf(acc[6], acc[7]));
            mx *= sl2;
            float m_new = m_run;
            bool resc = false;
            if (mx > m_run + RESCALE_THRESHOLD) {
                m_new = mx;
                resc = (i > 0);
            }
            float f = 1.f;
            if (__any_sync(0xffffffffu, resc)) {
                // O must hold P(i-1) V(i-1) before it is rescaled in place, and the
                // rescale must land before P(i) V(i) starts accumulating
                if (!warp_wait(bars.pv_done(t), (i - 1) & 1, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                f = resc ? ex2_approx(m_run - m_new) : 1.f;
#pragma unroll 1
                for (int c = 0; c < PP_D / 32; ++c) {
                    float o[32];
                    tmem_ld32(t_o + c * 32, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] *= f;
                    tmem_st32(t_o + c * 32, o);
                }
                tmem_wait_st();
            }
            // pass 2: the second half is in registers; its P goes to columns 96-127
            // (S columns already read) and is released to the tensor core at once;
            // then the first half is read again and its P goes to columns 64-95
            float2 sum2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) sum2[k] = make_float2(0.f, 0.f);
            exp_half(s, sl2, m_new, sum2);
            store_p_half(t_s + L::P_OFF + 32, s);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_half(t));  // P(i) of keys 64-127, (rescaled) O
            tmem_ld32(t_s, s);
            tmem_ld32(t_s + 32, s + 32);
            tmem_wait_ld();
            reg_fence32(s);
            reg_fence32(s + 32);
            exp_half(s, sl2, m_new, sum2);
            store_p_half(t_s + L::P_OFF, s);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_full(t));  // all of P(i)
            const float2 s01 = __fadd2_rn(sum2[0], sum2[1]);
            const float2 s23 = __fadd2_rn(sum2[2], sum2[3]);
            const float2 s03 = __fadd2_rn(s01, s23);
            l_run = l_run * f + (s03.x + s03.y);
            m_run = m_new;
        }
        if (ok && n > 0 && warp_wait(bars.pv_done(t), (n - 1) & 1, abort_flag, a.wait_ns)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const size_t grow = static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(qb) * PP_BN + row;
            __nv_bfloat16* orow = a.o + grow * PP_D;
#pragma unroll 1
            for (int c = 0; c < PP_D / 32; ++c) {
                float o[32];
                tmem_ld32(t_o + c * 32, o);
                tmem_wait_ld();
                reg_fence32(o);
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float* p = o + u * 8;
                    dst[u] = make_uint4(pack_bf16x2(p[0] * inv, p[1] * inv),
                                        pack_bf16x2(p[2] * inv, p[3] * inv),
                                        pack_bf16x2(p[4] * inv, p[5] * inv),
                                        pack_bf16x2(p[6] * inv, p[7] * inv));
                }
            }
            if (a.lse) a.lse[grow] = (m_run + log2f(l_run)) * 0.69314718055994531f;
        }
    }

    if (threadIdx.x == 0 && *abort_flag && a.status) atomicOr(a.status, VELOX_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == PP_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace

int attn_pp_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                   cudaStream_t st) {
    using L = PPLayout;
    CUtensorMap tq, tk, tv;
    const uint64_t bh = static_cast<uint64_t>(B) * a.H;
    if (!make_tmap(&tq, q, bh * a.Nq, PP_D, 128) || !make_tmap(&tk, k, bh * a.Nk, PP_D, PP_BN) ||
        !make_tmap(&tv, v, bh * a.Nk, PP_D, PP_BN))
        return VELOX_ECUDA;
    if (cudaFuncSetAttribute(attn_pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) !=
        cudaSuccess)
        return VELOX_ECUDA;
    dim3 grid((a.m + 1) / 2, a.H, B);
    attn_pp_kernel<<<grid, PP_THREADS, L::SMEM, st>>>(tq, tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

}  // namespace velox
