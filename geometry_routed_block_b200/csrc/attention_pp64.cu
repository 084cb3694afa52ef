// Block-sparse attention forward for sm_100a with 64-token blocks (head dim
// 128): two 128-row query tiles per CTA, each tile two query blocks.
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse" -- each query block attends only to the key blocks routed to
// it. A 64-token block is half of what one tcgen05 MMA covers (M = 128), so:
//
//   * a 128-row query tile holds two adjacent query blocks; they walk the
//     union of their two routed lists (ascending, each entry tagged with the
//     blocks that listed it), and scores of a key block that a query block did
//     not list get probability zero, so each query block sees its own list
//     and nothing else;
//   * a 128-key K or V tile holds two consecutive entries of that walk,
//     fetched as two 64-row boxes into the halves of the tile (the halves are
//     1024-byte aligned, so the 128-byte swizzle of the tile is that of one
//     128-row box and the MMAs are those of 128-token blocks). A walk of odd
//     length ends with a half that no query block listed.
//
// The CTA owns two such tiles, A (query blocks 4c, 4c + 1) and B (4c + 2,
// 4c + 3), and interleaves them on the tensor core as the 128-token
// two-block kernel does:
//
//   S_A(i) = Q_A K_A(i)^T,  O_B += P_B(i-1) V_B(i-1),  S_B(i) = Q_B K_B(i)^T,
//   O_A += P_A(i) V_A(i),   S_A(i+1) ...
//
// The two walks may differ in length; once the shorter one ends, the other
// tile runs on alone.
//
// CTA = 12 warps:
//   warps 0-3   softmax / correction / epilogue of tile A (row = TMEM lane;
//               warps 0-1 query block 4c, warps 2-3 query block 4c + 1)
//   warps 4-7   the same for tile B
//   warp 8      barrier set-up, Q loads, TMA producer of the K tiles
//   warp 9      tcgen05 issuer (one thread)
//   warp 10     builds tile A's walk, then TMA producer of the V tiles
//   warp 11     builds tile B's walk
// Shared memory: Q_A, Q_B, one K and one V tile per query tile (32 KB each,
// 128-byte swizzled), the two walks (16-bit entries) and their bitmaps.
// Tensor memory (512 columns): S_A, S_B (P as bf16 pairs overwrites the upper
// half of S once S has been read), O_A, O_B.
#include "attn_common.cuh"

namespace velox {

namespace {

constexpr int Q4_THREADS = 384;
constexpr int Q4_D = 128;
constexpr int Q4_T = 64;
constexpr int Q4_WARP_TMA_K = 8;
constexpr int Q4_WARP_MMA = 9;
constexpr int Q4_WARP_TMA_V = 10;
constexpr int Q4_WARP_WALK_B = 11;
constexpr int Q4_WALK_MAX = 4096;  // walk entries per tile: two lists of up to 2048 blocks
constexpr int Q4_WORDS = 512;      // bitmap words per list: up to 16384 key blocks
constexpr int Q4_KB_BITS = 14;     // a walk entry: key block (14 bits) | mask << 14
constexpr int Q4_KB_MASK = (1 << Q4_KB_BITS) - 1;

struct Q4Layout {
    static constexpr int TILE = 128 * 128 * 2;       // 128 rows x 128 bf16
    static constexpr int HALF = 64 * 128;            // 64 rows of one 64-column chunk
    static constexpr int OFF_Q = 0;                  // Q_A, Q_B
    static constexpr int OFF_K = 2 * TILE;           // K_A, K_B
    static constexpr int OFF_V = 4 * TILE;           // V_A, V_B
    static constexpr int OFF_WALK = 6 * TILE;        // uint16 [2][WALK_MAX]
    static constexpr int OFF_BITMAP = OFF_WALK + 2 * Q4_WALK_MAX * 2;  // uint32 [2][2][WORDS]
    static constexpr int OFF_BAR = OFF_BITMAP + 2 * 2 * Q4_WORDS * 4;
    // q_full, k_full[2], v_full[2], s_full[2], p_full[2], pv_done[2], p_half[2], mma_drain
    static constexpr int NBAR = 14;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, walk lengths[2]
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(OFF_BAR % 8 == 0, "barrier alignment");
    static constexpr int TMEM_COLS = 512;
    static constexpr int TMEM_O = 256;
    static constexpr int P_OFF = 64;
};

struct Q4Bars {
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    __device__ uint32_t k_full(int t) const { return base + 8 * (1 + t); }
    __device__ uint32_t v_full(int t) const { return base + 8 * (3 + t); }
    __device__ uint32_t s_full(int t) const { return base + 8 * (5 + t); }
    __device__ uint32_t p_full(int t) const { return base + 8 * (7 + t); }
    __device__ uint32_t pv_done(int t) const { return base + 8 * (9 + t); }
    __device__ uint32_t p_half(int t) const { return base + 8 * (11 + t); }
    __device__ uint32_t mma_drain() const { return base + 8 * 13; }
};

// 2^(x * sl2 - m) of 64 scores in place, sums into sum2 (4 chains of pairs)
__device__ __forceinline__ void exp64(float* s, float sl2, float m, float2* sum2) {
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

// 64 probabilities -> 32 bf16 pairs at tensor-memory column t_p
__device__ __forceinline__ void store_p64(uint32_t t_p, const float* s) {
    float pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = __uint_as_float(pack_bf16x2(s[2 * i], s[2 * i + 1]));
    tmem_st32(t_p, pk);
}

// probability zero for 64 keys the row's query block did not list
__device__ __forceinline__ void store_zero_p64(uint32_t t_p) {
    float z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0.f;
    tmem_st32(t_p, z);
}

__global__ void __launch_bounds__(Q4_THREADS, 1)
    attn_pp64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
    using L = Q4Layout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qb0 = 4 * blockIdx.x;           // first query block of tile A
    const int nq = min(4, a.m - qb0);         // query blocks of this CTA (1..4)
    const bool has_b = nq > 2;
    const int bh = blockIdx.z * a.H + blockIdx.y;
    const bool use_walk = a.idx != nullptr;

    Q4Bars bars{sbase + L::OFF_BAR};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    int* walk_len = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);
    uint16_t* walk = reinterpret_cast<uint16_t*>(smem + L::OFF_WALK);

    if (warp == Q4_WARP_TMA_K && lane == 0) {
        *abort_flag = 0;
        mbar_init(bars.q_full(), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars.k_full(t), 1);
            mbar_init(bars.v_full(t), 1);
            mbar_init(bars.s_full(t), 1);
            mbar_init(bars.p_full(t), 4);  // one elected arrive per softmax warp
            mbar_init(bars.p_half(t), 4);
            mbar_init(bars.pv_done(t), 1);
        }
        mbar_init(bars.mma_drain(), 1);
        fence_mbar_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        // Q of the CTA's query blocks (the rows of a missing fourth or third
        // block are never loaded; their P is zero and they are not stored)
        mbar_arrive_expect_tx(bars.q_full(), nq * 2 * L::HALF);
        const int qrow = bh * a.Nq + qb0 * Q4_T;
        for (int g = 0; g < nq; ++g) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
                tma_load_2d(sbase + L::OFF_Q + (g >> 1) * L::TILE + c * (128 * 128) +
                                (g & 1) * L::HALF,
                            &tmQ, bars.q_full(), c * 64, qrow + g * Q4_T);
        }
    }
    if (use_walk && (warp == Q4_WARP_TMA_V || (warp == Q4_WARP_WALK_B && has_b))) {
        const int t = warp == Q4_WARP_TMA_V ? 0 : 1;
        const int qb = qb0 + 2 * t;
        uint32_t* bm = reinterpret_cast<uint32_t*>(smem + L::OFF_BITMAP) + t * 2 * Q4_WORDS;
        const int len = build_walk<Q4_WORDS, uint16_t, Q4_KB_BITS>(
            a, bh, qb, qb + 1 < a.m, bm, walk + t * Q4_WALK_MAX, lane);
        if (lane == 0) walk_len[t] = len;
    }
    if (warp == Q4_WARP_MMA) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // walk lengths (entries) and iterations (key tiles of two entries) per tile
    const int len0 = use_walk ? walk_len[0] : a.n_kb;
    const int len1 = !has_b ? 0 : (use_walk ? walk_len[1] : a.n_kb);
    const int n0 = (len0 + 1) >> 1;
    const int n1 = (len1 + 1) >> 1;
    auto entry_kb = [&](int t, int j) -> int {
        return use_walk ? (walk[t * Q4_WALK_MAX + j] & Q4_KB_MASK) : j;
    };

    if (warp == Q4_WARP_TMA_K || warp == Q4_WARP_TMA_V) {
        // ------------------------------------------------------------ producers
        // one slot per tile; the slot of tile t is free for K_t(i) once S_t(i-1)
        // is complete (for V_t(i), once O_t += P_t(i-1) V_t(i-1) is)
        if (lane == 0) {
            const bool is_v = warp == Q4_WARP_TMA_V;
            const CUtensorMap* tm = is_v ? &tmV : &tmK;
            const uint32_t ring = sbase + (is_v ? L::OFF_V : L::OFF_K);
            const int krow0 = bh * a.Nk;
            const int nmax = max(n0, n1);
            int last[2] = {-1, -1};
            bool ok = true;
            for (int i = 0; ok && i < nmax; ++i) {
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int nt = t ? n1 : n0;
                    const int len = t ? len1 : len0;
                    if (!ok || i >= nt) continue;
                    if (i > 0) {
                        const uint32_t bar = is_v ? bars.pv_done(t) : bars.s_full(t);
                        if (!mbar_wait(bar, static_cast<uint32_t>((i - 1) & 1), abort_flag,
                                       a.wait_ns)) {
                            ok = false;
                            continue;
                        }
                    }
                    const int kb0 = entry_kb(t, 2 * i);
                    const int kb1 = 2 * i + 1 < len ? entry_kb(t, 2 * i + 1) : kb0;
                    const uint32_t full = is_v ? bars.v_full(t) : bars.k_full(t);
                    const uint32_t dst = ring + t * L::TILE;
                    mbar_arrive_expect_tx(full, L::TILE);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        tma_load_2d(dst + c * (128 * 128), tm, full, c * 64, krow0 + kb0 * Q4_T);
                        tma_load_2d(dst + c * (128 * 128) + L::HALF, tm, full, c * 64,
                                    krow0 + kb1 * Q4_T);
                    }
                    last[t] = i;
                }
            }
            // copies still in flight (only possible after an abort) land before exit
            if (!is_v) drain_wait(bars.q_full(), 0);
#pragma unroll
            for (int t = 0; t < 2; ++t)
                if (last[t] >= 0)
                    drain_wait(is_v ? bars.v_full(t) : bars.k_full(t),
                               static_cast<uint32_t>(last[t] & 1));
        }
    } else if (warp == Q4_WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // (with the skip_mma test hook it issues nothing: every wait on an MMA
        // completion then runs out, and the kernel reports the timeout)
        if (lane == 0 && !a.skip_mma) {
            constexpr uint32_t ID_S = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t ID_PV = idesc_bf16_f32(128, Q4_D, false, true);
            bool ok = mbar_wait(bars.q_full(), 0, abort_flag, a.wait_ns);
            tc_fence_after();
            auto issue_s = [&](int t, int i) -> bool {
                if (!mbar_wait(bars.k_full(t), static_cast<uint32_t>(i & 1), abort_flag,
                               a.wait_ns))
                    return false;
                tc_fence_after();
                const uint32_t d = tmem + t * 128;
#pragma unroll
                for (int kk = 0; kk < Q4_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sbase + L::OFF_Q + t * L::TILE + off, 16);
                    const uint64_t bd = smem_desc_sw128(sbase + L::OFF_K + t * L::TILE + off, 16);
                    mma_bf16_ss(d, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(bars.s_full(t));
                return true;
            };
            // O_t += P_t(i) V_t(i) in two halves of the keys: the second entry's
            // 64 keys once the softmax has stored their P (p_half), the first
            // entry's once all of P is stored (p_full)
            auto issue_pv = [&](int t, int i) -> bool {
                if (!mbar_wait(bars.v_full(t), static_cast<uint32_t>(i & 1), abort_flag,
                               a.wait_ns))
                    return false;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t bar = h == 0 ? bars.p_half(t) : bars.p_full(t);
                    if (!mbar_wait(bar, static_cast<uint32_t>(i & 1), abort_flag, a.wait_ns))
                        return false;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int kk = (h == 0 ? 4 : 0) + j;
                        const uint32_t at = tmem + t * 128 + L::P_OFF + kk * 8;
                        const uint64_t bd = smem_desc_sw128(
                            sbase + L::OFF_V + t * L::TILE + kk * (16 * 128), 128 * 128);
                        mma_bf16_ts(tmem + L::TMEM_O + t * 128, at, bd, ID_PV,
                                    (i > 0 || h > 0 || j > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bars.pv_done(t));
                return true;
            };
            const int nmax = max(n0, n1);
            for (int i = 0; ok && i < nmax; ++i) {
                if (i < n0 && !issue_s(0, i)) break;
                if (i > 0 && i - 1 < n1 && !issue_pv(1, i - 1)) break;
                if (i < n1 && !issue_s(1, i)) break;
                if (i < n0 && !issue_pv(0, i)) break;
                if (i == nmax - 1 && n1 == nmax) issue_pv(1, i);
            }
            // every MMA issued above has completed before this thread leaves (on
            // an abort, too), so none is in flight when tensor memory is freed
            mma_commit(bars.mma_drain());
            drain_wait(bars.mma_drain(), 0);
        }
    } else if (warp < 8 && (warp < 4 || has_b)) {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp >> 2;             // 0 = tile A, 1 = tile B
        const int g = (warp >> 1) & 1;       // which of the tile's two query blocks
        const int qb = qb0 + 2 * t + g;
        const bool present = qb < a.m;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + t * 128;
        const uint32_t t_o = tmem + lane_base + L::TMEM_O + t * 128;
        const int nt = t ? n1 : n0;
        const int len = t ? len1 : len0;
        const uint16_t* wk = walk + t * Q4_WALK_MAX;
        // did this warp's query block list walk entry j (the same for the whole warp)
        auto listed = [&](int j) -> bool {
            if (!present || j >= len) return false;
            if (!use_walk) return true;
            return ((wk[j] >> (Q4_KB_BITS + g)) & 1) != 0;
        };
        const float sl2 = a.scale_log2;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int i = 0; i < nt; ++i) {
            const bool l0 = listed(2 * i), l1 = listed(2 * i + 1);
            if (!warp_wait(bars.s_full(t), i & 1, abort_flag, a.wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // pass 1: row max over the listed halves of S (first entry: columns
            // 0-63, second: 64-127); the last half read stays in registers
            float s[64];
            float acc[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = -INFINITY;
            if (l0) {
                tmem_ld32(t_s, s);
                tmem_ld32(t_s + 32, s + 32);
                tmem_wait_ld();
                reg_fence32(s);
                reg_fence32(s + 32);
                max_range<0, 64>(s, acc);
            }
            if (l1) {
                tmem_ld32(t_s + 64, s);
                tmem_ld32(t_s + 96, s + 32);
                tmem_wait_ld();
                reg_fence32(s);
                reg_fence32(s + 32);
                max_range<0, 64>(s, acc);
            }
            float mx = max3f(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], acc[5]),
                             fmaxf(acc[6], acc[7]));
            mx *= sl2;
            float m_new = m_run;
            bool resc = false;
            if (mx > m_run + RESCALE_THRESHOLD) {
                m_new = mx;
                // nothing to rescale while no listed key has been seen (O and
                // the row sum are still zero)
                resc = i > 0 && m_run > -INFINITY;
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
                for (int c = 0; c < Q4_D / 32; ++c) {
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
            // pass 2: P of the second entry to columns 96-127 (S columns already
            // read), released at once; then the first entry's P to columns 64-95
            float2 sum2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) sum2[k] = make_float2(0.f, 0.f);
            if (l1) {
                exp64(s, sl2, m_new, sum2);
                store_p64(t_s + L::P_OFF + 32, s);
            } else {
                store_zero_p64(t_s + L::P_OFF + 32);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_half(t));  // P(i) of the second entry, (rescaled) O
            if (l0) {
                if (l1) {
                    tmem_ld32(t_s, s);
                    tmem_ld32(t_s + 32, s + 32);
                    tmem_wait_ld();
                    reg_fence32(s);
                    reg_fence32(s + 32);
                }
                exp64(s, sl2, m_new, sum2);
                store_p64(t_s + L::P_OFF, s);
            } else {
                store_zero_p64(t_s + L::P_OFF);
            }
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
        if (ok && present && nt > 0 &&
            warp_wait(bars.pv_done(t), (nt - 1) & 1, abort_flag, a.wait_ns)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const size_t grow = static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(qb) * Q4_T +
                                (row & (Q4_T - 1));
            __nv_bfloat16* orow = a.o + grow * Q4_D;
#pragma unroll 1
            for (int c = 0; c < Q4_D / 32; ++c) {
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
    if (warp == Q4_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

}  // namespace

bool attn_pp64_supported(const AttnArgs& a) {
    // a walk entry keeps the key block in 14 bits, and a tile's walk holds two lists
    return a.idx == nullptr || (a.n_sel <= Q4_WALK_MAX / 2 && a.n_kb <= (1 << Q4_KB_BITS));
}

int attn_pp64_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                     cudaStream_t st) {
    using L = Q4Layout;
    CUtensorMap tq, tk, tv;
    const uint64_t bh = static_cast<uint64_t>(B) * a.H;
    if (!make_tmap(&tq, q, bh * a.Nq, Q4_D, Q4_T) || !make_tmap(&tk, k, bh * a.Nk, Q4_D, Q4_T) ||
        !make_tmap(&tv, v, bh * a.Nk, Q4_D, Q4_T))
        return VELOX_ECUDA;
    if (cudaFuncSetAttribute(attn_pp64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::SMEM) != cudaSuccess)
        return VELOX_ECUDA;
    dim3 grid((a.m + 3) / 4, a.H, B);
    attn_pp64_kernel<<<grid, Q4_THREADS, L::SMEM, st>>>(tq, tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

}  // namespace velox
