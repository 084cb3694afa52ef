// Block-sparse attention forward for sm_100a on CTA pairs (head dim 128,
// 128-token blocks): the tensor-core MMAs of two SMs are issued as one.
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse" -- each query block attends only to the key blocks routed to
// it, at the granularity of the attention tile.
//
// A cluster of two CTAs owns four query blocks of one (batch, head) as two
// stages: stage s pairs block 4c + 2s (CTA rank 0) with block 4c + 2s + 1 (CTA
// rank 1). Every MMA of a stage is a pair MMA (tcgen05 cta_group::2, M = 256):
// each CTA supplies the 128 query rows of its own block and half of the key or
// value tile, and receives its own 128 rows of S and O in its tensor memory.
// The two blocks of a stage walk one list: the union of their routed lists
// (adjacent query blocks keep almost the same key blocks), each entry tagged
// with which of the two listed it; a block's softmax turns the S of a tile it
// did not list into P = 0, so each block attends exactly to its own list.
// Against one CTA per two blocks, this halves per SM the MMA instructions, the
// shared-memory reads of the B operand and the K/V tiles staged by TMA.
//
// The stages ping-pong on the tensor core as in the single-SM two-block
// kernel: S_0(i), O_1 += P_1(i-1) V_1(i-1), S_1(i), O_0 += P_0(i) V_0(i), ...;
// P V is issued in two halves of the keys (the half whose P is stored first
// goes first).
//
// CTA = 12 warps in both CTAs:
//   warps 0-3   softmax / epilogue of this CTA's block of stage 0 (row = TMEM lane)
//   warps 4-7   the same for stage 1
//   warp 8      TMA producer: Q, then this CTA's half of every K tile (64 keys)
//   warp 9      tensor-memory allocation for the pair; in CTA 0 the MMA issuer
//   warp 10     TMA producer: this CTA's half of every V tile (64 of the 128 dims)
//   warps 10-11 before the loop: build the walk of stage 1 / stage 0
// Barriers: the ones the issuer waits on (Q, K, V full; P half, P full) live
// in CTA 0 and count both CTAs' copies and arrivals; the MMA completions (S
// full, P V done) are committed to the same barrier in both CTAs, where the
// softmax and the producers of each CTA wait on them. Every wait is bounded.
#include "attn_common.cuh"

namespace velox {

namespace {

constexpr int PR_THREADS = 384;
constexpr int PR_D = 128;
constexpr int PR_BN = 128;
constexpr int PR_LIST = 4096;  // walk entries per stage: two lists of up to 2048 blocks
constexpr int PR_BITMAP_WORDS = 256;  // key blocks <= 8192 take the union by bitmap
constexpr int PR_WARP_TMA_K = 8;
constexpr int PR_WARP_MMA = 9;
constexpr int PR_WARP_TMA_V = 10;

struct PRLayout {
    static constexpr int Q_TILE = 128 * 128 * 2;   // 128 rows x 128 dims
    static constexpr int KV_HALF = 64 * 128 * 2;   // 64 keys x 128 dims, or 128 keys x 64 dims
    static constexpr int OFF_Q = 0;                // Q[2 stages]
    static constexpr int OFF_K = 2 * Q_TILE;       // K half-tiles, one slot per stage
    static constexpr int OFF_V = OFF_K + 2 * KV_HALF;
    static constexpr int OFF_LIST = OFF_V + 2 * KV_HALF;  // int32 walk[2][PR_LIST]
    static constexpr int OFF_BITMAP = OFF_LIST + 2 * PR_LIST * 4;  // uint32 [2 stages][2][256]
    static constexpr int OFF_BAR = OFF_BITMAP + 2 * 2 * PR_BITMAP_WORDS * 4;
    static constexpr int NBAR = 14;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, walk lengths
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
    static_assert(SMEM <= 232448, "shared memory budget");
    static constexpr int TMEM_COLS = 512;  // S_0, S_1, O_0, O_1
    static constexpr int TMEM_O = 256;
    static constexpr int P_OFF = 64;       // P inside S: columns 64..127
};

struct PRBars {
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    __device__ uint32_t k_full(int t) const { return base + 8 * (1 + t); }
    __device__ uint32_t v_full(int t) const { return base + 8 * (3 + t); }
    __device__ uint32_t s_full(int t) const { return base + 8 * (5 + t); }
    __device__ uint32_t pv_done(int t) const { return base + 8 * (7 + t); }
    __device__ uint32_t p_half(int t) const { return base + 8 * (9 + t); }
    __device__ uint32_t p_full(int t) const { return base + 8 * (11 + t); }
    __device__ uint32_t mma_drain() const { return base + 8 * 13; }
};

// Pairs 0 and 4 of every 8 go to the FMA pipe (Cody-Waite cubic), the rest to
// the ex2 unit. This kernel's MMA chain has room to spare, so its softmax sets
// the pace, and taking a quarter of the exponentials off the ex2 unit shortens
// it: 12 alternating rounds, chunk 48 / P = 8, routed 995 -> 1,061 / 957 -> 999
// and dense 1,101 -> 1,109 / 1,075 -> 1,130 TFLOP/s.
constexpr unsigned PR_EMU_MASK = 0x11;

// exponentials of 64 scores (one half row) in place, sums into sum2
__device__ __forceinline__ void pr_exp_half(float* s, float sl2, float m, float2* sum2) {
    const float2 sc2 = make_float2(sl2, sl2);
    const float2 ng2 = make_float2(-m, -m);
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
        float2 x = __ffma2_rn(make_float2(s[i], s[i + 1]), sc2, ng2);
        if ((PR_EMU_MASK >> ((i >> 1) & 7)) & 1) {
            x = exp2_poly2(x);
        } else {
            x.x = ex2_approx(x.x);
            x.y = ex2_approx(x.y);
        }
        s[i] = x.x;
        s[i + 1] = x.y;
        sum2[(i >> 1) & 3] = __fadd2_rn(sum2[(i >> 1) & 3], x);
    }
}

// 64 probabilities -> 32 bf16 pairs in tensor memory at column `t_p`
__device__ __forceinline__ void pr_store_p_half(uint32_t t_p, const float* s) {
    float pk[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = __uint_as_float(pack_bf16x2(s[2 * i], s[2 * i + 1]));
    tmem_st32(t_p, pk);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PR_THREADS, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnArgs a) {
    using L = PRLayout;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cl = blockIdx.x >> 1;  // cluster index within the (batch, head)
    const int bh = blockIdx.z * a.H + blockIdx.y;
    const int qb_first = 4 * cl;
    const int nstage = qb_first + 2 < a.m ? 2 : 1;
    // block of stage s held by CTA r: qb_first + 2 s + r (may be past the last block)
    auto member_qb = [&](int s, int r) { return qb_first + 2 * s + r; };

    PRBars bars{sbase + L::OFF_BAR};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    int* walk_len = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);  // [2]
    int* walk = reinterpret_cast<int*>(smem + L::OFF_LIST);          // [2][PR_LIST]

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bars.q_full(), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bars.k_full(t), 1);
            mbar_init(bars.v_full(t), 1);
            mbar_init(bars.s_full(t), 1);
            mbar_init(bars.pv_done(t), 1);
            mbar_init(bars.p_half(t), 8);  // one elected arrive per softmax warp, both CTAs
            mbar_init(bars.p_full(t), 8);
        }
        mbar_init(bars.mma_drain(), 1);
        fence_mbar_init();
    }
    if (warp == PR_WARP_MMA) {
        tmem_alloc_pair(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == PR_WARP_TMA_K && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    tc_fence_before();
    cluster_sync();  // barriers and the tensor-memory address are in place in both CTAs
    tc_fence_after();
    if (warp == PR_WARP_TMA_K && lane == 0) {
        // Q does not depend on the walks: its copies fly while they are built
        if (leader) mbar_arrive_expect_tx(bars.q_full(), 2 * nstage * L::Q_TILE);
        const uint32_t qbar = map_to_rank(bars.q_full(), 0);
        for (int s = 0; s < nstage; ++s) {
            const int qrow = bh * a.Nq + member_qb(s, rank) * PR_BN;
#pragma unroll
            for (int c = 0; c < 2; ++c)
                tma_load_2d_pair(sbase + L::OFF_Q + s * L::Q_TILE + c * (128 * 128), &tmQ, qbar,
                                 c * 64, qrow);
        }
    }
    if (warp == 10 || warp == 11) {
        const int s = warp == 11 ? 0 : 1;
        int len = 0;
        if (s < nstage) {
            const int qb0 = member_qb(s, 0);
            const bool has1 = qb0 + 1 < a.m;
            if (a.idx) {
                uint32_t* bm = reinterpret_cast<uint32_t*>(smem + L::OFF_BITMAP) +
                               s * 2 * PR_BITMAP_WORDS;
                len = build_walk<PR_BITMAP_WORDS>(a, bh, qb0, has1, bm, walk + s * PR_LIST, lane);
            } else {
                len = a.n_kb;  // dense: every block, listed by both
            }
        }
        if (lane == 0) walk_len[s] = len;
    }
    __syncthreads();  // the walks (each CTA builds its own copy)
    const uint32_t tmem = *tmem_slot;
    const int nw0 = walk_len[0], nw1 = walk_len[1];
    const int nmax = max(nw0, nw1);
    // entry i of stage t's walk: key block and which members listed it
    auto entry = [&](int t, int i) -> int {
        if (!a.idx) {
            const int pres = member_qb(t, 1) < a.m ? 3 : 1;
            return i | (pres << 16);
        }
        return walk[t * PR_LIST + i];
    };

    if (warp == PR_WARP_TMA_K || warp == PR_WARP_TMA_V) {
        // ------------------------------------------------------------ producers (both CTAs)
        if (lane == 0) {
            const bool is_v = warp == PR_WARP_TMA_V;
            const CUtensorMap* tm = is_v ? &tmV : &tmK;
            const uint32_t ring = sbase + (is_v ? L::OFF_V : L::OFF_K);
            auto full = [&](int t) { return is_v ? bars.v_full(t) : bars.k_full(t); };
            auto done = [&](int t) { return is_v ? bars.pv_done(t) : bars.s_full(t); };
            const int krow0 = bh * a.Nk;
            int issued[2] = {0, 0};
            bool ok = true;
            for (int i = 0; ok && i < nmax; ++i) {
                for (int t = 0; t < 2; ++t) {
                    if (i >= (t == 0 ? nw0 : nw1)) continue;
                    // slot t last held tile i-1 of stage t: free once its MMA is complete
                    if (i > 0 && !mbar_wait(done(t), (i - 1) & 1, abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    const int kb = entry(t, i) & 0xFFFF;
                    if (leader) mbar_arrive_expect_tx(full(t), 2 * L::KV_HALF);
                    const uint32_t fbar = map_to_rank(full(t), 0);
                    const uint32_t dst = ring + t * L::KV_HALF;
                    if (is_v) {
                        // this CTA's 64 of the 128 dims, all 128 keys
                        tma_load_2d_pair(dst, tm, fbar, 64 * static_cast<int>(rank),
                                         krow0 + kb * PR_BN);
                    } else {
                        // this CTA's 64 of the 128 keys, all 128 dims
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            tma_load_2d_pair(dst + c * (64 * 128), tm, fbar, c * 64,
                                             krow0 + kb * PR_BN + 64 * static_cast<int>(rank));
                    }
                    issued[t] = i + 1;
                }
            }
            // On an abort, copies may still be in flight: CTA 0 waits (bounded) for the
            // last phase of each of its full barriers, which count both CTAs' copies;
            // the final cluster barrier keeps CTA 1 alive until then.
            if (leader) {
                if (!is_v) drain_wait(bars.q_full(), 0);
                for (int t = 0; t < 2; ++t)
                    if (issued[t] > 0) drain_wait(full(t), (issued[t] - 1) & 1);
            }
        }
    } else if (warp == PR_WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer (CTA 0)
        // (with the skip_mma test hook it issues nothing: every wait on an MMA
        // completion then runs out, and the kernel reports the timeout)
        if (leader && lane == 0 && !a.skip_mma) {
            constexpr uint32_t ID_S = idesc_bf16_f32(256, PR_BN, false, false);
            constexpr uint32_t ID_PV = idesc_bf16_f32(256, PR_D, false, true);
            bool ok = mbar_wait(bars.q_full(), 0, abort_flag, a.wait_ns);
            tc_fence_after();
            auto issue_s = [&](int t, int i) -> bool {
                if (!mbar_wait(bars.k_full(t), i & 1, abort_flag, a.wait_ns)) return false;
                tc_fence_after();
                const uint32_t d = tmem + t * 128;
#pragma unroll
                for (int kk = 0; kk < PR_D / 16; ++kk) {
                    // A: this CTA's Q rows (K-major, 128-B swizzled, 64 dims per chunk);
                    // B: its 64 keys of the tile
                    const uint32_t off_a = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                    const uint32_t off_b = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sbase + L::OFF_Q + t * L::Q_TILE + off_a, 16);
                    const uint64_t bd = smem_desc_sw128(sbase + L::OFF_K + t * L::KV_HALF + off_b, 16);
                    mma_pair_bf16_ss(d, ad, bd, ID_S, kk > 0 ? 1u : 0u);
                }
                mma_commit_pair_both(bars.s_full(t));
                return true;
            };
            auto issue_pv = [&](int t, int i) -> bool {
                if (!mbar_wait(bars.v_full(t), i & 1, abort_flag, a.wait_ns)) return false;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t bar = h == 0 ? bars.p_half(t) : bars.p_full(t);
                    if (!mbar_wait(bar, i & 1, abort_flag, a.wait_ns)) return false;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < PR_BN / 32; ++j) {
                        const int kk = (h == 0 ? PR_BN / 32 : 0) + j;
                        // A: P in tensor memory (16 keys = 8 columns of bf16 pairs);
                        // B: this CTA's 64 dims of V, 16 keys (MN-major)
                        const uint32_t at = tmem + t * 128 + L::P_OFF + kk * 8;
                        const uint64_t bd = smem_desc_sw128(
                            sbase + L::OFF_V + t * L::KV_HALF + kk * (16 * 128), L::KV_HALF);
                        mma_pair_bf16_ts(tmem + L::TMEM_O + t * 128, at, bd, ID_PV,
                                         (i > 0 || h > 0 || j > 0) ? 1u : 0u);
                    }
                }
                mma_commit_pair_both(bars.pv_done(t));
                return true;
            };
            for (int i = 0; ok && i < nmax; ++i) {
                if (i < nw0 && !issue_s(0, i)) break;
                if (i > 0 && i - 1 < nw1 && !issue_pv(1, i - 1)) break;
                if (i < nw1 && !issue_s(1, i)) break;
                if (i < nw0 && !issue_pv(0, i)) break;
                if (i == nmax - 1 && nw1 > 0 && nw1 >= nw0 && !issue_pv(1, nw1 - 1)) break;
            }
            // every MMA issued above has completed before this thread leaves (on
            // an abort, too), so none is in flight when tensor memory is freed
            mma_commit_pair_local(bars.mma_drain());
            drain_wait(bars.mma_drain(), 0);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = warp >> 2;  // stage
        const int n = t == 0 ? nw0 : nw1;
        const int qb = member_qb(t, rank);
        const int mybit = 1 << rank;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + t * 128;
        const uint32_t t_o = tmem + lane_base + L::TMEM_O + t * 128;
        const uint32_t ph_bar = map_to_rank(bars.p_half(t), 0);
        const uint32_t pf_bar = map_to_rank(bars.p_full(t), 0);
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
            if (!((entry(t, i) >> 16) & mybit)) {
                // a tile of the walk this block did not list: P = 0
                float z[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) z[k] = 0.f;
                tmem_st32(t_s + L::P_OFF + 32, z);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(ph_bar);
                tmem_st32(t_s + L::P_OFF, z);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(pf_bar);
                continue;
            }
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
                // O is still exactly 0 before the first tile this block listed
                resc = m_run > -INFINITY;
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
                for (int c = 0; c < PR_D / 32; ++c) {
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
            pr_exp_half(s, sl2, m_new, sum2);
            pr_store_p_half(t_s + L::P_OFF + 32, s);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(ph_bar);
            tmem_ld32(t_s, s);
            tmem_ld32(t_s + 32, s + 32);
            tmem_wait_ld();
            reg_fence32(s);
            reg_fence32(s + 32);
            pr_exp_half(s, sl2, m_new, sum2);
            pr_store_p_half(t_s + L::P_OFF, s);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(pf_bar);
            const float2 s01 = __fadd2_rn(sum2[0], sum2[1]);
            const float2 s23 = __fadd2_rn(sum2[2], sum2[3]);
            const float2 s03 = __fadd2_rn(s01, s23);
            l_run = l_run * f + (s03.x + s03.y);
            m_run = m_new;
        }
        if (ok && n > 0 && qb < a.m &&
            warp_wait(bars.pv_done(t), (n - 1) & 1, abort_flag, a.wait_ns)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const size_t grow = static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(qb) * PR_BN + row;
            __nv_bfloat16* orow = a.o + grow * PR_D;
#pragma unroll 1
            for (int c = 0; c < PR_D / 32; ++c) {
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
    // neither CTA leaves (or frees tensor memory) while the pair's MMAs, copies
    // or arrivals may still touch the other's memory
    cluster_sync();
    if (warp == PR_WARP_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, L::TMEM_COLS);
    }
}

}  // namespace

bool attn_pair_supported(const AttnArgs& a) {
    // the walk of a stage holds two lists; entries keep the key block in 16 bits
    return (a.idx == nullptr || a.n_sel <= PR_LIST / 2) && a.n_kb <= 65535;
}

bool attn_pair_preferred(const AttnArgs& a) {
    // Measured at the chunk-48 shapes on one B200, same process, alternating:
    // the dense walk 1,114 TFLOP/s here against 1,071 for the single-SM
    // two-block kernel; routed lists 1,034 against 1,108 (there the two stages
    // walk different tile streams, where the single-SM kernel's two blocks
    // reuse each other's tiles from L2). Routed lists go to the two-block kernel.
    return a.idx == nullptr && attn_pair_supported(a);
}

int attn_pair_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                     cudaStream_t st) {
    using L = PRLayout;
    CUtensorMap tq, tk, tv;
    const uint64_t bh = static_cast<uint64_t>(B) * a.H;
    if (!make_tmap(&tq, q, bh * a.Nq, PR_D, 128) || !make_tmap(&tk, k, bh * a.Nk, PR_D, 64) ||
        !make_tmap(&tv, v, bh * a.Nk, PR_D, 128))
        return VELOX_ECUDA;
    if (cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::SMEM) != cudaSuccess)
        return VELOX_ECUDA;
    dim3 grid(2 * ((a.m + 3) / 4), a.H, B);
    attn_pair_kernel<<<grid, PR_THREADS, L::SMEM, st>>>(tq, tk, tv, a);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

}  // namespace velox
