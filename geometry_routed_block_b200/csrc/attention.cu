// Block-sparse attention forward for sm_100a over routed key blocks.
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse" -- the router decides at the granularity of the kernel's
// tile, so the kernel really skips the key blocks it is not given. Here one
// CTA owns a 128-row query tile of one (batch, head) and walks only the key
// blocks listed for it. With 128-token blocks the tile is one query block.
// With 64-token blocks it is two adjacent query blocks, which walk the union
// of their two routed lists (adjacent blocks keep almost the same key blocks),
// each entry tagged with which of the two listed it: the softmax warps of the
// block that did not list a tile turn its S into P = 0, so each block attends
// exactly to its own list and no MMA row is padding.
//
// CTA = 7 warps:
//   warps 0-3  softmax / correction / epilogue; thread i owns query row i,
//              which is TMEM lane i
//   warps 4, 6 TMA producers: K_j (warp 4) and V_j (warp 6) of every listed block
//              (128-byte swizzled tiles, no multicast)
//   warp 5     tcgen05 issuer (one thread): S_j = Q K_j^T into a double-buffered
//              TMEM S; O += P_j V_j. Q and P_j are A operands read from tensor
//              memory; only K_j and V_j come from shared memory.
// Tensor memory: S[2] (BN fp32 columns each), O (D fp32 columns), P (BN/2
// columns of bf16 pairs), Q (D/2 columns of bf16 pairs; written once by the
// softmax threads). Keeping Q and P out of shared memory halves the
// shared-memory traffic of a tile, which otherwise limits the tensor core.
// Online softmax in fp32, base-2 exponent; the running max is only raised
// when a row's max grows by more than 2^8, so O is rescaled rarely; the final
// normalisation divides by the running sum taken with the same max.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn_common.cuh"

namespace velox {

namespace {

constexpr int BM = 128;          // query rows per CTA tile (MMA M)
constexpr int NTHREADS = 224;    // 7 warps
constexpr int KST = 4;           // K ring depth
constexpr int VST = 3;           // V ring depth
constexpr int WARP_TMA_K = 4;
constexpr int WARP_MMA = 5;
constexpr int WARP_TMA_V = 6;

constexpr int WALK_MAX = 8192;           // walk entries: two lists of up to 4096 blocks
constexpr int WALK_BITMAP_WORDS = 512;   // key blocks <= 16384 take the union by bitmap

template <int D, int BN>
struct Layout {
    static constexpr bool PAIR = BN == 64;  // two 64-token query blocks per 128-row tile
    static constexpr int KV_TILE = BN * D * 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + KST * KV_TILE;
    static constexpr int OFF_WALK = OFF_V + VST * KV_TILE;  // int32 [WALK_MAX] (PAIR only)
    static constexpr int OFF_BITMAP = OFF_WALK + (PAIR ? WALK_MAX * 4 : 0);  // uint32 [2][WORDS]
    static constexpr int OFF_BAR = OFF_BITMAP + (PAIR ? 2 * WALK_BITMAP_WORDS * 4 : 0);
    // q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], p_full[2], pv_done[2]
    static constexpr int NBAR = 1 + 2 * KST + 2 * VST + 6;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag, walk length
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int SMEM = BYTES + 1024;  // slack for 1024-byte alignment
    // tensor memory columns: S[2] (fp32; P_j, as bf16 pairs, overwrites the
    // first BN/2 columns of S_j once S_j has been read), O (fp32), Q (bf16 pairs)
    static constexpr int TMEM_S = 0;
    static constexpr int TMEM_O = 2 * BN;
    static constexpr int TMEM_Q = 2 * BN + D;
    static constexpr int TMEM_USED = TMEM_Q + D / 2;
    static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "tensor memory budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Bars {
    uint32_t base;
    __device__ uint32_t q_full() const { return base; }
    static constexpr int R = 1 + 2 * KST + 2 * VST;  // first of the per-block barriers
    __device__ uint32_t k_full(int s) const { return base + 8 * (1 + s); }
    __device__ uint32_t k_empty(int s) const { return base + 8 * (1 + KST + s); }
    __device__ uint32_t v_full(int s) const { return base + 8 * (1 + 2 * KST + s); }
    __device__ uint32_t v_empty(int s) const { return base + 8 * (1 + 2 * KST + VST + s); }
    __device__ uint32_t s_full(int i) const { return base + 8 * (R + i); }
    __device__ uint32_t p_full(int i) const { return base + 8 * (R + 2 + i); }
    __device__ uint32_t pv_done(int i) const { return base + 8 * (R + 4 + i); }
};

template <int D, int BN>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const AttnArgs a) {
    using L = Layout<D, BN>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (sbase - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // first query block of the tile, and how many the tile holds (1 or 2)
    const bool pair = L::PAIR && a.pair_tiles;
    const int qb = pair ? 2 * blockIdx.x : blockIdx.x;
    const int nblk = pair ? min(2, a.m - qb) : 1;
    const int bh = blockIdx.z * a.H + blockIdx.y;

    Bars bars{sbase + L::OFF_BAR};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    int* walk_len = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);
    const int* walk = reinterpret_cast<const int*>(smem + L::OFF_WALK);
    const bool use_walk = pair && a.idx != nullptr;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(bars.q_full(), 4);  // the softmax warps' elected lanes, once Q is in TMEM
        for (int s = 0; s < KST; ++s) {
            mbar_init(bars.k_full(s), 1);
            mbar_init(bars.k_empty(s), 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(bars.v_full(s), 1);
            mbar_init(bars.v_empty(s), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bars.s_full(i), 1);
            mbar_init(bars.p_full(i), 4);  // one elected arrive per softmax warp
            mbar_init(bars.pv_done(i), 1);
        }
        fence_mbar_init();
    }
    if (warp == WARP_MMA) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == WARP_TMA_K && lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
    }
    if (use_walk && warp == WARP_TMA_V) {
        const int len = build_walk<WALK_BITMAP_WORDS>(
            a, bh, qb, nblk > 1, reinterpret_cast<uint32_t*>(smem + L::OFF_BITMAP),
            reinterpret_cast<int*>(smem + L::OFF_WALK), lane);
        if (lane == 0) *walk_len = len;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n = use_walk ? *walk_len : a.n_sel;
    // which of the tile's blocks listed entry j (bit g: block qb + g)
    auto listed = [&](int j) -> int {
        if (use_walk) return walk[j] >> 16;
        return pair ? (1 << nblk) - 1 : 1;
    };

    if (warp == WARP_TMA_K || warp == WARP_TMA_V) {
        // ------------------------------------------------------------ producers
        // one thread streams K_j, another V_j, each into its own ring, so a K
        // load never queues behind a V slot that is still being read
        if (lane == 0) {
            const bool is_v = warp == WARP_TMA_V;
            const int nst = is_v ? VST : KST;
            const CUtensorMap* tm = is_v ? &tmV : &tmK;
            const uint32_t ring = sbase + (is_v ? L::OFF_V : L::OFF_K);
            auto full = [&](int st) { return is_v ? bars.v_full(st) : bars.k_full(st); };
            auto empty = [&](int st) { return is_v ? bars.v_empty(st) : bars.k_empty(st); };
            const int krow0 = bh * a.Nk;
            const int32_t* row_idx =
                a.idx ? a.idx + (static_cast<size_t>(bh) * a.m + qb) * static_cast<size_t>(a.n_sel)
                      : nullptr;
            auto fetch = [&](int j) -> int {
                if (use_walk) return walk[j] & 0xFFFF;  // validated when it was built
                int kb = row_idx ? __ldg(row_idx + j) : j;
                if (kb < 0 || kb >= a.n_kb) {
                    if (a.status && !is_v) atomicOr(a.status, VELOX_STATUS_BAD_INDEX);
                    kb = 0;
                }
                return kb;
            };
            int kb = fetch(0);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j % nst;
                const int kb_next = (j + 1 < n) ? fetch(j + 1) : 0;
                if (j >= nst &&
                    !mbar_wait(empty(st), ((j / nst) - 1) & 1, abort_flag, a.wait_ns))
                    break;
                mbar_arrive_expect_tx(full(st), L::KV_TILE);
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tma_load_2d(ring + st * L::KV_TILE + c * (BN * 128), tm, full(st), c * 64,
                                krow0 + kb * BN);
                issued = j + 1;
                kb = kb_next;
            }
            // Copies still in flight (only possible after an abort) must land
            // before the CTA exits: wait for the last one of every slot.
            for (int j = issued - 1; j >= 0 && j >= issued - nst; --j)
                drain_wait(full(j % nst), (j / nst) & 1);
        }
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // (with the skip_mma test hook it issues nothing: every wait on an MMA
        // completion then runs out, and the kernel reports the timeout)
        if (lane == 0 && !a.skip_mma) {
            constexpr uint32_t ID_S = idesc_bf16_f32(BM, BN, false, false);
            constexpr uint32_t ID_PV = idesc_bf16_f32(BM, D, false, true);
            bool ok = mbar_wait(bars.q_full(), 0, abort_flag, a.wait_ns);
            tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int s = j % KST;
                const int bi = j & 1;
                if (!mbar_wait(bars.k_full(s), (j / KST) & 1, abort_flag, a.wait_ns))
                    return false;
                // S buffer bi last held P_{j-2}, read by PV_{j-2}, which this
                // thread issued earlier: MMAs from one thread run in issue order
                tc_fence_after();
                const uint32_t d_tmem = tmem + L::TMEM_S + bi * BN;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // A = Q from tensor memory (8 columns per 16 bf16); B = K_j, whose
                    // 16-element K slice sits 32 B into its 128-B swizzled row
                    const uint32_t at = tmem + L::TMEM_Q + kk * 8;
                    const uint64_t bd = smem_desc_sw128(
                        sbase + L::OFF_K + s * L::KV_TILE + (kk >> 2) * (BN * 128) + (kk & 3) * 32, 16);
                    mma_bf16_ts(d_tmem, at, bd, ID_S, kk > 0 ? 1u : 0u);
                }
                mma_commit(bars.k_empty(s));
                mma_commit(bars.s_full(bi));
                return true;
            };
            if (ok && n > 0) ok = issue_s(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !issue_s(j + 1)) break;
                const int s = j % VST;
                const int bi = j & 1;
                if (!mbar_wait(bars.v_full(s), (j / VST) & 1, abort_flag, a.wait_ns)) break;
                if (!mbar_wait(bars.p_full(bi), (j >> 1) & 1, abort_flag, a.wait_ns)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    // A = P_j from tensor memory: 16 bf16 of a row = 8 columns
                    const uint32_t at = tmem + L::TMEM_S + bi * BN + kk * 8;
                    const uint64_t bd = smem_desc_sw128(
                        sbase + L::OFF_V + s * L::KV_TILE + kk * (16 * 128), BN * 128);
                    mma_bf16_ts(tmem + L::TMEM_O, at, bd, ID_PV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bars.v_empty(s));
                mma_commit(bars.pv_done(bi));
            }
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroup
        const int row = threadIdx.x;  // 0..127
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t t_o = tmem + lane_base + L::TMEM_O;
        const float sl2 = a.scale_log2;
        // the tile row's block: rows 0-63 are block qb, rows 64-127 block qb + 1
        const int mybit = pair ? 1 << (warp >> 1) : 1;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        {
            // this thread's query row -> tensor memory as bf16 pairs, the A operand
            // of every S = Q K^T; rows past the end of Q read as zeros
            const long long grow =
                static_cast<long long>(bh) * a.Nq + static_cast<long long>(qb) * a.T + row;
            float qv[D / 2];
            if (grow < a.q_rows) {
                const uint4* src = reinterpret_cast<const uint4*>(a.q + grow * D);
#pragma unroll
                for (int u = 0; u < D / 8; ++u) {
                    const uint4 x = __ldg(src + u);
                    qv[4 * u + 0] = __uint_as_float(x.x);
                    qv[4 * u + 1] = __uint_as_float(x.y);
                    qv[4 * u + 2] = __uint_as_float(x.z);
                    qv[4 * u + 3] = __uint_as_float(x.w);
                }
            } else {
#pragma unroll
                for (int i = 0; i < D / 2; ++i) qv[i] = 0.f;
            }
            const uint32_t t_q = tmem + lane_base + L::TMEM_Q;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tmem_st32(t_q + c * 32, qv + c * 32);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.q_full());
        }
        for (int j = 0; j < n; ++j) {
            const int bi = j & 1;
            if (!warp_wait(bars.s_full(bi), (j >> 1) & 1, abort_flag, a.wait_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (!(listed(j) & mybit)) {
                // a tile of the walk this warp's block did not list: P = 0
                float z[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) z[k] = 0.f;
                const uint32_t t_p = tmem + lane_base + L::TMEM_S + bi * BN;
#pragma unroll
                for (int c = 0; c < BN / 64; ++c) tmem_st32(t_p + c * 32, z);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars.p_full(bi));
                continue;
            }
            float s[BN];
            const uint32_t t_s = tmem + lane_base + L::TMEM_S + bi * BN;
            // first half of the row, then the second half in flight while the
            // first half is reduced
            constexpr int HALF = BN / 2;
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) tmem_ld32(t_s + c * 32, s + c * 32);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) reg_fence32(s + c * 32);
#pragma unroll
            for (int c = HALF / 32; c < BN / 32; ++c) tmem_ld32(t_s + c * 32, s + c * 32);
            float acc[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) acc[k] = s[k];
            max_range<8, HALF>(s, acc);
            tmem_wait_ld();
#pragma unroll
            for (int c = HALF / 32; c < BN / 32; ++c) reg_fence32(s + c * 32);
            max_range<HALF, BN>(s, acc);
            float mx = max3f(max3f(acc[0], acc[1], acc[2]), max3f(acc[3], acc[4], acc[5]),
                             fmaxf(acc[6], acc[7]));
            mx *= sl2;
            float m_new = m_run;
            bool resc = false;
            if (mx > m_run + RESCALE_THRESHOLD) {
                m_new = mx;
                // O is still exactly 0 before the first tile this row's block listed
                resc = m_run > -INFINITY;
            }
            // p = 2^(s * scale * log2e - m), two lanes of fp32 per FFMA2 / FADD2;
            // the pairs selected by EXP2_EMU_MASK run on the FMA pipe, the rest
            // on the ex2 unit, so neither pipe alone bounds the loop
            const float2 sc2 = make_float2(sl2, sl2);
            const float2 ng2 = make_float2(-m_new, -m_new);
            float2 sum2[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) sum2[k] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < BN; i += 2) {
                float2 x = __ffma2_rn(make_float2(s[i], s[i + 1]), sc2, ng2);
                if ((EXP2_EMU_MASK >> ((i >> 1) & 7)) & 1) {
                    x = exp2_poly2(x);
                } else {
                    x.x = ex2_approx(x.x);
                    x.y = ex2_approx(x.y);
                }
                s[i] = x.x;
                s[i + 1] = x.y;
                sum2[(i >> 1) & 3] = __fadd2_rn(sum2[(i >> 1) & 3], x);
            }
            const float2 s01 = __fadd2_rn(sum2[0], sum2[1]);
            const float2 s23 = __fadd2_rn(sum2[2], sum2[3]);
            const float2 s03 = __fadd2_rn(s01, s23);
            const float rs = s03.x + s03.y;
            {
                // P_j (bf16 pairs, lower key in the low half) into tensor memory
                float pk[BN / 2];
#pragma unroll
                for (int i = 0; i < BN / 2; ++i)
                    pk[i] = __uint_as_float(pack_bf16x2(s[2 * i], s[2 * i + 1]));
                // into the S buffer just read: PV_j reads it from there
                const uint32_t t_p = tmem + lane_base + L::TMEM_S + bi * BN;
#pragma unroll
                for (int c = 0; c < BN / 64; ++c) tmem_st32(t_p + c * 32, pk + c * 32);
                tmem_wait_st();
            }
            if (__any_sync(0xffffffffu, resc)) {
                // O must hold PV_{j-1} before it is rescaled in place
                if (!warp_wait(bars.pv_done((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float f = resc ? ex2_approx(m_run - m_new) : 1.f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    float o[32];
                    tmem_ld32(t_o + c * 32, o);
                    tmem_wait_ld();
                    reg_fence32(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] *= f;
                    tmem_st32(t_o + c * 32, o);
                }
                tmem_wait_st();
                l_run *= f;
            }
            l_run += rs;
            m_run = m_new;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars.p_full(bi));  // P_j and (rescaled) O are ready
        }
        if (ok && n > 0 && warp_wait(bars.pv_done((n - 1) & 1), ((n - 1) >> 1) & 1, abort_flag, a.wait_ns)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            const bool store = row < nblk * a.T;
            const size_t grow = static_cast<size_t>(bh) * a.Nq + static_cast<size_t>(qb) * a.T + row;
            __nv_bfloat16* orow = a.o + grow * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float o[32];
                tmem_ld32(t_o + c * 32, o);
                tmem_wait_ld();
                reg_fence32(o);
                if (store) {
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
            }
            if (store && a.lse) a.lse[grow] = (m_run + log2f(l_run)) * 0.69314718055994531f;
        }
    }

    if (threadIdx.x == 0 && *abort_flag && a.status) atomicOr(a.status, VELOX_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int D, int BN>
int launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
           cudaStream_t st) {
    using L = Layout<D, BN>;
    CUtensorMap tk, tv;
    const uint64_t bh = static_cast<uint64_t>(B) * a.H;
    if (!make_tmap(&tk, k, bh * a.Nk, D, BN) || !make_tmap(&tv, v, bh * a.Nk, D, BN))
        return VELOX_ECUDA;
    AttnArgs args = a;
    args.q = static_cast<const __nv_bfloat16*>(q);
    args.q_rows = static_cast<long long>(bh) * a.Nq;
    // 64-token blocks: two per tile, unless a walk of two lists would not fit
    args.pair_tiles = L::PAIR && (a.idx == nullptr || (a.n_sel <= WALK_MAX / 2 && a.n_kb <= 65535));
    auto kern = attn_fwd_kernel<D, BN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) !=
        cudaSuccess)
        return VELOX_ECUDA;
    dim3 grid(args.pair_tiles ? (a.m + 1) / 2 : a.m, a.H, B);
    kern<<<grid, NTHREADS, L::SMEM, st>>>(tk, tv, args);
    return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA;
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag flag;
    std::call_once(flag, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// rows x cols bf16 matrix (row-major), boxes of box_rows x 64 columns, 128-byte swizzle
bool make_tmap(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols,
               uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int attn_fwd_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B, int d,
                    cudaStream_t st) {
    if (d == 128 && a.T == 128)
        return (attn_pair_preferred(a) || (a.force_pair && attn_pair_supported(a)))
                   ? attn_pair_launch(q, k, v, a, B, st)
                   : attn_pp_launch(q, k, v, a, B, st);
    if (d == 128 && a.T == 64)
        return attn_pp64_supported(a) ? attn_pp64_launch(q, k, v, a, B, st)
                                      : launch<128, 64>(q, k, v, a, B, st);
    if (d == 64 && a.T == 128) return launch<64, 128>(q, k, v, a, B, st);
    if (d == 64 && a.T == 64) return launch<64, 64>(q, k, v, a, B, st);
    return VELOX_EUNSUPPORTED;
}

}  // namespace velox
