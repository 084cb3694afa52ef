// Device helpers shared by the attention kernels (sm_100a), and the host-side
// tensor-map encoder they use.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "ptx.cuh"
#include "velox_internal.cuh"

namespace velox {

constexpr float RESCALE_THRESHOLD = 8.0f;          // log2 units

namespace {

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// acc[k] = max(acc[k], s[LO + k + 8 i]) over [LO, HI): 8 independent chains,
// three-input max where possible
template <int LO, int HI>
__device__ __forceinline__ void max_range(const float* s, float* acc) {
    int i = LO;
#pragma unroll
    for (; i + 16 <= HI; i += 16) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = max3f(acc[k], s[i + k], s[i + 8 + k]);
    }
#pragma unroll
    for (; i + 8 <= HI; i += 8) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = fmaxf(acc[k], s[i + k]);
    }
}

// 2^x for two lanes on the FMA pipe (Cody-Waite range reduction + minimax
// cubic; coefficients from geometry_routed_block_b200/exp2_poly.py, relative
// error < 1e-4). n = round(x) comes from the low mantissa bits of
// x + 1.5 * 2^23; f = x - n lies in [-1/2, 1/2]; the result is p(f) with n added
// to its exponent field. x is clamped to [-120, inf): below that 2^x is
// negligible next to the row sum, and the exponent cannot wrap.
constexpr float EXP2_C0 = 0.9999280571937561f;
constexpr float EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.2426111251115799f;
constexpr float EXP2_C3 = 0.0551716685295105f;
constexpr unsigned EXP2_EMU_MASK = 0x52;  // pairs 1, 4 and 6 of every 8

__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -120.f);
    x.y = fmaxf(x.y, -120.f);
    const float2 magic = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
    const float2 t = __fadd2_rn(x, magic);
    const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
    float2 p = __ffma2_rn(make_float2(EXP2_C3, EXP2_C3), f, make_float2(EXP2_C2, EXP2_C2));
    p = __ffma2_rn(p, f, make_float2(EXP2_C1, EXP2_C1));
    p = __ffma2_rn(p, f, make_float2(EXP2_C0, EXP2_C0));
    float2 r;
    r.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
    r.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
    return r;
}

// bounded wait, made uniform across the warp (a warp leaves together)
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          uint64_t limit_ns) {
    bool ok = mbar_wait(bar, parity, abort, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
    // waits for copies already in flight; ignores the abort flag, short limit
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > 100000000ull) return false;
    }
    return true;
}

// The walk of two adjacent query blocks, built by one warp: the union of the
// routed lists of query blocks qb0 and (if present) qb0 + 1, ascending, entry
// = kb | (mask << SHIFT) with bit g of mask set when list g holds kb (OutT and
// SHIFT: int and 16, or a 16-bit entry with SHIFT 14 when every key block
// index is below 2^14; bm: scratch
// bitmaps of 2 x WORDS words, so up to 32 * WORDS key blocks). A list that
// repeats a block, or more key blocks than the bitmap holds, gives the
// concatenation of the lists instead (masks one-hot), which keeps every listed
// block, repeats included. Indices out of range are replaced by block 0 and
// flagged in the status word. The same rows always give the same walk.
// Returns its length (at most twice the list length).
template <int WORDS, typename OutT = int, int SHIFT = 16>
__device__ int build_walk(const AttnArgs& a, int bh, int qb0, bool has1, uint32_t* bm, OutT* out,
                          int lane) {
    const unsigned FULL = 0xffffffffu;
    const int n = a.n_sel;
    const int32_t* r0 = a.idx + (static_cast<size_t>(bh) * a.m + qb0) * static_cast<size_t>(n);
    const int nlist = has1 ? 2 : 1;
    const int nw = (a.n_kb + 31) >> 5;
    bool bitmap = nw <= WORDS;
    bool bad = false;
    if (bitmap) {
        for (int w = lane; w < 2 * WORDS; w += 32) bm[w] = 0;
        __syncwarp();
        bool dup = false;
        for (int g = 0; g < nlist; ++g) {
            const int32_t* row = r0 + static_cast<size_t>(g) * n;
            for (int j = lane; j < n; j += 32) {
                int kb = __ldg(row + j);
                if (kb < 0 || kb >= a.n_kb) {
                    bad = true;
                    kb = 0;
                }
                const uint32_t bit = 1u << (kb & 31);
                const uint32_t old = atomicOr(&bm[g * WORDS + (kb >> 5)], bit);
                dup |= (old & bit) != 0;
            }
        }
        __syncwarp();
        bitmap = !__any_sync(FULL, dup);
    }
    if (__any_sync(FULL, bad) && lane == 0 && a.status) atomicOr(a.status, VELOX_STATUS_BAD_INDEX);
    if (bitmap) {
        constexpr int PER = WORDS / 32;  // words per lane
        const int w0 = lane * PER;
        int cnt = 0;
#pragma unroll
        for (int w = w0; w < w0 + PER; ++w)
            if (w < nw) cnt += __popc(bm[w] | bm[WORDS + w]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += v;
        }
        int pos = incl - cnt;
        const int total = __shfl_sync(FULL, incl, 31);
        for (int w = w0; w < w0 + PER && w < nw; ++w) {
            const uint32_t u0 = bm[w], u1 = bm[WORDS + w];
            uint32_t u = u0 | u1;
            while (u) {
                const int b = __ffs(u) - 1;
                u &= u - 1;
                const int mask = static_cast<int>(((u0 >> b) & 1u) | (((u1 >> b) & 1u) << 1));
                out[pos++] = static_cast<OutT>((w * 32 + b) | (mask << SHIFT));
            }
        }
        return total;
    }
    for (int g = 0; g < nlist; ++g) {
        const int32_t* row = r0 + static_cast<size_t>(g) * n;
        for (int j = lane; j < n; j += 32) {
            int kb = __ldg(row + j);
            if (kb < 0 || kb >= a.n_kb) kb = 0;
            out[g * n + j] = static_cast<OutT>(kb | ((1 << g) << SHIFT));
        }
    }
    return nlist * n;
}

}  // namespace

// rows x cols bf16 matrix (row-major), boxes of box_rows x 64 columns, 128-byte swizzle
bool make_tmap(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// The two-query-tile kernel (d = 128, T = 128); returns VELOX_* codes.
int attn_pp_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                   cudaStream_t st);

// The two-query-tile kernel for 64-token blocks (d = 128): each tile is two
// query blocks, each key tile two entries of their walk; the lists it takes.
bool attn_pp64_supported(const AttnArgs& a);
int attn_pp64_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                     cudaStream_t st);

// The CTA-pair kernel (d = 128, T = 128) and the lists it takes.
bool attn_pair_supported(const AttnArgs& a);
bool attn_pair_preferred(const AttnArgs& a);
int attn_pair_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                     cudaStream_t st);

}  // namespace velox
