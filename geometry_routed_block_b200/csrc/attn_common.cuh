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

}  // namespace

// rows x cols bf16 matrix (row-major), boxes of box_rows x 64 columns, 128-byte swizzle
bool make_tmap(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// The two-query-tile kernel (d = 128, T = 128); returns VELOX_* codes.
int attn_pp_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                   cudaStream_t st);

// The CTA-pair kernel (d = 128, T = 128) and the lists it takes.
bool attn_pair_supported(const AttnArgs& a);
bool attn_pair_preferred(const AttnArgs& a);
int attn_pair_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B,
                     cudaStream_t st);

}  // namespace velox
