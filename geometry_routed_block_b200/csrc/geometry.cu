// Geometry kernels for sm_100a: frustum slices, per-block slice overlap counts
// and the recency-priority multiwarp of past depth into the current view.
//
// Method: "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle", section
// "Tiefenanalyse", steps 1-3 (past chunk = camera-frustum slice with a depth
// interval; current depth from a recency-priority multiwarp; slice overlap per
// query-block region). All geometry runs in float64 with an explicit operation
// order through the round-to-nearest intrinsics (__dadd_rn, __dsub_rn,
// __dmul_rn, __ddiv_rn), which the compiler never fuses into FMAs, so counts
// and warped depths are exact, reproducible results of the stated formulas.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "velox_internal.cuh"

namespace velox {

namespace {

struct Cam64 {
    double R[9], t[3], fx, fy, cx, cy, znear, zfar;
};

__device__ __forceinline__ Cam64 widen_cam(const velox_slice_t& s) {
    Cam64 c;
#pragma unroll
    for (int i = 0; i < 9; ++i) c.R[i] = static_cast<double>(s.R[i]);
#pragma unroll
    for (int i = 0; i < 3; ++i) c.t[i] = static_cast<double>(s.t[i]);
    c.fx = s.fx;
    c.fy = s.fy;
    c.cx = s.cx;
    c.cy = s.cy;
    c.znear = s.znear;
    c.zfar = s.zfar;
    return c;
}

__device__ __forceinline__ bool depth_ok(float z) { return isfinite(z) && z > 0.0f; }

// pixel (r, c) at z-depth z -> world: p_c = ((u-cx)/fx*z, (v-cy)/fy*z, z),
// u = c + 0.5, v = r + 0.5; p_w = R^T (p_c - t), each row left to right
__device__ __forceinline__ void backproject(int r, int c, double z, const Cam64& k, double& xw,
                                            double& yw, double& zw) {
    const double u = __dadd_rn(static_cast<double>(c), 0.5);
    const double v = __dadd_rn(static_cast<double>(r), 0.5);
    const double xc = __dmul_rn(__ddiv_rn(__dsub_rn(u, k.cx), k.fx), z);
    const double yc = __dmul_rn(__ddiv_rn(__dsub_rn(v, k.cy), k.fy), z);
    const double dx = __dsub_rn(xc, k.t[0]);
    const double dy = __dsub_rn(yc, k.t[1]);
    const double dz = __dsub_rn(z, k.t[2]);
    xw = __dadd_rn(__dadd_rn(__dmul_rn(k.R[0], dx), __dmul_rn(k.R[3], dy)), __dmul_rn(k.R[6], dz));
    yw = __dadd_rn(__dadd_rn(__dmul_rn(k.R[1], dx), __dmul_rn(k.R[4], dy)), __dmul_rn(k.R[7], dz));
    zw = __dadd_rn(__dadd_rn(__dmul_rn(k.R[2], dx), __dmul_rn(k.R[5], dy)), __dmul_rn(k.R[8], dz));
}

// world -> camera: q = R p_w + t, each row left to right
__device__ __forceinline__ void to_camera(double xw, double yw, double zw, const Cam64& k, double& qx,
                                          double& qy, double& qz) {
    qx = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(k.R[0], xw), __dmul_rn(k.R[1], yw)),
                             __dmul_rn(k.R[2], zw)),
                   k.t[0]);
    qy = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(k.R[3], xw), __dmul_rn(k.R[4], yw)),
                             __dmul_rn(k.R[5], zw)),
                   k.t[1]);
    qz = __dadd_rn(__dadd_rn(__dadd_rn(__dmul_rn(k.R[6], xw), __dmul_rn(k.R[7], yw)),
                             __dmul_rn(k.R[8], zw)),
                   k.t[2]);
}

// continuous pixel coordinates u = fx*(qx/qz)+cx, v = fy*(qy/qz)+cy (qz > 0)
__device__ __forceinline__ double image_u(double qx, double qz, const Cam64& k) {
    return __dadd_rn(__dmul_rn(k.fx, __ddiv_rn(qx, qz)), k.cx);
}
__device__ __forceinline__ double image_v(double qy, double qz, const Cam64& k) {
    return __dadd_rn(__dmul_rn(k.fy, __ddiv_rn(qy, qz)), k.cy);
}
__device__ __forceinline__ void image_coords(double qx, double qy, double qz, const Cam64& k,
                                             double& uu, double& vv) {
    uu = image_u(qx, qz, k);
    vv = image_v(qy, qz, k);
}

// ---------------------------------------------------------------- slices

__global__ void __launch_bounds__(256) slices_kernel(const float* __restrict__ depth,
                                                     const float* __restrict__ poses,
                                                     const float* __restrict__ intr, int HW,
                                                     velox_slice_t* __restrict__ out) {
    __shared__ float s_lo[8], s_hi[8];
    const int j = blockIdx.x;
    const float* d = depth + static_cast<size_t>(j) * HW;
    float lo = __int_as_float(0x7f800000);   // +inf
    float hi = __int_as_float(0xff800000);   // -inf
    for (int i = threadIdx.x; i < HW; i += 256) {
        const float z = d[i];
        if (depth_ok(z)) {
            lo = fminf(lo, z);
            hi = fmaxf(hi, z);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((threadIdx.x & 31) == 0) {
        s_lo[threadIdx.x >> 5] = lo;
        s_hi[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < 8; ++w) {
            lo = fminf(lo, s_lo[w]);
            hi = fmaxf(hi, s_hi[w]);
        }
        velox_slice_t s;
        for (int i = 0; i < 9; ++i) s.R[i] = poses[j * 12 + i];
        for (int i = 0; i < 3; ++i) s.t[i] = poses[j * 12 + 9 + i];
        s.fx = intr[j * 4 + 0];
        s.fy = intr[j * 4 + 1];
        s.cx = intr[j * 4 + 2];
        s.cy = intr[j * 4 + 3];
        s.znear = lo;
        s.zfar = hi;
        out[j] = s;
    }
}

// ---------------------------------------------------------------- overlap counts

constexpr int CAMS_PER_CTA = 8;

// grid (m, ceil(P / CAMS_PER_CTA), B), one thread per token of the query block.
// The CTA's slices are widened to float64 once, into shared memory; a point
// whose horizontal coordinate is already off the grid skips the vertical one
// (the same operations decide the count, only fewer of them run).
__global__ void overlap_kernel(const float* __restrict__ depth, const velox_slice_t* __restrict__ cur,
                               const velox_slice_t* __restrict__ slices, int P, int Hp, int Wp,
                               int T, int m, int32_t* __restrict__ counts) {
    __shared__ Cam64 cams_s[CAMS_PER_CTA];
    const int qb = blockIdx.x;
    const int b = blockIdx.z;
    const int j0 = blockIdx.y * CAMS_PER_CTA;
    if (threadIdx.x < CAMS_PER_CTA && j0 + static_cast<int>(threadIdx.x) < P)
        cams_s[threadIdx.x] = widen_cam(slices[static_cast<size_t>(b) * P + j0 + threadIdx.x]);
    __syncthreads();
    const int HW = Hp * Wp;
    const int tau = qb * T + threadIdx.x;
    const int pix = tau % HW;
    const int r = pix / Wp, c = pix % Wp;
    const float zf = depth[static_cast<size_t>(b) * HW + pix];
    const bool valid = depth_ok(zf);
    double xw = 0.0, yw = 0.0, zw = 0.0;
    if (valid) {
        const Cam64 k = widen_cam(cur[b]);
        backproject(r, c, static_cast<double>(zf), k, xw, yw, zw);
    }
    const double Wd = static_cast<double>(Wp), Hd = static_cast<double>(Hp);
    for (int jj = 0; jj < CAMS_PER_CTA; ++jj) {
        const int j = j0 + jj;
        if (j >= P) break;  // uniform across the CTA
        bool inside = false;
        if (valid) {
            const Cam64& k = cams_s[jj];
            double qx, qy, qz;
            to_camera(xw, yw, zw, k, qx, qy, qz);
            if (qz > 0.0 && qz >= k.znear && qz <= k.zfar) {
                const double uu = image_u(qx, qz, k);
                if (uu >= 0.0 && uu < Wd) {
                    const double vv = image_v(qy, qz, k);
                    inside = vv >= 0.0 && vv < Hd;
                }
            }
        }
        const int cnt = __syncthreads_count(inside);
        if (threadIdx.x == 0) counts[(static_cast<size_t>(b) * m + qb) * P + j] = cnt;
    }
}

// ---------------------------------------------------------------- multiwarp

// Candidate of past pixel `gid` (chunk j = gid / HW): target pixel and its
// depth in the current camera, or false when it lands nowhere.
__device__ __forceinline__ bool mw_candidate(const float* __restrict__ past_depth,
                                             const velox_slice_t* __restrict__ past,
                                             const Cam64& cur, int gid, int Hp, int Wp, int& tp,
                                             double& qz) {
    const int HW = Hp * Wp;
    const int j = gid / HW, pix = gid % HW;
    const float zf = past_depth[gid];
    if (!depth_ok(zf)) return false;
    const Cam64 k = widen_cam(past[j]);
    double xw, yw, zw, qx, qy;
    backproject(pix / Wp, pix % Wp, static_cast<double>(zf), k, xw, yw, zw);
    to_camera(xw, yw, zw, cur, qx, qy, qz);
    if (!(qz > 0.0)) return false;
    double uu, vv;
    image_coords(qx, qy, qz, cur, uu, vv);
    if (!(uu >= 0.0 && uu < static_cast<double>(Wp) && vv >= 0.0 && vv < static_cast<double>(Hp)))
        return false;
    tp = static_cast<int>(floor(vv)) * Wp + static_cast<int>(floor(uu));
    return true;
}

__global__ void mw_init_kernel(unsigned long long* zmin, int* jwin, unsigned long long* zbest, int HW) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < HW) {
        zmin[i] = ~0ull;
        jwin[i] = -1;
        zbest[i] = ~0ull;
    }
}

// pass 1: nearest candidate depth per target pixel (positive doubles order like
// their bit patterns as unsigned integers)
__global__ void mw_zmin_kernel(const float* __restrict__ pd, const velox_slice_t* __restrict__ past,
                               const velox_slice_t* __restrict__ curp, int n, int Hp, int Wp,
                               unsigned long long* zmin) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n) return;
    const Cam64 cur = widen_cam(*curp);
    int tp;
    double qz;
    if (mw_candidate(pd, past, cur, gid, Hp, Wp, tp, qz))
        atomicMin(zmin + tp, static_cast<unsigned long long>(__double_as_longlong(qz)));
}

// pass 2: most recent chunk among candidates within (1 + rel_tol) of the nearest
__global__ void mw_winner_kernel(const float* __restrict__ pd, const velox_slice_t* __restrict__ past,
                                 const velox_slice_t* __restrict__ curp, int n, int Hp, int Wp,
                                 double factor, const unsigned long long* __restrict__ zmin, int* jwin) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n) return;
    const Cam64 cur = widen_cam(*curp);
    int tp;
    double qz;
    if (mw_candidate(pd, past, cur, gid, Hp, Wp, tp, qz)) {
        const double thr = __dmul_rn(__longlong_as_double(static_cast<long long>(zmin[tp])), factor);
        if (qz <= thr) atomicMax(jwin + tp, gid / (Hp * Wp));
    }
}

// pass 3: smallest depth of the winning chunk
__global__ void mw_depth_kernel(const float* __restrict__ pd, const velox_slice_t* __restrict__ past,
                                const velox_slice_t* __restrict__ curp, int n, int Hp, int Wp,
                                const int* __restrict__ jwin, unsigned long long* zbest) {
    const int gid = blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= n) return;
    const Cam64 cur = widen_cam(*curp);
    int tp;
    double qz;
    if (mw_candidate(pd, past, cur, gid, Hp, Wp, tp, qz) && jwin[tp] == gid / (Hp * Wp))
        atomicMin(zbest + tp, static_cast<unsigned long long>(__double_as_longlong(qz)));
}

__global__ void mw_final_kernel(const unsigned long long* __restrict__ zbest, int HW, float* out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < HW) {
        const unsigned long long z = zbest[i];
        out[i] = (z == ~0ull) ? __int_as_float(0x7fc00000)
                              : __double2float_rn(__longlong_as_double(static_cast<long long>(z)));
    }
}

__global__ void cast_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, size_t n) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        y[i] = __float2bfloat16_rn(x[i]);
}

inline int launch_status() { return cudaGetLastError() == cudaSuccess ? VELOX_OK : VELOX_ECUDA; }

}  // namespace

int slices_launch(const float* depth, const float* poses, const float* intr, int P, int HW,
                  velox_slice_t* out, cudaStream_t st) {
    slices_kernel<<<P, 256, 0, st>>>(depth, poses, intr, HW, out);
    return launch_status();
}

int overlap_launch(const float* depth, const velox_slice_t* cur, const velox_slice_t* slices, int B,
                   int P, int Hp, int Wp, int T, int m, int32_t* counts, cudaStream_t st) {
    dim3 grid(m, (P + CAMS_PER_CTA - 1) / CAMS_PER_CTA, B);
    overlap_kernel<<<grid, T, 0, st>>>(depth, cur, slices, P, Hp, Wp, T, m, counts);
    return launch_status();
}

// Scratch of the multiwarp for an HW-pixel grid: z_min and the winner's depth
// (64-bit each) and the winning chunk (32-bit), each array 256-byte aligned.
constexpr size_t mw_up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
constexpr size_t mw_ws_bytes(size_t HW) { return 2 * mw_up256(HW * 8) + mw_up256(HW * 4); }

size_t multiwarp_ws_bytes(int HW) { return mw_ws_bytes(static_cast<size_t>(HW)); }

int multiwarp_launch(const float* past_depth, const velox_slice_t* past, const velox_slice_t* cur,
                     int P, int Hp, int Wp, float rel_tol, float* out, void* ws, cudaStream_t st) {
    const int HW = Hp * Wp;
    char* w = static_cast<char*>(ws);
    auto* zmin = reinterpret_cast<unsigned long long*>(w);
    auto* zbest = reinterpret_cast<unsigned long long*>(w + mw_up256(static_cast<size_t>(HW) * 8));
    auto* jwin = reinterpret_cast<int*>(w + 2 * mw_up256(static_cast<size_t>(HW) * 8));
    // n = P * HW < 2^31 (checked by the callers); block counts in 64-bit arithmetic
    const int n = P * HW;
    const unsigned pix_blocks = static_cast<unsigned>((static_cast<long long>(HW) + 255) / 256);
    const unsigned pt_blocks = static_cast<unsigned>((static_cast<long long>(n) + 255) / 256);
    const double factor = 1.0 + static_cast<double>(rel_tol);
    mw_init_kernel<<<pix_blocks, 256, 0, st>>>(zmin, jwin, zbest, HW);
    mw_zmin_kernel<<<pt_blocks, 256, 0, st>>>(past_depth, past, cur, n, Hp, Wp, zmin);
    mw_winner_kernel<<<pt_blocks, 256, 0, st>>>(past_depth, past, cur, n, Hp, Wp, factor, zmin, jwin);
    mw_depth_kernel<<<pt_blocks, 256, 0, st>>>(past_depth, past, cur, n, Hp, Wp, jwin, zbest);
    mw_final_kernel<<<pix_blocks, 256, 0, st>>>(zbest, HW, out);
    return launch_status();
}

// float64 FMA throughput: 8 independent chains per thread (enough to cover the
// pipe latency with a few warps per scheduler); a chain converges to
// y / (1 - x), never to 0, so the store below never happens but the compiler
// cannot drop the work.
__global__ void fp64_fma_kernel(double* out, int iters) {
    const double x = 0.999999, y = 1e-7 * (threadIdx.x + 1);
    double a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = 1.0 + i + 1e-3 * threadIdx.x;
#pragma unroll 4
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fma(a[i], x, y);
    }
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += a[i];
    if (s == 0.0) out[0] = s;
}

int fp64_fma_launch(double* out, int blocks, int threads, int iters, cudaStream_t st) {
    fp64_fma_kernel<<<blocks, threads, 0, st>>>(out, iters);
    return launch_status();
}

int cast_bf16_launch(const float* x, uint16_t* y, size_t n, cudaStream_t st) {
    const size_t blocks = (n + 255) / 256;
    const int g = static_cast<int>(blocks < 148 * 16 ? (blocks ? blocks : 1) : 148 * 16);
    cast_bf16_kernel<<<g, 256, 0, st>>>(x, reinterpret_cast<__nv_bfloat16*>(y), n);
    return launch_status();
}

}  // namespace velox

// ---------------------------------------------------------------- multiwarp, library-owned scratch
//
// Some callers cannot allocate device memory: a plugin whose host hands it
// only its input and output buffers, or a latency-critical loop that must not
// call cudaMalloc (which can synchronise the device). For them the multiwarp's
// per-pixel scratch lives in a fixed array in this library's own device
// memory. Each GPU that loads the library holds the array until the process
// exits. All calls share it, so calls that overlap on the GPU race.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

namespace velox {
namespace {

constexpr int NOALLOC_MAX_PIXELS = VELOX_MULTIWARP_NOALLOC_MAX_PIXELS;
// the same layout (and 256-byte rounding) the launch uses to carve the scratch
constexpr size_t NOALLOC_BYTES = mw_ws_bytes(static_cast<size_t>(NOALLOC_MAX_PIXELS));
static_assert(NOALLOC_BYTES >= mw_ws_bytes(NOALLOC_MAX_PIXELS), "scratch array too small");
constexpr int NOALLOC_CACHE = 64;

static __device__ __align__(256) unsigned char g_multiwarp_scratch[NOALLOC_BYTES];

// The driver calls that identify the current context (a CUDA context has a
// process-unique id, so a context created after cudaDeviceReset never matches
// an older entry even if its handle is reused).
struct CtxApi {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxApi& ctx_api() {
    static CtxApi api;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            api.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    return api;
}

// Device address of the array in the current context. The host-side symbol is
// only a stand-in; the real address is looked up with cudaGetSymbolAddress the
// first time a context calls, and cached under that context's id.
void* multiwarp_scratch_in_current_context() {
    static std::mutex mu;
    static unsigned long long ids[NOALLOC_CACHE] = {};
    static void* addrs[NOALLOC_CACHE] = {};
    static int next = 0;
    const CtxApi& api = ctx_api();
    if (!api.get_current || !api.get_id) return nullptr;
    void* p = nullptr;
    CUcontext ctx = nullptr;
    if (api.get_current(&ctx) != CUDA_SUCCESS) return nullptr;
    if (ctx == nullptr) {
        // no context bound to this thread yet: the runtime lookup binds the
        // device's primary context
        if (cudaGetSymbolAddress(&p, g_multiwarp_scratch) != cudaSuccess) return nullptr;
        if (api.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return nullptr;
    }
    unsigned long long id = 0;
    if (api.get_id(ctx, &id) != CUDA_SUCCESS) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < NOALLOC_CACHE; ++i)
        if (addrs[i] != nullptr && ids[i] == id) return addrs[i];
    if (p == nullptr && cudaGetSymbolAddress(&p, g_multiwarp_scratch) != cudaSuccess) return nullptr;
    ids[next] = id;
    addrs[next] = p;
    next = (next + 1) % NOALLOC_CACHE;
    return p;
}

}  // namespace
}  // namespace velox

extern "C" int velox_depth_multiwarp_noalloc(const float* past_depth,
                                             const velox_slice_t* past_cams,
                                             const velox_slice_t* cur_cam, int P, int Hp, int Wp,
                                             float rel_tol, float* cur_depth, void* stream) {
    if (!past_depth || !past_cams || !cur_cam || !cur_depth) return VELOX_EINVAL;
    if (P < 1 || Hp < 1 || Wp < 1 || !(rel_tol >= 0.0f) || !isfinite(rel_tol)) return VELOX_EINVAL;
    if (static_cast<long long>(Hp) * Wp > velox::NOALLOC_MAX_PIXELS) return VELOX_EINVAL;
    if (static_cast<long long>(P) * Hp * Wp >= (1ll << 31)) return VELOX_EINVAL;
    void* scratch = velox::multiwarp_scratch_in_current_context();
    if (scratch == nullptr) return VELOX_ECUDA;
    // the launch sequence starts by resetting the per-pixel state it uses
    return velox::multiwarp_launch(past_depth, past_cams, cur_cam, P, Hp, Wp, rel_tol, cur_depth,
                                   scratch, static_cast<cudaStream_t>(stream));
}
