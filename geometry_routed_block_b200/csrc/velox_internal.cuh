// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/velox.h"

namespace velox {

// default limit of the attention kernels' bounded waits: 2 s, far above any
// legitimate wait
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;

struct AttnArgs {
    const int32_t* idx;  // [B*H][m][n_sel] or nullptr (dense)
    int n_sel;           // key blocks per query block
    int H, Nq, Nk, T, m, n_kb;
    float scale_log2;    // softmax scale * log2(e)
    __nv_bfloat16* o;
    float* lse;
    int32_t* status;
    const __nv_bfloat16* q;  // set by the launcher
    long long q_rows;        // B * H * Nq
    unsigned long long wait_ns;  // limit of every bounded wait
    int skip_mma;                // test hook: the tensor-core issuer issues nothing
    int force_pair;              // test hook: d = T = 128 on the CTA-pair kernel
    int pair_tiles;              // set by the launcher: two 64-token blocks per 128-row tile
};

int attn_fwd_launch(const void* q, const void* k, const void* v, const AttnArgs& a, int B, int d,
                    cudaStream_t st);

int slices_launch(const float* depth, const float* poses, const float* intr, int P, int HW,
                  velox_slice_t* out, cudaStream_t st);
int overlap_launch(const float* depth, const velox_slice_t* cur, const velox_slice_t* slices, int B,
                   int P, int Hp, int Wp, int T, int m, int32_t* counts, cudaStream_t st);
size_t multiwarp_ws_bytes(int HW);
int multiwarp_launch(const float* past_depth, const velox_slice_t* past, const velox_slice_t* cur,
                     int P, int Hp, int Wp, float rel_tol, float* out, void* ws, cudaStream_t st);

struct RouteArgs {
    int B, H, Nq, Nk, d, T, m, P, n_past, topk;
    const int32_t* counts;
    float alpha, inv_sqrt_d;
    int32_t* idx;
    float* qbar;    // workspace [B*H*m][d]
    float* scores;  // workspace [B*H*m][n_past]
    cudaEvent_t counts_ready;  // selection waits for it when set
    const float* kbar;         // k-bar cache [B*H][kbar_cap][d], or nullptr: pool K here
    int kbar_cap;              // blocks per (b, h) in the cache
    float* kbar_ws;            // workspace [B*H][n_past][d] when the scoring is split, else nullptr
};
// Whether routing without a k-bar cache pools every past key block into the
// workspace first and scores from there (instead of scoring each block as it
// is pooled): for the block shapes whose scoring per byte of K would hold
// the stream back.
bool route_split_scoring(int T, int d);
size_t route_ws_bytes(int B, int H, int m, int n_past, int d, int T);
int route_launch(const void* q, const void* k, int dtype, const RouteArgs& r, cudaStream_t st);

int kbar_append_launch(const void* k, int dtype, int BH, int Nk, int Nq, int d, int T, int chunk,
                       int cap, float* kbar, cudaStream_t st);

int cast_bf16_launch(const float* x, uint16_t* y, size_t n, cudaStream_t st);
int fp64_fma_launch(double* out, int blocks, int threads, int iters, cudaStream_t st);

}  // namespace velox
