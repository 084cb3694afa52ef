/*
 * velox.h -- C ABI of libvelox, the B200 (sm_100a) implementation of the Velox
 * geometry-routed block-sparse attention path.
 *
 * The method (pages "Velox: Raumgedaechtnis beschleunigt Video-Weltmodelle",
 * section "Tiefenanalyse", and "Velox: 공간 메모리로 비디오 월드 모델 추론 가속",
 * sections "배경" and "심층 분석") routes each query token block of the current
 * chunk of a chunked video-diffusion world model to a subset of the key blocks
 * of the growing KV cache:
 *   1. every past chunk is a camera-frustum slice with a depth interval;
 *   2. the current chunk's depth comes from a recency-priority multiwarp of
 *      past depth into the current view;
 *   3. the overlap of a query block's 3D region with each past slice softly
 *      modulates the block importance the model computes itself; regions that
 *      no history covers get no geometric bias;
 *   4. routing happens at token-block granularity, the attention tile, so the
 *      kernel really skips the blocks it was not given.
 * The pages fix no formula; the readings implemented here are stated on each
 * entry point below.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise. The library never allocates, frees or synchronises;
 *     scratch memory, where an operation needs it, is passed in by the caller
 *     (sizes from the matching *_workspace_size function). The one exception
 *     is velox_depth_multiwarp_noalloc, whose scratch is a fixed array owned
 *     by the library.
 *   - Tensors are dense, row-major, innermost dimension last. Q/K/V/O use the
 *     layout [B][H][N][d]. In the KV cache the past chunks come first (oldest
 *     first) and the current chunk occupies the last Nq keys.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream): it validates its arguments, enqueues kernels and returns.
 *     A rejected call (VELOX_EINVAL / VELOX_EUNSUPPORTED) launches nothing.
 *   - Calls hold no global state and may run concurrently on distinct streams
 *     with distinct outputs and workspaces -- except velox_depth_multiwarp_noalloc:
 *     all its calls share the library's scratch array, so they must not
 *     overlap on the GPU (serialise them, e.g. on one stream).
 *   - `status` arguments (may be NULL) point to one device int32 that kernels
 *     OR VELOX_STATUS_* bits into when they detect a bad index or give up a
 *     bounded wait; the caller zeroes it and reads it back.
 */
#ifndef VELOX_H
#define VELOX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VELOX_API __attribute__((visibility("default")))
#else
#define VELOX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define VELOX_OK 0
#define VELOX_EINVAL (-1)       /* bad shape, null or misaligned pointer, topk out of range */
#define VELOX_EUNSUPPORTED (-2) /* valid request outside the compiled variants (T, d, dtype) */
#define VELOX_ECUDA (-3)        /* a CUDA runtime / driver call or kernel launch failed */
#define VELOX_ETIMEOUT (-4)     /* reported through the status word: a bounded wait expired */
#define VELOX_EBOUNDS (-5)      /* reported through the status word: an index was out of range */

/* status-word bits */
#define VELOX_STATUS_BAD_INDEX 1
#define VELOX_STATUS_TIMEOUT 2

/* element types */
#define VELOX_BF16 0
#define VELOX_F32 1

/* A camera, and for a past chunk its frustum slice (72 bytes, float32).
 * R: world->camera rotation, row-major; x_c = R x_w + t. Camera axes follow
 * OpenCV (x right, y down, z forward); depth is z-depth (not ray length).
 * fx, fy, cx, cy: pinhole intrinsics in latent-grid pixel units; pixel (r, c)
 * has its centre at (c + 0.5, r + 0.5).
 * [znear, zfar]: closed depth interval of the slice; empty when znear > zfar
 * (the empty slice is [+inf, -inf]). Ignored where a call says so. */
typedef struct velox_slice_t {
    float R[9];
    float t[3];
    float fx, fy, cx, cy;
    float znear, zfar;
} velox_slice_t;

/* Library version (major*10000 + minor*100 + patch). */
VELOX_API int velox_version(void);

/* Human-readable text for a return code (static string, never NULL). */
VELOX_API const char* velox_strerror(int code);

/*
 * Frustum slices of past chunks (step 1 of "Tiefenanalyse": each past chunk is
 * a camera-frustum slice with a depth interval).
 *   depth  [P][Hp][Wp] float32  depth map of each past chunk (shared by its frames)
 *   poses  [P][12] float32      R (9, row-major) then t (3), world->camera
 *   intr   [P][4] float32       fx, fy, cx, cy
 *   slices [P] velox_slice_t    output
 * Reading: [znear, zfar] = [min, max] of the chunk's valid depth samples
 * (finite and > 0); a chunk with no valid sample gets the empty slice.
 * Errors: VELOX_EINVAL for P < 1, Hp < 1, Wp < 1 or a NULL pointer.
 */
VELOX_API int velox_slices_build(const float* depth, const float* poses, const float* intr, int P, int Hp,
                       int Wp, velox_slice_t* slices, void* stream);

/*
 * Query-block / past-slice overlap counts (steps 1 and 3 of "Tiefenanalyse";
 * region-level context choice of "배경").
 *   cur_depth [B][Hp][Wp] float32  current-chunk depth (NaN, inf or <= 0: no depth)
 *   cur_cam   [B] velox_slice_t    current camera (znear/zfar ignored)
 *   slices    [B][P] velox_slice_t past slices
 *   counts    [B][m][P] int32      output, m = F*Hp*Wp / T
 * Token tau of the current chunk (raster order frame, row, column) sits at the
 * centre of pixel (r, c) = ((tau mod Hp*Wp) / Wp, tau mod Wp) of the chunk's
 * depth map. It is back-projected with the current camera, moved into camera j
 * and counted for slice j when znear_j <= z <= zfar_j, z > 0 and its
 * projection lies in [0, Wp) x [0, Hp). Tokens without valid depth count as
 * outside. Geometry runs in float64 with a fixed operation order and no fused
 * multiply-add, so counts are exact and reproducible.
 * Errors: VELOX_EINVAL for non-positive sizes, F*Hp*Wp not a multiple of T,
 * or a NULL pointer.
 */
VELOX_API int velox_block_overlap(const float* cur_depth, const velox_slice_t* cur_cam,
                        const velox_slice_t* slices, int B, int P, int F, int Hp, int Wp, int T,
                        int32_t* counts, void* stream);

/* Bytes of scratch velox_route_topk needs for these sizes (0 on bad sizes):
 * q-bar (B*H*m*d floats) and the block scores (B*H*m*n_past floats); with
 * T = 64 also the pooled past keys (B*H*n_past*d floats), which that block
 * size scores from after pooling them all (see velox_route_topk). */
VELOX_API size_t velox_route_topk_workspace_size(int B, int H, int Nq, int Nk, int d, int T);

/*
 * Geometry-modulated block routing (step 3 of "Tiefenanalyse": the slice
 * overlap softly modulates the model's own block importance; step 4: regions
 * no history covers keep the model's own routing).
 *   q      [B][H][Nq][d], k [B][H][Nk][d]  dtype VELOX_BF16 or VELOX_F32
 *   counts [B][m][P] int32 from velox_block_overlap, or NULL (no geometry)
 *   idx    [B][H][m][topk] int32 output: selected key blocks, ascending
 *   ws     scratch of velox_route_topk_workspace_size bytes (256-B aligned)
 *   counts_ready  a cudaEvent_t or NULL. When set, only the final selection
 *          kernel waits for it (cudaStreamWaitEvent): pooling and scoring, which
 *          do not read the counts, run meanwhile -- so the geometry (slices,
 *          overlap) can be produced on another stream at the same time.
 * with m = Nq/T query blocks, P = Nk/Nq - 1 past chunks, n_past = P*m past key
 * blocks, and key block kb covering keys [kb*T, (kb+1)*T).
 * Readings implemented:
 *   s[qb][kb]  = mean_T(Q block qb) . mean_T(K block kb) / sqrt(d)   (fp32)
 *   s'[qb][kb] = s + alpha * counts[qb][kb / m] / T   if sum_j counts[qb][j] > 0
 *              = s                                    otherwise (no bias)
 *   per (b, h, qb): the m current-chunk blocks are always kept and the
 *   topk - m past blocks with the largest s' are added (equal s': the smaller
 *   kb first). topk counts the current blocks.
 * With T = 128 each key block is scored as it is pooled; with T = 64 (twice the
 * query blocks per byte of K) every past block is pooled into the workspace
 * first and scored from there. Both give bit-identical scores.
 * Errors: VELOX_EINVAL for sizes that are not multiples (Nq % T, Nk % Nq),
 * more than 8192 key blocks (Nk/T), topk < m or topk > Nk/T, ws_bytes too
 * small, NULL or misaligned (16 B) pointers; VELOX_EUNSUPPORTED for T not in
 * {64,128}, d not in {64,128}, or an unknown dtype.
 */
VELOX_API int velox_route_topk(const void* q, const void* k, int dtype, int B, int H, int Nq, int Nk, int d,
                     int T, const int32_t* counts, float alpha, int topk, int32_t* idx, void* ws,
                     size_t ws_bytes, void* counts_ready, void* stream);

/*
 * Block-sparse attention forward over the routed blocks (step 4 of
 * "Tiefenanalyse"; the kernel walks only the listed key blocks).
 *   q [B][H][Nq][d], k/v [B][H][Nk][d]  bf16
 *   idx  [B][H][m][topk] int32, or NULL for dense attention over all Nk/T blocks
 *   o    [B][H][Nq][d] bf16 output
 *   lse  [B][H][Nq] float32 output (natural log of the softmax denominator of
 *        the scaled scores), or NULL
 * For every query row i of block qb: O_i = sum_j softmax_j(scale * Q_i.K_j) V_j
 * over the keys j of the listed blocks (no mask inside blocks; a block listed
 * twice counts twice). Tensor cores (tcgen05, TMEM accumulators) compute
 * Q K^T and P V in bf16 with fp32 accumulation; the softmax runs online in fp32.
 * Out-of-range entries of idx are replaced by block 0 and flagged in *status
 * (VELOX_STATUS_BAD_INDEX); bounded internal waits flag VELOX_STATUS_TIMEOUT.
 * Errors: VELOX_EINVAL for Nq % T, Nk % T, topk outside [1, Nk/T] (when idx is
 * given), NULL or non-16-byte-aligned q/k/v/o; VELOX_EUNSUPPORTED for T or d
 * outside {64,128}; VELOX_ECUDA when a tensor map cannot be encoded or the
 * launch fails.
 */
VELOX_API int velox_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                          int topk, int B, int H, int Nq, int Nk, int d, int T, float scale,
                          void* o, float* lse, int32_t* status, void* stream);

/* test-hook flags of velox_sparse_attn_fwd_test */
#define VELOX_TEST_SKIP_MMA 1
#define VELOX_TEST_FORCE_PAIR 2

/*
 * velox_sparse_attn_fwd with two test hooks for its failure path; not a step
 * of the method. Every wait inside the attention kernels is bounded: a wait
 * that runs out sets VELOX_STATUS_TIMEOUT in *status, the CTA's other waits
 * give up, copies already in flight are drained and the kernel returns, so
 * the device stays usable. This entry point lets a test reach that path
 * without a fault:
 *   wait_limit_s  limit of each bounded wait, in seconds, in [1e-3, 10]
 *                 (velox_sparse_attn_fwd uses 2 s);
 *   flags         VELOX_TEST_SKIP_MMA: the tensor-core issuer issues nothing,
 *                 so no MMA completion ever arrives and the waits on them run
 *                 out (no MMA is in flight when tensor memory is freed); the
 *                 output is left unwritten.
 *                 VELOX_TEST_FORCE_PAIR: for d = T = 128, run the CTA-pair
 *                 kernel (two SMs per MMA, the union of two blocks' lists
 *                 walked once) also for routed lists, which otherwise go to the
 *                 single-SM two-block kernel; lists of more than 2048 blocks
 *                 still go there. 0: a normal call.
 * Other arguments, results and errors are those of velox_sparse_attn_fwd;
 * VELOX_EINVAL also for a limit outside the range or an unknown flag.
 */
VELOX_API int velox_sparse_attn_fwd_test(const void* q, const void* k, const void* v,
                                         const int32_t* idx, int topk, int B, int H, int Nq,
                                         int Nk, int d, int T, float scale, void* o, float* lse,
                                         int32_t* status, double wait_limit_s, int flags,
                                         void* stream);

/*
 * Pooled-key cache (an incremental form of the routing's key pooling; the
 * block importance the model computes in each layer, "Tiefenanalyse" step 3,
 * only ever needs the mean of each past key block, and a past chunk's keys
 * never change once the chunk is done).
 * The cache holds, per (b, h), the mean of each T-token key block of up to
 * max_past_chunks chunks: kbar [B][H][max_past_chunks * m][d] float32, m = Nq/T.
 */
VELOX_API size_t velox_kbar_cache_bytes(int B, int H, int max_past_chunks, int Nq, int d, int T);

/*
 * Pools the m key blocks of chunk `chunk` (keys [chunk*Nq, (chunk+1)*Nq) of every
 * (b, h) of the KV cache k [B][H][Nk][d], dtype VELOX_BF16 or VELOX_F32) into
 * kbar[b][h][chunk*m + i][:]. Call it once per chunk, when the chunk is done.
 * The values are bit-identical to the pooling velox_route_topk does itself.
 * Errors: VELOX_EINVAL for sizes that are not multiples, chunk outside
 * [0, max_past_chunks), keys [chunk*Nq, (chunk+1)*Nq) beyond Nk, NULL or
 * misaligned (16 B) pointers; VELOX_EUNSUPPORTED as velox_route_topk.
 */
VELOX_API int velox_kbar_append(const void* k, int dtype, int B, int H, int Nk, int Nq, int d, int T,
                                int chunk, float* kbar, int max_past_chunks, void* stream);

/*
 * velox_route_topk with the past key blocks taken from the pooled-key cache
 * instead of K: P past chunks (P <= max_past_chunks, chunks 0..P-1 appended)
 * and the current chunk, Nk = (P + 1) * Nq. Same arguments, semantics,
 * workspace (velox_route_topk_workspace_size(B, H, Nq, (P+1)*Nq, d, T)) and
 * errors; the selected blocks equal velox_route_topk's on the same keys.
 */
VELOX_API int velox_route_topk_cached(const void* q, int dtype, const float* kbar,
                                      int max_past_chunks, int B, int H, int Nq, int P, int d, int T,
                                      const int32_t* counts, float alpha, int topk, int32_t* idx,
                                      void* ws, size_t ws_bytes, void* counts_ready, void* stream);

/* Bytes of scratch velox_depth_multiwarp needs (0 on bad sizes). */
VELOX_API size_t velox_depth_multiwarp_workspace_size(int Hp, int Wp);

/*
 * Recency-priority multiwarp (step 2 of "Tiefenanalyse": past depth is warped
 * into the current view and recent history takes precedence).
 *   past_depth [P][Hp][Wp] float32, past_cams [P] velox_slice_t (znear/zfar
 *   ignored), cur_cam [1] velox_slice_t, cur_depth [Hp][Wp] float32 output.
 * Every valid past pixel (finite, > 0) is back-projected with its own camera,
 * moved into the current camera and, when in front of it and on the grid,
 * splatted on the pixel that contains its projection (floor). Per target
 * pixel: z_min = nearest candidate depth; candidates with
 * z <= z_min * (1 + rel_tol) win; the most recent winning chunk (largest
 * index) gives its smallest depth, rounded to float32. No candidate: NaN.
 * Float64 geometry, fixed operation order, no fused multiply-add.
 * ws: scratch of velox_depth_multiwarp_workspace_size bytes (8-B aligned).
 * Errors: VELOX_EINVAL for non-positive sizes, rel_tol < 0, a small workspace
 * or NULL pointers.
 */
VELOX_API int velox_depth_multiwarp(const float* past_depth, const velox_slice_t* past_cams,
                          const velox_slice_t* cur_cam, int P, int Hp, int Wp, float rel_tol,
                          float* cur_depth, void* ws, size_t ws_bytes, void* stream);

/* Largest grid (Hp * Wp) velox_depth_multiwarp_noalloc accepts. */
#define VELOX_MULTIWARP_NOALLOC_MAX_PIXELS 65536

/*
 * velox_depth_multiwarp without a caller workspace. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory -- e.g. a plugin whose host passes it only its input and output
 * buffers, or a latency-critical loop that must not call cudaMalloc, which can
 * synchronise the device. Arguments and results are those of
 * velox_depth_multiwarp, minus ws / ws_bytes. Nothing is allocated or freed:
 * the scratch (20 bytes per pixel) is a fixed array in the library's own
 * device memory, 1.25 MiB, held on every GPU that loads the library until the
 * process exits.
 *   - Hp * Wp above VELOX_MULTIWARP_NOALLOC_MAX_PIXELS returns VELOX_EINVAL and
 *     launches nothing.
 *   - The first call in a CUDA context (normally: the first call on a device,
 *     whose primary context the runtime uses) looks up the array's device
 *     address with that context current and caches it under the context's
 *     id; make that first call before any stream capture. A context created
 *     later for the same device (after cudaDeviceReset, say) gets its own
 *     lookup. A failed lookup returns VELOX_ECUDA.
 *   - Every call resets the scratch it uses before reading it, but all calls
 *     share one array: calls whose kernels overlap on the GPU (e.g. on two
 *     streams at once) race and give wrong depths. Serialise them.
 */
VELOX_API int velox_depth_multiwarp_noalloc(const float* past_depth,
                                            const velox_slice_t* past_cams,
                                            const velox_slice_t* cur_cam, int P, int Hp, int Wp,
                                            float rel_tol, float* cur_depth, void* stream);

/*
 * float32 -> bf16 (round to nearest even) for n elements; used where a
 * workload's Q/K/V arrive in float32 and the attention tiles take bf16.
 * Errors: VELOX_EINVAL for NULL pointers.
 */
VELOX_API int velox_cast_bf16(const float* x, uint16_t* y, size_t n, void* stream);

/*
 * Measurement helper, not a step of the method: blocks x threads threads each
 * run `iters` rounds of 8 independent float64 fused multiply-adds (2 FLOP each:
 * blocks * threads * iters * 16 FLOP per call), the ceiling that the float64
 * geometry (velox_block_overlap) is compared with. `out` (one double, device)
 * is written only in a case that does not occur, so the work cannot be
 * optimised away. Errors: VELOX_EINVAL for NULL out, blocks < 1, threads not a
 * multiple of 32 in [32, 1024], iters < 1.
 */
VELOX_API int velox_fp64_fma_bench(double* out, int blocks, int threads, int iters, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VELOX_H */
