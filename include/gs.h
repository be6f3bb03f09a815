/*
 * gs.h -- C ABI of the B200 differentiable tile rasterizer for 3D Gaussian
 * splats (libgs.so).
 *
 * The method: a per-view active-set cull, per-Gaussian EWA projection with
 * spherical-harmonic colour, binning of (Gaussian, tile) pairs by a 64-bit
 * key (tile_id << 32 | depth bits) with a stable radix sort, per-tile range
 * extraction, front-to-back alpha compositing per pixel over 16x16 tiles,
 * and the matching backward pass.
 *
 * Sources on the pages this library follows:
 *  - BlitzGS (CVPR 2026) write-up, section 2.3 "视图层级精细化修剪": per-view
 *    active set from a distance-LOD gate and an importance cull mask.
 *  - 4D-GS release page ("VisionTech 发布并开源 ... 120fps 实时渲染"), section
 *    "技术架构与关键机制": tiled rasterization with per-pixel alpha blending.
 *  - "像素扩散与CUDA内核优化" (Gsplat part), section 三.2: projection stages
 *    as separate parallel blocks; spatially local data staged in shared memory.
 *  - Spirula Studio quantised-training page, sections "先算一笔账" (full SH3
 *    colour, 45 coefficients per Gaussian) and "实测" (64-bit element addressing
 *    once element counts pass 2^31).
 *
 * Conventions for every entry point
 *  - Pointers marked [device] are CUDA device pointers owned by the caller;
 *    the library never allocates, frees or retains them. Pointers marked
 *    [host] are read during the call only.
 *  - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *    stream. Work is enqueued asynchronously on it unless stated otherwise.
 *  - Calls that need scratch memory take (workspace, workspace_bytes). With
 *    workspace == NULL the call only stores the required size in
 *    *workspace_bytes and returns GS_OK. The workspace must be 256-byte
 *    aligned and not shared by calls in flight at the same time.
 *  - Parameters use structure-of-arrays planes of float32, element counts in
 *    int64 (SH planes hold 48*N floats, past 2^31 elements at 45M Gaussians).
 *      means [3][N], log_scales [3][N], quats [4][N] as (w, x, y, z),
 *      opacity_logits [N], sh [K*3][N] with plane index k*3 + channel,
 *      K = (sh_degree + 1)^2.
 *  - Images are channel-planar: image [3][H][W]; per-pixel maps are [H][W].
 *    Pixel (u, v) is sampled at (u + 0.5, v + 0.5); tiles are 16x16 pixels,
 *    TW = ceil(W/16), TH = ceil(H/16), tile id = ty*TW + tx.
 *  - Return values are GS_* codes below; on an error the outputs are
 *    unspecified. GS_ERR_CUDA means a CUDA runtime call failed (the CUDA error
 *    is left for the caller to query with cudaGetLastError).
 *  - Arithmetic follows a fixed fp32 specification (operation order, explicit
 *    fused multiply-adds, a software exp2) so that every discrete result --
 *    cull masks, radii, tile rects, keys, sorted order, ranges and per-pixel
 *    contributor counts -- is reproducible bit for bit by an independent CPU
 *    implementation.
 */
#ifndef GS_H_
#define GS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GS_API __attribute__((visibility("default")))

enum {
  GS_OK = 0,
  GS_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad camera, ...  */
  GS_ERR_CAPACITY = 2,         /* more (Gaussian, tile) instances than capacity */
  GS_ERR_CUDA = 3,             /* a CUDA runtime call failed                    */
  GS_ERR_DEVICE_TIMEOUT = 4,   /* a bounded device-side wait gave up            */
  GS_ERR_UNSUPPORTED = 5       /* e.g. sh_degree > 3                            */
};

/* Pinhole camera, OpenCV axes (x right, y down, z forward). */
typedef struct gs_camera {
  float R[9];      /* world -> camera rotation, row-major                        */
  float t[3];      /* world -> camera translation: t_cam = R mu + t              */
  float campos[3]; /* camera centre in world coordinates (SH direction, LOD)     */
  float fx, fy, cx, cy; /* intrinsics in pixels                                   */
  float near_z;    /* Gaussians with camera-space z <= near_z are culled; >= 0    */
  int32_t width, height; /* image size in pixels, each in [1, 65535*16]          */
} gs_camera;

/* Projected records, one per active position (structure of small vectors).
 * A record is written in full only for a visible Gaussian (tiles_touched > 0);
 * all fields of other records are zero. */
typedef struct gs_projected {
  float* xyzo;            /* [device] [cap][4]: px, py, depth (camera z), opacity */
  float* conic;           /* [device] [cap][4]: A, B, C of Sigma'^-1, 0           */
  float* rgb;             /* [device] [cap][4]: r, g, b, 0                        */
  int32_t* radius;        /* [device] [cap]: ceil(3 sqrt(lambda_max(Sigma')))     */
  uint16_t* rect;         /* [device] [cap][4]: x0, y0, x1, y1 tile rect, end-excl*/
  int32_t* tiles_touched; /* [device] [cap]: (x1 - x0) * (y1 - y0)                */
} gs_projected;

GS_API int gs_version(void);
GS_API const char* gs_status_string(int status);

/* Per-view active-set cull (BlitzGS write-up, section 2.3: distance-LOD gate
 * and importance cull mask).
 *   keep(g) = [lod_dist <= 0 or |mu_g - campos|^2 <= lod_dist^2]
 *           and [importance_q == 0 or importance[g] >= tau]
 * with the squared distance in fp32 as ((dx*dx + dy*dy) + dz*dz) and tau the
 * value of rank floor(q*N) (0-based, ascending, total order on the fp32 bit
 * patterns) among all N weights. Then order-preserving compaction.
 *   means        [device] [3][N]
 *   importance   [device] [N], may be NULL when importance_q == 0
 *   N            number of Gaussians, 0 <= N < 2^31
 *   cam          [host] camera (campos is used)
 *   importance_q in [0, 1)
 *   mask         [device] [N] u8 out: 1 kept, 0 culled
 *   active_idx   [device] [N] i32 out: kept indices in increasing order
 *   n_active     [device] i32 out: number of kept Gaussians
 *   workspace    [device] scratch, see conventions
 * Asynchronous. */
GS_API int gs_cull(const float* means, const float* importance, int64_t N, const gs_camera* cam,
                   float lod_dist, float importance_q, uint8_t* mask, int32_t* active_idx,
                   int32_t* n_active, void* workspace, size_t* workspace_bytes, void* stream);

/* gs_cull without a workspace, for callers that cannot allocate device
 * memory: a plugin inside a host application that does not own the device
 * allocator, or a real-time loop that may not call cudaMalloc (it synchronises
 * the whole device). The pages have no counterpart of this entry point; it is
 * an interface convenience over gs_cull, whose results it reproduces exactly.
 * Its scratch is a 32 KiB array in the library image, which every GPU that
 * loads the library holds until the process exits. The call allocates
 * nothing.
 *   arguments    as for gs_cull, without workspace/workspace_bytes
 *   N            at most GS_CULL_NOALLOC_MAX_N; larger N returns
 *                GS_ERR_INVALID_ARGUMENT (use gs_cull with a workspace)
 * Each CUDA context that loads the library (a device's primary context, a
 * context the host application created itself, the primary context again
 * after cudaDeviceReset) holds its own copy of the array. The first call made
 * in a context looks up that copy's device address (cudaGetSymbolAddress) and
 * caches it under the context's unique id; make that first call before any
 * stream capture in the context. Every call shares the one array: each
 * clears what must start at zero, but calls that overlap on the GPU (other
 * streams or host threads) race on it. Asynchronous otherwise. */
#define GS_CULL_NOALLOC_MAX_N 16777216
GS_API int gs_cull_noalloc(const float* means, const float* importance, int64_t N, const gs_camera* cam,
                           float lod_dist, float importance_q, uint8_t* mask, int32_t* active_idx,
                           int32_t* n_active, void* stream);

/* Projection of every active Gaussian into records (EWA splatting):
 *   t = R mu + t, culled unless t.z > near_z; s = exp(log_s); q normalised;
 *   Sigma = Rq S S^T Rq^T; J = d(pinhole)/dt at t;
 *   Sigma' = J R Sigma R^T J^T + 0.3 I; culled unless det(Sigma') > 0;
 *   conic = Sigma'^-1; radius = ceil(3 sqrt(lambda_max)); centre
 *   (fx tx/tz + cx, fy ty/tz + cy); tile rect of the radius square clamped to
 *   the grid, culled if empty; opacity = 1/(1 + exp(-logit));
 *   colour = max(0, sum_k Y_k(dir) sh_k + 0.5) with dir = (mu - campos)/|.|
 *   and Y the real orthonormal SH basis (Condon-Shortley phase), l <= sh_degree.
 * Non-finite means, log-scales, quaternions or logits, and zero quaternions,
 * cull the Gaussian.
 *   active_idx   [device] [N] or NULL (record i is Gaussian i)
 *   n_active     [device] i32 or NULL (then N). Records i >= n_active get
 *                tiles_touched = 0.
 *   out          [host] struct of [device] arrays with capacity N
 * Asynchronous. */
GS_API int gs_preprocess(const float* means, const float* log_scales, const float* quats,
                         const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                         const int32_t* active_idx, const int32_t* n_active, const gs_camera* cam,
                         const gs_projected* out, void* stream);

/* Densification statistic of a view, from the raster backward's 2-D
 * gradients: for every record i that the view sees (tiles_touched > 0,
 * i < n_active), norm_sum[g] += sqrt(dpx^2 + dpy^2) and view_count[g] += 1,
 * with g = active_idx[i] (or i). Called once per view after
 * gs_rasterize_bwd(_2d); the mean norm_sum / view_count is the usual
 * densification criterion of Gaussian-splat training (positional gradient
 * in screen space). The pages print no formula for it; it pairs with the
 * importance weights (gs_rasterize_fwd_importance) as the two per-Gaussian
 * statistics a training schedule reads.
 *   grad2d        [device] [n_records][12] from gs_rasterize_bwd(_2d)
 *   tiles_touched [device] [n_records] i32 of the view's records
 *   active_idx, n_active [device] from gs_cull, or NULL
 *   norm_sum      [device] [N] f32 in/out (added to)
 *   view_count    [device] [N] i32 in/out (added to)
 * fp32: the norm is sqrt(fma(dpx, dpx, dpy * dpy)). Asynchronous. */
GS_API int gs_accumulate_grad2d_norm(const float* grad2d, const int32_t* tiles_touched,
                                     const int32_t* active_idx, const int32_t* n_active, int64_t n_records,
                                     float* norm_sum, int32_t* view_count, void* stream);

/* ---- Quantised SH training state (Spirula Studio page, sections
 * "先算一笔账", "一个开关" and the section on 8-bit Adam states): view-dependent
 * SH coefficients stored as 16-bit linear block codes, both Adam moments as
 * 8-bit linear block codes of their logarithms, gradients in fp32. A block is
 * 256 consecutive Gaussians of one unit plane (the transposed layout the page
 * describes); planes are [U][N] with U = 3 (K - 1) at SH degree with K
 * coefficients (the DC plane is not quantised), codes at row stride
 * Npad = 256 * ceil(N / 256), bounds [U][ceil(N / 256)][2] = (lo, hi) fp32.
 * Code, per block: step = (hi - lo) / Q, inv = Q / (hi - lo) (both 0 when
 * hi == lo: every code 0), Q = 2^bits - 1; q = rint((x - lo) * inv) clamped
 * to [0, Q]; decode lo + step * q (one multiplication per unit, as the page
 * says); fp32 without fused multiply-add. The page prints only the moment transform
 * log1p(sqrt(g2) / eps) and the decode; the rest is fixed as written here. */

/* Block codes of fp32 planes x [U][N] (row stride N); bits 8 or 16
 * (codes uint8 or uint16 [U][Npad]). Padding codes are 0. Asynchronous. */
GS_API int gs_quant_encode(const float* x, int64_t U, int64_t N, int bits, void* codes, float* bounds,
                           void* stream);

/* Decoded fp32 planes x [U][N] of block codes. Asynchronous. */
GS_API int gs_quant_decode(const void* codes, const float* bounds, int64_t U, int64_t N, int bits, float* x,
                           void* stream);

/* Hyperparameters of one Adam step (step counts from 1). */
typedef struct gs_adam_config {
  double lr, beta1, beta2, eps;
  double code_scale; /* e of the moment codes, > 0 */
  int64_t step;
} gs_adam_config;

/* One fused Adam step over quantised SH state, in place. Per unit: decode
 * the value p (16-bit), m from y_m = sign(m) log1p(|m| r) and v from
 * y_v = log1p(sqrt(v) r) (8-bit codes of y; r = 1 / e rounded from double,
 * decoded as e expm1(|y|) with y's sign); then
 *   m' = b1 m + (1 - b1) g,  v' = b2 v + (1 - b2) g^2,
 *   p' = p - lr (m' c1) / (sqrt(v' c2) + eps),
 * c1 = 1 / (1 - b1^step), c2 = 1 / (1 - b2^step); each block's new bounds
 * are the min and max of its new values (of y for the moments) and the
 * codes are rewritten. log1p(z) = ln 2 log2(1 + z) with a software log2
 * (atanh series) and expm1(y) = exp2(y log2 e) - 1 with the software exp2
 * of the raster, so the codes are reproducible bit for bit. The fp32
 * constants are the roundings of lr, b1, 1 - b1, b2, 1 - b2, c1, c2, eps,
 * e and 1 / e, each computed in double.
 *   grad          [device] [U][N] fp32 (e.g. d_sh + 3 N of gs_rasterize_bwd)
 *   value_codes   [device] [U][Npad] u16, value_bounds [U][nblk][2]
 *   m_codes, v_codes [device] [U][Npad] u8, m_bounds, v_bounds [U][nblk][2]
 * A zero state (all codes 0, all bounds 0) is m = v = 0. One warp per block;
 * HBM traffic 12 bytes per unit plus the bounds. Asynchronous. */
GS_API int gs_adam_sh_quant(const float* grad, int64_t U, int64_t N, uint16_t* value_codes, float* value_bounds,
                            uint8_t* m_codes, float* m_bounds, uint8_t* v_codes, float* v_bounds,
                            const gs_adam_config* cfg, void* stream);

/* ---- Index-interleaved multi-GPU rendering with one exchange (BlitzGS
 * write-up, section 2.1 "系统层级索引分割": Gaussians are dealt to GPUs by
 * index, each GPU projects its own, and one centralised exchange routes the
 * projected Gaussians to the GPUs that own the screen tiles they touch).
 * Readings: rank r of G holds Gaussians g = l G + r (local record l) and owns
 * the tile rows [floor(r TH / G), floor((r + 1) TH / G)); a record is sent to
 * every rank whose rows its rect reaches; no cull. The collective is the
 * caller's (counts, then one all-to-all of GS_WIRE_RECORD_BYTES-byte records;
 * after the backward the reverse all-to-all of 12-float gradient rows). */
#define GS_WIRE_RECORD_BYTES 64
#define GS_MAX_RANKS 32

/* CTAs of gs_route_count / gs_route_pack for n records (size of cta_counts
 * is gs_route_ctas(n) * n_ranks). */
GS_API int64_t gs_route_ctas(int64_t n);

/* Which ranks each visible record (tiles_touched > 0) goes to: rank q owns
 * the tile rows [band_starts[q], band_starts[q + 1]).
 *   band_starts [host] [n_ranks + 1] i32: non-decreasing, from 0 to tiles_y
 *               (else GS_ERR_INVALID_ARGUMENT); NULL: equal bands,
 *               band_starts[q] = floor(q tiles_y / n_ranks)
 *   mask        [device] [n] u32 out: bit q = sent to rank q
 *   cta_counts  [device] [gs_route_ctas(n)][n_ranks] u32 out: per-CTA
 *               exclusive offsets within each destination
 *   totals      [device] [n_ranks] i64 out: records for each destination
 *   dst_offsets [device] [n_ranks] i64 out, or NULL: the exclusive scan of
 *               totals (each destination's first slot in gs_route_pack's
 *               send buffer), so that the pack needs no host round trip
 * Asynchronous. */
GS_API int gs_route_count(const gs_projected* rec, int64_t n, int n_ranks, int tiles_y, const int32_t* band_starts,
                          uint32_t* mask, uint32_t* cta_counts, int64_t* totals, int64_t* dst_offsets,
                          void* stream);

/* Packs the records for every destination into send (wire records,
 * destination-major, each destination's records in ascending index);
 * dst_offsets [device] [n_ranks] i64 = exclusive scan of totals;
 * src_idx [device] [sum totals] i32 out = local record of each slot. The
 * global index sent is l * n_ranks + rank. Asynchronous. */
GS_API int gs_route_pack(const gs_projected* rec, const uint32_t* mask, int64_t n, int n_ranks, int rank,
                         const uint32_t* cta_offsets, const int64_t* dst_offsets, void* send, int32_t* src_idx,
                         void* stream);

/* The received wire records (n_ranks segments, seg_offsets [device]
 * [n_ranks + 1] i64, each ascending in global index) merged into records
 * ordered by global index, rects clamped to the tile rows
 * [tile_row_lo, tile_row_hi) (tiles_touched recomputed), so that bin/sort and
 * raster on them give this rank's rows exactly as one GPU renders them.
 *   out   records, capacity n_recv;  perm [device] [n_recv] i32 out: the
 *         received position of each merged record. Asynchronous. */
GS_API int gs_merge_received(const void* recv, const int64_t* seg_offsets, int n_ranks, int64_t n_recv,
                             int tile_row_lo, int tile_row_hi, const gs_projected* out, int32_t* perm,
                             void* stream);

/* back[perm[i]] = grad2d[i] (12 floats per record): the merged records'
 * 2-D gradients in received order, ready for the reverse exchange.
 * Asynchronous. */
GS_API int gs_unmerge_grad2d(const float* grad2d, const int32_t* perm, int64_t n, float* back, void* stream);

/* grad2d[src_idx[j]] += ret[j] for the n returned gradient rows (vector
 * atomics: a record sent to several ranks gets their sum). grad2d is the
 * sender's [n_local][12] array, zeroed first. Asynchronous. */
GS_API int gs_return_grad2d(const float* ret, const int32_t* src_idx, int64_t n, float* grad2d, void* stream);

/* Views per gs_preprocess_multiview call. */
#define GS_MAX_VIEWS 16

/* gs_preprocess for several views in one pass over the parameters: each
 * Gaussian's 11 + 3K parameters are read once and projected into every view
 * (the batched multi-view step for rendering many poses of one model, as
 * in the 10M-Gaussian eight-view 4K workload). Record i of view v is
 * Gaussian i; there is no cull (every Gaussian of every view is
 * projected), and outs[v] receives exactly what gs_preprocess with
 * cams[v], active_idx = NULL writes. The pages print no kernel for this;
 * the parameter layout and per-view records follow the Gsplat page's split
 * of per-Gaussian projection from the raster stages.
 *   cams         [host] [n_views] cameras (all may differ in size)
 *   n_views      0 .. GS_MAX_VIEWS
 *   outs         [host] [n_views] record sets, each of capacity N
 * HBM traffic: (11 + 3K) * 4 bytes read + n_views * 64 bytes written per
 * Gaussian, against n_views times both for separate calls. Asynchronous. */
GS_API int gs_preprocess_multiview(const float* means, const float* log_scales, const float* quats,
                                   const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                   const gs_camera* cams, int n_views, const gs_projected* outs,
                                   void* stream);

/* Tile binning: one (key, value) per (Gaussian, tile) instance with
 * key = (tile_id << 32) | bits(depth) and value = record index, tiles in
 * row-major order within the record's rect, sorted stably by key (equal keys
 * keep record order), then [start, end) per tile into tile_ranges (empty tiles
 * [0, 0)). The sort is an LSD radix sort with 8-bit digits (onesweep passes
 * with decoupled look-back): the 32 depth bits are sorted once per visible
 * record (tiles_touched > 0; compacted in record order, so equal depths keep
 * record order), the instances are emitted in that order, and only the
 * ceil(log2(TW*TH)) tile bits are sorted over the instances, which gives the
 * same order as sorting all key bits of every instance.
 *   in           [host] struct of [device] records, n entries
 *   offsets      [device] [n] i32 out, or NULL: exclusive scan of
 *                tiles_touched in record order
 *   keys, vals   [device] [capacity] out, sorted
 *   capacity     size of keys/vals, < 2^30
 *   tile_ranges  [device] [TW*TH][2] u32 out
 *   n_instances  [host] out: number of instances I
 * The instance count is read on the device between the scan and the sort,
 * so the whole call is enqueued at once; it then waits on `stream` once to
 * read I and the device status. Returns GS_ERR_CAPACITY (with *n_instances
 * set, nothing sorted, tile_ranges all empty) when I > capacity,
 * GS_ERR_DEVICE_TIMEOUT if a look-back wait hit its iteration limit
 * (tile_ranges are then all empty). */
GS_API int gs_bin_sort(const gs_projected* in, int64_t n, const gs_camera* cam, int32_t* offsets,
                       uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* tile_ranges,
                       int64_t* n_instances, void* workspace, size_t* workspace_bytes,
                       void* stream);

/* gs_bin_sort without the wait: the same work and outputs, enqueued on
 * `stream` only, so a caller can queue several views (and their raster
 * calls) without a host round trip. The workspace is the same as
 * gs_bin_sort's. The pages have no counterpart of this split; it exists
 * because the instance count is data-dependent and reading it on the host
 * stalls the device between views.
 *   result       [device] i64[2] out, or NULL: result[0] = I, result[1] =
 *                status (GS_OK, GS_ERR_CAPACITY: I > capacity, nothing sorted;
 *                GS_ERR_DEVICE_TIMEOUT: a look-back wait hit its limit); in
 *                both error cases tile_ranges are all empty, so a raster call
 *                on them reads nothing.
 * Grids of the instance kernels are sized for `capacity` (CTAs past I exit),
 * so a capacity far above I costs idle CTAs. Argument errors are returned
 * directly; device outcomes only through `result`. Asynchronous. */
GS_API int gs_bin_sort_async(const gs_projected* in, int64_t n, const gs_camera* cam, int32_t* offsets,
                             uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* tile_ranges,
                             int64_t* result, void* workspace, size_t* workspace_bytes, void* stream);

/* Tile schedule for the raster launches: the tile indices ordered by
 * descending floor(log2) of their list length (empty lists last), so that the
 * CTAs that take the longest lists start first and the launch does not end on
 * a few long tiles running alone (a longest-processing-time-first schedule;
 * without it, CTA b takes tile b). The order within one length class is
 * unspecified. The raster outputs do not depend on it. The pages describe
 * no launch schedule (the 4D-GS page's tiled rasterization fixes only what
 * each tile computes); this is an execution order, not a step of the method.
 *   tile_ranges  [device] [n_tiles] (start, end) u32 pairs from gs_bin_sort
 *   order        [device] [n_tiles] u32 out: a permutation of 0 .. n_tiles - 1
 * One CTA. Asynchronous; GS_ERR_INVALID_ARGUMENT on NULL pointers with
 * n_tiles > 0 or n_tiles outside [0, 2^31). */
GS_API int gs_tile_order(const uint32_t* tile_ranges, int64_t n_tiles, uint32_t* order, void* stream);

/* Forward compositing (tiled rasterization with alpha blending). For each
 * pixel, over its tile's sorted list: alpha = min(0.99, o exp(p)) with
 * p = -1/2 (A dx^2 + C dy^2) - B dx dy, (dx, dy) = (px - u - 0.5, py - v - 0.5);
 * skip alpha < 1/255; C += T alpha c; T *= 1 - alpha; stop once T < 1e-4
 * (the crossing Gaussian is blended). out = C + T bg.
 *   vals, tile_ranges [device] from gs_bin_sort
 *   tile_order   [device] [tiles] u32 from gs_tile_order, or NULL: the order
 *                in which the CTAs take the tiles; it changes no output bit
 *   bg           [host] 3 floats
 *   image        [device] [3][H][W] out
 *   final_T      [device] [H][W] out
 *   n_contrib    [device] [H][W] i32 out: blended Gaussians
 *   last         [device] [H][W] i32 out: 1 + list offset of the last blend
 *   hit_bits     [device] [n_instances rounded up to a multiple of 4] u8
 *                out, or NULL: one byte per sorted list entry (indexed as
 *                vals); bit f set when the entry blended at some pixel of the
 *                8x4 block f of its tile (block f at column (f & 1) * 8, row
 *                (f >> 1) * 4), clear otherwise. Every entry of every tile's
 *                list is written. The bits are OR-ed in with 32-bit atomics,
 *                so the pointer must be 4-byte aligned (else
 *                GS_ERR_INVALID_ARGUMENT). The backward's input of the same
 *                name.
 * Asynchronous. */
GS_API int gs_rasterize_fwd(const gs_projected* in, const uint32_t* vals,
                            const uint32_t* tile_ranges, const uint32_t* tile_order,
                            const gs_camera* cam, const float* bg,
                            float* image, float* final_T, int32_t* n_contrib, int32_t* last,
                            uint8_t* hit_bits, void* stream);

/* Importance pass: gs_rasterize_fwd plus the cross-view visibility weight
 * of every Gaussian (BlitzGS write-up, section 2.2 "模型层级重要性评分传递":
 * a weight per Gaussian for its total contribution over the views, used to
 * suppress the least important Gaussians and as the weights of the
 * view-level importance cull of gs_cull). The page prints no formula. It is
 * read as the sum over the view's pixels of the blend weight alpha * T of
 * each of the Gaussian's blends, with the forward's own fp32 values. The
 * image outputs equal gs_rasterize_fwd's bit for bit. tile_order and
 * hit_bits as for gs_rasterize_fwd.
 *   active_idx   [device] [n_records] i32 or NULL: Gaussian of record i
 *                (from gs_cull; NULL: record i is Gaussian i)
 *   importance   [device] [N] f32 in/out: this view's weights are ADDED, so
 *                zero it once and call once per view to sum over views
 * The sums are fp32 atomics in an unspecified order (a warp sum over an 8x8
 * pixel block, then one atomic per (Gaussian, block)). Asynchronous. */
GS_API int gs_rasterize_fwd_importance(const gs_projected* in, const uint32_t* vals,
                                       const uint32_t* tile_ranges, const uint32_t* tile_order,
                                       const gs_camera* cam, const float* bg,
                                       const int32_t* active_idx, float* image, float* final_T,
                                       int32_t* n_contrib, int32_t* last, float* importance,
                                       uint8_t* hit_bits, void* stream);

/* Backward pass: exact derivatives of the forward with every discrete decision
 * held fixed (visibility, tile lists, skips, the 0.99 clamp -- zero gradient
 * through a clamped alpha -- colour clamps, stop points).
 * Part 1 replays each pixel back to front and accumulates per-record 2-D
 * gradients into grad2d; part 2 chains them to the parameters.
 *   params, sh_degree, N, active_idx, n_active: as given to gs_preprocess
 *   mask         [device] [N] u8 from gs_cull or NULL (all active)
 *   in           records from gs_preprocess
 *   tile_order   as for gs_rasterize_fwd (any permutation, or NULL)
 *   hit_bits     [device] the forward's hit_bits for the same lists, or NULL.
 *                Given, each warp walks its own 8x8 block's entries and
 *                fetches only those that blended in one of its two 8x4
 *                halves, with no CTA-wide barrier; NULL, the kernel tests
 *                every entry's blend region itself. The results are the same either way
 *                up to the order of the fp32 atomic sums.
 *   final_T, last from gs_rasterize_fwd; dL_dimage [device] [3][H][W]
 *   grad2d       [device] [N][12] f32 out: (dpx, dpy, dopacity, 0,
 *                dA, dB, dC, 0, dr, dg, db, 0) per record
 *   d_*          [device] out, same layouts as the parameters; overwritten,
 *                zero for Gaussians that are culled or not visible
 * Asynchronous. */
GS_API int gs_rasterize_bwd(const float* means, const float* log_scales, const float* quats,
                            const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                            const int32_t* active_idx, const int32_t* n_active, const uint8_t* mask,
                            const gs_camera* cam, const gs_projected* in, const uint32_t* vals,
                            const uint32_t* tile_ranges, const uint32_t* tile_order,
                            const uint8_t* hit_bits, const float* bg,
                            const float* final_T, const int32_t* last, const float* dL_dimage,
                            float* grad2d, float* d_means, float* d_log_scales, float* d_quats,
                            float* d_opacity_logits, float* d_sh, void* stream);

/* Part 1 of gs_rasterize_bwd alone: the back-to-front replay that writes the
 * per-record 2-D gradients grad2d [device] [N][12] (zeroed first), without
 * chaining them to the parameters. Same arguments as the corresponding ones
 * of gs_rasterize_bwd; n_records = N. Asynchronous. */
GS_API int gs_rasterize_bwd_2d(const gs_projected* in, int64_t n_records, const uint32_t* vals,
                               const uint32_t* tile_ranges, const uint32_t* tile_order,
                               const uint8_t* hit_bits, const gs_camera* cam, const float* bg,
                               const float* final_T, const int32_t* last, const float* dL_dimage,
                               float* grad2d, void* stream);

/* Part 2 of gs_rasterize_bwd alone: parameter gradients from given per-record
 * 2-D gradients grad2d [device] [N][12] (input). Same outputs. Asynchronous. */
GS_API int gs_preprocess_bwd(const float* means, const float* log_scales, const float* quats,
                             const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                             const int32_t* active_idx, const int32_t* n_active,
                             const uint8_t* mask, const gs_camera* cam, const gs_projected* in,
                             const float* grad2d, float* d_means, float* d_log_scales,
                             float* d_quats, float* d_opacity_logits, float* d_sh, void* stream);

/* gs_preprocess_bwd that adds instead of overwriting: each visible record's
 * parameter gradient is added to its Gaussian's rows of d_* (read-modify-
 * write); rows of culled Gaussians and invisible records are not touched.
 * The gradient of a loss summed over several views is the sum of the views'
 * gradients, so a multi-view training step calls this once per view on
 * gradients it zeroed once (the problem statement's matching backward pass,
 * applied per view). Same arguments as gs_preprocess_bwd without the mask;
 * active_idx / n_active select the records as there. Calls that add into the
 * same rows must not overlap on the GPU (they would race); order them on one
 * stream. Asynchronous. */
GS_API int gs_preprocess_bwd_accumulate(const float* means, const float* log_scales, const float* quats,
                                        const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                        const int32_t* active_idx, const int32_t* n_active, const gs_camera* cam,
                                        const gs_projected* in, const float* grad2d, float* d_means,
                                        float* d_log_scales, float* d_quats, float* d_opacity_logits, float* d_sh,
                                        void* stream);

/* Backward of gs_preprocess_multiview: the parameter gradients of a loss
 * summed over several views of one model, from each view's per-record 2-D
 * gradients (gs_rasterize_bwd_2d), in one pass over the parameters. The
 * gradient of a sum over views is the sum of the views' gradients (the
 * problem statement's backward pass, applied per view); the pages print no
 * kernel for it. Record i of every view is Gaussian i, as
 * gs_preprocess_multiview writes them (no cull).
 *   params, sh_degree, N   as for gs_preprocess_multiview
 *   cams     [host] [n_views] the views' cameras
 *   n_views  1 .. GS_MAX_VIEWS
 *   ins      [host] [n_views] the views' records (capacity N each)
 *   grad2ds  [host] [n_views] pointers to each view's [device] [N][12] 2-D
 *            gradients
 *   d_*      [device] parameter-shaped gradients out: every row is written
 *            (zeros for a Gaussian that no view sees)
 * Per Gaussian the chain from the 3-D covariance to the log-scales and the
 * quaternion, and from the opacity to its logit, runs once on the summed
 * dL/dSigma and dL/dopacity (those chains are linear), so the result equals
 * the sum of gs_preprocess_bwd over the views up to fp32 rounding, not bit
 * for bit. HBM traffic: (11 + 3K) * 4 bytes read and written once, plus
 * 52 bytes per (Gaussian, view) of records and 2-D gradients. Asynchronous. */
GS_API int gs_preprocess_bwd_multiview(const float* means, const float* log_scales, const float* quats,
                                       const float* opacity_logits, const float* sh, int sh_degree, int64_t N,
                                       const gs_camera* cams, int n_views, const gs_projected* ins,
                                       const float* const* grad2ds, float* d_means, float* d_log_scales,
                                       float* d_quats, float* d_opacity_logits, float* d_sh, void* stream);

/* Number of kernels this library has launched in the process so far (all
 * devices, all streams). Host-side counter, for accounting in benchmarks. */
GS_API int64_t gs_debug_kernel_launches(void);

/* 1 in the checked build of the library (compiled with GS_CHECKED), else 0.
 * The checked build bounds-checks record and list gathers on the device: a
 * failed check records a code and skips the access instead of trapping. */
GS_API int gs_debug_is_checked_build(void);

/* The first failed device-side check since the last call (1: a list value or
 * active index past the record count, 2: a radix-sort scatter destination
 * past the key count, 3: a tile range that runs backwards), 0 if none,
 * 0xffffffff if the status could not be read; the status is cleared. Always
 * 0 in the unchecked build. Synchronous. */
GS_API uint32_t gs_debug_checked_status(void);

/* Fault-injection hook for tests of the bounded look-back wait: while set to
 * k >= 0, tile k of every radix-sort pass never publishes its counts, so its
 * successor's wait runs out and gs_bin_sort returns GS_ERR_DEVICE_TIMEOUT.
 * -1 (the default) disables it. Host-side state, not thread-safe. */
GS_API void gs_debug_set_stalled_sort_tile(int64_t tile);

#ifdef __cplusplus
}
#endif

#endif /* GS_H_ */
