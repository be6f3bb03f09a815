// Index-interleaved multi-GPU rendering with one exchange of projected
// records (BlitzGS write-up, section 2.1 "系统层级索引分割": Gaussians are
// dealt to GPUs by index, every GPU projects its own, and one exchange routes
// each projected Gaussian to the GPUs that own the screen tiles it touches).
//
// Rank r of G owns Gaussians g = r, r + G, r + 2G, ... (local record l is
// global Gaussian l G + r) and the tile rows [band(r), band(r + 1)) of a
// partition of the TH tile rows into G bands in rank order: by default
// band(q) = floor(q TH / G), or bounds the caller chose (for instance from
// the measured work per tile row). Kernels here, per rank:
//   route     which bands each visible local record reaches, and its slot in
//             the send buffer of each (records stay in local, hence global,
//             order within a destination);
//   pack      64-byte wire records (WireRecord): the record's xyzo, conic and
//             rgb vectors, its global index and radius in the two spare
//             lanes, and its rect;
//   merge     the G received segments, each ascending in global index, into
//             one record array in global order with rects clamped to the
//             own band (the bin sort is stable, so ties of equal depth then
//             resolve exactly as on one GPU);
//   return    2-D gradients of received records added back into the sender's
//             per-record gradients (a Gaussian reaching several bands gets
//             the sum of their contributions).
// The collective itself (counts, then one all-to-all of wire records, and
// the reverse one of gradients) is the caller's: NCCL through
// torch.distributed, or a copy when the ranks are emulated on one GPU.

#include "gs_device.cuh"
#include "gs_internal.cuh"

namespace gs {
namespace {

constexpr int kRouteBlock = 256;

// Mask of the bands that the rect rows [y0, y1) reach (bit q).
__device__ __forceinline__ uint32_t band_mask(int y0, int y1, int G, const BandStarts& b) {
  uint32_t m = 0;
  for (int q = 0; q < G; ++q)
    if (y0 < b.row[q + 1] && y1 > b.row[q]) m |= 1u << q;
  return m;
}

// Per record: its band mask; per CTA: the count of records for every band
// (cta_counts [n_ctas][G]).
__global__ void __launch_bounds__(kRouteBlock) route_count_kernel(const ushort4* rect, const int32_t* tiles,
                                                                  int64_t n, int G, BandStarts bands,
                                                                  uint32_t* mask, uint32_t* cta_counts) {
  __shared__ uint32_t s_cnt[kMaxRanks];
  if (threadIdx.x < kMaxRanks) s_cnt[threadIdx.x] = 0;
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * kRouteBlock + threadIdx.x;
  uint32_t m = 0;
  if (i < n && tiles[i] > 0) {
    const ushort4 r = rect[i];
    m = band_mask(r.y, r.w, G, bands);
  }
  if (i < n) mask[i] = m;
  for (int q = 0; q < G; ++q) {
    const uint32_t bal = __ballot_sync(0xffffffffu, (m >> q) & 1u);
    if ((threadIdx.x & 31) == 0 && bal) atomicAdd(&s_cnt[q], (uint32_t)__popc(bal));
  }
  __syncthreads();
  if (threadIdx.x < G) cta_counts[(int64_t)blockIdx.x * G + threadIdx.x] = s_cnt[threadIdx.x];
}

// Exclusive scan of cta_counts over CTAs for every band (one thread per
// band, sequential: G <= 32 bands and a few thousand CTAs), the totals, and
// (dst_off non-null) their exclusive scan: each destination's first slot in
// the send buffer, so the pack needs no host round trip.
__global__ void route_scan_kernel(uint32_t* cta_counts, int64_t n_ctas, int G, int64_t* totals,
                                  int64_t* dst_off) {
  const int q = threadIdx.x;
  int64_t run = 0;
  if (q < G) {
    for (int64_t c = 0; c < n_ctas; ++c) {
      const uint32_t v = cta_counts[c * G + q];
      cta_counts[c * G + q] = (uint32_t)run;
      run += v;
    }
    totals[q] = run;
  }
  if (dst_off) {
    int64_t x = q < G ? run : 0;  // inclusive warp scan of the totals
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (q >= o) x += y;
    }
    if (q < G) dst_off[q] = x - run;
  }
}

// Writes record i to slot dst_off[q] + (its rank among the records for band
// q) of the send buffer, for every band q in its mask; src_idx[slot] = i.
__global__ void __launch_bounds__(kRouteBlock) route_pack_kernel(Records rec, const uint32_t* mask, int64_t n,
                                                                 int G, int rank, const uint32_t* cta_offsets,
                                                                 const int64_t* dst_off, WireRecord* send,
                                                                 int32_t* src_idx) {
  __shared__ uint32_t s_warp[kRouteBlock / 32][kMaxRanks];
  const int64_t i = (int64_t)blockIdx.x * kRouteBlock + threadIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t m = i < n ? mask[i] : 0u;
  uint32_t below[kMaxRanks];
  for (int q = 0; q < G; ++q) {
    const uint32_t bal = __ballot_sync(0xffffffffu, (m >> q) & 1u);
    below[q] = (uint32_t)__popc(bal & ((1u << lane) - 1u));
    if (lane == 0) s_warp[warp][q] = (uint32_t)__popc(bal);
  }
  __syncthreads();
  if (!m) return;
  const float4 xyzo = rec.xyzo[i], conic = rec.conic[i], rgb = rec.rgb[i];
  const ushort4 r = rec.rect[i];
  for (int q = 0; q < G; ++q) {
    if (!((m >> q) & 1u)) continue;
    uint32_t before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w][q];
    const int64_t slot = dst_off[q] + cta_offsets[(int64_t)blockIdx.x * G + q] + before + below[q];
    WireRecord wr;
    wr.xyzo = xyzo;
    wr.conic = make_float4(conic.x, conic.y, conic.z, __int_as_float((int)(i * (int64_t)G + rank)));
    wr.rgb = make_float4(rgb.x, rgb.y, rgb.z, __int_as_float(rec.radius[i]));
    wr.rect = r;
    wr.pad = make_uint2(0u, 0u);
    send[slot] = wr;
    src_idx[slot] = (int32_t)i;
  }
}

__device__ __forceinline__ int32_t wire_gid(const WireRecord& w) { return __float_as_int(w.conic.w); }

// Merge of G segments (seg_off [G + 1] into recv), each ascending in global
// index, into global order; rects clamped to the band [y_lo, y_hi).
// perm[out] = position in recv of the record now at out.
__global__ void __launch_bounds__(256) merge_kernel(const WireRecord* recv, const int64_t* seg_off, int G,
                                                    int64_t n_recv, int y_lo, int y_hi, Records out,
                                                    int32_t* perm) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n_recv) return;
  int s = 0;
  while (k >= seg_off[s + 1]) ++s;
  const WireRecord w = recv[k];
  const int32_t gid = wire_gid(w);
  int64_t pos = k - seg_off[s];
  for (int t = 0; t < G; ++t) {
    if (t == s) continue;
    int64_t lo = seg_off[t], hi = seg_off[t + 1];  // first element with index > gid
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (wire_gid(recv[mid]) < gid) lo = mid + 1;
      else hi = mid;
    }
    pos += lo - seg_off[t];
  }
  const int y0 = max((int)w.rect.y, y_lo), y1 = min((int)w.rect.w, y_hi);
  out.xyzo[pos] = w.xyzo;
  out.conic[pos] = make_float4(w.conic.x, w.conic.y, w.conic.z, 0.0f);
  out.rgb[pos] = make_float4(w.rgb.x, w.rgb.y, w.rgb.z, 0.0f);
  out.radius[pos] = __float_as_int(w.rgb.w);
  out.rect[pos] = make_ushort4(w.rect.x, (unsigned short)y0, w.rect.z, (unsigned short)y1);
  out.tiles[pos] = ((int)w.rect.z - (int)w.rect.x) * (y1 - y0);
  perm[pos] = (int32_t)k;
}

// Gradients of the merged records back in receive order (for the reverse
// exchange): back[perm[i]] = grad2d[i].
__global__ void __launch_bounds__(256) unmerge_grad_kernel(const float4* grad2d, const int32_t* perm, int64_t n,
                                                           float4* back) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t k = perm[i];
  back[3 * k] = grad2d[3 * i];
  back[3 * k + 1] = grad2d[3 * i + 1];
  back[3 * k + 2] = grad2d[3 * i + 2];
}

// Returned gradients added into the sender's records: grad2d[src_idx[j]] +=
// ret[j] (a record sent to several bands receives several rows).
__global__ void __launch_bounds__(256) return_grad_kernel(const float4* ret, const int32_t* src_idx, int64_t n,
                                                          float4* grad2d) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  float4* dst = grad2d + 3 * (int64_t)src_idx[j];
  atomicAdd(dst, ret[3 * j]);
  atomicAdd(dst + 1, ret[3 * j + 1]);
  atomicAdd(dst + 2, ret[3 * j + 2]);
}

}  // namespace

int64_t route_ctas(int64_t n) { return (n + kRouteBlock - 1) / kRouteBlock; }

cudaError_t launch_route_count(const Records& rec, int64_t n, int G, const BandStarts& bands, uint32_t* mask,
                               uint32_t* cta_counts, int64_t* totals, int64_t* dst_off, cudaStream_t s) {
  const int64_t nc = route_ctas(n);
  if (nc > 0)
    route_count_kernel<<<(unsigned)nc, kRouteBlock, 0, s>>>(rec.rect, rec.tiles, n, G, bands, mask, cta_counts);
  route_scan_kernel<<<1, 32, 0, s>>>(cta_counts, nc, G, totals, dst_off);
  count_launches(nc > 0 ? 2 : 1);
  return cudaGetLastError();
}

cudaError_t launch_route_pack(const Records& rec, const uint32_t* mask, int64_t n, int G, int rank,
                              const uint32_t* cta_offsets, const int64_t* dst_off, WireRecord* send,
                              int32_t* src_idx, cudaStream_t s) {
  const int64_t nc = route_ctas(n);
  if (nc == 0) return cudaSuccess;
  route_pack_kernel<<<(unsigned)nc, kRouteBlock, 0, s>>>(rec, mask, n, G, rank, cta_offsets, dst_off, send, src_idx);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_merge(const WireRecord* recv, const int64_t* seg_off, int G, int64_t n_recv, int y_lo, int y_hi,
                         const Records& out, int32_t* perm, cudaStream_t s) {
  if (n_recv == 0) return cudaSuccess;
  merge_kernel<<<grid_for(n_recv, 256), 256, 0, s>>>(recv, seg_off, G, n_recv, y_lo, y_hi, out, perm);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_unmerge_grad(const float4* grad2d, const int32_t* perm, int64_t n, float4* back,
                                cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  unmerge_grad_kernel<<<grid_for(n, 256), 256, 0, s>>>(grad2d, perm, n, back);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_return_grad(const float4* ret, const int32_t* src_idx, int64_t n, float4* grad2d,
                               cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  return_grad_kernel<<<grid_for(n, 256), 256, 0, s>>>(ret, src_idx, n, grad2d);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace gs
