// Local permutation of (token, expert) pairs by expert -- the single-GPU
// stand-in for the dispatch step ("DeepSeek_V3_Report：Annotation",
// "Low-Precision Communication": tokens are quantised to FP8 first and the
// FP8 rows are what moves; "No Token-Dropping": no capacity limit).
//
// Deterministic and stable without atomics deciding any order:
//  1. count   -- per chunk of kChunkT tokens, a shared-memory histogram
//                (order-free integer adds) -> ws[chunk][E].
//  2. scan    -- one CTA: per expert a running sum over chunks (chunk bases),
//                then an exclusive scan over experts -> offsets, and the
//                128-row tile table of every segment.
//  3. scatter -- per chunk, four warps each walk a quarter of its tokens in
//                order, several tokens per step (lane = (token, k)), from
//                per-warp cursors (the chunk base plus the earlier quarters'
//                counts); lanes that picked the same expert are ranked with
//                __match_any_sync in lane order, which is token order, so
//                each expert's rows stay in ascending token order.
//  4. gather  -- one warp per destination row copies the FP8 row (16-byte
//                vectors, coalesced) and its 1x128 scales.
#include <mutex>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kChunkT = 128;
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(256) perm_count_kernel(const int32_t* __restrict__ idx, int T,
                                                         int K, int E, int32_t* __restrict__ ccount,
                                                         int32_t* dev_err) {
  extern __shared__ int32_t hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kChunkT;
  const int nt = min(kChunkT, T - t0);
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) {
    const int e = idx[static_cast<int64_t>(t0) * K + p];
    if (e < 0 || e >= E) {
      set_dev_err(dev_err, MOE_DEVERR_BAD_INDEX);
      continue;
    }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    ccount[static_cast<int64_t>(blockIdx.x) * E + e] = hist[e];
}

// Exclusive block scan of one int per thread (kScanThreads threads).
__device__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += n;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += n;
    }
    warp_sums[lane] = wi - w;  // exclusive prefix of the warp sums
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_sums[warp] + incl - v;
  __syncthreads();
  return r;
}

// Offsets and tile table from per-group row counts (one thread per group).
__device__ void write_tables(int cnt, int g, int groups, int32_t* offsets, int32_t* tile_group,
                             int32_t* tile_start, int32_t* n_tiles, int max_tiles,
                             int32_t* dev_err, int* smem) {
  int* warp_sums = smem;
  int* totals = smem + 32;
  const bool in = g < groups;
  const int off = block_excl_scan(in ? cnt : 0, warp_sums, &totals[0]);
  const int mt = in ? (cnt + 127) / 128 : 0;
  const int mstart = block_excl_scan(mt, warp_sums, &totals[1]);
  const int total_rows = totals[0];
  const int total_tiles = totals[1];
  const bool fits = total_tiles <= max_tiles;
  if (in) {
    offsets[g] = off;
    tile_start[g] = mstart;
    if (fits)
      for (int j = 0; j < mt; ++j) tile_group[mstart + j] = g;
  }
  if (threadIdx.x == 0) {
    offsets[groups] = total_rows;
    tile_start[groups] = total_tiles;
    *n_tiles = fits ? total_tiles : 0;
    if (!fits) set_dev_err(dev_err, MOE_DEVERR_BAD_TABLE);
  }
}

__global__ void __launch_bounds__(kScanThreads) perm_scan_kernel(
    int32_t* __restrict__ ccount, int n_chunks, int E, int T, int with_shared,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ tile_group,
    int32_t* __restrict__ tile_start, int32_t* __restrict__ n_tiles, int max_tiles,
    int32_t* dev_err) {
  __shared__ int smem[40];
  __shared__ int eoff[kScanThreads];
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    // running sum over chunks; loads batched so they overlap
    int c = 0;
    for (; c + 8 <= n_chunks; c += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = ccount[static_cast<int64_t>(c + j) * E + e];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ccount[static_cast<int64_t>(c + j) * E + e] = run;
        run += v[j];
      }
    }
    for (; c < n_chunks; ++c) {
      const int v = ccount[static_cast<int64_t>(c) * E + e];
      ccount[static_cast<int64_t>(c) * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  const int groups = E + (with_shared ? 1 : 0);
  const int cnt = (e < E) ? run : ((with_shared && e == E) ? T : 0);
  write_tables(cnt, e, groups, offsets, tile_group, tile_start, n_tiles, max_tiles, dev_err, smem);
  __syncthreads();
  if (e < E) eoff[e] = offsets[e];
  __syncthreads();
  // chunk bases become absolute row positions
  if (e < E) {
    const int base = eoff[e];
    for (int c = 0; c < n_chunks; ++c) ccount[static_cast<int64_t>(c) * E + e] += base;
  }
}

// One CTA per chunk, kScatterWarps warps: warp j places the pairs of tokens
// [j*kChunkT/kScatterWarps, ...) of the chunk.  Each warp's starting cursor
// per expert is the chunk base plus the pairs of that expert in the earlier
// warps' tokens (counted first), so the result is the one a single warp
// walking the whole chunk would produce.
constexpr int kScatterWarps = 4;
constexpr int kTokPerWarp = kChunkT / kScatterWarps;

__global__ void __launch_bounds__(32 * kScatterWarps) perm_scatter_kernel(
    const int32_t* __restrict__ idx, int T, int K, int E, const int32_t* __restrict__ cbase,
    int32_t* __restrict__ src_row, int32_t* __restrict__ dst_of) {
  extern __shared__ int32_t sm[];
  int32_t* cursor = sm;                       // [kScatterWarps][E]
  int32_t* hist = sm + kScatterWarps * E;     // [kScatterWarps][E]
  int32_t* sidx = sm + 2 * kScatterWarps * E; // [kChunkT * K]
  const int lane = threadIdx.x & 31, wj = threadIdx.x >> 5;
  const int t0 = blockIdx.x * kChunkT;
  const int nt = min(kChunkT, T - t0);
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) hist[i] = 0;
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) sidx[p] = idx[static_cast<int64_t>(t0) * K + p];
  __syncthreads();
  // pairs per expert in each warp's tokens (integer adds: order-free)
  const int wt0 = wj * kTokPerWarp, wt1 = min(nt, wt0 + kTokPerWarp);
  for (int p = wt0 * K + lane; p < wt1 * K; p += 32) {
    const int e = sidx[p];
    if (e >= 0 && e < E) atomicAdd(&hist[wj * E + e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = cbase[static_cast<int64_t>(blockIdx.x) * E + e];
    for (int j = 0; j < kScatterWarps; ++j) {
      cursor[j * E + e] = run;
      run += hist[j * E + e];
    }
  }
  __syncthreads();
  int32_t* cur = cursor + wj * E;
  const int tpi = 32 / K;  // tokens per step
  const int tl = lane / K, k = lane - (lane / K) * K;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int tb = wt0; tb < wt1; tb += tpi) {
    const int tt = tb + tl;
    int e = -1;
    if (tl < tpi && tt < wt1) e = sidx[tt * K + k];
    const bool active = e >= 0 && e < E;
    const unsigned amask = __ballot_sync(0xffffffffu, active);
    unsigned peers = 0;
    int pos = 0;
    if (active) {
      peers = __match_any_sync(amask, e);
      pos = cur[e] + __popc(peers & lt_mask);
    }
    __syncwarp();
    if (active && lane == __ffs(peers) - 1) cur[e] += __popc(peers);
    __syncwarp();
    if (active) {
      const int t = t0 + tt;
      src_row[pos] = t;
      dst_of[static_cast<int64_t>(t) * K + k] = pos;
    } else if (tl < tpi && tt < wt1) {
      dst_of[static_cast<int64_t>(t0 + tt) * K + k] = -1;  // flagged bad index: no row
    }
  }
}

// Scan and scatter fused: one CTA per chunk.  Every CTA sums the per-chunk
// counts itself -- the chunks before its own (its bases) and all of them
// (the expert totals) -- and scans the totals over the experts, so no
// separate single-CTA scan kernel runs between the count and the scatter.
// CTA 0 also writes counts, offsets and the tile table.  Warps 0..3 then
// place the chunk's pairs exactly as perm_scatter_kernel does.
__global__ void __launch_bounds__(kScanThreads) perm_scan_scatter_kernel(
    const int32_t* __restrict__ idx, int T, int K, int E, int with_shared,
    const int32_t* __restrict__ ccount, int n_chunks, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ tile_group,
    int32_t* __restrict__ tile_start, int32_t* __restrict__ n_tiles, int max_tiles,
    int32_t* __restrict__ src_row, int32_t* __restrict__ dst_of, int32_t* dev_err) {
  extern __shared__ int32_t sm[];
  __shared__ int scan_smem[40];
  int32_t* cursor = sm;                        // [kScatterWarps][E]
  int32_t* hist = sm + kScatterWarps * E;      // [kScatterWarps][E]
  int32_t* sidx = sm + 2 * kScatterWarps * E;  // [kChunkT * K]
  int32_t* cbase = sidx + kChunkT * K;         // [E]
  const int e = threadIdx.x;
  const int my = blockIdx.x;
  int before = 0, total = 0;
  if (e < E) {
    int c = 0;
    for (; c + 8 <= n_chunks; c += 8) {  // eight loads in flight
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = __ldg(ccount + static_cast<int64_t>(c + j) * E + e);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        before += (c + j < my) ? v[j] : 0;
        total += v[j];
      }
    }
    for (; c < n_chunks; ++c) {
      const int v = __ldg(ccount + static_cast<int64_t>(c) * E + e);
      before += (c < my) ? v : 0;
      total += v;
    }
  }
  int* warp_sums = scan_smem;
  const int off = block_excl_scan(e < E ? total : 0, warp_sums, &scan_smem[32]);
  if (e < E) cbase[e] = off + before;
  if (my == 0) {
    if (e < E) counts[e] = total;
    const int groups = E + (with_shared ? 1 : 0);
    const int cnt = (e < E) ? total : ((with_shared && e == E) ? T : 0);
    write_tables(cnt, e, groups, offsets, tile_group, tile_start, n_tiles, max_tiles, dev_err,
                 scan_smem);
  }
  const int lane = threadIdx.x & 31, wj = threadIdx.x >> 5;
  const int t0 = my * kChunkT;
  const int nt = min(kChunkT, T - t0);
  for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) hist[i] = 0;
  for (int p = threadIdx.x; p < nt * K; p += blockDim.x) sidx[p] = idx[static_cast<int64_t>(t0) * K + p];
  __syncthreads();
  const int wt0 = wj * kTokPerWarp, wt1 = min(nt, wt0 + kTokPerWarp);
  if (wj < kScatterWarps)
    for (int p = wt0 * K + lane; p < wt1 * K; p += 32) {
      const int ex = sidx[p];
      if (ex >= 0 && ex < E) atomicAdd(&hist[wj * E + ex], 1);
    }
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = cbase[x];
    for (int j = 0; j < kScatterWarps; ++j) {
      cursor[j * E + x] = run;
      run += hist[j * E + x];
    }
  }
  __syncthreads();
  if (wj >= kScatterWarps) return;
  int32_t* cur = cursor + wj * E;
  const int tpi = 32 / K;  // tokens per step
  const int tl = lane / K, k = lane - (lane / K) * K;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int tb = wt0; tb < wt1; tb += tpi) {
    const int tt = tb + tl;
    int ex = -1;
    if (tl < tpi && tt < wt1) ex = sidx[tt * K + k];
    const bool active = ex >= 0 && ex < E;
    const unsigned amask = __ballot_sync(0xffffffffu, active);
    unsigned peers = 0;
    int pos = 0;
    if (active) {
      peers = __match_any_sync(amask, ex);
      pos = cur[ex] + __popc(peers & lt_mask);
    }
    __syncwarp();
    if (active && lane == __ffs(peers) - 1) cur[ex] += __popc(peers);
    __syncwarp();
    if (active) {
      const int t = t0 + tt;
      src_row[pos] = t;
      dst_of[static_cast<int64_t>(t) * K + k] = pos;
    } else if (tl < tpi && tt < wt1) {
      dst_of[static_cast<int64_t>(t0 + tt) * K + k] = -1;  // flagged bad index: no row
    }
  }
}

size_t scan_scatter_smem(int E, int K) {
  return (2 * kScatterWarps * static_cast<size_t>(E) + kChunkT * K + E) * sizeof(int32_t);
}

// One warp per destination row: d bytes of FP8 plus d/128 fp32 scales.
__global__ void __launch_bounds__(256) perm_gather_kernel(
    const int32_t* __restrict__ src_row, int rows, int T, const uint8_t* __restrict__ xq,
    const float* __restrict__ xs, int d, uint8_t* __restrict__ xq_perm,
    float* __restrict__ xs_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int64_t s = src_row[r];
  // rows left unassigned after a flagged bad expert index hold no token
  if (s < 0 || s >= T) return;
  const uint4* src = reinterpret_cast<const uint4*>(xq + s * d);
  uint4* dst = reinterpret_cast<uint4*>(xq_perm + r * d);
  const int nv = d / 16;
  for (int v = lane; v < nv; v += 32) dst[v] = __ldg(src + v);
  const int ns = d / 128;
  for (int v = lane; v < ns; v += 32) xs_perm[r * ns + v] = __ldg(xs + s * ns + v);
}

__global__ void __launch_bounds__(kScanThreads) tile_table_kernel(
    const int32_t* __restrict__ offsets, int groups, int max_tiles, int32_t* __restrict__ tile_group,
    int32_t* __restrict__ tile_start, int32_t* __restrict__ n_tiles, int32_t* dev_err) {
  __shared__ int smem[40];
  __shared__ int32_t offs_copy[kScanThreads + 1];
  const int g = threadIdx.x;
  int cnt = 0;
  if (g < groups) {
    cnt = offsets[g + 1] - offsets[g];
    if (cnt < 0 || offsets[g] < 0) {
      set_dev_err(dev_err, MOE_DEVERR_BAD_TABLE);
      cnt = 0;
    }
  }
  // the caller's offsets are kept; only the tile table is written
  write_tables(cnt, g, groups, offs_copy, tile_group, tile_start, n_tiles, max_tiles, dev_err,
               smem);
}

// Segment ids of a source-major receive buffer (expert parallelism): the
// rows of segment s = counts[s] come after those of segments 0..s-1, and
// every row of segment s gets id s % E (its local expert).  Each CTA scans
// the <= 1024 counts itself, then labels its 4096 rows by binary search.
constexpr int kSegRowsPerCta = 4096;

__global__ void __launch_bounds__(kScanThreads) segment_ids_kernel(
    const int32_t* __restrict__ counts, int nseg, int E, int64_t lead, int64_t n_rows,
    int32_t* __restrict__ ids, int32_t* dev_err) {
  __shared__ int64_t incl[kScanThreads];
  const int t = threadIdx.x;
  int64_t c = t < nseg ? __ldg(counts + t) : 0;
  if (c < 0) {
    set_dev_err(dev_err, MOE_DEVERR_BAD_TABLE);
    c = 0;
  }
  incl[t] = c;
  __syncthreads();
  // inclusive scan over the segments actually present (log2 of their count
  // rounded up steps)
  for (int d = 1; d < nseg; d <<= 1) {
    const int64_t v = t >= d ? incl[t - d] : 0;
    __syncthreads();
    incl[t] += v;
    __syncthreads();
  }
  if (t == 0 && incl[nseg - 1] + lead != n_rows) set_dev_err(dev_err, MOE_DEVERR_BAD_TABLE);
  const int shift = lead > 0 ? 1 : 0;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kSegRowsPerCta;
  for (int64_t r = r0 + t; r < n_rows && r < r0 + kSegRowsPerCta; r += kScanThreads) {
    if (r < lead) {
      ids[r] = 0;
      continue;
    }
    const int64_t rr = r - lead;
    // first segment whose inclusive end exceeds rr
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (incl[mid] > rr) hi = mid;
      else lo = mid + 1;
    }
    ids[r] = shift + lo % E;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int n_chunks_of(int T) { return (T + kChunkT - 1) / kChunkT; }

}  // namespace
}  // namespace moe

extern "C" int moe_max_m_tiles(int T, int K, int E, int with_shared) {
  if (T < 0 || K < 0 || E < 0) return 0;
  const int64_t pairs = static_cast<int64_t>(T) * K;
  int64_t n = (pairs + static_cast<int64_t>(E) * 127) / 128;  // sum of ceil(c_e/128)
  if (with_shared) n += (T + 127) / 128;
  return static_cast<int>(n);
}

extern "C" moe_status moe_permute_workspace_size(int T, int K, int E, size_t* bytes) {
  if (!bytes || T < 0 || K <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  const size_t b = static_cast<size_t>(moe::n_chunks_of(T)) * E * sizeof(int32_t);
  *bytes = (b + 255) / 256 * 256;
  return MOE_OK;
}

namespace {

// Count, then the fused scan + scatter: counts, offsets, the tile table,
// src_row and dst_of (no row moves).  Arguments already validated.
moe_status permute_index_launch(const int32_t* topk_idx, int T, int K, int E, int with_shared,
                                int32_t* counts, int32_t* offsets, int32_t* src_row,
                                int32_t* dst_of, int32_t* tile_group, int32_t* tile_start,
                                int32_t* n_tiles, void* ws, int32_t* dev_err, cudaStream_t st) {
  using namespace moe;
  const int nch = n_chunks_of(T);
  int32_t* ccount = static_cast<int32_t*>(ws);
  const int max_tiles = moe_max_m_tiles(T, K, E, with_shared);
  if (nch == 0) {
    perm_scan_kernel<<<1, kScanThreads, 0, st>>>(ccount, nch, E, T, with_shared, counts, offsets,
                                                 tile_group, tile_start, n_tiles, max_tiles,
                                                 dev_err);
    MOE_CUDA_CHECK_LAUNCH();
    return MOE_OK;
  }
  perm_count_kernel<<<nch, 256, E * sizeof(int32_t), st>>>(topk_idx, T, K, E, ccount, dev_err);
  MOE_CUDA_CHECK_LAUNCH();
  const size_t sm = scan_scatter_smem(E, K);
  if (sm > 48 * 1024 &&
      cudaFuncSetAttribute(perm_scan_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(sm)) != cudaSuccess)
    return MOE_ERR_CUDA;
  perm_scan_scatter_kernel<<<nch, kScanThreads, sm, st>>>(
      topk_idx, T, K, E, with_shared, ccount, nch, counts, offsets, tile_group, tile_start,
      n_tiles, max_tiles, src_row, dst_of, dev_err);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

moe_status permute_index_check(const int32_t* topk_idx, int T, int K, int E, int32_t* counts,
                               int32_t* offsets, int32_t* src_row, int32_t* dst_of,
                               int32_t* tile_group, int32_t* tile_start, int32_t* n_tiles,
                               void* ws, size_t ws_bytes) {
  using namespace moe;
  if (T < 0 || K <= 0 || E <= 0) return MOE_ERR_INVALID_ARG;
  if (K > 32 || K > E) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets || !tile_start || !n_tiles || !tile_group) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !src_row || !dst_of)) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  moe_permute_workspace_size(T, K, E, &need);
  if (ws_bytes < need || (!ws && need)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute(const int32_t* topk_idx, int T, int K, int E, int with_shared,
                                  const uint8_t* xq, const float* xscale, int d, int32_t* counts,
                                  int32_t* offsets, int32_t* src_row, int32_t* dst_of,
                                  uint8_t* xq_perm, float* xscale_perm, int32_t* tile_group,
                                  int32_t* tile_start, int32_t* n_tiles, void* ws,
                                  size_t ws_bytes, int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (T < 0 || K <= 0 || E <= 0 || d <= 0) return MOE_ERR_INVALID_ARG;
  if (d % 128 != 0) return MOE_ERR_SHAPE;
  if (E + (with_shared ? 1 : 0) > kScanThreads) return MOE_ERR_UNSUPPORTED;
  moe_status r = permute_index_check(topk_idx, T, K, E, counts, offsets, src_row, dst_of,
                                     tile_group, tile_start, n_tiles, ws, ws_bytes);
  if (r != MOE_OK) return r;
  if (T > 0 && (!xq || !xscale || !xq_perm || !xscale_perm)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(xq_perm)) return MOE_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  r = permute_index_launch(topk_idx, T, K, E, with_shared, counts, offsets, src_row, dst_of,
                           tile_group, tile_start, n_tiles, ws, dev_err, st);
  if (r != MOE_OK || T == 0) return r;
  const int rows = T * K;
  perm_gather_kernel<<<(rows + 7) / 8, 256, 0, st>>>(src_row, rows, T, xq, xscale, d, xq_perm,
                                                     xscale_perm);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status moe_permute_index(const int32_t* topk_idx, int T, int K, int E,
                                        int with_shared, int32_t* counts, int32_t* offsets,
                                        int32_t* src_row, int32_t* dst_of, int32_t* tile_group,
                                        int32_t* tile_start, int32_t* n_tiles, void* ws,
                                        size_t ws_bytes, int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (E + (with_shared ? 1 : 0) > kScanThreads) return MOE_ERR_UNSUPPORTED;
  const moe_status r = permute_index_check(topk_idx, T, K, E, counts, offsets, src_row, dst_of,
                                           tile_group, tile_start, n_tiles, ws, ws_bytes);
  if (r != MOE_OK) return r;
  return permute_index_launch(topk_idx, T, K, E, with_shared, counts, offsets, src_row, dst_of,
                              tile_group, tile_start, n_tiles, ws, dev_err,
                              static_cast<cudaStream_t>(stream));
}

extern "C" moe_status moe_segment_ids(const int32_t* counts, int n_segments, int E,
                                      int64_t lead_rows, int64_t n_rows, int32_t* ids,
                                      int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (n_segments <= 0 || E <= 0 || n_rows < 0 || lead_rows < 0 || lead_rows > n_rows)
    return MOE_ERR_INVALID_ARG;
  if (n_segments % E != 0) return MOE_ERR_SHAPE;
  if (n_segments > kScanThreads) return MOE_ERR_UNSUPPORTED;
  if (n_rows == 0) return MOE_OK;
  if (!counts || !ids) return MOE_ERR_INVALID_ARG;
  const int64_t ctas = (n_rows + kSegRowsPerCta - 1) / kSegRowsPerCta;
  if (ctas > 0x7FFFFFFF) return MOE_ERR_UNSUPPORTED;
  segment_ids_kernel<<<static_cast<unsigned>(ctas), kScanThreads, 0,
                       static_cast<cudaStream_t>(stream)>>>(counts, n_segments, E, lead_rows,
                                                             n_rows, ids, dev_err);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

extern "C" moe_status moe_tile_table(const int32_t* offsets, int groups, int max_tiles,
                                     int32_t* tile_group, int32_t* tile_start, int32_t* n_tiles,
                                     int32_t* dev_err, moe_stream_t stream) {
  using namespace moe;
  if (groups <= 0 || max_tiles < 0 || !offsets || !tile_group || !tile_start || !n_tiles)
    return MOE_ERR_INVALID_ARG;
  if (groups > kScanThreads) return MOE_ERR_UNSUPPORTED;
  tile_table_kernel<<<1, kScanThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      offsets, groups, max_tiles, tile_group, tile_start, n_tiles, dev_err);
  MOE_CUDA_CHECK_LAUNCH();
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: moe_permute for callers that cannot allocate device
// memory at call time.  Inference-runtime plugins whose host framework owns
// and plans all device memory (and offers the plugin no workspace), and
// latency-critical paths that must not hit cudaMalloc's implicit device-wide
// synchronisation, can still run the permutation: its scratch (per-chunk
// expert counts) lives in a fixed file-scope device array instead of a
// caller buffer.
//
// The array is kNoAllocScratchInts int32 (1 MiB) and exists on every device
// that loads the library, for as long as the library stays loaded.  Every
// call shares it and it keeps the last call's contents; nothing in it needs
// clearing, because the count kernel overwrites every entry the later kernels
// read.  Calls that overlap on the GPU (two streams, or two host threads)
// race on the array and must be serialised by the caller.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchInts = size_t(1) << 18;
static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// Device address of the array for the current device; looked up once per
// device (host code may not use the symbol's name as a device pointer).
void* scratch_for_current_device(moe_status* st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    *st = MOE_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || !p) {
      *st = MOE_ERR_CUDA;
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  *st = MOE_OK;
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const int32_t* topk_idx, int T, int K, int E,
                                          int with_shared, const uint8_t* xq,
                                          const float* xscale, int d, int32_t* counts,
                                          int32_t* offsets, int32_t* src_row, int32_t* dst_of,
                                          uint8_t* xq_perm, float* xscale_perm,
                                          int32_t* tile_group, int32_t* tile_start,
                                          int32_t* n_tiles, int32_t* dev_err,
                                          moe_stream_t stream) {
  size_t need = 0;
  const moe_status q = moe_permute_workspace_size(T, K, E, &need);
  if (q != MOE_OK) return q;
  if (need > kNoAllocScratchInts * sizeof(int32_t)) return MOE_ERR_UNSUPPORTED;
  moe_status st = MOE_OK;
  void* ws = scratch_for_current_device(&st);
  if (st != MOE_OK) return st;
  return moe_permute(topk_idx, T, K, E, with_shared, xq, xscale, d, counts, offsets, src_row,
                     dst_of, xq_perm, xscale_perm, tile_group, tile_start, n_tiles, ws,
                     kNoAllocScratchInts * sizeof(int32_t), dev_err, stream);
}
