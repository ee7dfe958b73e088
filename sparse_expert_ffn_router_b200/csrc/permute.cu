// Scatter stage: per-expert histogram, prefix sum and the stable permutation that groups
// token rows by expert (www.trdm.cn/news/555962 §6.2: batch together the tokens that activate
// the same expert; www.pptc.cn/news/100465 §3.3: expert offsets as a running sum;
// www.hotelren.com/news/4731937 §2.3 dispatch_kernel).
//
// Row order inside an expert is ascending token index.  It is made deterministic without
// relying on atomic ordering:
//   route_count    one CTA per 256 tokens; each warp builds, per expert, the bit mask of its
//                  32 lanes (tokens) that chose that expert; a token's rank among the earlier
//                  tokens of its warp is popc(mask & lanes_below); warps are then prefixed in
//                  order, giving the rank inside the 256-token block and the block's counts.
//   route_scan     one CTA: per expert, exclusive prefix over blocks; counts; offsets[E+1]
//                  and the m-tile prefix the grouped GEMM schedules from (scans over experts).
//   route_scatter  one warp per token: final row = offsets[e] + block base + rank; writes
//                  src_row / dst_row and copies the token's row into each of its k grouped
//                  rows with 16-byte vector loads and stores.
// For int8 expert weights the copy is replaced by the token row's two int8 planes (and its
// scale), which is what the int8 expert kernels read; the bf16 grouped copy is then skipped.
#include "common.cuh"

namespace colibri {
namespace {

// Largest magnitude of the 8 bf16 values of one 16-byte vector.
__device__ __forceinline__ float vec_maxabs(const uint4& q) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f2 = __bfloat1622float2(h[i]);
    mx = fmaxf(mx, fmaxf(fabsf(f2.x), fabsf(f2.y)));
  }
  return mx;
}

// The int8 planes of the 8 bf16 values of one vector (row scale a), stored as vector v of each
// of the k grouped rows.
__device__ __forceinline__ void vec_planes_to_rows(const uint4& q, float a, float inv_a, int v, size_t d,
                                                   const int (&rows)[kMaxTopK], int k, const RowPlanes& P) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
  uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f2 = __bfloat1622float2(h[i]);
    int qh0, ql0, qh1, ql1;
    split_planes(f2.x, a, inv_a, qh0, ql0);
    split_planes(f2.y, a, inv_a, qh1, ql1);
    hw[i >> 1] |= (((uint32_t)qh0 & 0xffu) | (((uint32_t)qh1 & 0xffu) << 8)) << (16 * (i & 1));
    lw[i >> 1] |= (((uint32_t)ql0 & 0xffu) | (((uint32_t)ql1 & 0xffu) << 8)) << (16 * (i & 1));
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k) {
      reinterpret_cast<uint2*>(P.hi + (size_t)rows[j] * d)[v] = make_uint2(hw[0], hw[1]);
      reinterpret_cast<uint2*>(P.lo + (size_t)rows[j] * d)[v] = make_uint2(lw[0], lw[1]);
    }
  }
}

// One warp: the bf16 token row `src` (vec 16-byte vectors) split into int8 planes with the
// row's scale a = max|x| / 127, written to each of its k grouped rows.
__device__ __forceinline__ void warp_row_planes(const uint4* __restrict__ src, int vec, const int (&rows)[kMaxTopK],
                                                int k, const RowPlanes& P, int lane) {
  float mx = 0.f;
#pragma unroll 4
  for (int v = lane; v < vec; v += 32) mx = fmaxf(mx, vec_maxabs(__ldg(src + v)));
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const float a = plane_scale(mx), inv_a = __frcp_rn(a);  // correctly rounded 1 / a
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) P.scale[rows[j]] = a;
  }
  const size_t d = (size_t)vec * 8;
#pragma unroll 4
  for (int v = lane; v < vec; v += 32) vec_planes_to_rows(__ldg(src + v), a, inv_a, v, d, rows, k, P);
}

__global__ void __launch_bounds__(kCountBlock) route_count_kernel(const int32_t* __restrict__ idx,
                                                                  int T, int k, int E,
                                                                  int32_t* __restrict__ blk_counts,
                                                                  int32_t* __restrict__ local_rank) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t masks[];  // [warps][E]
  constexpr int W = kCountBlock / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kCountBlock + threadIdx.x;
  uint32_t* m = masks + warp * E;
  for (int e = lane; e < E; e += 32) m[e] = 0u;
  __syncwarp();
  int ids[kMaxTopK];
  int rank[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    ids[j] = 0;
    rank[j] = 0;
    if (j < k && t < T) {
      int e = idx[(size_t)t * k + j];
      e = min(max(e, 0), E - 1);
      ids[j] = e;
      atomicOr(&m[e], 1u << lane);
    }
  }
  __syncwarp();
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k && t < T) rank[j] = __popc(m[ids[j]] & below);
  __syncthreads();
  // per expert: exclusive prefix over the warps of this block (masks become bases)
  for (int e = threadIdx.x; e < E; e += kCountBlock) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int c = __popc(masks[w * E + e]);
      masks[w * E + e] = (uint32_t)run;
      run += c;
    }
    blk_counts[(size_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k && t < T) local_rank[(size_t)t * k + j] = (int)m[ids[j]] + rank[j];
}

__global__ void __launch_bounds__(256) route_scan_kernel(const int32_t* __restrict__ blk_counts,
                                                         int nblk, int E, int bm,
                                                         int32_t* __restrict__ blk_base,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ mt_prefix) {
  pdl_trigger();
  pdl_wait();
  __shared__ int wsum[2][8];
  const int e = threadIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // per expert: exclusive prefix over the blocks, eight block counts in flight at a time
  int run = 0;
  if (e < E) {
    int b = 0;
    for (; b + 8 <= nblk; b += 8) {
      int c[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = blk_counts[(size_t)(b + i) * E + e];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        blk_base[(size_t)(b + i) * E + e] = run;
        run += c[i];
      }
    }
    for (; b < nblk; ++b) {
      const int c = blk_counts[(size_t)b * E + e];
      blk_base[(size_t)b * E + e] = run;
      run += c;
    }
    counts[e] = run;
  }
  // offsets[] and the m-tile prefix: exclusive scans over the experts (warp scans, then warps)
  const int mt = (run + bm - 1) / bm;
  int io = run, im = mt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, io, o), c = __shfl_up_sync(0xffffffffu, im, o);
    if (lane >= o) {
      io += a;
      im += c;
    }
  }
  if (lane == 31) {
    wsum[0][warp] = io;
    wsum[1][warp] = im;
  }
  __syncthreads();
  int bo = 0, bmt = 0;
  for (int w = 0; w < warp; ++w) {
    bo += wsum[0][w];
    bmt += wsum[1][w];
  }
  if (e < E) {
    offsets[e] = bo + io - run;
    mt_prefix[e] = bmt + im - mt;
  }
  if (e == E - 1) {
    offsets[E] = bo + io;
    mt_prefix[E] = bmt + im;
  }
}

template <typename Tv>
__global__ void __launch_bounds__(256) route_scatter_kernel(
    const Tv* __restrict__ x, int T, int vec_per_row, int k, int E, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ blk_base, const int32_t* __restrict__ offsets, int32_t* __restrict__ dst_row,
    int32_t* __restrict__ src_row, Tv* __restrict__ Xp, RowPlanes P) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
    int r = 0;
    if (lane < k) {
      int e = idx[(size_t)t * k + lane];
      e = min(max(e, 0), E - 1);
      r = offsets[e] + blk_base[(size_t)(t / kCountBlock) * E + e] + dst_row[(size_t)t * k + lane];
      dst_row[(size_t)t * k + lane] = r;
      src_row[r] = t;
    }
    int rows[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, r, j);
    const Tv* src = x + (size_t)t * vec_per_row;
    if (P.hi) {
      warp_row_planes(src, vec_per_row, rows, k, P, lane);
      continue;
    }
    // four 16-byte loads in flight per lane before their k stores each
    int v = lane;
    for (; v + 96 < vec_per_row; v += 128) {
      Tv val[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) val[u] = __ldg(src + v + 32 * u);
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
#pragma unroll
          for (int u = 0; u < 4; ++u) Xp[(size_t)rows[j] * vec_per_row + v + 32 * u] = val[u];
        }
      }
    }
    for (; v < vec_per_row; v += 32) {
      const Tv val = __ldg(src + v);
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) Xp[(size_t)rows[j] * vec_per_row + v] = val;
    }
  }
}

// Small batches (T <= 64): histogram, prefix sum and scatter in one single-CTA launch.  Same
// rank rule as the three-kernel path: a token's rank inside its expert is the number of
// earlier tokens (warp masks, then a prefix over warps) that chose that expert.
template <typename Tv>
__global__ void __launch_bounds__(kFusedRouteThreads) route_fused_kernel(
    const Tv* __restrict__ x, int T, int vec_per_row, const int32_t* __restrict__ idx, int k, int E, int bm,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ mt_prefix,
    int32_t* __restrict__ src_row, int32_t* __restrict__ dst_row, Tv* __restrict__ Xp, RowPlanes P) {
  pdl_trigger();
  pdl_wait();
  constexpr int W = kFusedRouteThreads / 32;
  __shared__ uint32_t masks[W][kMaxExperts];
  __shared__ int off_s[kMaxExperts + 1];
  __shared__ int rows_s[kFusedRouteMaxT][kMaxTopK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, t = threadIdx.x;
  for (int e = lane; e < E; e += 32) masks[warp][e] = 0u;
  __syncwarp();
  int ids[kMaxTopK], rank[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    ids[j] = 0;
    rank[j] = 0;
    if (j < k && t < T) {
      ids[j] = min(max(idx[(size_t)t * k + j], 0), E - 1);
      atomicOr(&masks[warp][ids[j]], 1u << lane);
    }
  }
  __syncwarp();
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k && t < T) rank[j] = __popc(masks[warp][ids[j]] & below);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kFusedRouteThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const int c = __popc(masks[w][e]);
      masks[w][e] = (uint32_t)run;
      run += c;
    }
    off_s[e] = run;  // total for now
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int o = 0, mt = 0;
    for (int q = 0; q < E; ++q) {
      const int c = off_s[q];
      counts[q] = c;
      offsets[q] = o;
      mt_prefix[q] = mt;
      off_s[q] = o;
      o += c;
      mt += (c + bm - 1) / bm;
    }
    off_s[E] = o;
    offsets[E] = o;
    mt_prefix[E] = mt;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k && t < T) {
      const int r = off_s[ids[j]] + (int)masks[warp][ids[j]] + rank[j];
      dst_row[(size_t)t * k + j] = r;
      src_row[r] = t;
      rows_s[t][j] = r;
    }
  }
  __syncthreads();
  if (P.hi) {
    // int8 planes: G warps per token, G the largest power of two with G * T <= 32 warps, so a
    // handful of tokens still spreads its row over the whole CTA (one or two loads per thread)
    int G = 1;
    while (G * 2 * T <= W) G *= 2;
    const int groups = W / G, grp = warp / G;
    const int gt = (warp % G) * 32 + lane, gthreads = G * 32;
    __shared__ float gmax[W];
    const size_t d = (size_t)vec_per_row * 8;
    for (int base = 0; base < T; base += groups) {  // the same trip count in every warp
      const int tt = base + grp;
      const bool act = tt < T;
      const uint4* src = x + (size_t)(act ? tt : 0) * vec_per_row;
      float mx = 0.f;
      if (act) {
#pragma unroll 4
        for (int v = gt; v < vec_per_row; v += gthreads) mx = fmaxf(mx, vec_maxabs(__ldg(src + v)));
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (lane == 0) gmax[warp] = mx;
      __syncthreads();
      mx = 0.f;
      for (int g = 0; g < G; ++g) mx = fmaxf(mx, gmax[grp * G + g]);
      __syncthreads();  // gmax is reused by the next round
      if (act) {
        const float a = plane_scale(mx), inv_a = __frcp_rn(a);  // correctly rounded 1 / a
        int rows[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) rows[j] = j < k ? rows_s[tt][j] : 0;
        if (gt == 0) {
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k) P.scale[rows[j]] = a;
        }
#pragma unroll 4
        for (int v = gt; v < vec_per_row; v += gthreads)
          vec_planes_to_rows(__ldg(src + v), a, inv_a, v, d, rows, k, P);
      }
    }
    return;
  }
  // copy: the whole CTA walks (token, 16-byte vector) pairs
  for (int q = threadIdx.x; q < T * vec_per_row; q += kFusedRouteThreads) {
    const int tt = q / vec_per_row, v = q - tt * vec_per_row;
    const Tv val = __ldg(x + (size_t)tt * vec_per_row + v);
    for (int j = 0; j < k; ++j) Xp[(size_t)rows_s[tt][j] * vec_per_row + v] = val;
  }
}

}  // namespace

cudaError_t launch_route_fused(const void* x, int act, int T, int d, const int32_t* idx, int k, int E, int bm,
                               int32_t* counts, int32_t* offsets, int32_t* mt_prefix, int32_t* src_row,
                               int32_t* dst_row, void* Xp, const RowPlanes* planes, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (T > kFusedRouteMaxT) return cudaErrorInvalidValue;
  if (planes && act != COLIBRI_BF16) return cudaErrorInvalidValue;
  const int esize = (act == COLIBRI_BF16) ? 2 : 4;
  const int vec = d * esize / 16;
  const RowPlanes P = planes ? *planes : RowPlanes{nullptr, nullptr, nullptr};
  return launch_kernel(route_fused_kernel<uint4>, dim3(1), dim3(kFusedRouteThreads), 0, s, 1, (const uint4*)x, T, vec,
                       idx, k, E, bm, counts, offsets, mt_prefix, src_row, dst_row, (uint4*)Xp, P);
}

cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int32_t* blk_counts,
                               int32_t* local_rank, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int nblk = (T + kCountBlock - 1) / kCountBlock;
  const size_t smem = sizeof(uint32_t) * (kCountBlock / 32) * E;
  return launch_kernel(route_count_kernel, dim3(nblk), dim3(kCountBlock), smem, s, 1, idx, T, k, E, blk_counts,
                       local_rank);
}

cudaError_t launch_route_scan(const int32_t* blk_counts, int nblk, int E, int bm, int32_t* blk_base,
                              int32_t* counts, int32_t* offsets, int32_t* mt_prefix,
                              cudaStream_t s) {
  return launch_kernel(route_scan_kernel, dim3(1), dim3(256), 0, s, 1, blk_counts, nblk, E, bm, blk_base, counts,
                       offsets, mt_prefix);
}

cudaError_t launch_route_scatter(const void* x, int act, int T, int d, int k, int E,
                                 const int32_t* idx, const int32_t* blk_base, const int32_t* offsets,
                                 int32_t* dst_row, int32_t* src_row, void* Xp, const RowPlanes* planes,
                                 cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (planes && act != COLIBRI_BF16) return cudaErrorInvalidValue;
  const RowPlanes P = planes ? *planes : RowPlanes{nullptr, nullptr, nullptr};
  const int esize = (act == COLIBRI_BF16) ? 2 : 4;
  const int vec = d * esize / 16;  // d is a multiple of 64, rows are whole 16-byte vectors
  const int warps_per_cta = 8;
  int grid = (T + warps_per_cta - 1) / warps_per_cta;
  if (grid > 4096) grid = 4096;
  return launch_kernel(route_scatter_kernel<uint4>, dim3(grid), dim3(warps_per_cta * 32), 0, s, 1, (const uint4*)x,
                       T, vec, k, E, idx, blk_base, offsets, dst_row, src_row, (uint4*)Xp, P);
}

}  // namespace colibri
