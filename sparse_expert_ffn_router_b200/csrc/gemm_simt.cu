// Expert Compute stage for fp32 weights: grouped SwiGLU FFN with fp32 FMA (no TF32, so the
// result keeps fp32 accuracy).  Experts are addressed at a fixed stride in one buffer
// (www.mhpq.cn/news/563172 §2.1; www.0539edu.com/news/4774449 §2.2: one expert's parameters
// contiguous); rows are the grouped rows of each expert (www.trdm.cn/news/555962 §6.2).
//
//   gate/up:  H[r][n] = silu(sum_i A[r][i] W1_e[n][i]) * (sum_i A[r][i] W3_e[n][i])
//   down:     Y[r][n] = sum_i H[r][i] W2_e[n][i]
//
// 64 x 64 output tiles, K staged 16 at a time through shared memory, 4 x 4 register tile per
// thread.  Tiles are laid out on a (n-tile, m-tile) grid; m-tiles map to (expert, rows) through
// the device-side m-tile prefix, so no host synchronisation is needed.
#include "common.cuh"

namespace colibri {
namespace {

constexpr int BM = kSimtBM, BN = kSimtBN, BK = kSimtBK;

__device__ __forceinline__ bool simt_tile_rows(const SimtGroups& g, int mt, int& grp, int& row0,
                                               int& row_end) {
  if (g.offsets == nullptr) {
    grp = 0;
    row0 = mt * BM;
    row_end = g.rows_single;
    return row0 < row_end;
  }
  if (mt >= g.mt_prefix[g.G]) return false;
  int lo = 0, hi = g.G - 1;  // largest grp with mt_prefix[grp] <= mt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g.mt_prefix[mid] <= mt) lo = mid;
    else hi = mid - 1;
  }
  grp = lo;
  row0 = g.offsets[grp] + (mt - g.mt_prefix[grp]) * BM;
  row_end = g.offsets[grp + 1];
  return row0 < row_end;
}

template <bool kGateUp>
__global__ void __launch_bounds__(256) simt_ffn_kernel(const float* __restrict__ A, int lda, int K,
                                                       const float* __restrict__ W,
                                                       int64_t wstride, int d, int f,
                                                       SimtGroups groups,
                                                       float* __restrict__ out, int ldo, int N) {
  pdl_trigger();
  pdl_wait();
  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  __shared__ __align__(16) float Cs[kGateUp ? BK : 1][BN + 4];
  int grp, row0, row_end;
  if (!simt_tile_rows(groups, blockIdx.y, grp, row0, row_end)) return;
  const int n0 = blockIdx.x * BN;
  const float* base = W + (int64_t)grp * wstride;
  // gate/up: W1 rows [n][d] then W3 rows at +f*d; down: W2 rows [n][f] at +2*f*d
  const float* B1 = kGateUp ? base : base + 2 * (int64_t)f * d;
  const float* B3 = base + (int64_t)f * d;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int lr = tid >> 2, lk = (tid & 3) * 4;
  float acc1[4][4] = {}, acc3[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    {
      const int r = row0 + lr;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < row_end) v = *reinterpret_cast<const float4*>(A + (size_t)r * lda + k0 + lk);
      As[lk + 0][lr] = v.x; As[lk + 1][lr] = v.y; As[lk + 2][lr] = v.z; As[lk + 3][lr] = v.w;
      const int n = n0 + lr;
      float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n < N) b = *reinterpret_cast<const float4*>(B1 + (size_t)n * K + k0 + lk);
      Bs[lk + 0][lr] = b.x; Bs[lk + 1][lr] = b.y; Bs[lk + 2][lr] = b.z; Bs[lk + 3][lr] = b.w;
      if (kGateUp) {
        float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n < N) c = *reinterpret_cast<const float4*>(B3 + (size_t)n * K + k0 + lk);
        Cs[lk + 0][lr] = c.x; Cs[lk + 1][lr] = c.y; Cs[lk + 2][lr] = c.z; Cs[lk + 3][lr] = c.w;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc1[i][j] = fmaf(av[i], bv[j], acc1[i][j]);
      if (kGateUp) {
        const float4 c = *reinterpret_cast<const float4*>(&Cs[kk][tx * 4]);
        const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc3[i][j] = fmaf(av[i], cv[j], acc3[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty * 4 + i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc1[i][j];
      if (kGateUp) v = v / (1.0f + expf(-v)) * acc3[i][j];
      out[(size_t)r * ldo + n] = v;
    }
  }
}

}  // namespace

cudaError_t launch_simt_gateup(const float* A, int lda, const float* W, int64_t wstride, int d,
                               int f, SimtGroups g, int mt_bound, float* H, cudaStream_t s) {
  if (mt_bound <= 0) return cudaSuccess;
  const dim3 grid((f + BN - 1) / BN, mt_bound);
  return launch_kernel(simt_ffn_kernel<true>, grid, dim3(256), 0, s, 1, A, lda, d, W, wstride, d, f, g, H, f, f);
}

cudaError_t launch_simt_down(const float* H, int f, const float* W, int64_t wstride, int d,
                             SimtGroups g, int mt_bound, float* Y, cudaStream_t s) {
  if (mt_bound <= 0) return cudaSuccess;
  const dim3 grid((d + BN - 1) / BN, mt_bound);
  return launch_kernel(simt_ffn_kernel<false>, grid, dim3(256), 0, s, 1, H, f, f, W, wstride, d, f, g, Y, d, d);
}

}  // namespace colibri
