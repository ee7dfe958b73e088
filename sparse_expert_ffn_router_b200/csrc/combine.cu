// Gather stage: y[t] = sum_{j<k} w[t][j] * Yp[dst_row[t][j]]  (+ Ys[t] for the shared expert),
// summed in slot order j = 0..k-1 in fp32 and rounded once to the activation dtype
// (www.hotelren.com/news/4731937 §2.1 step 6 and §2.3 combine_kernel; the fixed-order k-way
// aggregation of www.pptc.cn/news/100465 §2.1, without the atomic accumulation of its §1 so
// that the result is deterministic).  One warp per token, 16-byte vector accesses.
#include <algorithm>

#include "common.cuh"

namespace colibri {
namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = q;
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

template <typename Tout, typename Typ>
__global__ void __launch_bounds__(256) combine_kernel(const Typ* __restrict__ Yp,
                                                      const int32_t* __restrict__ dst_row,
                                                      const float* __restrict__ w, int T, int k,
                                                      int d, const Typ* __restrict__ Ys,
                                                      Tout* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
    int r = 0;
    float wj = 0.f;
    if (lane < k) {
      r = dst_row[(size_t)t * k + lane];
      wj = w[(size_t)t * k + lane];
    }
    int rows[kMaxTopK];
    float ws[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      rows[j] = __shfl_sync(0xffffffffu, r, j);
      ws[j] = __shfl_sync(0xffffffffu, wj, j);
    }
    for (int c = lane * 8; c < d; c += 32 * 8) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
          float v[8];
          load8(Yp + (size_t)rows[j] * d + c, v);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(ws[j], v[i], acc[i]);
        }
      }
      if (Ys) {
        float v[8];
        load8(Ys + (size_t)t * d + c, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += v[i];
      }
      store8(y + (size_t)t * d + c, acc);
    }
  }
}

// int8 path: the down projection leaves `nsplit` K-partial sums per grouped row.  One thread
// per (token, 8 consecutive outputs): all k x nsplit partial loads of a thread are independent,
// so a handful of tokens is one short latency, not a serial walk.
template <typename Tout>
__global__ void __launch_bounds__(256) combine_split_kernel(const float* __restrict__ Ypart,
                                                            int nsplit, int rows,
                                                            const int32_t* __restrict__ dst_row,
                                                            const float* __restrict__ w, int T,
                                                            int k, int d, Tout* __restrict__ y) {
  const int chunks = d >> 3;
  const size_t split_stride = (size_t)rows * d;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < (long long)T * chunks;
       q += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(q / chunks), c = (int)(q - (long long)t * chunks) * 8;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k) {
        const int r = dst_row[(size_t)t * k + j];
        const float wj = w[(size_t)t * k + j];
        float part[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int sidx = 0; sidx < kDecSplitMax; ++sidx) {
          if (sidx < nsplit) {
            float v[8];
            load8(Ypart + sidx * split_stride + (size_t)r * d + c, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) part[i] += v[i];
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, part[i], acc[i]);
      }
    }
    store8(y + (size_t)t * d + c, acc);
  }
}

int grid_for_tokens(int T) {
  int g = (T + 7) / 8;
  return g > 8192 ? 8192 : g;
}

}  // namespace

cudaError_t launch_combine(const void* Yp, int yp_dtype, const int32_t* dst_row, const float* w,
                           int T, int k, int d, const void* Ys, void* y, int act, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const int grid = grid_for_tokens(T);
  if (yp_dtype == COLIBRI_BF16) {
    if (act == COLIBRI_BF16)
      combine_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, s>>>(
          (const __nv_bfloat16*)Yp, dst_row, w, T, k, d, (const __nv_bfloat16*)Ys,
          (__nv_bfloat16*)y);
    else
      combine_kernel<float, __nv_bfloat16><<<grid, 256, 0, s>>>(
          (const __nv_bfloat16*)Yp, dst_row, w, T, k, d, (const __nv_bfloat16*)Ys, (float*)y);
  } else {
    if (act == COLIBRI_BF16)
      combine_kernel<__nv_bfloat16, float><<<grid, 256, 0, s>>>(
          (const float*)Yp, dst_row, w, T, k, d, (const float*)Ys, (__nv_bfloat16*)y);
    else
      combine_kernel<float, float><<<grid, 256, 0, s>>>((const float*)Yp, dst_row, w, T, k, d,
                                                        (const float*)Ys, (float*)y);
  }
  return cudaGetLastError();
}

cudaError_t launch_combine_split(const float* Ypart, int nsplit, int rows, const int32_t* dst_row,
                                 const float* w, int T, int k, int d, void* y, int act,
                                 cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (nsplit > kDecSplitMax) return cudaErrorInvalidValue;
  long long threads = (long long)T * (d / 8);
  int grid = (int)std::min<long long>((threads + 255) / 256, 8192);
  if (act == COLIBRI_BF16)
    combine_split_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(Ypart, nsplit, rows, dst_row, w, T, k,
                                                             d, (__nv_bfloat16*)y);
  else
    combine_split_kernel<float><<<grid, 256, 0, s>>>(Ypart, nsplit, rows, dst_row, w, T, k, d,
                                                     (float*)y);
  return cudaGetLastError();
}

}  // namespace colibri
