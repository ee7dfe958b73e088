// Gather stage: y[t] = sum_{j<k} w[t][j] * Yp[dst_row[t][j]]  (+ Ys[t] for the shared expert),
// summed in slot order j = 0..k-1 in fp32 and rounded once to the activation dtype
// (www.hotelren.com/news/4731937 §2.1 step 6 and §2.3 combine_kernel; the fixed-order k-way
// aggregation of www.pptc.cn/news/100465 §2.1, without the atomic accumulation of its §1 so
// that the result is deterministic).  16-byte vector accesses.
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

// One thread per (token, 8 consecutive outputs): the k slot loads of a thread are independent,
// and a warp covers 512 contiguous bytes of each row it reads or writes.
template <typename Tout, typename Typ>
__global__ void __launch_bounds__(256) combine_kernel(const Typ* __restrict__ Yp,
                                                      const int32_t* __restrict__ dst_row,
                                                      const float* __restrict__ w, int T, int k,
                                                      int d, const Typ* __restrict__ Ys,
                                                      Tout* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int chunks = d >> 3;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < (long long)T * chunks;
       q += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(q / chunks), c = (int)(q - (long long)t * chunks) * 8;
    int rows[kMaxTopK];
    float ws[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      rows[j] = j < k ? dst_row[(size_t)t * k + j] : 0;
      ws[j] = j < k ? w[(size_t)t * k + j] : 0.f;
    }
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

// int8 path: the down projection leaves `nsplit` K-partial sums per grouped row.  One thread
// per (token, 4 consecutive outputs).  A slot's partials are loaded 8 at a time before they are
// summed (in split order), so a handful of tokens costs a few memory round trips, not one per
// partial.
__device__ __forceinline__ float4 ld4(const float* p) { return __ldg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ void add4(float4& a, const float4& b) {
  a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
}
__device__ __forceinline__ void store4(float* p, const float4& v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float4& v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 q;
  q.x = *reinterpret_cast<const uint32_t*>(&a);
  q.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = q;
}

template <typename Tout>
__global__ void __launch_bounds__(256) combine_split_kernel(const float* __restrict__ Ypart,
                                                            int nsplit, int rows,
                                                            const int32_t* __restrict__ dst_row,
                                                            const float* __restrict__ w, int T,
                                                            int k, int d, Tout* __restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int chunks = d >> 2;
  const size_t ss = (size_t)rows * d;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < (long long)T * chunks;
       q += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(q / chunks), c = (int)(q - (long long)t * chunks) * 4;
    int rs[kMaxTopK];
    float ws[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      rs[j] = j < k ? dst_row[(size_t)t * k + j] : 0;
      ws[j] = j < k ? w[(size_t)t * k + j] : 0.f;
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j >= k) break;
      const float* base = Ypart + (size_t)rs[j] * d + c;
      float4 part = make_float4(0.f, 0.f, 0.f, 0.f);
      int sp = 0;
      for (; sp + 8 <= nsplit; sp += 8) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = ld4(base + (size_t)(sp + i) * ss);
#pragma unroll
        for (int i = 0; i < 8; ++i) add4(part, v[i]);
      }
      for (; sp < nsplit; ++sp) add4(part, ld4(base + (size_t)sp * ss));
      acc.x = fmaf(ws[j], part.x, acc.x);
      acc.y = fmaf(ws[j], part.y, acc.y);
      acc.z = fmaf(ws[j], part.z, acc.z);
      acc.w = fmaf(ws[j], part.w, acc.w);
    }
    store4(y + (size_t)t * d + c, acc);
  }
}

int grid_for_rows(int T, int d) {
  const long long threads = (long long)T * (d / 8);
  return (int)std::min<long long>((threads + 255) / 256, 16384);
}

}  // namespace

cudaError_t launch_combine(const void* Yp, int yp_dtype, const int32_t* dst_row, const float* w,
                           int T, int k, int d, const void* Ys, void* y, int act, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const dim3 grid(grid_for_rows(T, d)), block(256);
  if (yp_dtype == COLIBRI_BF16) {
    const __nv_bfloat16* yp = (const __nv_bfloat16*)Yp;
    const __nv_bfloat16* ys = (const __nv_bfloat16*)Ys;
    if (act == COLIBRI_BF16)
      return launch_kernel(combine_kernel<__nv_bfloat16, __nv_bfloat16>, grid, block, 0, s, 1, yp, dst_row, w, T, k,
                           d, ys, (__nv_bfloat16*)y);
    return launch_kernel(combine_kernel<float, __nv_bfloat16>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys,
                         (float*)y);
  }
  const float* yp = (const float*)Yp;
  const float* ys = (const float*)Ys;
  if (act == COLIBRI_BF16)
    return launch_kernel(combine_kernel<__nv_bfloat16, float>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys,
                         (__nv_bfloat16*)y);
  return launch_kernel(combine_kernel<float, float>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys, (float*)y);
}

cudaError_t launch_combine_split(const float* Ypart, int nsplit, int rows, const int32_t* dst_row,
                                 const float* w, int T, int k, int d, void* y, int act,
                                 cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (nsplit > kDecSplitMax) return cudaErrorInvalidValue;
  long long threads = (long long)T * (d / 4);
  const dim3 grid((unsigned)std::min<long long>((threads + 255) / 256, 8192)), block(256);
  if (act == COLIBRI_BF16)
    return launch_kernel(combine_split_kernel<__nv_bfloat16>, grid, block, 0, s, 1, Ypart, nsplit, rows, dst_row, w,
                         T, k, d, (__nv_bfloat16*)y);
  return launch_kernel(combine_split_kernel<float>, grid, block, 0, s, 1, Ypart, nsplit, rows, dst_row, w, T, k, d,
                       (float*)y);
}

}  // namespace colibri
