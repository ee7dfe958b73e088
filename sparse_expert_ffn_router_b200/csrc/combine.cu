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

// One warp per token row: the routing state of the token is loaded once (one broadcast load per
// slot), then each lane sums 8 consecutive outputs at a time, U = 8 / KK such groups per step
// with all U x KK slot loads of the step (16 bytes each for bf16) issued before any is used, so
// a lane keeps 8 loads in flight and a warp covers 512 contiguous bytes of each row it reads or
// writes.  KK is the top-k (1, 2, 4 or 8; other k run with KK = 8 and the unused slots skipped).
template <typename Typ>
struct Raw8;  // 8 consecutive Yp values as loaded
template <>
struct Raw8<__nv_bfloat16> {
  uint4 q;
  __device__ void load(const __nv_bfloat16* p) { q = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ float get(int i) const {
    const uint32_t wv = i < 2 ? q.x : (i < 4 ? q.y : (i < 6 ? q.z : q.w));
    return __uint_as_float((i & 1) ? (wv & 0xffff0000u) : (wv << 16));
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ float get(int i) const {
    return i == 0 ? a.x : i == 1 ? a.y : i == 2 ? a.z : i == 3 ? a.w : i == 4 ? b.x : i == 5 ? b.y : i == 6 ? b.z : b.w;
  }
};

template <typename Tout, typename Typ, int KK>
__global__ void __launch_bounds__(256) combine_kernel(const Typ* __restrict__ Yp,
                                                      const int32_t* __restrict__ dst_row,
                                                      const float* __restrict__ w, int T, int k,
                                                      int d, const Typ* __restrict__ Ys,
                                                      Tout* __restrict__ y) {
  constexpr int U = 8 / KK;
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int chunks = d >> 3;
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long t = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
    int rows[KK];
    float ws[KK];
#pragma unroll
    for (int j = 0; j < KK; ++j) {
      rows[j] = j < k ? __ldg(dst_row + (size_t)t * k + j) : 0;
      ws[j] = j < k ? __ldg(w + (size_t)t * k + j) : 0.f;
    }
    for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
      Raw8<Typ> v[U][KK];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = (c0 + 32 * u) * 8;
#pragma unroll
        for (int j = 0; j < KK; ++j)
          if (j < k && c < d) v[u][j].load(Yp + (size_t)rows[j] * d + c);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = (c0 + 32 * u) * 8;
        if (c >= d) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < KK; ++j)
          if (j < k)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(ws[j], v[u][j].get(i), acc[i]);
        if (Ys) {
          float vs[8];
          load8(Ys + (size_t)t * d + c, vs);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] += vs[i];
        }
        store8(y + (size_t)t * d + c, acc);
      }
    }
  }
}

template <typename Tout, typename Typ>
cudaError_t launch_combine_k(const Typ* yp, const int32_t* dst_row, const float* w, int T, int k, int d, const Typ* ys,
                             Tout* y, dim3 grid, cudaStream_t s) {
  const dim3 block(256);
  switch (k) {
    case 1: return launch_kernel(combine_kernel<Tout, Typ, 1>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys, y);
    case 2: return launch_kernel(combine_kernel<Tout, Typ, 2>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys, y);
    case 3:
    case 4: return launch_kernel(combine_kernel<Tout, Typ, 4>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys, y);
    default: return launch_kernel(combine_kernel<Tout, Typ, 8>, grid, block, 0, s, 1, yp, dst_row, w, T, k, d, ys, y);
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

// one warp per token, up to 16 CTAs of 8 warps per SM of a 148-SM part
int grid_for_rows(int T) { return (int)std::min<long long>(((long long)T + 7) / 8, 148 * 16); }

}  // namespace

cudaError_t launch_combine(const void* Yp, int yp_dtype, const int32_t* dst_row, const float* w,
                           int T, int k, int d, const void* Ys, void* y, int act, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (k < 1 || k > kMaxTopK) return cudaErrorInvalidValue;
  const dim3 grid(grid_for_rows(T));
  if (yp_dtype == COLIBRI_BF16) {
    const __nv_bfloat16* yp = (const __nv_bfloat16*)Yp;
    const __nv_bfloat16* ys = (const __nv_bfloat16*)Ys;
    if (act == COLIBRI_BF16) return launch_combine_k(yp, dst_row, w, T, k, d, ys, (__nv_bfloat16*)y, grid, s);
    return launch_combine_k(yp, dst_row, w, T, k, d, ys, (float*)y, grid, s);
  }
  const float* yp = (const float*)Yp;
  const float* ys = (const float*)Ys;
  if (act == COLIBRI_BF16) return launch_combine_k(yp, dst_row, w, T, k, d, ys, (__nv_bfloat16*)y, grid, s);
  return launch_combine_k(yp, dst_row, w, T, k, d, ys, (float*)y, grid, s);
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
