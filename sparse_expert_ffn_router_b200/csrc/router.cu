// Gate stage: router logits, softmax and top-k.
//
// logits l[t][e] = b[e] + sum_i x[t][i] * Wr[e][i]      (www.hotelren.com/news/4731937 §3.2,
//                                                        www.0539edu.com/news/4774449 §2.1)
// top-k: order by (logit descending, expert index ascending), slot 0 = largest; ties keep
// the lower index, as the strict ">" scan of www.mhpq.cn/news/563172 §3.2 does.  The
// selection is made by k rounds of a warp-wide arg-max (the warp-shuffle top-k idea of
// www.pptc.cn/news/100465 §2.1, generalised from 2 to k <= 8 and to 256 experts).
// weights: softmax over all E renormalised over the k chosen, computed as
// exp(l_j - l_0) / sum_j' exp(l_j' - l_0) in fp32.
// Output layout [T][k] (www.pptc.cn/news/100465 §3.4).
#include "common.cuh"

namespace colibri {
namespace {

constexpr int kRouterTT = 32;  // tokens per CTA
constexpr int kRouterDK = 32;  // K chunk staged in shared memory
constexpr int kRouterThreads = 256;

// One warp selects the top-k of one token whose E logits sit in shared memory.
__device__ __forceinline__ void warp_topk(const float* lg, int E, int k, int lane, int32_t* idx_out,
                                          float* w_out) {
  float v[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int e = lane + 32 * m;
    v[m] = (e < E) ? lg[e] : -INFINITY;
  }
  uint32_t used = 0;
  float sel_v[kMaxTopK];
  int sel_e[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    sel_v[j] = -INFINITY;
    sel_e[j] = 0;
    if (j < k) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const int e = lane + 32 * m;
        if (e < E && !((used >> m) & 1u)) {
          if (v[m] > bv || (v[m] == bv && e < be)) {
            bv = v[m];
            be = e;
          }
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be & 31) == lane) used |= 1u << (be >> 5);
      sel_v[j] = bv;
      sel_e[j] = be;
    }
  }
  if (lane == 0) {
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) den += expf(sel_v[j] - sel_v[0]);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) {
        idx_out[j] = sel_e[j];
        w_out[j] = expf(sel_v[j] - sel_v[0]) / den;
      }
  }
}

// SIMT router: 32 tokens per CTA, warp w accumulates experts w, w+8, ... for the token of
// its lane; x and Wr chunks are staged in shared memory as fp32.
template <typename Tin>
__global__ void __launch_bounds__(kRouterThreads) router_topk_simt_kernel(
    const Tin* __restrict__ x, int T, int d, const Tin* __restrict__ wr, const float* __restrict__ b,
    int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  extern __shared__ float sm[];
  constexpr int P = kRouterDK + 1;
  float* xs = sm;                        // [TT][P]
  float* ws = xs + kRouterTT * P;        // [E][P]
  float* lg = ws + E * P;                // [TT][E+1]
  const int t0 = blockIdx.x * kRouterTT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc[32];
#pragma unroll
  for (int m = 0; m < 32; ++m) acc[m] = 0.f;

  for (int i0 = 0; i0 < d; i0 += kRouterDK) {
    for (int q = threadIdx.x; q < kRouterTT * kRouterDK; q += kRouterThreads) {
      const int r = q / kRouterDK, c = q % kRouterDK, t = t0 + r;
      xs[r * P + c] = (t < T && i0 + c < d) ? to_f32(x[(size_t)t * d + i0 + c]) : 0.f;
    }
    for (int q = threadIdx.x; q < E * kRouterDK; q += kRouterThreads) {
      const int r = q / kRouterDK, c = q % kRouterDK;
      ws[r * P + c] = (i0 + c < d) ? to_f32(wr[(size_t)r * d + i0 + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kRouterDK; ++c) {
      const float xv = xs[lane * P + c];
#pragma unroll
      for (int m = 0; m < 32; ++m) {
        const int e = warp + 8 * m;
        if (e < E) acc[m] = fmaf(xv, ws[e * P + c], acc[m]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int m = 0; m < 32; ++m) {
    const int e = warp + 8 * m;
    if (e < E) lg[lane * (E + 1) + e] = acc[m] + (b ? b[e] : 0.f);
  }
  __syncthreads();
  for (int tt = warp; tt < kRouterTT; tt += kRouterThreads / 32) {
    const int t = t0 + tt;
    if (t >= T) break;
    warp_topk(lg + tt * (E + 1), E, k, lane, idx_out + (size_t)t * k, w_out + (size_t)t * k);
  }
}

}  // namespace

cudaError_t launch_router_topk(const void* x, int act, int T, int d, const void* wr, const float* b,
                               int E, int k, int32_t* idx, float* w, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const size_t smem =
      sizeof(float) * ((size_t)kRouterTT * (kRouterDK + 1) + (size_t)E * (kRouterDK + 1) +
                       (size_t)kRouterTT * (E + 1));
  const dim3 grid((T + kRouterTT - 1) / kRouterTT);
  if (act == COLIBRI_BF16) {
    auto kern = router_topk_simt_kernel<__nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kRouterThreads, smem, s>>>((const __nv_bfloat16*)x, T, d,
                                            (const __nv_bfloat16*)wr, b, E, k, idx, w);
  } else {
    auto kern = router_topk_simt_kernel<float>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kRouterThreads, smem, s>>>((const float*)x, T, d, (const float*)wr, b, E, k, idx, w);
  }
  return cudaGetLastError();
}

}  // namespace colibri
