// Gate stage: router logits, softmax and top-k.  bf16 activations with E <= 128 use the
// tensor-core kernel below (the stage is bound by one read of x); fp32 activations, and more
// than 128 experts, use the SIMT kernel.
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

// ---------------------------------------------------------------------------------------
// bf16 router on the tensor cores (mma.sync m16n8k16, fp32 accumulation).  One warp owns 16
// tokens x all E experts (NB n-blocks of 8).  For a 32-wide K block a thread (g = lane / 4,
// c = lane % 4) loads 16 contiguous bytes [8c, 8c + 8) of token rows g and g + 8 and of expert
// row g of every n-block; MMA k-step s in {0, 1} takes elements 8c + 4s + {0,1} as logical
// k = 2c, 2c+1 and 8c + 4s + {2,3} as k = 2c+8, 2c+9 on both operands, so the K permutation
// cancels in the dot product.  The CTA's 4 warps cover TM token groups x KS K-slices
// (TM * KS = 4); K-slice partial logits are summed in fixed slice order in shared memory.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int NB, int TM>
__global__ void __launch_bounds__(128) router_topk_mma_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int d, const __nv_bfloat16* __restrict__ wr,
    const float* __restrict__ b, int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  constexpr int KS = 4 / TM;
  constexpr int TT = 16 * TM;
  extern __shared__ float sm[];
  float* part = sm;                       // [KS][TT][E]
  float* lg = part + KS * TT * E;         // [TT][E + 1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int tg = warp % TM, ks = warp / TM;
  const int t0 = blockIdx.x * TT + tg * 16;
  const int ta = min(t0 + g, T - 1), tb = min(t0 + g + 8, T - 1);
  const bool va = t0 + g < T, vb = t0 + g + 8 < T;
  const __nv_bfloat16* xa = x + (size_t)ta * d + 8 * c;
  const __nv_bfloat16* xb = x + (size_t)tb * d + 8 * c;
  const __nv_bfloat16* wrow[NB];
  bool wv[NB];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int e = nb * 8 + g;
    wv[nb] = e < E;
    wrow[nb] = wr + (size_t)min(e, E - 1) * d + 8 * c;
  }
  float acc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) acc[nb][0] = acc[nb][1] = acc[nb][2] = acc[nb][3] = 0.f;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  const int nkb = d / 32;
  for (int kb = ks; kb < nkb; kb += KS) {
    const int ko = kb * 32;
    const uint4 av = va ? ld_nc16(xa + ko) : zero;
    const uint4 bv4 = vb ? ld_nc16(xb + ko) : zero;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const uint4 wq = wv[nb] ? ld_nc16(wrow[nb] + ko) : zero;
      mma16816(acc[nb], av.x, bv4.x, av.y, bv4.y, wq.x, wq.y);  // k-step 0
      mma16816(acc[nb], av.z, bv4.z, av.w, bv4.w, wq.z, wq.w);  // k-step 1
    }
  }
  // C fragment: rows g / g + 8 (tokens), columns 2c, 2c + 1 (experts of the n-block)
  float* pw = part + (size_t)ks * TT * E;
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int row = tg * 16 + g + (q >> 1) * 8;
      const int e = nb * 8 + 2 * c + (q & 1);
      if (e < E) pw[row * E + e] = acc[nb][q];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < TT * E; i += 128) {
    const int row = i / E, e = i - row * E;
    float v = b ? b[e] : 0.f;
    float sum = 0.f;
#pragma unroll
    for (int s2 = 0; s2 < KS; ++s2) sum += part[(size_t)s2 * TT * E + i];
    lg[row * (E + 1) + e] = sum + v;
  }
  __syncthreads();
  for (int tt = warp; tt < TT; tt += 4) {
    const int t = blockIdx.x * TT + tt;
    if (t >= T) break;
    warp_topk(lg + tt * (E + 1), E, k, lane, idx_out + (size_t)t * k, w_out + (size_t)t * k);
  }
}

template <int NB, int TM>
cudaError_t launch_mma_router(const void* x, int T, int d, const void* wr, const float* b, int E, int k,
                              int32_t* idx, float* w, cudaStream_t s) {
  constexpr int KS = 4 / TM, TT = 16 * TM;
  const size_t smem = sizeof(float) * ((size_t)KS * TT * E + (size_t)TT * (E + 1));
  auto kern = router_topk_mma_kernel<NB, TM>;
  if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<(T + TT - 1) / TT, 128, smem, s>>>((const __nv_bfloat16*)x, T, d, (const __nv_bfloat16*)wr, b, E, k,
                                            idx, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_topk(const void* x, int act, int T, int d, const void* wr, const float* b,
                               int E, int k, int32_t* idx, float* w, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const size_t smem =
      sizeof(float) * ((size_t)kRouterTT * (kRouterDK + 1) + (size_t)E * (kRouterDK + 1) +
                       (size_t)kRouterTT * (E + 1));
  const dim3 grid((T + kRouterTT - 1) / kRouterTT);
  if (act == COLIBRI_BF16 && E <= 128) {
    // tensor-core router; token tile and K split chosen by the number of experts
    if (E <= 8) return launch_mma_router<1, 1>(x, T, d, wr, b, E, k, idx, w, s);
    if (E <= 16) return launch_mma_router<2, 1>(x, T, d, wr, b, E, k, idx, w, s);
    if (E <= 32) return launch_mma_router<4, 2>(x, T, d, wr, b, E, k, idx, w, s);
    if (E <= 64) return launch_mma_router<8, 4>(x, T, d, wr, b, E, k, idx, w, s);
    return launch_mma_router<16, 4>(x, T, d, wr, b, E, k, idx, w, s);
  }
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
