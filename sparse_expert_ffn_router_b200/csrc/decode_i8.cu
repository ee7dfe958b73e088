// Expert Compute stage for int8 weights with per-output-channel fp32 scales, dequantised in
// the kernel (www.0539edu.com/news/4774449 §3.1 stores int8 weights with scales; the scale
// here is per output channel).  For a handful of tokens the layer is a stream over the
// weights of the touched experts, bound by HBM bandwidth, so the design streams each weight
// byte once and keeps everything else off the critical path:
//
//   gate/up:  H[r][o]    = silu(s1[o] * sum_i q1[o][i] x[r][i]) * (s3[o] * sum_i q3[o][i] x[r][i])
//   down:     Yp_s[r][o] = s2[o] * sum_{i in split s} q2[o][i] H[r][i]
//
// W[o][i] = s[o] q[o][i], so the weight scale factors out of each dot product exactly.  The
// weights are never converted: each activation row (bf16) is first split, once, into two int8
// planes with a per-row scale, x ~= a * (hi + lo / 254) with a = max|x| / 127 (the residual
// after hi is at most a/2, so lo fits in [-127, 127]; the representation error is at most
// a / 508 = max|x| / 64516 per element, far below bf16's own rounding of the result).  The dot
// products then run on the integer tensor cores (mma.sync m16n8k32, s8 x s8 -> s32, exact
// integer accumulation), weights as the A operand (16 output channels), tokens as n-blocks
// of 8, and the epilogue forms s[o] * a * (acc_hi + acc_lo / 254) in fp32.
//
// Work decomposition: every warp is independent (no shared memory, no CTA barrier).  A work
// item is (touched expert, 16 output channels, K range); a persistent grid of warps walks the
// items of the experts that received rows only.  Per 256-wide K block a thread issues all of its
// 16-byte weight loads (ld.global.nc.L1::no_allocate, streamed once) before using any of them;
// activation planes are read through L1, where the warps of an SM working on the same expert
// share them.  The down projection is split over K into `nsplit` fp32 partial sums (summed in
// fixed order by the combine) so that a single token still spreads over every SM.
//
// Fragment bookkeeping: for each 64-wide K block a thread (g = lane/4, c = lane%4) loads 16
// consecutive weight bytes [16c, 16c + 16) of rows g and g + 8.  MMA k-step s (0, 1) uses bytes
// [16c + 8s, 16c + 8s + 8): the first four as logical k = 4c..4c+3 and the last four as
// k = 16+4c..16+4c+3.  The activation fragment of the same step is read from the same physical
// positions, so the permutation of K inside the block is the same on both operands and the
// dot product is unchanged.
#include <algorithm>

#include "common.cuh"

namespace colibri {
namespace {

constexpr int kWarpsPerCta = 8;
constexpr int KB = 256;  // K elements per streamed block (4 sub-blocks of 64)

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ldg_cached8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One warp per row: a = max|x| / 127, hi = rint(x / a), lo = rint((x - a * hi) * 254 / a).
__global__ void __launch_bounds__(256) dec_split_rows_kernel(const __nv_bfloat16* __restrict__ X, int R, int K,
                                                             int8_t* __restrict__ hi, int8_t* __restrict__ lo,
                                                             float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += nw) {
    const uint4* src = reinterpret_cast<const uint4*>(X + (size_t)r * K);
    float mx = 0.f;
    for (int v = lane; v < K / 8; v += 32) {
      const uint4 q = src[v];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(h[i]);
        mx = fmaxf(mx, fmaxf(fabsf(f2.x), fabsf(f2.y)));
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float a = mx > 0.f ? mx / 127.f : 1.f;
    const float inv_a = 1.f / a;
    if (lane == 0) scale[r] = a;
    for (int v = lane; v < K / 8; v += 32) {
      const uint4 q = src[v];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float xv = __bfloat162float(i & 1 ? h[i >> 1].y : h[i >> 1].x);
        const float qh = fminf(fmaxf(rintf(xv * inv_a), -127.f), 127.f);
        const float res = fmaf(-a, qh, xv);
        const float ql = fminf(fmaxf(rintf(res * inv_a * 254.f), -127.f), 127.f);
        hw[i >> 2] |= ((uint32_t)((int)qh) & 0xffu) << (8 * (i & 3));
        lw[i >> 2] |= ((uint32_t)((int)ql) & 0xffu) << (8 * (i & 3));
      }
      reinterpret_cast<uint2*>(hi + (size_t)r * K)[v] = make_uint2(hw[0], hw[1]);
      reinterpret_cast<uint2*>(lo + (size_t)r * K)[v] = make_uint2(lw[0], lw[1]);
    }
  }
}

// Map a work-item index onto (touched expert, item within that expert).  Experts that received
// no rows own no items.  Returns false when the index is past the last item.
__device__ __forceinline__ bool item_of(const int32_t* __restrict__ offsets, int E, int items_per_expert,
                                        int item, int& e, int& local) {
  int base = 0;
  for (int q = 0; q < E; ++q) {
    if (offsets[q + 1] - offsets[q] <= 0) continue;
    if (item < base + items_per_expert) {
      e = q;
      local = item - base;
      return true;
    }
    base += items_per_expert;
  }
  return false;
}

// One warp: 16 weight rows [o0, o0 + 16) of NMAT matrices (row m of matrix `mat` at
// wbase[mat] + m * ldw bytes) times token rows [r0, r0 + ntok) of the split activation planes
// (`ldx` bytes per row), over K range [kbeg, kend); NT n-blocks of 8 tokens.  acc[m][n][p][4]
// receives the s32 C fragments of plane p (0 = hi, 1 = lo).
template <int NMAT, int NT>
__device__ __forceinline__ void warp_stream(const int8_t* const (&wbase)[NMAT], int ldw,
                                            const int8_t* __restrict__ Xhi, const int8_t* __restrict__ Xlo, int ldx,
                                            int r0, int ntok, int kbeg, int kend, int lane,
                                            int (&acc)[NMAT][NT][2][4]) {
  const int g = lane >> 2, c = lane & 3;
  const int8_t* wrow_g[NMAT];
  const int8_t* wrow_g8[NMAT];
#pragma unroll
  for (int m = 0; m < NMAT; ++m) {
    wrow_g[m] = wbase[m] + (size_t)g * ldw;
    wrow_g8[m] = wbase[m] + (size_t)(g + 8) * ldw;
  }
  size_t xoff[NT];
  bool xv[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int t = n * 8 + g;
    xv[n] = t < ntok;
    xoff[n] = (size_t)(r0 + (xv[n] ? t : 0)) * ldx + 16 * c;
  }
  for (int k0 = kbeg; k0 < kend; k0 += KB) {
    const int nsub = min(4, (kend - k0) >> 6);
    uint4 wl[4][NMAT], wh[4][NMAT];
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      if (sub < nsub) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          wl[sub][m] = ldg_stream(wrow_g[m] + k0 + sub * 64 + 16 * c);
          wh[sub][m] = ldg_stream(wrow_g8[m] + k0 + sub * 64 + 16 * c);
        }
      }
    }
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      if (sub >= nsub) break;
      const int kx = k0 + sub * 64;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        uint4 xh = make_uint4(0u, 0u, 0u, 0u), xl = make_uint4(0u, 0u, 0u, 0u);
        if (xv[n]) {
          xh = *reinterpret_cast<const uint4*>(Xhi + xoff[n] + kx);
          xl = *reinterpret_cast<const uint4*>(Xlo + xoff[n] + kx);
        }
#pragma unroll
        for (int st = 0; st < 2; ++st) {
          const uint32_t bh0 = st ? xh.z : xh.x, bh1 = st ? xh.w : xh.y;
          const uint32_t bl0 = st ? xl.z : xl.x, bl1 = st ? xl.w : xl.y;
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint32_t a0 = st ? wl[sub][m].z : wl[sub][m].x, a2 = st ? wl[sub][m].w : wl[sub][m].y;
            const uint32_t a1 = st ? wh[sub][m].z : wh[sub][m].x, a3 = st ? wh[sub][m].w : wh[sub][m].y;
            mma_s8_16832(acc[m][n][0], a0, a1, a2, a3, bh0, bh1);
            mma_s8_16832(acc[m][n][1], a0, a1, a2, a3, bl0, bl1);
          }
        }
      }
    }
  }
}

// s32 accumulators of the two planes -> fp32 dot product in units of the row scale a
__device__ __forceinline__ float planes(const int (&hl)[2][4], int q) {
  return (float)hl[0][q] + (float)hl[1][q] * (1.0f / 254.0f);
}

// One CTA of 8 warps per SM for the 16- and 32-token variants (their accumulators need the
// registers), two per SM for the 8-token variant.
template <int NT>
__global__ void __launch_bounds__(kWarpsPerCta * 32, NT == 1 ? 2 : 1) dec_gateup_kernel(
    const int8_t* __restrict__ Xhi, const int8_t* __restrict__ Xlo, const float* __restrict__ xscale,
    const int8_t* __restrict__ W, const float* __restrict__ scales, int64_t wstride, int d, int f, int E,
    const int32_t* __restrict__ offsets, __nv_bfloat16* __restrict__ H) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int warp_id = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerCta;
  const int items_per_expert = f / 16;
  for (int item = warp_id;; item += nwarps) {
    int e, local;
    if (!item_of(offsets, E, items_per_expert, item, e, local)) break;
    const int row_base = offsets[e], cnt = offsets[e + 1] - row_base;
    const int o0 = local * 16;
    const int8_t* base = W + (int64_t)e * wstride;
    const int8_t* const wb[2] = {base + (size_t)o0 * d, base + (size_t)f * d + (size_t)o0 * d};
    const float* sc = scales + (int64_t)e * (2 * f + d);
    for (int tc0 = 0; tc0 < cnt; tc0 += NT * 8) {
      const int ntok = min(NT * 8, cnt - tc0);
      int acc[2][NT][2][4] = {};
      warp_stream<2, NT>(wb, d, Xhi, Xlo, d, row_base + tc0, ntok, 0, d, lane, acc);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {  // columns 2c, 2c + 1 (tokens)
          const int tk = n * 8 + 2 * c + cc;
          if (tk >= ntok) continue;
          const int row = row_base + tc0 + tk;
          const float a = xscale[row];
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // output rows g, g + 8
            const int o = o0 + g + 8 * h;
            const float gv = sc[o] * a * planes(acc[0][n], 2 * h + cc);
            const float uv = sc[f + o] * a * planes(acc[1][n], 2 * h + cc);
            H[(size_t)row * f + o] = __float2bfloat16_rn(silu_mul(gv, uv));
          }
        }
      }
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(kWarpsPerCta * 32, NT == 1 ? 2 : 1) dec_down_kernel(
    const int8_t* __restrict__ Hhi, const int8_t* __restrict__ Hlo, const float* __restrict__ hscale,
    const int8_t* __restrict__ W, const float* __restrict__ scales, int64_t wstride, int d, int f, int E,
    const int32_t* __restrict__ offsets, int nsplit, int rows, float* __restrict__ Ypart) {
  const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int warp_id = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * kWarpsPerCta;
  const int groups = d / 16;
  const int items_per_expert = groups * nsplit;
  const int kspan = f / nsplit;
  for (int item = warp_id;; item += nwarps) {
    int e, local;
    if (!item_of(offsets, E, items_per_expert, item, e, local)) break;
    const int split = local / groups, o0 = (local - split * groups) * 16;
    const int row_base = offsets[e], cnt = offsets[e + 1] - row_base;
    const int8_t* base = W + (int64_t)e * wstride + 2 * (size_t)f * d;
    const int8_t* const wb[1] = {base + (size_t)o0 * f};
    const float* s2 = scales + (int64_t)e * (2 * f + d) + 2 * f;
    float* out = Ypart + (size_t)split * rows * d;
    const int kbeg = split * kspan, kend = kbeg + kspan;
    for (int tc0 = 0; tc0 < cnt; tc0 += NT * 8) {
      const int ntok = min(NT * 8, cnt - tc0);
      int acc[1][NT][2][4] = {};
      warp_stream<1, NT>(wb, f, Hhi, Hlo, f, row_base + tc0, ntok, kbeg, kend, lane, acc);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int tk = n * 8 + 2 * c + cc;
          if (tk >= ntok) continue;
          const int row = row_base + tc0 + tk;
          const float a = hscale[row];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int o = o0 + g + 8 * h;
            out[(size_t)row * d + o] = s2[o] * a * planes(acc[0][n], 2 * h + cc);
          }
        }
      }
    }
  }
}

int persistent_ctas(int per_sm) {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms * per_sm;
}

}  // namespace

cudaError_t launch_dec_split(const __nv_bfloat16* X, int R, int K, int8_t* hi, int8_t* lo, float* scale,
                             cudaStream_t s) {
  if (R <= 0) return cudaSuccess;
  const int grid = std::min((R + 7) / 8, 4096);
  dec_split_rows_kernel<<<grid, 256, 0, s>>>(X, R, K, hi, lo, scale);
  return cudaGetLastError();
}

cudaError_t launch_dec_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const int8_t* W,
                              const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                              __nv_bfloat16* H, int max_rows_per_expert, cudaStream_t s) {
  const int grid = persistent_ctas(max_rows_per_expert <= 8 ? 2 : 1);
  const int threads = kWarpsPerCta * 32;
  if (max_rows_per_expert <= 8)
    dec_gateup_kernel<1><<<grid, threads, 0, s>>>(Xhi, Xlo, xscale, W, scales, wstride, d, f, E, offsets, H);
  else if (max_rows_per_expert <= 16)
    dec_gateup_kernel<2><<<grid, threads, 0, s>>>(Xhi, Xlo, xscale, W, scales, wstride, d, f, E, offsets, H);
  else
    dec_gateup_kernel<4><<<grid, threads, 0, s>>>(Xhi, Xlo, xscale, W, scales, wstride, d, f, E, offsets, H);
  return cudaGetLastError();
}

cudaError_t launch_dec_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const int8_t* W,
                            const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                            int nsplit, int rows, float* Ypart, int max_rows_per_expert, cudaStream_t s) {
  const int grid = persistent_ctas(max_rows_per_expert <= 8 ? 2 : 1);
  const int threads = kWarpsPerCta * 32;
  if (max_rows_per_expert <= 8)
    dec_down_kernel<1><<<grid, threads, 0, s>>>(Hhi, Hlo, hscale, W, scales, wstride, d, f, E, offsets, nsplit, rows,
                                                Ypart);
  else if (max_rows_per_expert <= 16)
    dec_down_kernel<2><<<grid, threads, 0, s>>>(Hhi, Hlo, hscale, W, scales, wstride, d, f, E, offsets, nsplit, rows,
                                                Ypart);
  else
    dec_down_kernel<4><<<grid, threads, 0, s>>>(Hhi, Hlo, hscale, W, scales, wstride, d, f, E, offsets, nsplit, rows,
                                                Ypart);
  return cudaGetLastError();
}

}  // namespace colibri
