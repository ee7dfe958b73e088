// Expert Compute stage for int8 weights with per-output-channel fp32 scales, dequantised in
// the kernel (www.0539edu.com/news/4774449 §3.1 stores int8 weights with scales; the scale
// here is per output channel).  For a handful of tokens the layer is a stream over the
// weights of the touched experts, bound by HBM bandwidth, so the design streams each weight
// byte once with 16-byte loads and keeps the arithmetic off the critical path:
//
//   gate/up:  H[r][o]  = silu(s1[o] * sum_i q1[o][i] x[r][i]) * (s3[o] * sum_i q3[o][i] x[r][i])
//   down:     Yp_s[r][o] = s2[o] * sum_{i in split s} q2[o][i] H[r][i]
//
// W[o][i] = s[o] q[o][i], so the scale factors out of each dot product exactly (up to fp32
// rounding).  q in [-127, 127] converts to bf16 exactly; products with bf16 activations run on
// the tensor cores (mma.sync m16n8k16, fp32 accumulation) with the weights as the A operand
// (16 output channels) and up to 32 token rows as four n-blocks of 8.  The down projection is
// split over K into `nsplit` partial sums (written to Ypart, summed in fixed order by the
// combine) so that even one token keeps every SM streaming.
//
// Fragment bookkeeping: for each 64-wide K block a thread (g = lane/4, c = lane%4) loads 16
// consecutive weight bytes [16c, 16c + 16) of rows g and g + 8.  MMA k-step s (0..3) uses
// bytes [16c + 4s, 16c + 4s + 4): its first two as logical k = 2c, 2c+1 and its last two as
// k = 2c+8, 2c+9.  The activation fragment of the same step is read from the same physical
// positions, so the permutation of K inside the block is the same on both operands and the
// dot product is unchanged.
#include "common.cuh"

namespace colibri {
namespace {

constexpr int KC = kDecKC;
constexpr int XPITCH = KC + 8;  // bf16 elements per staged row (16-byte aligned rows)

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Four signed bytes -> two bf16x2 words (bytes 0,1) and (bytes 2,3), exactly: each byte is
// biased to u = q + 128, placed in the mantissa of 2^23 (0x4B0000uu), and 2^23 + 128 is
// subtracted; the result is the integer q as fp32, whose bf16 is its upper half.
__device__ __forceinline__ void i8x4_to_bf16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)) - 8388736.0f;
  const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541)) - 8388736.0f;
  const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)) - 8388736.0f;
  const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543)) - 8388736.0f;
  lo = __byte_perm(__float_as_uint(f0), __float_as_uint(f1), 0x7632);
  hi = __byte_perm(__float_as_uint(f2), __float_as_uint(f3), 0x7632);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stage rows [r0, r0 + ntok) x columns [k0, k0 + kc) of a bf16 matrix into xs (zero padding).
__device__ __forceinline__ void stage_rows(__nv_bfloat16* xs, const __nv_bfloat16* src, int ld, int r0,
                                           int ntok, int k0, int kc) {
  const int vec_per_row = KC / 8;
  for (int q = threadIdx.x; q < kDecTokChunk * vec_per_row; q += blockDim.x) {
    const int r = q / vec_per_row, c8 = (q % vec_per_row) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < ntok && c8 < kc) v = *reinterpret_cast<const uint4*>(src + (size_t)(r0 + r) * ld + k0 + c8);
    *reinterpret_cast<uint4*>(xs + r * XPITCH + c8) = v;
  }
}

// Accumulate over one staged K chunk: `nmat` weight matrices (rows o_g and o_g + 8 of each),
// nb n-blocks of 8 tokens.
template <int NMAT>
__device__ __forceinline__ void mma_chunk(const int8_t* const (&wrow_lo)[NMAT],
                                          const int8_t* const (&wrow_hi)[NMAT], int k0, int kc,
                                          const __nv_bfloat16* xs, int nb, int g, int c,
                                          float (&acc)[NMAT][4][4]) {
#pragma unroll 2
  for (int sub = 0; sub < KC / 64; ++sub) {
    if (sub * 64 >= kc) break;
    uint4 wl[NMAT], wh[NMAT];
#pragma unroll
    for (int m = 0; m < NMAT; ++m) {
      wl[m] = ldg_stream(wrow_lo[m] + k0 + sub * 64 + 16 * c);
      wh[m] = ldg_stream(wrow_hi[m] + k0 + sub * 64 + 16 * c);
    }
#pragma unroll
    for (int st = 0; st < 4; ++st) {
      uint32_t a[NMAT][4];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) {
        const uint32_t lo_w = (&wl[m].x)[st], hi_w = (&wh[m].x)[st];
        i8x4_to_bf16x2x2(lo_w, a[m][0], a[m][2]);
        i8x4_to_bf16x2x2(hi_w, a[m][1], a[m][3]);
      }
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        if (n < nb) {
          const uint2 bv =
              *reinterpret_cast<const uint2*>(xs + (n * 8 + g) * XPITCH + sub * 64 + 16 * c + 4 * st);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) mma_bf16_16816(acc[m][n], a[m][0], a[m][1], a[m][2], a[m][3], bv.x, bv.y);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(128) dec_gateup_kernel(const __nv_bfloat16* __restrict__ Xp,
                                                         const int8_t* __restrict__ W,
                                                         const float* __restrict__ scales,
                                                         int64_t wstride, int d, int f,
                                                         const int32_t* __restrict__ offsets,
                                                         __nv_bfloat16* __restrict__ H) {
  __shared__ __align__(16) __nv_bfloat16 xs[kDecTokChunk * XPITCH];
  const int e = blockIdx.y;
  const int row_base = offsets[e], cnt = offsets[e + 1] - row_base;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int o0 = blockIdx.x * kDecRowsPerCta + warp * 16;
  const bool warp_active = o0 < f;
  const int8_t* base = W + (int64_t)e * wstride;
  const int og = min(o0 + g, f - 1), og8 = min(o0 + g + 8, f - 1);
  const int8_t* const lo[2] = {base + (size_t)og * d, base + (size_t)f * d + (size_t)og * d};
  const int8_t* const hi[2] = {base + (size_t)og8 * d, base + (size_t)f * d + (size_t)og8 * d};
  const float* sc = scales + (int64_t)e * (2 * f + d);
  for (int tc0 = 0; tc0 < cnt; tc0 += kDecTokChunk) {
    const int ntok = min(kDecTokChunk, cnt - tc0);
    const int nb = (ntok + 7) >> 3;
    float acc[2][4][4] = {};
    for (int k0 = 0; k0 < d; k0 += KC) {
      const int kc = min(KC, d - k0);
      __syncthreads();
      stage_rows(xs, Xp, d, row_base + tc0, ntok, k0, kc);
      __syncthreads();
      if (warp_active) mma_chunk<2>(lo, hi, k0, kc, xs, nb, g, c, acc);
    }
    if (warp_active) {
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        if (n >= nb) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {      // rows g, g + 8
          const int o = o0 + g + 8 * h;
          if (o >= f) continue;
          const float s1 = sc[o], s3 = sc[f + o];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {  // columns 2c, 2c + 1
            const int tk = n * 8 + 2 * c + cc;
            if (tk >= ntok) continue;
            const float gv = s1 * acc[0][n][2 * h + cc];
            const float uv = s3 * acc[1][n][2 * h + cc];
            H[(size_t)(row_base + tc0 + tk) * f + o] = __float2bfloat16_rn(silu_mul(gv, uv));
          }
        }
      }
    }
  }
}

__global__ void __launch_bounds__(128) dec_down_kernel(const __nv_bfloat16* __restrict__ H,
                                                       const int8_t* __restrict__ W,
                                                       const float* __restrict__ scales,
                                                       int64_t wstride, int d, int f,
                                                       const int32_t* __restrict__ offsets,
                                                       int nsplit, int rows,
                                                       float* __restrict__ Ypart) {
  __shared__ __align__(16) __nv_bfloat16 xs[kDecTokChunk * XPITCH];
  const int e = blockIdx.y, split = blockIdx.z;
  const int row_base = offsets[e], cnt = offsets[e + 1] - row_base;
  if (cnt <= 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
  const int o0 = blockIdx.x * kDecRowsPerCta + warp * 16;
  const bool warp_active = o0 < d;
  const int kspan = f / nsplit;
  const int kbeg = split * kspan, kend = kbeg + kspan;
  const int8_t* base = W + (int64_t)e * wstride + 2 * (size_t)f * d;
  const int og = min(o0 + g, d - 1), og8 = min(o0 + g + 8, d - 1);
  const int8_t* const lo[1] = {base + (size_t)og * f};
  const int8_t* const hi[1] = {base + (size_t)og8 * f};
  const float* s2 = scales + (int64_t)e * (2 * f + d) + 2 * f;
  float* out = Ypart + (size_t)split * rows * d;
  for (int tc0 = 0; tc0 < cnt; tc0 += kDecTokChunk) {
    const int ntok = min(kDecTokChunk, cnt - tc0);
    const int nb = (ntok + 7) >> 3;
    float acc[1][4][4] = {};
    for (int k0 = kbeg; k0 < kend; k0 += KC) {
      const int kc = min(KC, kend - k0);
      __syncthreads();
      stage_rows(xs, H, f, row_base + tc0, ntok, k0, kc);
      __syncthreads();
      if (warp_active) mma_chunk<1>(lo, hi, k0, kc, xs, nb, g, c, acc);
    }
    if (warp_active) {
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        if (n >= nb) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int o = o0 + g + 8 * h;
          if (o >= d) continue;
          const float s = s2[o];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int tk = n * 8 + 2 * c + cc;
            if (tk >= ntok) continue;
            out[(size_t)(row_base + tc0 + tk) * d + o] = s * acc[0][n][2 * h + cc];
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_dec_gateup(const __nv_bfloat16* Xp, const int8_t* W, const float* scales,
                              int64_t wstride, int d, int f, int E, const int32_t* offsets,
                              __nv_bfloat16* H, cudaStream_t s) {
  const dim3 grid((f + kDecRowsPerCta - 1) / kDecRowsPerCta, E);
  dec_gateup_kernel<<<grid, 128, 0, s>>>(Xp, W, scales, wstride, d, f, offsets, H);
  return cudaGetLastError();
}

cudaError_t launch_dec_down(const __nv_bfloat16* H, const int8_t* W, const float* scales,
                            int64_t wstride, int d, int f, int E, const int32_t* offsets,
                            int nsplit, int rows, float* Ypart, cudaStream_t s) {
  const dim3 grid((d + kDecRowsPerCta - 1) / kDecRowsPerCta, E, nsplit);
  dec_down_kernel<<<grid, 128, 0, s>>>(H, W, scales, wstride, d, f, offsets, nsplit, rows, Ypart);
  return cudaGetLastError();
}

}  // namespace colibri
