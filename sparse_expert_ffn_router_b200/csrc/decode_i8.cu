// Expert Compute stage for int8 weights with per-output-channel fp32 scales, dequantised in
// the kernel (www.0539edu.com/news/4774449 §3.1 stores int8 weights with scales; the scale
// here is per output channel).  For a handful of tokens the layer is a stream over the
// weights of the touched experts, bound by HBM bandwidth:
//
//   gate/up:  H[r][o]    = silu(s1[o] * sum_i q1[o][i] x[r][i]) * (s3[o] * sum_i q3[o][i] x[r][i])
//   down:     Yp_s[r][o] = s2[o] * sum_{i in split s} q2[o][i] H[r][i]
//
// W[o][i] = s[o] q[o][i], so the weight scale factors out of each dot product exactly.  The
// weights are never converted: each activation row (bf16) is split, once, into two int8 planes
// with a scale, x ~= a * (hi + lo / 254) with a = max|x| / 127 (the residual after hi is at most
// a/2, so lo fits in [-127, 127]; the representation error is at most a / 508 = max|x| / 64516
// per element, far below bf16's own rounding of the result).  The token rows x are split by the
// scatter as they are grouped (one scale per row); H is split by dec_finish_h with one scale
// per (row, K range of one down-projection split), the range that one accumulator covers.  The dot
// products then run on the 5th-generation tensor cores as kind::i8 MMAs with exact int32
// accumulation in TMEM: A = 128 weight rows (output channels) x 128 K bytes, B = the hi plane
// rows of up to 32 tokens stacked on their lo plane rows (N = 2 x tokens), so one MMA yields
// both planes.  The epilogue forms s[o] * a * (acc_hi + acc_lo / 254) in fp32.
//
// The stream kernel is persistent, one CTA per SM: warp 0 issues TMA copies of weight tiles
// (128-byte swizzle) and plane tiles into a ring of ~200 KB, warp 1 issues the MMAs, warps 2-5
// run the epilogue from double-buffered accumulators.  Work items (touched expert, 128-row tile
// of output channels, K split, 8/16/32-token chunk) are built on the device from the row
// offsets, so experts that received no rows cost nothing.  The down projection is split over K
// into fp32 partial sums (summed in fixed order by the combine) to spread one token over every
// SM.  Every wait is bounded.
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace colibri {
namespace {

// h = silu(g) * u from the gate/up partials (summed in split order), rounded to bf16 as the bf16
// path stores H, then split into int8 planes.  One CTA per (row, K range of one down split): the
// down projection accumulates each split separately, so each split may carry its own plane
// scale and no reduction crosses CTAs.  The range's bf16 values wait in shared memory between
// the max and the split.
constexpr int kFinishThreads = 256;
constexpr int kFinishMaxSmem = 2 * kDecMaxFF;  // one bf16 row of H
__global__ void __launch_bounds__(kFinishThreads) dec_finish_h_kernel(const float* __restrict__ GU, int gsplit, int R,
                                                                      int f, int dsplit, int8_t* __restrict__ hi,
                                                                      int8_t* __restrict__ lo,
                                                                      float* __restrict__ scale) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t hseg_raw[];  // [span] bf16
  __nv_bfloat16* hseg = reinterpret_cast<__nv_bfloat16*>(hseg_raw);
  __shared__ float red[kFinishThreads / 32];
  const int r = blockIdx.x / dsplit, ds = blockIdx.x - r * dsplit;
  const int span = f / dsplit, k0 = ds * span;
  const size_t plane = (size_t)R * f;
  const float* g0 = GU + (size_t)r * f + k0;
  float mx = 0.f;
  for (int j = threadIdx.x * 4; j < span; j += kFinishThreads * 4) {
    float4 g = __ldg(reinterpret_cast<const float4*>(g0 + j));
    float4 u = __ldg(reinterpret_cast<const float4*>(g0 + plane + j));
#pragma unroll 3
    for (int sp = 1; sp < gsplit; ++sp) {
      const float4 gs = __ldg(reinterpret_cast<const float4*>(g0 + (size_t)(2 * sp) * plane + j));
      const float4 us = __ldg(reinterpret_cast<const float4*>(g0 + (size_t)(2 * sp + 1) * plane + j));
      g.x += gs.x; g.y += gs.y; g.z += gs.z; g.w += gs.w;
      u.x += us.x; u.y += us.y; u.z += us.z; u.w += us.w;
    }
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(silu_mul(g.x, u.x), silu_mul(g.y, u.y));
    const __nv_bfloat162 h23 = __floats2bfloat162_rn(silu_mul(g.z, u.z), silu_mul(g.w, u.w));
    uint2 pk;
    pk.x = (uint32_t)__bfloat16_as_ushort(h01.x) | ((uint32_t)__bfloat16_as_ushort(h01.y) << 16);
    pk.y = (uint32_t)__bfloat16_as_ushort(h23.x) | ((uint32_t)__bfloat16_as_ushort(h23.y) << 16);
    *reinterpret_cast<uint2*>(hseg + j) = pk;
    const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f01.x), fabsf(f01.y)), fmaxf(fabsf(f23.x), fabsf(f23.y))));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int w = 0; w < kFinishThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  const float a = plane_scale(mx), inv_a = __frcp_rn(a);  // correctly rounded 1 / a
  if (threadIdx.x == 0) scale[(size_t)ds * R + r] = a;
  int8_t* hrow = hi + (size_t)r * f + k0;
  int8_t* lrow = lo + (size_t)r * f + k0;
  for (int j = threadIdx.x * 4; j < span; j += kFinishThreads * 4) {
    const uint2 pk = *reinterpret_cast<const uint2*>(hseg + j);
    const float2 f01 = make_float2(__bfloat162float(__ushort_as_bfloat16((unsigned short)(pk.x & 0xffffu))),
                                   __bfloat162float(__ushort_as_bfloat16((unsigned short)(pk.x >> 16))));
    const float2 f23 = make_float2(__bfloat162float(__ushort_as_bfloat16((unsigned short)(pk.y & 0xffffu))),
                                   __bfloat162float(__ushort_as_bfloat16((unsigned short)(pk.y >> 16))));
    int qh0, ql0, qh1, ql1, qh2, ql2, qh3, ql3;
    split_planes(f01.x, a, inv_a, qh0, ql0);
    split_planes(f01.y, a, inv_a, qh1, ql1);
    split_planes(f23.x, a, inv_a, qh2, ql2);
    split_planes(f23.y, a, inv_a, qh3, ql3);
    const uint32_t hw = ((uint32_t)qh0 & 0xffu) | (((uint32_t)qh1 & 0xffu) << 8) | (((uint32_t)qh2 & 0xffu) << 16) |
                        ((uint32_t)qh3 << 24);
    const uint32_t lw = ((uint32_t)ql0 & 0xffu) | (((uint32_t)ql1 & 0xffu) << 8) | (((uint32_t)ql2 & 0xffu) << 16) |
                        ((uint32_t)ql3 << 24);
    *reinterpret_cast<uint32_t*>(hrow + j) = hw;
    *reinterpret_cast<uint32_t*>(lrow + j) = lw;
  }
}

// ------------------------------------------------------------------------- stream kernel
constexpr int kDsThreads = 192;
constexpr int kDsTmemCols = 256;
constexpr size_t kDsRingBytes = 200 * 1024;
constexpr int kDsMaxStages = 12;

struct alignas(64) DecStreamParams {
  CUtensorMap mapW;   // int8 weights: gate/up {d, f, 2, E} (W1, W3); down {f, d, E} (W2)
  CUtensorMap mapHi;  // int8 activation planes {K, R}
  CUtensorMap mapLo;
  const float* wscale;      // expert scales base (per expert: s1[f] | s3[f] | s2[d])
  const float* rscale;      // plane scales: rscale[split * rscale_split_stride + row]
  int rscale_split_stride;  // 0: one scale per row (x planes); R: one per (K split, row) (H planes)
  const int32_t* offsets;   // [E+1]
  int E, d, f;
  int out_rows;             // f (gate/up) or d (down)
  int K, nsplit, kspan;     // kspan: K range of one split (a multiple of 128 unless nsplit == 1)
  int nt8;                  // tokens per chunk (8, 16 or 32); MMA N = 2 * nt8
  int R;                    // rows of the planes (T * k)
  uint32_t stage_bytes;
  int stages;
  float* GU;                // gate/up output: [nsplit, 2, R, f] fp32 partials (W1 . x, W3 . x, scaled)
  float* Ypart;             // down output [nsplit, R, d]
  uint32_t* err;
};

struct DecItem {
  int e, mat, tile, split, chunk, row0, ntok;
};

// Items of one touched expert: (matrix: W1 and W3 for gate/up, W2 for down) x 128-row tiles x
// K splits x token chunks, tile fastest.
template <bool kGateUp>
__device__ __forceinline__ bool dec_item(const DecStreamParams& p, const int32_t* touched, const int32_t* item_prefix,
                                         int ntouched, int L, DecItem& it) {
  if (L >= item_prefix[ntouched]) return false;
  int lo = 0, hi = ntouched - 1;  // largest ti with item_prefix[ti] <= L
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (item_prefix[mid] <= L) lo = mid;
    else hi = mid - 1;
  }
  const int e = touched[lo];
  const int tiles = (p.out_rows + 127) / 128;
  int local = L - item_prefix[lo];
  it.e = e;
  it.tile = local % tiles;
  local /= tiles;
  if (kGateUp) {
    it.mat = local & 1;
    local >>= 1;
  } else {
    it.mat = 0;
  }
  it.split = local % p.nsplit;
  it.chunk = local / p.nsplit;
  const int base = p.offsets[e], cnt = p.offsets[e + 1] - base;
  it.row0 = base + it.chunk * p.nt8;
  it.ntok = min(p.nt8, cnt - it.chunk * p.nt8);
  return true;
}

__device__ __forceinline__ bool ds_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitTimeoutNs) return false;
    }
  }
}

template <bool kGateUp>
__global__ void __launch_bounds__(kDsThreads, 1) dec_stream_kernel(const __grid_constant__ DecStreamParams p) {
  constexpr int NMAT = 1;  // one weight tile per item (W1 and W3 tiles of gate/up are separate items)
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(p.err, kErrWaitTimeout);
    return;
  }
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;    // [2]
  uint64_t* tempty = tfull + 2;   // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int32_t* ntouched_s = reinterpret_cast<int32_t*>(tmem_holder + 2);
  int32_t* issued_s = ntouched_s + 1;   // copies issued / stages consumed, for the error path
  int32_t* consumed_s = ntouched_s + 2;
  int32_t* touched = ntouched_s + 3;             // [E]
  int32_t* item_prefix = touched + kMaxExperts;  // [E + 1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *issued_s = 0;
    *consumed_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&p.mapW);
    tma_prefetch_desc(&p.mapHi);
    tma_prefetch_desc(&p.mapLo);
  }
  // Everything below may read what earlier kernels wrote.  TMEM is allocated only after the
  // wait too: the previous kernel has then released its own columns, so two kernels of the
  // chain never hold TMEM on one SM at the same time.
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(tmem_holder, kDsTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (threadIdx.x == 0) {
    // touched experts and the prefix of their work items
    const int tiles = (p.out_rows + 127) / 128;
    int n = 0, acc = 0;
    for (int e = 0; e < p.E; ++e) {
      const int cnt = p.offsets[e + 1] - p.offsets[e];
      if (cnt <= 0) continue;
      touched[n] = e;
      item_prefix[n] = acc;
      acc += tiles * (kGateUp ? 2 : 1) * p.nsplit * ((cnt + p.nt8 - 1) / p.nt8);
      ++n;
    }
    item_prefix[n] = acc;
    *ntouched_s = n;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int ntouched = *ntouched_s;
  const int N = 2 * p.nt8;
  const uint32_t a_bytes = 128u * 128u;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      const uint32_t tx = NMAT * a_bytes + (uint32_t)N * 128u;
      int issued = 0;
      bool ok = true;
      DecItem it;
      for (int L = blockIdx.x; ok && dec_item<kGateUp>(p, touched, item_prefix, ntouched, L, it); L += gridDim.x) {
        // The item's K blocks start at a rotated block (item index mod block count): items in
        // flight at the same time then read different column offsets of their weight rows, which
        // spreads the requests over the DRAM channels instead of hitting the same address bits
        // everywhere.  The accumulation is exact int32, so the block order does not matter.
        const int kbeg = it.split * p.kspan, kend = min(p.K, kbeg + p.kspan);
        const int nkb = (kend - kbeg + 127) / 128;
        int kb = L % nkb;
        for (int i = 0; i < nkb; ++i, kb = (kb + 1 == nkb) ? 0 : kb + 1) {
          const int kx = kbeg + kb * 128;
          if (!ds_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + (size_t)s * p.stage_bytes;
          mbar_arrive_expect_tx(&full[s], tx);
          if (kGateUp) tma_load_4d(st, &p.mapW, &full[s], kx, it.tile * 128, it.mat, it.e);
          else tma_load_3d(st, &p.mapW, &full[s], kx, it.tile * 128, it.e);
          uint8_t* sb = st + NMAT * a_bytes;
          tma_load_2d(sb, &p.mapHi, &full[s], kx, it.row0);
          tma_load_2d(sb + p.nt8 * 128, &p.mapLo, &full[s], kx, it.row0);
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.err, kErrWaitTimeout);
      }
      *issued_s = issued;
    }
    pdl_trigger();  // every copy of this CTA is issued: let the next kernel be scheduled
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_s8_s32(128, N);
      int s = 0;
      uint32_t ph = 0;
      int iter = 0, consumed = 0;
      bool ok = true;
      DecItem it;
      for (int L = blockIdx.x; ok && dec_item<kGateUp>(p, touched, item_prefix, ntouched, L, it);
           L += gridDim.x, ++iter) {
        const int a = iter & 1;
        const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
        if (!ds_wait(&tempty[a], aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dbase = tmem + (uint32_t)(a * NMAT * N);
        const int kbeg = it.split * p.kspan, kend = min(p.K, kbeg + p.kspan);
        bool first = true;
        for (int kx = kbeg; kx < kend; kx += 128) {
          if (!ds_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + (size_t)s * p.stage_bytes);
          const uint32_t sb = st + NMAT * a_bytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m)
              tc_mma_i8(dbase + (uint32_t)(m * N), smem_desc_sw128(st + m * a_bytes + kk * 32),
                        smem_desc_sw128(sb + kk * 32), idesc, (first && kk == 0) ? 0u : 1u);
          }
          first = false;
          tc_commit(&empty[s]);
          ++consumed;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[a]);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicOr(p.err, kErrWaitTimeout);
      }
      *consumed_s = consumed;
      tc_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    int iter = 0;
    DecItem it;
    for (int L = blockIdx.x; dec_item<kGateUp>(p, touched, item_prefix, ntouched, L, it); L += gridDim.x, ++iter) {
      const int a = iter & 1;
      const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
      const bool got = ds_wait(&tfull[a], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int o = it.tile * 128 + q * 32 + lane;
      const bool vo = o < p.out_rows;
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * NMAT * N);
      const float* es = p.wscale + (size_t)it.e * (2 * p.f + p.d);
      const float sc = vo ? es[(kGateUp ? it.mat * p.f : 2 * p.f) + o] : 0.f;
      // columns [0, nt8) hold the hi plane, [nt8, 2 nt8) the lo plane of the same tokens
      for (int j = 0; j < p.nt8; j += (p.nt8 == 8 ? 8 : 16)) {
        float hi[NMAT][16], lo[NMAT][16];
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          if (p.nt8 == 8) {  // one load: columns 0-7 hi, 8-15 lo
            float v[16];
            tmem_ld16(tb + m * N, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              hi[m][i] = (float)__float_as_int(v[i]);
              lo[m][i] = (float)__float_as_int(v[8 + i]);
            }
          } else {
            float vh[16], vl[16];
            tmem_ld16(tb + m * N + j, vh);
            tmem_ld16(tb + m * N + p.nt8 + j, vl);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              hi[m][i] = (float)__float_as_int(vh[i]);
              lo[m][i] = (float)__float_as_int(vl[i]);
            }
          }
        }
        const int width = p.nt8 == 8 ? 8 : 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = j + i;
          if (i >= width || t >= it.ntok || !vo) continue;
          const int row = it.row0 + t;
          const float v = sc * p.rscale[(size_t)it.split * p.rscale_split_stride + row] *
                          (hi[0][i] + lo[0][i] * (1.0f / 254.0f));
          if (kGateUp) p.GU[(((size_t)it.split * 2 + it.mat) * p.R + row) * p.f + o] = v;
          else p.Ypart[((size_t)it.split * p.R + row) * p.d + o] = v;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // copies issued but never consumed: wait (bounded) until they land before the CTA exits
    for (int i = *consumed_s; i < *issued_s; ++i) mbar_wait_bounded(&full[i % S], (uint32_t)(i / S) & 1u);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDsTmemCols);
  }
}

int dec_nt8(int max_rows_per_expert) { return max_rows_per_expert <= 8 ? 8 : (max_rows_per_expert <= 16 ? 16 : 32); }

int sm_count_current() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

template <bool kGateUp>
cudaError_t launch_stream(DecStreamParams& p, const int8_t* hi, const int8_t* lo, int K, cudaStream_t s) {
  constexpr int NMAT = 1;
  const uint64_t pd[2] = {(uint64_t)K, (uint64_t)p.R}, ps[1] = {(uint64_t)K};
  const uint32_t pb[2] = {128, (uint32_t)p.nt8};
  if (!make_tmap(&p.mapHi, CU_TENSOR_MAP_DATA_TYPE_UINT8, hi, 2, pd, ps, pb)) return cudaErrorInvalidValue;
  if (!make_tmap(&p.mapLo, CU_TENSOR_MAP_DATA_TYPE_UINT8, lo, 2, pd, ps, pb)) return cudaErrorInvalidValue;
  p.stage_bytes = (uint32_t)(NMAT * 128 * 128 + 2 * p.nt8 * 128);
  p.stages = (int)std::min<size_t>(kDsMaxStages, kDsRingBytes / p.stage_bytes);
  const size_t smem = (size_t)p.stages * p.stage_bytes + 4096;
  return launch_kernel(dec_stream_kernel<kGateUp>, dim3(sm_count_current()), dim3(kDsThreads), smem, s, 1, p);
}

}  // namespace

cudaError_t configure_dec_kernels() {
  const int smem = (int)(kDsRingBytes + 4096);
  cudaError_t e = cudaFuncSetAttribute(dec_stream_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_stream_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_finish_h_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFinishMaxSmem);
  return e;
}

cudaError_t launch_dec_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const int8_t* W,
                              const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                              int nsplit, float* GU, int R, int max_rows_per_expert, uint32_t* err, cudaStream_t s) {
  DecStreamParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)f, 2, (uint64_t)E};
  const uint64_t st[3] = {(uint64_t)d, (uint64_t)f * d, (uint64_t)wstride};
  const uint32_t box[4] = {128, 128, 1, 1};
  if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, 4, dims, st, box)) return cudaErrorInvalidValue;
  p.wscale = scales;
  p.rscale = xscale;
  p.offsets = offsets;
  p.E = E;
  p.d = d;
  p.f = f;
  p.out_rows = f;
  p.K = d;
  p.nsplit = nsplit;
  p.kspan = d / nsplit;
  p.nt8 = dec_nt8(max_rows_per_expert);
  p.R = R;
  p.GU = GU;
  p.err = err;
  return launch_stream<true>(p, Xhi, Xlo, d, s);
}

cudaError_t launch_dec_finish_h(const float* GU, int gsplit, int R, int f, int dsplit, int8_t* hi, int8_t* lo,
                                float* scale, cudaStream_t s) {
  if (R <= 0) return cudaSuccess;
  if (dsplit < 1 || f % dsplit != 0 || (f / dsplit) % 4 != 0) return cudaErrorInvalidValue;
  const size_t smem = (size_t)(f / dsplit) * sizeof(__nv_bfloat16);
  if (smem > (size_t)kFinishMaxSmem) return cudaErrorInvalidValue;
  return launch_kernel(dec_finish_h_kernel, dim3((unsigned)((size_t)R * dsplit)), dim3(kFinishThreads), smem, s, 1, GU,
                       gsplit, R, f, dsplit, hi, lo, scale);
}

cudaError_t launch_dec_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const int8_t* W,
                            const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                            int nsplit, int R, float* Ypart, int max_rows_per_expert, uint32_t* err,
                            cudaStream_t s) {
  DecStreamParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t dims[3] = {(uint64_t)f, (uint64_t)d, (uint64_t)E};
  const uint64_t st[2] = {(uint64_t)f, (uint64_t)wstride};
  const uint32_t box[3] = {128, 128, 1};
  if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W + 2 * (size_t)f * d, 3, dims, st, box))
    return cudaErrorInvalidValue;
  p.wscale = scales;
  p.rscale = hscale;
  p.rscale_split_stride = R;
  p.offsets = offsets;
  p.E = E;
  p.d = d;
  p.f = f;
  p.out_rows = d;
  p.K = f;
  p.nsplit = nsplit;
  p.kspan = f / nsplit;
  p.nt8 = dec_nt8(max_rows_per_expert);
  p.R = R;
  p.Ypart = Ypart;
  p.err = err;
  return launch_stream<false>(p, Hhi, Hlo, f, s);
}

}  // namespace colibri
