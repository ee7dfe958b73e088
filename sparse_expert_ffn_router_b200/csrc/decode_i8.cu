// Expert Compute stage for int8 weights with fp32 scales, dequantised in the kernel
// (www.0539edu.com/news/4774449 §3.1 stores int8 weights with a scale per weight matrix; the
// default here is one scale per output channel, the per-matrix layout is an option).  For a
// handful of tokens the layer is a stream over the weights of the touched experts, bound by HBM
// bandwidth:
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
//
// dec_fused_kernel runs the whole stage (for up to 64 tokens also the router, top-k and the
// grouping) as one cooperative launch whose phases are separated by grid barriers; the four
// separate kernels (dec_stream_kernel twice, dec_finish_h_kernel, and the combine) remain as the
// plan taken when the fused launch is turned off.
#include <algorithm>
#include <cstdlib>
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

// ------------------------------------------------------------------------- stream kernels
constexpr int kDsThreads = 192;
constexpr int kDsTmemCols = 256;
constexpr size_t kDsRingBytes = 200 * 1024;
constexpr int kDsMaxStages = 12;
constexpr int kDsMaxKbs = 4;

struct alignas(64) DecStreamParams {
  CUtensorMap mapW;   // int8 weights: gate/up {d, f, 2, E} (W1, W3); down {f, d, E} (W2)
  CUtensorMap mapHi;  // int8 activation planes {K, R}
  CUtensorMap mapLo;
  const float* wscale;      // expert scales: per expert s1[f] | s3[f] | s2[d], or [E][3] per matrix
  int scale_per_matrix;     // 1: one scale per weight matrix (W1, W3, W2) of each expert
  const float* rscale;      // plane scales: rscale[split * rscale_split_stride + row]
  int rscale_split_stride;  // 0: one scale per row (x planes); R: one per (K split, row) (H planes)
  const int32_t* offsets;   // [E+1]
  int E, d, f;
  int out_rows;             // f (gate/up) or d (down)
  int K, nsplit, kspan;     // kspan: K range of one split (a multiple of 128 unless nsplit == 1)
  int nt8;                  // tokens per chunk (8, 16 or 32); MMA N = 2 * nt8
  int R;                    // rows of the planes (T * k)
  int kbs;                  // 128-byte K blocks per ring stage (1..kDsMaxKbs)
  int evict_first;          // weight copies with an L2 evict-first policy (read once)
  uint32_t stage_bytes;     // kbs x (weight tile 128 x 128 + planes 2 nt8 x 128)
  int stages;
  float* GU;                // gate/up output: [nsplit, 2, R, f] fp32 partials (W1 . x, W3 . x, scaled)
  float* Ypart;             // down output [nsplit, R, d]
  uint32_t* err;
};

struct DecItem {
  int e, mat, tile, split, chunk, row0, ntok;
  int gchunk;  // chunk number over all touched experts
};

// Shared-memory control block of the stream kernels (after the ring).
struct DsCtl {
  uint64_t full[kDsMaxStages];
  uint64_t empty[kDsMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem;
  int abort;
  int issued;    // copies issued / stages consumed, for the error path
  int consumed;
  int flag;      // result of a grid-wide wait, broadcast to the epilogue warps
  int hpass;     // fused kernel: 1 once the epilogue warps passed the H barrier, -1 if it failed
  int first;     // this CTA's first work item (items first, first + gridDim.x, ...)
  int ntouched;
  int32_t off[kMaxExperts + 1];     // row offsets of the experts' groups
  int32_t touched[kMaxExperts];
  int32_t pre[2][kMaxExperts + 1];  // item prefix over the touched experts: [0] gate/up, [1] down
  int32_t cpre[kMaxExperts + 1];    // token-chunk prefix over the touched experts (chunk numbers)
  int32_t defer_row[kDsMaxStages];  // fused kernel: down stages whose plane copies wait for H
  int32_t defer_kx[kDsMaxStages][kDsMaxKbs];
  int32_t defer_nk[kDsMaxStages];
  int32_t defer_s[kDsMaxStages];
  float red[4];                     // fused kernel: per-warp maxima of the H pass
};
constexpr size_t kDsCtlBytes = 8192;
static_assert(sizeof(DsCtl) <= kDsCtlBytes, "stream-kernel control block");


// Items of one touched expert: (matrix: W1 and W3 for gate/up, W2 for down) x 128-row tiles x
// K splits x token chunks, tile fastest.
template <bool kGateUp, typename Ctl>
__device__ __forceinline__ bool dec_item(const DecStreamParams& p, const Ctl& c, int pre_idx, int L, DecItem& it) {
  const int32_t* item_prefix = c.pre[pre_idx];
  const int32_t* touched = c.touched;
  const int32_t* off = c.off;
  const int ntouched = c.ntouched;
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
  const int base = off[e], cnt = off[e + 1] - base;
  it.row0 = base + it.chunk * p.nt8;
  it.ntok = min(p.nt8, cnt - it.chunk * p.nt8);
  it.gchunk = c.cpre[lo] + it.chunk;
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

template <typename Ctl>
__device__ __forceinline__ void ds_abort(Ctl& c, uint32_t* err) {
  *(volatile int*)&c.abort = 1;
  atomicOr(err, kErrWaitTimeout);
}

// Ring position shared by the phases a role walks through.
struct DsRing {
  int s = 0;
  uint32_t ph = 0;
  int n = 0;  // copies issued (producer) or stages consumed (MMA)
  __device__ void advance(int S) {
    ++n;
    if (++s == S) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// Plane copies of K block j of a stage (hi rows, then lo rows of the same tokens).
__device__ __forceinline__ void ds_load_planes(const DecStreamParams& p, uint8_t* stage, uint64_t* full, int j, int kx,
                                               int row0) {
  uint8_t* sb = stage + (size_t)p.kbs * 128 * 128 + (size_t)j * (2 * p.nt8 * 128);
  tma_load_2d(sb, &p.mapHi, full, kx, row0);
  tma_load_2d(sb + p.nt8 * 128, &p.mapLo, full, kx, row0);
}

// Producer: every stage of one phase.  A stage carries kbs consecutive K blocks of one item, so
// each weight row is read kbs x 128 contiguous bytes at a time.  With `defer` the plane copies of
// the first ring-full of stages are held back (their weight copies go out at once) until
// `ready()` returns true.
template <bool kGateUp, typename Ready>
__device__ bool ds_produce(const DecStreamParams& p, uint8_t* smem, DsCtl& c, int S, int pre_idx, DsRing& r,
                           bool defer, Ready ready) {
  const uint32_t blk_bytes = 128u * 128u + (uint32_t)(2 * p.nt8) * 128u;
  const uint64_t policy = l2_evict_first_policy();
  int held = 0;
  bool released = !defer;
  auto release = [&]() {
    for (int h = 0; h < held; ++h) {
      uint8_t* st = smem + (size_t)c.defer_s[h] * p.stage_bytes;
      for (int j = 0; j < c.defer_nk[h]; ++j)
        ds_load_planes(p, st, &c.full[c.defer_s[h]], j, c.defer_kx[h][j], c.defer_row[h]);
    }
  };
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, pre_idx, L, it); L += gridDim.x) {
    // The item's K blocks start at a rotated block (item index mod block count): items in flight
    // at the same time then read different column offsets of their weight rows, which spreads
    // the requests over the DRAM channels instead of hitting the same address bits everywhere.
    // The accumulation is exact int32, so the block order does not matter.
    const int kbeg = it.split * p.kspan, kend = min(p.K, kbeg + p.kspan);
    const int nkb = (kend - kbeg + 127) / 128;
    int kb = L % nkb;
    for (int i = 0; i < nkb; i += p.kbs) {
      const int nk = min(p.kbs, nkb - i);
      if (!ds_wait(&c.empty[r.s], r.ph ^ 1u, &c.abort)) return false;
      uint8_t* st = smem + (size_t)r.s * p.stage_bytes;
      mbar_arrive_expect_tx(&c.full[r.s], (uint32_t)nk * blk_bytes);
      for (int j = 0; j < nk; ++j, kb = (kb + 1 == nkb) ? 0 : kb + 1) {
        const int kx = kbeg + kb * 128;
        uint8_t* sw = st + (size_t)j * 128 * 128;
        if (p.evict_first) {
          if (kGateUp) tma_load_4d_hint(sw, &p.mapW, &c.full[r.s], kx, it.tile * 128, it.mat, it.e, policy);
          else tma_load_3d_hint(sw, &p.mapW, &c.full[r.s], kx, it.tile * 128, it.e, policy);
        } else {
          if (kGateUp) tma_load_4d(sw, &p.mapW, &c.full[r.s], kx, it.tile * 128, it.mat, it.e);
          else tma_load_3d(sw, &p.mapW, &c.full[r.s], kx, it.tile * 128, it.e);
        }
        if (released) ds_load_planes(p, st, &c.full[r.s], j, kx, it.row0);
        else c.defer_kx[held][j] = kx;
      }
      if (!released) {
        c.defer_row[held] = it.row0;
        c.defer_nk[held] = nk;
        c.defer_s[held] = r.s;
        if (++held == S) {
          // The ring is full of weight copies and the planes are not ready yet.  (Pulling the
          // next weight blocks into L2 meanwhile measured slower: the extra requests delayed the
          // last items of the other CTAs and the grid barrier behind them.)
          // The held plane copies are issued even when the wait gave up, so that every issued
          // stage completes and the error path drains quickly
          const bool go = ready();
          release();
          if (!go) return false;
          released = true;
        }
      }
      c.issued = r.n + 1;
      r.advance(S);
    }
  }
  if (!released && held > 0) {
    const bool go = ready();
    release();
    if (!go) return false;
  }
  return true;
}

// MMA issuer: every item of one phase (A = 128 weight rows, B = hi rows stacked on lo rows).
template <bool kGateUp>
__device__ bool ds_mma(const DecStreamParams& p, uint8_t* smem, DsCtl& c, int S, int pre_idx, DsRing& r, int& iter,
                       uint32_t tmem) {
  const int N = 2 * p.nt8;
  const uint32_t idesc = idesc_s8_s32(128, N);
  const uint32_t plane_bytes = (uint32_t)(2 * p.nt8 * 128);
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, pre_idx, L, it);
       L += gridDim.x, ++iter) {
    const int a = iter & 1;
    const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
    if (!ds_wait(&c.tempty[a], aph ^ 1u, &c.abort)) return false;
    tc_fence_after();
    const uint32_t dbase = tmem + (uint32_t)(a * N);
    const int kbeg = it.split * p.kspan, kend = min(p.K, kbeg + p.kspan);
    const int nkb = (kend - kbeg + 127) / 128;
    bool first = true;
    for (int i = 0; i < nkb; i += p.kbs) {
      const int nk = min(p.kbs, nkb - i);
      if (!ds_wait(&c.full[r.s], r.ph, &c.abort)) return false;
      tc_fence_after();
      const uint32_t st = smem_u32(smem + (size_t)r.s * p.stage_bytes);
      const uint32_t sb = st + (uint32_t)p.kbs * 128u * 128u;
      for (int j = 0; j < nk; ++j) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          tc_mma_i8(dbase, smem_desc_sw128(st + j * 128u * 128u + kk * 32),
                    smem_desc_sw128(sb + j * plane_bytes + kk * 32), idesc, first ? 0u : 1u);
          first = false;
        }
      }
      tc_commit(&c.empty[r.s]);
      c.consumed = r.n + 1;
      r.advance(S);
    }
    tc_commit(&c.tfull[a]);
  }
  return true;
}

struct NoItemHook {
  __device__ bool operator()(const DecItem&, bool ok) const { return ok; }
};

// Epilogue (warps 2..5): every item of one phase; writes the scaled fp32 partial sums.  `after`
// runs in all four warps once an item's sums are written and its accumulator is released, and
// also when a warp's wait for the accumulator gave up (ok = false, with the CTA's abort flag set
// first), so that a hook that synchronises the four warps is reached by all of them for the same
// item; it returns false to stop the phase.
template <bool kGateUp, typename After = NoItemHook>
__device__ bool ds_epilogue(const DecStreamParams& p, DsCtl& c, int pre_idx, int& iter, uint32_t tmem, int warp,
                            int lane, After after = After()) {
  const int q = warp & 3;
  const int N = 2 * p.nt8;
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, pre_idx, L, it);
       L += gridDim.x, ++iter) {
    const int a = iter & 1;
    const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
    // the weight scale is an input of the call: loaded before the accumulator is waited for
    const int o = it.tile * 128 + q * 32 + lane;
    const bool vo = o < p.out_rows;
    const int m = kGateUp ? it.mat : 2;  // W1, W3 or W2
    const float* sp = p.scale_per_matrix ? p.wscale + (size_t)it.e * 3 + m
                                         : p.wscale + (size_t)it.e * (2 * p.f + p.d) + (size_t)m * p.f + o;
    const float sc = vo ? __ldg(sp) : 0.f;
    const bool got = ds_wait(&c.tfull[a], aph, &c.abort);
    if (!__all_sync(0xffffffffu, got)) {
      if (lane == 0) *(volatile int*)&c.abort = 1;
      __syncwarp();
      after(it, false);
      return false;
    }
    tc_fence_after();
    const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * N);
    // columns [0, nt8) hold the hi plane, [nt8, 2 nt8) the lo plane of the same tokens
    for (int j = 0; j < p.nt8; j += (p.nt8 == 8 ? 8 : 16)) {
      float hi[16], lo[16];
      if (p.nt8 == 8) {  // one load: columns 0-7 hi, 8-15 lo
        float v[16];
        tmem_ld16(tb, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hi[i] = (float)__float_as_int(v[i]);
          lo[i] = (float)__float_as_int(v[8 + i]);
        }
      } else {
        float vh[16], vl[16];
        tmem_ld16(tb + j, vh);
        tmem_ld16(tb + p.nt8 + j, vl);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          hi[i] = (float)__float_as_int(vh[i]);
          lo[i] = (float)__float_as_int(vl[i]);
        }
      }
      const int width = p.nt8 == 8 ? 8 : 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = j + i;
        if (i >= width || t >= it.ntok || !vo) continue;
        const int row = it.row0 + t;
        const float v = sc * __ldcg(p.rscale + (size_t)it.split * p.rscale_split_stride + row) *
                        (hi[i] + lo[i] * (1.0f / 254.0f));
        if (kGateUp) p.GU[(((size_t)it.split * 2 + it.mat) * p.R + row) * p.f + o] = v;
        else p.Ypart[((size_t)it.split * p.R + row) * p.d + o] = v;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.tempty[a]);
    if (!after(it, true)) return false;
  }
  return true;
}

// Barriers, descriptor prefetch, then (after the grid dependency wait) TMEM.
__device__ __forceinline__ void ds_init(const DecStreamParams* const* phases, int nphases, DsCtl& c, int S) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&c.tfull[a], 1);
      mbar_init(&c.tempty[a], 4);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    c.issued = 0;
    c.consumed = 0;
    c.flag = 0;
    c.hpass = 0;
    c.first = blockIdx.x;
    mbar_fence_init();
    for (int i = 0; i < nphases; ++i) {
      tma_prefetch_desc(&phases[i]->mapW);
      tma_prefetch_desc(&phases[i]->mapHi);
      tma_prefetch_desc(&phases[i]->mapLo);
    }
  }
  // Everything below may read what earlier kernels wrote.  TMEM is allocated only after the
  // wait too: the previous kernel has then released its own columns, so two kernels of the
  // chain never hold TMEM on one SM at the same time.
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(&c.tmem, kDsTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
}

// The experts' row offsets (from global memory, or already in c.off when `offsets` is NULL),
// the touched experts and the prefix of their work items per phase.
template <typename Ctl>
__device__ __forceinline__ void ds_items(const DecStreamParams* const* phases, int nphases, Ctl& c,
                                         const int32_t* offsets) {
  const int E = phases[0]->E;
  if (offsets)
    for (int e = threadIdx.x; e <= E; e += blockDim.x) c.off[e] = offsets[e];
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    int acc[2] = {0, 0};
    int chunks = 0;
    for (int e = 0; e < E; ++e) {
      const int cnt = c.off[e + 1] - c.off[e];
      if (cnt <= 0) continue;
      c.touched[n] = e;
      c.cpre[n] = chunks;
      chunks += (cnt + phases[0]->nt8 - 1) / phases[0]->nt8;
      for (int i = 0; i < nphases; ++i) {
        const DecStreamParams& p = *phases[i];
        const bool gateup = p.GU != nullptr;
        c.pre[i][n] = acc[i];
        acc[i] += (p.out_rows + 127) / 128 * (gateup ? 2 : 1) * p.nsplit * ((cnt + p.nt8 - 1) / p.nt8);
      }
      ++n;
    }
    for (int i = 0; i < nphases; ++i) c.pre[i][n] = acc[i];
    c.cpre[n] = chunks;
    c.ntouched = n;
  }
  __syncthreads();
  tc_fence_after();
}

// Copies issued but never consumed (error path): wait (bounded) until they land; then free TMEM.
__device__ __forceinline__ void ds_teardown(DsCtl& c, int S) {
  __syncthreads();
  if (threadIdx.x == 0 && c.abort) {
    for (int i = c.consumed; i < c.issued; ++i)
      if (!mbar_wait_bounded(&c.full[i % S], (uint32_t)(i / S) & 1u)) break;
  }
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(c.tmem, kDsTmemCols);
  }
}

template <bool kGateUp>
__global__ void __launch_bounds__(kDsThreads, 1) dec_stream_kernel(const __grid_constant__ DecStreamParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(p.err, kErrWaitTimeout);
    return;
  }
  const int S = p.stages;
  DsCtl& c = *reinterpret_cast<DsCtl*>(smem + (size_t)S * p.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DecStreamParams* phases[1] = {&p};
  ds_init(phases, 1, c, S);
  ds_items(phases, 1, c, p.offsets);
  const uint32_t tmem = c.tmem;
  if (warp == 0) {
    if (lane == 0) {
      DsRing r;
      if (!ds_produce<kGateUp>(p, smem, c, S, 0, r, false, [] { return true; })) ds_abort(c, p.err);
    }
    pdl_trigger();  // every copy of this CTA is issued: let the next kernel be scheduled
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      DsRing r;
      int iter = 0;
      if (!ds_mma<kGateUp>(p, smem, c, S, 0, r, iter, tmem)) ds_abort(c, p.err);
      tc_commit(&c.drain);  // wait until every MMA issued by this thread has completed
      mbar_wait_bounded(&c.drain, 0);
    }
    __syncwarp();
  } else {
    int iter = 0;
    if (!ds_epilogue<kGateUp>(p, c, 0, iter, tmem, warp, lane) && lane == 0) ds_abort(c, p.err);
  }
  ds_teardown(c, S);
}

// ------------------------------------------------------------------------- int4 stream kernel
// Group-wise int4 weights (www.mhpq.cn/news/563172 §4.2: INT4 packed in INT32, groups of 128
// inputs; www.trdm.cn/news/555962 §6.1: two 4-bit weights per byte, split apart at compute time):
//
//   W[o][i] = s[i / 128][o] * q[o][i],  q in [-8, 7] two's complement, element 2j in the low
//   nibble of byte j;  y[o] = sum_g s[g][o] * (sum_{i in g} q[o][i] x[i])
//
// The stream is the int8 one with two changes.  The packed tiles (128 rows x 64 bytes = one
// 128-wide K block) arrive unswizzled; converter warps widen them to int8, values unchanged, in
// the 128-byte swizzled layout of the MMA's A operand, so the MMA is the same exact kind::i8
// product against the activation planes.  And since every K block is one scale group, each K
// block accumulates into an accumulator of its own (a ring of kD4Bufs in TMEM) that the epilogue
// reads at once, scales by its group scale and adds into fp32 registers.
//
// Shared memory: kD4Slots widened A tiles (16 KB each), then the TMA ring whose stages hold the
// packed tiles and the plane tiles of kbs K blocks (so that the bytes in flight are packed ones).
// Warps: 0 TMA producer, 1 MMA issuer, 2-5 epilogue, 6-9 converters (one per SM sub-partition).
constexpr int kD4Threads = 320;
constexpr int kD4Bufs = 8;
constexpr int kD4Slots = 4;
constexpr int kD4RawBytes = 128 * 64;  // packed tile: 128 rows x 128 int4
constexpr size_t kD4SlotBytes = (size_t)kD4Slots * 128 * 128;

struct D4Ctl {
  uint64_t raw[kDsMaxStages];    // packed tiles landed (TMA bytes)
  uint64_t full[kDsMaxStages];   // plane tiles landed (TMA bytes)
  uint64_t empty[kDsMaxStages];  // stage free again (MMA commit)
  uint64_t afull[kD4Slots];      // widened A tile written (four converter warps)
  uint64_t aempty[kD4Slots];     // widened A tile read (MMA commit)
  uint64_t tfull[kD4Bufs];       // one K block's accumulator complete (MMA commit)
  uint64_t tempty[kD4Bufs];      // that accumulator read (four epilogue warps)
  uint64_t drain;
  uint32_t tmem;
  int abort;
  int issued;    // stages issued / consumed, for the error path
  int consumed;
  int first;
  int ntouched;
  int32_t off[kMaxExperts + 1];
  int32_t touched[kMaxExperts];
  int32_t pre[2][kMaxExperts + 1];
  int32_t cpre[kMaxExperts + 1];
};
static_assert(sizeof(D4Ctl) <= kDsCtlBytes, "int4 stream control block");

// One stage: plane tiles of its kbs K blocks, then their packed weight tiles.
__device__ __forceinline__ uint32_t d4_plane_bytes(const DecStreamParams& p) { return (uint32_t)(2 * p.nt8) * 128u; }
__device__ __forceinline__ uint8_t* d4_raw(const DecStreamParams& p, uint8_t* stage, int j) {
  return stage + (size_t)p.kbs * d4_plane_bytes(p) + (size_t)j * kD4RawBytes;
}

// Widen one packed word (8 int4, element 2j in the low nibble of byte j) to 8 int8 in order.
__device__ __forceinline__ uint2 widen_int4x8(uint32_t w) {
  // nibbles biased by 8 (q + 8 in [0, 15]), even elements in lo, odd elements in hi
  const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
  const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
  uint32_t a = __byte_perm(lo, hi, 0x5140);  // elements 0..3
  uint32_t b = __byte_perm(lo, hi, 0x7362);  // elements 4..7
  // per byte: (u + 0x78) ^ 0x80 = u - 8 (mod 256), no carry between bytes since u + 0x78 <= 0x87
  a = (a + 0x78787878u) ^ 0x80808080u;
  b = (b + 0x78787878u) ^ 0x80808080u;
  return make_uint2(a, b);
}

// The K blocks of an item, in the rotated order every role walks them.
struct D4Walk {
  int kbeg, nkb;
  __device__ D4Walk(const DecStreamParams& p, const DecItem& it) {
    kbeg = it.split * p.kspan;
    const int kend = min(p.K, kbeg + p.kspan);
    nkb = (kend - kbeg + 127) / 128;
  }
};

template <bool kGateUp>
__device__ bool d4_produce(const DecStreamParams& p, uint8_t* ring, D4Ctl& c, int S) {
  const uint32_t pb = d4_plane_bytes(p);
  const uint64_t policy = l2_evict_first_policy();
  DsRing r;
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, 0, L, it); L += gridDim.x) {
    const D4Walk w(p, it);
    int kb = L % w.nkb;
    for (int i = 0; i < w.nkb; i += p.kbs) {
      const int nk = min(p.kbs, w.nkb - i);
      if (!ds_wait(&c.empty[r.s], r.ph ^ 1u, &c.abort)) return false;
      uint8_t* st = ring + (size_t)r.s * p.stage_bytes;
      mbar_arrive_expect_tx(&c.raw[r.s], (uint32_t)nk * kD4RawBytes);
      mbar_arrive_expect_tx(&c.full[r.s], (uint32_t)nk * pb);
      for (int j = 0; j < nk; ++j, kb = (kb + 1 == w.nkb) ? 0 : kb + 1) {
        const int kx = w.kbeg + kb * 128;  // K element; the packed tile starts at byte kx / 2
        uint8_t* rw = d4_raw(p, st, j);
        if (kGateUp) tma_load_4d_hint(rw, &p.mapW, &c.raw[r.s], kx / 2, it.tile * 128, it.mat, it.e, policy);
        else tma_load_3d_hint(rw, &p.mapW, &c.raw[r.s], kx / 2, it.tile * 128, it.e, policy);
        uint8_t* pl = st + (size_t)j * pb;
        tma_load_2d(pl, &p.mapHi, &c.full[r.s], kx, it.row0);
        tma_load_2d(pl + p.nt8 * 128, &p.mapLo, &c.full[r.s], kx, it.row0);
      }
      c.issued = r.n + 1;
      r.advance(S);
    }
  }
  return true;
}

// Converter warps (warp cw = 0..3 of them): every K block, packed tile -> widened A tile in the
// next slot.  Each warp waits for itself (warp-uniform decisions, no barrier between the warps)
// and arrives on the slot's barrier once its share is written.
template <bool kGateUp>
__device__ bool d4_convert(const DecStreamParams& p, uint8_t* slots, uint8_t* ring, D4Ctl& c, int S, int cw, int lane) {
  DsRing r;
  uint32_t ka = 0;  // K blocks converted (slot ring position)
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, 0, L, it); L += gridDim.x) {
    const D4Walk w(p, it);
    for (int i = 0; i < w.nkb; i += p.kbs) {
      const int nk = min(p.kbs, w.nkb - i);
      if (!__all_sync(0xffffffffu, ds_wait(&c.raw[r.s], r.ph, &c.abort))) return false;
      uint8_t* st = ring + (size_t)r.s * p.stage_bytes;
      for (int j = 0; j < nk; ++j, ++ka) {
        const uint32_t a = ka % kD4Slots, aph = (ka / kD4Slots) & 1u;
        if (!__all_sync(0xffffffffu, ds_wait(&c.aempty[a], aph ^ 1u, &c.abort))) return false;
        const uint8_t* rw = d4_raw(p, st, j);
        uint8_t* at = slots + (size_t)a * 128 * 128;
        // this warp's 32 rows; a task is (row, 16-byte output chunk), so one instruction of the
        // warp reads 256 contiguous packed bytes (4 rows) and writes 4 whole swizzled rows.  All
        // eight packed loads are issued before the first store (a store may not be passed by a
        // later load the compiler cannot prove disjoint from it).
        uint2 v[8];
#pragma unroll
        for (int t8 = 0; t8 < 8; ++t8) {
          const int row = cw * 32 + t8 * 4 + (lane >> 3), ch = lane & 7;
          v[t8] = *reinterpret_cast<const uint2*>(rw + row * 64 + ch * 8);
        }
#pragma unroll
        for (int t8 = 0; t8 < 8; ++t8) {
          const int row = cw * 32 + t8 * 4 + (lane >> 3), ch = lane & 7;
          const uint2 e0 = widen_int4x8(v[t8].x), e1 = widen_int4x8(v[t8].y);
          *reinterpret_cast<uint4*>(at + row * 128 + ((ch ^ (row & 7)) << 4)) = make_uint4(e0.x, e0.y, e1.x, e1.y);
        }
        // the tensor core reads the tile through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.afull[a]);
      }
      r.advance(S);
    }
  }
  return true;
}

template <bool kGateUp>
__device__ bool d4_mma(const DecStreamParams& p, uint8_t* slots, uint8_t* ring, D4Ctl& c, int S, uint32_t tmem) {
  const int N = 2 * p.nt8;
  const uint32_t idesc = idesc_s8_s32(128, N);
  const uint32_t pb = d4_plane_bytes(p);
  DsRing r;
  uint32_t kc = 0;  // K blocks issued (slot and accumulator ring position)
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, 0, L, it); L += gridDim.x) {
    const D4Walk w(p, it);
    for (int i = 0; i < w.nkb; i += p.kbs) {
      const int nk = min(p.kbs, w.nkb - i);
      if (!ds_wait(&c.full[r.s], r.ph, &c.abort)) return false;
      const uint32_t st = smem_u32(ring + (size_t)r.s * p.stage_bytes);
      for (int j = 0; j < nk; ++j, ++kc) {
        const uint32_t a = kc % kD4Slots, aph = (kc / kD4Slots) & 1u;
        const uint32_t b = kc % kD4Bufs, bph = (kc / kD4Bufs) & 1u;
        if (!ds_wait(&c.afull[a], aph, &c.abort) || !ds_wait(&c.tempty[b], bph ^ 1u, &c.abort)) return false;
        tc_fence_after();
        const uint32_t at = smem_u32(slots + (size_t)a * 128 * 128);
        const uint32_t dbase = tmem + b * (uint32_t)N;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_i8(dbase, smem_desc_sw128(at + kk * 32), smem_desc_sw128(st + j * pb + kk * 32), idesc, kk ? 1u : 0u);
        tc_commit(&c.aempty[a]);
        tc_commit(&c.tfull[b]);
      }
      tc_commit(&c.empty[r.s]);
      c.consumed = r.n + 1;
      r.advance(S);
    }
  }
  return true;
}

// Epilogue: per K block, the accumulator scaled by that block's group scale is added into fp32
// registers (one per token of the chunk); per item the sums times the plane scale are written.
// K blocks are taken two at a time (both accumulators waited for, read, then released), so the
// fixed latencies of the wait and the TMEM load are paid once per pair.
__device__ __forceinline__ void d4_accumulate(float (&acc)[32], int nt8, int ntok, uint32_t tb, float s) {
  // columns [0, nt8) of the accumulator hold the hi plane, [nt8, 2 nt8) the lo plane; only the
  // 16-column groups that hold one of the item's ntok tokens are read
  if (nt8 == 8) {
    float v[16];
    tmem_ld16(tb, v);
    tmem_ld_wait();
#pragma unroll
    for (int t = 0; t < 8; ++t)
      acc[t] = fmaf(s, (float)__float_as_int(v[t]) + (float)__float_as_int(v[8 + t]) * (1.0f / 254.0f), acc[t]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; j += 16) {
      if (j >= nt8 || j >= ntok) break;
      float vh[16], vl[16];
      tmem_ld16(tb + j, vh);
      tmem_ld16(tb + nt8 + j, vl);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 16; ++t)
        acc[j + t] = fmaf(s, (float)__float_as_int(vh[t]) + (float)__float_as_int(vl[t]) * (1.0f / 254.0f), acc[j + t]);
    }
  }
}

template <bool kGateUp>
__device__ bool d4_epilogue(const DecStreamParams& p, D4Ctl& c, uint32_t tmem, int warp, int lane) {
  const int q = warp & 3;
  const int N = 2 * p.nt8;
  uint32_t kc = 0;
  DecItem it;
  for (int L = c.first; dec_item<kGateUp>(p, c, 0, L, it); L += gridDim.x) {
    const D4Walk w(p, it);
    const int kb0 = L % w.nkb;
    const int o = it.tile * 128 + q * 32 + lane;
    const bool vo = o < p.out_rows;
    // group scales of this matrix: [K / 128][out_rows], matrices W1 | W3 | W2 of each expert
    const int m = kGateUp ? it.mat : 2;
    const float* sg = p.wscale + (size_t)it.e * (3 * (size_t)p.d * p.f / 128) +
                      (size_t)m * ((size_t)p.d * p.f / 128) + (vo ? o : 0);
    auto group_scale = [&](int i) {  // scale of the i-th K block of the item's walk
      const int g = w.kbeg / 128 + (kb0 + i) % w.nkb;
      return (vo && i < w.nkb) ? __ldg(sg + (size_t)g * p.out_rows) : 0.f;
    };
    float acc[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) acc[t] = 0.f;
    float sc[8];  // the scales of K blocks i .. i + 7, loaded 8 blocks ahead
#pragma unroll
    for (int u = 0; u < 8; ++u) sc[u] = group_scale(u);
    for (int i0 = 0; i0 < w.nkb; i0 += 8) {
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        const int i = i0 + u;
        if (i >= w.nkb) break;
        const bool two = i + 1 < w.nkb;
        const uint32_t b0 = kc % kD4Bufs, ph0 = (kc / kD4Bufs) & 1u;
        const uint32_t b1 = (kc + 1) % kD4Bufs, ph1 = ((kc + 1) / kD4Bufs) & 1u;
        const bool got = ds_wait(&c.tfull[b0], ph0, &c.abort) && (!two || ds_wait(&c.tfull[b1], ph1, &c.abort));
        if (!__all_sync(0xffffffffu, got)) return false;
        tc_fence_after();
        const float s0 = sc[u], s1 = sc[u + 1];
        sc[u] = group_scale(i + 8);
        sc[u + 1] = group_scale(i + 9);
        const uint32_t lanes = (uint32_t)(q * 32) << 16;
        d4_accumulate(acc, p.nt8, it.ntok, tmem + lanes + b0 * (uint32_t)N, s0);
        if (two) d4_accumulate(acc, p.nt8, it.ntok, tmem + lanes + b1 * (uint32_t)N, s1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&c.tempty[b0]);
          if (two) mbar_arrive(&c.tempty[b1]);
        }
        kc += two ? 2 : 1;
      }
    }
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      if (t >= it.ntok || !vo) continue;
      const int row = it.row0 + t;
      const float v = __ldcg(p.rscale + (size_t)it.split * p.rscale_split_stride + row) * acc[t];
      if (kGateUp) p.GU[(((size_t)it.split * 2 + it.mat) * p.R + row) * p.f + o] = v;
      else p.Ypart[((size_t)it.split * p.R + row) * p.d + o] = v;
    }
  }
  return true;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kD4Threads, 1) dec_stream4_kernel(const __grid_constant__ DecStreamParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    pdl_wait();
    if (threadIdx.x == 0) atomicOr(p.err, kErrWaitTimeout);
    return;
  }
  const int S = p.stages;
  uint8_t* slots = smem;
  uint8_t* ring = smem + kD4SlotBytes;
  D4Ctl& c = *reinterpret_cast<D4Ctl*>(ring + (size_t)S * p.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tmem_cols = p.nt8 == 8 ? 128u : (p.nt8 == 16 ? 256u : 512u);  // kD4Bufs x 2 nt8
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&c.raw[s], 1);
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    for (int a = 0; a < kD4Slots; ++a) {
      mbar_init(&c.afull[a], 4);
      mbar_init(&c.aempty[a], 1);
    }
    for (int b = 0; b < kD4Bufs; ++b) {
      mbar_init(&c.tfull[b], 1);
      mbar_init(&c.tempty[b], 4);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    c.issued = 0;
    c.consumed = 0;
    c.first = blockIdx.x;
    mbar_fence_init();
    tma_prefetch_desc(&p.mapW);
    tma_prefetch_desc(&p.mapHi);
    tma_prefetch_desc(&p.mapLo);
  }
  pdl_wait();
  if (warp == 1) {
    tmem_alloc(&c.tmem, tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  const DecStreamParams* phases[1] = {&p};
  ds_items(phases, 1, c, p.offsets);  // starts and ends with a CTA barrier
  const uint32_t tmem = c.tmem;
  if (warp == 0) {
    if (lane == 0 && !d4_produce<kGateUp>(p, ring, c, S)) ds_abort(c, p.err);
    pdl_trigger();
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      if (!d4_mma<kGateUp>(p, slots, ring, c, S, tmem)) ds_abort(c, p.err);
      tc_commit(&c.drain);
      mbar_wait_bounded(&c.drain, 0);
    }
    __syncwarp();
  } else if (warp < 6) {
    if (!d4_epilogue<kGateUp>(p, c, tmem, warp, lane) && lane == 0) ds_abort(c, p.err);
  } else {
    if (!d4_convert<kGateUp>(p, slots, ring, c, S, warp - 6, lane) && lane == 0) ds_abort(c, p.err);
  }
  // error path: copies issued but never consumed land before the CTA exits; then TMEM is freed
  __syncthreads();
  if (threadIdx.x == 0 && c.abort) {
    for (int i = c.consumed; i < c.issued; ++i) {
      if (!mbar_wait_bounded(&c.raw[i % S], (uint32_t)(i / S) & 1u)) break;
      if (!mbar_wait_bounded(&c.full[i % S], (uint32_t)(i / S) & 1u)) break;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ------------------------------------------------------------------------- fused decode kernel
// The whole int8 expert stage in one cooperative launch (all CTAs resident, one per SM):
//   phase 1  gate/up weight stream -> GU partials                 (as dec_stream_kernel<true>)
//   barrier
//   phase 2  H = silu(g) * u -> int8 planes (epilogue warps, one (row, down split) unit at a
//            time; no shared-memory row buffer: the values are recomputed for the split pass),
//            while the producer already streams the first ring-full of down weights
//   barrier
//   phase 3  down weight stream -> Ypart                            (as dec_stream_kernel<false>)
//   barrier
//   phase 4  y[t] = sum_j w[t][j] * sum_split Ypart[split][dst_row[t][j]]  (fixed order)
// Grid barriers are arrival counters in global memory with bounded waits; the last CTA to
// leave resets them for the next launch.  One launch replaces four, the down stream starts
// with a full ring, and no kernel boundary separates the phases.
struct alignas(64) DecFusedParams {
  DecStreamParams gu;       // phase 1 (GU output)
  DecStreamParams dn;       // phase 3 (Ypart output); its planes are written by phase 2
  int8_t* hhi;              // H planes [R, f] and their scales [dsplit, R]
  int8_t* hlo;
  float* hscale;
  int32_t* dst_row;         // [T, k]
  float* topk_w;            // [T, k]
  int T, k;
  __nv_bfloat16* y;         // [T, d]
  int32_t* bar;             // [kFusedBars] arrival counters, zero between launches
  // phase 0 (route_in_kernel): router, top-k, grouping and the x planes in this launch
  int route_in_kernel;
  const __nv_bfloat16* x;   // [T, d]
  const __nv_bfloat16* router_w;  // [E, d]
  const float* router_b;    // [E] or NULL
  int router_flags;         // kRouterClamp | kRouterRaw
  int32_t* topk_idx;        // [T, k]
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E+1]
  int32_t* src_row;         // [T*k]
  int8_t* xhi;              // [R, d] x planes written by the routing phase (the buffers p.gu reads)
  int8_t* xlo;
  float* xscale;            // [R] scales of the x planes (the buffer p.gu.rscale reads)
};
// up to this many tokens every CTA of the fused kernel routes all of them itself
constexpr int kRedundantT = 1;
// grid-barrier counters: router done, x planes done, GU done, H done, Ypart done
enum { kBarRouter = 0, kBarPlanes, kBarGU, kBarH, kBarY, kFusedBars };
static_assert(kFusedBars <= kFusedBarCount, "grid-barrier counters of the fused kernel");

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid barriers are never reset.  A counter runs through [0, G * kBarLaps) (atom.inc wraps it
// to 0), and every launch that uses it adds exactly G: each CTA arrives once, also after an
// error.  A CTA's arrival returns the count before it; the round it belongs to started at the
// multiple of G below that, and the barrier is passed once the counter has moved G beyond that
// start.  The arrival (one thread, after a CTA barrier) is an acquire-release RMW, so every write
// the CTA made before its CTA barrier is visible to a CTA that acquires the counter later.
constexpr uint32_t kBarLaps = 1u << 16;
__device__ __forceinline__ uint32_t bar_arrive(int32_t* ctr, int G) {  // returns the count before
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.inc.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(ctr), "r"((uint32_t)G * kBarLaps - 1u)
               : "memory");
  return old;
}
__device__ __forceinline__ uint32_t bar_base(uint32_t old, int G) { return old - old % (uint32_t)G; }
__device__ __forceinline__ bool bar_passed(const int32_t* ctr, uint32_t base, int G) {
  const uint32_t wrap = (uint32_t)G * kBarLaps;
  return ((uint32_t)ld_acquire(ctr) + wrap - base) % wrap >= (uint32_t)G;
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// A flag in shared memory passed from one role of the CTA to another.
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta(int* p, int v) {
  asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Wait (bounded) until the round of the barrier `ctr` that started at `base` is complete.
__device__ bool grid_wait(const int32_t* ctr, uint32_t base, int G, volatile int* abort_flag) {
  const unsigned long long t0 = global_ns();
  while (!bar_passed(ctr, base, G)) {
    if (*abort_flag) return false;
    if (global_ns() - t0 > kWaitTimeoutNs) return false;
    __nanosleep(64);
  }
  return true;
}
// Arrive and wait; the last CTA to arrive completes the round and does not wait.
__device__ bool grid_sync(int32_t* ctr, int G, volatile int* abort_flag) {
  const uint32_t old = bar_arrive(ctr, G), base = bar_base(old, G);
  if (old - base == (uint32_t)G - 1u) return true;
  return grid_wait(ctr, base, G, abort_flag);
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Phase 0 (T <= 64): router + top-k (one CTA per token; skipped when the caller routed), a grid
// barrier, then in every CTA the
// grouping of all T x k choices (ranks from per-expert token bit masks, offsets by a scan; the
// same in every CTA, so no second exchange is needed), and for the CTA's own tokens: dst_row,
// src_row and the int8 planes of the token row in each of its k grouped rows.  The ring memory,
// idle until the producer starts, holds the scratch.  CTA 0 also writes counts and offsets.
// The caller then arrives on the planes barrier; the producer waits on it before its first plane
// copy.
__device__ void fused_route(const DecFusedParams& p, uint8_t* smem, DsCtl& c) {
  constexpr int kWarps = kDsThreads / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, T = p.T, k = p.k, E = p.gu.E, d = p.gu.d;
  const int nvec = d / 8;  // 16-byte slices of a bf16 row
  // scratch in the ring (idle until the producer starts)
  float* part = reinterpret_cast<float*>(smem);                         // [kWarps][kMaxExperts]
  float* lg = part + kWarps * kMaxExperts;                              // [kMaxExperts]
  int32_t* s_idx = reinterpret_cast<int32_t*>(smem + 8192);             // [T * k]
  float* s_w = reinterpret_cast<float*>(smem + 10240);                  // [T * k]
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(smem + 12288);  // [E] tokens choosing e
  float* red = reinterpret_cast<float*>(smem + 14336);                  // [kWarps]
  // A single token is routed by every CTA itself (the router weights are read from L2 by each
  // CTA), which saves a grid barrier; with more tokens CTA t routes token t and a barrier
  // follows (8 tokens routed in every CTA measured 20% slower at T=8).
  const bool redundant = p.route_in_kernel == 1 && T <= kRedundantT;
  for (int t = redundant ? 0 : blockIdx.x; p.route_in_kernel == 1 && t < T; t += redundant ? 1 : G) {
    const uint4* xv = reinterpret_cast<const uint4*>(p.x + (size_t)t * d);
    // the bias is loaded first (it is consumed last), and every slice of x and of the 8 expert
    // rows that a thread needs for one batch is loaded before any of them is used, so a batch
    // costs one memory round trip (d = 4096: one batch of 3 slices x 9 rows per thread)
    float bias[(kMaxExperts + kDsThreads - 1) / kDsThreads];
#pragma unroll
    for (int j = 0; j < (int)(sizeof(bias) / sizeof(float)); ++j) {
      const int e = tid + j * kDsThreads;
      bias[j] = (p.router_b && e < E) ? __ldg(p.router_b + e) : 0.f;
    }
    constexpr int kSlices = 3;
    for (int e0 = 0; e0 < E; e0 += 8) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
      for (int v0 = tid; v0 < nvec; v0 += kSlices * kDsThreads) {
        uint4 xq[kSlices], wq[kSlices][8];
#pragma unroll
        for (int u = 0; u < kSlices; ++u) {
          const int v = v0 + u * kDsThreads;
          xq[u] = v < nvec ? __ldg(xv + v) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            wq[u][i] = (v < nvec && e0 + i < E)
                           ? __ldg(reinterpret_cast<const uint4*>(p.router_w + (size_t)(e0 + i) * d) + v)
                           : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kSlices; ++u)
          if (v0 + u * kDsThreads < nvec)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = dot16(xq[u], wq[u][i], acc[i], p.x);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int off = 16; off; off >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
      }
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (e0 + i < E) part[warp * kMaxExperts + e0 + i] = acc[i];
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < (int)(sizeof(bias) / sizeof(float)); ++j) {
      const int e = tid + j * kDsThreads;
      if (e < E) {
        float sum = part[e];
        for (int w = 1; w < kWarps; ++w) sum += part[w * kMaxExperts + e];
        lg[e] = sum + bias[j];
      }
    }
    __syncthreads();
    if (warp == 0) {
      if (redundant) {
        warp_topk(lg, E, k, p.router_flags, lane, s_idx + (size_t)t * k, s_w + (size_t)t * k);
        __syncwarp();
        if (blockIdx.x == 0 && lane < k) {  // one CTA publishes the choices
          p.topk_idx[(size_t)t * k + lane] = s_idx[(size_t)t * k + lane];
          p.topk_w[(size_t)t * k + lane] = s_w[(size_t)t * k + lane];
        }
      } else {
        warp_topk(lg, E, k, p.router_flags, lane, p.topk_idx + (size_t)t * k, p.topk_w + (size_t)t * k);
      }
    }
    __syncthreads();
  }
  c.flag = 1;
  if (p.route_in_kernel == 1 && !redundant) {
    // every token's choices are needed below
    __syncthreads();
    if (tid == 0) {
      c.flag = grid_sync(&p.bar[kBarRouter], G, &c.abort) ? 1 : 0;
      if (!c.flag) ds_abort(c, p.gu.err);
    }
    __syncthreads();
  }
  // the choices: this CTA's own copy, or from global memory (another CTA's, or the caller's)
  auto choice = [&](int i) { return redundant ? s_idx[i] : __ldcg(p.topk_idx + i); };
  if (warp == 0) {  // per-expert token masks, then the offsets: exclusive scan of the counts
    for (int e = lane; e < E; e += 32) mask[e] = 0ull;
    __syncwarp();
    if (c.flag) {
      for (int i = lane; i < T * k; i += 32) {
        const int e = min(max(choice(i), 0), E - 1);
        atomicOr(&mask[e], 1ull << (i / k));
      }
    }
    __syncwarp();
    const int C = (E + 31) / 32;
    const int e0 = min(E, lane * C), e1 = min(E, e0 + C);
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += __popcll(mask[e]);
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += a;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
      const int cnt = __popcll(mask[e]);
      c.off[e] = run;
      if (blockIdx.x == 0) {
        p.counts[e] = cnt;
        p.offsets[e] = run;
      }
      run += cnt;
    }
    if (lane == 31) {
      c.off[E] = incl;
      if (blockIdx.x == 0) p.offsets[E] = incl;
    }
  }
  __syncthreads();
  for (int t = blockIdx.x; t < T && c.flag; t += G) {
    int rows[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      rows[j] = 0;
      if (j < k) {
        const int e = min(max(choice(t * k + j), 0), E - 1);
        rows[j] = c.off[e] + __popcll(mask[e] & ((1ull << t) - 1ull));
      }
    }
    if (tid < k) {
      const int r = rows[tid];
      p.dst_row[(size_t)t * k + tid] = r;
      p.src_row[r] = t;
    }
    const uint4* src = reinterpret_cast<const uint4*>(p.x + (size_t)t * d);
    float mx = 0.f;
    for (int v = tid; v < nvec; v += kDsThreads) {
      const uint4 q = __ldg(src + v);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(h2[i]);
        mx = fmaxf(mx, fmaxf(fabsf(f2.x), fabsf(f2.y)));
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
    for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, red[w]);
    __syncthreads();
    const float a = plane_scale(mx), inv_a = __frcp_rn(a);  // correctly rounded 1 / a
    if (tid < k) p.xscale[rows[tid]] = a;
    for (int v = tid; v < nvec; v += kDsThreads) {
      const uint4 q = __ldg(src + v);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
      uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f2 = __bfloat1622float2(h2[i]);
        int qh0, ql0, qh1, ql1;
        split_planes(f2.x, a, inv_a, qh0, ql0);
        split_planes(f2.y, a, inv_a, qh1, ql1);
        hw[i >> 1] |= (((uint32_t)qh0 & 0xffu) | (((uint32_t)qh1 & 0xffu) << 8)) << (16 * (i & 1));
        lw[i >> 1] |= (((uint32_t)ql0 & 0xffu) | (((uint32_t)ql1 & 0xffu) << 8)) << (16 * (i & 1));
      }
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
          reinterpret_cast<uint2*>(p.xhi + (size_t)rows[j] * d)[v] = make_uint2(hw[0], hw[1]);
          reinterpret_cast<uint2*>(p.xlo + (size_t)rows[j] * d)[v] = make_uint2(lw[0], lw[1]);
        }
      }
    }
  }
  // the planes are read next by TMA copies of other CTAs; the caller arrives on the planes
  // barrier after its next CTA barrier
  fence_proxy_async_global();
}

// H for one (row r, down split sp) unit, by the 128 epilogue threads of a CTA (tid 0..127): h =
// silu(g) * u over the columns of split sp, from the gate/up partials summed in split order, rounded
// to bf16, then split into int8 planes with one scale for the unit.  The caller makes the planes
// visible to the async proxy and publishes them.
__device__ void h_row_planes(const DecFusedParams& p, DsCtl& c, int r, int sp, int tid, int lane) {
  float* red = c.red;
  const int R = p.gu.R, f = p.gu.f, gs = p.gu.nsplit, ds = p.dn.nsplit;
  const size_t plane = (size_t)R * f;
  const int span = f / ds, k0 = sp * span;
  const float* g0 = p.gu.GU + (size_t)r * f + k0;
  // h for 4 consecutive columns: all gsplit partials are loaded before they are summed (in
  // split order), so one pass is one memory round trip per step
  auto hvals = [&](int j, float (&hv)[4]) {
    float4 gv[kDecGateSplitMax], uv[kDecGateSplitMax];
#pragma unroll
    for (int s2 = 0; s2 < kDecGateSplitMax; ++s2) {
      if (s2 < gs) {
        gv[s2] = __ldcg(reinterpret_cast<const float4*>(g0 + (size_t)(2 * s2) * plane + j));
        uv[s2] = __ldcg(reinterpret_cast<const float4*>(g0 + (size_t)(2 * s2 + 1) * plane + j));
      }
    }
    float4 g = gv[0], uu = uv[0];
#pragma unroll
    for (int s2 = 1; s2 < kDecGateSplitMax; ++s2) {
      if (s2 < gs) {
        g.x += gv[s2].x; g.y += gv[s2].y; g.z += gv[s2].z; g.w += gv[s2].w;
        uu.x += uv[s2].x; uu.y += uv[s2].y; uu.z += uv[s2].z; uu.w += uv[s2].w;
      }
    }
    hv[0] = __bfloat162float(__float2bfloat16_rn(silu_mul(g.x, uu.x)));
    hv[1] = __bfloat162float(__float2bfloat16_rn(silu_mul(g.y, uu.y)));
    hv[2] = __bfloat162float(__float2bfloat16_rn(silu_mul(g.z, uu.z)));
    hv[3] = __bfloat162float(__float2bfloat16_rn(silu_mul(g.w, uu.w)));
  };
  // A short unit (at most kHKeep steps per thread, e.g. one token's 896-column unit) keeps its
  // h values in registers between the max and the split; a longer one makes two passes over
  // the partials (holding every step measured slower: the kernel's register count doubled).
  constexpr int kHKeep = 2;
  const bool keep = span <= 128 * 4 * kHKeep;
  float hk[kHKeep][4];
  float mx = 0.f;
  if (keep) {
#pragma unroll
    for (int it = 0; it < kHKeep; ++it) {
      const int j = tid * 4 + it * 128 * 4;
      if (j < span) {
        hvals(j, hk[it]);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(hk[it][0]), fabsf(hk[it][1])), fmaxf(fabsf(hk[it][2]), fabsf(hk[it][3]))));
      }
      asm volatile("" ::: "memory");  // one step's partials in registers at a time
    }
  } else {
    for (int j = tid * 4; j < span; j += 128 * 4) {
      float hv[4];
      hvals(j, hv);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(hv[0]), fabsf(hv[1])), fmaxf(fabsf(hv[2]), fabsf(hv[3]))));
    }
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[tid >> 5] = mx;
  epi_sync();
  mx = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  epi_sync();  // red[] is rewritten by the next unit
  const float a = plane_scale(mx), inv_a = __frcp_rn(a);  // correctly rounded 1 / a
  if (tid == 0) p.hscale[(size_t)sp * R + r] = a;
  int8_t* hrow = p.hhi + (size_t)r * f + k0;
  int8_t* lrow = p.hlo + (size_t)r * f + k0;
  auto put = [&](int j, const float (&hv)[4]) {
    uint32_t hw = 0u, lw = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      int qh, ql;
      split_planes(hv[i], a, inv_a, qh, ql);
      hw |= ((uint32_t)qh & 0xffu) << (8 * i);
      lw |= ((uint32_t)ql & 0xffu) << (8 * i);
    }
    *reinterpret_cast<uint32_t*>(hrow + j) = hw;
    *reinterpret_cast<uint32_t*>(lrow + j) = lw;
  };
  if (keep) {
#pragma unroll
    for (int it = 0; it < kHKeep; ++it) {
      const int j = tid * 4 + it * 128 * 4;
      if (j < span) put(j, hk[it]);
    }
  } else {
    for (int j = tid * 4; j < span; j += 128 * 4) {  // the same values again, now split
      float hv[4];
      hvals(j, hv);
      put(j, hv);
    }
  }
}

__global__ void __launch_bounds__(kDsThreads, 1) dec_fused_kernel(const __grid_constant__ DecFusedParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int S = p.gu.stages;
  DsCtl& c = *reinterpret_cast<DsCtl*>(smem + (size_t)S * p.gu.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const bool aligned = (smem_u32(smem) & 1023u) == 0;  // the 128-byte swizzle needs 1024-byte stages
  const DecStreamParams* phases[2] = {&p.gu, &p.dn};
  uint32_t planes_old = 0;  // thread 0: the planes barrier count before its arrival
  if (aligned) {
    ds_init(phases, 2, c, S);
    if (p.route_in_kernel) {
      fused_route(p, smem, c);
      // CTAs 0..T-1 also split their token's planes and start last: the items are dealt so
      // that the CTAs that take one item more than the others are not among them
      if (threadIdx.x == 0) c.first = (int)((blockIdx.x + gridDim.x - (unsigned)min(p.T, (int)gridDim.x)) % gridDim.x);
      ds_items(phases, 2, c, nullptr);  // starts with a CTA barrier: this CTA's planes are written
      // Arrival on the planes barrier by the producer thread itself; the count it returns is
      // only needed when the producer waits, so the round trip overlaps its first copies.
      if (threadIdx.x == 0) planes_old = bar_arrive(&p.bar[kBarPlanes], G);
    } else {
      ds_items(phases, 2, c, p.gu.offsets);
    }
  }
  const uint32_t tmem = aligned ? c.tmem : 0u;
  if (!aligned) {
    if (threadIdx.x == 0) {  // report, and arrive at every barrier the others wait on
      atomicOr(p.gu.err, kErrWaitTimeout);
      if (p.route_in_kernel == 1 && p.T > kRedundantT) bar_arrive(&p.bar[kBarRouter], G);
      if (p.route_in_kernel) bar_arrive(&p.bar[kBarPlanes], G);
      for (int b = kBarGU; b <= kBarY; ++b) bar_arrive(&p.bar[b], G);
    }
  } else if (warp == 0) {
    if (lane == 0) {
      DsRing r;
      // with the routing done in this launch, the gate/up weights go out at once and the plane
      // copies wait until every CTA has written its tokens' planes
      bool ok = ds_produce<true>(p.gu, smem, c, S, 0, r, p.route_in_kernel != 0, [&] {
        if (!grid_wait(&p.bar[kBarPlanes], bar_base(planes_old, G), G, &c.abort)) return false;
        fence_proxy_async_global();
        return true;
      });
      // down weights go out at once; their plane copies wait until this CTA's epilogue warps
      // have passed the H barrier (phase 2 of every CTA done)
      if (ok)
        ok = ds_produce<false>(p.dn, smem, c, S, 1, r, true, [&] {
          const unsigned long long t0 = global_ns();
          int v;
          while ((v = ld_acquire_cta(&c.hpass)) == 0) {
            if (*(volatile int*)&c.abort || global_ns() - t0 > kWaitTimeoutNs) return false;
            __nanosleep(32);
          }
          if (v < 0) return false;
          fence_proxy_async_global();
          return true;
        });
      if (!ok) ds_abort(c, p.gu.err);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      DsRing r;
      int iter = 0;
      bool ok = ds_mma<true>(p.gu, smem, c, S, 0, r, iter, tmem);
      if (ok) ok = ds_mma<false>(p.dn, smem, c, S, 1, r, iter, tmem);
      if (!ok) ds_abort(c, p.gu.err);
      tc_commit(&c.drain);
      mbar_wait_bounded(&c.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue warps: phases 1-4
    const int tid = threadIdx.x - 64;  // 0..127
    int iter = 0;
    // Grid barrier over the epilogue warps of every CTA: each CTA arrives exactly once (also
    // after an error, so that the others are not kept waiting); the result is the same for all
    // four warps of a CTA (false once this CTA has aborted or the wait gave up).
    auto grid_barrier = [&](int idx) -> bool {
      epi_sync();
      if (tid == 0) {
        const uint32_t old = bar_arrive(&p.bar[idx], G), base = bar_base(old, G);
        const bool passed =
            !c.abort && (old - base == (uint32_t)G - 1u || grid_wait(&p.bar[idx], base, G, &c.abort));
        c.flag = passed ? 1 : 0;
        if (!passed && !c.abort) ds_abort(c, p.gu.err);
        if (idx == kBarH) st_release_cta(&c.hpass, passed ? 1 : -1);  // the producer waits on it
      }
      epi_sync();
      return *(volatile int*)&c.flag != 0;
    };
    bool ok = ds_epilogue<true>(p.gu, c, 0, iter, tmem, warp, lane);
    if (!__all_sync(0xffffffffu, ok) && lane == 0) ds_abort(c, p.gu.err);
    // barrier: every CTA's GU partials are written
    ok = grid_barrier(kBarGU);
    if (ok) {
      // phase 2: H planes, one (row, down split) unit per round
      const int R = p.gu.R, ds = p.dn.nsplit;
      for (int u = blockIdx.x; u < R * ds; u += G) {
        const int r = u / ds, sp = u - r * ds;
        h_row_planes(p, c, r, sp, tid, lane);
      }
      fence_proxy_async_global();  // the planes are read next by TMA copies of other CTAs
    }
    // barrier: every CTA's H planes are written (the producer waits on the same counter)
    ok = grid_barrier(kBarH);
    if (ok) ok = ds_epilogue<false>(p.dn, c, 1, iter, tmem, warp, lane);
    if (!__all_sync(0xffffffffu, ok) && lane == 0) ds_abort(c, p.gu.err);
    // barrier: every CTA's down partials are written
    ok = grid_barrier(kBarY);
    if (ok) {
      // phase 4: combine, one thread per (token, 4 consecutive outputs)
      const int d = p.dn.d, ns = p.dn.nsplit, k = p.k;
      const size_t ss = (size_t)p.dn.R * d;
      const int chunks = d >> 2;
      for (long long qi = (long long)blockIdx.x * 128 + tid; qi < (long long)p.T * chunks; qi += (long long)G * 128) {
        const int t = (int)(qi / chunks), cc = (int)(qi - (long long)t * chunks) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
          const int rr = __ldcg(p.dst_row + (size_t)t * k + j);
          const float wj = __ldcg(p.topk_w + (size_t)t * k + j);
          const float* base = p.dn.Ypart + (size_t)rr * d + cc;
          float4 part = make_float4(0.f, 0.f, 0.f, 0.f);
          int sp = 0;
          for (; sp + 4 <= ns; sp += 4) {
            float4 v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) v[i] = __ldcg(reinterpret_cast<const float4*>(base + (size_t)(sp + i) * ss));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              part.x += v[i].x; part.y += v[i].y; part.z += v[i].z; part.w += v[i].w;
            }
          }
          for (; sp < ns; ++sp) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(base + (size_t)sp * ss));
            part.x += v.x; part.y += v.y; part.z += v.z; part.w += v.w;
          }
          acc.x = fmaf(wj, part.x, acc.x);
          acc.y = fmaf(wj, part.y, acc.y);
          acc.z = fmaf(wj, part.z, acc.z);
          acc.w = fmaf(wj, part.w, acc.w);
        }
        const __nv_bfloat162 lo2 = __floats2bfloat162_rn(acc.x, acc.y), hi2 = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = (uint32_t)__bfloat16_as_ushort(lo2.x) | ((uint32_t)__bfloat16_as_ushort(lo2.y) << 16);
        pk.y = (uint32_t)__bfloat16_as_ushort(hi2.x) | ((uint32_t)__bfloat16_as_ushort(hi2.y) << 16);
        *reinterpret_cast<uint2*>(p.y + (size_t)t * d + cc) = pk;
      }
    }
  }
  if (aligned) ds_teardown(c, S);
  else __syncthreads();
}

// K blocks per ring stage: COLIBRI_DEC_KB (1..4), default 2.
int dec_kbs() {
  const char* v = getenv("COLIBRI_DEC_KB");
  const int k = v ? atoi(v) : 2;
  return k < 1 ? 1 : (k > kDsMaxKbs ? kDsMaxKbs : k);
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

bool plane_maps(DecStreamParams& p, const int8_t* hi, const int8_t* lo, int K) {
  const uint64_t pd[2] = {(uint64_t)K, (uint64_t)p.R}, ps[1] = {(uint64_t)K};
  const uint32_t pb[2] = {128, (uint32_t)p.nt8};
  if (!make_tmap(&p.mapHi, CU_TENSOR_MAP_DATA_TYPE_UINT8, hi, 2, pd, ps, pb)) return false;
  if (!make_tmap(&p.mapLo, CU_TENSOR_MAP_DATA_TYPE_UINT8, lo, 2, pd, ps, pb)) return false;
  p.kbs = dec_kbs();
  p.evict_first = !(getenv("COLIBRI_DEC_EVICT") && strcmp(getenv("COLIBRI_DEC_EVICT"), "0") == 0);
  p.stage_bytes = (uint32_t)(p.kbs * (128 * 128 + 2 * p.nt8 * 128));
  p.stages = (int)std::min<size_t>(kDsMaxStages, kDsRingBytes / p.stage_bytes);
  return true;
}

template <bool kGateUp>
cudaError_t launch_stream(const DecStreamParams& p, cudaStream_t s) {
  const size_t smem = (size_t)p.stages * p.stage_bytes + kDsCtlBytes;
  return launch_kernel(dec_stream_kernel<kGateUp>, dim3(sm_count_current()), dim3(kDsThreads), smem, s, 1, p);
}

}  // namespace

cudaError_t configure_dec_kernels() {
  const int smem = (int)(kDsRingBytes + kDsCtlBytes);
  cudaError_t e = cudaFuncSetAttribute(dec_stream_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_stream_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(dec_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_stream4_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_stream4_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(dec_finish_h_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFinishMaxSmem);
  return e;
}

namespace {

// Parameters of one stream phase (weights, planes, scales, outputs); false if a tensor map
// cannot be encoded.
bool dec_gateup_params(DecStreamParams& p, const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const int8_t* W,
                       const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                       const int32_t* offsets, int nsplit, float* GU, int R, int max_rows_per_expert, uint32_t* err) {
  memset(&p, 0, sizeof(p));
  const uint64_t dims[4] = {(uint64_t)d, (uint64_t)f, 2, (uint64_t)E};
  const uint64_t st[3] = {(uint64_t)d, (uint64_t)f * d, (uint64_t)wstride};
  const uint32_t box[4] = {128, 128, 1, 1};
  if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, 4, dims, st, box)) return false;
  p.wscale = scales;
  p.scale_per_matrix = scale_mode == COLIBRI_SCALE_PER_MATRIX;
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
  return plane_maps(p, Xhi, Xlo, d);
}

bool dec_down_params(DecStreamParams& p, const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const int8_t* W,
                     const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                     const int32_t* offsets, int nsplit, int R, float* Ypart, int max_rows_per_expert, uint32_t* err) {
  memset(&p, 0, sizeof(p));
  const uint64_t dims[3] = {(uint64_t)f, (uint64_t)d, (uint64_t)E};
  const uint64_t st[2] = {(uint64_t)f, (uint64_t)wstride};
  const uint32_t box[3] = {128, 128, 1};
  if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W + 2 * (size_t)f * d, 3, dims, st, box)) return false;
  p.wscale = scales;
  p.scale_per_matrix = scale_mode == COLIBRI_SCALE_PER_MATRIX;
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
  return plane_maps(p, Hhi, Hlo, f);
}

}  // namespace

cudaError_t launch_dec_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const int8_t* W,
                              const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                              const int32_t* offsets, int nsplit, float* GU, int R, int max_rows_per_expert,
                              uint32_t* err, cudaStream_t s) {
  DecStreamParams p;
  if (!dec_gateup_params(p, Xhi, Xlo, xscale, W, scales, scale_mode, wstride, d, f, E, offsets, nsplit, GU, R,
                         max_rows_per_expert, err))
    return cudaErrorInvalidValue;
  return launch_stream<true>(p, s);
}

namespace {

// Stream parameters of the int4 kernels: the packed weights are copied unswizzled, 64 bytes
// (128 K elements) of 128 rows per tile; the stage holds kbs such tiles and their plane tiles.
bool dec4_params(DecStreamParams& p, bool gateup, const int8_t* hi, const int8_t* lo, const float* rscale,
                 int rscale_split_stride, const uint8_t* W, const float* scales, int64_t wstride, int d, int f, int E,
                 const int32_t* offsets, int nsplit, float* out, int R, int max_rows_per_expert, uint32_t* err) {
  memset(&p, 0, sizeof(p));
  if (d % 128 || f % 128 || wstride % 256) return false;
  if (gateup) {
    const uint64_t dims[4] = {(uint64_t)d / 2, (uint64_t)f, 2, (uint64_t)E};
    const uint64_t st[3] = {(uint64_t)d / 2, (uint64_t)f * d / 2, (uint64_t)wstride / 2};
    const uint32_t box[4] = {64, 128, 1, 1};
    if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, 4, dims, st, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  } else {
    const uint64_t dims[3] = {(uint64_t)f / 2, (uint64_t)d, (uint64_t)E};
    const uint64_t st[2] = {(uint64_t)f / 2, (uint64_t)wstride / 2};
    const uint32_t box[3] = {64, 128, 1};
    if (!make_tmap(&p.mapW, CU_TENSOR_MAP_DATA_TYPE_UINT8, W + (size_t)f * d, 3, dims, st, box,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
      return false;
  }
  p.wscale = scales;
  p.rscale = rscale;
  p.rscale_split_stride = rscale_split_stride;
  p.offsets = offsets;
  p.E = E;
  p.d = d;
  p.f = f;
  p.out_rows = gateup ? f : d;
  p.K = gateup ? d : f;
  p.nsplit = nsplit;
  p.kspan = p.K / nsplit;
  p.nt8 = dec_nt8(max_rows_per_expert);
  p.R = R;
  if (gateup) p.GU = out;
  else p.Ypart = out;
  p.err = err;
  if (!plane_maps(p, hi, lo, p.K)) return false;
  p.stage_bytes = (uint32_t)((p.kbs * (2 * p.nt8 * 128 + kD4RawBytes) + 1023) / 1024 * 1024);
  p.stages = (int)std::min<size_t>(kDsMaxStages, (kDsRingBytes - kD4SlotBytes) / p.stage_bytes);
  return p.stages >= 2;
}

template <bool kGateUp>
cudaError_t launch_stream4(const DecStreamParams& p, cudaStream_t s) {
  const size_t smem = kD4SlotBytes + (size_t)p.stages * p.stage_bytes + kDsCtlBytes;
  return launch_kernel(dec_stream4_kernel<kGateUp>, dim3(sm_count_current()), dim3(kD4Threads), smem, s, 1, p);
}

}  // namespace

cudaError_t launch_dec4_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const uint8_t* W,
                               const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                               int nsplit, float* GU, int R, int max_rows_per_expert, uint32_t* err, cudaStream_t s) {
  DecStreamParams p;
  if (!dec4_params(p, true, Xhi, Xlo, xscale, 0, W, scales, wstride, d, f, E, offsets, nsplit, GU, R,
                   max_rows_per_expert, err))
    return cudaErrorInvalidValue;
  return launch_stream4<true>(p, s);
}

cudaError_t launch_dec4_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const uint8_t* W,
                             const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                             int nsplit, int R, float* Ypart, int max_rows_per_expert, uint32_t* err, cudaStream_t s) {
  DecStreamParams p;
  if (!dec4_params(p, false, Hhi, Hlo, hscale, R, W, scales, wstride, d, f, E, offsets, nsplit, Ypart, R,
                   max_rows_per_expert, err))
    return cudaErrorInvalidValue;
  return launch_stream4<false>(p, s);
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
                            const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                            const int32_t* offsets, int nsplit, int R, float* Ypart, int max_rows_per_expert,
                            uint32_t* err, cudaStream_t s) {
  DecStreamParams p;
  if (!dec_down_params(p, Hhi, Hlo, hscale, W, scales, scale_mode, wstride, d, f, E, offsets, nsplit, R, Ypart,
                       max_rows_per_expert, err))
    return cudaErrorInvalidValue;
  return launch_stream<false>(p, s);
}

cudaError_t launch_dec_fused(const DecFusedArgs& a, cudaStream_t s) {
  if (a.T <= 0) return cudaSuccess;
  if (a.f % a.dsplit != 0 || (a.f / a.dsplit) % 4 != 0 || a.d % 4 != 0) return cudaErrorInvalidValue;
  DecFusedParams p;
  memset(&p, 0, sizeof(p));
  const int R = a.T * a.k;
  // H is split into planes in place of the x planes (the gate/up phase has finished reading them)
  int8_t* hhi = a.planes_hi;
  int8_t* hlo = a.planes_lo;
  float* hsc = a.planes_scale;
  if (!dec_gateup_params(p.gu, a.planes_hi, a.planes_lo, a.planes_scale, a.W, a.scales, a.scale_mode, a.wstride, a.d,
                         a.f, a.E,
                         a.offsets, a.gsplit, a.GU, R, a.T, a.err) ||
      !dec_down_params(p.dn, hhi, hlo, hsc, a.W, a.scales, a.scale_mode, a.wstride, a.d, a.f, a.E, a.offsets, a.dsplit,
                       R, a.Ypart, a.T, a.err))
    return cudaErrorInvalidValue;
  p.hhi = hhi;
  p.hlo = hlo;
  p.hscale = hsc;
  p.dst_row = a.dst_row;
  p.topk_w = a.topk_w;
  p.T = a.T;
  p.k = a.k;
  p.y = a.y;
  p.bar = a.bar;
  p.route_in_kernel = a.route_in_kernel;
  p.x = a.x;
  p.router_w = a.router_w;
  p.router_b = a.router_b;
  p.router_flags = a.router_flags;
  p.topk_idx = a.topk_idx;
  p.counts = a.counts;
  p.offsets = a.offsets_out;
  p.src_row = a.src_row;
  p.xhi = a.planes_hi;
  p.xlo = a.planes_lo;
  p.xscale = a.planes_scale;
  if (a.route_in_kernel && (a.T > 64 || !a.x || !a.topk_idx || !a.counts || !a.offsets_out || !a.src_row ||
                            (a.route_in_kernel == 1 && !a.router_w)))
    return cudaErrorInvalidValue;
  const size_t smem = (size_t)p.gu.stages * p.gu.stage_bytes + kDsCtlBytes;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count_current());
  cfg.blockDim = dim3(kDsThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the grid barriers need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  launch_chain_break();  // an ordinary launch: the next one must not overlap it
  const cudaError_t e = cudaLaunchKernelEx(&cfg, dec_fused_kernel, p);
  launch_chain_break();
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace colibri
