// Gate stage: router logits, softmax and top-k.  bf16 activations use the tcgen05 kernel at the
// end of this file (the stage is bound by one read of x); fp32 activations use the SIMT kernel
// (fp32 FMA, no TF32).
//
// logits l[t][e] = b[e] + sum_i x[t][i] * Wr[e][i]      (www.hotelren.com/news/4731937 §3.2,
//                                                        www.0539edu.com/news/4774449 §2.1)
// top-k: order by (logit descending, expert index ascending), slot 0 = largest; ties keep
// the lower index, as the strict ">" scan of www.mhpq.cn/news/563172 §3.2 does.  The
// selection is made by k rounds of a warp-wide arg-max (the warp-shuffle top-k idea of
// www.pptc.cn/news/100465 §2.1, generalised from 2 to k <= 8 and to 256 experts).
// weights: softmax over all E renormalised over the k chosen, computed as
// exp(l_j - l_0) / sum_j' exp(l_j' - l_0) in fp32; or, on request, the raw chosen logits, and
// optionally with every logit clamped to [-50, 50] first (router_clamp / topk_weights).
// Output layout [T][k] (www.pptc.cn/news/100465 §3.4).
#include <algorithm>
#include <cstring>

#include "common.cuh"

namespace colibri {
namespace {

constexpr int kRouterTT = 32;  // tokens per CTA
constexpr int kRouterDK = 32;  // K chunk staged in shared memory
constexpr int kRouterThreads = 256;


// SIMT router: 32 tokens per CTA, warp w accumulates experts w, w+8, ... for the token of
// its lane; x and Wr chunks are staged in shared memory as fp32.
template <typename Tin>
__global__ void __launch_bounds__(kRouterThreads) router_topk_simt_kernel(
    const Tin* __restrict__ x, int T, int d, const Tin* __restrict__ wr, const float* __restrict__ b,
    int E, int k, int rflags, int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  pdl_trigger();
  pdl_wait();
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
    warp_topk(lg + tt * (E + 1), E, k, rflags, lane, idx_out + (size_t)t * k, w_out + (size_t)t * k);
  }
}

// ---------------------------------------------------------------------------------------
// Small batches (T <= 64): one CTA per token.  Warp w computes the logits of experts w, w + 8,
// ... with its lanes splitting d (16-byte loads; the token row is read through L1) and a
// shuffle reduction; then warp 0 selects the top-k.  Latency-bound work, so no tensor cores.
// ---------------------------------------------------------------------------------------

// Small batches: one CTA per token.  Every thread takes the same 16-byte slices of x and of 8
// expert rows at a time, so each thread has 9 independent loads per slice in flight; the 8
// partial dot products are reduced per warp by shuffles and then over the 8 warps in a fixed
// order (deterministic).
template <typename Tin>
__global__ void __launch_bounds__(256) router_small_kernel(const Tin* __restrict__ x, int d,
                                                           const Tin* __restrict__ wr, const float* __restrict__ b,
                                                           int E, int k, int rflags,
                                                           int32_t* __restrict__ idx_out,
                                                           float* __restrict__ w_out) {
  pdl_trigger();
  pdl_wait();
  constexpr int kWarps = 8, kChunk = 8;
  __shared__ float part[kWarps][kMaxExperts];
  __shared__ float lg[kMaxExperts];
  const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = d * (int)sizeof(Tin) / 16;
  const uint4* xv = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int e0 = 0; e0 < E; e0 += kChunk) {
    float acc[kChunk];
#pragma unroll
    for (int i = 0; i < kChunk; ++i) acc[i] = 0.f;
#pragma unroll 2
    for (int v = threadIdx.x; v < nvec; v += kWarps * 32) {
      const uint4 xq = __ldg(xv + v);
#pragma unroll
      for (int i = 0; i < kChunk; ++i)
        if (e0 + i < E) acc[i] = dot16(xq, __ldg(reinterpret_cast<const uint4*>(wr + (size_t)(e0 + i) * d) + v), acc[i], x);
    }
#pragma unroll
    for (int i = 0; i < kChunk; ++i) {
#pragma unroll
      for (int off = 16; off; off >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int i = 0; i < kChunk; ++i)
        if (e0 + i < E) part[warp][e0 + i] = acc[i];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kWarps * 32) {
    float sum = part[0][e];
#pragma unroll
    for (int wi = 1; wi < kWarps; ++wi) sum += part[wi][e];
    lg[e] = sum + (b ? b[e] : 0.f);
  }
  __syncthreads();
  if (warp == 0) warp_topk(lg, E, k, rflags, lane, idx_out + (size_t)t * k, w_out + (size_t)t * k);
}

// ---------------------------------------------------------------------------------------
// bf16 router on the 5th-generation tensor cores.  A CTA owns 128 tokens (the 128 TMEM lanes)
// and all experts padded to N = 16 * ceil(E / 16) columns: one elected thread streams x and Wr
// tiles (64-wide K blocks, 128-byte swizzle) through a 4-stage shared-memory ring with TMA and
// issues tcgen05.mma (M=128, N, K=16) into an fp32 accumulator in TMEM; padded expert rows are
// read as zeros and never selected.  Then every thread owns one token row: it reads that row's
// logits from TMEM 16 columns at a time, adds the bias and keeps the k best in registers by
// insertion with a strict ">" (so of two equal logits the lower expert index, seen first,
// stays ahead), then writes ids and the renormalised softmax weights.  Every wait is bounded.
// ---------------------------------------------------------------------------------------
constexpr int kRtMaxStages = 16;
constexpr int kRtABytes = 128 * 64 * 2;            // x tile: 128 tokens x 64 K
constexpr size_t kRtRingBytes = 200 * 1024;        // shared memory given to the ring

struct alignas(64) RouterTcParams {
  CUtensorMap mapX;  // [T, d], box {64, 128}
  CUtensorMap mapW;  // [E, d], box {64, N}
  const float* b;
  int T, d, E, k, N;
  int rflags;        // kRouterClamp | kRouterRaw
  int ksplit;        // CTAs per 128-token tile (one cluster, gridDim.x), each over d / ksplit
  int stages;  // ring depth: as many stages as fit in kRtRingBytes (small expert counts go deeper)
  int kbs;     // consecutive 64-wide K blocks per stage (1 or 2): each x row is read kbs x 128 bytes at a time
  uint32_t stage_bytes, tmem_cols;
  int32_t* idx;
  float* w;
  uint32_t* err;
};

__device__ __forceinline__ bool rt_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
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

// Insert (v, e) into a list of the k best kept in (logit descending, expert ascending) order.
template <int KK>
__device__ __forceinline__ void rt_insert_ordered(float (&bv)[KK], int (&bi)[KK], int k, float v, int e) {
#pragma unroll
  for (int j = 0; j < KK; ++j) {
    if (j < k && (v > bv[j] || (v == bv[j] && e < bi[j]))) {
      const float tv = bv[j];
      const int ti = bi[j];
      bv[j] = v;
      bi[j] = e;
      v = tv;
      e = ti;
    }
  }
}

constexpr int kRtThreads = 256;

// KK: the top-k list length the kernel is compiled for (k <= KK)
template <int KK>
__global__ void __launch_bounds__(kRtThreads, 1) router_tc_kernel(const __grid_constant__ RouterTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // the 128-byte swizzle needs 1024-byte aligned tiles
    pdl_wait();
    if (threadIdx.x == 0 && p.err) atomicOr(p.err, kErrWaitTimeout);
    return;
  }
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * p.stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* done = empty + S;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  int* issued_s = const_cast<int*>(abort_flag) + 1;  // copies issued / stages consumed (error path)
  int* consumed_s = issued_s + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *issued_s = 0;
    *consumed_s = 0;
    mbar_fence_init();
    tma_prefetch_desc(&p.mapX);
    tma_prefetch_desc(&p.mapW);
  }
  pdl_wait();  // below: reads of earlier kernels' output; TMEM once the previous kernel released its own
  if (warp == 0) {
    tmem_alloc(tmem_holder, p.tmem_cols);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int split = blockIdx.x, tile = blockIdx.y;  // the K slices of a tile form one cluster
  const int row0 = tile * 128;
  const int kspan = p.d / p.ksplit;               // a multiple of 64
  const int kb0 = split * (kspan / 64);
  const int nkb = kspan / 64;
  // A stage holds kbs consecutive K blocks: x tiles first, then the Wr tiles.
  const int kbs = p.kbs, nst = nkb / kbs;
  const uint32_t wtile = (uint32_t)p.N * 128u;
  const uint32_t bytes = (uint32_t)kbs * (kRtABytes + wtile);
  // The CTAs of a launch start their K walk at different stages (rotated by the tile index), so
  // the x rows read at one time do not all sit at the same column offset, which would put every
  // request on the same DRAM channels.  (This fixes, per tile, the order of the fp32 sum.)
  const int st_rot = tile % nst;
  if (warp == 0) {
    if (lane == 0) {
      // ----------------------------------------------------------- TMA producer
      bool ok = true;
      for (int i = 0; i < nst; ++i) {
        const int kb = ((st_rot + i) % nst) * kbs;
        const int s = i % S;
        const uint32_t ph = (uint32_t)(i / S) & 1u;
        if (!rt_wait(&empty[s], ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + (size_t)s * p.stage_bytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int j = 0; j < kbs; ++j) {
          tma_load_2d(sa + (size_t)j * kRtABytes, &p.mapX, &full[s], (kb0 + kb + j) * 64, row0);
          tma_load_2d(sa + (size_t)kbs * kRtABytes + (size_t)j * wtile, &p.mapW, &full[s], (kb0 + kb + j) * 64, 0);
        }
        *issued_s = i + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        if (p.err) atomicOr(p.err, kErrWaitTimeout);
      }
    }
    pdl_trigger();  // every copy of this CTA is issued: let the next kernel be scheduled
    __syncwarp();  // the other lanes wait here, not in a spin beside the producer
  } else if (warp == 1) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(128, p.N);
      bool ok = true;
      for (int i = 0; i < nst; ++i) {
        const int s = i % S;
        const uint32_t ph = (uint32_t)(i / S) & 1u;
        if (!rt_wait(&full[s], ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)s * p.stage_bytes);
        for (int j = 0; j < kbs; ++j) {
          const uint32_t xa = sa + (uint32_t)j * kRtABytes, wa = sa + (uint32_t)kbs * kRtABytes + (uint32_t)j * wtile;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_f16(tmem, smem_desc_sw128(xa + kk * 32), smem_desc_sw128(wa + kk * 32), idesc,
                       (i | j | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);  // frees the stage once these MMAs have read it
        *consumed_s = i + 1;
      }
      if (!ok) {
        *abort_flag = 1;
        if (p.err) atomicOr(p.err, kErrWaitTimeout);
      }
      tc_commit(done);  // arrives once every MMA issued above has completed
    }
    __syncwarp();
  }
  // ------------------------------------------------------------- epilogue
  const bool got = rt_wait(done, 0, abort_flag) && !*abort_flag;
  const bool warp_ok = __all_sync(0xffffffffu, got);
  tc_fence_after();
  const int q = warp & 3, half = warp >> 2;
  const int nchunks = p.N / 16, nc0 = (nchunks + 1) / 2;
  const int cbeg = half ? nc0 : 0, cend = half ? nchunks : nc0;
  const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
  __shared__ float merge_v[kRtThreads][KK];  // per-thread selections, merged per token
  __shared__ int merge_i[kRtThreads][KK];
  // Selection: order by (logit descending, expert ascending).  The experts a thread sees are
  // spread over kChains chains; each chain sees its experts in ascending order and keeps its k
  // best by insertion with a strict ">" (an equal logit never displaces the lower index seen
  // first), so every chain holds its exact top k; chains and threads are then merged comparing
  // (logit, index), which gives the exact top k of all experts.  Independent chains keep one
  // thread's compare-and-insert work from being one long dependent sequence.
  constexpr int kChains = 4;
  float bv[kChains][KK];
  int bi[kChains][KK];
  float thr[kChains];
#pragma unroll
  for (int g = 0; g < kChains; ++g) {
    thr[g] = -INFINITY;
#pragma unroll
    for (int j = 0; j < KK; ++j) {
      bv[g][j] = -INFINITY;
      bi[g][j] = 0x7fffffff;
    }
  }
  auto offer = [&](int g, int e, float l) {
    float cv = router_clamp(l + (p.b ? p.b[e] : 0.f), p.rflags);
    if (cv > thr[g]) {
      int ci = e;
#pragma unroll
      for (int j = 0; j < KK; ++j) {
        if (j < p.k && cv > bv[g][j]) {
          const float tv = bv[g][j];
          const int ti = bi[g][j];
          bv[g][j] = cv;
          bi[g][j] = ci;
          cv = tv;
          ci = ti;
        }
      }
      thr[g] = bv[g][0];
#pragma unroll
      for (int j = 1; j < KK; ++j) thr[g] = j < p.k ? bv[g][j] : thr[g];
    }
  };
  int tl, part, nparts;  // token within the tile this thread selects for, its share of the experts
  if (p.ksplit == 1) {
    // two threads per token: warp w reads TMEM lane quarter w & 3 (tokens 32 (w & 3) + lane)
    // and the 16-column chunks of expert half w >> 2
    tl = q * 32 + lane;
    part = half;
    nparts = 2;
    if (warp_ok) {
      for (int c = cbeg; c < cend; ++c) {
        float v[16];
        tmem_ld16(tbase + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c * 16 + i < p.E) offer(i % kChains, c * 16 + i, v[i]);
      }
    }
  } else {
    // The ksplit CTAs of the tile form a cluster; CTA r selects for the tokens
    // [r tpc, (r + 1) tpc), tpc = 128 / ksplit.  Every CTA pushes its slice of each token's logits
    // into the shared memory (the idle ring) of the CTA that owns the token, as
    // stage[slice][expert][token - owner tpc]; after one cluster barrier each CTA adds the slices
    // of its tokens in K order from its own shared memory.
    const int tpc = 128 / p.ksplit;
    float* stage = reinterpret_cast<float*>(smem);
    const int tq = q * 32 + lane;  // this thread's TMEM row
    const uint32_t dst = mapa_shared(smem_u32(stage), (uint32_t)(tq / tpc)) +
                         (uint32_t)(split * p.N * tpc + tq % tpc) * 4u;
    if (warp_ok) {
      for (int c = cbeg; c < cend; ++c) {
        float v[16];
        tmem_ld16(tbase + c * 16, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) st_shared_cluster_f32(dst + (uint32_t)((c * 16 + i) * tpc) * 4u, v[i]);
      }
    }
    cluster_sync_all();  // every slice has arrived (release / acquire at cluster scope)
    nparts = min(kRtThreads / tpc, (p.E + 7) / 8);  // at least 8 experts per thread
    tl = split * tpc + threadIdx.x % tpc;
    part = threadIdx.x / tpc;
    if (part < nparts) {
      const float* mine = stage + threadIdx.x % tpc;
      for (int e0 = part; e0 < p.E; e0 += nparts * kChains) {
        float v[kChains];
#pragma unroll
        for (int g = 0; g < kChains; ++g) v[g] = 0.f;
        for (int sp = 0; sp < p.ksplit; ++sp) {
#pragma unroll
          for (int g = 0; g < kChains; ++g) {
            const int e = e0 + g * nparts;
            v[g] += e < p.E ? mine[(sp * p.N + e) * tpc] : 0.f;
          }
        }
#pragma unroll
        for (int g = 0; g < kChains; ++g)
          if (e0 + g * nparts < p.E) offer(g, e0 + g * nparts, v[g]);
      }
    }
  }
  const bool select = __syncthreads_and(warp_ok) != 0;
  if (select) {
#pragma unroll
    for (int g = 1; g < kChains; ++g)
#pragma unroll
      for (int j = 0; j < KK; ++j)
        if (j < p.k) rt_insert_ordered<KK>(bv[0], bi[0], p.k, bv[g][j], bi[g][j]);
#pragma unroll
    for (int j = 0; j < KK; ++j) {
      merge_v[threadIdx.x][j] = bv[0][j];
      merge_i[threadIdx.x][j] = bi[0][j];
    }
  }
  __syncthreads();
  const int t = row0 + tl;
  if (select && part == 0) {
    const int stride = p.ksplit == 1 ? 128 : 128 / p.ksplit;  // threads of one token: tid + m * stride
    for (int m = 1; m < nparts; ++m) {
      const int o = threadIdx.x + m * stride;
#pragma unroll
      for (int j = 0; j < KK; ++j)
        if (j < p.k) rt_insert_ordered<KK>(bv[0], bi[0], p.k, merge_v[o][j], merge_i[o][j]);
    }
    if (t < p.T) {
      float sv[kMaxTopK], wv[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) sv[j] = j < KK ? bv[0][j < KK ? j : 0] : -INFINITY;
      topk_weights(sv, p.k, p.rflags, wv);
#pragma unroll
      for (int j = 0; j < KK; ++j)
        if (j < p.k) {
          p.idx[(size_t)t * p.k + j] = bi[0][j];
          p.w[(size_t)t * p.k + j] = wv[j];
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // copies issued but never consumed: wait (bounded) until they land before the CTA exits
    for (int i = *consumed_s; i < *issued_s; ++i) mbar_wait_bounded(&full[i % S], (uint32_t)(i / S) & 1u);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

constexpr size_t kRtMaxSmem = kRtRingBytes + 1024;

cudaError_t launch_router_tc(const void* x, int T, int d, const void* wr, const float* b, int E, int k,
                             int rflags, int32_t* idx, float* w, uint32_t* err, int ksplit, cudaStream_t s) {
  RouterTcParams p;
  memset(&p, 0, sizeof(p));
  p.N = (E + 15) / 16 * 16;
  {
    const uint64_t dims[2] = {(uint64_t)d, (uint64_t)T}, st[1] = {(uint64_t)d * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_bf16_tmap(&p.mapX, x, 2, dims, st, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)d, (uint64_t)E}, st[1] = {(uint64_t)d * 2};
    const uint32_t box[2] = {64, (uint32_t)p.N};
    if (!make_bf16_tmap(&p.mapW, wr, 2, dims, st, box)) return cudaErrorInvalidValue;
  }
  p.b = b;
  p.T = T;
  p.d = d;
  p.E = E;
  p.k = k;
  p.rflags = rflags;
  // two consecutive K blocks per stage when the slice has an even number of them (256 contiguous
  // bytes of each x row per copy pair instead of 128)
  auto ring = [&](int ks) {
    p.ksplit = ks;
    p.kbs = ((d / ks) / 64) % 2 == 0 ? 2 : 1;
    p.stage_bytes = (uint32_t)((p.kbs * (kRtABytes + p.N * 128) + 1023) / 1024 * 1024);
    p.stages = (int)std::min<size_t>(kRtMaxStages, kRtRingBytes / p.stage_bytes);
  };
  ring(ksplit);
  // a split tile stages its [N][128] fp32 logits in the ring
  if (ksplit > 1 && (size_t)p.N * 128 * 4 > (size_t)p.stages * p.stage_bytes) ring(1);
  p.tmem_cols = 32;
  while ((int)p.tmem_cols < p.N) p.tmem_cols <<= 1;
  p.idx = idx;
  p.w = w;
  p.err = err;
  const size_t smem = (size_t)p.stages * p.stage_bytes + 1024;
  const dim3 grid(p.ksplit, (T + 127) / 128);
  const unsigned cl = (unsigned)p.ksplit;
  if (k <= 2) return launch_kernel(router_tc_kernel<2>, grid, dim3(kRtThreads), smem, s, cl, p);
  if (k <= 4) return launch_kernel(router_tc_kernel<4>, grid, dim3(kRtThreads), smem, s, cl, p);
  return launch_kernel(router_tc_kernel<8>, grid, dim3(kRtThreads), smem, s, cl, p);
}

}  // namespace

// Largest dynamic shared memory the router kernels use (E = 256 on the SIMT kernel; 256 padded
// experts on the tensor-core kernel), set once per device at context creation.
cudaError_t configure_router_kernels() {
  const int simt = (int)(sizeof(float) * ((size_t)kRouterTT * (kRouterDK + 1) + (size_t)kMaxExperts * (kRouterDK + 1) +
                                          (size_t)kRouterTT * (kMaxExperts + 1)));
  cudaError_t e = cudaFuncSetAttribute(router_topk_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, simt);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(router_topk_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, simt);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(router_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtMaxSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(router_tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtMaxSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(router_tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRtMaxSmem);
  return e;
}

// K slices per 128-token tile: the most (up to 8, dividing the 64-wide K blocks) that keep the
// launch within about one CTA per SM.
int router_ksplit(int T, int d) {
  const int tiles = (T + 127) / 128;
  int ks = 1;
  while (ks < kRouterMaxSplit && tiles * ks * 2 <= kRouterCtaBudget && (d / 64) % (2 * ks) == 0) ks <<= 1;
  return ks;
}

cudaError_t launch_router_topk(const void* x, int act, int T, int d, const void* wr, const float* b,
                               int E, int k, int rflags, int32_t* idx, float* w, uint32_t* err, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (T <= kRouterSmallT) {
    if (act == COLIBRI_BF16)
      return launch_kernel(router_small_kernel<__nv_bfloat16>, dim3(T), dim3(256), 0, s, 1, (const __nv_bfloat16*)x, d,
                           (const __nv_bfloat16*)wr, b, E, k, rflags, idx, w);
    return launch_kernel(router_small_kernel<float>, dim3(T), dim3(256), 0, s, 1, (const float*)x, d,
                         (const float*)wr, b, E, k, rflags, idx, w);
  }
  if (act == COLIBRI_BF16) {
    return launch_router_tc(x, T, d, wr, b, E, k, rflags, idx, w, err, router_ksplit(T, d), s);
  }
  const size_t smem =
      sizeof(float) * ((size_t)kRouterTT * (kRouterDK + 1) + (size_t)E * (kRouterDK + 1) +
                       (size_t)kRouterTT * (E + 1));
  const dim3 grid((T + kRouterTT - 1) / kRouterTT);
  return launch_kernel(router_topk_simt_kernel<float>, grid, dim3(kRouterThreads), smem, s, 1, (const float*)x, T, d,
                       (const float*)wr, b, E, k, rflags, idx, w);
}

}  // namespace colibri
