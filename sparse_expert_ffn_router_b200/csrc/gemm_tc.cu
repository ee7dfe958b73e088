// Expert Compute stage for bf16 weights on 5th-generation tensor cores (sm_100a).
//
// Grouped SwiGLU FFN over the grouped rows of every expert (www.trdm.cn/news/555962 §6.2),
// expert e read at e * stride of one weight buffer (www.mhpq.cn/news/563172 §2.1,
// www.pptc.cn/news/100465 §3.3), weights stored [out, in] so both operands are K-major
// (www.hotelren.com/news/4731937 §4.2, the cuBLASLt layout note):
//
//   gate/up:  acc[r][0:128)   = Xp[r] . W1_e[n0 : n0+128]^T
//             acc[r][128:256) = Xp[r] . W3_e[n0 : n0+128]^T
//             H[r][n0 + c]    = silu(acc[r][c]) * acc[r][128 + c]          (bf16)
//   down:     Yp[r][n0 + c]   = H[r] . W2_e[n0 + c]^T,  c < 256             (bf16)
//
// Optionally the shared expert runs in the same launch as one more group whose rows are the
// T tokens of x (gate/up) or of Hs (down).
//
// Design (one CTA per SM, persistent, 192 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile 256 x 64 (bf16, 128-byte swizzle)
//               into a 4-stage shared-memory ring, completion on an mbarrier (expect-tx).
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators); one thread
//               issues tcgen05.mma (M=128, N=256, K=16) four times per stage and frees the
//               stage with tcgen05.commit; commits the finished accumulator to the epilogue.
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 16 columns, SwiGLU or convert, bf16 stores;
//               releases the accumulator so the next tile's MMAs overlap this epilogue.
// Tiles are numbered by a schedule built on the device from the per-expert row offsets:
// expert-major, then n-tile, then m-tile fastest, so the CTAs running at one time share the same
// weight tile through L2 and each weight byte leaves HBM about once; tiles of experts with a
// single m-tile (weight streaming) are interleaved with the others.  A CTA takes its first tile
// by its index and every later one from a global counter (claimed a few stages before its
// current tile's copies are all issued), so the tiles in flight always form one window of
// consecutive numbers however the CTAs' speeds differ, and a faster CTA simply takes more tiles.
// The producer hands each tile number to the MMA and epilogue roles through a small ring in
// shared memory; the last CTA to finish zeroes the counter for the next launch.
// Every wait is bounded (kWaitTimeoutNs); a wait that gives up sets the error word, makes the
// other roles leave their loops, drains outstanding copies and MMAs and frees TMEM.
#include <cstdlib>

#include "common.cuh"

namespace colibri {
namespace {

constexpr int BM = kTcBM, BN = kTcBN, BK = kTcBK, STAGES = kTcStages;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct alignas(64) TcParams {
  CUtensorMap mapA;     // routed A rows
  CUtensorMap mapA16;   // the same rows, boxes of 16, 32 and 64 rows (light tiles copy only what
  CUtensorMap mapA32;   // their MMAs read)
  CUtensorMap mapA64;
  CUtensorMap mapB16;   // gate/up weights viewed as [d, 16 rows, W1|W3, f / 16, E]: one box holds 4 x
                        // (16 W1 rows, the same 16 W3 rows) (pair light tiles)
  CUtensorMap mapB;     // routed weights
  CUtensorMap mapA_sh;  // shared-expert A rows
  CUtensorMap mapB_sh;  // shared-expert weights
  const int32_t* offsets;
  const int32_t* mt_prefix;
  uint32_t* sched;      // [2] tile counter, finished CTAs; nullptr: static round-robin
  int E;
  int n_tiles, n_tiles_sh;
  int mt_sh, rows_sh;
  int pair_light_rows;  // pair kernel: m-tiles with at most this many rows are swapped tails (<= 64)
  int num_kb, num_kb_sh;
  int n_out, n_out_sh;  // output row widths (elements)
  __nv_bfloat16* out;
  __nv_bfloat16* out_sh;
  uint32_t* err;
};

// Tile numbers in flight between the producer and the other roles (a sentinel -1 ends the loop).
constexpr int kTQ = 4;

struct SmemMisc {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t tq_full[kTQ];
  uint64_t tq_empty[kTQ];
  int32_t tq[kTQ];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int issued;
  int consumed;
  int mt_total;
  int32_t mt[kMaxExperts + 1];
  int32_t off[kMaxExperts + 1];
  int32_t hv[kMaxExperts + 1];  // m-tile prefix over experts with >= 2 m-tiles (compute-bound tiles)
  int32_t lt[kMaxExperts + 1];  // prefix over experts with exactly 1 m-tile (weight-streaming tiles)
};

constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + (size_t)STAGES * STAGE_BYTES + sizeof(SmemMisc);

struct Tile {
  bool sh;
  int e, row0, row_end, n0, num_kb;
  int mtiles;  // m-tiles of the tile's group
};

// An m-tile with at most kLightRows rows is computed with the operands swapped (one-CTA kernel):
// the weight tile is the M side (128 rows per MMA, two MMAs for the tile's 256 weight rows) and
// the tile's rows the N side (N = rows rounded up to 16), so a tile of a few rows costs a few
// percent of a 128 x 256 tile of MMAs and is bound by the stream of its weights.
constexpr int kLightRows = 64;

// Routed tiles come in two classes.  An expert with two or more m-tiles reuses each weight tile
// across its m-tiles (compute-bound); an expert with a single m-tile streams its weights once
// (bound by HBM).  When both classes exist (skewed routing) their tiles are interleaved in
// proportion, so that at any time some CTAs compute while others stream weights, instead of a
// compute-bound phase followed by a bandwidth-bound one.  Within a class the order is
// expert-major, then n-tile, then m-tile fastest (CTAs running together share a weight tile).
template <typename Misc>
__device__ void build_class_prefix(Misc& m, int E) {  // one full warp
  const int lane = threadIdx.x & 31;
  const int C = (E + 31) / 32;
  const int e0 = min(E, lane * C), e1 = min(E, e0 + C);
  int sh = 0, sl = 0;
  for (int e = e0; e < e1; ++e) {
    const int Me = m.mt[e + 1] - m.mt[e];
    sh += Me >= 2 ? Me : 0;
    sl += Me == 1 ? 1 : 0;
  }
  int ih = sh, il = sl;  // inclusive warp prefix
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ih, o), b = __shfl_up_sync(0xffffffffu, il, o);
    if (lane >= o) {
      ih += a;
      il += b;
    }
  }
  int ph = ih - sh, pl = il - sl;
  for (int e = e0; e < e1; ++e) {
    m.hv[e] = ph;
    m.lt[e] = pl;
    const int Me = m.mt[e + 1] - m.mt[e];
    ph += Me >= 2 ? Me : 0;
    pl += Me == 1 ? 1 : 0;
  }
  if (lane == 31) {
    m.hv[E] = ih;
    m.lt[E] = il;
  }
}

// largest e in [0, E) with pre[e] * n_tiles <= L
__device__ __forceinline__ int find_group(const int32_t* pre, int E, int n_tiles, int L) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] * n_tiles <= L) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <typename Misc>
__device__ __forceinline__ Tile decode_tile(const TcParams& p, const Misc& m, int L, int routed_total,
                                            bool gateup, int bm = BM) {
  Tile t;
  const int ncols = gateup ? BN / 2 : BN;
  if (L < routed_total) {
    const int nA = m.hv[p.E] * p.n_tiles, nB = m.lt[p.E] * p.n_tiles;
    const int32_t* pre = m.mt;
    int idx = L;
    if (nA > 0 && nB > 0) {
      const long long tot = (long long)nA + nB;
      const int b = (int)((long long)L * nB / tot);
      const bool light = (int)((long long)(L + 1) * nB / tot) > b;
      pre = light ? m.lt : m.hv;
      idx = light ? b : L - b;
    }
    const int lo = find_group(pre, p.E, p.n_tiles, idx);
    const int Me = m.mt[lo + 1] - m.mt[lo];
    const int Lp = idx - pre[lo] * p.n_tiles;
    const int n = Lp / Me, mm = Lp - n * Me;
    t.sh = false;
    t.mtiles = Me;
    t.e = lo;
    t.row0 = m.off[lo] + mm * bm;
    t.row_end = m.off[lo + 1];
    t.n0 = n * ncols;
    t.num_kb = p.num_kb;
  } else {
    const int Lp = L - routed_total;
    const int n = Lp / p.mt_sh, mm = Lp - n * p.mt_sh;
    t.sh = true;
    t.mtiles = p.mt_sh;
    t.e = 0;
    t.row0 = mm * bm;
    t.row_end = p.rows_sh;
    t.n0 = n * ncols;
    t.num_kb = p.num_kb_sh;
  }
  return t;
}

// Bounded wait that also gives up as soon as another role has aborted (kCluster: acquire at
// cluster scope, for barriers the other CTA of a pair arrives on).
template <bool kCluster = false>
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  auto try_wait = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (try_wait()) return true;
  const unsigned long long t0 = global_ns();
  uint32_t n = 0;
  while (true) {
    if (try_wait()) return true;
    if ((++n & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > kWaitTimeoutNs) return false;
    }
  }
}

// The tile after the current one: from the global counter (offset by the tiles the CTAs took by
// their index), or the static round-robin successor.
__device__ __forceinline__ int claim_next(uint32_t* sched, int L, int nworkers) {
  return sched ? (int)atomicAdd(sched, 1u) + nworkers : L + nworkers;
}

// Called once by every CTA of the launch on its way out, after its last claim: the last one to
// finish zeroes the counters for the next launch (launches of one forward are stream-ordered).
__device__ __forceinline__ void sched_finish(uint32_t* sched) {
  if (!sched) return;
  __threadfence();
  if (atomicAdd(sched + 1, 1u) == gridDim.x - 1) {
    atomicExch(sched, 0u);
    atomicExch(sched + 1, 0u);
  }
}

template <typename Misc>
__device__ __forceinline__ void raise_abort(Misc& m, uint32_t* err) {
  *(volatile int*)&m.abort = 1;
  atomicOr(err, kErrWaitTimeout);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <bool kGateUp>
__global__ void __launch_bounds__(NUM_THREADS, 1) tc_ffn_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  SmemMisc& m = *reinterpret_cast<SmemMisc*>(smem + (size_t)STAGES * STAGE_BYTES);
  volatile int* abort_flag = &m.abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&m.full[s], 1);
      mbar_init(&m.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&m.tfull[a], 1);
      mbar_init(&m.tempty[a], EPI_THREADS);
    }
    for (int i = 0; i < kTQ; ++i) {
      mbar_init(&m.tq_full[i], 1);
      mbar_init(&m.tq_empty[i], 1 + EPI_THREADS / 32);  // the MMA thread and the 4 epilogue warps
    }
    mbar_init(&m.drain, 1);
    m.abort = 0;
    m.issued = 0;
    m.consumed = 0;
    mbar_fence_init();
    tma_prefetch_desc(&p.mapA);
    tma_prefetch_desc(&p.mapA16);
    tma_prefetch_desc(&p.mapA64);
    tma_prefetch_desc(&p.mapB);
    if (p.mt_sh > 0) {
      tma_prefetch_desc(&p.mapA_sh);
      tma_prefetch_desc(&p.mapB_sh);
    }
  }
  pdl_wait();  // below: reads of earlier kernels' output; TMEM once the previous kernel released its own
  if (warp == 1) {
    tmem_alloc(&m.tmem_base, TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) {
    m.mt[i] = p.mt_prefix[i];
    m.off[i] = p.offsets[i];
  }
  __syncthreads();
  if (warp == 0) build_class_prefix(m, p.E);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = m.tmem_base;
  const int routed_total = m.mt[p.E] * p.n_tiles;
  const int total = routed_total + p.mt_sh * p.n_tiles_sh;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      int q = 0;
      uint32_t qph = 0;
      const uint64_t evict_first = l2_evict_first_policy();
      int L = blockIdx.x;
      while (true) {
        // publish the tile number (or the end) to the MMA and epilogue roles
        if (!wait_or_abort(&m.tq_empty[q], qph ^ 1u, abort_flag)) {
          raise_abort(m, p.err);
          break;
        }
        const int Lq = L < total ? L : -1;
        *(volatile int32_t*)&m.tq[q] = Lq;
        mbar_arrive(&m.tq_full[q]);
        if (++q == kTQ) {
          q = 0;
          qph ^= 1u;
        }
        if (Lq < 0) break;
        const Tile t = decode_tile(p, m, L, routed_total, kGateUp);
        const CUtensorMap* mA = t.sh ? &p.mapA_sh : &p.mapA;
        const CUtensorMap* mB = t.sh ? &p.mapB_sh : &p.mapB;
        const int claim_kb = t.num_kb > STAGES ? t.num_kb - STAGES : 0;
        int next = L;
        bool ok = true;
        for (int kb = 0; kb < t.num_kb; ++kb) {
          if (kb == claim_kb) next = claim_next(p.sched, L, (int)gridDim.x);
          if (!wait_or_abort(&m.empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = stage_base + (size_t)s * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          const int kx = kb * BK;
          // a light tile's MMAs read only its first 16 * ceil(rows / 16) rows of A: copy 16 or 64
          const int arows = t.row_end - t.row0;
          const uint32_t a_bytes = t.sh || arows > kLightRows ? (uint32_t)A_BYTES : (arows <= 16 ? 16u : 64u) * BK * 2;
          mbar_arrive_expect_tx(&m.full[s], a_bytes + (uint32_t)B_BYTES);
          tma_load_2d(sA, a_bytes == (uint32_t)A_BYTES ? mA : (arows <= 16 ? &p.mapA16 : &p.mapA64), &m.full[s], kx,
                      t.row0);
          // the weight tile of a group with a single (light) m-tile is read by this tile alone:
          // evict it first from L2
          const bool stream = t.mtiles == 1 && t.row_end - t.row0 <= kLightRows && !t.sh;
          if (kGateUp) {
            if (t.sh) {
              tma_load_3d(sB, mB, &m.full[s], kx, t.n0, 0);
              tma_load_3d(sB + B_BYTES / 2, mB, &m.full[s], kx, t.n0, 1);
            } else if (stream) {
              tma_load_4d_hint(sB, mB, &m.full[s], kx, t.n0, 0, t.e, evict_first);
              tma_load_4d_hint(sB + B_BYTES / 2, mB, &m.full[s], kx, t.n0, 1, t.e, evict_first);
            } else {
              tma_load_4d(sB, mB, &m.full[s], kx, t.n0, 0, t.e);
              tma_load_4d(sB + B_BYTES / 2, mB, &m.full[s], kx, t.n0, 1, t.e);
            }
          } else {
            // down projection: the W2 blocks of an expert with many m-tiles are evicted from L2
            // first (its m-tiles read each block within a short window), so that its H rows stay
            // for the n-tiles that start a tile later (measured: 1.15x -> 1.10x the algorithmic
            // bytes at T=2048 with two experts of ~2000 rows; not used for two m-tiles, where it
            // raised the traffic)
            if (t.sh) tma_load_2d(sB, mB, &m.full[s], kx, t.n0);
            else if (stream || t.mtiles > 2) tma_load_3d_hint(sB, mB, &m.full[s], kx, t.n0, t.e, evict_first);
            else tma_load_3d(sB, mB, &m.full[s], kx, t.n0, t.e);
          }
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          raise_abort(m, p.err);
          break;
        }
        L = next;
      }
      m.issued = issued;
    }
    pdl_trigger();  // every copy of this CTA is issued: let the next kernel be scheduled
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0, consumed = 0;
      int q = 0;
      uint32_t qph = 0;
      bool ok = true;
      for (;; ++it) {
        if (!wait_or_abort(&m.tq_full[q], qph, abort_flag)) {
          ok = false;
          break;
        }
        const int L = *(volatile int32_t*)&m.tq[q];
        mbar_arrive(&m.tq_empty[q]);
        if (++q == kTQ) {
          q = 0;
          qph ^= 1u;
        }
        if (L < 0) break;
        const Tile t = decode_tile(p, m, L, routed_total, kGateUp);
        const int a = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!wait_or_abort(&m.tempty[a], aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(a * BN);
        const int rows = t.row_end - t.row0;
        const bool light = rows <= kLightRows;
        const uint32_t idesc_l = idesc_bf16_f32(128, (rows + 15) / 16 * 16);
        for (int kb = 0; kb < t.num_kb; ++kb) {
          if (!wait_or_abort(&m.full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(stage_base + (size_t)s * STAGE_BYTES);
          const uint32_t sB = sA + A_BYTES;
          if (light) {
            // swapped: weight rows [0,128) -> columns [0,N), rows [128,256) -> columns [128,128+N)
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t xd = smem_desc_sw128(sA + kk * 32);
              const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
              tc_mma_f16(d_tmem, smem_desc_sw128(sB + kk * 32), xd, idesc_l, acc);
              tc_mma_f16(d_tmem + 128, smem_desc_sw128(sB + B_BYTES / 2 + kk * 32), xd, idesc_l, acc);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(sA + kk * 32);
              const uint64_t bd = smem_desc_sw128(sB + kk * 32);
              tc_mma_f16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&m.empty[s]);
          ++consumed;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&m.tfull[a]);
      }
      if (!ok) raise_abort(m, p.err);
      m.consumed = consumed;
      // drain: wait until every MMA issued by this thread has completed
      tc_commit(&m.drain);
      mbar_wait_bounded(&m.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int tq = 0;
    uint32_t tqph = 0;
    for (int it = 0;; ++it) {
      const bool gq = wait_or_abort(&m.tq_full[tq], tqph, abort_flag);
      if (!__all_sync(0xffffffffu, gq)) {
        if (lane == 0) raise_abort(m, p.err);
        break;
      }
      const int L = *(volatile int32_t*)&m.tq[tq];
      __syncwarp();
      if (lane == 0) mbar_arrive(&m.tq_empty[tq]);
      if (++tq == kTQ) {
        tq = 0;
        tqph ^= 1u;
      }
      if (L < 0) break;
      const Tile t = decode_tile(p, m, L, routed_total, kGateUp);
      const int a = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      const bool got = wait_or_abort(&m.tfull[a], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) raise_abort(m, p.err);
        break;
      }
      tc_fence_after();
      const int row = t.row0 + q * 32 + lane;
      const bool valid = row < t.row_end;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * BN);
      __nv_bfloat16* out = t.sh ? p.out_sh : p.out;
      const int n_out = t.sh ? p.n_out_sh : p.n_out;
      const int rows = t.row_end - t.row0;
      if (rows <= kLightRows) {
        // swapped tile: TMEM lane = weight row (output column), TMEM column = the tile's row
        const int ch = q * 32 + lane;  // gate/up: column n0 + ch; down: n0 + ch and n0 + 128 + ch
        for (int j0 = 0; j0 < rows; j0 += 16) {
          float v0[16], v1[16];
          tmem_ld16(tb + j0, v0);
          tmem_ld16(tb + 128 + j0, v1);
          tmem_ld_wait();
          if (kGateUp) {
            if (t.n0 + ch < n_out) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (j0 + i < rows)
                  out[(size_t)(t.row0 + j0 + i) * n_out + t.n0 + ch] = __float2bfloat16_rn(silu_mul(v0[i], v1[i]));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (j0 + i < rows) {
                __nv_bfloat16* o = out + (size_t)(t.row0 + j0 + i) * n_out + t.n0 + ch;
                if (t.n0 + ch < n_out) o[0] = __float2bfloat16_rn(v0[i]);
                if (t.n0 + 128 + ch < n_out) o[128] = __float2bfloat16_rn(v1[i]);
              }
            }
          }
        }
      } else if (kGateUp) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 16) {
          float g[16], u[16];
          tmem_ld16(tb + c, g);
          tmem_ld16(tb + BN / 2 + c, u);
          tmem_ld_wait();
          if (valid && t.n0 + c < n_out) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_bf16x2(silu_mul(g[2 * i], u[2 * i]), silu_mul(g[2 * i + 1], u[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * n_out + t.n0 + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(tb + c, v);
          tmem_ld_wait();
          if (valid && t.n0 + c < n_out) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * n_out + t.n0 + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&m.tempty[a]);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && m.abort) {
    // copies issued but never consumed: wait (bounded) until they land before exiting
    for (int i = m.consumed; i < m.issued; ++i)
      mbar_wait_bounded(&m.full[i % STAGES], (uint32_t)(i / STAGES) & 1u);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0) sched_finish(p.sched);
}

// ------------------------------------------------------------------------- pair kernel
// The same grouped GEMM with clusters of two CTAs and tcgen05 cta_group::2: a pair computes a
// 256 x 256 tile; each CTA loads its own 128 rows of A and its own 128 rows (N) of B (for
// gate/up: the leader W1, the peer W3), so a stage is 32 KB and six stages fit.  The leader
// issues the M=256 MMAs, which read both CTAs' shared memory and write 128 rows into each
// CTA's TMEM; its commits arrive on both CTAs' barriers (multicast commit).  Both CTAs' copies
// count on the leader's full barrier; both epilogues release the accumulator on the leader's
// barrier.  Per 128x256x64 unit of work a CTA moves 32 KB from L2 instead of 48 KB.
constexpr int BM2 = 256;
constexpr int STAGES2 = kTcPairStages;
// A pair m-tile with at most kPairLightRows rows (an expert's short last tile) is computed with
// the operands swapped, like the one-CTA light tiles: the weights are the M = 256 side (128 rows
// per CTA) and the tile's rows the N side (N = rows rounded up to 16, N / 2 rows per CTA), so the
// tail costs a fraction of a 256 x 256 tile and still reads its weight blocks from L2 in the same
// launch as the expert's other m-tiles.  For gate/up each CTA's 128 weight rows are 4 x (16 W1
// rows, the same 16 W3 rows), so that gate and up of one output column meet in one warp.
constexpr int kPairLightRows = 128;  // N <= 128: at most 64 token rows per CTA (a 32- or 64-row box)
constexpr int HALF_BYTES = 128 * BK * 2;          // 16 KB
constexpr int STAGE2_BYTES = 2 * HALF_BYTES;      // A half + B half
constexpr uint32_t IDESC2 = idesc_bf16_f32(BM2, BN);

struct SmemMisc2 {
  uint64_t full[STAGES2];    // used in the leader: both CTAs' copies (64 KB per phase)
  uint64_t empty[STAGES2];   // per CTA: freed by the leader's multicast commit
  uint64_t tfull[2];         // per CTA: accumulator ready (multicast commit)
  uint64_t tempty[2];        // used in the leader: 8 epilogue-warp arrivals (4 local, 4 peer)
  uint64_t tq_full[kTQ];     // per CTA: tile number published by the leader's producer
  uint64_t tq_empty[kTQ];    // used in the leader: MMA thread, peer producer, 8 epilogue warps
  int32_t tq[kTQ];           // per CTA: the leader writes both CTAs' copies
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int32_t mt[kMaxExperts + 1];
  int32_t off[kMaxExperts + 1];
  int32_t hv[kMaxExperts + 1];
  int32_t lt[kMaxExperts + 1];
};

// Light tails of at most 32 rows ("dense" light tiles) put the weights of two K blocks in a stage
// (A and B slots) and their 16-row token boxes in a ring of their own, so that the stream of
// weights has twice the bytes in flight
constexpr int kDenseLightRows = 32;
constexpr int TOK_BYTES = 16 * BK * 2;  // one 16-row token box
constexpr size_t TOK2_RING = (size_t)STAGES2 * 2 * TOK_BYTES;
constexpr size_t SMEM2_BYTES = (size_t)STAGES2 * STAGE2_BYTES + TOK2_RING + sizeof(SmemMisc2);
static_assert(SMEM2_BYTES <= 232448, "pair-tile stages exceed the shared memory of one CTA");

template <bool kGateUp>
__global__ void __launch_bounds__(NUM_THREADS, 1) tc2_ffn_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzle needs 1024-byte aligned stages; the dynamic shared window of a CTA
  // starts 1024-byte aligned (both CTAs of a pair take this branch together).
  if (smem_u32(smem_raw) & 1023u) {
    pdl_wait();
    if (threadIdx.x == 0) {
      atomicOr(p.err, kErrWaitTimeout);
      sched_finish(p.sched);
    }
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* stage_base = smem;
  uint8_t* tok_base = smem + (size_t)STAGES2 * STAGE2_BYTES;  // [STAGES2][2] token boxes (dense light tiles)
  SmemMisc2& m = *reinterpret_cast<SmemMisc2*>(smem + (size_t)STAGES2 * STAGE2_BYTES + TOK2_RING);
  volatile int* abort_flag = &m.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = (int)cluster_id_x(), npairs = (int)num_clusters_x();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(&m.full[s], 1);
      mbar_init(&m.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&m.tfull[a], 1);
      mbar_init(&m.tempty[a], 8);
    }
    for (int i = 0; i < kTQ; ++i) {
      mbar_init(&m.tq_full[i], 1);
      mbar_init(&m.tq_empty[i], 2 + 8);
    }
    mbar_init(&m.drain, 1);
    m.abort = 0;
    mbar_fence_init();
    tma_prefetch_desc(&p.mapA);
    tma_prefetch_desc(&p.mapB);
    tma_prefetch_desc(&p.mapA32);
    tma_prefetch_desc(&p.mapA16);
    tma_prefetch_desc(&p.mapA64);
    if (kGateUp) tma_prefetch_desc(&p.mapB16);
    if (p.mt_sh > 0) {
      tma_prefetch_desc(&p.mapA_sh);
      tma_prefetch_desc(&p.mapB_sh);
    }
  }
  pdl_wait();  // below: reads of earlier kernels' output; TMEM once the previous kernel released its own
  if (warp == 1) {
    tmem_alloc_pair(&m.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  for (int i = threadIdx.x; i <= p.E; i += NUM_THREADS) {
    m.mt[i] = p.mt_prefix[i];
    m.off[i] = p.offsets[i];
  }
  __syncthreads();
  if (warp == 0) build_class_prefix(m, p.E);
  __syncthreads();
  cluster_sync_all();  // the peer's barriers are initialised before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem_base = m.tmem_base;
  const int routed_total = m.mt[p.E] * p.n_tiles;
  const int total = routed_total + p.mt_sh * p.n_tiles_sh;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int q = 0;
      uint32_t qph = 0;
      int L = pair;
      const uint64_t evict_first = l2_evict_first_policy();
      while (true) {
        // the leader claims tiles and publishes each number to both CTAs; the peer reads its copy
        int Lq;
        if (rank == 0) {
          if (!wait_or_abort<true>(&m.tq_empty[q], qph ^ 1u, abort_flag)) {
            raise_abort(m, p.err);
            break;
          }
          Lq = L < total ? L : -1;
          *(volatile int32_t*)&m.tq[q] = Lq;
          st_shared_cluster_u32(mapa_shared(smem_u32(&m.tq[q]), 1), Lq);
          mbar_arrive(&m.tq_full[q]);
          mbar_arrive_cluster(mapa_shared(smem_u32(&m.tq_full[q]), 1));
        } else {
          if (!wait_or_abort<true>(&m.tq_full[q], qph, abort_flag)) {
            raise_abort(m, p.err);
            break;
          }
          Lq = *(volatile int32_t*)&m.tq[q];
          mbar_arrive_cluster(mapa_shared(smem_u32(&m.tq_empty[q]), 0));
        }
        if (++q == kTQ) {
          q = 0;
          qph ^= 1u;
        }
        if (Lq < 0) break;
        L = Lq;
        const Tile t = decode_tile(p, m, L, routed_total, kGateUp, BM2);
        const CUtensorMap* mA = t.sh ? &p.mapA_sh : &p.mapA;
        const CUtensorMap* mB = t.sh ? &p.mapB_sh : &p.mapB;
        const int arow = t.row0 + 128 * (int)rank;
        const bool light = !t.sh && t.row_end - t.row0 <= p.pair_light_rows;
        const bool dense = light && t.row_end - t.row0 <= kDenseLightRows;
        const int nh = (t.row_end - t.row0 + 15) / 16 * 8;  // light: token rows (N / 2) per CTA
        const int nsteps = dense ? (t.num_kb + 1) / 2 : t.num_kb;  // ring stages of the tile
        const int claim_step = nsteps > STAGES2 ? nsteps - STAGES2 : 0;
        int next = L;
        bool ok = true;
        for (int step = 0; step < nsteps; ++step) {
          if (rank == 0 && step == claim_step) next = claim_next(p.sched, L, npairs);
          if (!wait_or_abort(&m.empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = stage_base + (size_t)s * STAGE2_BYTES;
          uint8_t* sB = sA + HALF_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&m.full[s]), 0);
          const int kb = dense ? 2 * step : step;
          const int kx = kb * BK;
          if (dense) {
            // two K blocks of weights (A and B slots), their token boxes in the token ring
            const int nk = min(2, t.num_kb - kb);
            if (rank == 0) mbar_arrive_expect_tx(&m.full[s], (uint32_t)(2 * nk * (HALF_BYTES + TOK_BYTES)));
            for (int j = 0; j < nk; ++j) {
              uint8_t* wdst = sA + (size_t)j * HALF_BYTES;
              const int kxj = kx + j * BK;
              if (kGateUp) {
                if (t.mtiles == 1)
                  tma2_load_5d_hint(wdst, &p.mapB16, bar, kxj, 0, 0, (t.n0 + 64 * (int)rank) / 16, t.e, evict_first);
                else
                  tma2_load_5d(wdst, &p.mapB16, bar, kxj, 0, 0, (t.n0 + 64 * (int)rank) / 16, t.e);
              } else {
                if (t.mtiles == 1) tma2_load_3d_hint(wdst, mB, bar, kxj, t.n0 + 128 * (int)rank, t.e, evict_first);
                else tma2_load_3d(wdst, mB, bar, kxj, t.n0 + 128 * (int)rank, t.e);
              }
              tma2_load_2d(tok_base + (size_t)(2 * s + j) * TOK_BYTES, &p.mapA16, bar, kxj, t.row0 + (int)rank * nh);
            }
          } else if (light) {
            // swapped tail: weights into the A slot, the tile's token rows into the B slot
            const int box_rows = nh <= 32 ? 32 : 64;
            if (rank == 0) mbar_arrive_expect_tx(&m.full[s], 2 * (HALF_BYTES + box_rows * BK * 2));
            // an expert with this single m-tile streams its weights: evict them from L2 first
            if (kGateUp) {
              if (t.mtiles == 1)
                tma2_load_5d_hint(sA, &p.mapB16, bar, kx, 0, 0, (t.n0 + 64 * (int)rank) / 16, t.e, evict_first);
              else
                tma2_load_5d(sA, &p.mapB16, bar, kx, 0, 0, (t.n0 + 64 * (int)rank) / 16, t.e);
            } else {
              if (t.mtiles == 1) tma2_load_3d_hint(sA, mB, bar, kx, t.n0 + 128 * (int)rank, t.e, evict_first);
              else tma2_load_3d(sA, mB, bar, kx, t.n0 + 128 * (int)rank, t.e);
            }
            tma2_load_2d(sB, nh <= 32 ? &p.mapA32 : &p.mapA64, bar, kx, t.row0 + (int)rank * nh);
          } else {
            if (rank == 0) mbar_arrive_expect_tx(&m.full[s], 2 * STAGE2_BYTES);
            tma2_load_2d(sA, mA, bar, kx, arow);
            if (kGateUp) {
              if (t.sh) tma2_load_3d(sB, mB, bar, kx, t.n0, (int)rank);
              else tma2_load_4d(sB, mB, bar, kx, t.n0, (int)rank, t.e);
            } else {
              if (t.sh) tma2_load_2d(sB, mB, bar, kx, t.n0 + 128 * (int)rank);
              else tma2_load_3d(sB, mB, bar, kx, t.n0 + 128 * (int)rank, t.e);
            }
          }
          if (++s == STAGES2) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          raise_abort(m, p.err);
          break;
        }
        L = next;
      }
    }
    pdl_trigger();  // every copy of this CTA is issued: let the next kernel be scheduled
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      int q = 0;
      uint32_t qph = 0;
      bool ok = true;
      for (;; ++it) {
        if (!wait_or_abort(&m.tq_full[q], qph, abort_flag)) {
          ok = false;
          break;
        }
        const int L = *(volatile int32_t*)&m.tq[q];
        mbar_arrive(&m.tq_empty[q]);
        if (++q == kTQ) {
          q = 0;
          qph ^= 1u;
        }
        if (L < 0) break;
        const Tile t = decode_tile(p, m, L, routed_total, kGateUp, BM2);
        const int a = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!wait_or_abort(&m.tempty[a], aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(a * BN);
        const int trows = t.row_end - t.row0;
        // light tail: M = 256 weight rows, N = the tile's rows rounded up to 16
        const bool light = !t.sh && trows <= p.pair_light_rows;
        const bool dense = light && trows <= kDenseLightRows;
        const uint32_t idesc = light ? idesc_bf16_f32(BM2, (trows + 15) / 16 * 16) : IDESC2;
        const int nsteps = dense ? (t.num_kb + 1) / 2 : t.num_kb;
        for (int step = 0; step < nsteps; ++step) {
          if (!wait_or_abort(&m.full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(stage_base + (size_t)s * STAGE2_BYTES);
          const uint32_t sB = sA + HALF_BYTES;
          if (dense) {
            const int nk = min(2, t.num_kb - 2 * step);
            for (int j = 0; j < nk; ++j) {
              const uint32_t wa = sA + (uint32_t)(j * HALF_BYTES);
              const uint32_t tb = smem_u32(tok_base + (size_t)(2 * s + j) * TOK_BYTES);
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                tc_mma_f16_pair(d_tmem, smem_desc_sw128(wa + kk * 32), smem_desc_sw128(tb + kk * 32), idesc,
                                (step | j | kk) != 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(sA + kk * 32);
              const uint64_t bd = smem_desc_sw128(sB + kk * 32);
              tc_mma_f16_pair(d_tmem, ad, bd, idesc, (step | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit_pair_mc(&m.empty[s], 0x3);
          if (++s == STAGES2) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&m.tfull[a], 0x3);
      }
      if (!ok) raise_abort(m, p.err);
      tc_commit_pair(&m.drain);
      mbar_wait_bounded(&m.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&m.tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&m.tempty[1]), 0);
    int tq = 0;
    uint32_t tqph = 0;
    for (int it = 0;; ++it) {
      const bool gq = wait_or_abort<true>(&m.tq_full[tq], tqph, abort_flag);
      if (!__all_sync(0xffffffffu, gq)) {
        if (lane == 0) raise_abort(m, p.err);
        break;
      }
      const int L = *(volatile int32_t*)&m.tq[tq];
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&m.tq_empty[tq]), 0));
      if (++tq == kTQ) {
        tq = 0;
        tqph ^= 1u;
      }
      if (L < 0) break;
      const Tile t = decode_tile(p, m, L, routed_total, kGateUp, BM2);
      const int a = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      const bool got = wait_or_abort(&m.tfull[a], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) raise_abort(m, p.err);
        break;
      }
      tc_fence_after();
      const int row = t.row0 + 128 * (int)rank + q * 32 + lane;
      const bool valid = row < t.row_end;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * BN);
      __nv_bfloat16* out = t.sh ? p.out_sh : p.out;
      const int n_out = t.sh ? p.n_out_sh : p.n_out;
      const int trows = t.row_end - t.row0;
      if (!t.sh && trows <= p.pair_light_rows) {
        // swapped tail: TMEM lane = weight row of this CTA, column c = the tile's row t.row0 + c
        if (kGateUp) {
          // lanes 0-15 of warp q: gate of output column n0 + 64 rank + 16 q + lane; lanes 16-31: up
          const int oc = t.n0 + 64 * (int)rank + 16 * q + (lane & 15);
          for (int c = 0; c < trows; c += 16) {
            float v[16];
            tmem_ld16(tb + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float up = __shfl_down_sync(0xffffffffu, v[i], 16);
              if (lane < 16 && c + i < trows && oc < n_out)
                out[(size_t)(t.row0 + c + i) * n_out + oc] = __float2bfloat16_rn(silu_mul(v[i], up));
            }
          }
        } else {
          const int oc = t.n0 + 128 * (int)rank + q * 32 + lane;
          for (int c = 0; c < trows; c += 16) {
            float v[16];
            tmem_ld16(tb + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c + i < trows && oc < n_out) out[(size_t)(t.row0 + c + i) * n_out + oc] = __float2bfloat16_rn(v[i]);
          }
        }
      } else if (kGateUp) {
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 16) {
          float g[16], u[16];
          tmem_ld16(tb + c, g);
          tmem_ld16(tb + BN / 2 + c, u);
          tmem_ld_wait();
          if (valid && t.n0 + c < n_out) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pk[i] = pack_bf16x2(silu_mul(g[2 * i], u[2 * i]), silu_mul(g[2 * i + 1], u[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * n_out + t.n0 + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(tb + c, v);
          tmem_ld_wait();
          if (valid && t.n0 + c < n_out) {
            uint32_t pk[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * n_out + t.n0 + c);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(a ? tempty_leader1 : tempty_leader0);
    }
  }

  __syncthreads();
  if (threadIdx.x == 0 && m.abort) {
    // error path: give copies still in flight time to land before the CTA leaves
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < 2000000ull) {
    }
  }
  cluster_sync_all();  // the peer no longer reads this CTA's shared memory or arrives on it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0) sched_finish(p.sched);
}

// ------------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

// bf16 tensor map with a 64-element (128-byte) inner box and 128-byte swizzle; out-of-bounds
// elements of a box read as zero.
bool make_bf16_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box) {
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box);
}

bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  const CUresult r = enc(map, dtype, (cuuint32_t)rank, const_cast<void*>(base),
                         gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

bool make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  return make_bf16_tmap(map, base, rank, dims, strides_bytes, box);
}

template <bool kGateUp>
cudaError_t launch_tc(const TcGemmArgs& a, cudaStream_t s) {
  const bool pair = a.pair;
  const int bm = pair ? BM2 : BM;
  const uint32_t b_rows_down = pair ? 128 : BN;
  TcParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t d = a.d, f = a.f, fs = a.fs;
  const uint64_t S = (uint64_t)a.wstride * 2;  // bytes between experts
  bool ok = true;
  if (kGateUp) {
    // A: grouped rows Xp [rows, d] (and the light tiles' 16- and 64-row boxes)
    { uint64_t dims[2] = {d, (uint64_t)a.rows}, st[1] = {d * 2}; uint32_t box[2] = {BK, BM};
      ok &= make_map(&p.mapA, a.A, 2, dims, st, box);
      box[1] = 16;
      ok &= make_map(&p.mapA16, a.A, 2, dims, st, box);
      box[1] = 32;
      ok &= make_map(&p.mapA32, a.A, 2, dims, st, box);
      box[1] = 64;
      ok &= make_map(&p.mapA64, a.A, 2, dims, st, box); }
    // B: W1|W3 of every expert as [d, f, 2, E] (and in 16-row boxes)
    { uint64_t dims[4] = {d, f, 2, (uint64_t)a.E}, st[3] = {d * 2, f * d * 2, S};
      uint32_t box[4] = {BK, BN / 2, 1, 1};
      ok &= make_map(&p.mapB, a.W, 4, dims, st, box); }
    { uint64_t dims[5] = {d, 16, 2, f / 16, (uint64_t)a.E}, st[4] = {d * 2, f * d * 2, 16 * d * 2, S};
      uint32_t box[5] = {BK, 16, 2, 4, 1};
      ok &= f % 16 == 0 && make_map(&p.mapB16, a.W, 5, dims, st, box); }
    if (a.fs > 0) {
      { uint64_t dims[2] = {d, (uint64_t)a.rows_sh}, st[1] = {d * 2}; uint32_t box[2] = {BK, BM};
        ok &= make_map(&p.mapA_sh, a.A_sh, 2, dims, st, box); }
      { uint64_t dims[3] = {d, fs, 2}, st[2] = {d * 2, fs * d * 2}; uint32_t box[3] = {BK, BN / 2, 1};
        ok &= make_map(&p.mapB_sh, a.W_sh, 3, dims, st, box); }
    }
    p.n_tiles = (int)((f + BN / 2 - 1) / (BN / 2));
    p.n_tiles_sh = a.fs > 0 ? (int)((fs + BN / 2 - 1) / (BN / 2)) : 0;
    p.num_kb = (int)((d + BK - 1) / BK);
    p.num_kb_sh = p.num_kb;
    p.n_out = (int)f;
    p.n_out_sh = (int)fs;
  } else {
    // A: H [rows, f] (and the light tiles' 16- and 64-row boxes)
    { uint64_t dims[2] = {f, (uint64_t)a.rows}, st[1] = {f * 2}; uint32_t box[2] = {BK, BM};
      ok &= make_map(&p.mapA, a.A, 2, dims, st, box);
      box[1] = 16;
      ok &= make_map(&p.mapA16, a.A, 2, dims, st, box);
      box[1] = 32;
      ok &= make_map(&p.mapA32, a.A, 2, dims, st, box);
      box[1] = 64;
      ok &= make_map(&p.mapA64, a.A, 2, dims, st, box); }
    // B: W2 of every expert as [f, d, E], starting 2*f*d elements into the expert
    { uint64_t dims[3] = {f, d, (uint64_t)a.E}, st[2] = {f * 2, S}; uint32_t box[3] = {BK, b_rows_down, 1};
      ok &= make_map(&p.mapB, (const __nv_bfloat16*)a.W + 2 * f * d, 3, dims, st, box); }
    if (a.fs > 0) {
      { uint64_t dims[2] = {fs, (uint64_t)a.rows_sh}, st[1] = {fs * 2}; uint32_t box[2] = {BK, BM};
        ok &= make_map(&p.mapA_sh, a.A_sh, 2, dims, st, box); }
      { uint64_t dims[2] = {fs, d}, st[1] = {fs * 2}; uint32_t box[2] = {BK, b_rows_down};
        ok &= make_map(&p.mapB_sh, (const __nv_bfloat16*)a.W_sh + 2 * fs * d, 2, dims, st, box); }
    }
    p.n_tiles = (int)((d + BN - 1) / BN);
    p.n_tiles_sh = a.fs > 0 ? p.n_tiles : 0;
    p.num_kb = (int)((f + BK - 1) / BK);
    p.num_kb_sh = a.fs > 0 ? (int)((fs + BK - 1) / BK) : 0;
    p.n_out = (int)d;
    p.n_out_sh = (int)d;
  }
  if (!ok) return cudaErrorInvalidValue;
  p.offsets = a.offsets;
  p.mt_prefix = a.mt_prefix;
  p.sched = a.sched;
  p.E = a.E;
  p.mt_sh = a.fs > 0 ? (a.rows_sh + bm - 1) / bm : 0;
  p.rows_sh = a.rows_sh;
  {
    // COLIBRI_PAIR_LIGHT=0 computes every pair m-tile as a full 256 x 256 tile
    const char* v = getenv("COLIBRI_PAIR_LIGHT");
    p.pair_light_rows = v && atoi(v) == 0 ? 0 : kPairLightRows;
  }
  p.out = (__nv_bfloat16*)a.out;
  p.out_sh = (__nv_bfloat16*)a.out_sh;
  p.err = a.err;
  const long long bound = (long long)a.mt_bound * p.n_tiles + (long long)p.mt_sh * p.n_tiles_sh;
  if (!pair) {
    int grid = a.sm_count;
    if (bound < grid) grid = (int)bound;
    if (grid <= 0) return cudaSuccess;
    return launch_kernel(tc_ffn_kernel<kGateUp>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, s, 1, p);
  }
  int pairs = a.sm_count / 2;
  if (bound < pairs) pairs = (int)bound;
  if (pairs <= 0) return cudaSuccess;
  return launch_kernel(tc2_ffn_kernel<kGateUp>, dim3(2 * pairs), dim3(NUM_THREADS), SMEM2_BYTES, s, 2, p);
}

}  // namespace

// Done once per device at context creation, so that nothing in the launch path is a
// non-stream call (the launch sequence can then be captured into a CUDA graph).
cudaError_t configure_tc_kernels() {
  cudaError_t e = cudaFuncSetAttribute(tc_ffn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc_ffn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc2_ffn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM2_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc2_ffn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM2_BYTES);
  if (e == cudaSuccess && !get_encode()) e = cudaErrorNotSupported;
  return e;
}

cudaError_t launch_tc_gateup(const TcGemmArgs& a, cudaStream_t s) { return launch_tc<true>(a, s); }
cudaError_t launch_tc_down(const TcGemmArgs& a, cudaStream_t s) { return launch_tc<false>(a, s); }

}  // namespace colibri
