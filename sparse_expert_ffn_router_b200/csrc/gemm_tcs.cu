// Expert Compute stage for bf16 weights with the operands swapped: the weights are the M side of
// the tensor-core product (128 output channels per tile) and the grouped token rows the N side
// (16 to 256 rows, a multiple of 16).  Same arithmetic as the other grouped GEMMs
// (www.trdm.cn/news/555962 §6.2 grouping, www.mhpq.cn/news/563172 §2.1 fixed expert stride):
//
//   gate/up:  G[c][j] = W1_e[c0 + c] . X[r0 + j],   U[c][j] = W3_e[c0 + c] . X[r0 + j]
//             H[r0 + j][c0 + c] = silu(G[c][j]) * U[c][j]                           (bf16)
//   down:     Yp[r0 + j][c0 + c] = W2_e[c0 + c] . H[r0 + j]                         (bf16)
//
// A tile covers the group's remaining rows rounded up to 16 instead of a fixed 128 or 256, so
// experts that received a few hundred rows (fine-grained routing) compute little padding, and an
// expert with a handful of rows (skewed routing) costs the stream of its weights rather than a
// full tile of MMAs.
//
// Pipeline (one persistent CTA per SM, 192 threads), as in the other grouped GEMMs:
//   warp 0      TMA producer: per 64-wide K block the weight tile(s) (128 x 64, W1 and W3 for
//               gate/up) and the token rows (one or two boxes of 16 rows, else boxes of 64
//               rows), 128-byte swizzle, into a 4-stage ring of 48 KB;
//   warp 1      allocates 512 TMEM columns (two accumulators of 256 columns); one thread issues
//               tcgen05.mma (M=128, N=16..256, K=16) -- for gate/up two per K step, G into
//               columns [0, 128) and U into [128, 256) of the accumulator;
//   warps 2-5   epilogue: TMEM lane = output channel, column = token; SwiGLU or convert, bf16
//               stores; releases the accumulator so the next tile's MMAs overlap it.
// Work items (group, 128-channel tile, token chunk) are built on the device from the row
// offsets: group-major, then channel tile, then chunk fastest, so the CTAs running together
// share one weight tile through L2.  Groups with a single chunk (weight streaming) are
// interleaved in proportion with the others (compute-bound), so HBM and the tensor cores are
// busy at the same time.  The shared expert is one more group.  Every wait is bounded.
#include "common.cuh"

namespace colibri {
namespace {

constexpr int SW_THREADS = 192;
constexpr int SW_EPI_THREADS = 128;
constexpr int SW_BK = 64;                       // K elements per stage (128 bytes of bf16)
constexpr int SW_W_BYTES = 128 * SW_BK * 2;     // 16 KB: one 128-channel weight tile
constexpr int SW_BOX_ROWS = 16;                 // MMA N granularity; token rows of the small TMA box
constexpr int SW_BIG_ROWS = 64;                 // token rows of the large TMA box
constexpr int SW_STAGE_BYTES = 48 * 1024;       // gate/up: W1 + W3 + 128 rows; down: W2 + 256 rows
constexpr int SW_STAGES = 4;
constexpr int SW_TMEM_COLS = 512;
constexpr int SW_ACC_COLS = 256;
constexpr int SW_NT_GATEUP = 128;               // token rows per chunk
constexpr int SW_NT_DOWN = 256;
constexpr int SW_MAX_GROUPS = kMaxExperts + 1;  // routed experts + the shared expert

struct alignas(64) SwParams {
  CUtensorMap mapW;     // routed weights: gate/up [d, f, 2, E], down [f, d, E]; box 64 x 128
  CUtensorMap mapX;     // routed token rows [rows, K]; box 64 x 16
  CUtensorMap mapX64;   // the same rows; box 64 x 64
  CUtensorMap mapW_sh;  // shared-expert weights: gate/up [d, f_s, 2], down [f_s, d]
  CUtensorMap mapX_sh;  // shared-expert rows [T, K]; boxes 64 x 16 and 64 x 64
  CUtensorMap mapX64_sh;
  const int32_t* offsets;  // [E+1]
  int E;
  int rows_sh;             // rows of the shared expert (T), 0 = none
  int n_out, n_out_sh;     // output row widths (routed, shared)
  int num_kb, num_kb_sh;   // 64-wide K blocks (routed, shared)
  __nv_bfloat16* out;
  __nv_bfloat16* out_sh;
  uint32_t* err;
};

struct SwSmem {
  uint64_t full[SW_STAGES];
  uint64_t empty[SW_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int issued;
  int consumed;
  int ngroups;
  int32_t gstart[SW_MAX_GROUPS];   // first row of each group in its row matrix
  int32_t gcnt[SW_MAX_GROUPS];     // rows of each group
  int32_t hv[SW_MAX_GROUPS + 1];   // item prefix over groups with >= 2 chunks
  int32_t lt[SW_MAX_GROUPS + 1];   // item prefix over groups with exactly 1 chunk
};

constexpr size_t SW_SMEM_BYTES = 1024 /*align slack*/ + (size_t)SW_STAGES * SW_STAGE_BYTES + sizeof(SwSmem);

struct SwItem {
  bool sh;
  int e, row0, ntok, nb, c0;
  int nbig;  // token rows copied in 64-row boxes (0: in nb boxes of 16 rows)
};

template <bool kGateUp>
__device__ __forceinline__ int sw_nt() { return kGateUp ? SW_NT_GATEUP : SW_NT_DOWN; }

template <bool kGateUp>
__device__ __forceinline__ int sw_ctiles(const SwParams& p, bool sh) {
  return ((sh ? p.n_out_sh : p.n_out) + 127) / 128;
}

// Item prefix by class over the groups (one full warp).
template <bool kGateUp>
__device__ void sw_build_prefix(SwSmem& m, const SwParams& p) {
  const int lane = threadIdx.x & 31;
  const int G = m.ngroups;
  const int C = (G + 31) / 32;
  const int g0 = min(G, lane * C), g1 = min(G, g0 + C);
  auto items = [&](int g, bool& heavy) {
    const int chunks = (m.gcnt[g] + sw_nt<kGateUp>() - 1) / sw_nt<kGateUp>();
    heavy = chunks >= 2;
    return chunks * sw_ctiles<kGateUp>(p, g >= p.E);
  };
  int sh = 0, sl = 0;
  for (int g = g0; g < g1; ++g) {
    bool heavy;
    const int n = items(g, heavy);
    sh += heavy ? n : 0;
    sl += heavy ? 0 : n;
  }
  int ih = sh, il = sl;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ih, o), b = __shfl_up_sync(0xffffffffu, il, o);
    if (lane >= o) {
      ih += a;
      il += b;
    }
  }
  int ph = ih - sh, pl = il - sl;
  for (int g = g0; g < g1; ++g) {
    m.hv[g] = ph;
    m.lt[g] = pl;
    bool heavy;
    const int n = items(g, heavy);
    ph += heavy ? n : 0;
    pl += heavy ? 0 : n;
  }
  if (lane == 31) {
    m.hv[G] = ih;
    m.lt[G] = il;
  }
}

template <bool kGateUp>
__device__ __forceinline__ bool sw_item(const SwParams& p, const SwSmem& m, int L, SwItem& it) {
  const int G = m.ngroups;
  const int nA = m.hv[G], nB = m.lt[G];
  if (L >= nA + nB) return false;
  const int32_t* pre = nA > 0 ? m.hv : m.lt;
  int idx = L;
  if (nA > 0 && nB > 0) {
    const long long tot = (long long)nA + nB;
    const int b = (int)((long long)L * nB / tot);
    const bool light = (int)((long long)(L + 1) * nB / tot) > b;
    pre = light ? m.lt : m.hv;
    idx = light ? b : L - b;
  }
  int lo = 0, hi = G - 1;  // largest g with pre[g] <= idx
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= idx) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int NT = sw_nt<kGateUp>();
  const int chunks = (m.gcnt[g] + NT - 1) / NT;
  const int local = idx - pre[g];
  const int ct = local / chunks, ch = local - ct * chunks;
  it.sh = g >= p.E;
  it.e = it.sh ? 0 : g;
  it.row0 = m.gstart[g] + ch * NT;
  it.ntok = min(NT, m.gcnt[g] - ch * NT);
  it.nb = (it.ntok + SW_BOX_ROWS - 1) / SW_BOX_ROWS;
  // more than two small boxes: copy the rows in 64-row boxes instead (fewer copy instructions;
  // the rows past the group's end are loaded but not used)
  it.nbig = it.nb > 2 ? (it.ntok + SW_BIG_ROWS - 1) / SW_BIG_ROWS : 0;
  it.c0 = ct * 128;
  return true;
}

__device__ __forceinline__ bool sw_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
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

__device__ __forceinline__ void sw_abort(SwSmem& m, uint32_t* err) {
  *(volatile int*)&m.abort = 1;
  atomicOr(err, kErrWaitTimeout);
}

template <bool kGateUp>
__global__ void __launch_bounds__(SW_THREADS, 1) tcs_ffn_kernel(const __grid_constant__ SwParams p) {
  constexpr int NMAT = kGateUp ? 2 : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage_base =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SwSmem& m = *reinterpret_cast<SwSmem*>(stage_base + (size_t)SW_STAGES * SW_STAGE_BYTES);
  volatile int* abort_flag = &m.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW_STAGES; ++s) {
      mbar_init(&m.full[s], 1);
      mbar_init(&m.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&m.tfull[a], 1);
      mbar_init(&m.tempty[a], SW_EPI_THREADS);
    }
    mbar_init(&m.drain, 1);
    m.abort = 0;
    m.issued = 0;
    m.consumed = 0;
    m.ngroups = p.E + (p.rows_sh > 0 ? 1 : 0);
    mbar_fence_init();
    tma_prefetch_desc(&p.mapW);
    tma_prefetch_desc(&p.mapX);
    tma_prefetch_desc(&p.mapX64);
    if (p.rows_sh > 0) {
      tma_prefetch_desc(&p.mapW_sh);
      tma_prefetch_desc(&p.mapX_sh);
      tma_prefetch_desc(&p.mapX64_sh);
    }
  }
  pdl_wait();  // below: reads of earlier kernels' output; TMEM once the previous kernel released its own
  if (warp == 1) {
    tmem_alloc(&m.tmem_base, SW_TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  for (int g = threadIdx.x; g < p.E; g += SW_THREADS) {
    const int o = p.offsets[g];
    m.gstart[g] = o;
    m.gcnt[g] = p.offsets[g + 1] - o;
  }
  if (threadIdx.x == 0 && p.rows_sh > 0) {
    m.gstart[p.E] = 0;
    m.gcnt[p.E] = p.rows_sh;
  }
  __syncthreads();
  if (warp == 0) sw_build_prefix<kGateUp>(m, p);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = m.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      SwItem it;
      for (int L = blockIdx.x; sw_item<kGateUp>(p, m, L, it); L += gridDim.x) {
        const CUtensorMap* mW = it.sh ? &p.mapW_sh : &p.mapW;
        const CUtensorMap* mX = it.nbig ? (it.sh ? &p.mapX64_sh : &p.mapX64) : (it.sh ? &p.mapX_sh : &p.mapX);
        const int num_kb = it.sh ? p.num_kb_sh : p.num_kb;
        const int nx = it.nbig ? it.nbig : it.nb;
        const int xrows = it.nbig ? SW_BIG_ROWS : SW_BOX_ROWS;
        const uint32_t tx = (uint32_t)(NMAT * SW_W_BYTES + nx * xrows * SW_BK * 2);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!sw_wait(&m.empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sW = stage_base + (size_t)s * SW_STAGE_BYTES;
          uint8_t* sX = sW + NMAT * SW_W_BYTES;
          mbar_arrive_expect_tx(&m.full[s], tx);
          const int kx = kb * SW_BK;
          if (kGateUp) {
            if (it.sh) {
              tma_load_3d(sW, mW, &m.full[s], kx, it.c0, 0);
              tma_load_3d(sW + SW_W_BYTES, mW, &m.full[s], kx, it.c0, 1);
            } else {
              tma_load_4d(sW, mW, &m.full[s], kx, it.c0, 0, it.e);
              tma_load_4d(sW + SW_W_BYTES, mW, &m.full[s], kx, it.c0, 1, it.e);
            }
          } else {
            if (it.sh) tma_load_2d(sW, mW, &m.full[s], kx, it.c0);
            else tma_load_3d(sW, mW, &m.full[s], kx, it.c0, it.e);
          }
          for (int b = 0; b < nx; ++b)
            tma_load_2d(sX + b * xrows * SW_BK * 2, mX, &m.full[s], kx, it.row0 + b * xrows);
          ++issued;
          if (++s == SW_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) {
          sw_abort(m, p.err);
          break;
        }
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
      int iter = 0, consumed = 0;
      bool ok = true;
      SwItem it;
      for (int L = blockIdx.x; ok && sw_item<kGateUp>(p, m, L, it); L += gridDim.x, ++iter) {
        const int a = iter & 1;
        const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
        if (!sw_wait(&m.tempty[a], aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(a * SW_ACC_COLS);
        const uint32_t idesc = idesc_bf16_f32(128, it.nb * SW_BOX_ROWS);
        const int num_kb = it.sh ? p.num_kb_sh : p.num_kb;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!sw_wait(&m.full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sW = smem_u32(stage_base + (size_t)s * SW_STAGE_BYTES);
          const uint32_t sX = sW + NMAT * SW_W_BYTES;
#pragma unroll
          for (int kk = 0; kk < SW_BK / 16; ++kk) {
            const uint64_t xd = smem_desc_sw128(sX + kk * 32);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_f16(d_tmem, smem_desc_sw128(sW + kk * 32), xd, idesc, acc);
            if (kGateUp) tc_mma_f16(d_tmem + 128, smem_desc_sw128(sW + SW_W_BYTES + kk * 32), xd, idesc, acc);
          }
          tc_commit(&m.empty[s]);
          ++consumed;
          if (++s == SW_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&m.tfull[a]);
      }
      if (!ok) sw_abort(m, p.err);
      m.consumed = consumed;
      tc_commit(&m.drain);  // drain: wait until every MMA issued by this thread has completed
      mbar_wait_bounded(&m.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int iter = 0;
    SwItem it;
    for (int L = blockIdx.x; sw_item<kGateUp>(p, m, L, it); L += gridDim.x, ++iter) {
      const int a = iter & 1;
      const uint32_t aph = (uint32_t)(iter >> 1) & 1u;
      const bool got = sw_wait(&m.tfull[a], aph, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) sw_abort(m, p.err);
        break;
      }
      tc_fence_after();
      const int n_out = it.sh ? p.n_out_sh : p.n_out;
      __nv_bfloat16* out = it.sh ? p.out_sh : p.out;
      const int ch = it.c0 + q * 32 + lane;
      const bool vch = ch < n_out;
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * SW_ACC_COLS);
      __nv_bfloat16* col = out + (size_t)it.row0 * n_out + ch;
#pragma unroll 1
      for (int j0 = 0; j0 < it.nb * SW_BOX_ROWS; j0 += 16) {
        float v[16];
        if (kGateUp) {
          float u[16];
          tmem_ld16(tb + j0, v);
          tmem_ld16(tb + 128 + j0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = silu_mul(v[i], u[i]);
        } else {
          tmem_ld16(tb + j0, v);
          tmem_ld_wait();
        }
        if (vch) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (j0 + i < it.ntok) col[(size_t)(j0 + i) * n_out] = __float2bfloat16_rn(v[i]);
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
      mbar_wait_bounded(&m.full[i % SW_STAGES], (uint32_t)(i / SW_STAGES) & 1u);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, SW_TMEM_COLS);
  }
}

// Token-row maps of a [rows, K] bf16 matrix with 16-row and 64-row boxes.
bool row_maps(CUtensorMap* m16, CUtensorMap* m64, const void* base, uint64_t K, int rows) {
  const uint64_t dims[2] = {K, (uint64_t)rows}, st[1] = {K * 2};
  const uint32_t b16[2] = {SW_BK, SW_BOX_ROWS}, b64[2] = {SW_BK, SW_BIG_ROWS};
  return make_bf16_tmap(m16, base, 2, dims, st, b16) && make_bf16_tmap(m64, base, 2, dims, st, b64);
}

template <bool kGateUp>
cudaError_t launch_tcs(const TcGemmArgs& a, cudaStream_t s) {
  SwParams p;
  memset(&p, 0, sizeof(p));
  const uint64_t d = a.d, f = a.f, fs = a.fs;
  const uint64_t S = (uint64_t)a.wstride * 2;  // bytes between experts
  const bool sh = a.fs > 0 && a.rows_sh > 0;
  bool ok = true;
  if (kGateUp) {
    { uint64_t dims[4] = {d, f, 2, (uint64_t)a.E}, st[3] = {d * 2, f * d * 2, S};
      uint32_t box[4] = {SW_BK, 128, 1, 1};
      ok &= make_bf16_tmap(&p.mapW, a.W, 4, dims, st, box); }
    ok &= row_maps(&p.mapX, &p.mapX64, a.A, d, a.rows);
    if (sh) {
      { uint64_t dims[3] = {d, fs, 2}, st[2] = {d * 2, fs * d * 2}; uint32_t box[3] = {SW_BK, 128, 1};
        ok &= make_bf16_tmap(&p.mapW_sh, a.W_sh, 3, dims, st, box); }
      ok &= row_maps(&p.mapX_sh, &p.mapX64_sh, a.A_sh, d, a.rows_sh);
    }
    p.n_out = (int)f;
    p.n_out_sh = (int)fs;
    p.num_kb = (int)((d + SW_BK - 1) / SW_BK);
    p.num_kb_sh = p.num_kb;
  } else {
    { uint64_t dims[3] = {f, d, (uint64_t)a.E}, st[2] = {f * 2, S}; uint32_t box[3] = {SW_BK, 128, 1};
      ok &= make_bf16_tmap(&p.mapW, (const __nv_bfloat16*)a.W + 2 * f * d, 3, dims, st, box); }
    ok &= row_maps(&p.mapX, &p.mapX64, a.A, f, a.rows);
    if (sh) {
      { uint64_t dims[2] = {fs, d}, st[1] = {fs * 2}; uint32_t box[2] = {SW_BK, 128};
        ok &= make_bf16_tmap(&p.mapW_sh, (const __nv_bfloat16*)a.W_sh + 2 * fs * d, 2, dims, st, box); }
      ok &= row_maps(&p.mapX_sh, &p.mapX64_sh, a.A_sh, fs, a.rows_sh);
    }
    p.n_out = (int)d;
    p.n_out_sh = (int)d;
    p.num_kb = (int)((f + SW_BK - 1) / SW_BK);
    p.num_kb_sh = sh ? (int)((fs + SW_BK - 1) / SW_BK) : 0;
  }
  if (!ok) return cudaErrorInvalidValue;
  p.offsets = a.offsets;
  p.E = a.E;
  p.rows_sh = sh ? a.rows_sh : 0;
  p.out = (__nv_bfloat16*)a.out;
  p.out_sh = (__nv_bfloat16*)a.out_sh;
  p.err = a.err;
  if (a.sm_count <= 0) return cudaSuccess;
  return launch_kernel(tcs_ffn_kernel<kGateUp>, dim3(a.sm_count), dim3(SW_THREADS), SW_SMEM_BYTES, s, 1, p);
}

}  // namespace

cudaError_t configure_tcs_kernels() {
  cudaError_t e =
      cudaFuncSetAttribute(tcs_ffn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SW_SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tcs_ffn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SW_SMEM_BYTES);
  return e;
}

cudaError_t launch_tcs_gateup(const TcGemmArgs& a, cudaStream_t s) { return launch_tcs<true>(a, s); }
cudaError_t launch_tcs_down(const TcGemmArgs& a, cudaStream_t s) { return launch_tcs<false>(a, s); }

}  // namespace colibri
