// Expert Compute stage for fp32 weights: grouped SwiGLU FFN with fp32 FMA (no TF32, so the
// result keeps fp32 accuracy).  Experts are addressed at a fixed stride in one buffer
// (www.mhpq.cn/news/563172 §2.1; www.0539edu.com/news/4774449 §2.2: one expert's parameters
// contiguous); rows are the grouped rows of each expert (www.trdm.cn/news/555962 §6.2).
//
//   gate/up:  H[r][n] = silu(sum_i A[r][i] W1_e[n][i]) * (sum_i A[r][i] W3_e[n][i])
//   down:     Y[r][n] = sum_i H[r][i] W2_e[n][i]
//
// 32 x 32 output tiles (down: 32 x 16): an expert of a small layer has few rows (a 64-row tile
// spent most of its multiply-adds on padding), and narrow tiles give such a layer enough CTAs to
// keep the memory system busy.  K advances 32 at a time through a 4-stage shared-memory ring filled by
// cp.async (16-byte copies, rows past a group's end or past N zero-filled), so three K slices are
// in flight while one is multiplied: the tiles of a small layer are bound by the memory round
// trip, which a load-then-compute loop paid once per slice.  Thread (ty, tx) of 16 x 16 owns the
// outputs (ty + 16 i, tx + 16 j), i < 2, j < 2 (down: j < 1), each accumulated with one fmaf per K in ascending K
// order.  Tiles are laid out on a (n-tile, m-tile) grid; m-tiles map to (expert, rows) through the
// device-side m-tile prefix, so no host synchronisation is needed.
#include "common.cuh"

namespace colibri {
namespace {

constexpr int BM = kSimtBM;
constexpr int MI = BM / 16;  // rows per thread
static_assert(BM % 16 == 0, "16 x 16 threads: BM / 16 rows each");
// Tile width: gate/up 32 columns; down 16 (its N = d_model is the smaller side of a small layer, and
// narrower tiles give it as many CTAs as gate/up has)
template <bool kGateUp>
constexpr int simt_bn() { return kGateUp ? kSimtBN : kSimtBN / 2; }
constexpr int SK = 32;       // K per stage (d_model and d_ff are multiples of 64)
constexpr int SS = 4;        // stages
constexpr int SP = SK + 4;   // floats per staged row: 16-byte aligned rows, and the 8 lanes of one
                             // 128-bit shared load hit distinct banks
template <bool kGateUp>
constexpr size_t simt_smem_bytes() { return (size_t)SS * (BM + simt_bn<kGateUp>() * (kGateUp ? 2 : 1)) * SP * 4; }

__device__ __forceinline__ void cp_async16(float* dst, const float* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ bool simt_tile_rows(const SimtGroups& g, int mt, int& grp, int& row0,
                                               int& row_end) {
  if (g.offsets == nullptr) {
    grp = 0;
    row0 = mt * BM;
    row_end = g.rows_single;
    return row0 < row_end;
  }
  if (mt >= g.mt_prefix[g.G]) return false;
  int lo = 0, hi = g.G - 1;  // largest grp with mt_prefix[grp] <= mt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (g.mt_prefix[mid] <= mt) lo = mid;
    else hi = mid - 1;
  }
  grp = lo;
  row0 = g.offsets[grp] + (mt - g.mt_prefix[grp]) * BM;
  row_end = g.offsets[grp + 1];
  return row0 < row_end;
}

template <bool kGateUp>
__global__ void __launch_bounds__(256) simt_ffn_kernel(const float* __restrict__ A, int lda, int K,
                                                       const float* __restrict__ W,
                                                       int64_t wstride, int d, int f,
                                                       SimtGroups groups,
                                                       float* __restrict__ out, int ldo, int N) {
  constexpr int BN = simt_bn<kGateUp>();
  constexpr int NJ = BN / 16;  // columns per thread
  static_assert(BN % 16 == 0, "16 x 16 threads: BN / 16 columns each");
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) float sm[];
  float (*As)[BM][SP] = reinterpret_cast<float (*)[BM][SP]>(sm);                      // [SS][BM][SP]
  float (*Bs)[BN][SP] = reinterpret_cast<float (*)[BN][SP]>(sm + SS * BM * SP);        // [SS][BN][SP]
  float (*Cs)[BN][SP] = reinterpret_cast<float (*)[BN][SP]>(sm + SS * (BM + BN) * SP);  // gate/up: W3
  int grp, row0, row_end;
  if (!simt_tile_rows(groups, blockIdx.y, grp, row0, row_end)) return;
  const int n0 = blockIdx.x * BN;
  const float* base = W + (int64_t)grp * wstride;
  // gate/up: W1 rows [n][d] then W3 rows at +f*d; down: W2 rows [n][f] at +2*f*d
  const float* B1 = kGateUp ? base : base + 2 * (int64_t)f * d;
  const float* B3 = base + (int64_t)f * d;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int nk = K / SK;
  // copies of K slice kt into ring slot `slot`: 64 rows x 8 chunks of 16 bytes per operand
  auto issue = [&](int kt, int slot) {
    const int k0 = kt * SK;
#pragma unroll
    for (int q = tid; q < BM * (SK / 4); q += 256) {
      const int rr = q >> 3, c4 = (q & 7) * 4;
      const int r = row0 + rr;
      const bool vr = r < row_end;
      cp_async16(&As[slot][rr][c4], A + (size_t)(vr ? r : row0) * lda + k0 + c4, vr);
    }
#pragma unroll
    for (int q = tid; q < BN * (SK / 4); q += 256) {
      const int rr = q >> 3, c4 = (q & 7) * 4;
      const int n = n0 + rr;
      const bool vn = n < N;
      cp_async16(&Bs[slot][rr][c4], B1 + (size_t)(vn ? n : n0) * K + k0 + c4, vn);
      if (kGateUp) cp_async16(&Cs[slot][rr][c4], B3 + (size_t)(vn ? n : n0) * K + k0 + c4, vn);
    }
  };
#pragma unroll
  for (int st = 0; st < SS - 1; ++st) {
    if (st < nk) issue(st, st);
    cp_async_commit();
  }
  float acc1[MI][NJ] = {}, acc3[MI][NJ] = {};
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait<SS - 2>();  // this thread's copies of slice kt have landed
    __syncthreads();          // everyone's have, and every thread is done with slice kt - 1
    if (kt + SS - 1 < nk) issue(kt + SS - 1, (kt + SS - 1) % SS);
    cp_async_commit();
    const int slot = kt % SS;
#pragma unroll
    for (int k4 = 0; k4 < SK; k4 += 4) {
      float4 a[MI], b[NJ], c[NJ];
#pragma unroll
      for (int i = 0; i < MI; ++i) a[i] = *reinterpret_cast<const float4*>(&As[slot][ty + 16 * i][k4]);
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        b[j] = *reinterpret_cast<const float4*>(&Bs[slot][tx + 16 * j][k4]);
        if (kGateUp) c[j] = *reinterpret_cast<const float4*>(&Cs[slot][tx + 16 * j][k4]);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int i = 0; i < MI; ++i) {
          const float av = kk == 0 ? a[i].x : kk == 1 ? a[i].y : kk == 2 ? a[i].z : a[i].w;
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            const float bv = kk == 0 ? b[j].x : kk == 1 ? b[j].y : kk == 2 ? b[j].z : b[j].w;
            acc1[i][j] = fmaf(av, bv, acc1[i][j]);
            if (kGateUp) {
              const float cv = kk == 0 ? c[j].x : kk == 1 ? c[j].y : kk == 2 ? c[j].z : c[j].w;
              acc3[i][j] = fmaf(av, cv, acc3[i][j]);
            }
          }
        }
      }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int i = 0; i < MI; ++i) {
    const int r = row0 + ty + 16 * i;
    if (r >= row_end) continue;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      float v = acc1[i][j];
      if (kGateUp) v = v / (1.0f + expf(-v)) * acc3[i][j];
      out[(size_t)r * ldo + n] = v;
    }
  }
}

}  // namespace

cudaError_t launch_simt_gateup(const float* A, int lda, const float* W, int64_t wstride, int d,
                               int f, SimtGroups g, int mt_bound, float* H, cudaStream_t s) {
  if (mt_bound <= 0) return cudaSuccess;
  constexpr int BN = simt_bn<true>();
  const dim3 grid((f + BN - 1) / BN, mt_bound);
  return launch_kernel(simt_ffn_kernel<true>, grid, dim3(256), simt_smem_bytes<true>(), s, 1, A, lda, d, W, wstride, d,
                       f, g, H, f, f);
}

cudaError_t launch_simt_down(const float* H, int f, const float* W, int64_t wstride, int d,
                             SimtGroups g, int mt_bound, float* Y, cudaStream_t s) {
  if (mt_bound <= 0) return cudaSuccess;
  constexpr int BN = simt_bn<false>();
  const dim3 grid((d + BN - 1) / BN, mt_bound);
  return launch_kernel(simt_ffn_kernel<false>, grid, dim3(256), simt_smem_bytes<false>(), s, 1, H, f, f, W, wstride, d,
                       f, g, Y, d, d);
}

// Done once per device at context creation (nothing in the launch path is a non-stream call).
cudaError_t configure_simt_kernels() {
  cudaError_t e = cudaFuncSetAttribute(simt_ffn_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)simt_smem_bytes<true>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(simt_ffn_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)simt_smem_bytes<false>());
  return e;
}

}  // namespace colibri
