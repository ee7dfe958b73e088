// Expert Compute stage for group-wise int4 weights at decode sizes, on the CUDA cores.
//
// With a few tokens each packed weight byte meets only a few rows of activations, so the work
// is a stream over the touched experts' weights and the tensor-core path (which first widens each
// packed tile to int8 in shared memory) spends more time on that hand-off than on the stream.
// Here the dot products run as dp4a on the same int8 activation planes the tensor-core path uses
// (x ~= a (hi + lo / 254) per row; H likewise per row and down-projection K split), with the
// weights read straight from global memory into registers:
//
//   gate/up:  GU[m][r][o]    = a_r * sum_g s_g[o] (S_hi + S_lo / 254),   m = W1 | W3
//   down:     Ypart[sp][r][o] = a_(sp,r) * sum_(g in split sp) s_g[o] (S_hi + S_lo / 254)
//
// where S = sum over the group's 128 K of q[o][k] * plane[r][k] (exact int32) and s_g[o] the
// group scale (www.mhpq.cn/news/563172 §4.2: a scale per 128 input channels of each output row;
// storage: two's complement nibbles, element 2j in the low nibble of byte j, scales [K/128][out]).
// A nibble q placed in the high half of a byte reads as the int8 16 q, so the packed word is
// split into even and odd elements with one shift and two masks and fed to dp4a against the
// activation bytes permuted the same way; the factor 16 is exact and folded into the scale.  The
// sums are formed per 32-element chunk (a quarter of a group) and added in a fixed order (chunk
// order within a lane, then a butterfly over the lanes), so results do not vary run to run; they
// differ from the tensor-core path's (whole groups, another order) only by fp32 rounding.
//
// Work: one warp per task = (touched expert, matrix, 8 consecutive output rows, K split), for all
// of the expert's rows; tasks are enumerated over the touched experts only, consecutive warps on
// consecutive rows of one matrix, so the activation chunks they share stay in L1 (the weight
// stream bypasses it).  This dp4a kernel serves one or two rows per expert; from three rows on the
// warp-level MMA kernel below takes over (up to 8 rows per instruction).
#include <algorithm>
#include <cstdlib>

#include "common.cuh"

namespace colibri {
namespace {

constexpr int kG4Threads = 384;  // 12 warps: ~170 registers each, two chunk steps of loads in flight
constexpr int kG4Rows = 8;       // output rows per task

struct Gemv4Params {
  const uint8_t* W;        // packed expert buffer (expert e at e * wstride / 2 bytes)
  const float* wscale;     // group scales, [E][3][K/128][out] per matrix (W1, W3 with K = d; W2 with K = f)
  int64_t wstride;         // elements between experts
  const int8_t* hi;        // [R, K] activation planes (grouped rows)
  const int8_t* lo;
  const float* rscale;     // [nsplit][R] (down) or [R] (gate/up) plane scales
  int rscale_split_stride;
  const int32_t* offsets;  // [E+1] grouped-row offsets
  int E, d, f, R;
  int K, out_rows, mats;   // gate/up: K = d, out = f, 2 matrices; down: K = f, out = d, 1
  int nsplit, kspan;       // K splits (down), each kspan wide (a multiple of 1024)
  float* out;              // GU [2][R][f] or Ypart [nsplit][R][d]
  bool gateup;
};

// 16 bytes of the weight stream: read once, so kept out of L1 (the activation planes, re-read by
// every warp of the expert, stay there)
__device__ __forceinline__ uint4 ld_stream16(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}

__device__ __forceinline__ float exact_i2f(int v) {  // |v| < 2^22: the float of v without I2F
  return __int_as_float(v + 0x4B400000) - 12582912.0f;
}

// One task: 8 output rows of one matrix of one touched expert over one K split, for all of the
// expert's rows (NR at a time; a second pass over the same weights finds them in L1).  Lane l
// takes the 32-element chunks l, l + 32, ... of the split, so one load instruction of the warp
// reads 512 contiguous bytes of a row; each chunk's exact int32 sums are scaled by its group's
// scale.  The next chunk step's weight loads are issued before the current one is used.
template <int NR>
__global__ void __launch_bounds__(kG4Threads, 1) gemv4_kernel(const __grid_constant__ Gemv4Params p) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t off_s[kMaxExperts + 1];
  __shared__ int32_t touched[kMaxExperts];
  __shared__ int32_t n_touched;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) off_s[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x < 32) {
    // the experts that received rows, in order (E <= 256: 8 ballots)
    int base = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + (int)threadIdx.x;
      const bool has = e < p.E && off_s[e + 1] > off_s[e];
      const unsigned m = __ballot_sync(0xffffffffu, has);
      if (has) touched[base + __popc(m & ((1u << threadIdx.x) - 1u))] = e;
      base += __popc(m);
    }
    if (threadIdx.x == 0) n_touched = base;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int ngroups = p.out_rows / kG4Rows;
  const int per_e = p.mats * p.nsplit * ngroups;
  const int tasks = n_touched * per_e;
  const size_t mat_bytes = (size_t)p.d * p.f / 2;
  const size_t scales_per_mat = (size_t)p.d * p.f / 128;
  const size_t row_bytes = (size_t)p.K / 2;

  for (int task = blockIdx.x * (kG4Threads / 32) + (threadIdx.x >> 5); task < tasks;
       task += gridDim.x * (kG4Threads / 32)) {
    const int te = task / per_e;
    int rest = task - te * per_e;
    const int og = rest % ngroups;
    rest /= ngroups;
    const int sp = rest % p.nsplit;
    const int m = rest / p.nsplit;
    const int e = touched[te];
    const int r_beg = off_s[e], r_end = off_s[e + 1];
    const int o0 = og * kG4Rows;
    const int kbeg = sp * p.kspan;
    const uint8_t* wbase = p.W + (size_t)e * (size_t)(p.wstride / 2) +
                           (p.gateup ? (size_t)m * mat_bytes : 2 * mat_bytes) + (size_t)o0 * row_bytes + kbeg / 2;
    const float* sbase = p.wscale + (size_t)e * 3 * scales_per_mat + (size_t)(p.gateup ? m : 2) * scales_per_mat +
                         (size_t)(kbeg / 128) * p.out_rows + o0;

    for (int row0 = r_beg; row0 < r_end; row0 += NR) {
      const int nr = min(NR, r_end - row0);
      float acc[kG4Rows][NR];
#pragma unroll
      for (int r = 0; r < kG4Rows; ++r)
#pragma unroll
        for (int t = 0; t < NR; ++t) acc[r][t] = 0.f;
      // chunk steps of this lane: step n is the 32-element chunk lane + 32 n of the split (16
      // packed bytes of each row; a warp's load covers 512 contiguous bytes of a row)
      const int nchunks = p.kspan / 32;
      const int nsteps = nchunks > lane ? (nchunks - lane + 31) / 32 : 0;
      uint4 wcur[kG4Rows], wnext[kG4Rows];
      auto load_w = [&](uint4 (&dst)[kG4Rows], int n) {
        const uint8_t* src = wbase + (size_t)(lane + 32 * n) * 16;
#pragma unroll
        for (int r = 0; r < kG4Rows; ++r) dst[r] = ld_stream16(src + (size_t)r * row_bytes);
      };
      if (nsteps > 0) load_w(wcur, 0);
      for (int n = 0; n < nsteps; ++n) {
        if (n + 1 < nsteps) load_w(wnext, n + 1);
        const int ch = lane + 32 * n;
        const int kx = kbeg + ch * 32;  // first K element of the chunk
        // the chunk lies in K group ch / 4: its scales for the 8 rows, divided by 16 (exact)
        const float4 s03 = __ldg(reinterpret_cast<const float4*>(sbase + (size_t)(ch >> 2) * p.out_rows));
        const float4 s47 = __ldg(reinterpret_cast<const float4*>(sbase + (size_t)(ch >> 2) * p.out_rows + 4));
        const float sg[kG4Rows] = {s03.x * 0.0625f, s03.y * 0.0625f, s03.z * 0.0625f, s03.w * 0.0625f,
                                   s47.x * 0.0625f, s47.y * 0.0625f, s47.z * 0.0625f, s47.w * 0.0625f};
#pragma unroll
        for (int t = 0; t < NR; ++t) {
          if (t < nr) {
            const int8_t* hp = p.hi + (size_t)(row0 + t) * p.K + kx;
            const int8_t* lp = p.lo + (size_t)(row0 + t) * p.K + kx;
            const uint4 h0 = __ldg(reinterpret_cast<const uint4*>(hp)), h1 = __ldg(reinterpret_cast<const uint4*>(hp + 16));
            const uint4 l0 = __ldg(reinterpret_cast<const uint4*>(lp)), l1 = __ldg(reinterpret_cast<const uint4*>(lp + 16));
            const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            const uint32_t lw[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
            uint32_t he[4], ho[4], le[4], lo2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              he[i] = __byte_perm(hw[2 * i], hw[2 * i + 1], 0x6420);
              ho[i] = __byte_perm(hw[2 * i], hw[2 * i + 1], 0x7531);
              le[i] = __byte_perm(lw[2 * i], lw[2 * i + 1], 0x6420);
              lo2[i] = __byte_perm(lw[2 * i], lw[2 * i + 1], 0x7531);
            }
#pragma unroll
            for (int r = 0; r < kG4Rows; ++r) {
              const uint32_t wv[4] = {wcur[r].x, wcur[r].y, wcur[r].z, wcur[r].w};
              int sh = 0, sl = 0;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                // even elements 16 q in ev, odd ones in od
                const int ev = (int)((wv[i] << 4) & 0xF0F0F0F0u), od = (int)(wv[i] & 0xF0F0F0F0u);
                sh = __dp4a(ev, (int)he[i], sh);
                sh = __dp4a(od, (int)ho[i], sh);
                sl = __dp4a(ev, (int)le[i], sl);
                sl = __dp4a(od, (int)lo2[i], sl);
              }
              acc[r][t] = fmaf(sg[r], exact_i2f(sh) + exact_i2f(sl) * (1.0f / 254.0f), acc[r][t]);
            }
          }
        }
        if (n + 1 < nsteps) {
#pragma unroll
          for (int r = 0; r < kG4Rows; ++r) wcur[r] = wnext[r];
        }
      }
      // sum over the lanes (butterfly: every lane ends with every sum), then lane t writes
      // row t's 8 consecutive outputs
#pragma unroll
      for (int t = 0; t < NR; ++t) {
        if (t < nr) {
#pragma unroll
          for (int r = 0; r < kG4Rows; ++r) {
#pragma unroll
            for (int o = 16; o; o >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], o);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < NR; ++t) {
        if (t < nr && lane == t) {
          const int row = row0 + t;
          const float a = __ldcg(p.rscale + (size_t)sp * p.rscale_split_stride + row);
          float* dst = p.gateup ? p.out + (((size_t)sp * 2 + m) * p.R + row) * p.f + o0
                                : p.out + ((size_t)sp * p.R + row) * p.d + o0;
          reinterpret_cast<float4*>(dst)[0] = make_float4(a * acc[0][t], a * acc[1][t], a * acc[2][t], a * acc[3][t]);
          reinterpret_cast<float4*>(dst)[1] = make_float4(a * acc[4][t], a * acc[5][t], a * acc[6][t], a * acc[7][t]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------------- warp-level MMA plan
// The same contraction on the tensor cores through the warp-level mma.sync.m16n8k32 (s8 x s8 ->
// s32), the weights unpacked in registers (no shared-memory staging): up to 8 tokens share each
// instruction, so the work per weight byte no longer grows with the token count.  A warp task is
// (touched expert, matrix, 32 output rows, K split) for all of the expert's rows, 8 at a time.
// Lane (g = lane / 4, t = lane % 4) reads, per K group (128 elements), the 16 packed bytes
// [32 t, 32 t + 32) of rows g, g + 8, g + 16, g + 24; MMA kk (0..3) of the group takes from every
// lane the 8 elements 32 t + 8 kk + [0, 8) of its rows — even elements (16 q, as above) in the
// A register of columns 4 t.., odd ones in that of columns 16 + 4 t.. — and the activation bytes
// of token g at the same K positions, permuted the same way, as B.  The contraction order over K
// is thereby permuted identically in A and B, which leaves the exact int32 group sums unchanged.
// Per group and plane the MMA accumulators (rows g, g + 8 of each 16-row half, tokens 2 t, 2 t + 1)
// are scaled by the group scale and added into fp32 registers.
constexpr int kG4mThreads = 384;
constexpr int kG4mRows = 32;
constexpr int kG4mAhead = 2;  // K groups of weight loads in flight per warp beyond the current one

__device__ __forceinline__ void mma_s8_16x8x32(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kG4mThreads, 1) gemv4m_kernel(const __grid_constant__ Gemv4Params p) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t off_s[kMaxExperts + 1];
  __shared__ int32_t touched[kMaxExperts];
  __shared__ int32_t n_touched;
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) off_s[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x < 32) {
    int base = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const int e = e0 + (int)threadIdx.x;
      const bool has = e < p.E && off_s[e + 1] > off_s[e];
      const unsigned m = __ballot_sync(0xffffffffu, has);
      if (has) touched[base + __popc(m & ((1u << threadIdx.x) - 1u))] = e;
      base += __popc(m);
    }
    if (threadIdx.x == 0) n_touched = base;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ntiles = p.out_rows / kG4mRows;
  const int per_e = p.mats * p.nsplit * ntiles;
  const int tasks = n_touched * per_e;
  const int ngr = p.kspan / 128;
  const size_t mat_bytes = (size_t)p.d * p.f / 2;
  const size_t scales_per_mat = (size_t)p.d * p.f / 128;
  const size_t row_bytes = (size_t)p.K / 2;

  for (int task = blockIdx.x * (kG4mThreads / 32) + (threadIdx.x >> 5); task < tasks;
       task += gridDim.x * (kG4mThreads / 32)) {
    const int te = task / per_e;
    int rest = task - te * per_e;
    const int ot = rest % ntiles;
    rest /= ntiles;
    const int sp = rest % p.nsplit;
    const int m = rest / p.nsplit;
    const int e = touched[te];
    const int r_beg = off_s[e], r_end = off_s[e + 1];
    const int o0 = ot * kG4mRows;
    const int kbeg = sp * p.kspan;
    // this lane's packed bytes: rows o0 + g + 8 j, bytes [16 t, 16 t + 16) of every 64-byte group
    const uint8_t* wbase = p.W + (size_t)e * (size_t)(p.wstride / 2) +
                           (p.gateup ? (size_t)m * mat_bytes : 2 * mat_bytes) + (size_t)(o0 + g) * row_bytes +
                           kbeg / 2 + 16 * t;
    const float* sbase = p.wscale + (size_t)e * 3 * scales_per_mat + (size_t)(p.gateup ? m : 2) * scales_per_mat +
                         (size_t)(kbeg / 128) * p.out_rows + o0 + g;

    for (int row0 = r_beg; row0 < r_end; row0 += 8) {
      const int nr = min(8, r_end - row0);
      const bool has_tok = g < nr;  // this lane supplies B for token g
      const int8_t* hp = p.hi + (size_t)(row0 + (has_tok ? g : 0)) * p.K + kbeg + 32 * t;
      const int8_t* lp = p.lo + (size_t)(row0 + (has_tok ? g : 0)) * p.K + kbeg + 32 * t;
      float acc[4][2];  // rows g + 8 j, tokens 2 t, 2 t + 1
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = 0.f;
      uint4 wq[kG4mAhead + 1][4];
      auto load_w = [&](uint4 (&dst)[4], int gi) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[j] = ld_stream16(wbase + (size_t)(8 * j) * row_bytes + (size_t)gi * 64);
      };
#pragma unroll
      for (int a = 0; a < kG4mAhead; ++a)
        if (a < ngr) load_w(wq[a], a);
      for (int gi = 0; gi < ngr; ++gi) {
        // rotate the prefetch window (register arrays indexed by constants only)
        if (gi + kG4mAhead < ngr) load_w(wq[kG4mAhead], gi + kG4mAhead);
        uint4 w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = wq[0][j];
#pragma unroll
        for (int a = 0; a < kG4mAhead; ++a)
#pragma unroll
          for (int j = 0; j < 4; ++j) wq[a][j] = wq[a + 1][j];
        // activation bytes of token g at K 128 gi + 32 t + [0, 32), both planes
        uint4 h0 = make_uint4(0, 0, 0, 0), h1 = h0, l0 = h0, l1 = h0;
        if (has_tok) {
          h0 = __ldg(reinterpret_cast<const uint4*>(hp + 128 * gi));
          h1 = __ldg(reinterpret_cast<const uint4*>(hp + 128 * gi + 16));
          l0 = __ldg(reinterpret_cast<const uint4*>(lp + 128 * gi));
          l1 = __ldg(reinterpret_cast<const uint4*>(lp + 128 * gi + 16));
        }
        const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
        const uint32_t lw[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
        int dh[2][4], dl[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 4; ++i) dh[h][i] = dl[h][i] = 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // B: token g's 8 bytes at 32 t + 8 kk, even ones then odd ones
          const uint32_t bhe = __byte_perm(hw[2 * kk], hw[2 * kk + 1], 0x6420);
          const uint32_t bho = __byte_perm(hw[2 * kk], hw[2 * kk + 1], 0x7531);
          const uint32_t ble = __byte_perm(lw[2 * kk], lw[2 * kk + 1], 0x6420);
          const uint32_t blo = __byte_perm(lw[2 * kk], lw[2 * kk + 1], 0x7531);
#pragma unroll
          for (int h = 0; h < 2; ++h) {  // 16-row halves: rows g + 16 h and g + 8 + 16 h
            const uint32_t wa = (kk == 0 ? w[2 * h].x : kk == 1 ? w[2 * h].y : kk == 2 ? w[2 * h].z : w[2 * h].w);
            const uint32_t wb = (kk == 0 ? w[2 * h + 1].x : kk == 1 ? w[2 * h + 1].y : kk == 2 ? w[2 * h + 1].z
                                                                                          : w[2 * h + 1].w);
            const uint32_t a[4] = {(wa << 4) & 0xF0F0F0F0u, (wb << 4) & 0xF0F0F0F0u, wa & 0xF0F0F0F0u,
                                   wb & 0xF0F0F0F0u};
            mma_s8_16x8x32(dh[h], a, bhe, bho);
            mma_s8_16x8x32(dl[h], a, ble, blo);
          }
        }
        // the group's exact sums (x 16) times its scales / 16
        const float* sg = sbase + (size_t)gi * p.out_rows;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float s0 = __ldg(sg + 16 * h) * 0.0625f, s1 = __ldg(sg + 16 * h + 8) * 0.0625f;
          acc[2 * h][0] = fmaf(s0, exact_i2f(dh[h][0]) + exact_i2f(dl[h][0]) * (1.0f / 254.0f), acc[2 * h][0]);
          acc[2 * h][1] = fmaf(s0, exact_i2f(dh[h][1]) + exact_i2f(dl[h][1]) * (1.0f / 254.0f), acc[2 * h][1]);
          acc[2 * h + 1][0] = fmaf(s1, exact_i2f(dh[h][2]) + exact_i2f(dl[h][2]) * (1.0f / 254.0f), acc[2 * h + 1][0]);
          acc[2 * h + 1][1] = fmaf(s1, exact_i2f(dh[h][3]) + exact_i2f(dl[h][3]) * (1.0f / 254.0f), acc[2 * h + 1][1]);
        }
      }
      // lane (g, t) holds rows o0 + g + 8 j for tokens 2 t and 2 t + 1
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int tok = 2 * t + c;
        if (tok < nr) {
          const int row = row0 + tok;
          const float a = __ldcg(p.rscale + (size_t)sp * p.rscale_split_stride + row);
          float* dst = p.gateup ? p.out + (((size_t)sp * 2 + m) * p.R + row) * p.f + o0 + g
                                : p.out + ((size_t)sp * p.R + row) * p.d + o0 + g;
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[8 * j] = a * acc[j][c];
        }
      }
    }
  }
}

int sm_count_here() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

cudaError_t launch_gemv4(const Gemv4Params& p, int max_rows_per_expert, cudaStream_t s) {
  const int grid = sm_count_here();
  // up to 2 rows per expert the dp4a kernel, beyond that the warp-MMA one (measured on B200:
  // 4096 x 14336 layer, T = 1: 87 against 123 us per call; T = 8: 380 against 242 us);
  // COLIBRI_I4_GEMV_MMA=0 / 1 forces one of them
  const char* force = getenv("COLIBRI_I4_GEMV_MMA");
  const bool mma_plan = force ? atoi(force) != 0 : max_rows_per_expert > 2;
  if (mma_plan) return launch_kernel(gemv4m_kernel, dim3(grid), dim3(kG4mThreads), 0, s, 1, p);
  if (max_rows_per_expert <= 1) return launch_kernel(gemv4_kernel<1>, dim3(grid), dim3(kG4Threads), 0, s, 1, p);
  return launch_kernel(gemv4_kernel<2>, dim3(grid), dim3(kG4Threads), 0, s, 1, p);
}

}  // namespace

bool gemv4_supported(int d, int f) { return d % 1024 == 0 && f % 1024 == 0; }

// a second K split of the gate/up projection doubles its tasks when only one or two experts are
// touched (fewer tasks than warps otherwise leave SMs idle at the end)
int gemv4_gateup_split(int d, int T) { return T <= 2 && (d / 1024) % 2 == 0 ? 2 : 1; }

// K splits of the down projection: the largest divisor of f / 1024 up to 8 (f = 14336: 7 splits of
// 2048), so that the H-plane kernel (one CTA per row and split) and the down GEMV both get enough
// CTAs and tasks for a single token
int gemv4_down_split(int f, int max_split) {
  int ns = 1;
  for (int c = 2; c <= 8 && c <= max_split; ++c)
    if ((f / 1024) % c == 0) ns = c;
  return ns;
}

cudaError_t launch_gemv4_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const uint8_t* W,
                                const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                                int gsplit, float* GU, int R, int max_rows_per_expert, cudaStream_t s) {
  if (!gemv4_supported(d, f) || gsplit < 1 || (d / gsplit) % 1024 != 0) return cudaErrorInvalidValue;
  Gemv4Params p{};
  p.W = W;
  p.wscale = scales;
  p.wstride = wstride;
  p.hi = Xhi;
  p.lo = Xlo;
  p.rscale = xscale;
  p.rscale_split_stride = 0;
  p.offsets = offsets;
  p.E = E;
  p.d = d;
  p.f = f;
  p.R = R;
  p.K = d;
  p.out_rows = f;
  p.mats = 2;
  p.nsplit = gsplit;
  p.kspan = d / gsplit;
  p.out = GU;
  p.gateup = true;
  return launch_gemv4(p, max_rows_per_expert, s);
}

cudaError_t launch_gemv4_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const uint8_t* W,
                              const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                              int nsplit, int R, float* Ypart, int max_rows_per_expert, cudaStream_t s) {
  if (!gemv4_supported(d, f) || nsplit < 1 || (f / nsplit) % 1024 != 0) return cudaErrorInvalidValue;
  Gemv4Params p{};
  p.W = W;
  p.wscale = scales;
  p.wstride = wstride;
  p.hi = Hhi;
  p.lo = Hlo;
  p.rscale = hscale;
  p.rscale_split_stride = R;
  p.offsets = offsets;
  p.E = E;
  p.d = d;
  p.f = f;
  p.R = R;
  p.K = f;
  p.out_rows = d;
  p.mats = 1;
  p.nsplit = nsplit;
  p.kspan = f / nsplit;
  p.out = Ypart;
  p.gateup = false;
  return launch_gemv4(p, max_rows_per_expert, s);
}

}  // namespace colibri
