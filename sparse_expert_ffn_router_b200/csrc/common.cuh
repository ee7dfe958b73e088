// Internal declarations shared by the sm_100a kernels and the host orchestration of the
// MoE layer forward.  Nothing here is part of the public C ABI (include/colibri.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "colibri.h"

namespace colibri {

// ---------------------------------------------------------------------------------------
// Limits and tile shapes
// ---------------------------------------------------------------------------------------
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 8;
constexpr int kCountBlock = 256;  // tokens per block of the histogram / rank kernel
constexpr int kFusedRouteMaxT = 64;       // largest T routed by the single-CTA fused kernel
constexpr int kFusedRouteThreads = 1024;  // its threads (the row copies use all of them)

// tcgen05 grouped GEMM tile: BM x BN accumulator, BK = one 128-byte swizzle atom of bf16
constexpr int kTcBM = 128;
constexpr int kTcBN = 256;
constexpr int kTcBK = 64;
#ifndef COLIBRI_TC_STAGES
#define COLIBRI_TC_STAGES 4
#endif
#ifndef COLIBRI_TC2_STAGES
#define COLIBRI_TC2_STAGES 6
#endif
constexpr int kTcStages = COLIBRI_TC_STAGES;    // 48 KB stages, one CTA per tile
constexpr int kTcPairStages = COLIBRI_TC2_STAGES;  // 32 KB stages, pair tiles
constexpr int kTcPairBM = 256;  // rows of a pair tile (two CTAs, cta_group::2)

// SIMT fp32 grouped GEMM tile
constexpr int kSimtBM = 32;
constexpr int kSimtBN = 32;

// int8 weight-streaming decode path
constexpr int kDecSplitMax = 16;     // K splits of the down projection
constexpr int kDecMaxFF = 65536;     // largest d_ff of the int8 path (one H row in shared memory)
constexpr int kDecGateSplitMax = 4;  // K splits of the gate/up projection (small batches)
constexpr int kDecGateSplitRows = 64;  // routed rows up to which the gate/up projection may split

// Device error word bits (ctx->err)
constexpr uint32_t kErrWaitTimeout = 1u;

// Bounded waits: a device wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitTimeoutNs = 4000000000ull;

// ---------------------------------------------------------------------------------------
// Context
// ---------------------------------------------------------------------------------------
struct Workspace {
  void* x_stage = nullptr;  // [M, d] act, for host x
  void* y_stage = nullptr;  // [M, d] act, for host y
  void* x_stage2 = nullptr;  // the second pair: staged calls alternate between the two
  void* y_stage2 = nullptr;
  int32_t* topk_idx = nullptr;  // [M, k]
  float* topk_w = nullptr;      // [M, k]
  int32_t* dst_row = nullptr;   // [M, k]
  int32_t* src_row = nullptr;   // [M*k]
  int32_t* blk_counts = nullptr;  // [nblk, E]
  int32_t* blk_base = nullptr;    // [nblk, E]
  int32_t* counts = nullptr;      // [E]
  int32_t* offsets = nullptr;     // [E+1]
  int32_t* mt_prefix = nullptr;   // [E+1] m-tiles prefix for the GEMM schedule
  void* Xp = nullptr;   // [M*k, d] act (grouped rows)
  void* H = nullptr;    // [M*k, f] bf16 (bf16 path), f32 (fp32 path), [2, M*k, f] f32 gate/up partials (int8)
  void* Yp = nullptr;   // [M*k, d] bf16 or f32
  void* Hs = nullptr;   // [M, fs]
  void* Ys = nullptr;   // [M, d]
  float* Ypart = nullptr;  // [split, M*k, d] f32, int8 path
  int32_t* grid_bar = nullptr;       // [4] grid-barrier counters of the fused int8 kernel (zero between calls)
  int8_t* plane_hi = nullptr;  // [M*k, max(d, f)] int8 activation planes, int8 path
  int8_t* plane_lo = nullptr;
  float* plane_scale = nullptr;  // [M*k]
  uint32_t* err = nullptr;
  uint32_t* tile_sched = nullptr;  // [4] tile counters of the bf16 GEMMs (gate/up, down; zero between calls)
};

}  // namespace colibri

struct colibri_ctx {
  colibri_desc desc;
  int sm_count = 0;
  int64_t expert_stride = 0;
  int nblk_max = 0;
  int dec_split = 1;
  colibri::Workspace ws;
  void* ws_base = nullptr;
  size_t ws_bytes = 0;
  int last_T = -1;
  std::string last_error;
  bool profile = false;                // COLIBRI_PROFILE=1: print one line per call
  cudaEvent_t ev[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  // colibri_profile_begin/end: 6 events per recorded call
  std::vector<cudaEvent_t> prof_ev;
  int prof_max = 0;
  int prof_n = 0;
  bool prof_on = false;
  // CUDA graphs of the launch sequence, keyed by the forward's arguments
  struct GraphEntry {
    uintptr_t key[14];
    cudaGraphExec_t exec;
    uint64_t last_use;
    // graphs captured while colibri_profile_begin is active also hold one event-record node per
    // stage boundary; the graph is kept so that each replay can point them at that call's events
    cudaGraph_t graph = nullptr;
    cudaGraphNode_t ev_node[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  };
  cudaEvent_t cap_ev[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};  // events the nodes are captured with
  std::vector<GraphEntry> graphs;
  uint64_t graph_clock = 0;
  bool use_graphs = true;
  bool tile_static = false;  // bf16 GEMMs: static round-robin tiles instead of the claimed schedule
  bool i4_gemv = true;       // int4 weights, T <= kGemv4MaxT: GEMV kernels instead of the stream kernels
  bool use_pdl = false;  // programmatic dependent launch between the kernels of a forward (opt-in)
  bool dec_fused = true;  // int8 weights: the one-launch expert stage (COLIBRI_DEC_FUSED=0: four launches)
  bool dec_route = true;  // int8, T <= 64: routing inside that launch too (COLIBRI_DEC_ROUTE=0: not)
  // staged calls (host x or y): copy streams, events [2 staging pairs][x free, x in, forward done,
  // y out], and the pair the next call takes (COLIBRI_STAGED=0: copies on the caller's stream)
  bool staged = true;
  cudaStream_t cs_in = nullptr, cs_out = nullptr;
  cudaEvent_t st_ev[8] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  int stage_next = 0;
};

namespace colibri {

// ---------------------------------------------------------------------------------------
// Launches.  Every kernel goes through launch_kernel().  Inside a LaunchScope that enables it,
// each launch after the first of the scope uses programmatic dependent launch: its CTAs may be
// scheduled while the previous kernel still runs, so they do their set-up (barriers, TMEM,
// descriptor prefetch) in its shadow.  Every kernel therefore calls pdl_wait() before it reads
// anything an earlier launch wrote, on every path (so that a kernel never completes before its
// predecessor), and pdl_trigger() to let its successor be scheduled; both are no-ops for a
// launch without the attribute.  A copy or memset between two launches breaks the chain
// (launch_chain_break): the launch after it is an ordinary one.
// ---------------------------------------------------------------------------------------
namespace detail {
inline thread_local bool tl_pdl = false;   // launches of the current scope may overlap
inline thread_local int tl_chain = 0;      // launches since the scope began or the chain broke
}  // namespace detail
struct LaunchScope {
  explicit LaunchScope(bool pdl) {
    detail::tl_pdl = pdl;
    detail::tl_chain = 0;
  }
  ~LaunchScope() {
    detail::tl_pdl = false;
    detail::tl_chain = 0;
  }
};
inline void launch_chain_break() { detail::tl_chain = 0; }

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (detail::tl_pdl && detail::tl_chain > 0) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  ++detail::tl_chain;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------------------
// Kernel launchers (each returns cudaGetLastError() of its launch)
// ---------------------------------------------------------------------------------------
// err: the context's device error word for bounded waits that give up (may be NULL).
constexpr int kRouterSmallT = 64;       // T up to which one CTA per token computes the logits
constexpr int kRouterMaxSplit = 4;      // K slices per token tile of the tensor-core router (a cluster)
constexpr int kRouterCtaBudget = 160;   // CTAs the tensor-core router aims to stay within
int router_ksplit(int T, int d);
cudaError_t launch_router_topk(const void* x, int act, int T, int d, const void* wr, const float* b,
                               int E, int k, int rflags, int32_t* idx, float* w, uint32_t* err, cudaStream_t s);
cudaError_t launch_route_count(const int32_t* idx, int T, int k, int E, int32_t* blk_counts,
                               int32_t* local_rank, cudaStream_t s);
cudaError_t launch_route_scan(const int32_t* blk_counts, int nblk, int E, int bm, int32_t* blk_base,
                              int32_t* counts, int32_t* offsets, int32_t* mt_prefix, cudaStream_t s);
// Grouped rows go to Xp (a copy of the token row), or -- when `planes` is given (bf16 input,
// int8 weights) -- to the int8 planes of the token row instead: planes->hi/lo [R, d] and the
// per-row scale planes->scale [R] (x ~= scale * (hi + lo / 254)); Xp is then not written.
struct RowPlanes {
  int8_t* hi;
  int8_t* lo;
  float* scale;
};
// blk_base: per (block, expert) exclusive prefix of the block counts (without offsets[e])
cudaError_t launch_route_scatter(const void* x, int act, int T, int d, int k, int E,
                                 const int32_t* idx, const int32_t* blk_base, const int32_t* offsets,
                                 int32_t* dst_row, int32_t* src_row, void* Xp, const RowPlanes* planes,
                                 cudaStream_t s);
// T <= kFusedRouteMaxT: count + scan + scatter in one single-CTA launch
cudaError_t launch_route_fused(const void* x, int act, int T, int d, const int32_t* idx, int k, int E, int bm,
                               int32_t* counts, int32_t* offsets, int32_t* mt_prefix, int32_t* src_row,
                               int32_t* dst_row, void* Xp, const RowPlanes* planes, cudaStream_t s);
cudaError_t launch_combine(const void* Yp, int yp_dtype, const int32_t* dst_row, const float* w,
                           int T, int k, int d, const void* Ys, void* y, int act, cudaStream_t s);
cudaError_t launch_combine_split(const float* Ypart, int nsplit, int rows, const int32_t* dst_row,
                                 const float* w, int T, int k, int d, void* y, int act,
                                 cudaStream_t s);

// fp32 SIMT grouped SwiGLU expert FFN
struct SimtGroups {
  const int32_t* offsets;    // [G+1] row ranges (device), or nullptr with rows_single
  const int32_t* mt_prefix;  // [G+1] m-tile prefix (device), or nullptr with rows_single
  int G;
  int rows_single;           // rows of the single group when offsets == nullptr
};
cudaError_t launch_simt_gateup(const float* A, int lda, const float* W, int64_t wstride, int d,
                               int f, SimtGroups g, int mt_bound, float* H, cudaStream_t s);
cudaError_t launch_simt_down(const float* H, int f, const float* W, int64_t wstride, int d,
                             SimtGroups g, int mt_bound, float* Y, cudaStream_t s);

// tcgen05 grouped GEMM (bf16 x bf16 -> fp32 TMEM), see gemm_tc.cu
struct TcGemmArgs {
  // routed groups
  const void* A;        // [rows, K] bf16 grouped rows
  int rows;             // T*k
  const int32_t* offsets;    // [E+1] device
  const int32_t* mt_prefix;  // [E+1] device
  int E;
  const void* W;        // expert buffer base (bf16)
  int64_t wstride;      // elements between experts
  void* out;            // [rows, N_out] bf16
  // shared expert (optional, rows = T tokens of x / Hs)
  const void* A_sh;     // [T, K_sh] bf16 or nullptr
  int rows_sh;
  const void* W_sh;     // shared buffer base or nullptr
  void* out_sh;         // [T, N_out_sh]
  // sizes
  int d;                // d_model
  int f;                // routed d_ff
  int fs;               // shared d_ff (0 = none)
  int mt_bound;         // upper bound on routed m-tiles
  uint32_t* err;
  uint32_t* sched;      // [2] tile counter and finished-CTA counter (zero between launches), or
                        // nullptr for the static round-robin schedule
  int sm_count;
  bool pair;            // clusters of two CTAs with 256-row pair tiles (cta_group::2)
};
// Tensor map, zero fill out of bounds; 128-byte swizzle (with a 128-byte inner box) unless told
// otherwise
bool make_tmap(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int rank, const uint64_t* dims,
               const uint64_t* strides_bytes, const uint32_t* box,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);
// bf16 tensor map: 64-element (128-byte) inner box, 128-byte swizzle, zero fill out of bounds
bool make_bf16_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box);
cudaError_t configure_tc_kernels();      // once per device, before any launch
cudaError_t configure_router_kernels();  // once per device, before any launch
cudaError_t launch_tc_gateup(const TcGemmArgs& a, cudaStream_t s);
cudaError_t launch_tc_down(const TcGemmArgs& a, cudaStream_t s);

// int8 weight-streaming decode path, see decode_i8.cu (the x planes come from the scatter)
// max_rows_per_expert: an upper bound (T) that picks the token chunk (8, 16 or 32 rows).
cudaError_t configure_dec_kernels();  // once per device, before any launch
cudaError_t configure_simt_kernels();  // once per device, before any launch
// gate/up: W1 . x and W3 . x (scaled) as fp32 K-split partials GU [nsplit, 2, R, f]
// scale_mode: COLIBRI_SCALE_PER_CHANNEL (scales per expert [f | f | d]) or
// COLIBRI_SCALE_PER_MATRIX (scales [E][3]: W1, W3, W2)
cudaError_t launch_dec_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const int8_t* W,
                              const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                              const int32_t* offsets, int nsplit, float* GU, int R, int max_rows_per_expert,
                              uint32_t* err, cudaStream_t s);
// H = silu(sum g) * (sum u) (bf16) from the gsplit partials GU, split into int8 planes with one
// scale per (down K split, row): scale[ds * R + r] covers H[r][ds * f / dsplit, (ds + 1) * f / dsplit).
cudaError_t launch_dec_finish_h(const float* GU, int gsplit, int R, int f, int dsplit, int8_t* hi, int8_t* lo,
                                float* scale, cudaStream_t s);
cudaError_t launch_dec_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const int8_t* W,
                            const float* scales, int scale_mode, int64_t wstride, int d, int f, int E,
                            const int32_t* offsets, int nsplit, int R, float* Ypart, int max_rows_per_expert,
                            uint32_t* err, cudaStream_t s);
// Group-wise int4 weights (two per byte along K, group scales [K / 128][out] per matrix, per
// expert W1 | W3 | W2): the same outputs as launch_dec_gateup / launch_dec_down.  wstride counts
// int4 elements (a multiple of 256); d and f must be multiples of 128.
cudaError_t launch_dec4_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const uint8_t* W,
                               const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                               int nsplit, float* GU, int R, int max_rows_per_expert, uint32_t* err, cudaStream_t s);
cudaError_t launch_dec4_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const uint8_t* W,
                             const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                             int nsplit, int R, float* Ypart, int max_rows_per_expert, uint32_t* err, cudaStream_t s);
// Group-wise int4 weights at decode sizes: GEMV kernels over the same planes and outputs as the
// two stream kernels above (gate/up with gsplit K splits, down with nsplit, each split a multiple
// of 1024 wide).  Needs d and f multiples of 1024.
constexpr int kGemv4MaxT = 16;  // tokens up to which the int4 path uses the GEMV kernels
bool gemv4_supported(int d, int f);
int gemv4_down_split(int f, int max_split);
int gemv4_gateup_split(int d, int T);
cudaError_t launch_gemv4_gateup(const int8_t* Xhi, const int8_t* Xlo, const float* xscale, const uint8_t* W,
                                const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                                int gsplit, float* GU, int R, int max_rows_per_expert, cudaStream_t s);
cudaError_t launch_gemv4_down(const int8_t* Hhi, const int8_t* Hlo, const float* hscale, const uint8_t* W,
                              const float* scales, int64_t wstride, int d, int f, int E, const int32_t* offsets,
                              int nsplit, int R, float* Ypart, int max_rows_per_expert, cudaStream_t s);
// The whole int8 expert stage (gate/up stream, H planes, down stream, combine) in one
// cooperative launch with grid barriers; the x planes must already be in planes_hi/lo/scale.
struct DecFusedArgs {
  int8_t* planes_hi;        // [R, max(d, f)]: x planes in, H planes written in place
  int8_t* planes_lo;
  float* planes_scale;      // x scales [R] in; H scales [dsplit, R] written
  const int8_t* W;          // expert buffer (int8) and its per-channel scales
  const float* scales;
  int scale_mode;           // COLIBRI_SCALE_PER_CHANNEL or COLIBRI_SCALE_PER_MATRIX
  int64_t wstride;
  int d, f, E, T, k;
  const int32_t* offsets;   // [E+1] (written by an earlier launch unless route_in_kernel)
  int32_t* dst_row;         // [T, k]
  float* topk_w;            // [T, k]
  int gsplit, dsplit;       // K splits of gate/up and of down
  float* GU;                // [gsplit, 2, R, f]
  float* Ypart;             // [dsplit, R, d]
  __nv_bfloat16* y;         // [T, d]
  int32_t* bar;             // [kFusedBarCount] grid-barrier counters: zero at first use, then
                            // owned by the kernel (never reset between launches)
  uint32_t* err;
  // T <= 64: 1 = router, top-k and grouping in the same launch; 2 = grouping only (topk_idx and
  // topk_w given); 0 = all done by earlier launches
  int route_in_kernel = 0;
  const __nv_bfloat16* x = nullptr;         // [T, d]
  const __nv_bfloat16* router_w = nullptr;  // [E, d]
  const float* router_b = nullptr;
  int router_flags = 0;                     // kRouterClamp | kRouterRaw
  int32_t* topk_idx = nullptr;              // [T, k]
  int32_t* counts = nullptr;                // [E]
  int32_t* offsets_out = nullptr;           // [E+1]
  int32_t* src_row = nullptr;               // [T*k]
};
constexpr int kFusedBarCount = 8;
cudaError_t launch_dec_fused(const DecFusedArgs& a, cudaStream_t s);

// ---------------------------------------------------------------------------------------
// Small device helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// Two int8 planes of a value, given the row scale a and 1/a: hi = rint(x / a), lo = rint((x - a hi)
// * 254 / a), both clamped to [-127, 127], so that x ~= a * (hi + lo / 254).
__device__ __forceinline__ void split_planes(float x, float a, float inv_a, int& qh, int& ql) {
  const float h = fminf(fmaxf(rintf(x * inv_a), -127.f), 127.f);
  const float l = fminf(fmaxf(rintf(fmaf(-a, h, x) * inv_a * 254.f), -127.f), 127.f);
  qh = (int)h;
  ql = (int)l;
}
// Router variants (colibri_desc.router_flags).  kRouterClamp limits every logit to [-50, 50]
// before selection and weighting (the gate-softmax clip option of
// www.0539edu.com/news/4774449 §5.2); kRouterRaw makes the combine weights the chosen logits
// themselves, with no softmax (www.hotelren.com/news/4731937 §3.2).  Selection is unchanged.
constexpr int kRouterClamp = 1;
constexpr int kRouterRaw = 2;
__device__ __forceinline__ float router_clamp(float l, int flags) {
  return (flags & kRouterClamp) ? fminf(fmaxf(l, -50.f), 50.f) : l;
}
// Combine weights of the k chosen logits (slot 0 the largest).
__device__ __forceinline__ void topk_weights(const float* sel_v, int k, int flags, float* w) {
  if (flags & kRouterRaw) {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) w[j] = sel_v[j];
    return;
  }
  float den = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k) den += expf(sel_v[j] - sel_v[0]);
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < k) w[j] = expf(sel_v[j] - sel_v[0]) / den;
}
// One warp selects the top-k of one token whose E logits (bias added, not yet clamped) sit in
// shared memory.
__device__ __forceinline__ void warp_topk(const float* lg, int E, int k, int flags, int lane, int32_t* idx_out,
                                          float* w_out) {
  float v[8];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int e = lane + 32 * m;
    v[m] = (e < E) ? router_clamp(lg[e], flags) : -INFINITY;
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
    float w[kMaxTopK];
    topk_weights(sel_v, k, flags, w);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) {
        idx_out[j] = sel_e[j];
        w_out[j] = w[j];
      }
  }
}

// 8 products of one 16-byte slice of x and of a router row, accumulated in order.
__device__ __forceinline__ float dot16(const uint4& xa, const uint4& wa, float acc, const __nv_bfloat16*) {
  const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xa);
  const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wa);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 xf = __bfloat1622float2(xh[i]), wf = __bfloat1622float2(wh[i]);
    acc = fmaf(xf.x, wf.x, acc);
    acc = fmaf(xf.y, wf.y, acc);
  }
  return acc;
}
__device__ __forceinline__ float dot16(const uint4& xa, const uint4& wa, float acc, const float*) {
  acc = fmaf(__uint_as_float(xa.x), __uint_as_float(wa.x), acc);
  acc = fmaf(__uint_as_float(xa.y), __uint_as_float(wa.y), acc);
  acc = fmaf(__uint_as_float(xa.z), __uint_as_float(wa.z), acc);
  acc = fmaf(__uint_as_float(xa.w), __uint_as_float(wa.w), acc);
  return acc;
}

// Plane scale of a row from its largest magnitude (an all-zero row gets 1).
__device__ __forceinline__ float plane_scale(float maxabs) { return maxabs > 0.f ? maxabs / 127.f : 1.f; }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// The same wait with cluster-scope acquire: for a barrier whose arrivals (and the shared data
// they publish) come from the other CTA of a cluster.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; give up after kWaitTimeoutNs.
// Returns false on timeout (the caller records the error and leaves its loop).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 255u) == 0 && global_ns() - t0 > kWaitTimeoutNs) return false;
  }
}

// ---------------------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// L2 policy for data read exactly once (a weight stream): evict it first, so it does not push
// out tiles that other CTAs still re-read.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// The same tensor copies with an L2 cache policy.
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                                 int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                                 int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, "
      "%4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Prefetch of a tensor tile into L2 only (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on an mbarrier once every previously issued tcgen05.mma of this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 32 lanes x 32 bits, 16 consecutive columns per thread
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------------------------------
// Clusters of two CTAs (tcgen05 cta_group::2)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address, in the cluster shared window, of the same shared variable in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 32-bit store into the shared memory of a CTA of the cluster (address from mapa_shared).
__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, int32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_shared_cluster_f32(uint32_t cluster_addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA loads into this CTA's shared memory whose completion is counted on an mbarrier of the
// pair's leader CTA (cluster address).  No multicast.
__device__ __forceinline__ void tma2_load_2d(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma2_load_3d(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma2_load_4d(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma2_load_5d(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                             int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}
// The same pair copies with an L2 cache policy (weights read by a single tile: evict first).
__device__ __forceinline__ void tma2_load_3d_hint(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                  int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
      "[%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma2_load_5d_hint(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int c0,
                                                  int c1, int c2, int c3, int c4, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
      "[%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Pair MMA issued by the leader CTA: A rows 0-127 and B rows (N) 0-127 from the leader's shared
// memory, A rows 128-255 and B rows 128-255 from the peer's, at the same descriptor addresses.
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at this shared offset in every CTA of `cta_mask` when the pair
// MMAs issued so far by this thread complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with 128-byte
// swizzle: rows of 128 bytes, 8-row core groups 1024 bytes apart (stride byte offset), the
// leading byte offset unused by this layout (encoded as 16 bytes), descriptor version 1,
// layout type 2 = 128-byte swizzle.  The tile base must be 1024-byte aligned; stepping K by
// 16 bf16 inside the atom adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address >> 4, bits 0-13
  desc |= (uint64_t)(16u >> 4) << 16;                // leading byte offset >> 4, bits 16-29
  desc |= (uint64_t)(1024u >> 4) << 32;              // stride byte offset >> 4, bits 32-45
  desc |= (uint64_t)1 << 46;                         // version, bits 46-47
  desc |= (uint64_t)2 << 61;                         // 128-byte swizzle, bits 61-63
  return desc;
}

// Instruction descriptor, kind::i8: signed int8 A and B, s32 D, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_s8_s32(int M, int N) {
  return (2u << 4)                          // D format: s32
         | (1u << 7)                        // A format: signed 8-bit
         | (1u << 10)                       // B format: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)       // N >> 3
         | ((uint32_t)(M >> 4) << 24);      // M >> 4
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::i8 (int8 inputs, s32 accumulate)
__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((uint32_t)(N >> 3) << 17)       // N >> 3
         | ((uint32_t)(M >> 4) << 24);      // M >> 4
}

}  // namespace colibri
