// Host side of the C ABI declared in include/colibri.h: argument validation, workspace
// ownership, host/device pointer handling and the stream-ordered launch sequence
//   router_topk -> route_count -> route_scan -> route_scatter -> expert FFN -> combine.
// No host synchronisation inside a forward (unless COLIBRI_PROFILE=1).
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>

#include "common.cuh"

using namespace colibri;

namespace {

thread_local std::string g_last_error;

bool env_flag(const char* name) {
  const char* v = getenv(name);
  return v && *v && strcmp(v, "0") != 0;
}

colibri_status fail(colibri_ctx* ctx, colibri_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  if (ctx) ctx->last_error = buf;
  if (env_flag("COLIBRI_DEBUG")) fprintf(stderr, "[colibri] %s: %s\n", colibri_status_string(st), buf);
  return st;
}

size_t dtype_size(int dt) { return dt == COLIBRI_F32 ? 4 : (dt == COLIBRI_BF16 ? 2 : 1); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool changed = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) {
      changed = cudaSetDevice(dev) == cudaSuccess;
    }
  }
  ~DeviceGuard() {
    if (changed) cudaSetDevice(prev);
  }
};

enum PtrKind { kPtrDevice, kPtrHost, kPtrBad };

PtrKind classify(const void* p, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return kPtrHost;
  }
  switch (at.type) {
    case cudaMemoryTypeDevice:
      return at.device == dev ? kPtrDevice : kPtrBad;
    case cudaMemoryTypeManaged:
      return kPtrDevice;
    case cudaMemoryTypeHost:
    case cudaMemoryTypeUnregistered:
    default:
      return kPtrHost;
  }
}

// K splits of the int8 down projection: each split must cover whole 128-byte K blocks.
int pick_dec_split(int f) {
  if (f % 128 != 0) return 1;
  const int blocks = f / 128;
  for (int s = kDecSplitMax; s > 1; s >>= 1)
    if (blocks % s == 0) return s;
  return 1;
}

// Tile shape of the bf16 expert GEMMs: 0 = one CTA, 128 rows x 256 columns; 1 = pairs of CTAs
// (cta_group::2), 256 x 256.  Pair tiles by default: a CTA moves 32 KB from L2 per 128x256x64
// unit instead of 48 KB, and an expert's last m-tile of at most 128 rows runs with swapped
// operands, so the 256-row tile no longer pads small groups (measured on B200: the 128-expert
// layer 678 against 711 us per step, the skewed layer 998 against 1027 us, the Mixtral-shaped
// layer unchanged in mode).  COLIBRI_GEMM_CTA=1 or 2 forces a mode (both are exact).
enum GemmMode { kGemmOne = 0, kGemmPair = 1 };
int gemm_mode(int /*avg_rows_per_expert*/) {
  const char* v = getenv("COLIBRI_GEMM_CTA");
  if (v && v[0] == '1') return kGemmOne;
  return kGemmPair;
}

constexpr size_t kMaxGraphs = 8;  // captured forwards kept per context (least recently used evicted)

// Workspace carve-out: every buffer 256-byte aligned inside one allocation.
struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  }
};

}  // namespace

namespace colibri {
// Records the reason of a failure of a context-free entry point (read by colibri_last_error(NULL)).
void record_error(const char* msg) {
  g_last_error = msg;
  if (env_flag("COLIBRI_DEBUG")) fprintf(stderr, "[colibri] %s\n", msg);
}
// Records the reason of a failure on a context (or on no context) and returns `st`.
colibri_status report(colibri_ctx* ctx, colibri_status st, const char* msg) { return fail(ctx, st, "%s", msg); }
}  // namespace colibri

extern "C" {

const char* colibri_status_string(colibri_status st) {
  switch (st) {
    case COLIBRI_OK: return "COLIBRI_OK";
    case COLIBRI_ERR_INVALID_ARG: return "COLIBRI_ERR_INVALID_ARG: invalid argument";
    case COLIBRI_ERR_ALIGNMENT: return "COLIBRI_ERR_ALIGNMENT: tensor not 16-byte aligned";
    case COLIBRI_ERR_UNSUPPORTED: return "COLIBRI_ERR_UNSUPPORTED: configuration not supported";
    case COLIBRI_ERR_OOM: return "COLIBRI_ERR_OOM: workspace allocation failed";
    case COLIBRI_ERR_CUDA: return "COLIBRI_ERR_CUDA: CUDA call or launch failed";
    case COLIBRI_ERR_TIMEOUT: return "COLIBRI_ERR_TIMEOUT: a device-side wait gave up";
  }
  return "COLIBRI: unknown status";
}

const char* colibri_last_error(const colibri_ctx* ctx) {
  if (ctx) return ctx->last_error.c_str();
  return g_last_error.c_str();
}

int64_t colibri_expert_stride(const colibri_ctx* ctx) { return ctx ? ctx->expert_stride : -1; }

colibri_status colibri_init(const colibri_desc* desc, colibri_ctx** out) {
  if (!out) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!desc) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "desc is NULL");
  const colibri_desc& D = *desc;
  if (D.d_model < 64 || D.d_model % 64 != 0 || D.d_model > 65536)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "d_model=%d must be a positive multiple of 64 (<= 65536)", D.d_model);
  if (D.d_ff < 64 || D.d_ff % 64 != 0 || D.d_ff > 262144)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "d_ff=%d must be a positive multiple of 64 (<= 262144)", D.d_ff);
  if (D.shared_d_ff < 0 || D.shared_d_ff % 64 != 0 || D.shared_d_ff > 262144)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "shared_d_ff=%d must be 0 or a multiple of 64", D.shared_d_ff);
  if (D.num_experts < 1 || D.num_experts > kMaxExperts)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "num_experts=%d must be in [1, %d]", D.num_experts, kMaxExperts);
  if (D.top_k < 1 || D.top_k > kMaxTopK || D.top_k > D.num_experts)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "top_k=%d must be in [1, min(E, %d)]", D.top_k, kMaxTopK);
  if (D.max_tokens < 1)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "max_tokens=%d must be >= 1", D.max_tokens);
  if (D.router_flags & ~(COLIBRI_ROUTER_CLAMP | COLIBRI_ROUTER_RAW_WEIGHTS))
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "router_flags=0x%x has unknown bits", (unsigned)D.router_flags);
  if (D.weight_scale_mode != COLIBRI_SCALE_PER_CHANNEL && D.weight_scale_mode != COLIBRI_SCALE_PER_MATRIX)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "weight_scale_mode=%d unknown", D.weight_scale_mode);
  if ((int64_t)D.max_tokens * D.top_k > (1ll << 30))
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "max_tokens * top_k too large");
  const bool f32 = D.act_dtype == COLIBRI_F32 && D.weight_dtype == COLIBRI_F32;
  const bool bf16 = D.act_dtype == COLIBRI_BF16 && D.weight_dtype == COLIBRI_BF16;
  const bool w8 = D.act_dtype == COLIBRI_BF16 && D.weight_dtype == COLIBRI_I8;
  const bool w4 = D.act_dtype == COLIBRI_BF16 && D.weight_dtype == COLIBRI_I4;
  const bool i8 = w8 || w4;  // the weight-streaming path (int8 tensor cores over activation planes)
  if (D.act_dtype < 0 || D.act_dtype > 2 || D.weight_dtype < 0 || D.weight_dtype > 3)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "unknown dtype code (act=%d, weight=%d)", D.act_dtype, D.weight_dtype);
  if (!f32 && !bf16 && !i8)
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "dtype pair (act=%d, weight=%d) not supported", D.act_dtype, D.weight_dtype);
  if (i8 && D.shared_d_ff > 0)
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "shared expert with int8 / int4 weights is not supported");
  if (i8 && D.d_ff > kDecMaxFF)
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "int8 / int4 weights support d_ff <= %d", kDecMaxFF);
  if (w4 && (D.d_model % 128 != 0 || D.d_ff % 128 != 0))
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "int4 weights need d_model and d_ff multiples of 128 (the scale group)");
  if (!w8 && D.weight_scale_mode != COLIBRI_SCALE_PER_CHANNEL)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "weight_scale_mode applies to int8 weights only");
  if (f32 && ((int64_t)D.max_tokens * D.top_k / kSimtBM + D.num_experts > 65535 ||
              ((int64_t)D.max_tokens + kSimtBM - 1) / kSimtBM > 65535))
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "fp32 path limited to max_tokens * top_k < 4M rows");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return fail(nullptr, COLIBRI_ERR_CUDA, "no CUDA device available");
  }
  if (D.device_id < 0 || D.device_id >= ndev)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "device_id=%d out of range (%d devices)", D.device_id, ndev);
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, D.device_id) != cudaSuccess)
    return fail(nullptr, COLIBRI_ERR_CUDA, "cudaGetDeviceProperties failed");
  if (prop.major != 10)
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                D.device_id, prop.major, prop.minor);

  colibri_ctx* ctx = new (std::nothrow) colibri_ctx();
  if (!ctx) return fail(nullptr, COLIBRI_ERR_OOM, "host allocation failed");
  ctx->desc = D;
  ctx->sm_count = prop.multiProcessorCount;
  // int4: 256 elements = 128 bytes, so every expert still starts on a 128-byte boundary
  const int64_t stride_unit = D.weight_dtype == COLIBRI_I4 ? 256 : 128;
  ctx->expert_stride = ((int64_t)3 * D.d_model * D.d_ff + stride_unit - 1) / stride_unit * stride_unit;
  ctx->profile = env_flag("COLIBRI_PROFILE");
  ctx->dec_split = i8 ? pick_dec_split(D.d_ff) : 1;

  const int64_t M = D.max_tokens, R = M * D.top_k, d = D.d_model, f = D.d_ff, fs = D.shared_d_ff;
  const int E = D.num_experts;
  const size_t as = dtype_size(D.act_dtype);
  const size_t hs = f32 ? 4 : 2;
  const int nblk = (int)((M + kCountBlock - 1) / kCountBlock);
  ctx->nblk_max = nblk;
  Carver c;
  const size_t o_xs = c.take(M * d * as), o_ys = c.take(M * d * as);
  const size_t o_xs2 = c.take(M * d * as), o_ys2 = c.take(M * d * as);  // second pair (staged calls alternate)
  const size_t o_idx = c.take(R * 4), o_w = c.take(R * 4), o_dst = c.take(R * 4), o_src = c.take(R * 4);
  const size_t o_bc = c.take((size_t)nblk * E * 4), o_bb = c.take((size_t)nblk * E * 4);
  const size_t o_cnt = c.take(E * 4), o_off = c.take((E + 1) * 4), o_mt = c.take((E + 1) * 4);
  const size_t o_xp = c.take(i8 ? 0 : R * d * as);  // int8 weights read the row planes instead
  const size_t o_h = c.take(i8 ? std::max<int64_t>(2 * R, 2 * kDecGateSplitMax * std::min<int64_t>(R, kDecGateSplitRows)) * f * 4
                             : R * f * hs);
  const size_t o_yp = i8 ? c.take(0) : c.take(R * d * hs);
  const size_t o_hs = c.take(fs > 0 ? M * fs * hs : 0);
  const size_t o_ysh = c.take(fs > 0 ? M * d * hs : 0);
  const int64_t part_rows = i8 ? std::max<int64_t>(R, (int64_t)ctx->dec_split * std::min<int64_t>(R, 256)) : 0;
  const size_t o_part = c.take(part_rows * d * 4);
  const size_t plane_w = (size_t)std::max<int64_t>(d, f);
  const size_t o_phi = c.take(i8 ? R * plane_w : 0), o_plo = c.take(i8 ? R * plane_w : 0);
  const size_t o_psc = c.take(i8 ? part_rows * 4 : 0);  // per (down K split, row) scales of the H planes
  const size_t o_err = c.take(4);
  const size_t o_tsched = c.take(4 * 4);
  const size_t o_gbar = c.take(i8 ? kFusedBarCount * 4 : 0);
  ctx->ws_bytes = c.off;

  DeviceGuard guard(D.device_id);
  if (cudaMalloc(&ctx->ws_base, ctx->ws_bytes) != cudaSuccess) {
    cudaGetLastError();
    const size_t want = ctx->ws_bytes;
    delete ctx;
    return fail(nullptr, COLIBRI_ERR_OOM, "cudaMalloc of %zu workspace bytes failed", want);
  }
  uint8_t* b = static_cast<uint8_t*>(ctx->ws_base);
  Workspace& w = ctx->ws;
  w.x_stage = b + o_xs;
  w.y_stage = b + o_ys;
  w.x_stage2 = b + o_xs2;
  w.y_stage2 = b + o_ys2;
  w.topk_idx = reinterpret_cast<int32_t*>(b + o_idx);
  w.topk_w = reinterpret_cast<float*>(b + o_w);
  w.dst_row = reinterpret_cast<int32_t*>(b + o_dst);
  w.src_row = reinterpret_cast<int32_t*>(b + o_src);
  w.blk_counts = reinterpret_cast<int32_t*>(b + o_bc);
  w.blk_base = reinterpret_cast<int32_t*>(b + o_bb);
  w.counts = reinterpret_cast<int32_t*>(b + o_cnt);
  w.offsets = reinterpret_cast<int32_t*>(b + o_off);
  w.mt_prefix = reinterpret_cast<int32_t*>(b + o_mt);
  w.Xp = b + o_xp;
  w.H = b + o_h;
  w.Yp = b + o_yp;
  w.Hs = b + o_hs;
  w.Ys = b + o_ysh;
  w.Ypart = reinterpret_cast<float*>(b + o_part);
  w.plane_hi = reinterpret_cast<int8_t*>(b + o_phi);
  w.plane_lo = reinterpret_cast<int8_t*>(b + o_plo);
  w.plane_scale = reinterpret_cast<float*>(b + o_psc);
  w.err = reinterpret_cast<uint32_t*>(b + o_err);
  w.tile_sched = reinterpret_cast<uint32_t*>(b + o_tsched);
  w.grid_bar = i8 ? reinterpret_cast<int32_t*>(b + o_gbar) : nullptr;
  if (cudaMemset(w.err, 0, 4) != cudaSuccess || cudaMemset(w.tile_sched, 0, 4 * 4) != cudaSuccess ||
      (i8 && cudaMemset(w.grid_bar, 0, kFusedBarCount * 4) != cudaSuccess)) {
    cudaFree(ctx->ws_base);
    delete ctx;
    return fail(nullptr, COLIBRI_ERR_CUDA, "cudaMemset failed");
  }
  if (ctx->profile) {
    for (auto& e : ctx->ev) cudaEventCreate(&e);
  }
  for (auto& e : ctx->cap_ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      e = nullptr;
    }
  }
  ctx->use_graphs = !(getenv("COLIBRI_GRAPHS") && strcmp(getenv("COLIBRI_GRAPHS"), "0") == 0);
  // COLIBRI_TILE_SCHED=static: the bf16 GEMMs walk their tiles round-robin instead of claiming them
  ctx->tile_static = getenv("COLIBRI_TILE_SCHED") && strcmp(getenv("COLIBRI_TILE_SCHED"), "static") == 0;
  // COLIBRI_I4_GEMV=0: int4 weights always take the tensor-core stream kernels
  ctx->i4_gemv = !(getenv("COLIBRI_I4_GEMV") && strcmp(getenv("COLIBRI_I4_GEMV"), "0") == 0);
  // Programmatic dependent launch measured slower on the small-batch decode chain and neutral on
  // prefill, so it is opt-in (COLIBRI_PDL=1).
  ctx->use_pdl = env_flag("COLIBRI_PDL");
  ctx->dec_fused = !(getenv("COLIBRI_DEC_FUSED") && strcmp(getenv("COLIBRI_DEC_FUSED"), "0") == 0);
  ctx->dec_route = !(getenv("COLIBRI_DEC_ROUTE") && strcmp(getenv("COLIBRI_DEC_ROUTE"), "0") == 0);
  cudaError_t ce = configure_router_kernels();
  if (ce == cudaSuccess) ce = configure_tc_kernels();
  if (ce == cudaSuccess) ce = configure_dec_kernels();
  if (ce == cudaSuccess) ce = configure_simt_kernels();
  if (ce != cudaSuccess) {
    cudaGetLastError();
    cudaFree(ctx->ws_base);
    delete ctx;
    return fail(nullptr, COLIBRI_ERR_CUDA, "kernel configuration failed: %s", cudaGetErrorString(ce));
  }
  // copy streams and events of staged (host x / y) calls; without them such calls copy on the
  // caller's stream
  {
    bool ok = cudaStreamCreateWithFlags(&ctx->cs_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&ctx->cs_out, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& e : ctx->st_ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) cudaGetLastError();
    ctx->staged = ok && !(getenv("COLIBRI_STAGED") && strcmp(getenv("COLIBRI_STAGED"), "0") == 0);
  }
  *out = ctx;
  return COLIBRI_OK;
}

void colibri_free(colibri_ctx* ctx) {
  if (!ctx) return;
  {
    DeviceGuard guard(ctx->desc.device_id);
    if (ctx->ws_base) cudaFree(ctx->ws_base);
    for (auto& e : ctx->ev)
      if (e) cudaEventDestroy(e);
    for (auto& e : ctx->prof_ev)
      if (e) cudaEventDestroy(e);
    for (auto& e : ctx->cap_ev)
      if (e) cudaEventDestroy(e);
    for (auto& g : ctx->graphs) {
      cudaGraphExecDestroy(g.exec);
      if (g.graph) cudaGraphDestroy(g.graph);
    }
    for (auto& e : ctx->st_ev)
      if (e) cudaEventDestroy(e);
    if (ctx->cs_in) cudaStreamDestroy(ctx->cs_in);
    if (ctx->cs_out) cudaStreamDestroy(ctx->cs_out);
  }
  delete ctx;
}

}  // extern "C"

namespace {

colibri_status check_launch(colibri_ctx* ctx, cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(ctx, COLIBRI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return COLIBRI_OK;
}

#define COLIBRI_TRY(expr, what)                                 \
  do {                                                          \
    colibri_status st_ = check_launch(ctx, (expr), (what));     \
    if (st_ != COLIBRI_OK) return st_;                          \
  } while (0)

// The launch sequence of one forward (stream-ordered, no host synchronisation unless
// COLIBRI_PROFILE printing is on).
// stage_ev: NULL, or 6 events recorded at the stage boundaries (as event-record nodes when
// `ev_nodes` is set: the forward is then being captured into a graph for timed replays).
colibri_status enqueue_forward(colibri_ctx* ctx, const void* x, PtrKind xk, int32_t T, const void* router_w,
                               const float* router_b, const int32_t* user_idx, const float* user_w,
                               const void* expert_w, const float* expert_scales, const void* shared_w, void* y,
                               PtrKind yk, cudaStream_t s, int gemm, cudaEvent_t* stage_ev, bool ev_nodes) {
  const colibri_desc& D = ctx->desc;
  const bool routed_by_caller = user_idx != nullptr;
  Workspace& w = ctx->ws;
  const int d = D.d_model, f = D.d_ff, fs = D.shared_d_ff, E = D.num_experts, k = D.top_k;
  const int act = D.act_dtype;
  const size_t row_bytes = (size_t)d * dtype_size(act);
  const int R = T * k;
  const void* xd = x;
  void* yd = y;
  // Kernels after the first may overlap their predecessor's tail (not while stage events are
  // recorded between them: the events would then not bound the stages).
  LaunchScope launch_scope(ctx->use_pdl && !ctx->profile && stage_ev == nullptr);
  if (xk == kPtrHost) {
    COLIBRI_TRY(cudaMemcpyAsync(w.x_stage, x, (size_t)T * row_bytes, cudaMemcpyHostToDevice, s), "copy x to device");
    launch_chain_break();
    xd = w.x_stage;
  }
  if (yk == kPtrHost) yd = w.y_stage;
  // stage boundary events: COLIBRI_PROFILE printing and/or colibri_profile_begin recording
  auto mark = [&](int i) {
    if (ctx->profile) cudaEventRecord(ctx->ev[i], s);
    if (stage_ev) {
      if (ev_nodes) cudaEventRecordWithFlags(stage_ev[i], s, cudaEventRecordExternal);
      else cudaEventRecord(stage_ev[i], s);
    }
  };
  mark(0);

  // int8 weights, T <= 64: router, top-k and grouping run as phase 0 of the fused expert launch
  // (COLIBRI_DEC_ROUTE=0: as two launches before it).  With the weight streams evicted first
  // from L2 the router's inputs stay resident and the one launch is the faster plan (T=1: 0.0856
  // against 0.0874 ms per step, T=8: 0.198 against 0.204 ms).
  const bool route_in_dec =
      D.weight_dtype == COLIBRI_I8 && ctx->dec_fused && ctx->dec_route && T <= kFusedRouteMaxT;
  const bool quant = D.weight_dtype == COLIBRI_I8 || D.weight_dtype == COLIBRI_I4;

  // ---- Gate
  if (routed_by_caller) {
    COLIBRI_TRY(cudaMemcpyAsync(w.topk_idx, user_idx, (size_t)R * 4, cudaMemcpyDeviceToDevice, s), "copy topk_idx");
    COLIBRI_TRY(cudaMemcpyAsync(w.topk_w, user_w, (size_t)R * 4, cudaMemcpyDeviceToDevice, s), "copy topk_w");
    launch_chain_break();
  } else if (!route_in_dec) {
    COLIBRI_TRY(launch_router_topk(xd, act, T, d, router_w, router_b, E, k, D.router_flags, w.topk_idx, w.topk_w, w.err, s),
                "router_topk");
  }
  mark(1);

  // ---- Scatter
  const int nblk = (T + kCountBlock - 1) / kCountBlock;
  const int bm = D.weight_dtype == COLIBRI_F32 ? kSimtBM : (gemm == kGemmPair ? kTcPairBM : kTcBM);
  const RowPlanes xplanes{w.plane_hi, w.plane_lo, w.plane_scale};
  const RowPlanes* planes = quant ? &xplanes : nullptr;
  if (route_in_dec) {
    // grouping and the x planes are phase 0 of the fused expert launch
  } else if (T <= kFusedRouteMaxT) {
    COLIBRI_TRY(launch_route_fused(xd, act, T, d, w.topk_idx, k, E, bm, w.counts, w.offsets, w.mt_prefix,
                                   w.src_row, w.dst_row, w.Xp, planes, s), "route_fused");
  } else {
    COLIBRI_TRY(launch_route_count(w.topk_idx, T, k, E, w.blk_counts, w.dst_row, s), "route_count");
    COLIBRI_TRY(launch_route_scan(w.blk_counts, nblk, E, bm, w.blk_base, w.counts, w.offsets, w.mt_prefix, s),
                "route_scan");
    COLIBRI_TRY(launch_route_scatter(xd, act, T, d, k, E, w.topk_idx, w.blk_base, w.offsets, w.dst_row, w.src_row,
                                     w.Xp, planes, s), "route_scatter");
  }
  mark(2);

  // ---- Expert compute
  const int64_t stride = ctx->expert_stride;
  int nsplit = 1;
  if (D.weight_dtype == COLIBRI_F32) {
    SimtGroups g{w.offsets, w.mt_prefix, E, 0};
    const int mt_bound = R / kSimtBM + E;
    SimtGroups gs{nullptr, nullptr, 1, T};
    const int mts = (T + kSimtBM - 1) / kSimtBM;
    COLIBRI_TRY(launch_simt_gateup((const float*)w.Xp, d, (const float*)expert_w, stride, d, f, g, mt_bound,
                                   (float*)w.H, s), "simt_gateup");
    if (fs > 0)
      COLIBRI_TRY(launch_simt_gateup((const float*)xd, d, (const float*)shared_w, 0, d, fs, gs, mts,
                                     (float*)w.Hs, s), "simt_gateup_shared");
    mark(3);
    COLIBRI_TRY(launch_simt_down((const float*)w.H, f, (const float*)expert_w, stride, d, g, mt_bound,
                                 (float*)w.Yp, s), "simt_down");
    if (fs > 0)
      COLIBRI_TRY(launch_simt_down((const float*)w.Hs, fs, (const float*)shared_w, 0, d, gs, mts,
                                   (float*)w.Ys, s), "simt_down_shared");
  } else if (D.weight_dtype == COLIBRI_BF16) {
    TcGemmArgs a;
    a.A = w.Xp;
    a.rows = R;
    a.offsets = w.offsets;
    a.mt_prefix = w.mt_prefix;
    a.E = E;
    a.W = expert_w;
    a.wstride = stride;
    a.out = w.H;
    a.A_sh = xd;
    a.rows_sh = T;
    a.W_sh = shared_w;
    a.out_sh = w.Hs;
    a.d = d;
    a.f = f;
    a.fs = fs;
    a.mt_bound = R / bm + E;
    a.err = w.err;
    a.sm_count = ctx->sm_count;
    a.pair = gemm == kGemmPair;
    a.sched = ctx->tile_static ? nullptr : w.tile_sched;
    COLIBRI_TRY(launch_tc_gateup(a, s), "tc_gateup");
    mark(3);
    a.sched = ctx->tile_static ? nullptr : w.tile_sched + 2;
    a.A = w.H;
    a.out = w.Yp;
    a.A_sh = w.Hs;
    a.out_sh = w.Ys;
    COLIBRI_TRY(launch_tc_down(a, s), "tc_down");
  } else {
    // K splits of the down projection: enough work items to cover every SM a few times
    nsplit = 1;
    if (R <= 256) {
      const int touched = std::min(E, R), tiles = (d + 127) / 128;
      while (nsplit < ctx->dec_split && touched * tiles * nsplit < 4 * ctx->sm_count) nsplit <<= 1;
    }
    // K splits of the gate/up projection (partials summed before SiLU by the finishing kernel).
    // Up to 4: 8 splits (64 KB items) measured slower for one token (gate/up phase 5 us longer).
    int gsplit = 1;
    if (R <= kDecGateSplitRows && d % 128 == 0) {
      const int touched = std::min(E, R), tiles = 2 * ((f + 127) / 128);
      while (gsplit < kDecGateSplitMax && (d / 128) % (2 * gsplit) == 0 &&
             touched * tiles * gsplit < 8 * ctx->sm_count)
        gsplit <<= 1;
    }
    if (D.weight_dtype == COLIBRI_I4 && ctx->i4_gemv && T <= kGemv4MaxT && gemv4_supported(d, f)) {
      // int4 at decode sizes: dp4a GEMV for gate/up, H planes, dp4a GEMV for down
      nsplit = gemv4_down_split(f, ctx->dec_split);
      const int g4split = gemv4_gateup_split(d, T);
      COLIBRI_TRY(launch_gemv4_gateup(w.plane_hi, w.plane_lo, w.plane_scale, (const uint8_t*)expert_w, expert_scales,
                                      stride, d, f, E, w.offsets, g4split, (float*)w.H, R, T, s), "gemv4_gateup");
      mark(3);
      COLIBRI_TRY(launch_dec_finish_h((const float*)w.H, g4split, R, f, nsplit, w.plane_hi, w.plane_lo,
                                      w.plane_scale, s), "dec_finish_h");
      COLIBRI_TRY(launch_gemv4_down(w.plane_hi, w.plane_lo, w.plane_scale, (const uint8_t*)expert_w, expert_scales,
                                    stride, d, f, E, w.offsets, nsplit, R, w.Ypart, T, s), "gemv4_down");
    } else if (D.weight_dtype == COLIBRI_I4) {
      // int4: the stream kernels that widen the packed tiles, then H planes, then down
      COLIBRI_TRY(launch_dec4_gateup(w.plane_hi, w.plane_lo, w.plane_scale, (const uint8_t*)expert_w, expert_scales,
                                     stride, d, f, E, w.offsets, gsplit, (float*)w.H, R, T, w.err, s), "dec4_gateup");
      mark(3);
      COLIBRI_TRY(launch_dec_finish_h((const float*)w.H, gsplit, R, f, nsplit, w.plane_hi, w.plane_lo,
                                      w.plane_scale, s), "dec_finish_h");
      COLIBRI_TRY(launch_dec4_down(w.plane_hi, w.plane_lo, w.plane_scale, (const uint8_t*)expert_w, expert_scales,
                                   stride, d, f, E, w.offsets, nsplit, R, w.Ypart, T, w.err, s), "dec4_down");
    } else if (ctx->dec_fused) {
      // one cooperative launch for gate/up, H, down and the combine (stages 3-5 are empty)
      DecFusedArgs fa;
      fa.planes_hi = w.plane_hi;
      fa.planes_lo = w.plane_lo;
      fa.planes_scale = w.plane_scale;
      fa.W = (const int8_t*)expert_w;
      fa.scales = expert_scales;
      fa.scale_mode = D.weight_scale_mode;
      fa.wstride = stride;
      fa.d = d;
      fa.f = f;
      fa.E = E;
      fa.T = T;
      fa.k = k;
      fa.offsets = w.offsets;
      fa.dst_row = w.dst_row;
      fa.topk_w = w.topk_w;
      fa.gsplit = gsplit;
      fa.dsplit = nsplit;
      fa.GU = (float*)w.H;
      fa.Ypart = w.Ypart;
      fa.y = (__nv_bfloat16*)yd;
      fa.bar = w.grid_bar;
      fa.err = w.err;
      if (route_in_dec) {
        fa.route_in_kernel = routed_by_caller ? 2 : 1;
        fa.x = (const __nv_bfloat16*)xd;
        fa.router_w = (const __nv_bfloat16*)router_w;
        fa.router_b = router_b;
        fa.router_flags = D.router_flags;
        fa.topk_idx = w.topk_idx;
        fa.counts = w.counts;
        fa.offsets_out = w.offsets;
        fa.src_row = w.src_row;
      }
      COLIBRI_TRY(launch_dec_fused(fa, s), "dec_fused");
      mark(3);
    } else {
      COLIBRI_TRY(launch_dec_gateup(w.plane_hi, w.plane_lo, w.plane_scale, (const int8_t*)expert_w, expert_scales,
                                    D.weight_scale_mode, stride, d, f, E, w.offsets, gsplit, (float*)w.H, R, T, w.err, s), "dec_gateup");
      mark(3);
      COLIBRI_TRY(launch_dec_finish_h((const float*)w.H, gsplit, R, f, nsplit, w.plane_hi, w.plane_lo,
                                      w.plane_scale, s), "dec_finish_h");
      COLIBRI_TRY(launch_dec_down(w.plane_hi, w.plane_lo, w.plane_scale, (const int8_t*)expert_w, expert_scales,
                                  D.weight_scale_mode, stride, d, f, E, w.offsets, nsplit, R, w.Ypart, T, w.err, s), "dec_down");
    }
  }
  mark(4);

  // ---- Gather
  if (D.weight_dtype == COLIBRI_I8 && ctx->dec_fused) {
    // done inside the fused kernel
  } else if (quant) {
    COLIBRI_TRY(launch_combine_split(w.Ypart, nsplit, R, w.dst_row, w.topk_w, T, k, d, yd, act, s),
                "combine_split");
  } else {
    const int yp_dtype = D.weight_dtype == COLIBRI_F32 ? COLIBRI_F32 : COLIBRI_BF16;
    COLIBRI_TRY(launch_combine(w.Yp, yp_dtype, w.dst_row, w.topk_w, T, k, d, fs > 0 ? w.Ys : nullptr, yd, act, s),
                "combine");
  }
  mark(5);
  if (yk == kPtrHost)
    COLIBRI_TRY(cudaMemcpyAsync(y, yd, (size_t)T * row_bytes, cudaMemcpyDeviceToHost, s), "copy y to host");

  if (ctx->profile) {
    cudaStreamSynchronize(s);
    float ms[5] = {0, 0, 0, 0, 0}, tot = 0;
    for (int i = 0; i < 5; ++i) cudaEventElapsedTime(&ms[i], ctx->ev[i], ctx->ev[i + 1]);
    cudaEventElapsedTime(&tot, ctx->ev[0], ctx->ev[5]);
    fprintf(stderr, "[colibri] T=%d Gate %.4f ms | Scatter %.4f ms | ExpertCompute %.4f ms | Gather %.4f ms | Total %.4f ms\n",
            T, ms[0], ms[1], ms[2] + ms[3], ms[4], tot);
  }
  return COLIBRI_OK;
}

colibri_status forward_device(colibri_ctx* ctx, const void* x, PtrKind xk, int32_t T, const void* router_w,
                              const float* router_b, const int32_t* user_idx, const float* user_w,
                              const void* expert_w, const float* expert_scales, const void* shared_w, void* y,
                              PtrKind yk, cudaStream_t s);

bool stream_capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return true;
  }
  return cs != cudaStreamCaptureStatusNone;
}

// Host x and/or y: the call alternates between two device staging pairs, and its copies run on
// the context's two copy streams, ordered by events:
//   cs_in:  waits until the forward two calls back has read this pair's x buffer, copies x in;
//   stream: waits for that copy, runs the forward on device pointers (a replayed graph);
//   cs_out: waits for the forward, copies y out; stream then waits for that copy.
// So the next call's input copy overlaps this call's compute, host y is valid once `stream` has
// been synchronised (as for the single-stream path), and every later use of a staging buffer on
// `stream` comes after the copies that read it.
colibri_status forward_staged(colibri_ctx* ctx, const void* x, PtrKind xk, int32_t T, const void* router_w,
                              const float* router_b, const int32_t* user_idx, const float* user_w,
                              const void* expert_w, const float* expert_scales, const void* shared_w, void* y,
                              PtrKind yk, cudaStream_t s) {
  const colibri_desc& D = ctx->desc;
  Workspace& w = ctx->ws;
  const size_t bytes = (size_t)T * D.d_model * (D.act_dtype == COLIBRI_F32 ? 4 : 2);
  const int b = ctx->stage_next;
  ctx->stage_next ^= 1;
  cudaEvent_t* ev = ctx->st_ev + 4 * b;  // x buffer free, x copied in, forward done, y copied out
  void* xs = b ? w.x_stage2 : w.x_stage;
  void* ys = b ? w.y_stage2 : w.y_stage;
  const void* xd = x;
  void* yd = y;
  if (xk == kPtrHost) {
    COLIBRI_TRY(cudaStreamWaitEvent(ctx->cs_in, ev[0], 0), "staged: wait for the x buffer");
    COLIBRI_TRY(cudaMemcpyAsync(xs, x, bytes, cudaMemcpyHostToDevice, ctx->cs_in), "staged: copy x to device");
    COLIBRI_TRY(cudaEventRecord(ev[1], ctx->cs_in), "staged: record x copy");
    COLIBRI_TRY(cudaStreamWaitEvent(s, ev[1], 0), "staged: wait for the x copy");
    xd = xs;
  }
  if (yk == kPtrHost) yd = ys;
  const colibri_status st = forward_device(ctx, xd, kPtrDevice, T, router_w, router_b, user_idx, user_w, expert_w,
                                           expert_scales, shared_w, yd, kPtrDevice, s);
  if (st != COLIBRI_OK) return st;
  if (xk == kPtrHost) COLIBRI_TRY(cudaEventRecord(ev[0], s), "staged: record x buffer free");
  if (yk == kPtrHost) {
    COLIBRI_TRY(cudaEventRecord(ev[2], s), "staged: record forward done");
    COLIBRI_TRY(cudaStreamWaitEvent(ctx->cs_out, ev[2], 0), "staged: wait for the forward");
    COLIBRI_TRY(cudaMemcpyAsync(y, ys, bytes, cudaMemcpyDeviceToHost, ctx->cs_out), "staged: copy y to host");
    COLIBRI_TRY(cudaEventRecord(ev[3], ctx->cs_out), "staged: record y copy");
    COLIBRI_TRY(cudaStreamWaitEvent(s, ev[3], 0), "staged: wait for the y copy");
  }
  return COLIBRI_OK;
}

// Shared body of both forward entry points.  topk_idx/topk_w non-NULL = caller routing.
colibri_status forward_impl(colibri_ctx* ctx, const void* x, int32_t T, const void* router_w,
                            const float* router_b, const int32_t* user_idx, const float* user_w,
                            const void* expert_w, const float* expert_scales, const void* shared_w,
                            void* y, void* stream_ptr) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  const colibri_desc& D = ctx->desc;
  const bool routed_by_caller = user_idx != nullptr || user_w != nullptr;
  if (T < 0 || T > D.max_tokens)
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, D.max_tokens);
  if (!x || !expert_w || !y) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "x, expert_w and y must be non-NULL");
  if (routed_by_caller) {
    if (!user_idx || !user_w) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "topk_idx and topk_w must both be given");
  } else if (!router_w) {
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "router_w is NULL");
  }
  const bool quant = D.weight_dtype == COLIBRI_I8 || D.weight_dtype == COLIBRI_I4;
  if (quant != (expert_scales != nullptr))
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "expert_scales must be given exactly when weights are int8 or int4");
  if ((D.shared_d_ff > 0) != (shared_w != nullptr))
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "shared_w must be given exactly when shared_d_ff > 0");
  const void* ptrs[] = {x, router_w, router_b, expert_w, expert_scales, shared_w, y, user_idx, user_w};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(ctx, COLIBRI_ERR_ALIGNMENT, "pointer %p is not 16-byte aligned", p);
  ctx->last_T = T;
  if (T == 0) return COLIBRI_OK;

  DeviceGuard guard(D.device_id);
  const int dev = D.device_id;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_ptr);
  const void* dev_only[] = {router_w, router_b, expert_w, expert_scales, shared_w, user_idx, user_w};
  for (const void* p : dev_only)
    if (p && classify(p, dev) != kPtrDevice)
      return fail(ctx, COLIBRI_ERR_INVALID_ARG, "pointer %p is not device memory of device %d", p, dev);
  const PtrKind xk = classify(x, dev), yk = classify(y, dev);
  if (xk == kPtrBad || yk == kPtrBad)
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "x or y is device memory of another device");
  if ((xk == kPtrHost || yk == kPtrHost) && ctx->staged && !ctx->profile && !stream_capturing(s))
    return forward_staged(ctx, x, xk, T, router_w, router_b, user_idx, user_w, expert_w, expert_scales, shared_w, y,
                          yk, s);
  return forward_device(ctx, x, xk, T, router_w, router_b, user_idx, user_w, expert_w, expert_scales, shared_w, y,
                        yk, s);
}

// The forward once x and y are classified: a replayed graph when possible, else the launches.
colibri_status forward_device(colibri_ctx* ctx, const void* x, PtrKind xk, int32_t T, const void* router_w,
                              const float* router_b, const int32_t* user_idx, const float* user_w,
                              const void* expert_w, const float* expert_scales, const void* shared_w, void* y,
                              PtrKind yk, cudaStream_t s) {
  const colibri_desc& D = ctx->desc;
  // bf16 weights: the tiling of the expert GEMMs (see gemm_mode)
  const int gemm = D.weight_dtype == COLIBRI_BF16 ? gemm_mode(T * D.top_k / D.num_experts) : kGemmOne;

  // Stage events of colibri_profile_begin: the events of this call, if it is still recorded.
  const bool prof_rec = ctx->prof_on && ctx->prof_n < ctx->prof_max;
  cudaEvent_t* call_ev = prof_rec ? &ctx->prof_ev[(size_t)ctx->prof_n * 6] : nullptr;
  if (prof_rec) ctx->prof_n++;

  // Replay a captured CUDA graph of this exact call when possible: device x and y, a stream
  // other than the legacy default stream that is not itself being captured, and no COLIBRI_PROFILE
  // printing.  While stage events are recorded a second graph of the same call is used whose
  // event-record nodes sit at the stage boundaries; before each replay they are pointed at that
  // call's events, so the recorded stages are those of the replayed graph.
  const bool graphable = ctx->use_graphs && reinterpret_cast<uintptr_t>(s) > 2 && xk == kPtrDevice &&
                         yk == kPtrDevice && !ctx->profile && (!prof_rec || ctx->cap_ev[0] != nullptr);
  if (graphable) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
      cudaGetLastError();
      cs = cudaStreamCaptureStatusActive;
    }
    if (cs == cudaStreamCaptureStatusNone) {
      const uintptr_t key[14] = {(uintptr_t)x,        (uintptr_t)T,        (uintptr_t)router_w, (uintptr_t)router_b,
                                 (uintptr_t)user_idx, (uintptr_t)user_w,   (uintptr_t)expert_w, (uintptr_t)expert_scales,
                                 (uintptr_t)shared_w, (uintptr_t)y,        (uintptr_t)s,        (uintptr_t)gemm,
                                 (uintptr_t)prof_rec, 0};
      // points the stage-event nodes of a timed graph at this call's events, then launches it
      auto replay = [&](colibri_ctx::GraphEntry& g) -> colibri_status {
        if (prof_rec)
          for (int i = 0; i < 6; ++i)
            COLIBRI_TRY(cudaGraphExecEventRecordNodeSetEvent(g.exec, g.ev_node[i], call_ev[i]), "set stage event");
        g.last_use = ++ctx->graph_clock;
        COLIBRI_TRY(cudaGraphLaunch(g.exec, s), "graph launch");
        return COLIBRI_OK;
      };
      for (auto& g : ctx->graphs)
        if (memcmp(g.key, key, sizeof(key)) == 0) return replay(g);
      COLIBRI_TRY(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal), "begin capture");
      const colibri_status st = enqueue_forward(ctx, x, xk, T, router_w, router_b, user_idx, user_w, expert_w,
                                                expert_scales, shared_w, y, yk, s, gemm,
                                                prof_rec ? ctx->cap_ev : nullptr, prof_rec);
      cudaGraph_t graph = nullptr;
      const cudaError_t ce = cudaStreamEndCapture(s, &graph);
      if (st != COLIBRI_OK) {
        if (graph) cudaGraphDestroy(graph);
        cudaGetLastError();
        return st;
      }
      if (ce != cudaSuccess) return check_launch(ctx, ce, "end capture");
      colibri_ctx::GraphEntry ge;
      memcpy(ge.key, key, sizeof(key));
      if (prof_rec) {
        // find the event-record node of each stage boundary by the event it was captured with
        size_t n = 0;
        cudaError_t ne = cudaGraphGetNodes(graph, nullptr, &n);
        std::vector<cudaGraphNode_t> nodes(n);
        if (ne == cudaSuccess && n) ne = cudaGraphGetNodes(graph, nodes.data(), &n);
        for (size_t j = 0; ne == cudaSuccess && j < n; ++j) {
          cudaGraphNodeType t;
          ne = cudaGraphNodeGetType(nodes[j], &t);
          if (ne != cudaSuccess || t != cudaGraphNodeTypeEventRecord) continue;
          cudaEvent_t ev = nullptr;
          ne = cudaGraphEventRecordNodeGetEvent(nodes[j], &ev);
          for (int i = 0; ne == cudaSuccess && i < 6; ++i)
            if (ev == ctx->cap_ev[i]) ge.ev_node[i] = nodes[j];
        }
        bool found = ne == cudaSuccess;
        for (int i = 0; i < 6; ++i) found = found && ge.ev_node[i] != nullptr;
        if (!found) {
          cudaGraphDestroy(graph);
          cudaGetLastError();
          return fail(ctx, COLIBRI_ERR_CUDA, "stage-event nodes not found in the captured forward");
        }
      }
      cudaGraphExec_t exec = nullptr;
      const cudaError_t ie = cudaGraphInstantiate(&exec, graph, 0);
      if (ie != cudaSuccess || !prof_rec) cudaGraphDestroy(graph);
      if (ie != cudaSuccess) return check_launch(ctx, ie, "graph instantiate");
      if (ctx->graphs.size() >= kMaxGraphs) {
        size_t lru = 0;
        for (size_t i = 1; i < ctx->graphs.size(); ++i)
          if (ctx->graphs[i].last_use < ctx->graphs[lru].last_use) lru = i;
        cudaGraphExecDestroy(ctx->graphs[lru].exec);
        if (ctx->graphs[lru].graph) cudaGraphDestroy(ctx->graphs[lru].graph);
        ctx->graphs.erase(ctx->graphs.begin() + lru);
      }
      ge.exec = exec;
      ge.graph = prof_rec ? graph : nullptr;
      ctx->graphs.push_back(ge);
      return replay(ctx->graphs.back());
    }
  }
  return enqueue_forward(ctx, x, xk, T, router_w, router_b, user_idx, user_w, expert_w, expert_scales, shared_w, y,
                         yk, s, gemm, call_ev, false);
}

}  // namespace

extern "C" {

colibri_status colibri_moe_forward(colibri_ctx* ctx, const void* x, int32_t T, const void* router_w,
                                   const float* router_b, const void* expert_w,
                                   const float* expert_scales, const void* shared_w, void* y,
                                   void* stream) {
  return forward_impl(ctx, x, T, router_w, router_b, nullptr, nullptr, expert_w, expert_scales, shared_w, y,
                      stream);
}

colibri_status colibri_moe_forward_routed(colibri_ctx* ctx, const void* x, int32_t T,
                                          const int32_t* topk_idx, const float* topk_w,
                                          const void* expert_w, const float* expert_scales,
                                          const void* shared_w, void* y, void* stream) {
  if (!topk_idx || !topk_w) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "topk_idx and topk_w must be non-NULL");
  return forward_impl(ctx, x, T, nullptr, nullptr, topk_idx, topk_w, expert_w, expert_scales, shared_w, y,
                      stream);
}

colibri_status colibri_get_routing(colibri_ctx* ctx, int32_t* topk_idx, float* topk_w, int32_t* counts,
                                   int32_t* offsets, int32_t* src_row, int32_t* dst_row, void* stream) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  if (ctx->last_T < 0) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "no forward has run on this context");
  const int T = ctx->last_T, k = ctx->desc.top_k, E = ctx->desc.num_experts;
  if (T == 0) return COLIBRI_OK;
  DeviceGuard guard(ctx->desc.device_id);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Workspace& w = ctx->ws;
  struct Copy {
    void* dst;
    const void* src;
    size_t bytes;
  } copies[] = {{topk_idx, w.topk_idx, (size_t)T * k * 4}, {topk_w, w.topk_w, (size_t)T * k * 4},
                {counts, w.counts, (size_t)E * 4},          {offsets, w.offsets, (size_t)(E + 1) * 4},
                {src_row, w.src_row, (size_t)T * k * 4},    {dst_row, w.dst_row, (size_t)T * k * 4}};
  for (const Copy& c : copies)
    if (c.dst) COLIBRI_TRY(cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDefault, s), "copy routing state");
  return COLIBRI_OK;
}

colibri_status colibri_combine(const void* Yp, int32_t act_dtype, const int32_t* dst_row, const float* topk_w,
                               int32_t T, int32_t top_k, int32_t d_model, void* y, void* stream) {
  if (act_dtype != COLIBRI_F32 && act_dtype != COLIBRI_BF16)
    return fail(nullptr, COLIBRI_ERR_UNSUPPORTED, "act_dtype must be COLIBRI_F32 or COLIBRI_BF16");
  if (T < 0 || top_k < 1 || top_k > kMaxTopK || d_model < 8 || d_model % 8 != 0)
    return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "T >= 0, 1 <= top_k <= 8 and d_model a positive multiple of 8");
  if (T == 0) return COLIBRI_OK;
  if (!Yp || !dst_row || !topk_w || !y) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "NULL buffer");
  const void* ptrs[] = {Yp, dst_row, topk_w, y};
  for (const void* p : ptrs)
    if (!aligned16(p)) return fail(nullptr, COLIBRI_ERR_ALIGNMENT, "every buffer must be 16-byte aligned");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, COLIBRI_ERR_CUDA, "cudaGetDevice failed");
  }
  for (const void* p : ptrs)
    if (classify(p, dev) != kPtrDevice)
      return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "every buffer must be device memory of the current device");
  const cudaError_t e = launch_combine(Yp, act_dtype, dst_row, topk_w, T, top_k, d_model, nullptr, y, act_dtype,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(nullptr, COLIBRI_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  }
  return COLIBRI_OK;
}

colibri_status colibri_sync_status(colibri_ctx* ctx, void* stream) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  DeviceGuard guard(ctx->desc.device_id);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  COLIBRI_TRY(cudaStreamSynchronize(s), "stream synchronize");
  uint32_t err = 0;
  COLIBRI_TRY(cudaMemcpy(&err, ctx->ws.err, 4, cudaMemcpyDeviceToHost), "read error word");
  if (err) {
    COLIBRI_TRY(cudaMemset(ctx->ws.err, 0, 4), "clear error word");
    // a wait that gave up may leave the fused kernel's grid-barrier counters out of step
    if (ctx->ws.grid_bar)
      COLIBRI_TRY(cudaMemset(ctx->ws.grid_bar, 0, kFusedBarCount * 4), "reset grid-barrier counters");
    COLIBRI_TRY(cudaMemset(ctx->ws.tile_sched, 0, 4 * 4), "reset tile counters");
    return fail(ctx, COLIBRI_ERR_TIMEOUT, "device error word 0x%x (a bounded wait gave up)", err);
  }
  return COLIBRI_OK;
}

colibri_status colibri_profile_begin(colibri_ctx* ctx, int32_t max_calls) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  if (max_calls < 1 || max_calls > 65536)
    return fail(ctx, COLIBRI_ERR_INVALID_ARG, "max_calls=%d outside [1, 65536]", max_calls);
  DeviceGuard guard(ctx->desc.device_id);
  const size_t need = (size_t)max_calls * 6;
  while (ctx->prof_ev.size() < need) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      return fail(ctx, COLIBRI_ERR_OOM, "cudaEventCreate failed");
    }
    ctx->prof_ev.push_back(e);
  }
  ctx->prof_max = max_calls;
  ctx->prof_n = 0;
  ctx->prof_on = true;
  return COLIBRI_OK;
}

colibri_status colibri_profile_end(colibri_ctx* ctx, float* stage_ms, int32_t* ncalls) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  if (!ctx->prof_on) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "colibri_profile_begin was not called");
  DeviceGuard guard(ctx->desc.device_id);
  ctx->prof_on = false;
  double tot[COLIBRI_NUM_STAGES] = {0, 0, 0, 0, 0};
  for (int c = 0; c < ctx->prof_n; ++c) {
    cudaEvent_t* ev = &ctx->prof_ev[(size_t)c * 6];
    COLIBRI_TRY(cudaEventSynchronize(ev[5]), "event synchronize");
    for (int i = 0; i < COLIBRI_NUM_STAGES; ++i) {
      float ms = 0.f;
      COLIBRI_TRY(cudaEventElapsedTime(&ms, ev[i], ev[i + 1]), "event elapsed time");
      tot[i] += ms;
    }
  }
  if (stage_ms)
    for (int i = 0; i < COLIBRI_NUM_STAGES; ++i) stage_ms[i] = (float)tot[i];
  if (ncalls) *ncalls = ctx->prof_n;
  return COLIBRI_OK;
}

colibri_status colibri_profile_calls(colibri_ctx* ctx, float* call_stage_ms, int32_t max_calls) {
  if (!ctx) return fail(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  if (ctx->prof_on) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "colibri_profile_end was not called");
  if (!call_stage_ms || max_calls < 0) return fail(ctx, COLIBRI_ERR_INVALID_ARG, "bad output buffer");
  DeviceGuard guard(ctx->desc.device_id);
  const int n = std::min(max_calls, ctx->prof_n);
  for (int c = 0; c < n; ++c) {
    cudaEvent_t* ev = &ctx->prof_ev[(size_t)c * 6];
    COLIBRI_TRY(cudaEventSynchronize(ev[5]), "event synchronize");
    for (int i = 0; i < COLIBRI_NUM_STAGES; ++i) {
      float ms = 0.f;
      COLIBRI_TRY(cudaEventElapsedTime(&ms, ev[i], ev[i + 1]), "event elapsed time");
      call_stage_ms[(size_t)c * COLIBRI_NUM_STAGES + i] = ms;
    }
  }
  return COLIBRI_OK;
}

}  // extern "C"
