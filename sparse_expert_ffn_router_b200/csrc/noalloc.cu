// colibri_route_noalloc: the Gate and Scatter stages (router logits, softmax, top-k, per-expert
// histogram, prefix sum, stable grouping of token rows) without a context and without any
// device allocation.
//
// Who needs it: callers that cannot call cudaMalloc -- for example an engine whose device memory
// is entirely reserved up front by its own allocator (weights, KV cache and activation pools),
// where an extra cudaMalloc would fail or fragment that reservation, or a latency-critical loop
// that must not pay cudaMalloc's implicit device synchronisation.  They pass every input and
// output buffer themselves; the only scratch this call needs (per-block expert counts and their
// prefix bases) lives in the file-scope array below.
//
// The scratch array is a static __device__ object: every GPU that loads this library holds its
// 257 KB until the process exits.  Host code may not use its name as an address (on the host the
// name is only a stand-in), so every call looks up the device address with cudaGetSymbolAddress,
// with the caller's device current, and raises the router kernels' shared-memory limit there
// (both cheap once the module is loaded, and both stay right if the context is torn down and
// re-created).  The first call on each device loads the module and should come before any stream
// capture.  Every call shares the array and it keeps the last call's contents: every entry a call
// reads is written by that call first, and the error word the tensor-core router sets when a
// bounded wait gives up is cleared at the start of each call (a stream-ordered memset, not an
// allocation); colibri_route_noalloc_check reads it.  Calls that overlap on the GPU (two streams,
// or two host threads) race on the array.
#include "common.cuh"

namespace colibri {
void record_error(const char* msg);
}

using namespace colibri;

namespace {

constexpr int kNoAllocMaxBlockExperts = 32768;  // ceil(T / 256) * num_experts
// block counts | block bases | m-tile prefix [E+1] | device error word
constexpr size_t kErrWordOffset = 2 * (size_t)kNoAllocMaxBlockExperts + (kMaxExperts + 1);
constexpr size_t kScratchInts = kErrWordOffset + 1;

static __device__ __align__(256) int32_t g_route_scratch[kScratchInts];


colibri_status nf_fail(colibri_status st, const char* msg) {
  record_error(msg);
  return st;
}

// Device address of g_route_scratch on the current device, after setting the router kernels'
// shared-memory limits there (both cheap once the module is loaded; done on every call so that
// they stay right if the caller tears the context down and re-creates it).
colibri_status scratch_address(int32_t** out) {
  if (configure_router_kernels() != cudaSuccess) {
    cudaGetLastError();
    return nf_fail(COLIBRI_ERR_CUDA, "router kernel configuration failed");
  }
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
  if (e != cudaSuccess || !p) {
    cudaGetLastError();
    return nf_fail(COLIBRI_ERR_CUDA, "cudaGetSymbolAddress of the routing scratch array failed");
  }
  *out = static_cast<int32_t*>(p);
  return COLIBRI_OK;
}

bool is_device_ptr(const void* p, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (at.type == cudaMemoryTypeDevice && at.device == dev) || at.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" colibri_status colibri_route_noalloc(const void* x, int32_t act_dtype, int32_t T,
                                                int32_t d_model, const void* router_w,
                                                const float* router_b, int32_t num_experts,
                                                int32_t top_k, int32_t* topk_idx, float* topk_w,
                                                int32_t* counts, int32_t* offsets,
                                                int32_t* src_row, int32_t* dst_row, void* Xp,
                                                void* stream) {
  if (act_dtype != COLIBRI_F32 && act_dtype != COLIBRI_BF16)
    return nf_fail(COLIBRI_ERR_UNSUPPORTED, "act_dtype must be COLIBRI_F32 or COLIBRI_BF16");
  if (d_model < 64 || d_model % 64 != 0)
    return nf_fail(COLIBRI_ERR_INVALID_ARG, "d_model must be a positive multiple of 64");
  if (num_experts < 1 || num_experts > kMaxExperts)
    return nf_fail(COLIBRI_ERR_INVALID_ARG, "num_experts must be in [1, 256]");
  if (top_k < 1 || top_k > kMaxTopK || top_k > num_experts)
    return nf_fail(COLIBRI_ERR_INVALID_ARG, "top_k must be in [1, min(num_experts, 8)]");
  if (T < 0) return nf_fail(COLIBRI_ERR_INVALID_ARG, "T must be >= 0");
  const int64_t nblk = ((int64_t)T + kCountBlock - 1) / kCountBlock;
  if (nblk * num_experts > kNoAllocMaxBlockExperts)
    return nf_fail(COLIBRI_ERR_INVALID_ARG,
                   "ceil(T / 256) * num_experts exceeds 32768, the size of the built-in scratch array");
  if (T == 0) return COLIBRI_OK;
  const void* ptrs[] = {x, router_w, topk_idx, topk_w, counts, offsets, src_row, dst_row, Xp};
  for (const void* p : ptrs)
    if (!p) return nf_fail(COLIBRI_ERR_INVALID_ARG, "every buffer except router_b must be non-NULL");
  const void* all[] = {x, router_w, router_b, topk_idx, topk_w, counts, offsets, src_row, dst_row, Xp};
  for (const void* p : all)
    if (p && (reinterpret_cast<uintptr_t>(p) & 15u))
      return nf_fail(COLIBRI_ERR_ALIGNMENT, "every buffer must be 16-byte aligned");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return nf_fail(COLIBRI_ERR_CUDA, "cudaGetDevice failed");
  }
  for (const void* p : all)
    if (p && !is_device_ptr(p, dev))
      return nf_fail(COLIBRI_ERR_INVALID_ARG, "every buffer must be device memory of the current device");
  int32_t* scratch = nullptr;
  const colibri_status st = scratch_address(&scratch);
  if (st != COLIBRI_OK) return st;
  int32_t* blk_counts = scratch;
  int32_t* blk_base = scratch + kNoAllocMaxBlockExperts;
  int32_t* mt_prefix = scratch + 2 * kNoAllocMaxBlockExperts;
  uint32_t* err = reinterpret_cast<uint32_t*>(scratch + kErrWordOffset);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess)
    e = launch_router_topk(x, act_dtype, T, d_model, router_w, router_b, num_experts, top_k, 0, topk_idx, topk_w,
                           err, s);
  if (e == cudaSuccess) e = launch_route_count(topk_idx, T, top_k, num_experts, blk_counts, dst_row, s);
  if (e == cudaSuccess)
    e = launch_route_scan(blk_counts, (int)nblk, num_experts, kTcBM, blk_base, counts, offsets, mt_prefix, s);
  if (e == cudaSuccess)
    e = launch_route_scatter(x, act_dtype, T, d_model, top_k, num_experts, topk_idx, blk_base, offsets, dst_row,
                             src_row, Xp, nullptr, s);
  if (e != cudaSuccess) return nf_fail(COLIBRI_ERR_CUDA, cudaGetErrorString(e));
  return COLIBRI_OK;
}

extern "C" colibri_status colibri_route_noalloc_check(void* stream) {
  int32_t* scratch = nullptr;
  const colibri_status st = scratch_address(&scratch);
  if (st != COLIBRI_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return nf_fail(COLIBRI_ERR_CUDA, "stream synchronize failed");
  }
  uint32_t word = 0;
  if (cudaMemcpy(&word, scratch + kErrWordOffset, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return nf_fail(COLIBRI_ERR_CUDA, "reading the error word failed");
  }
  if (word) return nf_fail(COLIBRI_ERR_TIMEOUT, "a bounded device wait of colibri_route_noalloc gave up");
  return COLIBRI_OK;
}
