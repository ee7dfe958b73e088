// colibri_selftest_wait_timeout: exercises the failure-detection path without any fault.
//
// Every pipeline wait of the library's kernels (TMA/MMA mbarrier waits) is bounded; a wait that
// gives up sets a bit in the context's device error word and its kernel returns, and
// colibri_sync_status later reports COLIBRI_ERR_TIMEOUT (the error reporting of
// www.mhpq.cn/news/563172 §4.3).  This call launches one CTA whose single thread waits on an
// mbarrier that nothing ever arrives on, with the caller's limit instead of the pipelines' 4 s,
// so that path can be tested: the wait runs out, the error word is set, nothing faults or hangs
// and the context stays usable.
#include "common.cuh"

namespace colibri {
colibri_status report(colibri_ctx* ctx, colibri_status st, const char* msg);
}

using namespace colibri;

namespace {

__global__ void selftest_wait_kernel(uint32_t* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_fence_init();
  const unsigned long long t0 = global_ns();
  bool completed = false;
  while (true) {
    if (mbar_try_wait(&bar, 0)) {  // phase 0 never completes: no thread arrives
      completed = true;
      break;
    }
    if (global_ns() - t0 > limit_ns) break;
  }
  if (!completed) atomicOr(err, kErrWaitTimeout);
}

}  // namespace

extern "C" colibri_status colibri_selftest_wait_timeout(colibri_ctx* ctx, int32_t timeout_us, void* stream) {
  if (!ctx) return report(nullptr, COLIBRI_ERR_INVALID_ARG, "ctx is NULL");
  if (timeout_us < 1 || timeout_us > 1000000)
    return report(ctx, COLIBRI_ERR_INVALID_ARG, "timeout_us outside [1, 1000000]");
  int prev = -1;
  cudaGetDevice(&prev);
  if (prev != ctx->desc.device_id) cudaSetDevice(ctx->desc.device_id);
  const cudaError_t e = launch_kernel(selftest_wait_kernel, dim3(1), dim3(32), 0,
                                      reinterpret_cast<cudaStream_t>(stream), 1, ctx->ws.err,
                                      (unsigned long long)timeout_us * 1000ull);
  if (prev >= 0 && prev != ctx->desc.device_id) cudaSetDevice(prev);
  return e == cudaSuccess ? COLIBRI_OK : report(ctx, COLIBRI_ERR_CUDA, cudaGetErrorString(e));
}
