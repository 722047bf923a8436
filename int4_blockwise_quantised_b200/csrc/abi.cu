// Library-wide entry points: version, error text, device error word.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "vv_device.cuh"
#include "vv_internal.h"

namespace vv {

__device__ int g_device_error = 0;

namespace {
thread_local vv_status t_last_code = VV_OK;
thread_local char t_last_text[512] = "";
}  // namespace

vv_status set_error(vv_status code, const char* fmt, ...) {
  t_last_code = code;
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_text, sizeof(t_last_text), fmt, ap);
  va_end(ap);
  return code;
}

vv_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return VV_OK;
  return set_error(VV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

namespace {
// Self-test of the bounded waits: one CTA waits, through the same helpers the kernels use, on a
// signal that never comes (an mbarrier nobody arrives at; a counter nobody increments).
__global__ void wait_selftest_kernel(int which, uint64_t limit_ns, unsigned* counter) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  if (which == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0, limit_ns);
  } else {
    wait_counter_geq(counter, 1u, limit_ns);
  }
}
}  // namespace

}  // namespace vv

extern "C" {

const char* vv_version(void) { return "libvv 0.1 (sm_100a)"; }

vv_status vv_last_error(char* buf, size_t n) {
  if (buf && n) {
    strncpy(buf, vv::t_last_text, n - 1);
    buf[n - 1] = '\0';
  }
  return vv::t_last_code;
}

vv_status vv_wait_selftest(int32_t which, int64_t limit_ns, void* scratch, vv_stream stream) {
  VV_CHECK_ARG(which == 0 || which == 1, "vv_wait_selftest: which %d (0 or 1)", which);
  VV_CHECK_ARG(limit_ns >= 1000 && limit_ns <= 100000000, "vv_wait_selftest: limit %lld ns",
               (long long)limit_ns);
  VV_CHECK_ARG(which == 0 || (scratch && vv::aligned16(scratch)),
               "vv_wait_selftest: counter scratch null or misaligned");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (which == 1) VV_CUDA(cudaMemsetAsync(scratch, 0, 16, s));
  vv::wait_selftest_kernel<<<1, 32, 0, s>>>(which, (uint64_t)limit_ns,
                                            static_cast<unsigned*>(scratch));
  VV_CUDA(cudaGetLastError());
  return VV_OK;
}

vv_status vv_sync_status(vv_stream stream) {
  VV_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int err = 0;
  VV_CUDA(cudaMemcpyFromSymbol(&err, vv::g_device_error, sizeof(int)));
  if (err != 0) {
    const int zero = 0;
    VV_CUDA(cudaMemcpyToSymbol(vv::g_device_error, &zero, sizeof(int)));
    return vv::set_error(err, "device-side error %d recorded by a kernel", err);
  }
  return VV_OK;
}

}  // extern "C"
