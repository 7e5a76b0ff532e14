// Test probe of the library's bounded on-chip waits (not part of libqlin.so).
//
// One CTA allocates tensor memory, initialises one mbarrier that nothing ever
// arrives on (no TMA, bulk copy or MMA is in flight) and waits on it with the
// library's own bounded wait.  The wait must run out after the library's wait
// limit, store QLIN_ERR_TIMEOUT into the caller's status word through the
// library's own reporting helper, release the tensor memory and return, so
// that the CUDA context stays usable for the calls that follow.
#include "qlin_internal.cuh"

namespace {

__global__ void __launch_bounds__(128, 1) never_arrived_kernel(int32_t* dev_status,
                                                               unsigned long long* out) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    qlin::mbar_init(&bar, 1);
    qlin::fence_barrier_init();
  }
  if (warp == 0) {
    qlin::tmem_alloc(&tmem_slot, 32);
    qlin::tmem_relinquish();
  }
  qlin::tc_fence_before();
  __syncthreads();
  qlin::tc_fence_after();
  const unsigned long long t0 = qlin::global_ns();
  bool ok = true;
  if (threadIdx.x == 0) {
    ok = qlin::mbar_wait(&bar, 0);  // phase 0 never completes
    if (!ok) qlin::report_timeout(dev_status);
    out[0] = ok ? 1ull : 2ull;
    out[1] = qlin::global_ns() - t0;
  }
  qlin::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    qlin::tc_fence_after();
    qlin::tmem_dealloc(tmem_slot, 32);
  }
}

}  // namespace

// out: two u64 words on the device -- [0] 2 if the wait ran out (1 if it
// completed), [1] nanoseconds the wait took.  Returns a cudaError_t.
extern "C" __attribute__((visibility("default"))) int probe_never_arrived(int32_t* dev_status,
                                                                          void* out, void* stream) {
  never_arrived_kernel<<<1, 128, 0, (cudaStream_t)stream>>>(dev_status, (unsigned long long*)out);
  return (int)cudaGetLastError();
}

// The library's wait limit in nanoseconds (what the test expects the wait to take).
extern "C" __attribute__((visibility("default"))) unsigned long long probe_wait_limit_ns() {
  return qlin::kWaitLimitNs;
}
