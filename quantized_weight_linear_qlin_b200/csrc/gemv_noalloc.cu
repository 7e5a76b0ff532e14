// qlin_gemv_noalloc: qlin_gemv with its scratch in a fixed device array that
// lives inside this library, for callers that cannot hand it a workspace.
//
// Who cannot allocate: a caller whose device memory is planned once at start-up
// and must not grow afterwards (a serving engine with a fixed memory budget, or
// plain C code that owns only the weights, x and y buffers), and a caller that
// would otherwise have to allocate while work is being recorded for replay.
// qlin_gemv needs a caller-provided workspace (split-tile counters and FP32
// partial sums, or the FP32 accumulator of the CUDA-core kernel); this entry
// point supplies one from a file-scope __device__ array instead.
//
// First call per device: resolves the array's device address with
// cudaGetSymbolAddress (this may load the module on that device) and zero-fills
// the array with a synchronous cudaMemset.  Make that first call before any
// stream capture and outside any latency-critical section.  Later calls only
// enqueue a cudaMemsetAsync of the split-tile counters and the kernel(s).
//
// The array is shared by every call on a device: calls that may overlap in time
// (different streams, different host threads without ordering) race on it and
// must be serialized by the caller.
#include <atomic>
#include <mutex>

#include "qlin_internal.cuh"

namespace qlin {
namespace {

constexpr size_t kNoAllocBytes = (size_t)16 << 20;  // 16 MiB per device
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's array (the device must be current); null on failure.
void* scratch_for(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = g_scratch[dev].load(std::memory_order_acquire);
  if (p) return p;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  p = g_scratch[dev].load(std::memory_order_relaxed);
  if (p) return p;
  void* q = nullptr;
  if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || q == nullptr) return nullptr;
  if (cudaMemset(q, 0, kNoAllocBytes) != cudaSuccess) return nullptr;
  g_scratch[dev].store(q, std::memory_order_release);
  return q;
}

}  // namespace
}  // namespace qlin

extern "C" QLIN_API int qlin_gemv_noalloc(const qlin_weights* w, const uint16_t* x_bf16, int64_t t,
                                          void* y, int y_dtype, void* stream, int32_t* dev_status) {
  // every argument check of qlin_gemv first: a rejected call enqueues nothing
  int rc = qlin::check_gemv_args(w, x_bf16, t, y, y_dtype);
  if (rc != QLIN_OK) return rc;
  size_t need = 0;
  rc = qlin_gemv_workspace_bytes(w, t, &need);
  if (rc != QLIN_OK) return rc;
  if (need > qlin::kNoAllocBytes) return QLIN_ERR_WORKSPACE;  // larger than the fixed array
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLIN_ERR_CUDA;
  void* scratch = qlin::scratch_for(dev);
  if (scratch == nullptr) return QLIN_ERR_CUDA;
  // split-tile counters must read zero when the kernel starts; a call whose
  // on-chip wait timed out may have left some set, so clear them every call
  const int64_t tiles = (w->n + 127) / 128;
  const size_t counters = ((size_t)tiles * sizeof(int) + 255) / 256 * 256;
  if (need > 0 && cudaMemsetAsync(scratch, 0, counters < need ? counters : need, (cudaStream_t)stream) != cudaSuccess)
    return QLIN_ERR_CUDA;
  qlin_exec ex;
  ex.stream = stream;
  ex.dev_status = dev_status;
  ex.workspace = need > 0 ? scratch : nullptr;
  ex.workspace_bytes = need > 0 ? qlin::kNoAllocBytes : 0;
  return qlin_gemv(w, x_bf16, t, y, y_dtype, &ex);
}
