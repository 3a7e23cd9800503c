// gsq_pool.cu -- the library's device memory.  Every buffer of a context
// (layer, block stage, K-Quant), the init-time staging and the GPTQ
// workspace come from one memory pool per device that the library owns.  The
// pool keeps freed memory reserved (all of it by default, or up to the limit
// gsq_set_cached_memory_limit sets), so that the next context or call of a
// similar size maps no new pages: mapping device memory costs tens of
// milliseconds per GB here, as much as hundreds of reconstruction steps of a
// layer, and a block's MLP stage alone takes about 45 GB.
// gsq_release_cached_memory hands the reserve back to the driver.
//
// pool_malloc has cudaMalloc's contract (the memory may be used on any stream
// once it returns): it allocates on a private stream of the device and
// waits for that stream.  pool_free has cudaFree's (nothing in flight still
// uses the memory): it frees on the same private stream, so a later
// pool_malloc reuses the memory in stream order.
#include <atomic>
#include <mutex>

#include "../../include/gsq.h"
#include "gsq_internal.h"

namespace gsq {

namespace {

constexpr int kMaxDevices = 64;

std::mutex g_mu;
uint64_t g_keep = ~0ull;  // release threshold of every pool
// test hook: allocations left before one fails (negative: none fails)
std::atomic<int64_t> g_fail_after{-1};
cudaMemPool_t g_pool[kMaxDevices] = {};
cudaStream_t g_stream[kMaxDevices] = {};

// pool and private stream of device dev (created on first use); false when
// either cannot be created
bool device_pool(int dev, cudaMemPool_t* pool, cudaStream_t* stream) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    uint64_t keep = g_keep;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    cudaGetLastError();
    g_pool[dev] = p;
  }
  if (!g_stream[dev]) {
    int cur = 0;
    if (cudaGetDevice(&cur) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    cudaStream_t s = nullptr;
    const bool switched = cur != dev && cudaSetDevice(dev) == cudaSuccess;
    const cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    if (switched) cudaSetDevice(cur);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    g_stream[dev] = s;
  }
  *pool = g_pool[dev];
  *stream = g_stream[dev];
  return true;
}

}  // namespace

bool pool_fail_injected() {
  int64_t n = g_fail_after.load();
  while (n >= 0) {
    if (g_fail_after.compare_exchange_weak(n, n - 1)) return n == 0;
  }
  return false;
}

cudaMemPool_t library_pool(int dev) {
  cudaMemPool_t p = nullptr;
  cudaStream_t s = nullptr;
  return device_pool(dev, &p, &s) ? p : nullptr;
}

cudaError_t pool_malloc(void** p, size_t bytes) {
  *p = nullptr;
  if (pool_fail_injected()) return cudaErrorMemoryAllocation;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  cudaMemPool_t pool = nullptr;
  cudaStream_t s = nullptr;
  if (!device_pool(dev, &pool, &s)) return cudaErrorMemoryAllocation;
  e = cudaMallocFromPoolAsync(p, bytes, pool, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    if (*p) cudaFreeAsync(*p, s);
    *p = nullptr;
  }
  return e;
}

void pool_free(void* p) {
  if (!p) return;
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  cudaMemPool_t pool = nullptr;
  cudaStream_t s = nullptr;
  if (device_pool(at.device, &pool, &s)) cudaFreeAsync(p, s);
  cudaGetLastError();
}

}  // namespace gsq

extern "C" {

int gsq_set_cached_memory_limit(uint64_t bytes) {
  using namespace gsq;
  std::lock_guard<std::mutex> lk(g_mu);
  g_keep = bytes;
  int rc = GSQ_OK;
  for (int d = 0; d < kMaxDevices; ++d) {
    if (!g_pool[d]) continue;
    uint64_t keep = bytes;
    if (cudaMemPoolSetAttribute(g_pool[d], cudaMemPoolAttrReleaseThreshold, &keep) !=
        cudaSuccess) {
      cudaGetLastError();
      rc = GSQ_ERR_CUDA;
    }
  }
  return rc;
}

int gsq_debug_fail_alloc(int64_t after) {
  gsq::g_fail_after.store(after < 0 ? -1 : after);
  return GSQ_OK;
}

int gsq_debug_pool_used(int device, uint64_t* bytes) {
  using namespace gsq;
  if (!bytes || device < 0 || device >= kMaxDevices) return GSQ_ERR_INVALID_ARG;
  *bytes = 0;
  cudaMemPool_t pool = nullptr;
  cudaStream_t s = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    pool = g_pool[device];
    s = g_stream[device];
  }
  if (!pool) return GSQ_OK;  // nothing allocated on that device yet
  uint64_t used = 0;
  // frees queued on the private stream are done before the count is read
  if ((s && cudaStreamSynchronize(s) != cudaSuccess) ||
      cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &used) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  *bytes = used;
  return GSQ_OK;
}

int gsq_release_cached_memory(void) {
  using namespace gsq;
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = GSQ_OK;
  for (int d = 0; d < kMaxDevices; ++d) {
    if (!g_pool[d]) continue;
    // the frees queued on the private stream are done before the trim
    if ((g_stream[d] && cudaStreamSynchronize(g_stream[d]) != cudaSuccess) ||
        cudaMemPoolTrimTo(g_pool[d], 0) != cudaSuccess) {
      cudaGetLastError();
      rc = GSQ_ERR_CUDA;
    }
  }
  return rc;
}

}  // extern "C"
