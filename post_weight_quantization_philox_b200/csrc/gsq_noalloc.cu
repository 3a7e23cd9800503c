// gsq_noalloc.cu -- gsq_uniforms_noalloc: the step's Philox uniforms without
// any device allocation.
//
// Some callers cannot call cudaMalloc: a process whose device memory is
// fully reserved by another allocator (a caching allocator or a fixed pool
// that owns the whole budget), or code that runs inside a framework that
// forbids device allocation on its execution path.  They still may want to
// reproduce or audit the noise a GSQ step draws.  This entry point runs the
// same uniform-generation kernel as gsq_debug_uniforms, but its device
// staging buffer is the file-scope array below instead of memory obtained
// from cudaMalloc.  The array lives on every GPU that loads the library
// until the process exits.
#include <mutex>

#include "../../include/gsq.h"
#include "gsq_internal.h"

namespace {

// Five uniforms per coordinate at most (3-bit local shift).
constexpr int64_t kScratchFloats = (int64_t)GSQ_NOALLOC_MAX_COORDS * 5;

static __device__ __align__(256) float g_uniform_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
float* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The calling thread's current driver context (null if it cannot be read).
CUcontext current_context() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<CtxGetCurrentFn>(p);
    return (CtxGetCurrentFn) nullptr;
  }();
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in, so the address comes from
// cudaGetSymbolAddress, with that device current: once per device, and again
// whenever the device's context is no longer the one the address was taken
// in (after cudaDeviceReset the old address is gone).
int scratch_address(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return GSQ_ERR_UNSUPPORTED;
  // null until the runtime has made the device's context current; the
  // lookup below does that, and the context is read again after it
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_uniform_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return GSQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
    g_scratch_ctx[dev] = ctx ? ctx : current_context();
  }
  *out = g_scratch_ptr[dev];
  return GSQ_OK;
}

}  // namespace

extern "C" GSQ_API int gsq_uniforms_noalloc(int grid_mode, uint64_t seed,
                                            uint32_t t, uint64_t coord0,
                                            int64_t count, float* out,
                                            void* stream) {
  if (!out || count <= 0 || grid_mode < GSQ_GRID_2BIT ||
      grid_mode > GSQ_GRID_3BIT_LOCAL)
    return GSQ_ERR_INVALID_ARG;
  if (count > GSQ_NOALLOC_MAX_COORDS) return GSQ_ERR_INVALID_ARG;
  float* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != GSQ_OK) return rc;
  const int L = grid_mode == GSQ_GRID_3BIT_LOCAL ? 5 : 4;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The kernel writes every one of the count * L entries that are copied
  // out, so nothing in the scratch has to start at zero.
  cudaError_t e = gsq::launch_uniforms(grid_mode, seed, t, coord0, count,
                                       scratch, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out, scratch, (size_t)count * L * sizeof(float),
                        cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  return GSQ_OK;
}
