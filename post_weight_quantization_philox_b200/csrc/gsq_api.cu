// gsq_api.cu -- the C ABI of libgsq (declared in include/gsq.h): context
// life cycle, the step driver and the host side of every entry point.
// Every entry point validates on the host before touching the device, maps
// CUDA failures to status codes and never throws across the ABI.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/gsq.h"
#include "gsq_internal.h"

using namespace gsq;

namespace {

constexpr int kGroup = 128;
constexpr int kLossRing = 4096;
constexpr int kMaxPartials = 1024;
constexpr uint64_t kStateMagic = 0x3130515347ull;  // "GSQ01"

int num_logits(int mode) {
  return mode == GSQ_GRID_3BIT_LOCAL ? 5 : (mode == GSQ_GRID_2BIT || mode == GSQ_GRID_TERNARY) ? 4 : -1;
}

struct Timing {
  cudaEvent_t ev[5];
  bool soft;    // the soft-weight phase launched a kernel in this step
  bool next;    // the backward also built the next step's soft weight
  bool merged;  // one launch ran both GEMMs (timed as the forward phase)
};

}  // namespace

struct gsq_ctx {
  int mode = 0, L = 0, group = kGroup;
  // logits and Lion momenta stored as bf16 (the reduced-memory state); the
  // pointers below keep their float type and the launchers reinterpret them
  int state16 = 0;
  int64_t N = 0, K = 0, T = 0, Tp = 0, G = 0;
  uint64_t seed = 0, t = 0;
  // global coordinate of local coordinate 0 (row0 K for a shard of rows)
  uint64_t coord0 = 0;
  int noise = 1;
  cudaStream_t st = nullptr;
  int dev = 0, sms = 148;
  int failed = 0;  // sticky status (negative) once something went wrong
  int stall_probe = 0;  // test hook: the next forward GEMM runs the probe
  // both GEMMs of a step in one launch (layers with fewer than 24 row tiles):
  // per-band counters of the forward tiles done, and the launch generation
  bool merged = false;
  unsigned* band_done = nullptr;
  uint32_t merge_gen = 0;

  __nv_bfloat16 *Xb = nullptr, *Xt = nullptr, *What = nullptr, *dYt = nullptr;
  float *YrefT = nullptr, *dW = nullptr, *logits = nullptr, *mom = nullptr;
  float *s = nullptr, *ms = nullptr;
  int8_t* i0 = nullptr;
  double *partials = nullptr, *loss_hist = nullptr, *scratch = nullptr;
  unsigned* ticket = nullptr;
  int* err = nullptr;
  float *wsoft32 = nullptr, *dl = nullptr, *ds = nullptr;  // debug, lazy
  // What holds the soft weight of step what_t at temperature what_tau
  // (what_t < 0: nothing precomputed)
  int64_t what_t = -1;
  float what_tau = 0.f;
  // level codes of the hard choice of the current logits (scale-only steps)
  int8_t* hcode = nullptr;
  bool hcode_valid = false;
  double yref_sq = 0.0;
  CUtensorMap tm_What, tm_Xb, tm_dYt, tm_Xt;  // GEMM operands
  EpiMaps em_forward;  // dY^T (bf16) out, Y_ref^T in
  EpiMaps em_wgrad;    // dW (fp32) out
  std::vector<void*> allocs;

  bool timing = false;
  std::vector<Timing> tev;
  size_t tev_used = 0;
};

namespace {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GSQ_OK;
  if (e == cudaErrorMemoryAllocation) return GSQ_ERR_OOM;
  return GSQ_ERR_CUDA;
}

int fail(gsq_ctx* c, int status) {
  if (c && status != GSQ_OK && c->failed == 0) c->failed = status;
  return status;
}

#define CK(call)                                   \
  do {                                             \
    cudaError_t e_ = (call);                       \
    if (e_ != cudaSuccess) return fail(c, cuda_status(e_)); \
  } while (0)

template <typename T>
int dalloc(gsq_ctx* c, T** p, size_t count) {
  void* q = nullptr;
  cudaError_t e = pool_malloc(&q, count * sizeof(T) + 16);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_OOM;
  }
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return GSQ_OK;
}

void free_all(gsq_ctx* c) {
  for (void* p : c->allocs) pool_free(p);
  c->allocs.clear();
  for (auto& te : c->tev)
    for (auto& e : te.ev) cudaEventDestroy(e);
  c->tev.clear();
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

// Reads the device error word (syncs) and turns it into a sticky status.
int check_device(gsq_ctx* c) {
  cudaError_t e = cudaStreamSynchronize(c->st);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  int h = 0;
  e = cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  switch (h) {
    case DEV_OK: return GSQ_OK;
    case DEV_ERR_TIMEOUT: return fail(c, GSQ_ERR_TIMEOUT);
    case DEV_ERR_NONFINITE: return fail(c, GSQ_ERR_NONFINITE);
    case DEV_ERR_BAD_INIT: return fail(c, GSQ_ERR_INVALID_ARG);
    default: return fail(c, GSQ_ERR_CUDA);
  }
}

int usable(gsq_ctx* c) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  return GSQ_OK;
}

StepArgs step_args(gsq_ctx* c, float tau) {
  StepArgs a;
  a.mode = c->mode;
  a.N = c->N;
  a.K = c->K;
  a.G = c->G;
  a.logits = c->logits;
  a.logits_w = c->logits;
  a.mom = c->mom;
  a.s = c->s;
  a.ms = c->ms;
  a.i0 = c->i0;
  a.seed = c->seed;
  a.t = (uint32_t)c->t;
  a.noise = c->noise;
  a.tau = tau;
  a.state16 = c->state16;
  a.coord0 = c->coord0;
  return a;
}

// bytes of one full logit (or momentum) state: L x N x K elements
size_t state_plane_bytes(const gsq_ctx* c) {
  return (size_t)c->L * c->N * c->K * (c->state16 ? 2 : 4);
}

EpiParams forward_params(gsq_ctx* c, double* loss_out) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.partials = c->partials;
  ep.ticket = c->ticket;
  ep.loss_out = loss_out;
  ep.err = c->err;
  return ep;
}

cudaError_t run_forward(gsq_ctx* c, double* loss_out, int epi) {
  EpiParams ep = forward_params(c, loss_out);
  ep.stall_probe = c->stall_probe;
  c->stall_probe = 0;
  return launch_gemm(c->tm_What, c->tm_Xb, c->em_forward, c->N, c->Tp, c->K,
                     epi, ep, c->sms,
                     c->st);
}

// Forward GEMM (loss and dY) and weight-gradient GEMM in one persistent
// launch: a band's weight-gradient tiles start once its forward tiles are done.
cudaError_t run_gemms_merged(gsq_ctx* c, double* loss_out) {
  EpiParams ep = forward_params(c, loss_out);
  ep.stall_probe = c->stall_probe;
  c->stall_probe = 0;
  MergeArgs mg;
  mg.tmA2 = c->tm_dYt;
  mg.tmB2 = c->tm_Xt;
  mg.tmO2 = c->em_wgrad.out;
  mg.N2 = c->K;
  mg.Kc2 = c->Tp;
  mg.band_done = c->band_done;
  c->merge_gen += 1;
  mg.target = c->merge_gen * (unsigned)merged_band_tiles(c->Tp) * 8u;
  return launch_gemm_merged(c->tm_What, c->tm_Xb, c->em_forward, c->N, c->Tp, c->K, mg, ep,
                            c->sms, c->st);
}

cudaError_t run_weight_grad(gsq_ctx* c) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.err = c->err;
  return launch_gemm(c->tm_dYt, c->tm_Xt, c->em_wgrad, c->N, c->K, c->Tp,
                     EPI_STORE_F32, ep,
                     c->sms, c->st);
}

bool step_args_ok(float tau, float lr, float b1, float b2) {
  return tau > 0.f && std::isfinite(tau) && lr >= 0.f && std::isfinite(lr) &&
         b1 >= 0.f && b1 < 1.f && b2 >= 0.f && b2 < 1.f;
}

}  // namespace

extern "C" {

const char* gsq_error_string(int status) {
  switch (status) {
    case GSQ_OK: return "ok";
    case GSQ_ERR_INVALID_ARG: return "invalid argument";
    case GSQ_ERR_CUDA: return "CUDA error";
    case GSQ_ERR_OOM: return "out of device memory";
    case GSQ_ERR_NONFINITE: return "non-finite value";
    case GSQ_ERR_STATE: return "context failed or destroyed";
    case GSQ_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case GSQ_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

int gsq_init_gptq(gsq_ctx** out, const void* W, int w_dtype, const void* X, int x_dtype,
                  int64_t N, int64_t K, int64_t T, int group, int grid_mode, float damp,
                  uint64_t seed, void* stream) {
  if (!out) return GSQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (N <= 0 || K <= 0 || group <= 0 || K % group != 0) return GSQ_ERR_INVALID_ARG;
  int8_t* lev = nullptr;
  float* sc = nullptr;
  if (pool_malloc(&lev, (size_t)N * K) != cudaSuccess ||
      pool_malloc(&sc, (size_t)N * (K / group) * 4) != cudaSuccess) {
    cudaGetLastError();
    pool_free(lev);
    return GSQ_ERR_OOM;
  }
  int rc = gsq_gptq(W, w_dtype, X, x_dtype, N, K, T, group, grid_mode, damp, lev, sc, stream);
  if (!rc) rc = gsq_init(out, W, w_dtype, X, x_dtype, N, K, T, group, grid_mode, lev, seed,
                         stream);
  if (!rc) {
    gsq_ctx* c = *out;
    if (cudaMemcpyAsync(c->s, sc, (size_t)N * c->G * 4, cudaMemcpyDeviceToDevice, c->st) !=
            cudaSuccess ||
        cudaStreamSynchronize(c->st) != cudaSuccess) {
      cudaGetLastError();
      gsq_destroy(c);
      *out = nullptr;
      rc = GSQ_ERR_CUDA;
    }
  }
  pool_free(lev);
  pool_free(sc);
  return rc;
}

int gsq_packed_bytes(int grid_mode, int64_t N, int64_t K, size_t* bytes) {
  if (!bytes || N <= 0 || K <= 0 || K % kGroup != 0 || num_logits(grid_mode) < 0)
    return GSQ_ERR_INVALID_ARG;
  const int b = grid_mode == GSQ_GRID_3BIT_LOCAL ? 3 : 2;
  *bytes = (size_t)N * (size_t)K * b / 8;
  return GSQ_OK;
}

}  // extern "C"

namespace {

int init_impl(gsq_ctx** out, const void* W, int w_dtype, const void* X,
              int x_dtype, int64_t N, int64_t K, int64_t T, int group,
              int grid_mode, const int8_t* init_idx, uint64_t seed,
              void* stream, int state16, int64_t row0 = 0) {
  if (!out) return GSQ_ERR_INVALID_ARG;
  *out = nullptr;
  // the global coordinates row0 K .. (row0 + N) K must fit the 64-bit
  // counter words
  if (row0 < 0 || (K > 0 && row0 > (((int64_t)1 << 62) / K) - N)) return GSQ_ERR_INVALID_ARG;
  if (!W || !X || N <= 0 || K <= 0 || T <= 0 || group <= 0 ||
      (w_dtype != GSQ_F32 && w_dtype != GSQ_BF16) ||
      (x_dtype != GSQ_F32 && x_dtype != GSQ_BF16) || num_logits(grid_mode) < 0 ||
      K % group != 0 || N > (int64_t)1 << 31 || T > (int64_t)1 << 31)
    return GSQ_ERR_INVALID_ARG;
  if (group != kGroup) return GSQ_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return GSQ_ERR_CUDA;
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;

  gsq_ctx* c = new (std::nothrow) gsq_ctx();
  if (!c) return GSQ_ERR_OOM;
  c->mode = grid_mode;
  c->L = num_logits(grid_mode);
  c->state16 = state16 ? 1 : 0;
  c->N = N;
  c->K = K;
  c->T = T;
  c->Tp = (T + 63) / 64 * 64;
  c->G = K / kGroup;
  c->seed = seed;
  c->coord0 = (uint64_t)row0 * (uint64_t)K;
  c->st = static_cast<cudaStream_t>(stream);
  c->dev = dev;
  c->sms = prop.multiProcessorCount;

  const int64_t NK = N * K, Tp = c->Tp;
  const bool split = (w_dtype == GSQ_F32);
  int rc = GSQ_OK;
#define AL(p, n) \
  if (rc == GSQ_OK) rc = dalloc(c, &(p), (size_t)(n))
  AL(c->Xb, Tp * K);
  AL(c->Xt, K * Tp);
  AL(c->What, NK);
  AL(c->dYt, N * Tp);
  AL(c->YrefT, N * Tp);
  AL(c->dW, NK);
  // bf16 state: half as many 4-byte words
  AL(c->logits, state16 ? (c->L * NK + 1) / 2 : c->L * NK);
  AL(c->mom, state16 ? (c->L * NK + 1) / 2 : c->L * NK);
  AL(c->s, N * c->G);
  AL(c->ms, N * c->G);
  AL(c->i0, NK);
  AL(c->hcode, NK);
  AL(c->partials, kMaxPartials);
  AL(c->loss_hist, kLossRing);
  AL(c->scratch, 4);
  AL(c->ticket, 4);
  AL(c->err, 4);
  {
    // both GEMMs of a step in one launch when the GEMMs' B operand (X, Tp x
    // K bf16) fits well inside L2: the merged launch runs each 256-row
    // band's column tiles together, so a wave reads every column tile of B
    // and one band of A.  (Measured on one B200: q_proj 4096 x 4096 -4.5%
    // per step, gate_proj 14336 x 4096 -0.8% (its GEMMs -6%); with a 117 MB
    // or 268 MB B, down_proj 4096 x 14336 and the 70B k_proj, +3% and +10%.)
    // Larger B keeps two launches, with the banded tile order from 24 row
    // tiles.
    const int64_t m_tiles = (N + 255) / 256;
    c->merged = (double)Tp * (double)K * 2.0 <= 64.0 * 1024 * 1024;
    AL(c->band_done, m_tiles);
  }
  // init-only staging
  float* W32 = nullptr;
  __nv_bfloat16 *Wop = nullptr, *Xcat = nullptr;
  void *Wd = nullptr, *Xd = nullptr;
  int8_t* idx_d = nullptr;
  std::vector<void*> staging;
  auto salloc = [&](void** p, size_t bytes) {
    if (rc != GSQ_OK) return;
    if (pool_malloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      rc = GSQ_ERR_OOM;
      return;
    }
    staging.push_back(*p);
  };
  salloc((void**)&W32, (size_t)NK * 4);
  salloc((void**)&Wop, (size_t)NK * 2 * (split ? 2 : 1));
  if (split) salloc((void**)&Xcat, (size_t)Tp * 2 * K * 2);
  const size_t wbytes = (size_t)NK * (w_dtype == GSQ_F32 ? 4 : 2);
  const size_t xbytes = (size_t)T * K * (x_dtype == GSQ_F32 ? 4 : 2);
  if (rc == GSQ_OK) {
    if (is_device_ptr(W)) Wd = const_cast<void*>(W);
    else salloc(&Wd, wbytes);
    if (is_device_ptr(X)) Xd = const_cast<void*>(X);
    else salloc(&Xd, xbytes);
    if (init_idx) {
      if (is_device_ptr(init_idx)) idx_d = const_cast<int8_t*>(init_idx);
      else salloc((void**)&idx_d, (size_t)NK);
    }
  }
  auto cleanup_fail = [&](int status) {
    cudaStreamSynchronize(c->st);
    cudaGetLastError();
    for (void* p : staging) pool_free(p);
    free_all(c);
    delete c;
    return status;
  };
  if (rc != GSQ_OK) return cleanup_fail(rc);

  cudaStream_t st = c->st;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
    return e == cudaSuccess;
  };
  if (Wd != W) ok(cudaMemcpyAsync(Wd, W, wbytes, cudaMemcpyDefault, st));
  if (Xd != X) ok(cudaMemcpyAsync(Xd, X, xbytes, cudaMemcpyDefault, st));
  if (init_idx && idx_d != init_idx)
    ok(cudaMemcpyAsync(idx_d, init_idx, (size_t)NK, cudaMemcpyDefault, st));
  ok(cudaMemsetAsync(c->err, 0, 4 * sizeof(int), st));
  ok(cudaMemsetAsync(c->ticket, 0, 4 * sizeof(unsigned), st));
  ok(cudaMemsetAsync(c->band_done, 0, (size_t)((N + 255) / 256) * sizeof(unsigned), st));
  ok(cudaMemsetAsync(c->loss_hist, 0, kLossRing * sizeof(double), st));
  ok(cudaMemsetAsync(c->mom, 0, state_plane_bytes(c), st));
  ok(cudaMemsetAsync(c->ms, 0, (size_t)N * c->G * 4, st));
  ok(cudaMemsetAsync(c->dW, 0, (size_t)NK * 4, st));
  ok(cudaMemsetAsync(c->dYt, 0, (size_t)N * Tp * 2, st));
  ok(launch_convert_x(Xd, x_dtype, T, K, Tp, c->Xb, c->Xt, Xcat, c->err, st));
  ok(launch_convert_w(Wd, w_dtype, N, K, W32, Wop, split ? 1 : 0, c->err, st));
  if (e != cudaSuccess) return cleanup_fail(cuda_status(e));

  // tensor maps of the persistent operands
  const int kw = split ? 2 : 1;
  CUtensorMap tmW, tmXr;
  if (make_tmap_bf16(&c->tm_What, c->What, N, K, K, kGemmBoxRowsA) ||
      make_tmap_bf16(&c->tm_Xb, c->Xb, Tp, K, K, kGemmBoxRowsB) ||
      make_tmap_bf16(&c->tm_dYt, c->dYt, N, Tp, Tp, kGemmBoxRowsA) ||
      make_tmap_bf16(&c->tm_Xt, c->Xt, K, Tp, Tp, kGemmBoxRowsB) ||
      make_tmap_bf16(&tmW, Wop, N, kw * K, kw * K, kGemmBoxRowsA) ||
      make_tmap_bf16(&tmXr, split ? Xcat : c->Xb, Tp, kw * K, kw * K, kGemmBoxRowsB) ||
      make_tmap_epi_bf16(&c->em_forward.out, c->dYt, N, Tp, Tp) ||
      make_tmap_epi_f32(&c->em_forward.yref, c->YrefT, N, Tp, Tp) ||
      make_tmap_epi_f32(&c->em_wgrad.out, c->dW, N, K, K))
    return cleanup_fail(GSQ_ERR_CUDA);
  c->em_wgrad.yref = c->em_forward.yref;  // unused by the fp32-store epilogue

  // Y_ref^T = W . bf16(X)^T (fp32 accumulate; W at its own precision)
  {
    EpiParams ep;
    std::memset(&ep, 0, sizeof(ep));
    ep.err = c->err;
    EpiMaps em;
    em.out = c->em_forward.yref;  // Y_ref^T is this GEMM's fp32 output
    em.yref = c->em_forward.yref;
    ok(launch_gemm(tmW, tmXr, em, N, Tp, kw * K, EPI_STORE_F32, ep, c->sms, st));
  }
  ok(launch_init_state(grid_mode, W32, idx_d, N, K, c->s, c->i0, c->logits,
                       c->err, st, c->state16));
  ok(launch_sumsq(c->YrefT, N * Tp, c->partials, c->ticket, c->scratch, st));
  if (e != cudaSuccess) return cleanup_fail(cuda_status(e));
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cleanup_fail(cuda_status(e));
  int h = 0;
  double ysq = 0.0;
  if (cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(&ysq, c->scratch, sizeof(double), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cleanup_fail(GSQ_ERR_CUDA);
  if (h == DEV_ERR_NONFINITE) return cleanup_fail(GSQ_ERR_NONFINITE);
  if (h == DEV_ERR_BAD_INIT) return cleanup_fail(GSQ_ERR_INVALID_ARG);
  if (h != DEV_OK) return cleanup_fail(h == DEV_ERR_TIMEOUT ? GSQ_ERR_TIMEOUT : GSQ_ERR_CUDA);
  c->yref_sq = ysq;
  for (void* p : staging) pool_free(p);
  *out = c;
  return GSQ_OK;
#undef AL
}

}  // namespace

extern "C" {

int gsq_init(gsq_ctx** out, const void* W, int w_dtype, const void* X,
             int x_dtype, int64_t N, int64_t K, int64_t T, int group,
             int grid_mode, const int8_t* init_idx, uint64_t seed,
             void* stream) {
  return init_impl(out, W, w_dtype, X, x_dtype, N, K, T, group, grid_mode, init_idx, seed,
                   stream, 0);
}

int gsq_init_bf16_state(gsq_ctx** out, const void* W, int w_dtype, const void* X,
                        int x_dtype, int64_t N, int64_t K, int64_t T, int group,
                        int grid_mode, const int8_t* init_idx, uint64_t seed,
                        void* stream) {
  return init_impl(out, W, w_dtype, X, x_dtype, N, K, T, group, grid_mode, init_idx, seed,
                   stream, 1);
}

int gsq_init_rows(gsq_ctx** out, const void* W, int w_dtype, const void* X, int x_dtype,
                  int64_t N, int64_t K, int64_t T, int group, int grid_mode,
                  const int8_t* init_idx, uint64_t seed, int64_t row0, int state_bf16,
                  void* stream) {
  if (state_bf16 != 0 && state_bf16 != 1) return GSQ_ERR_INVALID_ARG;
  return init_impl(out, W, w_dtype, X, x_dtype, N, K, T, group, grid_mode, init_idx, seed,
                   stream, state_bf16, row0);
}

}  // extern "C"

namespace {

// One step t at temperature tau; with tau_next > 0 the backward also builds
// the soft weight of step t + 1 (which the next call then skips).
int run_step(gsq_ctx* c, float tau, float tau_next, float lr, float beta1,
             float beta2) {
  if (c->t >= 0xFFFFFFFEull) return GSQ_ERR_UNSUPPORTED;  // 32-bit counter word
  const StepArgs a = step_args(c, tau);
  Timing* tm = nullptr;
  if (c->timing) {
    if (c->tev_used == c->tev.size()) {
      Timing te;
      for (auto& ev : te.ev) CK(cudaEventCreate(&ev));
      c->tev.push_back(te);
    }
    tm = &c->tev[c->tev_used++];
    CK(cudaEventRecord(tm->ev[0], c->st));
  }
  NvtxRange step_range("gsq_step");
  const bool soft = !(c->what_t == (int64_t)c->t && c->what_tau == tau);
  if (soft) {
    NvtxRange r("soft_weight");
    CK(launch_soft_weight(a, c->What, nullptr, c->sms, c->st));
  }
  if (tm) {
    tm->soft = soft;
    tm->next = tau_next > 0.f;
    CK(cudaEventRecord(tm->ev[1], c->st));
  }
  if (c->merged) {
    NvtxRange r("gemms_merged");
    CK(run_gemms_merged(c, c->loss_hist + (c->t % kLossRing)));
    if (tm) {
      tm->merged = true;
      CK(cudaEventRecord(tm->ev[2], c->st));
      CK(cudaEventRecord(tm->ev[3], c->st));
    }
  } else {
    {
      NvtxRange r("forward_gemm");
      CK(run_forward(c, c->loss_hist + (c->t % kLossRing), EPI_LOSS_DY));
    }
    if (tm) {
      tm->merged = false;
      CK(cudaEventRecord(tm->ev[2], c->st));
    }
    {
      NvtxRange r("weight_grad_gemm");
      CK(run_weight_grad(c));
    }
    if (tm) CK(cudaEventRecord(tm->ev[3], c->st));
  }
  {
    NvtxRange r(tau_next > 0.f ? "backward_lion_next_soft" : "backward_lion");
    CK(launch_backward_lion(a, c->dW, lr, beta1, beta2, tau_next, c->What, nullptr, nullptr,
                            c->sms, c->st));
  }
  if (tm) CK(cudaEventRecord(tm->ev[4], c->st));
  c->t += 1;
  c->hcode_valid = false;  // the logits moved
  if (tau_next > 0.f) {
    c->what_t = (int64_t)c->t;
    c->what_tau = tau_next;
  } else {
    c->what_t = -1;
  }
  return GSQ_OK;
}

// codes of the hard choice of the current logits, computed once per logits
cudaError_t ensure_hard_codes(gsq_ctx* c) {
  if (c->hcode_valid) return cudaSuccess;
  cudaError_t e = launch_hard_codes(c->mode, c->N, c->K, c->logits, c->i0, c->hcode, c->st,
                                    c->state16);
  if (e == cudaSuccess) c->hcode_valid = true;
  return e;
}

// One scale-only step: hard weight from the frozen codes and the current
// scales, forward + loss, weight gradient, scale gradient + Lion on s.
int run_scale_step(gsq_ctx* c, float lr, float beta1, float beta2) {
  if (c->t >= 0xFFFFFFFEull) return GSQ_ERR_UNSUPPORTED;
  CK(ensure_hard_codes(c));
  CK(launch_code_weight(c->mode, c->N, c->K, c->hcode, c->s, c->What, c->st));
  CK(run_forward(c, c->loss_hist + (c->t % kLossRing), EPI_LOSS_DY));
  CK(run_weight_grad(c));
  CK(launch_scale_lion(c->mode, c->N, c->K, c->hcode, c->dW, c->s, c->ms, lr, beta1, beta2,
                       nullptr, c->sms, c->st));
  c->t += 1;
  c->what_t = -1;
  return GSQ_OK;
}

}  // namespace

extern "C" {

int gsq_scale_step(gsq_ctx* c, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(1.0f, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  return run_scale_step(c, lr, beta1, beta2);
}

int gsq_scale_run(gsq_ctx* c, int64_t n, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (n <= 0 || !step_args_ok(1.0f, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int rc = run_scale_step(c, lr, beta1, beta2);
    if (rc) return rc;
  }
  return GSQ_OK;
}

int gsq_step(gsq_ctx* c, float tau, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  return run_step(c, tau, 0.f, lr, beta1, beta2);
}

int gsq_step_next(gsq_ctx* c, float tau, float tau_next, float lr, float beta1,
                  float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(tau, lr, beta1, beta2) || !(tau_next > 0.f && std::isfinite(tau_next)))
    return GSQ_ERR_INVALID_ARG;
  return run_step(c, tau, tau_next, lr, beta1, beta2);
}

int gsq_run(gsq_ctx* c, const float* taus, int64_t n, float lr, float beta1,
            float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!taus || n <= 0) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i)
    if (!step_args_ok(taus[i], lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int rc = run_step(c, taus[i], i + 1 < n ? taus[i + 1] : 0.f, lr,
                            beta1, beta2);
    if (rc) return rc;
  }
  return GSQ_OK;
}

int gsq_last_loss(gsq_ctx* c, double* loss) {
  int u = usable(c);
  if (u) return u;
  if (!loss) return GSQ_ERR_INVALID_ARG;
  if (c->t == 0) return GSQ_ERR_STATE;
  int rc = check_device(c);
  if (rc) return rc;
  CK(cudaMemcpy(loss, c->loss_hist + ((c->t - 1) % kLossRing), sizeof(double),
                cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_loss_history(gsq_ctx* c, uint64_t t0, int64_t n, double* host_out) {
  int u = usable(c);
  if (u) return u;
  if (!host_out || n < 0 || t0 + (uint64_t)n > c->t || n > kLossRing ||
      c->t - t0 > (uint64_t)kLossRing)
    return GSQ_ERR_INVALID_ARG;
  int rc = check_device(c);
  if (rc) return rc;
  std::vector<double> ring(kLossRing);
  CK(cudaMemcpy(ring.data(), c->loss_hist, kLossRing * sizeof(double),
                cudaMemcpyDeviceToHost));
  for (int64_t i = 0; i < n; ++i) host_out[i] = ring[(t0 + i) % kLossRing];
  return GSQ_OK;
}

int gsq_harden_pack(gsq_ctx* c, void* packed, uint16_t* scales_f16,
                    float* scales_f32) {
  int u = usable(c);
  if (u) return u;
  if (!packed) return GSQ_ERR_INVALID_ARG;
  size_t pbytes = 0;
  gsq_packed_bytes(c->mode, c->N, c->K, &pbytes);
  const int64_t ng = c->N * c->G;
  // kernels write device memory: caller's if it is device, else staging
  const bool pd = is_device_ptr(packed);
  const bool hd = !scales_f16 || is_device_ptr(scales_f16);
  const bool fd = !scales_f32 || is_device_ptr(scales_f32);
  void* stage = nullptr;
  size_t sbytes = (pd ? 0 : pbytes) + (hd ? 0 : ng * 2) + (fd ? 0 : ng * 4) + 64;
  CK(pool_malloc(&stage, sbytes));
  char* sp = static_cast<char*>(stage);
  uint32_t* pk = pd ? static_cast<uint32_t*>(packed) : reinterpret_cast<uint32_t*>(sp);
  if (!pd) sp += (pbytes + 15) / 16 * 16;
  uint16_t* h16 = scales_f16 ? (hd ? scales_f16 : reinterpret_cast<uint16_t*>(sp)) : nullptr;
  if (scales_f16 && !hd) sp += (ng * 2 + 15) / 16 * 16;
  float* f32 = scales_f32 ? (fd ? scales_f32 : reinterpret_cast<float*>(sp)) : nullptr;
  cudaError_t e = launch_harden_pack(c->mode, c->N, c->K, c->logits, c->i0, pk, c->st,
                                     c->state16);
  if (e == cudaSuccess && (h16 || f32))
    e = launch_export_scales(c->s, ng, h16, f32, c->st);
  if (e == cudaSuccess && !pd)
    e = cudaMemcpyAsync(packed, pk, pbytes, cudaMemcpyDefault, c->st);
  if (e == cudaSuccess && scales_f16 && !hd)
    e = cudaMemcpyAsync(scales_f16, h16, ng * 2, cudaMemcpyDefault, c->st);
  if (e == cudaSuccess && scales_f32 && !fd)
    e = cudaMemcpyAsync(scales_f32, f32, ng * 4, cudaMemcpyDefault, c->st);
  cudaError_t e2 = cudaStreamSynchronize(c->st);
  pool_free(stage);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  if (e2 != cudaSuccess) return fail(c, cuda_status(e2));
  return check_device(c);
}

int gsq_recon_error(gsq_ctx* c, int mode, float tau, double* abs_err,
                    double* rel_err) {
  int u = usable(c);
  if (u) return u;
  if (!abs_err || (mode != GSQ_RECON_HARD && mode != GSQ_RECON_SOFT) ||
      (mode == GSQ_RECON_SOFT && !(tau > 0.f && std::isfinite(tau))))
    return GSQ_ERR_INVALID_ARG;
  c->what_t = -1;  // What is overwritten below
  if (mode == GSQ_RECON_HARD) {
    CK(launch_hard_weight(c->mode, c->N, c->K, c->logits, c->s, c->i0, c->What, c->st,
                          c->state16));
  } else {
    StepArgs a = step_args(c, tau);
    a.noise = 0;
    CK(launch_soft_weight(a, c->What, nullptr, c->sms, c->st));
  }
  CK(run_forward(c, c->scratch, EPI_LOSS));
  int rc = check_device(c);
  if (rc) return rc;
  double v = 0.0;
  CK(cudaMemcpy(&v, c->scratch, sizeof(double), cudaMemcpyDeviceToHost));
  *abs_err = v;
  if (rel_err) *rel_err = c->yref_sq > 0.0 ? v / c->yref_sq : 0.0;
  return GSQ_OK;
}

int gsq_state_bytes(gsq_ctx* c, size_t* bytes) {
  if (!c || !bytes) return GSQ_ERR_INVALID_ARG;
  *bytes = 8 * sizeof(uint64_t) + state_plane_bytes(c) * 2 + (size_t)c->N * c->G * 4 * 2;
  return GSQ_OK;
}

int gsq_export_state(gsq_ctx* c, void* host_buf, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  size_t need = 0;
  gsq_state_bytes(c, &need);
  if (!host_buf || bytes != need) return GSQ_ERR_INVALID_ARG;
  int rc = check_device(c);
  if (rc) return rc;
  uint64_t* h = static_cast<uint64_t*>(host_buf);
  h[0] = kStateMagic;
  h[1] = (uint64_t)c->mode;
  h[2] = (uint64_t)c->N;
  h[3] = (uint64_t)c->K;
  h[4] = (uint64_t)c->group;
  h[5] = c->t;
  h[6] = c->seed;
  h[7] = (uint64_t)c->state16;
  char* p = static_cast<char*>(host_buf) + 8 * sizeof(uint64_t);
  const size_t lb = state_plane_bytes(c), sb = (size_t)c->N * c->G * 4;
  CK(cudaMemcpy(p, c->logits, lb, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(p + lb, c->mom, lb, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(p + 2 * lb, c->s, sb, cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(p + 2 * lb + sb, c->ms, sb, cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_import_state(gsq_ctx* c, const void* host_buf, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  size_t need = 0;
  gsq_state_bytes(c, &need);
  if (!host_buf || bytes != need) return GSQ_ERR_INVALID_ARG;
  const uint64_t* h = static_cast<const uint64_t*>(host_buf);
  if (h[0] != kStateMagic || h[1] != (uint64_t)c->mode || h[2] != (uint64_t)c->N ||
      h[3] != (uint64_t)c->K || h[4] != (uint64_t)c->group || h[6] != c->seed ||
      h[7] != (uint64_t)c->state16)
    return GSQ_ERR_INVALID_ARG;
  CK(cudaStreamSynchronize(c->st));
  const char* p = static_cast<const char*>(host_buf) + 8 * sizeof(uint64_t);
  const size_t lb = state_plane_bytes(c), sb = (size_t)c->N * c->G * 4;
  CK(cudaMemcpy(c->logits, p, lb, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(c->mom, p + lb, lb, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(c->s, p + 2 * lb, sb, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(c->ms, p + 2 * lb + sb, sb, cudaMemcpyHostToDevice));
  c->t = h[5];
  c->what_t = -1;
  c->hcode_valid = false;
  return GSQ_OK;
}

int gsq_get_step(gsq_ctx* c, uint64_t* t) {
  if (!c || !t) return GSQ_ERR_INVALID_ARG;
  *t = c->t;
  return GSQ_OK;
}

int gsq_destroy(gsq_ctx* c) {
  if (!c) return GSQ_OK;
  cudaStreamSynchronize(c->st);
  cudaGetLastError();
  free_all(c);
  delete c;
  return GSQ_OK;
}

// ------------------------------------------------------------- timing

int gsq_set_timing(gsq_ctx* c, int on) {
  int u = usable(c);
  if (u) return u;
  c->timing = on != 0;
  return GSQ_OK;
}

int gsq_phase_times(gsq_ctx* c, double* ms, int64_t* launches) {
  int u = usable(c);
  if (u) return u;
  if (!ms) return GSQ_ERR_INVALID_ARG;
  CK(cudaStreamSynchronize(c->st));
  double acc[5] = {0, 0, 0, 0, 0};
  int64_t n[5] = {0, 0, 0, 0, 0};
  for (size_t i = 0; i < c->tev_used; ++i) {
    const Timing& te = c->tev[i];
    for (int p = 0; p < 4; ++p) {
      float x = 0.f;
      CK(cudaEventElapsedTime(&x, te.ev[p], te.ev[p + 1]));
      // backward launches that also built the next soft weight count apart
      const int slot = (p == 3 && te.next) ? 4 : p;
      acc[slot] += x;
      // a merged launch is one launch in the forward slot; the weight-gradient
      // slot then holds two back-to-back events
      if ((p != 0 || te.soft) && !(p == 2 && te.merged)) n[slot] += 1;
    }
  }
  for (int p = 0; p < 5; ++p) {
    ms[p] = acc[p];
    if (launches) launches[p] = n[p];
  }
  c->tev_used = 0;
  return GSQ_OK;
}

// ------------------------------------------------------------- debug

static int debug_buffer(gsq_ctx* c, int which, void** p, size_t* bytes) {
  const size_t NK = (size_t)c->N * c->K, LNK = (size_t)c->L * NK,
               NG = (size_t)c->N * c->G;
  int rc = GSQ_OK;
  switch (which) {
    case GSQ_DBG_LOGITS: *p = c->logits; *bytes = state_plane_bytes(c); break;
    case GSQ_DBG_MOM: *p = c->mom; *bytes = state_plane_bytes(c); break;
    case GSQ_DBG_SCALES: *p = c->s; *bytes = NG * 4; break;
    case GSQ_DBG_SMOM: *p = c->ms; *bytes = NG * 4; break;
    case GSQ_DBG_I0: *p = c->i0; *bytes = NK; break;
    case GSQ_DBG_WHAT: *p = c->What; *bytes = NK * 2; break;
    case GSQ_DBG_WSOFT32:
      if (!c->wsoft32) rc = dalloc(c, &c->wsoft32, NK);
      *p = c->wsoft32; *bytes = NK * 4; break;
    case GSQ_DBG_DW: *p = c->dW; *bytes = NK * 4; break;
    case GSQ_DBG_DYT: *p = c->dYt; *bytes = (size_t)c->N * c->Tp * 2; break;
    case GSQ_DBG_YREFT: *p = c->YrefT; *bytes = (size_t)c->N * c->Tp * 4; break;
    case GSQ_DBG_DL:
      if (!c->dl) rc = dalloc(c, &c->dl, LNK);
      *p = c->dl; *bytes = LNK * 4; break;
    case GSQ_DBG_DS:
      if (!c->ds) rc = dalloc(c, &c->ds, NG);
      *p = c->ds; *bytes = NG * 4; break;
    default: return GSQ_ERR_INVALID_ARG;
  }
  return rc;
}

int gsq_debug_get(gsq_ctx* c, int which, void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = debug_buffer(c, which, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  rc = check_device(c);
  if (rc) return rc;
  CK(cudaMemcpy(host, p, nb, cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_debug_set(gsq_ctx* c, int which, const void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = debug_buffer(c, which, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  CK(cudaStreamSynchronize(c->st));
  CK(cudaMemcpy(p, host, nb, cudaMemcpyHostToDevice));
  c->what_t = -1;  // any state change invalidates a precomputed soft weight
  c->hcode_valid = false;  // and the hard codes
  return GSQ_OK;
}

int gsq_debug_noise(gsq_ctx* c, int on) {
  int u = usable(c);
  if (u) return u;
  c->noise = on ? 1 : 0;
  c->what_t = -1;
  return GSQ_OK;
}

int gsq_debug_uniforms(gsq_ctx* c, uint32_t t, uint64_t coord0, int64_t count,
                       float* host_out) {
  int u = usable(c);
  if (u) return u;
  if (!host_out || count <= 0) return GSQ_ERR_INVALID_ARG;
  float* d = nullptr;
  CK(pool_malloc(&d, (size_t)count * c->L * 4));
  cudaError_t e = launch_uniforms(c->mode, c->seed, t, coord0, count, d, c->st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->st);
  if (e == cudaSuccess)
    e = cudaMemcpy(host_out, d, (size_t)count * c->L * 4, cudaMemcpyDeviceToHost);
  pool_free(d);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  return GSQ_OK;
}

int gsq_debug_noise_log2(gsq_ctx* c, uint32_t m0, int64_t count, float* host_out) {
  int u = usable(c);
  if (u) return u;
  if (!host_out || count <= 0 || (int64_t)m0 + count > ((int64_t)1 << 23))
    return GSQ_ERR_INVALID_ARG;
  float* d = nullptr;
  CK(pool_malloc(&d, (size_t)count * 4));
  cudaError_t e = launch_log2_unit(m0, count, d, c->st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(c->st);
  if (e == cudaSuccess) e = cudaMemcpy(host_out, d, (size_t)count * 4, cudaMemcpyDeviceToHost);
  pool_free(d);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  return GSQ_OK;
}

int gsq_debug_stall_probe(gsq_ctx* c) {
  int u = usable(c);
  if (u) return u;
  c->stall_probe = 1;
  return GSQ_OK;
}

int gsq_debug_soft_weight(gsq_ctx* c, float tau) {
  int u = usable(c);
  if (u) return u;
  if (!(tau > 0.f && std::isfinite(tau))) return GSQ_ERR_INVALID_ARG;
  void* p;
  size_t nb;
  int rc = debug_buffer(c, GSQ_DBG_WSOFT32, &p, &nb);
  if (rc) return rc;
  CK(launch_soft_weight(step_args(c, tau), c->What, c->wsoft32, c->sms, c->st));
  c->what_t = (int64_t)c->t;
  c->what_tau = tau;
  return check_device(c);
}

int gsq_debug_forward(gsq_ctx* c, double* loss) {
  int u = usable(c);
  if (u) return u;
  if (!loss) return GSQ_ERR_INVALID_ARG;
  CK(run_forward(c, c->scratch, EPI_LOSS_DY));
  int rc = check_device(c);
  if (rc) return rc;
  CK(cudaMemcpy(loss, c->scratch, sizeof(double), cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_debug_weight_grad(gsq_ctx* c) {
  int u = usable(c);
  if (u) return u;
  CK(run_weight_grad(c));
  return check_device(c);
}

int gsq_debug_backward(gsq_ctx* c, float tau, float lr, float beta1,
                       float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  void* p;
  size_t nb;
  int rc = debug_buffer(c, GSQ_DBG_DL, &p, &nb);
  if (!rc) rc = debug_buffer(c, GSQ_DBG_DS, &p, &nb);
  if (rc) return rc;
  // the backward draws the step's probabilities itself
  const StepArgs a = step_args(c, tau);
  CK(launch_backward_lion(a, c->dW, lr, beta1, beta2, 0.f, c->What,
                          c->dl, c->ds, c->sms, c->st));
  c->what_t = -1;
  c->hcode_valid = false;
  return check_device(c);
}

int gsq_debug_scale_backward(gsq_ctx* c, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(1.0f, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  void* p;
  size_t nb;
  int rc = debug_buffer(c, GSQ_DBG_DS, &p, &nb);
  if (rc) return rc;
  CK(ensure_hard_codes(c));
  CK(launch_scale_lion(c->mode, c->N, c->K, c->hcode, c->dW, c->s, c->ms, lr, beta1, beta2,
                       c->ds, c->sms, c->st));
  return check_device(c);
}

}  // extern "C"

namespace {

// C (M x N fp32, ldc = N) = A B^T (EPI_STORE_F32) or C -= A B^T (EPI_SUB_F32)
int gemm_bf16_abt_mode(const void* A, const void* B, float* Cout, int64_t M, int64_t N,
                       int64_t Kc, int mode, void* stream) {
  if (!A || !B || !Cout || M <= 0 || N <= 0 || Kc <= 0 || Kc % 8 != 0 ||
      N % 4 != 0 || (reinterpret_cast<uintptr_t>(Cout) & 15) ||
      (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(B) & 15))
    return GSQ_ERR_INVALID_ARG;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap ta, tb;
  if (make_tmap_bf16(&ta, A, M, Kc, Kc, kGemmBoxRowsA) ||
      make_tmap_bf16(&tb, B, N, Kc, Kc, kGemmBoxRowsB))
    return GSQ_ERR_CUDA;
  int* err = nullptr;
  if (pool_malloc(&err, 16) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_OOM;
  }
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.err = err;
  EpiMaps em;
  if (make_tmap_epi_f32(&em.out, Cout, M, N, N)) {
    pool_free(err);
    return GSQ_ERR_CUDA;
  }
  em.yref = em.out;
  cudaError_t e = cudaMemsetAsync(err, 0, 16, st);
  if (e == cudaSuccess)
    e = launch_gemm(ta, tb, em, M, N, Kc, mode, ep, prop.multiProcessorCount, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  int h = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost);
  pool_free(err);
  if (e != cudaSuccess) return cuda_status(e);
  return h == DEV_OK ? GSQ_OK : GSQ_ERR_TIMEOUT;
}

}  // namespace

extern "C" {

int gsq_gemm_bf16_abt(const void* A, const void* B, float* Cout, int64_t M,
                      int64_t N, int64_t Kc, void* stream) {
  return gemm_bf16_abt_mode(A, B, Cout, M, N, Kc, EPI_STORE_F32, stream);
}

int gsq_gemm_bf16_abt_sub(const void* A, const void* B, float* C, int64_t M, int64_t N,
                          int64_t Kc, void* stream) {
  return gemm_bf16_abt_mode(A, B, C, M, N, Kc, EPI_SUB_F32, stream);
}

}  // extern "C"
