// gsq_mlp.cu -- the block's MLP stage: joint reconstruction of the gate, up
// and down projections of a SwiGLU MLP against the block output (GSQ staging,
// agihunt.info summary, optimisation paragraph: the MLP is trained on the
// block output after the attention stages).
//
// Per step t at temperature tau (all GEMMs on the CTA-pair tcgen05 kernel,
// both operands K-major; "^T" layouts are chosen so that every contraction
// is A . B^T):
//   soft weights G, U (F x H), D (H x F)      (own Philox stream per weight)
//   a^T = G . Xn^T, b^T = U . Xn^T             (F x T, fp32)
//   h^T = bf16(silu(a^T) b^T), h = (h^T)^T     (bf16)
//   pred^T = D . h^T^T; E = pred^T - R^T; loss = sum E^2; dp^T = bf16(2E)
//   dD = dp^T . (h^T)^T                        (H x F)
//   dh^T = D^T . dp^T^T  (D^T, dp transposed copies)   (F x T, fp32)
//   da^T = bf16(dh^T b^T silu'(a^T)), db^T = bf16(dh^T silu(a^T))
//   dG = da^T . Xn, dU = db^T . Xn             (F x H; Xn^T as B)
//   backward + Lion per weight (optionally building step t+1's soft weight)
#include <cmath>
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

struct Weight {
  int64_t N = 0, K = 0, G = 0;
  uint64_t seed = 0;
  float *logits = nullptr, *mom = nullptr, *s = nullptr, *ms = nullptr;
  float* dW = nullptr;
  int8_t* i0 = nullptr;
  __nv_bfloat16* What = nullptr;
  CUtensorMap tmA;  // What as GEMM operand A
  EpiMaps em_dW;    // dW as fp32 epilogue output
};

}  // namespace

struct gsq_mlp {
  int mode = 0, L = 0;
  PhaseClock clock;  // per-phase device time (gsq_mlp_set_timing)
  int64_t T = 0, H = 0, F = 0;
  uint64_t t = 0;
  int noise = 1;
  cudaStream_t st = nullptr;
  int sms = 148;
  int failed = 0;
  Weight w[3];  // gate (F x H), up (F x H), down (H x F)
  __nv_bfloat16 *Xn = nullptr, *XnT = nullptr, *hT = nullptr, *h = nullptr;
  __nv_bfloat16 *dpT = nullptr, *dp = nullptr, *WdT = nullptr;
  __nv_bfloat16 *daT = nullptr, *dbT = nullptr;
  float *RT = nullptr, *aT = nullptr, *bT = nullptr, *dhT = nullptr;
  double *partials = nullptr, *loss_hist = nullptr, *scratch = nullptr;
  unsigned* ticket = nullptr;
  int* err = nullptr;
  double r_sq = 0.0;
  int64_t what_t = -1;
  float what_tau = 0.f;
  CUtensorMap tmB_Xn, tmB_h, tmB_hT, tmB_dp, tmB_XnT;
  CUtensorMap tmA_dpT, tmA_WdT, tmA_daT, tmA_dbT;
  EpiMaps em_aT, em_bT, em_pred, em_dhT;
  std::vector<void*> allocs;
};

namespace {

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GSQ_OK;
  if (e == cudaErrorMemoryAllocation) return GSQ_ERR_OOM;
  return GSQ_ERR_CUDA;
}

int fail(gsq_mlp* c, int status) {
  if (c && status != GSQ_OK && c->failed == 0) c->failed = status;
  return status;
}

#define CKM(call)                                           \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return fail(c, cuda_status(e_)); \
  } while (0)

template <typename T>
int alloc(gsq_mlp* c, T** p, size_t count) {
  void* q = nullptr;
  if (pool_malloc(&q, count * sizeof(T) + 16) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_OOM;
  }
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return GSQ_OK;
}

void free_all(gsq_mlp* c) {
  for (void* p : c->allocs) pool_free(p);
  c->allocs.clear();
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

int check_device(gsq_mlp* c) {
  cudaError_t e = cudaStreamSynchronize(c->st);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  int h = 0;
  e = cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  switch (h) {
    case DEV_OK: return GSQ_OK;
    case DEV_ERR_TIMEOUT: return fail(c, GSQ_ERR_TIMEOUT);
    case DEV_ERR_NONFINITE: return fail(c, GSQ_ERR_NONFINITE);
    default: return fail(c, GSQ_ERR_CUDA);
  }
}

int usable(gsq_mlp* c) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  return GSQ_OK;
}

StepArgs weight_args(gsq_mlp* c, int i, float tau) {
  const Weight& w = c->w[i];
  StepArgs a;
  a.mode = c->mode;
  a.N = w.N;
  a.K = w.K;
  a.G = w.G;
  a.logits = w.logits;
  a.logits_w = w.logits;
  a.mom = w.mom;
  a.s = w.s;
  a.ms = w.ms;
  a.i0 = w.i0;
  a.seed = w.seed;
  a.t = (uint32_t)c->t;
  a.noise = c->noise;
  a.tau = tau;
  return a;
}

EpiParams epi(gsq_mlp* c, double* loss_out) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.partials = c->partials;
  ep.ticket = c->ticket;
  ep.loss_out = loss_out;
  ep.err = c->err;
  return ep;
}

// forward from the weights in w[i].What: a^T, b^T, h^T, h, then pred^T with
// the loss (and dp^T when with_dp) into *loss_out
cudaError_t forward(gsq_mlp* c, double* loss_out, bool with_dp) {
  const int64_t T = c->T, H = c->H, F = c->F;
  cudaError_t e;
  EpiParams ep = epi(c, loss_out);
  PhaseClock& k = c->clock;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  if ((e = launch_gemm(c->w[0].tmA, c->tmB_Xn, c->em_aT, F, T, H, EPI_STORE_F32, ep,
                       c->sms, c->st)) != cudaSuccess) return e;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  if ((e = launch_gemm(c->w[1].tmA, c->tmB_Xn, c->em_bT, F, T, H, EPI_STORE_F32, ep,
                       c->sms, c->st)) != cudaSuccess) return e;
  if ((e = k.mark(c->st, PH_ELEM)) != cudaSuccess) return e;
  if ((e = launch_swiglu_fwd(c->aT, c->bT, F * T, c->hT, c->sms, c->st)) != cudaSuccess)
    return e;
  if ((e = k.mark(c->st, PH_ELEM)) != cudaSuccess) return e;
  if ((e = launch_transpose_bf16(c->hT, F, T, c->h, c->st)) != cudaSuccess) return e;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  return launch_gemm(c->w[2].tmA, c->tmB_h, c->em_pred, H, T, F,
                     with_dp ? EPI_LOSS_DY : EPI_LOSS, ep, c->sms, c->st);
}

bool step_args_ok(float tau, float lr, float b1, float b2) {
  return tau > 0.f && std::isfinite(tau) && lr >= 0.f && std::isfinite(lr) &&
         b1 >= 0.f && b1 < 1.f && b2 >= 0.f && b2 < 1.f;
}

int run_step(gsq_mlp* c, float tau, float tau_next, float lr, float b1, float b2) {
  if (c->t >= 0xFFFFFFFEull) return GSQ_ERR_UNSUPPORTED;
  NvtxRange step_range("gsq_mlp_step");
  const int64_t T = c->T, H = c->H, F = c->F;
  PhaseClock& k = c->clock;
  if (!(c->what_t == (int64_t)c->t && c->what_tau == tau))
    for (int i = 0; i < 3; ++i) {
      CKM(k.mark(c->st, PH_SOFT));
      CKM(launch_soft_weight(weight_args(c, i, tau), c->w[i].What, nullptr, c->sms,
                             c->st));
    }
  CKM(forward(c, c->loss_hist + (c->t % kLossRing), true));
  EpiParams ep = epi(c, nullptr);
  // dD = dp^T . (h^T)^T
  CKM(k.mark(c->st, PH_GEMM));
  CKM(launch_gemm(c->tmA_dpT, c->tmB_hT, c->w[2].em_dW, H, F, T, EPI_STORE_F32, ep,
                  c->sms, c->st));
  // dh^T = D^T . dp^T  (transposed copies of D and dp^T)
  CKM(k.mark(c->st, PH_ELEM));
  CKM(launch_transpose_bf16(c->w[2].What, H, F, c->WdT, c->st));
  CKM(k.mark(c->st, PH_ELEM));
  CKM(launch_transpose_bf16(c->dpT, H, T, c->dp, c->st));
  CKM(k.mark(c->st, PH_GEMM));
  CKM(launch_gemm(c->tmA_WdT, c->tmB_dp, c->em_dhT, F, T, H, EPI_STORE_F32, ep,
                  c->sms, c->st));
  CKM(k.mark(c->st, PH_ELEM));
  CKM(launch_swiglu_bwd(c->aT, c->bT, c->dhT, F * T, c->daT, c->dbT, c->sms, c->st));
  // dG = da^T . Xn, dU = db^T . Xn
  CKM(k.mark(c->st, PH_GEMM));
  CKM(launch_gemm(c->tmA_daT, c->tmB_XnT, c->w[0].em_dW, F, H, T, EPI_STORE_F32, ep,
                  c->sms, c->st));
  CKM(k.mark(c->st, PH_GEMM));
  CKM(launch_gemm(c->tmA_dbT, c->tmB_XnT, c->w[1].em_dW, F, H, T, EPI_STORE_F32, ep,
                  c->sms, c->st));
  for (int i = 0; i < 3; ++i) {
    CKM(k.mark(c->st, PH_BACKWARD));
    CKM(launch_backward_lion(weight_args(c, i, tau), c->w[i].dW, lr, b1,
                             b2, tau_next, c->w[i].What, nullptr, nullptr, c->sms,
                             c->st));
  }
  CKM(k.mark(c->st, -1));
  c->t += 1;
  if (tau_next > 0.f) {
    c->what_t = (int64_t)c->t;
    c->what_tau = tau_next;
  } else {
    c->what_t = -1;
  }
  return GSQ_OK;
}

int num_logits(int mode) {
  return mode == GSQ_GRID_3BIT_LOCAL ? 5 : (mode == GSQ_GRID_2BIT || mode == GSQ_GRID_TERNARY) ? 4 : -1;
}

}  // namespace

extern "C" {

int gsq_mlp_init(gsq_mlp** out, const void* Xn, int x_dtype, const void* R,
                 int r_dtype, const void* Wg, const void* Wu, const void* Wd,
                 int w_dtype, int64_t T, int64_t H, int64_t F, int group,
                 int grid_mode, uint64_t seed, void* stream) {
  if (!out) return GSQ_ERR_INVALID_ARG;
  *out = nullptr;
  auto dt_ok = [](int d) { return d == GSQ_F32 || d == GSQ_BF16; };
  if (!Xn || !R || !Wg || !Wu || !Wd || T <= 0 || H <= 0 || F <= 0 ||
      !dt_ok(x_dtype) || !dt_ok(r_dtype) || !dt_ok(w_dtype) ||
      num_logits(grid_mode) < 0 || group <= 0 || H % group != 0 ||
      F % group != 0 || T % 64 != 0 || T > (int64_t)1 << 31)
    return GSQ_ERR_INVALID_ARG;
  if (group != kGroup) return GSQ_ERR_UNSUPPORTED;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  gsq_mlp* c = new (std::nothrow) gsq_mlp();
  if (!c) return GSQ_ERR_OOM;
  c->mode = grid_mode;
  c->L = num_logits(grid_mode);
  c->T = T;
  c->H = H;
  c->F = F;
  c->st = static_cast<cudaStream_t>(stream);
  c->sms = prop.multiProcessorCount;
  const int64_t dims[3][2] = {{F, H}, {F, H}, {H, F}};
  int rc = GSQ_OK;
#define ALM(p, n) \
  if (rc == GSQ_OK) rc = alloc(c, &(p), (size_t)(n))
  for (int i = 0; i < 3; ++i) {
    Weight& w = c->w[i];
    w.N = dims[i][0];
    w.K = dims[i][1];
    w.G = w.K / kGroup;
    // own Philox key per weight: high key word xor (weight index << 16)
    w.seed = seed ^ ((uint64_t)i << 48);
    const int64_t NK = w.N * w.K;
    ALM(w.logits, c->L * NK);
    ALM(w.mom, c->L * NK);
    ALM(w.s, w.N * w.G);
    ALM(w.ms, w.N * w.G);
    ALM(w.i0, NK);
    ALM(w.What, NK);
    ALM(w.dW, NK);
  }
  ALM(c->Xn, T * H);
  ALM(c->XnT, H * T);
  ALM(c->RT, H * T);
  ALM(c->aT, F * T);
  ALM(c->bT, F * T);
  ALM(c->hT, F * T);
  ALM(c->h, T * F);
  ALM(c->dpT, H * T);
  ALM(c->dp, T * H);
  ALM(c->WdT, F * H);
  ALM(c->dhT, F * T);
  ALM(c->daT, F * T);
  ALM(c->dbT, F * T);
  ALM(c->partials, kMaxPartials);
  ALM(c->loss_hist, kLossRing);
  ALM(c->scratch, 4);
  ALM(c->ticket, 4);
  ALM(c->err, 4);
#undef ALM
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
  auto cleanup_fail = [&](int status) {
    cudaStreamSynchronize(c->st);
    cudaGetLastError();
    for (void* p : staging) pool_free(p);
    free_all(c);
    delete c;
    return status;
  };
  const int64_t maxNK = F * H;
  float* W32 = nullptr;
  __nv_bfloat16* Wop = nullptr;
  salloc((void**)&W32, (size_t)maxNK * 4);
  salloc((void**)&Wop, (size_t)maxNK * 2);
  const size_t xb = (size_t)T * H * (x_dtype == GSQ_F32 ? 4 : 2);
  const size_t rb = (size_t)T * H * (r_dtype == GSQ_F32 ? 4 : 2);
  const size_t wb = (size_t)maxNK * (w_dtype == GSQ_F32 ? 4 : 2);
  const void* Xd = Xn;
  const void* Rd = R;
  void* tmp = nullptr;
  if (rc == GSQ_OK && !is_device_ptr(Xn)) { salloc(&tmp, xb); Xd = tmp; }
  if (rc == GSQ_OK && !is_device_ptr(R)) { salloc(&tmp, rb); Rd = tmp; }
  void* Wstage = nullptr;
  const bool any_host_w = !is_device_ptr(Wg) || !is_device_ptr(Wu) || !is_device_ptr(Wd);
  if (rc == GSQ_OK && any_host_w) salloc(&Wstage, wb);
  if (rc != GSQ_OK) return cleanup_fail(rc);

  cudaStream_t st = c->st;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
    return e == cudaSuccess;
  };
  if (Xd != Xn) ok(cudaMemcpyAsync(const_cast<void*>(Xd), Xn, xb, cudaMemcpyDefault, st));
  if (Rd != R) ok(cudaMemcpyAsync(const_cast<void*>(Rd), R, rb, cudaMemcpyDefault, st));
  ok(cudaMemsetAsync(c->err, 0, 16, st));
  ok(cudaMemsetAsync(c->ticket, 0, 16, st));
  ok(cudaMemsetAsync(c->loss_hist, 0, kLossRing * sizeof(double), st));
  ok(launch_convert_x(Xd, x_dtype, T, H, T, c->Xn, c->XnT, nullptr, c->err, st));
  ok(launch_transpose_to_f32(Rd, r_dtype == GSQ_BF16, T, H, c->RT, st));
  const void* Ws[3] = {Wg, Wu, Wd};
  for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
    Weight& w = c->w[i];
    const int64_t NK = w.N * w.K;
    const void* src = Ws[i];
    if (!is_device_ptr(src)) {
      ok(cudaMemcpyAsync(Wstage, src, (size_t)NK * (w_dtype == GSQ_F32 ? 4 : 2),
                         cudaMemcpyDefault, st));
      src = Wstage;
    }
    ok(cudaMemsetAsync(w.mom, 0, (size_t)c->L * NK * 4, st));
    ok(cudaMemsetAsync(w.ms, 0, (size_t)w.N * w.G * 4, st));
    ok(cudaMemsetAsync(w.dW, 0, (size_t)NK * 4, st));
    ok(launch_convert_w(src, w_dtype, w.N, w.K, W32, Wop, 0, c->err, st));
    ok(launch_init_state(grid_mode, W32, nullptr, w.N, w.K, w.s, w.i0, w.logits,
                         c->err, st));
    // the staging buffers are reused by the next weight: finish this one
    ok(cudaStreamSynchronize(st));
  }
  ok(launch_sumsq(c->RT, H * T, c->partials, c->ticket, c->scratch, st));
  if (e != cudaSuccess) return cleanup_fail(cuda_status(e));

  // tensor maps
  bool bad = false;
  for (int i = 0; i < 3; ++i) {
    Weight& w = c->w[i];
    bad |= make_tmap_bf16(&w.tmA, w.What, w.N, w.K, w.K, kGemmBoxRowsA) != 0;
    bad |= make_tmap_epi_f32(&w.em_dW.out, w.dW, w.N, w.K, w.K) != 0;
    w.em_dW.yref = w.em_dW.out;
  }
  bad |= make_tmap_bf16(&c->tmB_Xn, c->Xn, T, H, H, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_h, c->h, T, F, F, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_hT, c->hT, F, T, T, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_dp, c->dp, T, H, H, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_XnT, c->XnT, H, T, T, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmA_dpT, c->dpT, H, T, T, kGemmBoxRowsA) != 0;
  bad |= make_tmap_bf16(&c->tmA_WdT, c->WdT, F, H, H, kGemmBoxRowsA) != 0;
  bad |= make_tmap_bf16(&c->tmA_daT, c->daT, F, T, T, kGemmBoxRowsA) != 0;
  bad |= make_tmap_bf16(&c->tmA_dbT, c->dbT, F, T, T, kGemmBoxRowsA) != 0;
  bad |= make_tmap_epi_f32(&c->em_aT.out, c->aT, F, T, T) != 0;
  bad |= make_tmap_epi_f32(&c->em_bT.out, c->bT, F, T, T) != 0;
  bad |= make_tmap_epi_f32(&c->em_dhT.out, c->dhT, F, T, T) != 0;
  bad |= make_tmap_epi_bf16(&c->em_pred.out, c->dpT, H, T, T) != 0;
  bad |= make_tmap_epi_f32(&c->em_pred.yref, c->RT, H, T, T) != 0;
  c->em_aT.yref = c->em_aT.out;
  c->em_bT.yref = c->em_bT.out;
  c->em_dhT.yref = c->em_dhT.out;
  if (bad) return cleanup_fail(GSQ_ERR_CUDA);

  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cleanup_fail(cuda_status(e));
  int h = 0;
  double rsq = 0.0;
  if (cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(&rsq, c->scratch, sizeof(double), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cleanup_fail(GSQ_ERR_CUDA);
  if (h == DEV_ERR_NONFINITE) return cleanup_fail(GSQ_ERR_NONFINITE);
  if (h != DEV_OK) return cleanup_fail(GSQ_ERR_CUDA);
  c->r_sq = rsq;
  for (void* p : staging) pool_free(p);
  *out = c;
  return GSQ_OK;
}

int gsq_mlp_step(gsq_mlp* c, float tau, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  return run_step(c, tau, 0.f, lr, beta1, beta2);
}

int gsq_mlp_run(gsq_mlp* c, const float* taus, int64_t n, float lr, float beta1,
                float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!taus || n <= 0) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i)
    if (!step_args_ok(taus[i], lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int rc = run_step(c, taus[i], i + 1 < n ? taus[i + 1] : 0.f, lr, beta1, beta2);
    if (rc) return rc;
  }
  return GSQ_OK;
}

int gsq_mlp_last_loss(gsq_mlp* c, double* loss) {
  int u = usable(c);
  if (u) return u;
  if (!loss) return GSQ_ERR_INVALID_ARG;
  if (c->t == 0) return GSQ_ERR_STATE;
  int rc = check_device(c);
  if (rc) return rc;
  CKM(cudaMemcpy(loss, c->loss_hist + ((c->t - 1) % kLossRing), sizeof(double),
                 cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_mlp_recon_error(gsq_mlp* c, int mode, float tau, double* abs_err,
                        double* rel_err) {
  int u = usable(c);
  if (u) return u;
  if (!abs_err || (mode != GSQ_RECON_HARD && mode != GSQ_RECON_SOFT) ||
      (mode == GSQ_RECON_SOFT && !(tau > 0.f && std::isfinite(tau))))
    return GSQ_ERR_INVALID_ARG;
  c->what_t = -1;
  for (int i = 0; i < 3; ++i) {
    Weight& w = c->w[i];
    if (mode == GSQ_RECON_HARD) {
      CKM(launch_hard_weight(c->mode, w.N, w.K, w.logits, w.s, w.i0, w.What, c->st));
    } else {
      StepArgs a = weight_args(c, i, tau);
      a.noise = 0;
      CKM(launch_soft_weight(a, w.What, nullptr, c->sms, c->st));
    }
  }
  CKM(forward(c, c->scratch, false));
  int rc = check_device(c);
  if (rc) return rc;
  double v = 0.0;
  CKM(cudaMemcpy(&v, c->scratch, sizeof(double), cudaMemcpyDeviceToHost));
  *abs_err = v;
  if (rel_err) *rel_err = c->r_sq > 0.0 ? v / c->r_sq : 0.0;
  return GSQ_OK;
}

int gsq_mlp_harden_pack(gsq_mlp* c, int which, void* packed, uint16_t* scales_f16,
                        float* scales_f32) {
  int u = usable(c);
  if (u) return u;
  if (which < 0 || which > 2 || !packed) return GSQ_ERR_INVALID_ARG;
  Weight& w = c->w[which];
  size_t pbytes = 0;
  gsq_packed_bytes(c->mode, w.N, w.K, &pbytes);
  const int64_t ng = w.N * w.G;
  void* buf = nullptr;
  CKM(pool_malloc(&buf, pbytes + (size_t)ng * 6 + 64));
  uint32_t* pk = static_cast<uint32_t*>(buf);
  uint16_t* h16 = reinterpret_cast<uint16_t*>(static_cast<char*>(buf) + (pbytes + 15) / 16 * 16);
  float* f32 = reinterpret_cast<float*>(reinterpret_cast<char*>(h16) + ((size_t)ng * 2 + 15) / 16 * 16);
  cudaError_t e = launch_harden_pack(c->mode, w.N, w.K, w.logits, w.i0, pk, c->st);
  if (e == cudaSuccess) e = launch_export_scales(w.s, ng, h16, f32, c->st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(packed, pk, pbytes, cudaMemcpyDefault, c->st);
  if (e == cudaSuccess && scales_f16)
    e = cudaMemcpyAsync(scales_f16, h16, (size_t)ng * 2, cudaMemcpyDefault, c->st);
  if (e == cudaSuccess && scales_f32)
    e = cudaMemcpyAsync(scales_f32, f32, (size_t)ng * 4, cudaMemcpyDefault, c->st);
  cudaError_t e2 = cudaStreamSynchronize(c->st);
  pool_free(buf);
  if (e != cudaSuccess) return fail(c, cuda_status(e));
  if (e2 != cudaSuccess) return fail(c, cuda_status(e2));
  return check_device(c);
}

static int mlp_buffer(gsq_mlp* c, int which, int buf, void** p, size_t* bytes) {
  if (which >= 0 && which <= 2) {
    Weight& w = c->w[which];
    const size_t NK = (size_t)w.N * w.K, LNK = (size_t)c->L * NK, NG = (size_t)w.N * w.G;
    switch (buf) {
      case GSQ_DBG_LOGITS: *p = w.logits; *bytes = LNK * 4; return GSQ_OK;
      case GSQ_DBG_MOM: *p = w.mom; *bytes = LNK * 4; return GSQ_OK;
      case GSQ_DBG_SCALES: *p = w.s; *bytes = NG * 4; return GSQ_OK;
      case GSQ_DBG_SMOM: *p = w.ms; *bytes = NG * 4; return GSQ_OK;
      case GSQ_DBG_I0: *p = w.i0; *bytes = NK; return GSQ_OK;
      case GSQ_DBG_WHAT: *p = w.What; *bytes = NK * 2; return GSQ_OK;
      case GSQ_DBG_DW: *p = w.dW; *bytes = NK * 4; return GSQ_OK;
      default: return GSQ_ERR_INVALID_ARG;
    }
  }
  if (which != GSQ_MLP_STAGE) return GSQ_ERR_INVALID_ARG;
  const size_t FT = (size_t)c->F * c->T, HT = (size_t)c->H * c->T;
  switch (buf) {
    case GSQ_MLP_DBG_AT: *p = c->aT; *bytes = FT * 4; return GSQ_OK;
    case GSQ_MLP_DBG_BT: *p = c->bT; *bytes = FT * 4; return GSQ_OK;
    case GSQ_MLP_DBG_HT: *p = c->hT; *bytes = FT * 2; return GSQ_OK;
    case GSQ_MLP_DBG_DPT: *p = c->dpT; *bytes = HT * 2; return GSQ_OK;
    case GSQ_MLP_DBG_DHT: *p = c->dhT; *bytes = FT * 4; return GSQ_OK;
    case GSQ_MLP_DBG_DAT: *p = c->daT; *bytes = FT * 2; return GSQ_OK;
    case GSQ_MLP_DBG_DBT: *p = c->dbT; *bytes = FT * 2; return GSQ_OK;
    case GSQ_MLP_DBG_RT: *p = c->RT; *bytes = HT * 4; return GSQ_OK;
    default: return GSQ_ERR_INVALID_ARG;
  }
}

int gsq_mlp_debug_get(gsq_mlp* c, int which, int buf, void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = mlp_buffer(c, which, buf, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  rc = check_device(c);
  if (rc) return rc;
  CKM(cudaMemcpy(host, p, nb, cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_mlp_debug_set(gsq_mlp* c, int which, int buf, const void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = mlp_buffer(c, which, buf, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  CKM(cudaStreamSynchronize(c->st));
  CKM(cudaMemcpy(p, host, nb, cudaMemcpyHostToDevice));
  c->what_t = -1;
  return GSQ_OK;
}

int gsq_mlp_get_step(gsq_mlp* c, uint64_t* t) {
  if (!c || !t) return GSQ_ERR_INVALID_ARG;
  *t = c->t;
  return GSQ_OK;
}

int gsq_mlp_destroy(gsq_mlp* c) {
  if (!c) return GSQ_OK;
  cudaStreamSynchronize(c->st);
  cudaGetLastError();
  c->clock.release();
  free_all(c);
  delete c;
  return GSQ_OK;
}

int gsq_mlp_set_timing(gsq_mlp* c, int on) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  c->clock.on = on != 0;
  return GSQ_OK;
}

int gsq_mlp_phase_times(gsq_mlp* c, double* ms, int64_t* launches) {
  if (!c || !ms || !launches) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  CKM(c->clock.collect(PH_COUNT, ms, launches));
  return GSQ_OK;
}

}  // extern "C"
