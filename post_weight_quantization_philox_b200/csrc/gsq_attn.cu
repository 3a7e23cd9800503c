// gsq_attn.cu -- the block's attention V/O stage: the value and output
// projections quantized jointly while the attention probabilities, built from
// the frozen (already quantized) query and key projections, stay fixed (GSQ
// staging, agihunt.info summary, optimisation paragraph: Q and K first, then
// V and O jointly).
//
// Once, at init (per sequence s and head h, group g = h / grp):
//   Q = Xa Wq^T, K = Xa Wk^T (fp32), rotary embedding -> bf16,
//   scores = Q_(s,h) K_(s,g)^T, P_(s,h) = causal softmax(scores / sqrt(d)),
//   kept as bf16 in two layouts: P[s][h][q][key] and
//   P^T[s][g][key][hig][q] (hig = h - g grp), i.e. one K-major operand per
//   (s, g) for the value gradient.
// Per step t (CTA-pair tcgen05 GEMMs, all A . B^T with K-major operands):
//   V^T = bf16(Wv Xa^T)                               (Hk x T)
//   o_(s,g-heads) = bf16(P_(s, g's heads) . V_(s,g))   (grp S x d per (s, g),
//                   written straight into o, T x H)
//   pred^T = Wo o^T; E = pred^T - R^T; loss; dp^T = bf16(2E)
//   dWo = dp^T . o ;  do^T = bf16(Wo^T dp^T)           (H x T)
//   dV_(s,g) = bf16(P^T_(s,g) . do_(s, g's heads))     (S x d, K = grp S: one
//              K segment per head, read from do^T in place)
//   dWv = dV^T . Xa ; backward + Lion for Wv and Wo.
// The per-(s, g) products run as one batched launch each, on 256 x 128
// tiles (N = d = 128).  When S is a multiple of 256 they skip the zero half
// of the causal P: o tiles of queries [q0, q0 + 256) contract over keys
// [0, q0 + 256) only, dV tiles of keys [k0, k0 + 256) over queries [k0, S) of
// each head.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "gsq_stage.h"

using namespace gsq;

struct gsq_attn {
  int mode = 0, L = 0;
  PhaseClock clock;  // per-phase device time (gsq_attn_set_timing)
  int64_t nseq = 0, S = 0, nh = 0, nkv = 0, d = 0, grp = 0, T = 0, H = 0, Hk = 0;
  uint64_t t = 0;
  int noise = 1;
  cudaStream_t st = nullptr;
  int sms = 148;
  int failed = 0;
  StageWeight w[2];  // value (Hk x H), output (H x H)
  __nv_bfloat16 *Xa = nullptr, *XaT = nullptr, *P = nullptr, *PT = nullptr;
  __nv_bfloat16 *VT = nullptr, *o = nullptr, *oT = nullptr, *dpT = nullptr, *dp = nullptr;
  __nv_bfloat16 *WoT = nullptr, *doT = nullptr, *dVb = nullptr, *dVT = nullptr;
  float* RT = nullptr;
  double *partials = nullptr, *loss_hist = nullptr, *scratch = nullptr;
  unsigned* ticket = nullptr;
  int* err = nullptr;
  double r_sq = 0.0;
  int64_t what_t = -1;
  float what_tau = 0.f;
  CUtensorMap tmB_Xa, tmB_o, tmB_oT, tmB_dp, tmB_XaT, tmA_dpT, tmA_WoT, tmA_dVT;
  EpiMaps em_VT, em_pred, em_doT;
  // all (s, g) problems of a step in one launch each (GemmSched)
  CUtensorMap tmA_P, tmB_VT, tm_o, tmA_PT, tmB_doT, tm_dV;
  GemmSched sc_pv, sc_dv;
  std::vector<void*> allocs;
};

namespace {

int fail(gsq_attn* c, int status) {
  if (c && status != GSQ_OK && c->failed == 0) c->failed = status;
  return status;
}

#define CKA(call)                                                 \
  do {                                                            \
    cudaError_t e_ = (call);                                      \
    if (e_ != cudaSuccess) return fail(c, stage_cuda_status(e_)); \
  } while (0)

template <typename T>
int alloc(gsq_attn* c, T** p, size_t count) {
  void* q = nullptr;
  if (pool_malloc(&q, count * sizeof(T) + 16) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_OOM;
  }
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return GSQ_OK;
}

void free_all(gsq_attn* c) {
  for (void* p : c->allocs) pool_free(p);
  c->allocs.clear();
}

int usable(gsq_attn* c) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  return GSQ_OK;
}

int check_device(gsq_attn* c) {
  cudaError_t e = cudaStreamSynchronize(c->st);
  if (e != cudaSuccess) return fail(c, stage_cuda_status(e));
  int h = 0;
  e = cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(c, stage_cuda_status(e));
  switch (h) {
    case DEV_OK: return GSQ_OK;
    case DEV_ERR_TIMEOUT: return fail(c, GSQ_ERR_TIMEOUT);
    case DEV_ERR_NONFINITE: return fail(c, GSQ_ERR_NONFINITE);
    default: return fail(c, GSQ_ERR_CUDA);
  }
}

EpiParams epi(gsq_attn* c, double* loss_out) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.partials = c->partials;
  ep.ticket = c->ticket;
  ep.loss_out = loss_out;
  ep.err = c->err;
  return ep;
}

EpiMaps out_only(const CUtensorMap& m) {
  EpiMaps e;
  e.out = m;
  e.yref = m;
  return e;
}

// forward from the weights in w[i].What: V, attention outputs, o, o^T and
// pred^T with the loss (and dp^T when with_dp) into *loss_out
cudaError_t forward(gsq_attn* c, double* loss_out, bool with_dp) {
  const int64_t T = c->T, H = c->H, Hk = c->Hk, S = c->S;
  cudaError_t e;
  EpiParams ep = epi(c, loss_out);
  PhaseClock& k = c->clock;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  if ((e = launch_gemm(c->w[0].tmA, c->tmB_Xa, c->em_VT, Hk, T, H, EPI_STORE_BF16, ep,
                       c->sms, c->st)) != cudaSuccess) return e;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  if ((e = launch_gemm_batched(c->tmA_P, c->tmB_VT, c->tm_o, c->grp * S, c->d, S, 128,
                               c->sc_pv, EPI_STORE_BF16, ep, c->sms, c->st)) != cudaSuccess)
    return e;
  if ((e = k.mark(c->st, PH_ELEM)) != cudaSuccess) return e;
  if ((e = launch_transpose_bf16(c->o, T, H, c->oT, c->st)) != cudaSuccess) return e;
  if ((e = k.mark(c->st, PH_GEMM)) != cudaSuccess) return e;
  return launch_gemm(c->w[1].tmA, c->tmB_o, c->em_pred, H, T, H,
                     with_dp ? EPI_LOSS_DY : EPI_LOSS, ep, c->sms, c->st);
}

int run_step(gsq_attn* c, float tau, float tau_next, float lr, float b1, float b2) {
  if (c->t >= 0xFFFFFFFEull) return GSQ_ERR_UNSUPPORTED;
  NvtxRange step_range("gsq_attn_step");
  const int64_t T = c->T, H = c->H, Hk = c->Hk, S = c->S;
  PhaseClock& k = c->clock;
  if (!(c->what_t == (int64_t)c->t && c->what_tau == tau))
    for (int i = 0; i < 2; ++i) {
      CKA(k.mark(c->st, PH_SOFT));
      CKA(launch_soft_weight(stage_weight_args(c->w[i], c->mode, c->t, c->noise, tau),
                             c->w[i].What, nullptr, c->sms, c->st));
    }
  CKA(forward(c, c->loss_hist + (c->t % kStageLossRing), true));
  EpiParams ep = epi(c, nullptr);
  // dWo = dp^T . o
  CKA(k.mark(c->st, PH_GEMM));
  CKA(launch_gemm(c->tmA_dpT, c->tmB_oT, c->w[1].em_dW, H, H, T, EPI_STORE_F32, ep,
                  c->sms, c->st));
  // do^T = Wo^T . dp^T
  CKA(k.mark(c->st, PH_ELEM));
  CKA(launch_transpose_bf16(c->w[1].What, H, H, c->WoT, c->st));
  CKA(k.mark(c->st, PH_ELEM));
  CKA(launch_transpose_bf16(c->dpT, H, T, c->dp, c->st));
  CKA(k.mark(c->st, PH_GEMM));
  CKA(launch_gemm(c->tmA_WoT, c->tmB_dp, c->em_doT, H, T, H, EPI_STORE_BF16, ep, c->sms,
                  c->st));
  // dV_(s,g) = P^T_(s,g) . do_(s, g's heads)
  CKA(k.mark(c->st, PH_GEMM));
  CKA(launch_gemm_batched(c->tmA_PT, c->tmB_doT, c->tm_dV, S, c->d, c->grp * S, 128,
                          c->sc_dv, EPI_STORE_BF16, ep, c->sms, c->st));
  // dWv = dV^T . Xa
  CKA(k.mark(c->st, PH_ELEM));
  CKA(launch_transpose_bf16(c->dVb, T, Hk, c->dVT, c->st));
  CKA(k.mark(c->st, PH_GEMM));
  CKA(launch_gemm(c->tmA_dVT, c->tmB_XaT, c->w[0].em_dW, Hk, H, T, EPI_STORE_F32, ep,
                  c->sms, c->st));
  for (int i = 0; i < 2; ++i) {
    CKA(k.mark(c->st, PH_BACKWARD));
    CKA(launch_backward_lion(stage_weight_args(c->w[i], c->mode, c->t, c->noise, tau),
                             c->w[i].dW, lr, b1, b2, tau_next,
                             c->w[i].What, nullptr, nullptr, c->sms, c->st));
  }
  CKA(k.mark(c->st, -1));
  c->t += 1;
  if (tau_next > 0.f) {
    c->what_t = (int64_t)c->t;
    c->what_tau = tau_next;
  } else {
    c->what_t = -1;
  }
  return GSQ_OK;
}

int attn_buffer(gsq_attn* c, int which, int buf, void** p, size_t* bytes) {
  if (which == 0 || which == 1) return stage_weight_buffer(c->w[which], c->L, buf, p, bytes);
  if (which != GSQ_ATTN_STAGE) return GSQ_ERR_INVALID_ARG;
  const size_t PS = (size_t)c->nseq * c->nh * c->S * c->S;
  const size_t TH = (size_t)c->T * c->H, TK = (size_t)c->T * c->Hk;
  switch (buf) {
    case GSQ_ATTN_DBG_P: *p = c->P; *bytes = PS * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_PT: *p = c->PT; *bytes = PS * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_VT: *p = c->VT; *bytes = TK * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_O: *p = c->o; *bytes = TH * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_DPT: *p = c->dpT; *bytes = TH * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_DV: *p = c->dVb; *bytes = TK * 2; return GSQ_OK;
    case GSQ_ATTN_DBG_RT: *p = c->RT; *bytes = TH * 4; return GSQ_OK;
    default: return GSQ_ERR_INVALID_ARG;
  }
}

}  // namespace

extern "C" {

int gsq_attn_init(gsq_attn** out, const void* Xa, int x_dtype, const void* R,
                  int r_dtype, const void* Wq, const void* Wk, const void* Wv,
                  const void* Wo, int w_dtype, int64_t n_seq, int64_t seq_len,
                  int64_t n_heads, int64_t n_kv_heads, int64_t head_dim,
                  double rope_theta, int group, int grid_mode, uint64_t seed,
                  void* stream) {
  if (!out) return GSQ_ERR_INVALID_ARG;
  *out = nullptr;
  auto dt_ok = [](int dt) { return dt == GSQ_F32 || dt == GSQ_BF16; };
  if (!Xa || !R || !Wq || !Wk || !Wv || !Wo || !dt_ok(x_dtype) || !dt_ok(r_dtype) ||
      !dt_ok(w_dtype) || n_seq <= 0 || seq_len <= 0 || n_heads <= 0 ||
      n_kv_heads <= 0 || n_heads % n_kv_heads != 0 || stage_num_logits(grid_mode) < 0 ||
      group <= 0 || !(rope_theta > 0.0) || n_seq * seq_len > (int64_t)1 << 31)
    return GSQ_ERR_INVALID_ARG;
  if (group != kStageGroup || head_dim != 128 || seq_len % 128 != 0 || seq_len > 65536)
    return GSQ_ERR_UNSUPPORTED;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  gsq_attn* c = new (std::nothrow) gsq_attn();
  if (!c) return GSQ_ERR_OOM;
  c->mode = grid_mode;
  c->L = stage_num_logits(grid_mode);
  c->nseq = n_seq;
  c->S = seq_len;
  c->nh = n_heads;
  c->nkv = n_kv_heads;
  c->d = head_dim;
  c->grp = n_heads / n_kv_heads;
  c->T = n_seq * seq_len;
  c->H = n_heads * head_dim;
  c->Hk = n_kv_heads * head_dim;
  c->st = static_cast<cudaStream_t>(stream);
  c->sms = prop.multiProcessorCount;
  const int64_t T = c->T, H = c->H, Hk = c->Hk, S = c->S, grp = c->grp, d = c->d;
  const int64_t PS = c->nseq * c->nh * S * S;
  const int64_t dims[2][2] = {{Hk, H}, {H, H}};
  int rc = GSQ_OK;
#define ALA(p, n) \
  if (rc == GSQ_OK) rc = alloc(c, &(p), (size_t)(n))
  for (int i = 0; i < 2; ++i) {
    StageWeight& w = c->w[i];
    w.N = dims[i][0];
    w.K = dims[i][1];
    w.G = w.K / kStageGroup;
    w.seed = seed ^ ((uint64_t)i << 48);  // own Philox key per weight
    const int64_t NK = w.N * w.K;
    ALA(w.logits, c->L * NK);
    ALA(w.mom, c->L * NK);
    ALA(w.s, w.N * w.G);
    ALA(w.ms, w.N * w.G);
    ALA(w.i0, NK);
    ALA(w.What, NK);
    ALA(w.dW, NK);
  }
  ALA(c->Xa, T * H);
  ALA(c->XaT, H * T);
  ALA(c->RT, H * T);
  ALA(c->P, PS);
  ALA(c->PT, PS);
  ALA(c->VT, Hk * T);
  ALA(c->o, T * H);
  ALA(c->oT, H * T);
  ALA(c->dpT, H * T);
  ALA(c->dp, T * H);
  ALA(c->WoT, H * H);
  ALA(c->doT, H * T);
  ALA(c->dVb, T * Hk);
  ALA(c->dVT, Hk * T);
  ALA(c->partials, kStagePartials);
  ALA(c->loss_hist, kStageLossRing);
  ALA(c->scratch, 4);
  ALA(c->ticket, 4);
  ALA(c->err, 4);
#undef ALA
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
  // init-only buffers
  float *W32 = nullptr, *Q32 = nullptr, *K32 = nullptr, *scores = nullptr;
  __nv_bfloat16 *Wqb = nullptr, *Wkb = nullptr, *Qr = nullptr, *Kr = nullptr, *Wop = nullptr;
  salloc((void**)&W32, (size_t)H * H * 4);
  salloc((void**)&Wop, (size_t)H * H * 2);
  salloc((void**)&Wqb, (size_t)H * H * 2);
  salloc((void**)&Wkb, (size_t)Hk * H * 2);
  salloc((void**)&Q32, (size_t)T * H * 4);
  salloc((void**)&K32, (size_t)T * Hk * 4);
  salloc((void**)&Qr, (size_t)T * H * 2);
  salloc((void**)&Kr, (size_t)T * Hk * 2);
  salloc((void**)&scores, (size_t)S * S * 4);
  const size_t es_x = x_dtype == GSQ_F32 ? 4 : 2, es_r = r_dtype == GSQ_F32 ? 4 : 2;
  const size_t es_w = w_dtype == GSQ_F32 ? 4 : 2;
  const void* Xd = Xa;
  const void* Rd = R;
  void* tmp = nullptr;
  if (rc == GSQ_OK && !stage_is_device_ptr(Xa)) { salloc(&tmp, (size_t)T * H * es_x); Xd = tmp; }
  if (rc == GSQ_OK && !stage_is_device_ptr(R)) { salloc(&tmp, (size_t)T * H * es_r); Rd = tmp; }
  void* Wstage = nullptr;
  salloc(&Wstage, (size_t)H * H * es_w);
  if (rc != GSQ_OK) return cleanup_fail(rc);

  cudaStream_t st = c->st;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
    return e == cudaSuccess;
  };
  if (Xd != Xa) ok(cudaMemcpyAsync(const_cast<void*>(Xd), Xa, (size_t)T * H * es_x, cudaMemcpyDefault, st));
  if (Rd != R) ok(cudaMemcpyAsync(const_cast<void*>(Rd), R, (size_t)T * H * es_r, cudaMemcpyDefault, st));
  ok(cudaMemsetAsync(c->err, 0, 16, st));
  ok(cudaMemsetAsync(c->ticket, 0, 16, st));
  ok(cudaMemsetAsync(c->loss_hist, 0, kStageLossRing * sizeof(double), st));
  ok(launch_convert_x(Xd, x_dtype, T, H, T, c->Xa, c->XaT, nullptr, c->err, st));
  ok(launch_transpose_to_f32(Rd, r_dtype == GSQ_BF16, T, H, c->RT, st));
  // bf16 copies of the frozen query / key weights; quantization state of V, O
  auto to_dev = [&](const void* src, int64_t n) -> const void* {
    if (stage_is_device_ptr(src)) return src;
    ok(cudaMemcpyAsync(Wstage, src, (size_t)n * es_w, cudaMemcpyDefault, st));
    return Wstage;
  };
  ok(launch_convert_w(to_dev(Wq, H * H), w_dtype, H, H, W32, Wqb, 0, c->err, st));
  ok(cudaStreamSynchronize(st));
  ok(launch_convert_w(to_dev(Wk, Hk * H), w_dtype, Hk, H, W32, Wkb, 0, c->err, st));
  ok(cudaStreamSynchronize(st));
  const void* Wvo[2] = {Wv, Wo};
  for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
    StageWeight& w = c->w[i];
    const int64_t NK = w.N * w.K;
    ok(cudaMemsetAsync(w.mom, 0, (size_t)c->L * NK * 4, st));
    ok(cudaMemsetAsync(w.ms, 0, (size_t)w.N * w.G * 4, st));
    ok(cudaMemsetAsync(w.dW, 0, (size_t)NK * 4, st));
    ok(launch_convert_w(to_dev(Wvo[i], NK), w_dtype, w.N, w.K, W32, Wop, 0, c->err, st));
    ok(launch_init_state(grid_mode, W32, nullptr, w.N, w.K, w.s, w.i0, w.logits, c->err, st));
    ok(cudaStreamSynchronize(st));
  }
  ok(launch_sumsq(c->RT, H * T, c->partials, c->ticket, c->scratch, st));
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));

  // persistent tensor maps
  bool bad = false;
  for (int i = 0; i < 2; ++i) {
    StageWeight& w = c->w[i];
    bad |= make_tmap_bf16(&w.tmA, w.What, w.N, w.K, w.K, kGemmBoxRowsA) != 0;
    CUtensorMap m;
    bad |= make_tmap_epi_f32(&m, w.dW, w.N, w.K, w.K) != 0;
    w.em_dW = out_only(m);
  }
  bad |= make_tmap_bf16(&c->tmB_Xa, c->Xa, T, H, H, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_o, c->o, T, H, H, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_oT, c->oT, H, T, T, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_dp, c->dp, T, H, H, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmB_XaT, c->XaT, H, T, T, kGemmBoxRowsB) != 0;
  bad |= make_tmap_bf16(&c->tmA_dpT, c->dpT, H, T, T, kGemmBoxRowsA) != 0;
  bad |= make_tmap_bf16(&c->tmA_WoT, c->WoT, H, H, H, kGemmBoxRowsA) != 0;
  bad |= make_tmap_bf16(&c->tmA_dVT, c->dVT, Hk, T, T, kGemmBoxRowsA) != 0;
  {
    CUtensorMap m;
    bad |= make_tmap_epi_bf16(&m, c->VT, Hk, T, T) != 0;
    c->em_VT = out_only(m);
    bad |= make_tmap_epi_bf16(&m, c->doT, H, T, T) != 0;
    c->em_doT = out_only(m);
    bad |= make_tmap_epi_bf16(&c->em_pred.out, c->dpT, H, T, T) != 0;
    bad |= make_tmap_epi_f32(&c->em_pred.yref, c->RT, H, T, T) != 0;
  }
  {
    // P as (nseq nh S) x S: problem (s, g) is the grp S rows of g's heads
    bad |= make_tmap_bf16(&c->tmA_P, c->P, c->nseq * c->nh * S, S, S, kGemmBoxRowsA) != 0;
    // V^T (Hk x T): problem (s, g) is rows g d.., columns s S..
    bad |= make_tmap_bf16(&c->tmB_VT, c->VT, Hk, T, T, kGemmBoxRowsBNarrow) != 0;
    // o (T x H): problem (s, g) rows (hig, q) land at row s S + q, columns
    // (g grp + hig) d..
    bad |= make_tmap_epi_bf16(&c->tm_o, c->o, T, H, H) != 0;
    // P^T as (nseq nkv S) x (grp S)
    bad |= make_tmap_bf16(&c->tmA_PT, c->PT, c->nseq * c->nkv * S, grp * S, grp * S,
                          kGemmBoxRowsA) != 0;
    // do^T (H x T): K segment hig of problem (s, g) is rows (g grp + hig) d..,
    // columns s S..
    bad |= make_tmap_bf16(&c->tmB_doT, c->doT, H, T, T, kGemmBoxRowsBNarrow) != 0;
    // dV (T x Hk): problem (s, g) is rows s S.., columns g d..
    bad |= make_tmap_epi_bf16(&c->tm_dV, c->dVb, T, Hk, Hk) != 0;
    // problem p = s nkv + g; causal K ranges when a period holds whole tiles
    const bool causal = S % 256 == 0;
    GemmSched& a = c->sc_pv;
    a.count = (int)(c->nseq * c->nkv);
    a.inner = (int)c->nkv;
    a.a_row[0] = c->nh * S;
    a.a_row[1] = grp * S;
    a.b_row[1] = d;
    a.b_k[0] = S;
    a.o_row[0] = S;
    a.o_col[1] = grp * d;
    a.o_fold = S;
    a.o_fold_col = d;
    a.causal = causal ? 1 : 0;
    a.seg = S;
    GemmSched& b = c->sc_dv;
    b.count = (int)(c->nseq * c->nkv);
    b.inner = (int)c->nkv;
    b.a_row[0] = c->nkv * S;
    b.a_row[1] = S;
    b.b_row[1] = grp * d;
    b.b_k[0] = S;
    b.o_row[0] = S;
    b.o_col[1] = d;
    b.causal = causal ? 2 : 0;
    b.seg = S;
    b.nseg = (int)grp;
    b.a_seg_k = S;
    b.b_seg_row = d;
  }
  if (bad) return cleanup_fail(GSQ_ERR_CUDA);

  // attention probabilities from the frozen Q and K projections
  {
    EpiParams ep = epi(c, nullptr);
    CUtensorMap ta, tb, tc;
    bad |= make_tmap_bf16(&ta, c->Xa, T, H, H, kGemmBoxRowsA) != 0;
    bad |= make_tmap_bf16(&tb, Wqb, H, H, H, kGemmBoxRowsB) != 0;
    bad |= make_tmap_epi_f32(&tc, Q32, T, H, H) != 0;
    if (bad) return cleanup_fail(GSQ_ERR_CUDA);
    ok(launch_gemm(ta, tb, out_only(tc), T, H, H, EPI_STORE_F32, ep, c->sms, st));
    bad |= make_tmap_bf16(&tb, Wkb, Hk, H, H, kGemmBoxRowsB) != 0;
    bad |= make_tmap_epi_f32(&tc, K32, T, Hk, Hk) != 0;
    if (bad) return cleanup_fail(GSQ_ERR_CUDA);
    ok(launch_gemm(ta, tb, out_only(tc), T, Hk, H, EPI_STORE_F32, ep, c->sms, st));
    ok(launch_rope(Q32, T, H, S, (int)d, rope_theta, Qr, c->sms, st));
    ok(launch_rope(K32, T, Hk, S, (int)d, rope_theta, Kr, c->sms, st));
    const float scale = (float)(1.0 / std::sqrt((double)d));
    for (int64_t s = 0; s < c->nseq && e == cudaSuccess; ++s)
      for (int64_t h = 0; h < c->nh && e == cudaSuccess; ++h) {
        const int64_t g = h / grp, hig = h % grp;
        bad |= make_tmap_bf16(&ta, Qr + s * S * H + h * d, S, d, H, kGemmBoxRowsA) != 0;
        bad |= make_tmap_bf16(&tb, Kr + s * S * Hk + g * d, S, d, Hk, kGemmBoxRowsB) != 0;
        bad |= make_tmap_epi_f32(&tc, scores, S, S, S) != 0;
        if (bad) return cleanup_fail(GSQ_ERR_CUDA);
        ok(launch_gemm(ta, tb, out_only(tc), S, S, d, EPI_STORE_F32, ep, c->sms, st));
        __nv_bfloat16* Ph = c->P + (s * c->nh + h) * S * S;
        ok(launch_causal_softmax(scores, S, scale, Ph, st));
        ok(launch_transpose_ld(Ph, S, S, S, c->PT + (s * c->nkv + g) * S * grp * S + hig * S,
                               grp * S, st));
      }
  }
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));
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

int gsq_attn_step(gsq_attn* c, float tau, float lr, float beta1, float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!stage_step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  return run_step(c, tau, 0.f, lr, beta1, beta2);
}

int gsq_attn_run(gsq_attn* c, const float* taus, int64_t n, float lr, float beta1,
                 float beta2) {
  int u = usable(c);
  if (u) return u;
  if (!taus || n <= 0) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i)
    if (!stage_step_args_ok(taus[i], lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int rc = run_step(c, taus[i], i + 1 < n ? taus[i + 1] : 0.f, lr, beta1, beta2);
    if (rc) return rc;
  }
  return GSQ_OK;
}

int gsq_attn_last_loss(gsq_attn* c, double* loss) {
  int u = usable(c);
  if (u) return u;
  if (!loss) return GSQ_ERR_INVALID_ARG;
  if (c->t == 0) return GSQ_ERR_STATE;
  int rc = check_device(c);
  if (rc) return rc;
  CKA(cudaMemcpy(loss, c->loss_hist + ((c->t - 1) % kStageLossRing), sizeof(double),
                 cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_attn_recon_error(gsq_attn* c, int mode, float tau, double* abs_err,
                         double* rel_err) {
  int u = usable(c);
  if (u) return u;
  if (!abs_err || (mode != GSQ_RECON_HARD && mode != GSQ_RECON_SOFT) ||
      (mode == GSQ_RECON_SOFT && !(tau > 0.f && std::isfinite(tau))))
    return GSQ_ERR_INVALID_ARG;
  c->what_t = -1;
  for (int i = 0; i < 2; ++i) {
    StageWeight& w = c->w[i];
    if (mode == GSQ_RECON_HARD) {
      CKA(launch_hard_weight(c->mode, w.N, w.K, w.logits, w.s, w.i0, w.What, c->st));
    } else {
      StepArgs a = stage_weight_args(w, c->mode, c->t, 0, tau);
      CKA(launch_soft_weight(a, w.What, nullptr, c->sms, c->st));
    }
  }
  CKA(forward(c, c->scratch, false));
  int rc = check_device(c);
  if (rc) return rc;
  double v = 0.0;
  CKA(cudaMemcpy(&v, c->scratch, sizeof(double), cudaMemcpyDeviceToHost));
  *abs_err = v;
  if (rel_err) *rel_err = c->r_sq > 0.0 ? v / c->r_sq : 0.0;
  return GSQ_OK;
}

int gsq_attn_harden_pack(gsq_attn* c, int which, void* packed, uint16_t* scales_f16,
                         float* scales_f32) {
  int u = usable(c);
  if (u) return u;
  if (which < 0 || which > 1 || !packed) return GSQ_ERR_INVALID_ARG;
  StageWeight& w = c->w[which];
  size_t pbytes = 0;
  gsq_packed_bytes(c->mode, w.N, w.K, &pbytes);
  const int64_t ng = w.N * w.G;
  void* buf = nullptr;
  CKA(pool_malloc(&buf, pbytes + (size_t)ng * 6 + 64));
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
  if (e != cudaSuccess) return fail(c, stage_cuda_status(e));
  if (e2 != cudaSuccess) return fail(c, stage_cuda_status(e2));
  return check_device(c);
}

int gsq_attn_debug_get(gsq_attn* c, int which, int buf, void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = attn_buffer(c, which, buf, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  rc = check_device(c);
  if (rc) return rc;
  CKA(cudaMemcpy(host, p, nb, cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_attn_debug_set(gsq_attn* c, int which, int buf, const void* host, size_t bytes) {
  int u = usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t nb = 0;
  int rc = attn_buffer(c, which, buf, &p, &nb);
  if (rc) return rc;
  if (!host || bytes != nb) return GSQ_ERR_INVALID_ARG;
  CKA(cudaStreamSynchronize(c->st));
  CKA(cudaMemcpy(p, host, nb, cudaMemcpyHostToDevice));
  c->what_t = -1;
  return GSQ_OK;
}

int gsq_attn_get_step(gsq_attn* c, uint64_t* t) {
  if (!c || !t) return GSQ_ERR_INVALID_ARG;
  *t = c->t;
  return GSQ_OK;
}

int gsq_attn_destroy(gsq_attn* c) {
  if (!c) return GSQ_OK;
  cudaStreamSynchronize(c->st);
  cudaGetLastError();
  free_all(c);
  c->clock.release();
  delete c;
  return GSQ_OK;
}

int gsq_attn_set_timing(gsq_attn* c, int on) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  c->clock.on = on != 0;
  return GSQ_OK;
}

int gsq_attn_phase_times(gsq_attn* c, double* ms, int64_t* launches) {
  if (!c || !ms || !launches) return GSQ_ERR_INVALID_ARG;
  if (c->failed) return GSQ_ERR_STATE;
  CKA(c->clock.collect(PH_COUNT, ms, launches));
  return GSQ_OK;
}

}  // extern "C"
