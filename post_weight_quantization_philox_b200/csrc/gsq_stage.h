// gsq_stage.h -- host-side pieces shared by the block-stage contexts (MLP,
// attention V/O): the quantization state of one weight and small helpers.
#pragma once

#include <cstring>

#include "../../include/gsq.h"
#include "gsq_internal.h"

namespace gsq {

constexpr int kStageGroup = 128;
constexpr int kStageLossRing = 4096;
constexpr int kStagePartials = 1024;

// quantization state of one weight of a stage (N x K, groups along K)
struct StageWeight {
  int64_t N = 0, K = 0, G = 0;
  uint64_t seed = 0;
  float *logits = nullptr, *mom = nullptr, *s = nullptr, *ms = nullptr;
  float* dW = nullptr;
  int8_t* i0 = nullptr;
  __nv_bfloat16* What = nullptr;
  CUtensorMap tmA;  // What as GEMM operand A
  EpiMaps em_dW;    // dW as fp32 epilogue output
};

inline int stage_cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GSQ_OK;
  if (e == cudaErrorMemoryAllocation) return GSQ_ERR_OOM;
  return GSQ_ERR_CUDA;
}

inline bool stage_is_device_ptr(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

inline int stage_num_logits(int mode) {
  return mode == GSQ_GRID_3BIT_LOCAL ? 5
                                     : (mode == GSQ_GRID_2BIT || mode == GSQ_GRID_TERNARY) ? 4 : -1;
}

inline bool stage_step_args_ok(float tau, float lr, float b1, float b2) {
  return tau > 0.f && tau < 3.0e38f && lr >= 0.f && lr < 3.0e38f && b1 >= 0.f &&
         b1 < 1.f && b2 >= 0.f && b2 < 1.f;
}

inline StepArgs stage_weight_args(const StageWeight& w, int mode, uint64_t t,
                                  int noise, float tau) {
  StepArgs a;
  a.mode = mode;
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
  a.t = (uint32_t)t;
  a.noise = noise;
  a.tau = tau;
  return a;
}

// buffer of a stage weight for the debug accessors (GSQ_DBG_* codes)
inline int stage_weight_buffer(const StageWeight& w, int L, int buf, void** p,
                               size_t* bytes) {
  const size_t NK = (size_t)w.N * w.K, LNK = (size_t)L * NK, NG = (size_t)w.N * w.G;
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

}  // namespace gsq
