// gsq_gemm_epi.cuh -- small pieces of the GEMM epilogue: bf16 packing and
// the deterministic cross-CTA loss reduction.
#pragma once

#include "gsq_device.cuh"
#include "gsq_internal.h"

namespace gsq {

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Deterministic loss: the CTA's partial in a fixed slot; the last CTA to
// finish adds all partials in slot order and resets the ticket.  Called by
// one thread per CTA.
__device__ __forceinline__ void loss_finish(double cta, const EpiParams& ep) {
  ep.partials[blockIdx.x] = cta;
  __threadfence();
  const unsigned tk = atomicAdd(ep.ticket, 1u);
  if (tk == gridDim.x - 1) {
    __threadfence();
    double tot = 0.0;
    for (unsigned b = 0; b < gridDim.x; ++b) tot += *((volatile double*)ep.partials + b);
    *ep.loss_out = tot;
    if (!isfinite(tot)) atomicCAS(ep.err, 0, DEV_ERR_NONFINITE);
    *ep.ticket = 0u;
  }
}

}  // namespace gsq
