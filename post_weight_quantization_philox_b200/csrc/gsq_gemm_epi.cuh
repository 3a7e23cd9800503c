// gsq_gemm_epi.cuh -- epilogue of one 32-column chunk of a GEMM output row,
// shared by the single-CTA and the CTA-pair GEMM kernels.
#pragma once

#include "gsq_device.cuh"
#include "gsq_internal.h"

namespace gsq {

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// v: accumulator row `row`, columns col0 .. col0+31 (fp32 bit patterns).
//   EPI_STORE_F32  C[row, col] = v (bounds-checked for ragged N)
//   EPI_LOSS(_DY)  E = v - Yref[row, col]; part += sum E^2;
//                  (_DY) dY[row, col] = bf16(2E).  N is a multiple of 64 for
//                  these modes, so chunks are whole.
template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&v)[32],
                                               int64_t row, int64_t col0,
                                               int64_t M, int64_t N,
                                               const EpiParams& ep,
                                               float& part) {
  if (row >= M || col0 >= N) return;
  if (EPI == EPI_STORE_F32) {
    float* dst = ep.out + row * ep.ldo + col0;
    if (col0 + 32 <= N && (ep.ldo & 3) == 0) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4*>(dst)[j] =
            make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                        __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < N) dst[j] = __uint_as_float(v[j]);
    }
  } else {
    const float4* yr = reinterpret_cast<const float4*>(ep.yref + row * ep.ldy + col0);
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 y4 = __ldg(yr + j);
      const float e0 = __uint_as_float(v[4 * j]) - y4.x;
      const float e1 = __uint_as_float(v[4 * j + 1]) - y4.y;
      const float e2 = __uint_as_float(v[4 * j + 2]) - y4.z;
      const float e3 = __uint_as_float(v[4 * j + 3]) - y4.w;
      part = fmaf(e0, e0, part);
      part = fmaf(e1, e1, part);
      part = fmaf(e2, e2, part);
      part = fmaf(e3, e3, part);
      pk[2 * j] = pack_bf16x2(2.f * e0, 2.f * e1);
      pk[2 * j + 1] = pack_bf16x2(2.f * e2, 2.f * e3);
    }
    if (EPI == EPI_LOSS_DY) {
      uint4* dst = reinterpret_cast<uint4*>(ep.dy + row * ep.lddy + col0);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
    }
  }
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
