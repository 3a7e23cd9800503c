// gsq_kquant.cu -- GSQ on GGUF K-Quant formats: start from a K-Quant (a
// released checkpoint's blocks, or a min-max K-Quant of W), optimise the
// per-coordinate assignment and the per-sub-block parameters with the GSQ
// step, and project the result back into the same format (agihunt.info
// summary, optimisation and results paragraphs: Q2_K / Q3_K_M, format
// unchanged).
//
// Formats: 256-weight super-blocks of 16 sub-blocks of 16 consecutive
// weights of a row.
//   Q2_K  w = d sc_j q - dmin m_j,  q 0..3, sc_j and m_j 4-bit, d, dmin fp16
//   Q3_K  w = d sc_j q,  q -4..3, sc_j 6-bit signed, d fp16
// Block bytes (the GGUF encodings of these two types):
//   Q2_K  [0,16) sc_j | m_j << 4, [16,80) 2-bit codes, [80,82) d, [82,84) dmin
//   Q3_K  [0,32) high code bits, [32,96) low 2 code bits, [96,108) 6-bit
//         scales, [108,110) d
//   a 2-bit field of weight i = 128 h + 32 s + r lives in code byte 32 h + r
//   at bit 2 s; the Q3_K high bit of weight i in byte i % 32 at bit i / 32;
//   the Q3_K scale u_j = sc_j + 32 has its low 4 bits in byte j % 8 at bit
//   4 (j / 8) and its high 2 bits in byte 8 + j % 4 at bit 2 (j / 4).
// One warp per super-block for the block codecs: lane r owns the eight
// weights 128 h + 32 s + r, i.e. exactly the code bytes 32 h + r (and Q3_K
// high-bit byte r).
//
// GSQ on the format: logits over q (Q2_K: 4, the full grid; Q3_K: 5 shifts
// -2..+2 around the start code, clamped to [-4, 3]); soft weight
// w = a_j sum_k y_k c_k - b_j with a_j, b_j continuous and trained by Lion
// beside the logits (starting at d sc_j, dmin m_j); Gumbel noise and the
// tempered softmax exactly as the 2-bit (Q2_K) and 3-bit local (Q3_K) grids
// draw and form them (the same counters and the same function), drawn again
// in the backward instead of kept between the soft weight and the backward.
// Projection back: hard codes by argmax, a_j and b_j re-encoded as the start
// encodes them.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "gsq_device.cuh"
#include "gsq_stage.h"

using namespace gsq;

namespace {

constexpr int KQ_Q2 = GSQ_KQ_Q2_K, KQ_Q3 = GSQ_KQ_Q3_K;
constexpr int kSub = 16, kSuper = 256;

template <int F>
struct KqT {
  static constexpr int L = F == KQ_Q2 ? 4 : 5;
  static constexpr int BYTES = F == KQ_Q2 ? 84 : 110;
  static constexpr int QMIN = F == KQ_Q2 ? 0 : -4;
  static constexpr int QMAX = 3;
};

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ uint16_t float_to_half_bits(float x) {
  return __half_as_ushort(__float2half_rn(x));
}

// Sub-block codes of the format from continuous a[16] (and b[16]) -- the
// same in every lane: (sc, m) codes, fp16 d, dmin (as fp32 values).
template <int F>
__device__ __forceinline__ void kq_project(const float* a_in, const float* b_in, int* sc,
                                           int* m, float& d, float& dmin) {
  if (F == KQ_Q2) {
    float a[16], b[16], amax = 0.f, bmax = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      a[j] = fmaxf(a_in[j], 0.f);
      b[j] = fmaxf(b_in[j], 0.f);
      amax = fmaxf(amax, a[j]);
      bmax = fmaxf(bmax, b[j]);
    }
    d = __half2float(__float2half_rn(__fdiv_rn(amax, 15.f)));
    dmin = __half2float(__float2half_rn(__fdiv_rn(bmax, 15.f)));
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      sc[j] = d > 0.f ? (int)fminf(fmaxf(rintf(__fdiv_rn(a[j], d)), 0.f), 15.f) : 0;
      m[j] = dmin > 0.f ? (int)fminf(fmaxf(rintf(__fdiv_rn(b[j], dmin)), 0.f), 15.f) : 0;
    }
  } else {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(a_in[j]));
    d = __half2float(__float2half_rn(__fdiv_rn(amax, 31.f)));
    dmin = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      sc[j] = d > 0.f ? (int)fminf(fmaxf(rintf(__fdiv_rn(a_in[j], d)), -32.f), 31.f) : 0;
      m[j] = 0;
    }
  }
}

// Writes one block from this lane's eight codes q[h * 4 + s] (weights
// 128 h + 32 s + r) and the block's sub-block codes (identical in every lane).
template <int F>
__device__ __forceinline__ void kq_encode(uint8_t* blk, int r, const int* q, const int* sc,
                                          const int* m, float d, float dmin) {
  if (F == KQ_Q2) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t byte = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) byte |= (uint32_t)(q[h * 4 + s] & 3) << (2 * s);
      blk[16 + 32 * h + r] = (uint8_t)byte;
    }
    if (r < 16) blk[r] = (uint8_t)(sc[r] | (m[r] << 4));
    if (r == 0) {
      // both fp16 factors in one aligned 4-byte store (84 bi + 80 is a
      // multiple of 4), little-endian
      *reinterpret_cast<uint32_t*>(blk + 80) =
          (uint32_t)float_to_half_bits(d) | ((uint32_t)float_to_half_bits(dmin) << 16);
    }
  } else {
    uint32_t hib = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t byte = 0;
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        const uint32_t u = (uint32_t)(q[h * 4 + s] + 4);
        byte |= (u & 3u) << (2 * s);
        hib |= (u >> 2) << (4 * h + s);
      }
      blk[32 + 32 * h + r] = (uint8_t)byte;
    }
    blk[r] = (uint8_t)hib;
    if (r < 8)
      blk[96 + r] = (uint8_t)(((sc[r] + 32) & 15) | (((sc[r + 8] + 32) & 15) << 4));
    if (r < 4) {
      uint32_t byte = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) byte |= (uint32_t)(((sc[r + 4 * p] + 32) >> 4) & 3) << (2 * p);
      blk[104 + r] = (uint8_t)byte;
    }
    if (r == 0) {
      // one aligned 2-byte store (110 bi + 108 is even), little-endian
      *reinterpret_cast<uint16_t*>(blk + 108) = float_to_half_bits(d);
    }
  }
}

// Reads this lane's eight codes and the block's sub-block codes.
template <int F>
__device__ __forceinline__ void kq_decode(const uint8_t* blk, int r, int* q, int* sc, int* m,
                                          float& d, float& dmin) {
  if (F == KQ_Q2) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t byte = blk[16 + 32 * h + r];
#pragma unroll
      for (int s = 0; s < 4; ++s) q[h * 4 + s] = (int)((byte >> (2 * s)) & 3u);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      sc[j] = blk[j] & 15;
      m[j] = blk[j] >> 4;
    }
    d = half_bits_to_float((uint16_t)(blk[80] | (blk[81] << 8)));
    dmin = half_bits_to_float((uint16_t)(blk[82] | (blk[83] << 8)));
  } else {
    const uint32_t hib = blk[r];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t byte = blk[32 + 32 * h + r];
#pragma unroll
      for (int s = 0; s < 4; ++s)
        q[h * 4 + s] = (int)((byte >> (2 * s)) & 3u) + 4 * (int)((hib >> (4 * h + s)) & 1u) - 4;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int lo = (blk[96 + (j & 7)] >> (4 * (j >> 3))) & 15;
      const int hi = (blk[104 + (j & 3)] >> (2 * (j >> 2))) & 3;
      sc[j] = (lo | (hi << 4)) - 32;
      m[j] = 0;
    }
    d = half_bits_to_float((uint16_t)(blk[108] | (blk[109] << 8)));
    dmin = 0.f;
  }
}

// Min-max K-Quant of W32 (the start when no blocks are given): per sub-block
// continuous parameters, projected to the format, then every weight's
// nearest level (first on ties), all in fp32 without contraction.
template <int F>
__global__ void __launch_bounds__(256) k_kq_start(const float* __restrict__ W32, int64_t nblk,
                                                  uint8_t* __restrict__ blocks) {
  const int r = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t bi = warp; bi < nblk; bi += nwarps) {
    const float* w0 = W32 + bi * kSuper;
    float w[8], a[16], b[16];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int s = 0; s < 4; ++s) w[h * 4 + s] = w0[128 * h + 32 * s + r];
#pragma unroll
    for (int hs = 0; hs < 8; ++hs) {
      // the half-warp of lanes r (r < 16 or r >= 16) holds sub-block
      // 2 hs + (r >= 16)
      float mn = w[hs], mx = w[hs], am = fabsf(w[hs]), wa = w[hs];
      int ia = r & 15;
#pragma unroll
      for (int off = 1; off < 16; off <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float am2 = __shfl_xor_sync(0xffffffffu, am, off);
        const float wa2 = __shfl_xor_sync(0xffffffffu, wa, off);
        const int ia2 = __shfl_xor_sync(0xffffffffu, ia, off);
        // the largest magnitude, first position on ties
        if (am2 > am || (am2 == am && ia2 < ia)) {
          am = am2;
          wa = wa2;
          ia = ia2;
        }
      }
      float av, bv;
      if (F == KQ_Q2) {
        mn = fminf(mn, 0.f);
        av = __fdiv_rn(__fsub_rn(mx, mn), 3.f);
        bv = -mn;
      } else {
        av = __fdiv_rn(-wa, 4.f);
        bv = 0.f;
      }
      a[2 * hs] = __shfl_sync(0xffffffffu, av, 0);
      a[2 * hs + 1] = __shfl_sync(0xffffffffu, av, 16);
      b[2 * hs] = __shfl_sync(0xffffffffu, bv, 0);
      b[2 * hs + 1] = __shfl_sync(0xffffffffu, bv, 16);
    }
    int sc[16], m[16], q[8];
    float d, dmin;
    kq_project<F>(a, b, sc, m, d, dmin);
#pragma unroll
    for (int hs = 0; hs < 8; ++hs) {
      const int j = 2 * hs + (r >= 16 ? 1 : 0);
      const float aq = __fmul_rn(d, (float)sc[j]), bq = __fmul_rn(dmin, (float)m[j]);
      int best = KqT<F>::QMIN;
      float bd = INFINITY;
#pragma unroll
      for (int k = KqT<F>::QMIN; k <= KqT<F>::QMAX; ++k) {
        const float dist = fabsf(__fsub_rn(w[hs], __fsub_rn(__fmul_rn(aq, (float)k), bq)));
        if (dist < bd) {
          bd = dist;
          best = k;
        }
      }
      q[hs] = best;
    }
    kq_encode<F>(blocks + bi * KqT<F>::BYTES, r, q, sc, m, d, dmin);
  }
}

// State from blocks: a_j = d sc_j, b_j = dmin m_j, start codes, logits +2
// on the start code (Q2_K) or on shift 0 (Q3_K), momenta zero elsewhere.
template <int F>
__global__ void __launch_bounds__(256) k_kq_init(const uint8_t* __restrict__ blocks,
                                                 int64_t nblk, int64_t NK, float* __restrict__ a,
                                                 float* __restrict__ b, int8_t* __restrict__ q0,
                                                 float* __restrict__ logits) {
  constexpr int L = KqT<F>::L;
  const int r = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t bi = warp; bi < nblk; bi += nwarps) {
    int q[8], sc[16], m[16];
    float d, dmin;
    kq_decode<F>(blocks + bi * KqT<F>::BYTES, r, q, sc, m, d, dmin);
    if (r < 16) {
      a[bi * 16 + r] = __fmul_rn(d, (float)sc[r]);
      b[bi * 16 + r] = __fmul_rn(dmin, (float)m[r]);
    }
#pragma unroll
    for (int hs = 0; hs < 8; ++hs) {
      const int64_t c = bi * kSuper + 128 * (hs >> 2) + 32 * (hs & 3) + r;
      q0[c] = (int8_t)q[hs];
#pragma unroll
      for (int p = 0; p < L; ++p) {
        const bool on = F == KQ_Q2 ? (p == q[hs]) : (p == 2);
        logits[p * NK + c] = on ? 2.f : 0.f;
      }
    }
  }
}

// Level values of a coordinate's logits.
template <int F>
__device__ __forceinline__ void kq_cand(int q0, float* c) {
#pragma unroll
  for (int k = 0; k < KqT<F>::L; ++k)
    c[k] = F == KQ_Q2 ? (float)k : (float)min(max(q0 + k - 2, -4), 3);
}

// Philox words of the aligned quad c0 .. c0 + 3 (c0 % 4 == 0) at step t:
// block 0 of each coordinate and, with `five` (Q3_K), the quad's one block-1
// draw, coordinate c0 + j taking its word j -- the counters of the GSQ grids.
__device__ __forceinline__ void kq_quad_words(uint64_t c0, uint32_t t, const PhiloxKeys& ks,
                                              bool five, uint32_t w[4][5]) {
  const uint32_t hi = (uint32_t)(c0 >> 32);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 r = philox4x32_10(make_uint4((uint32_t)c0 + (uint32_t)j, hi, t, 0u), ks);
    w[j][0] = r.x;
    w[j][1] = r.y;
    w[j][2] = r.z;
    w[j][3] = r.w;
  }
  uint4 r1 = make_uint4(0u, 0u, 0u, 0u);
  if (five) r1 = philox4x32_10(make_uint4((uint32_t)c0, hi, t, 1u), ks);
  w[0][4] = r1.x;
  w[1][4] = r1.y;
  w[2][4] = r1.z;
  w[3][4] = r1.w;
}

// y = softmax((l + g) / tau) with the GSQ grids' noise (gsoftmax2: the same
// words, the same arithmetic) and v = sum_k y_k c_k
template <int L>
__device__ __forceinline__ float kq_value(const float* l, const uint32_t* w, bool noise,
                                          float inv_tau, const float2* cells, const float* c,
                                          float* y) {
  const float r = gsoftmax2<L, false>(l, w, noise, inv_tau, cells, y);
  float v = 0.f;
#pragma unroll
  for (int k = 0; k < L; ++k) v = fmaf(y[k], c[k], v);
#pragma unroll
  for (int k = 0; k < L; ++k) y[k] *= r;
  return v * r;
}

// Soft weight w = bf16(a_j v - b_j) of step t.  Nothing else is kept: the
// backward draws the same noise again from the same counters.  Four
// coordinates per thread.
template <int F>
__global__ void __launch_bounds__(256) k_kq_soft(const float* __restrict__ logits,
                                                 const float* __restrict__ a,
                                                 const float* __restrict__ b,
                                                 const int8_t* __restrict__ q0, int64_t NK,
                                                 const PhiloxKeys ks, uint32_t t, int noise,
                                                 float inv_tau, __nv_bfloat16* __restrict__ What,
                                                 float* __restrict__ wsoft32) {
  constexpr int L = KqT<F>::L;
  __shared__ float2 l2cells[kLog2Cells];
  log2_cells_init(l2cells);
  __syncthreads();
  for (int64_t qd = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; qd < NK / 4;
       qd += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c0 = qd * 4;
    const float aj = a[c0 / kSub], bj = b[c0 / kSub];
    const char4 qv = *reinterpret_cast<const char4*>(q0 + c0);
    const int qq[4] = {qv.x, qv.y, qv.z, qv.w};
    float4 lp[L];
#pragma unroll
    for (int p = 0; p < L; ++p) lp[p] = *reinterpret_cast<const float4*>(logits + p * NK + c0);
    uint32_t wd[4][5] = {};
    if (noise) kq_quad_words((uint64_t)c0, t, ks, L == 5, wd);
    float wv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l[L], c[L], y[L];
#pragma unroll
      for (int p = 0; p < L; ++p)
        l[p] = j == 0 ? lp[p].x : j == 1 ? lp[p].y : j == 2 ? lp[p].z : lp[p].w;
      kq_cand<F>(qq[j], c);
      const float v = kq_value<L>(l, wd[j], noise, inv_tau, l2cells, c, y);
      wv[j] = fmaf(aj, v, -bj);
    }
    __nv_bfloat162 p01 = __floats2bfloat162_rn(wv[0], wv[1]);
    __nv_bfloat162 p23 = __floats2bfloat162_rn(wv[2], wv[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&p01);
    pk.y = *reinterpret_cast<uint32_t*>(&p23);
    *reinterpret_cast<uint2*>(What + c0) = pk;
    if (wsoft32) *reinterpret_cast<float4*>(wsoft32 + c0) = make_float4(wv[0], wv[1], wv[2], wv[3]);
  }
}

// Backward + Lion from dW: per coordinate the step's probabilities are drawn
// again from the pre-update logits and the words of step t (the soft
// weight's counters, so the same values), then
// dl_k = (a_j dw / tau) y_k sum_m y_m (c_k - c_m); per sub-block
// da_j = sum dw v, db_j = -sum dw (the four lanes of a sub-block combine by
// shuffles, which leaves the same sum in all four); Lion on the logits, a_j
// and (Q2_K) b_j.  With NEXT the kernel goes on to the soft weight of step
// t + 1 at 1 / inv_tau_next from the updated logits, a_j and b_j -- the
// same arithmetic as k_kq_soft -- and writes it to What.
//
// One warp per 128 consecutive coordinates (8 sub-blocks); lane j owns the
// four coordinates 4j..4j+3.  The warp's next 128 coordinates are staged in
// shared memory by per-lane 16-byte async copies (each lane copies exactly
// what it will read) and their sub-block parameters loaded into registers
// while the current ones are computed, so the loads of one group overlap the
// arithmetic of the previous one.
template <int F>
struct KqBwdCfg {
  static constexpr int L = KqT<F>::L;
  // per-warp staging of 128 coordinates: dW, logits, momenta, q0
  static constexpr int OFF_L = 512, OFF_M = OFF_L + L * 512;
  static constexpr int OFF_Q = OFF_M + L * 512;
  static constexpr int BUF = OFF_Q + 128;
  static constexpr int WARPS = 8;  // warps per CTA
  static constexpr int CTAS = 2;   // CTAs per SM
  static constexpr int SMEM = WARPS * 2 * BUF;
};

template <int F, bool DBG, bool NEXT>
__global__ void __launch_bounds__(KqBwdCfg<F>::WARPS * 32, KqBwdCfg<F>::CTAS) k_kq_backward(
    float* __restrict__ logits, float* __restrict__ mom, float* __restrict__ a,
    float* __restrict__ ma, float* __restrict__ b, float* __restrict__ mb,
    const int8_t* __restrict__ q0, const float* __restrict__ dW, int64_t NK, float inv_tau,
    float lr, float b1, float omb1, float b2, float omb2, float* __restrict__ dl_dbg,
    float* __restrict__ da_dbg, float* __restrict__ db_dbg, const PhiloxKeys ks, uint32_t t,
    int noise, float inv_tau_next, __nv_bfloat16* __restrict__ What) {
  using C = KqBwdCfg<F>;
  constexpr int L = C::L;
  extern __shared__ __align__(16) uint8_t kq_smem[];
  __shared__ float2 l2cells[kLog2Cells];
  log2_cells_init(l2cells);
  __syncthreads();
  const int64_t groups = NK / 128;  // K % 256 == 0
  const int lane = threadIdx.x & 31, wic = threadIdx.x >> 5;
  const int64_t nwarps = (int64_t)gridDim.x * C::WARPS;
  const uint32_t wbuf = smem_u32(kq_smem) + (uint32_t)(wic * 2 * C::BUF);
  auto prefetch = [&](int64_t gi, int buf) {
    const int64_t c = gi * 128 + 4 * lane;
    const uint32_t d = wbuf + (uint32_t)(buf * C::BUF + 16 * lane);
    cp_async16(d, dW + c);
#pragma unroll
    for (int p = 0; p < L; ++p) {
      cp_async16(d + (uint32_t)(C::OFF_L + p * 512), logits + p * NK + c);
      cp_async16(d + (uint32_t)(C::OFF_M + p * 512), mom + p * NK + c);
    }
    cp_async4(wbuf + (uint32_t)(buf * C::BUF + C::OFF_Q + 4 * lane), q0 + c);
  };
  int64_t gi = (int64_t)blockIdx.x * C::WARPS + wic;
  // the lane's sub-block parameters, one group ahead like the staging (each
  // sub-block is read and written by the four lanes of one warp only)
  auto params = [&](int64_t g, float* v) {
    const int64_t sb = (g * 128 + 4 * lane) / kSub;
    v[0] = a[sb];
    v[1] = ma[sb];
    v[2] = b[sb];
    v[3] = F == KQ_Q2 ? mb[sb] : 0.f;
  };
  float pn[4] = {0.f, 0.f, 0.f, 0.f};
  if (gi < groups) {
    prefetch(gi, 0);
    params(gi, pn);
  }
  cp_async_commit();
  for (int buf = 0; gi < groups; gi += nwarps, buf ^= 1) {
    const float aj = pn[0], maj = pn[1], bj = pn[2], mbj = pn[3];
    if (gi + nwarps < groups) {
      prefetch(gi + nwarps, buf ^ 1);
      params(gi + nwarps, pn);
    }
    cp_async_commit();
    cp_async_wait<1>();  // this lane's copies of group gi have landed
    const uint8_t* sbuf = kq_smem + wic * 2 * C::BUF + buf * C::BUF + 16 * lane;
    const int64_t c0 = gi * 128 + 4 * lane;
    const int64_t sb = c0 / kSub;
    float dw[4], lr_[L][4], mr[L][4];
    *reinterpret_cast<float4*>(dw) = *reinterpret_cast<const float4*>(sbuf);
#pragma unroll
    for (int p = 0; p < L; ++p) {
      *reinterpret_cast<float4*>(lr_[p]) =
          *reinterpret_cast<const float4*>(sbuf + C::OFF_L + p * 512);
      *reinterpret_cast<float4*>(mr[p]) =
          *reinterpret_cast<const float4*>(sbuf + C::OFF_M + p * 512);
    }
    const uint32_t q4 = *reinterpret_cast<const uint32_t*>(
        kq_smem + wic * 2 * C::BUF + buf * C::BUF + C::OFF_Q + 4 * lane);
    int qq[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) qq[j] = (int)(int8_t)((q4 >> (8 * j)) & 0xFFu);
    // pass 1: this step's probabilities (pre-update logits, words of step t)
    uint32_t wd[4][5] = {};
    if (noise) kq_quad_words((uint64_t)c0, t, ks, L == 5, wd);
    float da_part = 0.f, db_part = 0.f;
    float dlo[DBG ? L : 1][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l[L], y[L], c[L];
#pragma unroll
      for (int p = 0; p < L; ++p) l[p] = lr_[p][j];
      kq_cand<F>(qq[j], c);
      const float v = kq_value<L>(l, wd[j], noise, inv_tau, l2cells, c, y);
      da_part = fmaf(dw[j], v, da_part);
      db_part -= dw[j];
      const float sc = aj * dw[j] * inv_tau;
      // sum_k y_k (c_p - c_k) = c_p Sy - Vy, Sy = sum_k y_k, Vy = sum_k y_k c_k
      float Sy = 0.f, Vy = 0.f;
#pragma unroll
      for (int k = 0; k < L; ++k) {
        Sy += y[k];
        Vy = fmaf(y[k], c[k], Vy);
      }
#pragma unroll
      for (int p = 0; p < L; ++p) {
        const float g = sc * y[p] * fmaf(c[p], Sy, -Vy);
        float th = lr_[p][j], mm = mr[p][j];
        lion_update(th, mm, g, lr, b1, omb1, b2, omb2);
        lr_[p][j] = th;
        mr[p][j] = mm;
        if (DBG) dlo[DBG ? p : 0][j] = g;
      }
    }
#pragma unroll
    for (int p = 0; p < L; ++p) {
      *reinterpret_cast<float4*>(logits + p * NK + c0) = *reinterpret_cast<float4*>(lr_[p]);
      *reinterpret_cast<float4*>(mom + p * NK + c0) = *reinterpret_cast<float4*>(mr[p]);
      if (DBG)
        *reinterpret_cast<float4*>(dl_dbg + p * NK + c0) =
            *reinterpret_cast<float4*>(dlo[DBG ? p : 0]);
    }
    // the four lanes of the sub-block (lanes 4k..4k+3)
    da_part += __shfl_xor_sync(0xffffffffu, da_part, 1);
    da_part += __shfl_xor_sync(0xffffffffu, da_part, 2);
    db_part += __shfl_xor_sync(0xffffffffu, db_part, 1);
    db_part += __shfl_xor_sync(0xffffffffu, db_part, 2);
    // every lane of the sub-block updates its parameters alike; the first stores
    float av = aj, mav = maj, bv = bj, mbv = mbj;
    lion_update(av, mav, da_part, lr, b1, omb1, b2, omb2);
    if (F == KQ_Q2) lion_update(bv, mbv, db_part, lr, b1, omb1, b2, omb2);
    if ((lane & 3) == 0) {
      a[sb] = av;
      ma[sb] = mav;
      if (F == KQ_Q2) {
        b[sb] = bv;
        mb[sb] = mbv;
      }
      if (DBG) {
        da_dbg[sb] = da_part;
        db_dbg[sb] = db_part;
      }
    }
    if (NEXT) {
      // pass 2: the soft weight of step t + 1 (updated logits and parameters)
      if (noise) kq_quad_words((uint64_t)c0, t + 1u, ks, L == 5, wd);
      float wv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float l[L], c[L], y[L];
#pragma unroll
        for (int p = 0; p < L; ++p) l[p] = lr_[p][j];
        kq_cand<F>(qq[j], c);
        const float v = kq_value<L>(l, wd[j], noise, inv_tau_next, l2cells, c, y);
        wv[j] = fmaf(av, v, -bv);
      }
      __nv_bfloat162 p01 = __floats2bfloat162_rn(wv[0], wv[1]);
      __nv_bfloat162 p23 = __floats2bfloat162_rn(wv[2], wv[3]);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&p01);
      pk.y = *reinterpret_cast<uint32_t*>(&p23);
      *reinterpret_cast<uint2*>(What + c0) = pk;
    }
  }
  cp_async_wait<0>();
}

// Projection back into the format: hard codes (argmax, first maximum) and
// the sub-block parameters re-encoded.
template <int F>
__global__ void __launch_bounds__(256) k_kq_export(const float* __restrict__ logits,
                                                   const float* __restrict__ a,
                                                   const float* __restrict__ b,
                                                   const int8_t* __restrict__ q0, int64_t nblk,
                                                   int64_t NK, uint8_t* __restrict__ blocks) {
  constexpr int L = KqT<F>::L;
  const int r = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t bi = warp; bi < nblk; bi += nwarps) {
    float av[16], bv[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      av[j] = a[bi * 16 + j];
      bv[j] = b[bi * 16 + j];
    }
    int sc[16], m[16], q[8];
    float d, dmin;
    kq_project<F>(av, bv, sc, m, d, dmin);
#pragma unroll
    for (int hs = 0; hs < 8; ++hs) {
      const int64_t c = bi * kSuper + 128 * (hs >> 2) + 32 * (hs & 3) + r;
      int best = 0;
      float bl = logits[c];
#pragma unroll
      for (int p = 1; p < L; ++p) {
        const float l = logits[p * NK + c];
        if (l > bl) {
          bl = l;
          best = p;
        }
      }
      q[hs] = F == KQ_Q2 ? best : min(max((int)q0[c] + best - 2, -4), 3);
    }
    kq_encode<F>(blocks + bi * KqT<F>::BYTES, r, q, sc, m, d, dmin);
  }
}

// Weights of the format: w = bf16((d sc_j) q - dmin m_j) in fp32 without
// contraction (the products and the difference rounded separately).
template <int F>
__global__ void __launch_bounds__(256) k_kq_dequant(const uint8_t* __restrict__ blocks,
                                                    int64_t nblk, __nv_bfloat16* __restrict__ W,
                                                    float* __restrict__ W32) {
  const int r = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t bi = warp; bi < nblk; bi += nwarps) {
    int q[8], sc[16], m[16];
    float d, dmin;
    kq_decode<F>(blocks + bi * KqT<F>::BYTES, r, q, sc, m, d, dmin);
#pragma unroll
    for (int hs = 0; hs < 8; ++hs) {
      const int j = 2 * hs + (r >= 16 ? 1 : 0);
      const float w = __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc[j]), (float)q[hs]),
                                __fmul_rn(dmin, (float)m[j]));
      const int64_t c = bi * kSuper + 128 * (hs >> 2) + 32 * (hs & 3) + r;
      if (W) W[c] = __float2bfloat16_rn(w);
      if (W32) W32[c] = w;
    }
  }
}

int kq_grid(int64_t work_threads, int sms) {
  const int64_t b = (work_threads + 255) / 256;
  const int64_t cap = (int64_t)sms * 16;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

}  // namespace

// ------------------------------------------------------------- the context

struct gsq_kq {
  int fmt = 0, L = 0;
  int64_t N = 0, K = 0, T = 0, Tp = 0, nblk = 0;
  uint64_t seed = 0, t = 0;
  int noise = 1;
  // What holds the soft weight of step what_t at what_tau
  // (what_t < 0: nothing precomputed)
  int64_t what_t = -1;
  float what_tau = 0.f;
  cudaStream_t st = nullptr;
  int sms = 148, failed = 0;
  __nv_bfloat16 *Xb = nullptr, *Xt = nullptr, *What = nullptr, *dYt = nullptr;
  float *YrefT = nullptr, *dW = nullptr, *logits = nullptr, *mom = nullptr;
  float *a = nullptr, *ma = nullptr, *b = nullptr, *mb = nullptr;
  float *dl = nullptr, *da = nullptr, *db = nullptr, *wsoft32 = nullptr;  // debug, lazy
  int8_t* q0 = nullptr;
  uint8_t *start = nullptr, *exp = nullptr;
  double *partials = nullptr, *loss_hist = nullptr, *scratch = nullptr;
  unsigned* ticket = nullptr;
  int* err = nullptr;
  double yref_sq = 0.0;
  CUtensorMap tm_What, tm_Xb, tm_dYt, tm_Xt;
  EpiMaps em_forward, em_wgrad;
  std::vector<void*> allocs;
};

namespace {

int kq_fail(gsq_kq* c, int status) {
  if (c && status != GSQ_OK && c->failed == 0) c->failed = status;
  return status;
}

#define CKQ(call)                                                    \
  do {                                                               \
    cudaError_t e_ = (call);                                         \
    if (e_ != cudaSuccess) return kq_fail(c, stage_cuda_status(e_)); \
  } while (0)

template <typename T>
int kq_alloc(gsq_kq* c, T** p, size_t count) {
  void* q = nullptr;
  if (pool_malloc(&q, count * sizeof(T) + 16) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_OOM;
  }
  c->allocs.push_back(q);
  *p = static_cast<T*>(q);
  return GSQ_OK;
}

void kq_free_all(gsq_kq* c) {
  for (void* p : c->allocs) pool_free(p);
  c->allocs.clear();
}

int kq_usable(gsq_kq* c) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  return c->failed ? GSQ_ERR_STATE : GSQ_OK;
}

int kq_check_device(gsq_kq* c) {
  cudaError_t e = cudaStreamSynchronize(c->st);
  if (e != cudaSuccess) return kq_fail(c, stage_cuda_status(e));
  int h = 0;
  e = cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return kq_fail(c, stage_cuda_status(e));
  switch (h) {
    case DEV_OK: return GSQ_OK;
    case DEV_ERR_TIMEOUT: return kq_fail(c, GSQ_ERR_TIMEOUT);
    case DEV_ERR_NONFINITE: return kq_fail(c, GSQ_ERR_NONFINITE);
    default: return kq_fail(c, GSQ_ERR_CUDA);
  }
}

EpiParams kq_epi(gsq_kq* c, double* loss_out) {
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.partials = c->partials;
  ep.ticket = c->ticket;
  ep.loss_out = loss_out;
  ep.err = c->err;
  return ep;
}

size_t kq_block_bytes(int fmt) { return fmt == KQ_Q2 ? 84 : 110; }

cudaError_t kq_launch_soft(gsq_kq* c, float tau, float* wsoft32) {
  const uint32_t k0 = (uint32_t)c->seed, k1 = (uint32_t)(c->seed >> 32);
  const int64_t NK = c->N * c->K;
  const int g = kq_grid(NK / 4, c->sms);
  if (c->fmt == KQ_Q2)
    k_kq_soft<KQ_Q2><<<g, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, NK,
                                           philox_keys(k0, k1), (uint32_t)c->t, c->noise,
                                           1.f / tau, c->What, wsoft32);
  else
    k_kq_soft<KQ_Q3><<<g, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, NK,
                                           philox_keys(k0, k1), (uint32_t)c->t, c->noise,
                                           1.f / tau, c->What, wsoft32);
  return cudaGetLastError();
}

// The backward of step t; next_tau > 0 (not with dbg): also the soft weight
// of step t + 1 at next_tau.
template <int F, bool DBG, bool NEXT>
cudaError_t kq_backward_launch(gsq_kq* c, float it, float lr, float b1, float b2, float itn) {
  using Cf = KqBwdCfg<F>;
  {
    const cudaError_t e = smem_optin<k_kq_backward<F, DBG, NEXT>>(Cf::SMEM);
    if (e != cudaSuccess) return e;
  }
  const int64_t NK = c->N * c->K, groups = NK / 128;
  const int64_t need = (groups + Cf::WARPS - 1) / Cf::WARPS;
  const int64_t cap = (int64_t)c->sms * Cf::CTAS;
  const unsigned blocks = (unsigned)(need < cap ? need : cap);
  k_kq_backward<F, DBG, NEXT><<<blocks, Cf::WARPS * 32, Cf::SMEM, c->st>>>(
      c->logits, c->mom, c->a, c->ma, c->b, c->mb, c->q0, c->dW, NK, it, lr, b1, 1.f - b1, b2,
      1.f - b2, c->dl, c->da, c->db, philox_keys((uint32_t)c->seed, (uint32_t)(c->seed >> 32)),
      (uint32_t)c->t, c->noise, itn, c->What);
  return cudaGetLastError();
}

cudaError_t kq_launch_backward(gsq_kq* c, float tau, float lr, float b1, float b2, bool dbg,
                               float next_tau = 0.f) {
  const float it = 1.f / tau;
  const bool next = !dbg && next_tau > 0.f;
  const float itn = next ? 1.f / next_tau : 0.f;
  if (c->fmt == KQ_Q2) {
    if (dbg) return kq_backward_launch<KQ_Q2, true, false>(c, it, lr, b1, b2, itn);
    if (next) return kq_backward_launch<KQ_Q2, false, true>(c, it, lr, b1, b2, itn);
    return kq_backward_launch<KQ_Q2, false, false>(c, it, lr, b1, b2, itn);
  }
  if (dbg) return kq_backward_launch<KQ_Q3, true, false>(c, it, lr, b1, b2, itn);
  if (next) return kq_backward_launch<KQ_Q3, false, true>(c, it, lr, b1, b2, itn);
  return kq_backward_launch<KQ_Q3, false, false>(c, it, lr, b1, b2, itn);
}

cudaError_t kq_launch_dequant(int fmt, const uint8_t* blocks, int64_t nblk, __nv_bfloat16* W,
                              float* W32, int sms, cudaStream_t st) {
  const int g = kq_grid(nblk * 32, sms);
  if (fmt == KQ_Q2) k_kq_dequant<KQ_Q2><<<g, 256, 0, st>>>(blocks, nblk, W, W32);
  else k_kq_dequant<KQ_Q3><<<g, 256, 0, st>>>(blocks, nblk, W, W32);
  return cudaGetLastError();
}

// One step at tau; next_tau > 0: the backward also forms the soft weight of
// the next step at next_tau (What then holds step t + 1's, recorded
// in what_t / what_tau, and the next step at that tau skips its own).
int kq_step(gsq_kq* c, float tau, float lr, float b1, float b2, float next_tau = 0.f) {
  if (c->t >= 0xFFFFFFFEull) return GSQ_ERR_UNSUPPORTED;
  if (!(c->what_t == (int64_t)c->t && c->what_tau == tau)) CKQ(kq_launch_soft(c, tau, nullptr));
  c->what_t = -1;
  EpiParams ep = kq_epi(c, c->loss_hist + (c->t % kStageLossRing));
  CKQ(launch_gemm(c->tm_What, c->tm_Xb, c->em_forward, c->N, c->Tp, c->K, EPI_LOSS_DY, ep,
                  c->sms, c->st));
  EpiParams ep2 = kq_epi(c, nullptr);
  CKQ(launch_gemm(c->tm_dYt, c->tm_Xt, c->em_wgrad, c->N, c->K, c->Tp, EPI_STORE_F32, ep2,
                  c->sms, c->st));
  CKQ(kq_launch_backward(c, tau, lr, b1, b2, false, next_tau));
  c->t += 1;
  if (next_tau > 0.f) {
    c->what_t = (int64_t)c->t;
    c->what_tau = next_tau;
  }
  return GSQ_OK;
}

int kq_buffer(gsq_kq* c, int which, void** p, size_t* bytes) {
  const size_t NK = (size_t)c->N * c->K, LNK = (size_t)c->L * NK, NS = NK / kSub;
  int rc = GSQ_OK;
  switch (which) {
    case GSQ_KQ_DBG_LOGITS: *p = c->logits; *bytes = LNK * 4; break;
    case GSQ_KQ_DBG_MOM: *p = c->mom; *bytes = LNK * 4; break;
    case GSQ_KQ_DBG_A: *p = c->a; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_MA: *p = c->ma; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_B: *p = c->b; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_MB: *p = c->mb; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_Q0: *p = c->q0; *bytes = NK; break;
    case GSQ_KQ_DBG_WHAT: *p = c->What; *bytes = NK * 2; break;
    case GSQ_KQ_DBG_DW: *p = c->dW; *bytes = NK * 4; break;
    case GSQ_KQ_DBG_DL:
      if (!c->dl) rc = kq_alloc(c, &c->dl, LNK);
      *p = c->dl; *bytes = LNK * 4; break;
    case GSQ_KQ_DBG_DA:
      if (!c->da) rc = kq_alloc(c, &c->da, NS);
      *p = c->da; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_DB:
      if (!c->db) rc = kq_alloc(c, &c->db, NS);
      *p = c->db; *bytes = NS * 4; break;
    case GSQ_KQ_DBG_WSOFT32:
      if (!c->wsoft32) rc = kq_alloc(c, &c->wsoft32, NK);
      *p = c->wsoft32; *bytes = NK * 4; break;
    default: return GSQ_ERR_INVALID_ARG;
  }
  return rc;
}

}  // namespace

extern "C" {

int gsq_kq_block_bytes(int format, int64_t N, int64_t K, size_t* bytes) {
  if (!bytes || (format != KQ_Q2 && format != KQ_Q3) || N <= 0 || K <= 0 || K % kSuper)
    return GSQ_ERR_INVALID_ARG;
  *bytes = (size_t)(N * K / kSuper) * kq_block_bytes(format);
  return GSQ_OK;
}

int gsq_kq_init(gsq_kq** out, const void* W, int w_dtype, const void* X, int x_dtype,
                int64_t N, int64_t K, int64_t T, int format, const void* start_blocks,
                uint64_t seed, void* stream) {
  if (!out) return GSQ_ERR_INVALID_ARG;
  *out = nullptr;
  auto dt_ok = [](int dt) { return dt == GSQ_F32 || dt == GSQ_BF16; };
  if (!W || !X || !dt_ok(w_dtype) || !dt_ok(x_dtype) || N <= 0 || K <= 0 || T <= 0 ||
      K % kSuper != 0 || (format != KQ_Q2 && format != KQ_Q3) || N > ((int64_t)1 << 31) ||
      T > ((int64_t)1 << 31))
    return GSQ_ERR_INVALID_ARG;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  gsq_kq* c = new (std::nothrow) gsq_kq();
  if (!c) return GSQ_ERR_OOM;
  c->fmt = format;
  c->L = format == KQ_Q2 ? 4 : 5;
  c->N = N;
  c->K = K;
  c->T = T;
  c->Tp = (T + 63) / 64 * 64;
  c->nblk = N * K / kSuper;
  c->seed = seed;
  c->st = static_cast<cudaStream_t>(stream);
  c->sms = prop.multiProcessorCount;
  const int64_t NK = N * K, Tp = c->Tp, NS = NK / kSub;
  const size_t bb = (size_t)c->nblk * kq_block_bytes(format);
  const bool split = w_dtype == GSQ_F32;
  int rc = GSQ_OK;
#define ALQ(p, n) \
  if (rc == GSQ_OK) rc = kq_alloc(c, &(p), (size_t)(n))
  ALQ(c->Xb, Tp * K);
  ALQ(c->Xt, K * Tp);
  ALQ(c->What, NK);
  ALQ(c->dYt, N * Tp);
  ALQ(c->YrefT, N * Tp);
  ALQ(c->dW, NK);
  ALQ(c->logits, c->L * NK);
  ALQ(c->mom, c->L * NK);
  ALQ(c->a, NS);
  ALQ(c->ma, NS);
  ALQ(c->b, NS);
  ALQ(c->mb, NS);
  ALQ(c->q0, NK);
  ALQ(c->start, bb);
  ALQ(c->exp, bb);
  ALQ(c->partials, kStagePartials);
  ALQ(c->loss_hist, kStageLossRing);
  ALQ(c->scratch, 4);
  ALQ(c->ticket, 4);
  ALQ(c->err, 4);
#undef ALQ
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
    kq_free_all(c);
    delete c;
    return status;
  };
  float* W32 = nullptr;
  __nv_bfloat16 *Wop = nullptr, *Xcat = nullptr;
  salloc((void**)&W32, (size_t)NK * 4);
  salloc((void**)&Wop, (size_t)NK * 2 * (split ? 2 : 1));
  if (split) salloc((void**)&Xcat, (size_t)Tp * 2 * K * 2);
  const size_t wbytes = (size_t)NK * (w_dtype == GSQ_F32 ? 4 : 2);
  const size_t xbytes = (size_t)T * K * (x_dtype == GSQ_F32 ? 4 : 2);
  const void* Wd = W;
  const void* Xd = X;
  void* tmp = nullptr;
  if (rc == GSQ_OK && !stage_is_device_ptr(W)) { salloc(&tmp, wbytes); Wd = tmp; }
  if (rc == GSQ_OK && !stage_is_device_ptr(X)) { salloc(&tmp, xbytes); Xd = tmp; }
  if (rc != GSQ_OK) return cleanup_fail(rc);
  cudaStream_t st = c->st;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
    return e == cudaSuccess;
  };
  if (Wd != W) ok(cudaMemcpyAsync(const_cast<void*>(Wd), W, wbytes, cudaMemcpyDefault, st));
  if (Xd != X) ok(cudaMemcpyAsync(const_cast<void*>(Xd), X, xbytes, cudaMemcpyDefault, st));
  ok(cudaMemsetAsync(c->err, 0, 16, st));
  ok(cudaMemsetAsync(c->ticket, 0, 16, st));
  ok(cudaMemsetAsync(c->loss_hist, 0, kStageLossRing * sizeof(double), st));
  ok(cudaMemsetAsync(c->mom, 0, (size_t)c->L * NK * 4, st));
  ok(cudaMemsetAsync(c->ma, 0, (size_t)NS * 4, st));
  ok(cudaMemsetAsync(c->mb, 0, (size_t)NS * 4, st));
  ok(cudaMemsetAsync(c->dW, 0, (size_t)NK * 4, st));
  ok(cudaMemsetAsync(c->dYt, 0, (size_t)N * Tp * 2, st));
  ok(launch_convert_x(Xd, x_dtype, T, K, Tp, c->Xb, c->Xt, Xcat, c->err, st));
  ok(launch_convert_w(Wd, w_dtype, N, K, W32, Wop, split ? 1 : 0, c->err, st));
  // the start: the caller's blocks, or the min-max K-Quant of W
  const int gq = kq_grid(c->nblk * 32, c->sms);
  if (start_blocks) {
    ok(cudaMemcpyAsync(c->start, start_blocks, bb, cudaMemcpyDefault, st));
  } else if (format == KQ_Q2) {
    k_kq_start<KQ_Q2><<<gq, 256, 0, st>>>(W32, c->nblk, c->start);
    ok(cudaGetLastError());
  } else {
    k_kq_start<KQ_Q3><<<gq, 256, 0, st>>>(W32, c->nblk, c->start);
    ok(cudaGetLastError());
  }
  if (format == KQ_Q2)
    k_kq_init<KQ_Q2><<<gq, 256, 0, st>>>(c->start, c->nblk, NK, c->a, c->b, c->q0, c->logits);
  else
    k_kq_init<KQ_Q3><<<gq, 256, 0, st>>>(c->start, c->nblk, NK, c->a, c->b, c->q0, c->logits);
  ok(cudaGetLastError());
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));
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
  c->em_wgrad.yref = c->em_forward.yref;
  {
    EpiMaps em;
    em.out = c->em_forward.yref;
    em.yref = c->em_forward.yref;
    ok(launch_gemm(tmW, tmXr, em, N, Tp, kw * K, EPI_STORE_F32, kq_epi(c, nullptr), c->sms, st));
  }
  ok(launch_sumsq(c->YrefT, N * Tp, c->partials, c->ticket, c->scratch, st));
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cleanup_fail(stage_cuda_status(e));
  int h = 0;
  double ysq = 0.0;
  if (cudaMemcpy(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(&ysq, c->scratch, sizeof(double), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cleanup_fail(GSQ_ERR_CUDA);
  if (h == DEV_ERR_NONFINITE) return cleanup_fail(GSQ_ERR_NONFINITE);
  if (h != DEV_OK) return cleanup_fail(h == DEV_ERR_TIMEOUT ? GSQ_ERR_TIMEOUT : GSQ_ERR_CUDA);
  c->yref_sq = ysq;
  for (void* p : staging) pool_free(p);
  *out = c;
  return GSQ_OK;
}

int gsq_kq_step(gsq_kq* c, float tau, float lr, float beta1, float beta2) {
  int u = kq_usable(c);
  if (u) return u;
  if (!stage_step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  return kq_step(c, tau, lr, beta1, beta2);
}

int gsq_kq_run(gsq_kq* c, const float* taus, int64_t n, float lr, float beta1, float beta2) {
  int u = kq_usable(c);
  if (u) return u;
  if (!taus || n <= 0) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i)
    if (!stage_step_args_ok(taus[i], lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int rc = kq_step(c, taus[i], lr, beta1, beta2, i + 1 < n ? taus[i + 1] : 0.f);
    if (rc) return rc;
  }
  return GSQ_OK;
}

int gsq_kq_last_loss(gsq_kq* c, double* loss) {
  int u = kq_usable(c);
  if (u) return u;
  if (!loss) return GSQ_ERR_INVALID_ARG;
  if (c->t == 0) return GSQ_ERR_STATE;
  int rc = kq_check_device(c);
  if (rc) return rc;
  CKQ(cudaMemcpy(loss, c->loss_hist + ((c->t - 1) % kStageLossRing), sizeof(double),
                 cudaMemcpyDeviceToHost));
  if (!std::isfinite(*loss)) return kq_fail(c, GSQ_ERR_NONFINITE);
  return GSQ_OK;
}

int gsq_kq_export(gsq_kq* c, void* blocks) {
  int u = kq_usable(c);
  if (u) return u;
  if (!blocks) return GSQ_ERR_INVALID_ARG;
  const int gq = kq_grid(c->nblk * 32, c->sms);
  const int64_t NK = c->N * c->K;
  if (c->fmt == KQ_Q2)
    k_kq_export<KQ_Q2><<<gq, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, c->nblk, NK, c->exp);
  else
    k_kq_export<KQ_Q3><<<gq, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, c->nblk, NK, c->exp);
  CKQ(cudaGetLastError());
  CKQ(cudaMemcpyAsync(blocks, c->exp, (size_t)c->nblk * kq_block_bytes(c->fmt),
                      cudaMemcpyDefault, c->st));
  return kq_check_device(c);
}

int gsq_kq_start_blocks(gsq_kq* c, void* blocks) {
  int u = kq_usable(c);
  if (u) return u;
  if (!blocks) return GSQ_ERR_INVALID_ARG;
  CKQ(cudaMemcpyAsync(blocks, c->start, (size_t)c->nblk * kq_block_bytes(c->fmt),
                      cudaMemcpyDefault, c->st));
  return kq_check_device(c);
}

int gsq_kq_recon_error(gsq_kq* c, int which, double* abs_err, double* rel_err) {
  int u = kq_usable(c);
  if (u) return u;
  if (!abs_err || (which != 0 && which != 1)) return GSQ_ERR_INVALID_ARG;
  if (which == 0) {
    const int gq = kq_grid(c->nblk * 32, c->sms);
    const int64_t NK = c->N * c->K;
    if (c->fmt == KQ_Q2)
      k_kq_export<KQ_Q2><<<gq, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, c->nblk, NK, c->exp);
    else
      k_kq_export<KQ_Q3><<<gq, 256, 0, c->st>>>(c->logits, c->a, c->b, c->q0, c->nblk, NK, c->exp);
    CKQ(cudaGetLastError());
  }
  c->what_t = -1;  // What now holds the dequantized blocks
  CKQ(kq_launch_dequant(c->fmt, which == 0 ? c->exp : c->start, c->nblk, c->What, nullptr,
                        c->sms, c->st));
  CKQ(launch_gemm(c->tm_What, c->tm_Xb, c->em_forward, c->N, c->Tp, c->K, EPI_LOSS,
                  kq_epi(c, c->scratch), c->sms, c->st));
  int rc = kq_check_device(c);
  if (rc) return rc;
  double v = 0.0;
  CKQ(cudaMemcpy(&v, c->scratch, sizeof(double), cudaMemcpyDeviceToHost));
  *abs_err = v;
  if (rel_err) *rel_err = c->yref_sq > 0.0 ? v / c->yref_sq : 0.0;
  return GSQ_OK;
}

int gsq_kq_dequant(int format, const void* blocks, int64_t N, int64_t K, void* W_bf16,
                   void* stream) {
  if (!blocks || !W_bf16 || (format != KQ_Q2 && format != KQ_Q3) || N <= 0 || K <= 0 ||
      K % kSuper)
    return GSQ_ERR_INVALID_ARG;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nblk = N * K / kSuper;
  const size_t bb = (size_t)nblk * kq_block_bytes(format), wb = (size_t)N * K * 2;
  std::vector<void*> tmp;
  auto dev_or_copy = [&](const void* p, size_t bytes, bool in) -> void* {
    if (stage_is_device_ptr(p)) return const_cast<void*>(p);
    void* q = nullptr;
    if (pool_malloc(&q, bytes) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    tmp.push_back(q);
    if (in && cudaMemcpyAsync(q, p, bytes, cudaMemcpyDefault, st) != cudaSuccess) return nullptr;
    return q;
  };
  int rc = GSQ_OK;
  void* bd = dev_or_copy(blocks, bb, true);
  void* wd = bd ? dev_or_copy(W_bf16, wb, false) : nullptr;
  if (!bd || !wd) rc = GSQ_ERR_OOM;
  if (rc == GSQ_OK &&
      kq_launch_dequant(format, static_cast<const uint8_t*>(bd), nblk,
                        static_cast<__nv_bfloat16*>(wd), nullptr, prop.multiProcessorCount,
                        st) != cudaSuccess)
    rc = GSQ_ERR_CUDA;
  if (rc == GSQ_OK && wd != W_bf16 &&
      cudaMemcpyAsync(W_bf16, wd, wb, cudaMemcpyDefault, st) != cudaSuccess)
    rc = GSQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess && rc == GSQ_OK) rc = GSQ_ERR_CUDA;
  cudaGetLastError();
  for (void* p : tmp) pool_free(p);
  return rc;
}

int gsq_kq_debug_get(gsq_kq* c, int which, void* host, size_t bytes) {
  int u = kq_usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t need = 0;
  int rc = kq_buffer(c, which, &p, &need);
  if (rc) return rc;
  if (!host || bytes != need) return GSQ_ERR_INVALID_ARG;
  rc = kq_check_device(c);
  if (rc) return rc;
  CKQ(cudaMemcpy(host, p, need, cudaMemcpyDeviceToHost));
  return GSQ_OK;
}

int gsq_kq_debug_set(gsq_kq* c, int which, const void* host, size_t bytes) {
  int u = kq_usable(c);
  if (u) return u;
  void* p = nullptr;
  size_t need = 0;
  int rc = kq_buffer(c, which, &p, &need);
  if (rc) return rc;
  if (!host || bytes != need) return GSQ_ERR_INVALID_ARG;
  CKQ(cudaStreamSynchronize(c->st));
  CKQ(cudaMemcpy(p, host, need, cudaMemcpyHostToDevice));
  c->what_t = -1;
  return GSQ_OK;
}

int gsq_kq_debug_soft_weight(gsq_kq* c, float tau) {
  int u = kq_usable(c);
  if (u) return u;
  if (!(tau > 0.f) || !std::isfinite(tau)) return GSQ_ERR_INVALID_ARG;
  void* p = nullptr;
  size_t need = 0;
  int rc = kq_buffer(c, GSQ_KQ_DBG_WSOFT32, &p, &need);
  if (rc) return rc;
  c->what_t = -1;
  CKQ(kq_launch_soft(c, tau, c->wsoft32));
  return kq_check_device(c);
}

int gsq_kq_debug_backward(gsq_kq* c, float tau, float lr, float beta1, float beta2) {
  int u = kq_usable(c);
  if (u) return u;
  if (!stage_step_args_ok(tau, lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  void* p = nullptr;
  size_t need = 0;
  int rc = kq_buffer(c, GSQ_KQ_DBG_DL, &p, &need);
  if (!rc) rc = kq_buffer(c, GSQ_KQ_DBG_DA, &p, &need);
  if (!rc) rc = kq_buffer(c, GSQ_KQ_DBG_DB, &p, &need);
  if (rc) return rc;
  // the backward from the current dW (it draws the step's probabilities
  // again itself, as inside a step)
  c->what_t = -1;
  CKQ(kq_launch_backward(c, tau, lr, beta1, beta2, true));
  return kq_check_device(c);
}

int gsq_kq_debug_noise(gsq_kq* c, int on) {
  if (!c) return GSQ_ERR_INVALID_ARG;
  c->noise = on ? 1 : 0;
  c->what_t = -1;
  return GSQ_OK;
}

int gsq_kq_get_step(gsq_kq* c, uint64_t* t) {
  if (!c || !t) return GSQ_ERR_INVALID_ARG;
  *t = c->t;
  return GSQ_OK;
}

int gsq_kq_destroy(gsq_kq* c) {
  if (!c) return GSQ_OK;
  cudaStreamSynchronize(c->st);
  cudaGetLastError();
  kq_free_all(c);
  delete c;
  return GSQ_OK;
}

}  // extern "C"
