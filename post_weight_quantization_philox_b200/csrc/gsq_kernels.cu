// gsq_kernels.cu -- the bandwidth-bound kernels of the GSQ step:
//   init (operand conversion, scales, initial level, logits),
//   soft weight (Philox Gumbel noise + tempered softmax + dequantisation),
//   backward (softmax-Jacobian logit gradients, group-scale gradient by warp
//   shuffle over the 128-wide group, Lion in place),
//   harden + pack, scale export, and small reductions.
// Method: GSQ (arXiv 2604.18556), method and optimisation paragraphs of the
// agihunt.info summary; Approach section on atlas.scime.ai.
#include "gsq_device.cuh"
#include "gsq_internal.h"

namespace gsq {

namespace {

constexpr int kGroup = 128;

// Logit and Lion-momentum planes hold fp32, or bf16 in the reduced-memory
// state mode; St<TS> loads them as fp32 and stores fp32 values.
template <typename TS>
struct St;
template <>
struct St<float> {
  __device__ static float ld(const float* p) { return __ldg(p); }
  __device__ static float4 ld4(const float* p) {
    return __ldg(reinterpret_cast<const float4*>(p));
  }
  __device__ static void st(float* p, float v) { *p = v; }
};
template <>
struct St<__nv_bfloat16> {
  __device__ static float ld(const __nv_bfloat16* p) { return __bfloat162float(__ldg(p)); }
  __device__ static float4 ld4(const __nv_bfloat16* p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
  }
  // every value stored through here is already a bf16 value
  __device__ static void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// bf16 by stochastic rounding with a 9-bit threshold r: r << 7 is added to
// the fp32 bit pattern and the low half dropped (the magnitude rounds up
// with probability low16 / 2^16, to 2^-9 of a bf16 unit); returned as the
// fp32 value of the bf16 result.
__device__ __forceinline__ float bf16_sr(float x, uint32_t r) {
  return __uint_as_float((__float_as_uint(x) + ((r & 0x1FFu) << 7)) & 0xFFFF0000u);
}
__device__ __forceinline__ float bf16_rn(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

__device__ __forceinline__ void set_err(int* err, int code) {
  atomicCAS(err, 0, code);
}

// ------------------------------------------------------------ conversion

// X (T x K, fp32 or bf16) -> Xb (Tp x K bf16, row-major) and
// Xt (K x Tp bf16, transposed); optional Xcat (Tp x 2K) = [Xb | Xb] for the
// split-precision reference GEMM.  64 x 64 tiles through shared memory.
__global__ void k_convert_x(const void* __restrict__ X, int dtype, int64_t T,
                            int64_t K, int64_t Tp, __nv_bfloat16* __restrict__ Xb,
                            __nv_bfloat16* __restrict__ Xt,
                            __nv_bfloat16* __restrict__ Xcat, int* err) {
  __shared__ __nv_bfloat16 tile[64][66];
  const int64_t t0 = (int64_t)blockIdx.y * 64, k0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 64 x 4
  bool bad = false;
  for (int r = ty; r < 64; r += 4) {
    const int64_t t = t0 + r, k = k0 + tx;
    float v = 0.f;
    if (t < T && k < K) {
      v = dtype == 0 ? ((const float*)X)[t * K + k]
                     : __bfloat162float(((const __nv_bfloat16*)X)[t * K + k]);
      bad |= !isfinite(v);
    }
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    tile[r][tx] = b;
    if (t < Tp && k < K) {
      Xb[t * K + k] = b;
      if (Xcat) {
        Xcat[t * 2 * K + k] = b;
        Xcat[t * 2 * K + K + k] = b;
      }
    }
  }
  if (bad) set_err(err, DEV_ERR_NONFINITE);
  __syncthreads();
  for (int r = ty; r < 64; r += 4) {
    const int64_t k = k0 + r, t = t0 + tx;
    if (k < K && t < Tp) Xt[k * Tp + t] = tile[tx][r];
  }
}

// W (N x K, fp32 or bf16) -> W32 (fp32 copy for init) and the reference-GEMM
// operand: bf16 W (split = 0) or [hi | lo] (N x 2K) with hi = bf16(W),
// lo = bf16(W - hi) (split = 1), so that hi + lo carries ~16 bits of W.
__global__ void k_convert_w(const void* __restrict__ W, int dtype, int64_t N,
                            int64_t K, float* __restrict__ W32,
                            __nv_bfloat16* __restrict__ Wop, int split,
                            int* err) {
  const int64_t n_el = N * K;
  bool bad = false;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_el;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float w = dtype == 0
                        ? ((const float*)W)[i]
                        : __bfloat162float(((const __nv_bfloat16*)W)[i]);
    bad |= !isfinite(w);
    W32[i] = w;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    if (split) {
      const int64_t n = i / K, k = i % K;
      Wop[n * 2 * K + k] = hi;
      Wop[n * 2 * K + K + k] = __float2bfloat16_rn(w - __bfloat162float(hi));
    } else {
      Wop[i] = hi;
    }
  }
  if (bad) set_err(err, DEV_ERR_NONFINITE);
}

// ------------------------------------------------------------------ init

// One warp per group of 128: s = absmax / c_max; initial level by
// round-to-nearest of w / s (first level on ties, s = 0 -> w / s := 0) or
// from init_idx; logits +2 on the initial slot.  All comparisons in fp32.
template <int MODE, typename TS>
__global__ void k_init_state(const float* __restrict__ W32,
                             const int8_t* __restrict__ init_idx, int64_t N,
                             int64_t K, float* __restrict__ s,
                             int8_t* __restrict__ i0,
                             TS* __restrict__ logits, int* err) {
  using Gr = GridT<MODE>;
  const int64_t G = K / kGroup, NK = N * K;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t gi = warp; gi < N * G; gi += nwarps) {
    const int64_t n = gi / G, g = gi % G;
    const int64_t base = n * K + g * kGroup + lane * 4;
    float w[4];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[j] = W32[base + j];
      amax = fmaxf(amax, fabsf(w[j]));
    }
    amax = warp_max(amax);
    const float sg = amax / Gr::CMAX;
    if (lane == 0) s[gi] = sg;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = base + j;
      int lev;
      if (init_idx) {
        lev = init_idx[c];
        if (lev < 0 || lev >= Gr::LEVELS) {
          set_err(err, DEV_ERR_BAD_INIT);
          lev = 0;
        }
      } else {
        const float q = sg > 0.f ? w[j] / sg : 0.f;
        lev = 0;
        float best = fabsf(q - Gr::level(0));
#pragma unroll
        for (int l = 1; l < Gr::LEVELS; ++l) {
          const float d = fabsf(q - Gr::level(l));
          if (d < best) {
            best = d;
            lev = l;
          }
        }
      }
      i0[c] = (int8_t)lev;
      float lg[Gr::L];
#pragma unroll
      for (int p = 0; p < Gr::L; ++p) lg[p] = 0.f;
      if (MODE == GRID_2BIT) {
#pragma unroll
        for (int p = 0; p < Gr::L; ++p) lg[p] = (p == lev) ? 2.f : 0.f;
      } else if (MODE == GRID_3BIT_LOCAL) {
        lg[2] = 2.f;  // shift 0
      } else {
        // ternary: mask (zero, nonzero), sign (minus, plus); sign of w when
        // the initial level is zero (w = 0 counts as plus)
        const bool nonzero = lev != 1;
        const bool plus = (lev == 2) || (lev == 1 && !(w[j] < 0.f));
        lg[nonzero ? 1 : 0] = 2.f;
        lg[plus ? 3 : 2] = 2.f;
      }
#pragma unroll
      for (int p = 0; p < Gr::L; ++p) St<TS>::st(logits + p * NK + c, lg[p]);
    }
  }
}

// ----------------------------------------------------- soft weight (A1+A2)

template <int MODE>
__device__ __forceinline__ void candidates(int lev0, float* cand) {
  if (MODE == GRID_2BIT) {
#pragma unroll
    for (int k = 0; k < 4; ++k) cand[k] = (float)k - 1.5f;
  } else if (MODE == GRID_3BIT_LOCAL) {
#pragma unroll
    for (int k = 0; k < 5; ++k) {
      const int j = min(max(lev0 + k - 2, 0), 7);
      cand[k] = (float)j - 3.5f;
    }
  }
}

// Tempered Gumbel-softmax of one coordinate at a step, from its logits l and
// its Philox words w, and its unit value v.  Categorical modes: e holds the
// unnormalised e_k, r[0] = 1 / sum e, and v = r[0] sum_k e_k c_k over the
// candidate values cand[]; an e_k below 2^-126 is flushed (its share of v is
// far below v's rounding, as the largest e_k is 1).  Ternary (one softmax
// over the mask pair, one over the sign pair): e holds the normalised
// probabilities p0, p1, q-, q+ and v = p1 (q+ - q-); v is itself as small as
// p1, so subnormal probabilities are kept.
template <int MODE>
__device__ __forceinline__ float coord_value(const float* l, const uint32_t* w, bool noise,
                                             float inv_tau, const float2* cells,
                                             const float* cand, float* e, float* r) {
  if (MODE == GRID_TERNARY) {
    const float rm = gsoftmax2<2, true>(l, w, noise, inv_tau, cells, e);
    const float rs = gsoftmax2<2, true>(l + 2, w + 2, noise, inv_tau, cells, e + 2);
    e[0] *= rm;
    e[1] *= rm;
    e[2] *= rs;
    e[3] *= rs;
    r[0] = 1.f;
    return e[1] * (e[3] - e[2]);
  } else {
    r[0] = gsoftmax2<GridT<MODE>::L, false>(l, w, noise, inv_tau, cells, e);
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < GridT<MODE>::L; ++k) v = fmaf(e[k], cand[k], v);
    return v * r[0];
  }
}

// Block-0 words of coordinate c at step t (words 0..3 of its noise).  The
// callers pass the high word of the aligned quad's first coordinate: the four
// coordinates of a quad share it (a quad never straddles a multiple of
// 2^32), so the rounds that depend only on it and on t are formed once.
__device__ __forceinline__ void block0_words(uint64_t c, uint32_t c_hi, uint32_t t,
                                             const PhiloxKeys& ks, uint32_t* w) {
  const uint4 r = philox4x32_10(make_uint4((uint32_t)c, c_hi, t, 0u), ks);
  w[0] = r.x;
  w[1] = r.y;
  w[2] = r.z;
  w[3] = r.w;
}
// Block-1 draw of the aligned quad starting at c0 (the 3-bit grid's fifth
// word: coordinate c0 + j takes word j).
__device__ __forceinline__ void block1_words(uint64_t c0, uint32_t t, const PhiloxKeys& ks,
                                             uint32_t* w) {
  const uint4 r = philox4x32_10(make_uint4((uint32_t)c0, (uint32_t)(c0 >> 32), t, 1u), ks);
  w[0] = r.x;
  w[1] = r.y;
  w[2] = r.z;
  w[3] = r.w;
}

__device__ __forceinline__ void store_bf16x4(__nv_bfloat16* dst, const float* w) {
  __nv_bfloat162 b01 = __floats2bfloat162_rn(w[0], w[1]);
  __nv_bfloat162 b23 = __floats2bfloat162_rn(w[2], w[3]);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&b01);
  pk.y = *reinterpret_cast<uint32_t*>(&b23);
  *reinterpret_cast<uint2*>(dst) = pk;
}

// The soft weight and the fused backward give one warp a group of 128
// coordinates of one row; lane j takes the aligned quad 4j .. 4j + 3, so every
// access to a plane is one 16-byte access per lane (512 contiguous bytes per
// warp) and the quad shares its 3-bit block-1 Philox draw.

// Soft weight (A1 + A2): w = bf16(s * v), v the unit value of the tempered
// Gumbel-softmax of the logits.  Nothing else is kept: the backward draws the
// same noise again from the same counters.
template <int MODE, bool DBG, typename TS>
__global__ void __launch_bounds__(256) k_soft_weight(
    const TS* __restrict__ logits, const float* __restrict__ s,
    const int8_t* __restrict__ i0, int64_t N, int64_t K, const PhiloxKeys ks,
    uint64_t coord0, uint32_t t, int noise, float inv_tau, __nv_bfloat16* __restrict__ What,
    float* __restrict__ wsoft32) {
  constexpr int L = GridT<MODE>::L;
  __shared__ float2 l2cells[kLog2Cells];
  log2_cells_init(l2cells);
  __syncthreads();
  const int64_t NK = N * K, G = K / kGroup;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t gi = warp; gi < N * G; gi += nwarps) {
    // K = G * 128: group gi starts at coordinate 128 gi
    const int64_t c0 = gi * kGroup + 4 * lane;
    const float sg = __ldg(s + gi);
    float lj[4][L];
#pragma unroll
    for (int p = 0; p < L; ++p) {
      const float4 v = St<TS>::ld4(logits + p * NK + c0);
      lj[0][p] = v.x;
      lj[1][p] = v.y;
      lj[2][p] = v.z;
      lj[3][p] = v.w;
    }
    int levj[4] = {0, 0, 0, 0};
    if (MODE == GRID_3BIT_LOCAL) {
      const uint32_t b4 = __ldg(reinterpret_cast<const uint32_t*>(i0 + c0));
#pragma unroll
      for (int j = 0; j < 4; ++j) levj[j] = (int)(int8_t)((b4 >> (8 * j)) & 0xFFu);
    }
    // Philox counters take the global coordinate (a multiple of 4 here)
    const uint64_t gc0 = coord0 + (uint64_t)c0;
    uint32_t q1[4] = {0u, 0u, 0u, 0u};
    if (L == 5 && noise) block1_words(gc0, t, ks, q1);
    float w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t wd[5] = {0u, 0u, 0u, 0u, 0u};
      if (noise) block0_words(gc0 + j, (uint32_t)(gc0 >> 32), t, ks, wd);
      wd[4] = q1[j];
      float cand[5], e[L], r;
      candidates<MODE>(levj[j], cand);
      w[j] = sg * coord_value<MODE>(lj[j], wd, noise, inv_tau, l2cells, cand, e, &r);
    }
    store_bf16x4(What + c0, w);
    if (DBG) *reinterpret_cast<float4*>(wsoft32 + c0) = make_float4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------- backward + Lion (A5)

// Backward + Lion (A5), optionally fused with the next step's A1 + A2.  One
// warp per 128-group; lane j owns the four consecutive coordinates 4j..4j+3.
// The warp's next group is staged into shared memory with per-lane 16-byte
// async copies (each lane copies exactly the pieces it will read) while the
// current group is computed, so the loads of one group overlap the
// arithmetic of the previous one.  Every global access is 16 bytes wide
// (8 bytes for bf16 state planes).
//
// Per coordinate, from the pre-update logits and the step's Philox words
// (the counters of the step's soft weight, so the same probabilities):
//   a = s dW / tau,  dl_k = a y_k sum_j y_j (c_k - c_j)   (categorical),
//   dl_mask1 = a (q+ - q-) p1 p0 = -dl_mask0, dl_sign+ = 2 a p1 q+ q- =
//   -dl_sign- (ternary),  ds = sum over the group of dW v (warp shuffle),
// then Lion on the logits and the group scale.  With NEXT it also forms the
// soft weight of step t + 1 from the updated logits and scale with the words
// of step t + 1: the values a separate soft-weight launch would produce.
template <int MODE, typename TS = float>
struct BwdCfg {
  static constexpr int L = GridT<MODE>::L;
  // per-warp staging of one group: dW, logits, momenta (, i0); the logit and
  // momentum planes take 128 sizeof(TS) bytes each
  static constexpr int SP = 128 * (int)sizeof(TS);
  static constexpr int OFF_L = 512, OFF_M = OFF_L + L * SP, OFF_I = OFF_M + L * SP;
  static constexpr int BUF = OFF_I + (MODE == GRID_3BIT_LOCAL ? 128 : 0);
  static constexpr int WARPS = L == 5 ? 8 : 12;  // warps per CTA
  static constexpr int CTAS = 2;                 // CTAs per SM
  static constexpr int SMEM = WARPS * 2 * BUF;
};

// With TS = bf16 (the reduced-memory state) the updated logits are rounded
// stochastically, thresholds from the low 9 bits of the Philox words of
// step t + 1 (the words of the next step's noise), and the momenta to
// nearest.
template <int MODE, bool DBG, bool NEXT, typename TS>
__global__ void __launch_bounds__(BwdCfg<MODE, TS>::WARPS * 32, BwdCfg<MODE, TS>::CTAS)
    k_backward_lion(TS* __restrict__ logits, TS* __restrict__ mom,
                    float* __restrict__ s, float* __restrict__ ms,
                    const int8_t* __restrict__ i0, const float* __restrict__ dW,
                    int64_t N, int64_t K, const PhiloxKeys ks, uint64_t coord0, uint32_t t,
                    int noise, float inv_tau, float inv_tau_next, float lr, float b1, float omb1,
                    float b2, float omb2, __nv_bfloat16* __restrict__ What,
                    float* __restrict__ dl_dbg, float* __restrict__ ds_dbg) {
  using C = BwdCfg<MODE, TS>;
  constexpr int L = C::L;
  constexpr bool S16 = sizeof(TS) == 2;
  extern __shared__ __align__(16) uint8_t bwd_smem[];
  __shared__ float2 l2cells[kLog2Cells];
  pdl_trigger();  // persistent grid: every CTA is resident
  log2_cells_init(l2cells);
  pdl_wait();     // dW (and the state) of the previous kernels are complete
  __syncthreads();
  const int64_t NK = N * K, G = K / kGroup, groups = N * G;
  const int lane = threadIdx.x & 31, wic = threadIdx.x >> 5;
  const int64_t warp = (int64_t)blockIdx.x * C::WARPS + wic;
  const int64_t nwarps = (int64_t)gridDim.x * C::WARPS;
  const uint32_t wbuf = smem_u32(bwd_smem) + (uint32_t)(wic * 2 * C::BUF);
  const uint32_t t1 = t + 1u;
  // shared-memory plane order: dW, logits 0..L-1, momenta, (i0)
  auto prefetch = [&](int64_t gi, int buf) {
    const int64_t c = gi * kGroup + 4 * lane;  // K = G * 128
    const uint32_t d = wbuf + (uint32_t)(buf * C::BUF + 16 * lane);
    cp_async16(d, dW + c);
    const uint32_t ds_ = wbuf + (uint32_t)(buf * C::BUF + (S16 ? 8 : 16) * lane);
#pragma unroll
    for (int p = 0; p < L; ++p) {
      if (S16) {
        cp_async8(ds_ + (uint32_t)(C::OFF_L + p * C::SP), logits + p * NK + c);
        cp_async8(ds_ + (uint32_t)(C::OFF_M + p * C::SP), mom + p * NK + c);
      } else {
        cp_async16(ds_ + (uint32_t)(C::OFF_L + p * C::SP), logits + p * NK + c);
        cp_async16(ds_ + (uint32_t)(C::OFF_M + p * C::SP), mom + p * NK + c);
      }
    }
    if (MODE == GRID_3BIT_LOCAL)
      cp_async4(wbuf + (uint32_t)(buf * C::BUF + C::OFF_I + 4 * lane), i0 + c);
  };
  int64_t gi = warp;
  if (gi < groups) prefetch(gi, 0);
  // the group's scale and its momentum, one group ahead like the staging
  // (each group's scale is read and written by its own warp only)
  float s_nx = gi < groups ? s[gi] : 0.f, ms_nx = gi < groups ? ms[gi] : 0.f;
  cp_async_commit();
  for (int buf = 0; gi < groups; gi += nwarps, buf ^= 1) {
    const float sg = s_nx;
    const float msg = ms_nx;
    if (gi + nwarps < groups) {
      prefetch(gi + nwarps, buf ^ 1);
      s_nx = s[gi + nwarps];
      ms_nx = ms[gi + nwarps];
    }
    cp_async_commit();
    cp_async_wait<1>();  // this lane's copies of group gi have landed
    const uint8_t* sb = bwd_smem + wic * 2 * C::BUF + buf * C::BUF + 16 * lane;
    const uint8_t* sb_s = bwd_smem + wic * 2 * C::BUF + buf * C::BUF + (S16 ? 8 : 16) * lane;
    const int64_t c0 = gi * kGroup + 4 * lane;
    float Dr[4], Lr[L][4], Mr[L][4];
    *reinterpret_cast<float4*>(Dr) = *reinterpret_cast<const float4*>(sb);
#pragma unroll
    for (int p = 0; p < L; ++p) {
      if (S16) {
        const uint2 lu = *reinterpret_cast<const uint2*>(sb_s + C::OFF_L + p * C::SP);
        const uint2 mu = *reinterpret_cast<const uint2*>(sb_s + C::OFF_M + p * C::SP);
        Lr[p][0] = __uint_as_float(lu.x << 16);
        Lr[p][1] = __uint_as_float(lu.x & 0xFFFF0000u);
        Lr[p][2] = __uint_as_float(lu.y << 16);
        Lr[p][3] = __uint_as_float(lu.y & 0xFFFF0000u);
        Mr[p][0] = __uint_as_float(mu.x << 16);
        Mr[p][1] = __uint_as_float(mu.x & 0xFFFF0000u);
        Mr[p][2] = __uint_as_float(mu.y << 16);
        Mr[p][3] = __uint_as_float(mu.y & 0xFFFF0000u);
      } else {
        *reinterpret_cast<float4*>(Lr[p]) =
            *reinterpret_cast<const float4*>(sb + C::OFF_L + p * C::SP);
        *reinterpret_cast<float4*>(Mr[p]) =
            *reinterpret_cast<const float4*>(sb + C::OFF_M + p * C::SP);
      }
    }
    int lev[4] = {0, 0, 0, 0};
    if (MODE == GRID_3BIT_LOCAL) {
      const uint32_t b4 = *reinterpret_cast<const uint32_t*>(
          bwd_smem + wic * 2 * C::BUF + buf * C::BUF + C::OFF_I + 4 * lane);
#pragma unroll
      for (int j = 0; j < 4; ++j) lev[j] = (int)(int8_t)((b4 >> (8 * j)) & 0xFFu);
    }
    // pass 1: this step's probabilities (pre-update logits, words of step t),
    // gradients and Lion.  Philox counters take the global coordinate.
    const uint64_t gc0 = coord0 + (uint64_t)c0;
    uint32_t q1[4] = {0u, 0u, 0u, 0u};
    if (L == 5 && noise) block1_words(gc0, t, ks, q1);
    float ds_part = 0.f;
    float Do[DBG ? L : 1][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t wd[5] = {0u, 0u, 0u, 0u, 0u};
      if (noise) block0_words(gc0 + j, (uint32_t)(gc0 >> 32), t, ks, wd);
      wd[4] = q1[j];
      // e: unnormalised e_k (categorical) or the probabilities (ternary)
      float l[L], e[L], cand[5], r;
#pragma unroll
      for (int p = 0; p < L; ++p) l[p] = Lr[p][j];
      candidates<MODE>(lev[j], cand);
      const float v = coord_value<MODE>(l, wd, noise, inv_tau, l2cells, cand, e, &r);
      const float dw = Dr[j];
      ds_part = fmaf(dw, v, ds_part);
      const float a = sg * dw * inv_tau;
      float dl[L];
      if (MODE == GRID_TERNARY) {
        const float gm = a * (e[3] - e[2]) * e[1] * e[0];
        const float gs = 2.f * a * e[1] * e[3] * e[2];
        dl[0] = -gm;
        dl[1] = gm;
        dl[2] = -gs;
        dl[3] = gs;
      } else {
        // y_k = e_k r: dl_k = (a r^2) e_k sum_j e_j (c_k - c_j)
        //                   = (a r^2) e_k (c_k S - V),
        // S = sum_j e_j and V = sum_j e_j c_j (the sums coord_value formed,
        // in the same order)
        const float a2 = a * r * r;
        float S = 0.f, V = 0.f;
#pragma unroll
        for (int q = 0; q < L; ++q) S += e[q];
#pragma unroll
        for (int q = 0; q < L; ++q) V = fmaf(e[q], cand[q], V);
#pragma unroll
        for (int p = 0; p < L; ++p) dl[p] = a2 * e[p] * fmaf(cand[p], S, -V);
      }
#pragma unroll
      for (int p = 0; p < L; ++p) {
        float th = l[p], mm = Mr[p][j];
        lion_update(th, mm, dl[p], lr, b1, omb1, b2, omb2);
        Lr[p][j] = th;  // fp32; rounded in pass 2 with bf16 state
        Mr[p][j] = S16 ? bf16_rn(mm) : mm;
        if (DBG) Do[DBG ? p : 0][j] = dl[p];
      }
    }
#pragma unroll
    for (int p = 0; p < L; ++p) {
      if (S16) {
        // the values are bf16 already: keep their top halves
        *reinterpret_cast<uint2*>(mom + p * NK + c0) =
            make_uint2((__float_as_uint(Mr[p][0]) >> 16) | (__float_as_uint(Mr[p][1]) & 0xFFFF0000u),
                       (__float_as_uint(Mr[p][2]) >> 16) | (__float_as_uint(Mr[p][3]) & 0xFFFF0000u));
      } else {
        *reinterpret_cast<float4*>(logits + p * NK + c0) = *reinterpret_cast<float4*>(Lr[p]);
        *reinterpret_cast<float4*>(mom + p * NK + c0) = *reinterpret_cast<float4*>(Mr[p]);
      }
      if (DBG)
        *reinterpret_cast<float4*>(dl_dbg + p * NK + c0) =
            *reinterpret_cast<float4*>(Do[DBG ? p : 0]);
    }
    // every lane takes lane 0's sum so that all lanes hold the same new scale
    const float ds = __shfl_sync(0xffffffffu, warp_sum(ds_part), 0);
    float s_new = sg, ms_new = msg;
    lion_update(s_new, ms_new, ds, lr, b1, omb1, b2, omb2);
    if (lane == 0) {
      s[gi] = s_new;
      ms[gi] = ms_new;
      if (DBG) ds_dbg[gi] = ds;
    }
    // pass 2 (NEXT, or bf16 state): the words of step t + 1 give the
    // stochastic-rounding thresholds of the updated logits and the next
    // step's noise
    if (NEXT || S16) {
      uint32_t r1[4] = {0u, 0u, 0u, 0u};
      if (L == 5 && (S16 || noise)) block1_words(gc0, t1, ks, r1);
      float w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t wd[5] = {0u, 0u, 0u, 0u, 0u};
        if (S16 || noise) block0_words(gc0 + j, (uint32_t)(gc0 >> 32), t1, ks, wd);
        wd[4] = r1[j];
        float l[L];
#pragma unroll
        for (int p = 0; p < L; ++p) {
          if (S16) Lr[p][j] = bf16_sr(Lr[p][j], wd[p]);
          l[p] = Lr[p][j];
        }
        if (NEXT) {
          float e[L], cand[5], r;
          candidates<MODE>(lev[j], cand);
          w[j] = s_new * coord_value<MODE>(l, wd, noise, inv_tau_next, l2cells, cand, e, &r);
        }
      }
      if (S16) {
#pragma unroll
        for (int p = 0; p < L; ++p)
          *reinterpret_cast<uint2*>(logits + p * NK + c0) =
              make_uint2((__float_as_uint(Lr[p][0]) >> 16) | (__float_as_uint(Lr[p][1]) & 0xFFFF0000u),
                         (__float_as_uint(Lr[p][2]) >> 16) | (__float_as_uint(Lr[p][3]) & 0xFFFF0000u));
      }
      if (NEXT) store_bf16x4(What + c0, w);
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------- harden + pack (A6)

template <int MODE>
__device__ __forceinline__ int hard_level(const float* l, int lev0) {
  if (MODE == GRID_TERNARY) {
    const bool nonzero = l[1] > l[0];  // first maximum: ties -> zero
    const bool plus = l[3] > l[2];     // ties -> minus
    return nonzero ? (plus ? 2 : 0) : 1;
  }
  constexpr int L = GridT<MODE>::L;
  int best = 0;
#pragma unroll
  for (int k = 1; k < L; ++k)
    if (l[k] > l[best]) best = k;
  if (MODE == GRID_3BIT_LOCAL) return min(max(lev0 + best - 2, 0), 7);
  return best;
}

// ------------------------------------------------- scale-only step

// Level codes of the hard choice (argmax of the logits, no noise), four
// coordinates per thread.
template <int MODE, typename TS>
__global__ void __launch_bounds__(256) k_hard_codes(const TS* __restrict__ logits,
                                                    const int8_t* __restrict__ i0,
                                                    int64_t NK, int8_t* __restrict__ code) {
  constexpr int L = GridT<MODE>::L;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < NK / 4;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c0 = q * 4;
    float4 lp[L];
#pragma unroll
    for (int p = 0; p < L; ++p) lp[p] = St<TS>::ld4(logits + p * NK + c0);
    char4 iv = make_char4(0, 0, 0, 0);
    if (MODE == GRID_3BIT_LOCAL) iv = *reinterpret_cast<const char4*>(i0 + c0);
    const int lev0[4] = {iv.x, iv.y, iv.z, iv.w};
    int out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l[L];
#pragma unroll
      for (int p = 0; p < L; ++p)
        l[p] = j == 0 ? lp[p].x : j == 1 ? lp[p].y : j == 2 ? lp[p].z : lp[p].w;
      out[j] = hard_level<MODE>(l, lev0[j]);
    }
    *reinterpret_cast<char4*>(code + c0) =
        make_char4((signed char)out[0], (signed char)out[1], (signed char)out[2],
                   (signed char)out[3]);
  }
}

// w = bf16(s_g c_code), four coordinates per thread
template <int MODE>
__global__ void __launch_bounds__(256) k_code_weight(const int8_t* __restrict__ code,
                                                     const float* __restrict__ s, int64_t N,
                                                     int64_t K, __nv_bfloat16* __restrict__ What) {
  const int64_t NK = N * K, G = K / kGroup;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < NK / 4;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c0 = q * 4, n = c0 / K, k = c0 - n * K;
    const float sg = __ldg(s + n * G + k / kGroup);
    const char4 cv = *reinterpret_cast<const char4*>(code + c0);
    const float w[4] = {sg * GridT<MODE>::level(cv.x), sg * GridT<MODE>::level(cv.y),
                        sg * GridT<MODE>::level(cv.z), sg * GridT<MODE>::level(cv.w)};
    store_bf16x4(What + c0, w);
  }
}

// Scale-only backward + Lion: ds_g = sum over the group of dW_i c_code(i)
// (one warp per group, four consecutive coordinates per lane, warp-shuffle
// sum), then Lion on s and its momentum.
template <int MODE>
__global__ void __launch_bounds__(256) k_scale_lion(const int8_t* __restrict__ code,
                                                    const float* __restrict__ dW,
                                                    float* __restrict__ s,
                                                    float* __restrict__ ms, int64_t N,
                                                    int64_t K, float lr, float b1, float omb1,
                                                    float b2, float omb2,
                                                    float* __restrict__ ds_dbg) {
  const int64_t G = K / kGroup;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t gi = warp; gi < N * G; gi += nwarps) {
    const int64_t c0 = (gi / G) * K + (gi % G) * kGroup + 4 * lane;
    const float4 d4 = __ldg(reinterpret_cast<const float4*>(dW + c0));
    const char4 cv = *reinterpret_cast<const char4*>(code + c0);
    float part = d4.x * GridT<MODE>::level(cv.x);
    part = fmaf(d4.y, GridT<MODE>::level(cv.y), part);
    part = fmaf(d4.z, GridT<MODE>::level(cv.z), part);
    part = fmaf(d4.w, GridT<MODE>::level(cv.w), part);
    const float ds = __shfl_sync(0xffffffffu, warp_sum(part), 0);
    if (lane == 0) {
      float sv = s[gi], mv = ms[gi];
      lion_update(sv, mv, ds, lr, b1, omb1, b2, omb2);
      s[gi] = sv;
      ms[gi] = mv;
      if (ds_dbg) ds_dbg[gi] = ds;
    }
  }
}

// 2-bit / ternary: 16 codes -> one 32-bit word per thread.
// 3-bit: 32 codes -> three 32-bit words per thread.  Codes never straddle
// rows because K is a multiple of 128.
template <int MODE, typename TS>
__global__ void __launch_bounds__(256) k_harden_pack(
    const TS* __restrict__ logits, const int8_t* __restrict__ i0,
    int64_t N, int64_t K, uint32_t* __restrict__ packed) {
  constexpr int L = GridT<MODE>::L;
  constexpr int CPT = (MODE == GRID_3BIT_LOCAL) ? 32 : 16;  // codes / thread
  const int64_t NK = N * K, nthr = NK / CPT;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nthr;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c0 = q * CPT;
    uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
    for (int j4 = 0; j4 < CPT / 4; ++j4) {
      float4 lp[L];
#pragma unroll
      for (int p = 0; p < L; ++p)
        lp[p] = St<TS>::ld4(logits + p * NK + c0 + j4 * 4);
      char4 iv = make_char4(0, 0, 0, 0);
      if (MODE == GRID_3BIT_LOCAL)
        iv = __ldg(reinterpret_cast<const char4*>(i0 + c0 + j4 * 4));
      const int lev0[4] = {iv.x, iv.y, iv.z, iv.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float l[L];
#pragma unroll
        for (int p = 0; p < L; ++p)
          l[p] = j == 0 ? lp[p].x : j == 1 ? lp[p].y : j == 2 ? lp[p].z : lp[p].w;
        const uint32_t code = (uint32_t)hard_level<MODE>(l, lev0[j]);
        const int idx = j4 * 4 + j;
        if (MODE == GRID_3BIT_LOCAL) {
          const int bit = idx * 3;
          w[bit >> 5] |= code << (bit & 31);
          if ((bit & 31) > 29) w[(bit >> 5) + 1] |= code >> (32 - (bit & 31));
        } else {
          w[0] |= code << (idx * 2);
        }
      }
    }
    if (MODE == GRID_3BIT_LOCAL) {
      packed[q * 3 + 0] = w[0];
      packed[q * 3 + 1] = w[1];
      packed[q * 3 + 2] = w[2];
    } else {
      packed[q] = w[0];
    }
  }
}

// bf16(s * level) of the hard choice, four coordinates per thread
template <int MODE, typename TS>
__global__ void __launch_bounds__(256) k_hard_weight(
    const TS* __restrict__ logits, const float* __restrict__ s,
    const int8_t* __restrict__ i0, int64_t N, int64_t K,
    __nv_bfloat16* __restrict__ What) {
  constexpr int L = GridT<MODE>::L;
  const int64_t NK = N * K, G = K / kGroup, n4 = NK / 4;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < n4;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c0 = q * 4;
    const int64_t n = c0 / K, k = c0 - n * K;
    const float sg = s[n * G + k / kGroup];
    float4 lp[L];
#pragma unroll
    for (int p = 0; p < L; ++p) lp[p] = St<TS>::ld4(logits + p * NK + c0);
    char4 iv = make_char4(0, 0, 0, 0);
    if (MODE == GRID_3BIT_LOCAL) iv = *reinterpret_cast<const char4*>(i0 + c0);
    const int lev0[4] = {iv.x, iv.y, iv.z, iv.w};
    float wv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l[L];
#pragma unroll
      for (int p = 0; p < L; ++p)
        l[p] = j == 0 ? lp[p].x : j == 1 ? lp[p].y : j == 2 ? lp[p].z : lp[p].w;
      wv[j] = sg * GridT<MODE>::level(hard_level<MODE>(l, lev0[j]));
    }
    __nv_bfloat162 b01 = __floats2bfloat162_rn(wv[0], wv[1]);
    __nv_bfloat162 b23 = __floats2bfloat162_rn(wv[2], wv[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&b01);
    pk.y = *reinterpret_cast<uint32_t*>(&b23);
    *reinterpret_cast<uint2*>(What + c0) = pk;
  }
}

__global__ void k_export_scales(const float* __restrict__ s, int64_t n,
                                uint16_t* __restrict__ f16,
                                float* __restrict__ f32) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = s[i];
    if (f16) {
      const __half h = __float2half_rn(v);
      f16[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
    if (f32) f32[i] = v;
  }
}

template <int MODE>
__global__ void k_uniforms(uint64_t seed, uint32_t t, uint64_t coord0,
                           int64_t count, float* __restrict__ out) {
  constexpr int L = GridT<MODE>::L;
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t c = coord0 + (uint64_t)i;
    uint32_t w[5];
    coord_words5(c, t, k0, k1, L == 5, w);
#pragma unroll
    for (int p = 0; p < L; ++p) out[i * L + p] = word_to_unit(w[p]);
  }
}

// log2(u) of the uniforms u = (m + 1/2) 2^-23, m = m0 .. m0 + count - 1, as
// the noise of every step forms it (log2_unit on the word m << 9).
__global__ void __launch_bounds__(256) k_log2_unit(uint32_t m0, int64_t count,
                                                   float* __restrict__ out) {
  __shared__ float2 l2cells[kLog2Cells];
  log2_cells_init(l2cells);
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = log2_unit((m0 + (uint32_t)i) << 9, l2cells);
}

// sum of squares with per-block fp64 partials; the last block to finish
// adds the partials in block order (deterministic) and resets the ticket.
__global__ void __launch_bounds__(256) k_sumsq(const float* __restrict__ x,
                                               int64_t n,
                                               double* __restrict__ partials,
                                               unsigned* ticket,
                                               double* __restrict__ out) {
  __shared__ double red[8];
  __shared__ bool last;
  double acc = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double v = x[i];
    acc += v * v;
  }
  acc = warp_sum_d(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b += red[w];
    partials[blockIdx.x] = b;
    __threadfence();
    last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    double tot = 0.0;
    for (unsigned b = 0; b < gridDim.x; ++b)
      tot += *((volatile double*)partials + b);
    *out = tot;
    *ticket = 0u;
  }
}

// ------------------------------------------------------ SwiGLU pieces
// (the block's MLP stage: h = silu(a) * b and its derivatives)

__device__ __forceinline__ float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }


// hT = bf16(silu(aT) * bT), elementwise over n entries
__global__ void __launch_bounds__(256) k_swiglu_fwd(const float* __restrict__ a,
                                                    const float* __restrict__ b,
                                                    int64_t n,
                                                    __nv_bfloat16* __restrict__ h) {
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 a4 = __ldg(reinterpret_cast<const float4*>(a + i));
    const float4 b4 = __ldg(reinterpret_cast<const float4*>(b + i));
    const float hv[4] = {a4.x * sigmoidf_(a4.x) * b4.x, a4.y * sigmoidf_(a4.y) * b4.y,
                         a4.z * sigmoidf_(a4.z) * b4.z, a4.w * sigmoidf_(a4.w) * b4.w};
    store_bf16x4(h + i, hv);
  }
}

// da = bf16(dh * b * silu'(a)), db = bf16(dh * silu(a)),
// silu'(a) = sigma(a) (1 + a (1 - sigma(a)))
__global__ void __launch_bounds__(256) k_swiglu_bwd(const float* __restrict__ a,
                                                    const float* __restrict__ b,
                                                    const float* __restrict__ dh,
                                                    int64_t n,
                                                    __nv_bfloat16* __restrict__ da,
                                                    __nv_bfloat16* __restrict__ db) {
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 a4 = __ldg(reinterpret_cast<const float4*>(a + i));
    const float4 b4 = __ldg(reinterpret_cast<const float4*>(b + i));
    const float4 d4 = __ldg(reinterpret_cast<const float4*>(dh + i));
    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
    const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
    const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
    float ga[4], gb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float sg = sigmoidf_(av[j]);
      ga[j] = dv[j] * bv[j] * (sg * (1.f + av[j] * (1.f - sg)));
      gb[j] = dv[j] * av[j] * sg;
    }
    store_bf16x4(da + i, ga);
    store_bf16x4(db + i, gb);
  }
}

// out (cols x rows) = in (rows x cols)^T, 64 x 64 tiles through shared memory
template <typename TIn, typename TOut>
__global__ void k_transpose(const TIn* __restrict__ in, int64_t rows,
                            int64_t cols, TOut* __restrict__ out) {
  __shared__ float tile[64][65];
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 64 x 4
  for (int r = ty; r < 64; r += 4) {
    const int64_t rr = r0 + r, cc = c0 + tx;
    float v = 0.f;
    if (rr < rows && cc < cols) {
      if constexpr (sizeof(TIn) == 2)
        v = __bfloat162float(in[rr * cols + cc]);
      else
        v = in[rr * cols + cc];
    }
    tile[r][tx] = v;
  }
  __syncthreads();
  for (int c = ty; c < 64; c += 4) {
    const int64_t cc = c0 + c, rr = r0 + tx;
    if (cc < cols && rr < rows) {
      if constexpr (sizeof(TOut) == 2)
        out[cc * rows + rr] = __float2bfloat16_rn(tile[tx][c]);
      else
        out[cc * rows + rr] = tile[tx][c];
    }
  }
}

// ------------------------------------------------ attention V/O pieces

// Rotary embedding (rotate-half pairs (i, i + d/2), angle p theta^(-2i/d) at
// the position p = t % S within the sequence; angles in double precision) of
// an fp32 projection (T x cols, cols = heads * d), written as bf16.
__global__ void k_rope(const float* __restrict__ x, int64_t T, int64_t cols,
                       int64_t S, int d, double theta,
                       __nv_bfloat16* __restrict__ out) {
  const int half = d / 2;
  const int64_t pairs = T * (cols / 2);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < pairs;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / (cols / 2);
    const int64_t r = i % (cols / 2);
    const int64_t head = r / half;
    const int j = (int)(r % half);
    const int64_t c0 = head * d + j, c1 = c0 + half;
    const double ang = (double)(t % S) * pow(theta, -2.0 * (double)j / (double)d);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const float a = x[t * cols + c0], b = x[t * cols + c1];
    out[t * cols + c0] = __float2bfloat16_rn((float)((double)a * cs - (double)b * sn));
    out[t * cols + c1] = __float2bfloat16_rn((float)((double)b * cs + (double)a * sn));
  }
}

// Causal softmax of scaled scores: one block per query row q of one (s, h)
// slice (S x S fp32); P row written as bf16 (zeros above the diagonal).
__global__ void __launch_bounds__(256) k_causal_softmax(
    const float* __restrict__ scores, int64_t S, float scale,
    __nv_bfloat16* __restrict__ P) {
  __shared__ float red[32];
  const int64_t q = blockIdx.x;
  const float* row = scores + q * S;
  __nv_bfloat16* out = P + q * S;
  float mx = -INFINITY;
  for (int64_t k = threadIdx.x; k <= q; k += blockDim.x) mx = fmaxf(mx, row[k] * scale);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : -INFINITY;
    v = warp_max(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  mx = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int64_t k = threadIdx.x; k <= q; k += blockDim.x) sum += expf(row[k] * scale - mx);
  sum = warp_sum(sum);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv = 1.f / red[0];
  for (int64_t k = threadIdx.x; k < S; k += blockDim.x)
    out[k] = __float2bfloat16_rn(k <= q ? expf(row[k] * scale - mx) * inv : 0.f);
}

// out[c * ld_out + r] = in[r * ld_in + c] for an rows x cols bf16 block
__global__ void k_transpose_ld(const __nv_bfloat16* __restrict__ in, int64_t rows,
                               int64_t cols, int64_t ld_in,
                               __nv_bfloat16* __restrict__ out, int64_t ld_out) {
  __shared__ __nv_bfloat16 tile[64][66];
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 64 x 4
  for (int r = ty; r < 64; r += 4) {
    const int64_t rr = r0 + r, cc = c0 + tx;
    tile[r][tx] = (rr < rows && cc < cols) ? in[rr * ld_in + cc] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  for (int c = ty; c < 64; c += 4) {
    const int64_t cc = c0 + c, rr = r0 + tx;
    if (cc < cols && rr < rows) out[cc * ld_out + rr] = tile[tx][c];
  }
}

// The same transpose with 16-byte accesses (rows, cols, ld_in, ld_out and
// both pointers multiples of 8 elements / 16 bytes): a 64 x 64 tile per
// iteration, held in shared memory as 32-bit words (two neighbouring
// columns); an output word pairs rows 2p and 2p + 1 of one column, taken
// from two words with one byte permute.  Each lane writes 32 contiguous
// output bytes (16 rows of one column).
__global__ void __launch_bounds__(256) k_transpose_b16v(
    const __nv_bfloat16* __restrict__ in, int64_t rows, int64_t cols,
    int64_t ld_in, __nv_bfloat16* __restrict__ out, int64_t ld_out) {
  __shared__ uint32_t tile[64][33];
  const int tid = threadIdx.x;
  const int64_t tr = (rows + 63) / 64, tc = (cols + 63) / 64;
  for (int64_t t = blockIdx.x; t < tr * tc; t += gridDim.x) {
    const int64_t r0 = (t / tc) * 64, c0 = (t % tc) * 64;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int id = tid + 256 * i, r = id >> 3, ch = id & 7;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r0 + r < rows && c0 + ch * 8 < cols)
        v = __ldg(reinterpret_cast<const uint4*>(in + (r0 + r) * ld_in + c0 + ch * 8));
      tile[r][ch * 4] = v.x;
      tile[r][ch * 4 + 1] = v.y;
      tile[r][ch * 4 + 2] = v.z;
      tile[r][ch * 4 + 3] = v.w;
    }
    __syncthreads();
    {
      const int c = tid & 63, q = tid >> 6;  // output row c0 + c, rows 16 q ..
      const uint32_t sel = (c & 1) ? 0x7632u : 0x5410u;  // high or low halves
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int r = 16 * q + 2 * k;
        w[k] = __byte_perm(tile[r][c >> 1], tile[r + 1][c >> 1], sel);
      }
      if (c0 + c < cols) {
        __nv_bfloat16* o = out + (c0 + c) * ld_out + r0 + 16 * q;
        if (r0 + 16 * q < rows)
          *reinterpret_cast<uint4*>(o) = make_uint4(w[0], w[1], w[2], w[3]);
        if (r0 + 16 * q + 8 < rows)
          *reinterpret_cast<uint4*>(o + 8) = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    __syncthreads();
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ in, int64_t n,
                              __nv_bfloat16* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(in[i]);
}

int grid_for(int64_t work, int threads, int cap) {
  int64_t b = (work + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return (int)b;
}

}  // namespace

// ------------------------------------------------------------ launchers

cudaError_t launch_convert_x(const void* X, int dtype, int64_t T, int64_t K,
                             int64_t Tp, __nv_bfloat16* Xb, __nv_bfloat16* Xt,
                             __nv_bfloat16* Xcat, int* err, cudaStream_t st) {
  dim3 grid((unsigned)((K + 63) / 64), (unsigned)((Tp + 63) / 64));
  k_convert_x<<<grid, dim3(64, 4), 0, st>>>(X, dtype, T, K, Tp, Xb, Xt, Xcat,
                                            err);
  return cudaGetLastError();
}

cudaError_t launch_convert_w(const void* W, int dtype, int64_t N, int64_t K,
                             float* W32, __nv_bfloat16* Wop, int split,
                             int* err, cudaStream_t st) {
  k_convert_w<<<grid_for(N * K, 256, 4096), 256, 0, st>>>(W, dtype, N, K, W32,
                                                          Wop, split, err);
  return cudaGetLastError();
}

cudaError_t launch_init_state(int mode, const float* W32,
                              const int8_t* init_idx, int64_t N, int64_t K,
                              float* s, int8_t* i0, float* logits, int* err,
                              cudaStream_t st, int state16) {
  const int64_t groups = N * (K / kGroup);
  const int blocks = grid_for(groups * 32, 256, 8192);
  __nv_bfloat16* l16 = reinterpret_cast<__nv_bfloat16*>(logits);
  switch (mode * 2 + (state16 ? 1 : 0)) {
    case GRID_2BIT * 2:
      k_init_state<GRID_2BIT, float><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, logits, err);
      break;
    case GRID_2BIT * 2 + 1:
      k_init_state<GRID_2BIT, __nv_bfloat16><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, l16, err);
      break;
    case GRID_TERNARY * 2:
      k_init_state<GRID_TERNARY, float><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, logits, err);
      break;
    case GRID_TERNARY * 2 + 1:
      k_init_state<GRID_TERNARY, __nv_bfloat16><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, l16, err);
      break;
    case GRID_3BIT_LOCAL * 2:
      k_init_state<GRID_3BIT_LOCAL, float><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, logits, err);
      break;
    default:
      k_init_state<GRID_3BIT_LOCAL, __nv_bfloat16><<<blocks, 256, 0, st>>>(W32, init_idx, N, K, s, i0, l16, err);
  }
  return cudaGetLastError();
}

template <int MODE, typename TS>
static void soft_weight_ts(const StepArgs& a, __nv_bfloat16* What, float* wsoft32, int blocks,
                           cudaStream_t st) {
  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32);
  const float inv_tau = 1.0f / a.tau;
  const TS* lg = reinterpret_cast<const TS*>(a.logits);
  if (wsoft32)
    k_soft_weight<MODE, true, TS><<<blocks, 256, 0, st>>>(lg, a.s, a.i0, a.N, a.K,
                                                          philox_keys(k0, k1), a.coord0, a.t,
                                                          a.noise, inv_tau, What, wsoft32);
  else
    k_soft_weight<MODE, false, TS><<<blocks, 256, 0, st>>>(lg, a.s, a.i0, a.N, a.K,
                                                           philox_keys(k0, k1), a.coord0, a.t,
                                                           a.noise, inv_tau, What, nullptr);
}

template <int MODE>
static void soft_weight_mode(const StepArgs& a, __nv_bfloat16* What, float* wsoft32, int blocks,
                             cudaStream_t st) {
  if (a.state16)
    soft_weight_ts<MODE, __nv_bfloat16>(a, What, wsoft32, blocks, st);
  else
    soft_weight_ts<MODE, float>(a, What, wsoft32, blocks, st);
}

cudaError_t launch_soft_weight(const StepArgs& a, __nv_bfloat16* What, float* wsoft32,
                               int sm_count, cudaStream_t st) {
  const int64_t groups = a.N * (a.K / kGroup);
  const int blocks = grid_for(groups * 32, 256, sm_count * 8);
  switch (a.mode) {
    case GRID_2BIT: soft_weight_mode<GRID_2BIT>(a, What, wsoft32, blocks, st); break;
    case GRID_TERNARY: soft_weight_mode<GRID_TERNARY>(a, What, wsoft32, blocks, st); break;
    default: soft_weight_mode<GRID_3BIT_LOCAL>(a, What, wsoft32, blocks, st);
  }
  return cudaGetLastError();
}

template <int MODE, bool NEXT, typename TS>
static void backward_mode(const StepArgs& a, const float* dW, float lr, float b1, float b2, float tau_next,
                          __nv_bfloat16* What, float* dl_dbg, float* ds_dbg,
                          int blocks, cudaStream_t st) {
  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32);
  const float inv_tau = 1.0f / a.tau;
  const float inv_tau_next = NEXT ? 1.0f / tau_next : 0.f;
  const float omb1 = 1.0f - b1, omb2 = 1.0f - b2;
  using C = BwdCfg<MODE, TS>;
  TS* lg = reinterpret_cast<TS*>(a.logits_w);
  TS* mm = reinterpret_cast<TS*>(a.mom);
  // a failed opt-in leaves the launch to fail, and the launcher's caller
  // reads that error from cudaGetLastError
  // launched with programmatic stream serialisation: the CTAs start as the
  // weight-gradient GEMM's finish and wait in the kernel for its dW
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(C::WARPS * 32);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dl_dbg) {
    smem_optin<k_backward_lion<MODE, true, NEXT, TS>>(C::SMEM);
    cudaLaunchKernelEx(&cfg, k_backward_lion<MODE, true, NEXT, TS>, lg, mm, a.s, a.ms, a.i0,
                       dW, a.N, a.K, philox_keys(k0, k1), a.coord0, a.t, a.noise, inv_tau,
                       inv_tau_next, lr, b1, omb1, b2, omb2, What, dl_dbg, ds_dbg);
  } else {
    smem_optin<k_backward_lion<MODE, false, NEXT, TS>>(C::SMEM);
    cudaLaunchKernelEx(&cfg, k_backward_lion<MODE, false, NEXT, TS>, lg, mm, a.s, a.ms, a.i0,
                       dW, a.N, a.K, philox_keys(k0, k1), a.coord0, a.t, a.noise, inv_tau,
                       inv_tau_next, lr, b1, omb1, b2, omb2, What, (float*)nullptr,
                       (float*)nullptr);
  }
}

template <int MODE>
static void backward_dispatch(const StepArgs& a, const float* dW, float lr, float b1, float b2, float tau_next,
                              __nv_bfloat16* What, float* dl_dbg,
                              float* ds_dbg, int blocks, cudaStream_t st) {
  const bool next = tau_next > 0.f;
  if (a.state16) {
    if (next)
      backward_mode<MODE, true, __nv_bfloat16>(a, dW, lr, b1, b2, tau_next, What, dl_dbg,
                                               ds_dbg, blocks, st);
    else
      backward_mode<MODE, false, __nv_bfloat16>(a, dW, lr, b1, b2, tau_next, What,
                                                dl_dbg, ds_dbg, blocks, st);
  } else {
    if (next)
      backward_mode<MODE, true, float>(a, dW, lr, b1, b2, tau_next, What, dl_dbg, ds_dbg,
                                       blocks, st);
    else
      backward_mode<MODE, false, float>(a, dW, lr, b1, b2, tau_next, What, dl_dbg,
                                        ds_dbg, blocks, st);
  }
}

cudaError_t launch_backward_lion(const StepArgs& a, const float* dW, float lr, float b1, float b2,
                                 float tau_next, __nv_bfloat16* What,
                                 float* dl_dbg, float* ds_dbg, int sm_count,
                                 cudaStream_t st) {
  const int64_t groups = a.N * (a.K / kGroup);
  // persistent: as many CTAs as fit on the SMs at once, fewer for small layers
  auto blocks_for = [&](int warps, int ctas) {
    const int64_t need = (groups + warps - 1) / warps;
    const int64_t cap = (int64_t)sm_count * ctas;
    return (int)(need < cap ? need : cap);
  };
  const int blocks = a.mode == GRID_3BIT_LOCAL
                         ? blocks_for(BwdCfg<GRID_3BIT_LOCAL>::WARPS, BwdCfg<GRID_3BIT_LOCAL>::CTAS)
                         : blocks_for(BwdCfg<GRID_2BIT>::WARPS, BwdCfg<GRID_2BIT>::CTAS);
  switch (a.mode) {
    case GRID_2BIT: backward_dispatch<GRID_2BIT>(a, dW, lr, b1, b2, tau_next, What, dl_dbg, ds_dbg, blocks, st); break;
    case GRID_TERNARY: backward_dispatch<GRID_TERNARY>(a, dW, lr, b1, b2, tau_next, What, dl_dbg, ds_dbg, blocks, st); break;
    default: backward_dispatch<GRID_3BIT_LOCAL>(a, dW, lr, b1, b2, tau_next, What, dl_dbg, ds_dbg, blocks, st);
  }
  return cudaGetLastError();
}

cudaError_t launch_hard_weight(int mode, int64_t N, int64_t K,
                               const float* logits, const float* s,
                               const int8_t* i0, __nv_bfloat16* What,
                               cudaStream_t st, int state16) {
  const int blocks = grid_for(N * K / 4, 256, 4096);
  const __nv_bfloat16* l16 = reinterpret_cast<const __nv_bfloat16*>(logits);
  switch (mode * 2 + (state16 ? 1 : 0)) {
    case GRID_2BIT * 2: k_hard_weight<GRID_2BIT, float><<<blocks, 256, 0, st>>>(logits, s, i0, N, K, What); break;
    case GRID_2BIT * 2 + 1: k_hard_weight<GRID_2BIT, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, s, i0, N, K, What); break;
    case GRID_TERNARY * 2: k_hard_weight<GRID_TERNARY, float><<<blocks, 256, 0, st>>>(logits, s, i0, N, K, What); break;
    case GRID_TERNARY * 2 + 1: k_hard_weight<GRID_TERNARY, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, s, i0, N, K, What); break;
    case GRID_3BIT_LOCAL * 2: k_hard_weight<GRID_3BIT_LOCAL, float><<<blocks, 256, 0, st>>>(logits, s, i0, N, K, What); break;
    default: k_hard_weight<GRID_3BIT_LOCAL, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, s, i0, N, K, What);
  }
  return cudaGetLastError();
}

cudaError_t launch_hard_codes(int mode, int64_t N, int64_t K, const float* logits,
                              const int8_t* i0, int8_t* code, cudaStream_t st, int state16) {
  const int blocks = grid_for(N * K / 4, 256, 4096);
  const __nv_bfloat16* l16 = reinterpret_cast<const __nv_bfloat16*>(logits);
  switch (mode * 2 + (state16 ? 1 : 0)) {
    case GRID_2BIT * 2: k_hard_codes<GRID_2BIT, float><<<blocks, 256, 0, st>>>(logits, i0, N * K, code); break;
    case GRID_2BIT * 2 + 1: k_hard_codes<GRID_2BIT, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, i0, N * K, code); break;
    case GRID_TERNARY * 2: k_hard_codes<GRID_TERNARY, float><<<blocks, 256, 0, st>>>(logits, i0, N * K, code); break;
    case GRID_TERNARY * 2 + 1: k_hard_codes<GRID_TERNARY, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, i0, N * K, code); break;
    case GRID_3BIT_LOCAL * 2: k_hard_codes<GRID_3BIT_LOCAL, float><<<blocks, 256, 0, st>>>(logits, i0, N * K, code); break;
    default: k_hard_codes<GRID_3BIT_LOCAL, __nv_bfloat16><<<blocks, 256, 0, st>>>(l16, i0, N * K, code);
  }
  return cudaGetLastError();
}

cudaError_t launch_code_weight(int mode, int64_t N, int64_t K, const int8_t* code,
                               const float* s, __nv_bfloat16* What, cudaStream_t st) {
  const int blocks = grid_for(N * K / 4, 256, 4096);
  switch (mode) {
    case GRID_2BIT: k_code_weight<GRID_2BIT><<<blocks, 256, 0, st>>>(code, s, N, K, What); break;
    case GRID_TERNARY: k_code_weight<GRID_TERNARY><<<blocks, 256, 0, st>>>(code, s, N, K, What); break;
    default: k_code_weight<GRID_3BIT_LOCAL><<<blocks, 256, 0, st>>>(code, s, N, K, What);
  }
  return cudaGetLastError();
}

cudaError_t launch_scale_lion(int mode, int64_t N, int64_t K, const int8_t* code,
                              const float* dW, float* s, float* ms, float lr, float b1,
                              float b2, float* ds_dbg, int sm_count, cudaStream_t st) {
  const int64_t groups = N * (K / kGroup);
  const int blocks = grid_for(groups * 32, 256, sm_count * 8);
  const float omb1 = 1.0f - b1, omb2 = 1.0f - b2;
  switch (mode) {
    case GRID_2BIT:
      k_scale_lion<GRID_2BIT><<<blocks, 256, 0, st>>>(code, dW, s, ms, N, K, lr, b1, omb1, b2,
                                                     omb2, ds_dbg);
      break;
    case GRID_TERNARY:
      k_scale_lion<GRID_TERNARY><<<blocks, 256, 0, st>>>(code, dW, s, ms, N, K, lr, b1, omb1,
                                                        b2, omb2, ds_dbg);
      break;
    default:
      k_scale_lion<GRID_3BIT_LOCAL><<<blocks, 256, 0, st>>>(code, dW, s, ms, N, K, lr, b1,
                                                           omb1, b2, omb2, ds_dbg);
  }
  return cudaGetLastError();
}

cudaError_t launch_harden_pack(int mode, int64_t N, int64_t K,
                               const float* logits, const int8_t* i0,
                               uint32_t* packed, cudaStream_t st, int state16) {
  const __nv_bfloat16* l16 = reinterpret_cast<const __nv_bfloat16*>(logits);
  const int b16 = grid_for(N * K / 16, 256, 4096), b32 = grid_for(N * K / 32, 256, 4096);
  switch (mode * 2 + (state16 ? 1 : 0)) {
    case GRID_2BIT * 2: k_harden_pack<GRID_2BIT, float><<<b16, 256, 0, st>>>(logits, i0, N, K, packed); break;
    case GRID_2BIT * 2 + 1: k_harden_pack<GRID_2BIT, __nv_bfloat16><<<b16, 256, 0, st>>>(l16, i0, N, K, packed); break;
    case GRID_TERNARY * 2: k_harden_pack<GRID_TERNARY, float><<<b16, 256, 0, st>>>(logits, i0, N, K, packed); break;
    case GRID_TERNARY * 2 + 1: k_harden_pack<GRID_TERNARY, __nv_bfloat16><<<b16, 256, 0, st>>>(l16, i0, N, K, packed); break;
    case GRID_3BIT_LOCAL * 2: k_harden_pack<GRID_3BIT_LOCAL, float><<<b32, 256, 0, st>>>(logits, i0, N, K, packed); break;
    default: k_harden_pack<GRID_3BIT_LOCAL, __nv_bfloat16><<<b32, 256, 0, st>>>(l16, i0, N, K, packed);
  }
  return cudaGetLastError();
}

cudaError_t launch_export_scales(const float* s, int64_t n, uint16_t* f16,
                                 float* f32, cudaStream_t st) {
  k_export_scales<<<grid_for(n, 256, 1024), 256, 0, st>>>(s, n, f16, f32);
  return cudaGetLastError();
}

cudaError_t launch_uniforms(int mode, uint64_t seed, uint32_t t,
                            uint64_t coord0, int64_t count, float* out,
                            cudaStream_t st) {
  const int blocks = grid_for(count, 256, 4096);
  switch (mode) {
    case GRID_2BIT: k_uniforms<GRID_2BIT><<<blocks, 256, 0, st>>>(seed, t, coord0, count, out); break;
    case GRID_TERNARY: k_uniforms<GRID_TERNARY><<<blocks, 256, 0, st>>>(seed, t, coord0, count, out); break;
    default: k_uniforms<GRID_3BIT_LOCAL><<<blocks, 256, 0, st>>>(seed, t, coord0, count, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_log2_unit(uint32_t m0, int64_t count, float* out, cudaStream_t st) {
  k_log2_unit<<<grid_for(count, 256, 4096), 256, 0, st>>>(m0, count, out);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_fwd(const float* a, const float* b, int64_t n,
                              __nv_bfloat16* h, int sm_count, cudaStream_t st) {
  k_swiglu_fwd<<<grid_for(n / 4, 256, sm_count * 8), 256, 0, st>>>(a, b, n, h);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_bwd(const float* a, const float* b, const float* dh,
                              int64_t n, __nv_bfloat16* da, __nv_bfloat16* db,
                              int sm_count, cudaStream_t st) {
  k_swiglu_bwd<<<grid_for(n / 4, 256, sm_count * 8), 256, 0, st>>>(a, b, dh, n, da, db);
  return cudaGetLastError();
}

namespace {
bool b16v_ok(const void* in, int64_t rows, int64_t cols, int64_t ld_in,
             const void* out, int64_t ld_out) {
  return rows % 8 == 0 && cols % 8 == 0 && ld_in % 8 == 0 && ld_out % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(in) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(out) & 15) == 0;
}
cudaError_t launch_b16v(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                        int64_t ld_in, __nv_bfloat16* out, int64_t ld_out,
                        cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ((rows + 63) / 64) * ((cols + 63) / 64);
  const int64_t cap = (int64_t)sms * 8;
  k_transpose_b16v<<<(unsigned)(tiles < cap ? tiles : cap), 256, 0, st>>>(in, rows, cols,
                                                                         ld_in, out, ld_out);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_transpose_bf16(const __nv_bfloat16* in, int64_t rows,
                                  int64_t cols, __nv_bfloat16* out,
                                  cudaStream_t st) {
  if (rows > 0 && cols > 0 && b16v_ok(in, rows, cols, cols, out, rows))
    return launch_b16v(in, rows, cols, cols, out, rows, st);
  dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
  k_transpose<__nv_bfloat16, __nv_bfloat16><<<grid, dim3(64, 4), 0, st>>>(in, rows, cols, out);
  return cudaGetLastError();
}

cudaError_t launch_transpose_to_f32(const void* in, int in_bf16, int64_t rows,
                                    int64_t cols, float* out, cudaStream_t st) {
  dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
  if (in_bf16)
    k_transpose<__nv_bfloat16, float><<<grid, dim3(64, 4), 0, st>>>(
        (const __nv_bfloat16*)in, rows, cols, out);
  else
    k_transpose<float, float><<<grid, dim3(64, 4), 0, st>>>((const float*)in, rows, cols, out);
  return cudaGetLastError();
}

cudaError_t launch_rope(const float* x, int64_t T, int64_t cols, int64_t S, int d,
                        double theta, __nv_bfloat16* out, int sm_count, cudaStream_t st) {
  k_rope<<<grid_for(T * cols / 2, 256, sm_count * 8), 256, 0, st>>>(x, T, cols, S, d, theta, out);
  return cudaGetLastError();
}

cudaError_t launch_causal_softmax(const float* scores, int64_t S, float scale,
                                  __nv_bfloat16* P, cudaStream_t st) {
  k_causal_softmax<<<(unsigned)S, 256, 0, st>>>(scores, S, scale, P);
  return cudaGetLastError();
}

cudaError_t launch_transpose_ld(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                int64_t ld_in, __nv_bfloat16* out, int64_t ld_out,
                                cudaStream_t st) {
  if (rows > 0 && cols > 0 && b16v_ok(in, rows, cols, ld_in, out, ld_out))
    return launch_b16v(in, rows, cols, ld_in, out, ld_out, st);
  dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows + 63) / 64));
  k_transpose_ld<<<grid, dim3(64, 4), 0, st>>>(in, rows, cols, ld_in, out, ld_out);
  return cudaGetLastError();
}

cudaError_t launch_f32_to_bf16(const float* in, int64_t n, __nv_bfloat16* out,
                               int sm_count, cudaStream_t st) {
  k_f32_to_bf16<<<grid_for(n, 256, sm_count * 8), 256, 0, st>>>(in, n, out);
  return cudaGetLastError();
}

cudaError_t launch_sumsq(const float* x, int64_t n, double* partials,
                         unsigned* ticket, double* out, cudaStream_t st) {
  k_sumsq<<<grid_for(n, 256, 1024), 256, 0, st>>>(x, n, partials, ticket, out);
  return cudaGetLastError();
}

}  // namespace gsq
