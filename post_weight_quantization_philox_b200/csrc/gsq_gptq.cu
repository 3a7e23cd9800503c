// gsq_gptq.cu -- GPTQ initial assignment for the GSQ grids on the GPU.
//
// GSQ starts its logits from a GPTQ solution (agihunt.info summary,
// optimisation paragraph).  GPTQ is the algorithm of Frantar, Ashkboos,
// Hoefler and Alistarh ("GPTQ: Accurate Post-Training Quantization for
// Generative Pre-trained Transformers", ICLR 2023): columns are quantized in
// input order and each column's rounding error is pushed onto the columns
// not yet quantized through U, the upper Cholesky factor of H^-1
// (H^-1 = U^T U, H = X^T X damped).  Here, for the symmetric group-128 GSQ
// grids, in fp32:
//
//   H      = Xt Xt^T on the tensor cores (bf16 operands, fp32 accumulation)
//   dead inputs (H_ii = 0): H_ii = 1, W[:, i] = 0; H_ii += damp mean(diag H)
//   U      = J L^-1 J with L L^T = J H J (J reverses the index order), so
//            U^T U = J (J H J)^-1 J = H^-1 and U is upper triangular;
//            L from a blocked right-looking Cholesky (64 x 64 diagonal
//            blocks in one CTA, the panel times the block's inverse, the
//            trailing update on the tensor cores), L^-1 by block forward
//            substitution (the row block times the diagonal block's inverse,
//            the update of the later row blocks on the tensor cores)
//   per group of 128 columns: one thread per row carries the row's 128
//            weights in shared memory, sets the group scale absmax / c_max
//            from the updated weights, rounds each column to the nearest
//            level (first on ties) and feeds its error
//            e_j = (w_j - s c) / U_jj forward within the group; the error
//            block E (128 x N) then updates every later column at once:
//            W[:, j1:] -= E^T U[j0:j1, j1:]   (tensor cores)
//
// The tensor-core updates keep fp32 accuracy: each fp32 operand is split
// into three bf16 terms and every product is formed from six bf16 products
// (one GEMM of six-fold depth, fp32 accumulation) whose epilogue subtracts
// the result from the fp32 matrix in place.  The small products with the
// diagonal blocks' inverses stay on a SIMT fp32 kernel.
//
// This runs once per layer before the reconstruction steps; none of it is on
// the per-step path.
#include <cmath>
#include <vector>

#include "../../include/gsq.h"
#include "gsq_device.cuh"
#include "gsq_internal.h"
#include "gsq_stage.h"

namespace gsq {
namespace {

constexpr int kNb = 64;     // Cholesky / inverse block
constexpr int kCols = 128;  // GPTQ column block (= the quantization group)

int grid_cap(int64_t work, int threads, int cap) {
  const int64_t b = (work + threads - 1) / threads;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

// dead inputs (H_ii = 0 -> 1, flagged), then H_ii += damp * mean(diag H);
// one block
__global__ void k_gptq_damp(float* __restrict__ H, int64_t K, float damp,
                            int* __restrict__ dead) {
  __shared__ double red[32];
  double sum = 0.0;
  for (int64_t i = threadIdx.x; i < K; i += blockDim.x) {
    float d = H[i * K + i];
    const int z = d == 0.f;
    dead[i] = z;
    if (z) {
      d = 1.f;
      H[i * K + i] = 1.f;
    }
    sum += (double)d;
  }
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float add = (float)((double)damp * red[0] / (double)K);
  for (int64_t i = threadIdx.x; i < K; i += blockDim.x) H[i * K + i] += add;
}

__global__ void k_zero_dead_cols(float* __restrict__ W, int64_t N, int64_t K,
                                 const int* __restrict__ dead) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < N * K;
       i += (int64_t)gridDim.x * blockDim.x)
    if (dead[i % K]) W[i] = 0.f;
}

// dst[i][j] = src[K-1-i][K-1-j]
__global__ void k_reverse(const float* __restrict__ src, float* __restrict__ dst, int64_t K) {
  const int64_t KK = K * K;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < KK;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[KK - 1 - i];
}

// Lower Cholesky factor L of the 64 x 64 diagonal block at (k0, k0), in place
// (lower triangle only), right-looking, and X = L^-T into Xinv (64 x 64,
// row-major).  64 threads, thread r holding row r of the block in registers
// (every loop below is unrolled, so the row is indexed statically):
//   column c: thread c takes the pivot's square root, every row r > c forms
//   l_rc = a_rc / sqrt(a_cc) and publishes it, then each row takes the
//   rank-1 update a_rs -= l_rc l_sc of its entries c < s <= r;
//   row r of X solves x L^T = e_r by forward substitution
//   (x_c = (delta_rc - sum_{s<c} x_s L_cs) / L_cc, x_c = 0 for c < r, so the
//   dot product needs no bound on s).
// A pivot that is not positive is recorded and replaced by 1 so that nothing
// downstream turns into NaN.  The triangular solves against L become GEMMs
// with X.
constexpr int kPotrfThreads = kNb;
__global__ void __launch_bounds__(kPotrfThreads) k_potrf64(float* __restrict__ A, int64_t K,
                                                           int64_t k0, int* __restrict__ err,
                                                           float* __restrict__ Xinv) {
  __shared__ float ls[kNb][kNb + 1];  // the block (rows), then L
  __shared__ float col[kNb];          // the current column of L
  __shared__ float piv;               // its diagonal entry
  const int r = threadIdx.x;
  {
    // coalesced: thread r loads column r of each row, all 64 loads in
    // flight before the first store (the block is often not in L2)
    float v[kNb];
#pragma unroll
    for (int i = 0; i < kNb; ++i) v[i] = A[(k0 + i) * K + k0 + r];
#pragma unroll
    for (int i = 0; i < kNb; ++i) ls[i][r] = v[i];
  }
  __syncthreads();
  float a[kNb];
#pragma unroll
  for (int s = 0; s < kNb; ++s) a[s] = s <= r ? ls[r][s] : 0.f;
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kNb; ++c) {
    if (r == c) {
      float d = a[c];
      const bool bad = !(d > 0.f) || !isfinite(d);
      if (bad) {
        d = 1.f;
        atomicCAS(err, 0, DEV_ERR_NONFINITE);
      }
      piv = sqrtf(d);
    }
    // the pivot's root; every row is also done with the previous column's
    // update, so col can be rewritten (and piv was read before the barrier
    // below in the previous column)
    __syncthreads();
    const float sd = piv;
    const float l = r > c ? a[c] / sd : (r == c ? sd : 0.f);
    if (r > c) col[r] = l;
    __syncthreads();  // the column
    if (r >= c) a[c] = l;
#pragma unroll
    for (int s = c + 1; s < kNb; ++s)
      if (r > c && s <= r) a[s] -= l * col[s];
  }
#pragma unroll
  for (int s = 0; s < kNb; ++s) ls[r][s] = s <= r ? a[s] : 0.f;
  __syncthreads();
  for (int i = 0; i < kNb; ++i)
    if (r <= i) A[(k0 + i) * K + k0 + r] = ls[i][r];
  // X = L^-T, row r in registers; four partial sums for the dot products
  float x[kNb];
#pragma unroll
  for (int c = 0; c < kNb; ++c) {
    float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
    for (int q = 0; q + 3 < c; q += 4) {
      p0 = fmaf(x[q], ls[c][q], p0);
      p1 = fmaf(x[q + 1], ls[c][q + 1], p1);
      p2 = fmaf(x[q + 2], ls[c][q + 2], p2);
      p3 = fmaf(x[q + 3], ls[c][q + 3], p3);
    }
#pragma unroll
    for (int q = c & ~3; q < c; ++q) p0 = fmaf(x[q], ls[c][q], p0);
    const float part = (p0 + p1) + (p2 + p3);
    x[c] = c < r ? 0.f : ((c == r ? 1.f : 0.f) - part) / ls[c][c];
  }
  __syncthreads();  // L is read by every thread above; reuse ls for X
#pragma unroll
  for (int c = 0; c < kNb; ++c) ls[r][c] = x[c];
  __syncthreads();
  for (int i = 0; i < kNb; ++i) Xinv[i * kNb + r] = ls[i][r];
}

// C[m][n] -= sum_k A(m, k) B(k, n) (or =, with assign) with A(m, k) = A[m a_rs + k a_cs] and
// B(k, n) = B[k b_rs + n b_cs]; C has leading dimension ldc; Kd % 8 == 0.
// 128 x 128 tiles, 8-deep K slices double-buffered in shared memory (the
// next slice is fetched into registers while the current one computes),
// 8 x 8 outputs per thread in two 4-wide row and column strips 64 apart (so
// the shared-memory reads of a warp are contiguous 16-byte vectors).  Global
// reads run along whichever operand axis is contiguous (a_cs == 1: along k,
// else along m; likewise for B), so they coalesce at every call site.  With
// lower, tiles wholly above the diagonal (n0 > m0 + 127) are skipped.
struct SubGemm {
  int64_t M, N, Kd;
  const float* A;
  int64_t a_rs, a_cs;
  const float* B;
  int64_t b_rs, b_cs;
  float* C;
  int64_t ldc;
  int lower;
  int assign = 0;  // C = A B instead of C -= A B
};

constexpr int kGT = 128, kGK = 8;

__global__ void __launch_bounds__(256) k_gemm_sub(const SubGemm g) {
  __shared__ __align__(16) float as[2][kGK][kGT + 4];
  __shared__ __align__(16) float bs[2][kGK][kGT + 4];
  const int64_t m0 = (int64_t)blockIdx.y * kGT, n0 = (int64_t)blockIdx.x * kGT;
  if (g.lower && n0 > m0 + kGT - 1) return;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const bool a_k = g.a_cs == 1, b_k = g.b_rs == 1;
  // this thread's four elements of each slice: (row of the tile, k)
  auto a_pos = [&](int e, int& mm, int& kk) {
    const int idx = tid + 256 * e;  // 0..1023
    if (a_k) { kk = idx & 7; mm = idx >> 3; } else { mm = idx & 127; kk = idx >> 7; }
  };
  auto b_pos = [&](int e, int& nn, int& kk) {
    const int idx = tid + 256 * e;
    if (b_k) { kk = idx & 7; nn = idx >> 3; } else { nn = idx & 127; kk = idx >> 7; }
  };
  float ra[4], rb[4];
  auto fetch = [&](int64_t k0) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int mm, kk;
      a_pos(e, mm, kk);
      const int64_t m = m0 + mm, k = k0 + kk;
      ra[e] = m < g.M ? g.A[m * g.a_rs + k * g.a_cs] : 0.f;
      int nn, kb;
      b_pos(e, nn, kb);
      const int64_t n = n0 + nn, kq = k0 + kb;
      rb[e] = n < g.N ? g.B[kq * g.b_rs + n * g.b_cs] : 0.f;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      int mm, kk;
      a_pos(e, mm, kk);
      as[buf][kk][mm] = ra[e];
      int nn, kb;
      b_pos(e, nn, kb);
      bs[buf][kb][nn] = rb[e];
    }
  };
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int64_t k0 = 0; k0 < g.Kd; k0 += kGK) {
    const bool more = k0 + kGK < g.Kd;
    if (more) fetch(k0 + kGK);
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float av[8], bv[8];
      *reinterpret_cast<float4*>(av) = *reinterpret_cast<const float4*>(&as[buf][kk][ty * 4]);
      *reinterpret_cast<float4*>(av + 4) =
          *reinterpret_cast<const float4*>(&as[buf][kk][64 + ty * 4]);
      *reinterpret_cast<float4*>(bv) = *reinterpret_cast<const float4*>(&bs[buf][kk][tx * 4]);
      *reinterpret_cast<float4*>(bv + 4) =
          *reinterpret_cast<const float4*>(&bs[buf][kk][64 + tx * 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) {
      stash(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
      const int64_t n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (m < g.M && n < g.N) {
        if (g.assign) g.C[m * g.ldc + n] = acc[i][j];
        else g.C[m * g.ldc + n] -= acc[i][j];
      }
    }
}

// Products of fp32 matrices on the bf16 tensor cores, to fp32 accuracy:
// every value is split into three bf16 terms, x = x1 + x2 + x3 + r with each
// term the bf16 rounding of what the earlier ones leave (|r| about 2^-24 |x|,
// every subtraction exact), and sum_k x_k y_k is formed from the six products
// x1 y1 + x1 y2 + x2 y1 + x1 y3 + x2 y2 + x3 y1 (the dropped ones are below
// 2^-24 of the product).  The six go into one GEMM with a six-fold depth: A's
// K blocks hold the terms (1, 1, 2, 1, 2, 3) of x, B's (1, 2, 1, 3, 2, 1) of
// y.  bf16 x bf16 products are exact in the fp32 accumulator.
__device__ __forceinline__ void split3_bf16(float x, __nv_bfloat16* t) {
  t[0] = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(t[0]);
  t[1] = __float2bfloat16_rn(r1);
  t[2] = __float2bfloat16_rn(r1 - __bfloat162float(t[1]));
}
__device__ __forceinline__ int split_term(int b_side, int q) {
  // A: 0 0 1 0 1 2, B: 0 1 0 2 1 0
  return b_side ? (0x010210 >> (4 * (5 - q))) & 15 : (0x001012 >> (4 * (5 - q))) & 15;
}

// dst (cols x 6 depth, row-major, leading dimension 6 depth) from the
// transpose of src (depth x cols, leading dimension lds): row n of dst holds
// the split terms of column n of src, K block q holding term split_term(q).
// 32 x 32 tiles through shared memory so that both sides coalesce.
__global__ void __launch_bounds__(256) k_split_t(const float* __restrict__ src, int64_t lds,
                                                 int depth, int64_t cols,
                                                 __nv_bfloat16* __restrict__ dst, int b_side) {
  __shared__ float tile[32][33];
  const int64_t c0 = (int64_t)blockIdx.x * 32;
  const int r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i;
    const int64_t c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < depth && c < cols) ? src[(int64_t)r * lds + c] : 0.f;
  }
  __syncthreads();
  const int64_t ldd = 6 * (int64_t)depth;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int64_t c = c0 + i;
    const int r = r0 + threadIdx.x;
    if (c < cols && r < depth) {
      __nv_bfloat16 t[3];
      split3_bf16(tile[threadIdx.x][i], t);
#pragma unroll
      for (int q = 0; q < 6; ++q) dst[c * ldd + q * depth + r] = t[split_term(b_side, q)];
    }
  }
}

// dst (rows x 6 depth) from src (rows x depth, leading dimension lds), no
// transpose.
__global__ void __launch_bounds__(256) k_split_rows(const float* __restrict__ src, int64_t lds,
                                                    int64_t rows, int depth,
                                                    __nv_bfloat16* __restrict__ dst,
                                                    int b_side) {
  const int64_t ldd = 6 * (int64_t)depth;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * depth;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / depth;
    const int k = (int)(i - r * depth);
    __nv_bfloat16 t[3];
    split3_bf16(src[r * lds + k], t);
#pragma unroll
    for (int q = 0; q < 6; ++q) dst[r * ldd + q * depth + k] = t[split_term(b_side, q)];
  }
}

// M[i][i] = 1 for all i
__global__ void k_unit_diag(float* __restrict__ M, int64_t K) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < K;
       i += (int64_t)gridDim.x * blockDim.x)
    M[i * K + i] = 1.f;
}

// Nearest level of w / s (first level on ties; s = 0 gives w / s := 0), in fp32.
template <int MODE>
__device__ __forceinline__ int gptq_round(float w, float s) {
  using Gr = GridT<MODE>;
  const float q = s > 0.f ? w / s : 0.f;
  int best = 0;
  float bd = fabsf(q - Gr::level(0));
#pragma unroll
  for (int k = 1; k < Gr::LEVELS; ++k) {
    const float d = fabsf(q - Gr::level(k));
    if (d < bd) {
      bd = d;
      best = k;
    }
  }
  return best;
}

// One block of 128 columns [j0, j0 + 128): one warp per row, lane l holding
// the row's columns l, l + 32, l + 64, l + 96; 16 rows per CTA share the
// block's 128 x 128 upper triangle of U in shared memory (rows of U read
// across lanes: conflict-free).  The row's group scale is set from its
// updated weights at the block start (warp max); then column by column the
// owner lane's weight is broadcast, rounded to the nearest level (first on
// ties), its error e = (w - s c) / U_jj written to E[j][n] and fed forward
// to the later columns of the block, every lane updating its own columns.
constexpr int kColRows = 16;
constexpr int kColsSmem = kCols * kCols * 4;

template <int MODE>
__global__ void __launch_bounds__(kColRows * 32) k_gptq_cols(
    const float* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ U, int64_t j0,
    int8_t* __restrict__ levels, float* __restrict__ scales, float* __restrict__ E) {
  using Gr = GridT<MODE>;
  extern __shared__ __align__(16) uint8_t gsm[];
  float (*us)[kCols] = reinterpret_cast<float (*)[kCols]>(gsm);
  // eight loads in flight per thread before their stores (the block of U
  // is usually not in L2); kCols * kCols is a multiple of 8 x the block
  constexpr int kBatch = 8;
  static_assert((kCols * kCols) % (kBatch * kColRows * 32) == 0, "U block load batches");
  for (int e0 = threadIdx.x; e0 < kCols * kCols; e0 += kBatch * blockDim.x) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u * blockDim.x;
      const int r = e / kCols, c = e % kCols;
      v[u] = c >= r ? U[(j0 + r) * K + j0 + c] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u * blockDim.x;
      us[e / kCols][e % kCols] = v[u];
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)blockIdx.x * kColRows + (threadIdx.x >> 5);
  if (n >= N) return;  // whole warps
  float w[4];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w[i] = W[n * K + j0 + lane + 32 * i];
    amax = fmaxf(amax, fabsf(w[i]));
  }
  amax = warp_max(amax);
  const float s = amax / Gr::CMAX;
  if (lane == 0) scales[n * (K / kCols) + j0 / kCols] = s;
  int lev_own[4] = {0, 0, 0, 0};
  for (int j = 0; j < kCols; ++j) {
    const int slot = j >> 5;
    const float mine = slot == 0 ? w[0] : slot == 1 ? w[1] : slot == 2 ? w[2] : w[3];
    const float wj = __shfl_sync(0xffffffffu, mine, j & 31);
    const int lev = gptq_round<MODE>(wj, s);
    const float e = (wj - s * Gr::level(lev)) / us[j][j];
    if (lane == (j & 31)) {
      lev_own[0] = slot == 0 ? lev : lev_own[0];
      lev_own[1] = slot == 1 ? lev : lev_own[1];
      lev_own[2] = slot == 2 ? lev : lev_own[2];
      lev_own[3] = slot == 3 ? lev : lev_own[3];
    }
    if (lane == 0) E[(int64_t)j * N + n] = e;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = lane + 32 * i;
      if (c > j) w[i] = fmaf(-e, us[j][c], w[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) levels[n * K + j0 + lane + 32 * i] = (int8_t)lev_own[i];
}

}  // namespace

namespace {

// C (rows x cols, leading dimension ldc) -= X Y^T with X rows x depth
// (leading dimension ldx) and Y^T given either as cols x depth (ldy, b_t
// false) or as depth x cols (b_t true), on the tensor cores with the
// three-term split: X and Y are split into Sa and Sb, and the GEMM's
// epilogue subtracts the product from C in place.  depth <= 128.
cudaError_t sub_split_gemm(const float* X, int64_t ldx, int64_t rows, const float* Y,
                           int64_t ldy, int64_t cols, int depth, bool b_t, float* C,
                           int64_t ldc, __nv_bfloat16* Sa, __nv_bfloat16* Sb,
                           const EpiParams& ep, int sm_count, cudaStream_t st) {
  const int kd = 6 * depth;
  k_split_rows<<<grid_cap(rows * depth, 256, sm_count * 8), 256, 0, st>>>(X, ldx, rows, depth,
                                                                          Sa, 0);
  if (b_t)
    k_split_t<<<dim3((unsigned)((cols + 31) / 32), (unsigned)((depth + 31) / 32)), dim3(32, 8),
                0, st>>>(Y, ldy, depth, cols, Sb, 1);
  else
    k_split_rows<<<grid_cap(cols * depth, 256, sm_count * 8), 256, 0, st>>>(Y, ldy, cols,
                                                                            depth, Sb, 1);
  CUtensorMap ta, tb;
  EpiMaps em;
  if (make_tmap_bf16(&ta, Sa, rows, kd, kd, kGemmBoxRowsA) ||
      make_tmap_bf16(&tb, Sb, cols, kd, kd, kGemmBoxRowsB) ||
      make_tmap_epi_f32(&em.out, C, rows, cols, ldc))
    return cudaErrorInvalidValue;
  em.yref = em.out;
  return launch_gemm(ta, tb, em, rows, cols, kd, EPI_SUB_F32, ep, sm_count, st);
}

// W[:, j1:] -= E^T U[j0:j1, j1:] for each block of 128 columns, on the tensor
// cores with the three-term split (fp32 accuracy): A = split of E^T (N x
// 768), B = split of U[j0:j1, j1:]^T (rest x 768), and the GEMM's epilogue
// subtracts the product from W's columns j1.. in place.
template <int MODE>
cudaError_t gptq_columns(float* W32, int64_t N, int64_t K, const float* U, int8_t* levels,
                         float* scales, float* E, __nv_bfloat16* Es, __nv_bfloat16* Us,
                         const EpiParams& ep, int sm_count, cudaStream_t st) {
  {
    const cudaError_t e = smem_optin<k_gptq_cols<MODE>>(kColsSmem);
    if (e != cudaSuccess) return e;
  }
  const unsigned rb = (unsigned)((N + kColRows - 1) / kColRows);
  for (int64_t j0 = 0; j0 < K; j0 += kCols) {
    k_gptq_cols<MODE><<<rb, kColRows * 32, kColsSmem, st>>>(W32, N, K, U, j0, levels, scales, E);
    const int64_t j1 = j0 + kCols, rest = K - j1;
    if (rest > 0) {
      k_split_t<<<dim3((unsigned)((N + 31) / 32), kCols / 32), dim3(32, 8), 0, st>>>(
          E, N, kCols, N, Es, 0);
      k_split_t<<<dim3((unsigned)((rest + 31) / 32), kCols / 32), dim3(32, 8), 0, st>>>(
          U + j0 * K + j1, K, kCols, rest, Us, 1);
      CUtensorMap ta, tb;
      EpiMaps em;
      if (make_tmap_bf16(&ta, Es, N, 6 * kCols, 6 * kCols, kGemmBoxRowsA) ||
          make_tmap_bf16(&tb, Us, rest, 6 * kCols, 6 * kCols, kGemmBoxRowsB) ||
          make_tmap_epi_f32(&em.out, W32 + j1, N, rest, K))
        return cudaErrorInvalidValue;
      em.yref = em.out;
      const cudaError_t e =
          launch_gemm(ta, tb, em, N, rest, 6 * kCols, EPI_SUB_F32, ep, sm_count, st);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace

// GPTQ on device inputs; levels (N x K int8) and scales (N x K/128 fp32) are
// device buffers.  Allocates its workspace stream-ordered on `st` from the
// library's pool (no device synchronisation, and the pool keeps the memory
// for the next call), synchronises the stream, frees.
int gptq_run(int mode, const void* Wd, int w_dtype, const void* Xd, int x_dtype, int64_t N,
             int64_t K, int64_t T, float damp, int8_t* levels, float* scales, int sm_count,
             cudaStream_t st) {
  const int64_t Tp = (T + 63) / 64 * 64, NK = N * K, KK = K * K;
  std::vector<void*> bufs;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaMemPool_t pool = library_pool(dev);
  bool oom = pool == nullptr;
  auto alloc = [&](size_t bytes) -> void* {
    void* p = nullptr;
    if (oom || cudaMallocFromPoolAsync(&p, bytes, pool, st) != cudaSuccess) {
      cudaGetLastError();
      oom = true;
      return nullptr;
    }
    bufs.push_back(p);
    return p;
  };
  float* W32 = (float*)alloc((size_t)NK * 4);
  __nv_bfloat16* Wop = (__nv_bfloat16*)alloc((size_t)NK * 2);
  __nv_bfloat16* Xb = (__nv_bfloat16*)alloc((size_t)Tp * K * 2);
  __nv_bfloat16* Xt = (__nv_bfloat16*)alloc((size_t)K * Tp * 2);
  float* B1 = (float*)alloc((size_t)KK * 4);
  float* B2 = (float*)alloc((size_t)KK * 4);
  int* dead = (int*)alloc((size_t)K * 4);
  float* E = (float*)alloc((size_t)kCols * N * 4);
  // split operands of the tensor-core updates (up to 6 x 128 bf16 per row)
  __nv_bfloat16* Sa = (__nv_bfloat16*)alloc((size_t)(N > K ? N : K) * 6 * kCols * 2);
  __nv_bfloat16* Sb = (__nv_bfloat16*)alloc((size_t)K * 6 * kCols * 2);
  float* Xinv = (float*)alloc((size_t)K * kNb * 4);  // L_kk^-T of every diagonal block
  int* err = (int*)alloc(64);
  double* partials = (double*)alloc(4096 * 8);
  unsigned* ticket = (unsigned*)alloc(16);
  auto finish = [&](int status) {
    cudaGetLastError();
    for (void* p : bufs) cudaFreeAsync(p, st);
    cudaStreamSynchronize(st);
    cudaGetLastError();
    return status;
  };
  if (oom) return finish(GSQ_ERR_OOM);

  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t x) {
    if (e == cudaSuccess) e = x;
    return e == cudaSuccess;
  };
  ok(cudaMemsetAsync(err, 0, 64, st));
  ok(cudaMemsetAsync(ticket, 0, 16, st));
  ok(cudaMemsetAsync(Xt, 0, (size_t)K * Tp * 2, st));
  ok(cudaMemsetAsync(Xb, 0, (size_t)Tp * K * 2, st));
  ok(launch_convert_x(Xd, x_dtype, T, K, Tp, Xb, Xt, nullptr, err, st));
  ok(launch_convert_w(Wd, w_dtype, N, K, W32, Wop, 0, err, st));

  // H = Xt Xt^T (fp32) into B1
  CUtensorMap ta, tb;
  EpiMaps em;
  if (make_tmap_bf16(&ta, Xt, K, Tp, Tp, kGemmBoxRowsA) ||
      make_tmap_bf16(&tb, Xt, K, Tp, Tp, kGemmBoxRowsB) ||
      make_tmap_epi_f32(&em.out, B1, K, K, K))
    return finish(GSQ_ERR_CUDA);
  em.yref = em.out;
  EpiParams ep;
  ep.partials = partials;
  ep.ticket = ticket;
  ep.loss_out = nullptr;
  ep.err = err;
  ok(launch_gemm(ta, tb, em, K, K, Tp, EPI_STORE_F32, ep, sm_count, st));
  k_gptq_damp<<<1, 1024, 0, st>>>(B1, K, damp, dead);
  k_zero_dead_cols<<<grid_cap(NK, 256, sm_count * 8), 256, 0, st>>>(W32, N, K, dead);
  ok(cudaGetLastError());

  // A = J H J into B2, lower Cholesky in place
  const int rgrid = grid_cap(KK, 256, sm_count * 8);
  k_reverse<<<rgrid, 256, 0, st>>>(B1, B2, K);
  float* A = B2;
  for (int64_t k0 = 0; k0 < K && e == cudaSuccess; k0 += kNb) {
    float* Xk = Xinv + (k0 / kNb) * kNb * kNb;  // L_kk^-T
    k_potrf64<<<1, kPotrfThreads, 0, st>>>(A, K, k0, err, Xk);
    const int64_t rest = K - k0 - kNb;
    if (rest > 0) {
      float* P = A + (k0 + kNb) * K + k0;
      // the panel below: P = P L_kk^-T, in place (each CTA's rows are its own)
      SubGemm gs{rest, kNb, kNb, P, K, 1, Xk, kNb, 1, P, K, 0};
      gs.assign = 1;
      k_gemm_sub<<<dim3(1, (unsigned)((rest + kGT - 1) / kGT)), 256, 0, st>>>(gs);
      // the trailing matrix: A[c1:, c1:] -= P P^T on the tensor cores (the
      // whole square; only its lower triangle is ever read)
      ok(sub_split_gemm(P, K, rest, P, K, rest, kNb, false, A + (k0 + kNb) * K + k0 + kNb, K,
                        Sa, Sb, ep, sm_count, st));
    }
    ok(cudaGetLastError());
  }
  // M = L^-1 into B1, right-looking block forward substitution: M starts
  // as I; row block k0 is solved against its diagonal block once every
  // earlier block has been subtracted from it, then subtracted from all
  // later row blocks at once (one wide GEMM per block instead of a 64-row
  // strip with the whole K depth)
  float* M = B1;
  ok(cudaMemsetAsync(M, 0, (size_t)KK * 4, st));
  k_unit_diag<<<grid_cap(K, 256, 1024), 256, 0, st>>>(M, K);
  for (int64_t k0 = 0; k0 < K && e == cudaSuccess; k0 += kNb) {
    const int64_t c1 = k0 + kNb, rest = K - c1;
    // the row block: M[k0:c1, :c1] = L_kk^-1 M[k0:c1, :c1], in place (each
    // CTA's columns are its own); L_kk^-1 (m, k) = Xinv_k (k, m)
    {
      SubGemm gs{kNb, c1, kNb, Xinv + (k0 / kNb) * kNb * kNb, 1, kNb, M + k0 * K, K, 1,
                 M + k0 * K, K, 0};
      gs.assign = 1;
      k_gemm_sub<<<dim3((unsigned)((c1 + kGT - 1) / kGT), 1), 256, 0, st>>>(gs);
    }
    if (rest > 0) {
      // M[c1:, :c1] -= L[c1:, k0:c1] M[k0:c1, :c1] on the tensor cores
      ok(sub_split_gemm(A + c1 * K + k0, K, rest, M + k0 * K, K, c1, kNb, true, M + c1 * K, K,
                        Sa, Sb, ep, sm_count, st));
    }
    ok(cudaGetLastError());
  }
  // U = J M J into B2
  k_reverse<<<rgrid, 256, 0, st>>>(M, B2, K);
  ok(cudaGetLastError());
  const float* U = B2;
  if (e == cudaSuccess) {
    switch (mode) {
      case GRID_2BIT:
        ok(gptq_columns<GRID_2BIT>(W32, N, K, U, levels, scales, E, Sa, Sb, ep, sm_count, st));
        break;
      case GRID_TERNARY:
        ok(gptq_columns<GRID_TERNARY>(W32, N, K, U, levels, scales, E, Sa, Sb, ep, sm_count,
                                      st));
        break;
      default:
        ok(gptq_columns<GRID_3BIT_LOCAL>(W32, N, K, U, levels, scales, E, Sa, Sb, ep, sm_count,
                                         st));
    }
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  int h = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess)
    return finish(e == cudaErrorMemoryAllocation ? GSQ_ERR_OOM : GSQ_ERR_CUDA);
  if (h == DEV_ERR_NONFINITE) return finish(GSQ_ERR_NONFINITE);
  if (h == DEV_ERR_TIMEOUT) return finish(GSQ_ERR_TIMEOUT);
  if (h != DEV_OK) return finish(GSQ_ERR_CUDA);
  return finish(GSQ_OK);
}

}  // namespace gsq

extern "C" {

int gsq_gptq(const void* W, int w_dtype, const void* X, int x_dtype, int64_t N, int64_t K,
             int64_t T, int group, int grid_mode, float damp, int8_t* levels, float* scales,
             void* stream) {
  using namespace gsq;
  if (!W || !X || !levels || !scales || N <= 0 || K <= 0 || T <= 0 || group <= 0 ||
      (w_dtype != GSQ_F32 && w_dtype != GSQ_BF16) ||
      (x_dtype != GSQ_F32 && x_dtype != GSQ_BF16) || stage_num_logits(grid_mode) < 0 ||
      K % group != 0 || !(damp >= 0.f) || !std::isfinite(damp) || N > ((int64_t)1 << 31) ||
      T > ((int64_t)1 << 31) || K > 65536)
    return GSQ_ERR_INVALID_ARG;
  if (group != kStageGroup) return GSQ_ERR_UNSUPPORTED;
  int dev = 0, major = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (major != 10) return GSQ_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t wbytes = (size_t)N * K * (w_dtype == GSQ_F32 ? 4 : 2);
  const size_t xbytes = (size_t)T * K * (x_dtype == GSQ_F32 ? 4 : 2);
  const size_t lbytes = (size_t)N * K, sbytes = (size_t)N * (K / group) * 4;
  std::vector<void*> tmp;
  auto dev_copy = [&](const void* p, size_t bytes, void** out) -> int {
    if (stage_is_device_ptr(p)) {
      *out = const_cast<void*>(p);
      return GSQ_OK;
    }
    if (pool_malloc(out, bytes) != cudaSuccess) {
      cudaGetLastError();
      return GSQ_ERR_OOM;
    }
    tmp.push_back(*out);
    return GSQ_OK;
  };
  void *Wd = nullptr, *Xd = nullptr, *Ld = nullptr, *Sd = nullptr;
  int rc = dev_copy(W, wbytes, &Wd);
  if (!rc) rc = dev_copy(X, xbytes, &Xd);
  if (!rc) rc = dev_copy(levels, lbytes, &Ld);
  if (!rc) rc = dev_copy(scales, sbytes, &Sd);
  cudaError_t e = cudaSuccess;
  if (!rc && Wd != W) e = cudaMemcpyAsync(Wd, W, wbytes, cudaMemcpyDefault, st);
  if (!rc && e == cudaSuccess && Xd != X) e = cudaMemcpyAsync(Xd, X, xbytes, cudaMemcpyDefault, st);
  if (!rc && e != cudaSuccess) rc = GSQ_ERR_CUDA;
  if (!rc)
    rc = gptq_run(grid_mode, Wd, w_dtype, Xd, x_dtype, N, K, T, damp, (int8_t*)Ld, (float*)Sd,
                  sms, st);
  if (!rc && Ld != levels &&
      cudaMemcpy(levels, Ld, lbytes, cudaMemcpyDeviceToHost) != cudaSuccess)
    rc = GSQ_ERR_CUDA;
  if (!rc && Sd != scales &&
      cudaMemcpy(scales, Sd, sbytes, cudaMemcpyDeviceToHost) != cudaSuccess)
    rc = GSQ_ERR_CUDA;
  cudaStreamSynchronize(st);
  cudaGetLastError();
  for (void* p : tmp) pool_free(p);
  return rc;
}

}  // extern "C"
