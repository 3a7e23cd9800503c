// gsq_block.cu -- the staged block pipeline: GSQ quantizes the blocks of a
// model in order, each block from the output of the already quantized prefix,
// and inside a block the query and key projections first (each against its
// own output), then the value and output projections together, then the MLP
// on the block output (agihunt.info summary, optimisation paragraph).
//
// The block is a pre-norm Llama block on an fp32 residual stream x (T x H):
//   xa = bf16(RMSNorm(x)), attn = Attn(xa), h = x + attn,
//   xm = bf16(RMSNorm(h)),  y = h + (bf16(silu(xm Wg^T) * xm Wu^T)) Wd^T,
// RMSNorm with unit gain, rotary embedding (rotate-half), causal attention
// with grouped key/value heads; every GEMM runs on the CTA-pair tcgen05
// kernel with bf16 operands and fp32 accumulation.
//
// gsq_block_quantize, for one block:
//   1. the full-precision forward: the V/O target attn_fp and y_fp;
//   2. Q and K: single-layer contexts on xa (target: the full-precision
//      weight's own output);
//   3. V and O: the joint attention stage, probabilities from the frozen
//      quantized Q, K, target attn_fp;
//   4. h_q = x + Attn_q(xa), xm_q = bf16(RMSNorm(h_q)), the MLP stage on
//      xm_q with target y_fp - h_q (so its loss is the block-output error);
//   5. x_out = h_q + MLP_q(xm_q): the input of the next block.
// Each stage hardens its weights (harden/pack, then gsq_dequant), so the
// later stages and the next block see exactly the packed result.
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "gsq_device.cuh"
#include "gsq_stage.h"

using namespace gsq;

namespace {

constexpr int kBlkThreads = 256;

// ------------------------------------------------------------------ kernels

__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) red[wid] = v;
  __syncthreads();
  if (wid == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    v = warp_sum(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  const float s = red[0];
  __syncthreads();
  return s;
}

// One block per row: v = x (+ a); h_out = v; xn = bf16(v / sqrt(mean(v^2) +
// eps)); r_out = yfp - v.  a, h_out, yfp / r_out nullable.  H % 4 == 0.
__global__ void __launch_bounds__(kBlkThreads) k_residual_rmsnorm(
    const float* __restrict__ x, const float* __restrict__ a, int64_t H, float eps,
    float* __restrict__ h_out, __nv_bfloat16* __restrict__ xn,
    const float* __restrict__ yfp, float* __restrict__ r_out) {
  __shared__ float red[32];
  const int64_t off = (int64_t)blockIdx.x * H;
  float ss = 0.f;
  for (int64_t i = threadIdx.x * 4; i < H; i += (int64_t)blockDim.x * 4) {
    float4 v = *reinterpret_cast<const float4*>(x + off + i);
    if (a) {
      const float4 b = *reinterpret_cast<const float4*>(a + off + i);
      v.x += b.x; v.y += b.y; v.z += b.z; v.w += b.w;
    }
    if (h_out) *reinterpret_cast<float4*>(h_out + off + i) = v;
    if (r_out) {
      const float4 y = *reinterpret_cast<const float4*>(yfp + off + i);
      *reinterpret_cast<float4*>(r_out + off + i) =
          make_float4(y.x - v.x, y.y - v.y, y.z - v.z, y.w - v.w);
    }
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum(ss, red);
  const float r = 1.f / sqrtf(ss / (float)H + eps);
  for (int64_t i = threadIdx.x * 4; i < H; i += (int64_t)blockDim.x * 4) {
    float4 v = *reinterpret_cast<const float4*>(x + off + i);
    if (a) {
      const float4 b = *reinterpret_cast<const float4*>(a + off + i);
      v.x += b.x; v.y += b.y; v.z += b.z; v.w += b.w;
    }
    __nv_bfloat162 p0 = __floats2bfloat162_rn(v.x * r, v.y * r);
    __nv_bfloat162 p1 = __floats2bfloat162_rn(v.z * r, v.w * r);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&p0);
    pk.y = *reinterpret_cast<uint32_t*>(&p1);
    *reinterpret_cast<uint2*>(xn + off + i) = pk;
  }
}

// y = h + m (n % 4 == 0)
__global__ void __launch_bounds__(256) k_add(const float* __restrict__ h,
                                             const float* __restrict__ m, int64_t n,
                                             float* __restrict__ y) {
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n;
       i += (int64_t)gridDim.x * blockDim.x * 4) {
    const float4 a = *reinterpret_cast<const float4*>(h + i);
    const float4 b = *reinterpret_cast<const float4*>(m + i);
    *reinterpret_cast<float4*>(y + i) = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  }
}

// w = bf16(s_g level(code)) from the LSB-first code stream of a row: b = 2
// bits (16 codes per 32-bit word) or 3 bits (32 codes per 3 words).  One
// thread per 32 codes.
template <int MODE>
__global__ void __launch_bounds__(256) k_dequant(const uint32_t* __restrict__ packed,
                                                 const float* __restrict__ s, int64_t N,
                                                 int64_t K, __nv_bfloat16* __restrict__ W) {
  constexpr int B = MODE == GRID_3BIT_LOCAL ? 3 : 2;
  const int64_t per_row = K / 32, G = K / 128, wpr = K * B / 32;
  for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < N * per_row;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = q / per_row, j0 = (q - n * per_row) * 32;
    const uint32_t* src = packed + n * wpr + j0 * B / 32;
    uint64_t lo, hi = 0;
    if (B == 2) {
      lo = (uint64_t)src[0] | ((uint64_t)src[1] << 32);
    } else {
      lo = (uint64_t)src[0] | ((uint64_t)src[1] << 32);
      hi = src[2];
    }
    const float sg = s[n * G + j0 / 128];
    float w[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int bit = j * B;
      uint32_t code;
      if (bit + B <= 64)
        code = (uint32_t)(lo >> bit) & ((1u << B) - 1u);
      else if (bit >= 64)
        code = (uint32_t)(hi >> (bit - 64)) & ((1u << B) - 1u);
      else
        code = (uint32_t)((lo >> bit) | (hi << (64 - bit))) & ((1u << B) - 1u);
      w[j] = sg * GridT<MODE>::level((int)code);
    }
    __nv_bfloat16* dst = W + n * K + j0;
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      __nv_bfloat162 p[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) p[u] = __floats2bfloat162_rn(w[j + 2 * u], w[j + 2 * u + 1]);
      *reinterpret_cast<uint4*>(dst + j) = *reinterpret_cast<uint4*>(p);
    }
  }
}

int grid_cap(int64_t work, int threads, int cap) {
  const int64_t b = (work + threads - 1) / threads;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

cudaError_t launch_dequant(int mode, const uint32_t* packed, const float* s, int64_t N,
                           int64_t K, __nv_bfloat16* W, int sms, cudaStream_t st) {
  const int blocks = grid_cap(N * (K / 32), 256, sms * 16);
  switch (mode) {
    case GRID_2BIT: k_dequant<GRID_2BIT><<<blocks, 256, 0, st>>>(packed, s, N, K, W); break;
    case GRID_TERNARY: k_dequant<GRID_TERNARY><<<blocks, 256, 0, st>>>(packed, s, N, K, W); break;
    default: k_dequant<GRID_3BIT_LOCAL><<<blocks, 256, 0, st>>>(packed, s, N, K, W);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ host helpers

struct Dims {
  int64_t nseq = 0, S = 0, nh = 0, nkv = 0, d = 0, F = 0, T = 0, H = 0, Hk = 0, grp = 0;
  double theta = 0.0;
  float eps = 0.f;
  int64_t rows(int i) const {  // q k v o gate up down
    const int64_t r[7] = {H, Hk, Hk, H, F, F, H};
    return r[i];
  }
  int64_t cols(int i) const { return i == 6 ? F : H; }
};

int check_dims(Dims* D, int64_t n_seq, int64_t seq_len, int64_t n_heads, int64_t n_kv_heads,
               int64_t head_dim, int64_t ffn, double theta, float eps) {
  if (n_seq <= 0 || seq_len <= 0 || n_heads <= 0 || n_kv_heads <= 0 || ffn <= 0 ||
      n_heads % n_kv_heads != 0 || !(theta > 0.0) || !(eps >= 0.f) || !std::isfinite(eps) ||
      n_seq * seq_len > ((int64_t)1 << 31))
    return GSQ_ERR_INVALID_ARG;
  if (head_dim != 128 || seq_len % 128 != 0 || seq_len > 65536 || ffn % 128 != 0)
    return GSQ_ERR_UNSUPPORTED;
  D->nseq = n_seq;
  D->S = seq_len;
  D->nh = n_heads;
  D->nkv = n_kv_heads;
  D->d = head_dim;
  D->F = ffn;
  D->T = n_seq * seq_len;
  D->H = n_heads * head_dim;
  D->Hk = n_kv_heads * head_dim;
  D->grp = n_heads / n_kv_heads;
  D->theta = theta;
  D->eps = eps;
  return GSQ_OK;
}

int sm100_sms(int* sms) {
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return GSQ_ERR_CUDA;
  }
  if (prop.major != 10) return GSQ_ERR_UNSUPPORTED;
  *sms = prop.multiProcessorCount;
  return GSQ_OK;
}

// Device allocations of one call, freed on every exit path.
struct Arena {
  std::vector<void*> ptrs;
  int status = GSQ_OK;
  cudaStream_t st = nullptr;
  ~Arena() {
    if (st) cudaStreamSynchronize(st);
    cudaGetLastError();
    for (void* p : ptrs) pool_free(p);
  }
  template <typename T>
  T* get(size_t count) {
    if (status != GSQ_OK) return nullptr;
    void* p = nullptr;
    if (pool_malloc(&p, count * sizeof(T) + 16) != cudaSuccess) {
      cudaGetLastError();
      status = GSQ_ERR_OOM;
      return nullptr;
    }
    ptrs.push_back(p);
    return static_cast<T*>(p);
  }
  void release(void* p) {
    if (!p) return;
    for (auto& q : ptrs)
      if (q == p) {
        cudaStreamSynchronize(st);
        pool_free(q);
        q = nullptr;
      }
  }
  // e != cudaSuccess -> sticky status
  bool ok(cudaError_t e) {
    if (status == GSQ_OK && e != cudaSuccess) status = stage_cuda_status(e);
    return status == GSQ_OK;
  }
  bool ok_status(int s) {
    if (status == GSQ_OK && s != GSQ_OK) status = s;
    return status == GSQ_OK;
  }
};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// a device copy of a caller buffer when it is host memory or not 16-byte
// aligned (the kernels use 16-byte vector accesses and TMA)
const void* device_view(Arena& A, const void* p, size_t bytes) {
  if (A.status != GSQ_OK) return nullptr;
  if (stage_is_device_ptr(p) && aligned16(p)) return p;
  void* d = A.get<char>(bytes);
  if (d) A.ok(cudaMemcpyAsync(d, p, bytes, cudaMemcpyDefault, A.st));
  return d;
}

struct Gemm {
  Arena* A;
  int sms;
  double* partials;
  unsigned* ticket;
  int* err;
  EpiParams ep() const {
    EpiParams e;
    std::memset(&e, 0, sizeof(e));
    e.partials = partials;
    e.ticket = ticket;
    e.loss_out = nullptr;
    e.err = err;
    return e;
  }
  // C (M x N) = Am (M x Kc, ld lda) . Bm (N x Kc, ld ldb)^T, fp32 or bf16 out
  bool run(const __nv_bfloat16* Am, int64_t M, int64_t lda, const __nv_bfloat16* Bm,
           int64_t N, int64_t ldb, int64_t Kc, void* C, int64_t ldc, bool bf16_out) {
    if (A->status != GSQ_OK) return false;
    CUtensorMap ta, tb;
    EpiMaps em;
    bool bad = make_tmap_bf16(&ta, Am, M, Kc, lda, kGemmBoxRowsA) != 0;
    bad |= make_tmap_bf16(&tb, Bm, N, Kc, ldb, kGemmBoxRowsB) != 0;
    bad |= (bf16_out ? make_tmap_epi_bf16(&em.out, C, M, N, ldc)
                     : make_tmap_epi_f32(&em.out, C, M, N, ldc)) != 0;
    em.yref = em.out;
    if (bad) return A->ok_status(GSQ_ERR_CUDA);
    return A->ok(launch_gemm(ta, tb, em, M, N, Kc, bf16_out ? EPI_STORE_BF16 : EPI_STORE_F32,
                             ep(), sms, A->st));
  }
};

// out32 (T x H) = o Wo^T with o_(s,h) = P_(s,h) V_(s, h / grp), P from Wq, Wk
bool attn_sublayer(const Dims& D, Gemm& G, const __nv_bfloat16* xa, const __nv_bfloat16* const* W,
                   float* out32) {
  Arena& A = *G.A;
  const int64_t T = D.T, H = D.H, Hk = D.Hk, S = D.S, d = D.d;
  float* Q32 = A.get<float>(T * H);
  float* K32 = A.get<float>(T * Hk);
  __nv_bfloat16* Qr = A.get<__nv_bfloat16>(T * H);
  __nv_bfloat16* Kr = A.get<__nv_bfloat16>(T * Hk);
  float* scores = A.get<float>(S * S);
  __nv_bfloat16* P = A.get<__nv_bfloat16>(D.nseq * D.nh * S * S);
  __nv_bfloat16* VT = A.get<__nv_bfloat16>(Hk * T);
  __nv_bfloat16* o = A.get<__nv_bfloat16>(T * H);
  if (A.status != GSQ_OK) return false;
  G.run(xa, T, H, W[0], H, H, H, Q32, H, false);
  G.run(xa, T, H, W[1], Hk, H, H, K32, Hk, false);
  A.ok(launch_rope(Q32, T, H, S, (int)d, D.theta, Qr, G.sms, A.st));
  A.ok(launch_rope(K32, T, Hk, S, (int)d, D.theta, Kr, G.sms, A.st));
  const float scale = (float)(1.0 / std::sqrt((double)d));
  for (int64_t s = 0; s < D.nseq && A.status == GSQ_OK; ++s)
    for (int64_t h = 0; h < D.nh && A.status == GSQ_OK; ++h) {
      const int64_t g = h / D.grp;
      G.run(Qr + s * S * H + h * d, S, H, Kr + s * S * Hk + g * d, S, Hk, d, scores, S, false);
      A.ok(launch_causal_softmax(scores, S, scale, P + (s * D.nh + h) * S * S, A.st));
    }
  // V^T = Wv xa^T (Hk x T)
  G.run(W[2], Hk, H, xa, T, H, H, VT, T, true);
  // o: all (s, g) problems in one batched launch (grp S x d each)
  {
    CUtensorMap tmA_P, tmB_VT, tm_o;
    bool bad = make_tmap_bf16(&tmA_P, P, D.nseq * D.nh * S, S, S, kGemmBoxRowsA) != 0;
    bad |= make_tmap_bf16(&tmB_VT, VT, Hk, T, T, kGemmBoxRowsBNarrow) != 0;
    bad |= make_tmap_epi_bf16(&tm_o, o, T, H, H) != 0;
    if (bad) return A.ok_status(GSQ_ERR_CUDA);
    GemmSched a;
    a.count = (int)(D.nseq * D.nkv);
    a.inner = (int)D.nkv;
    a.a_row[0] = D.nh * S;
    a.a_row[1] = D.grp * S;
    a.b_row[1] = d;
    a.b_k[0] = S;
    a.o_row[0] = S;
    a.o_col[1] = D.grp * d;
    a.o_fold = S;
    a.o_fold_col = d;
    a.causal = S % 256 == 0 ? 1 : 0;
    a.seg = S;
    A.ok(launch_gemm_batched(tmA_P, tmB_VT, tm_o, D.grp * S, d, S, 128, a, EPI_STORE_BF16,
                             G.ep(), G.sms, A.st));
  }
  G.run(o, T, H, W[3], H, H, H, out32, H, false);
  for (void* p : {(void*)Q32, (void*)K32, (void*)Qr, (void*)Kr, (void*)scores, (void*)P,
                  (void*)VT, (void*)o})
    A.release(p);
  return A.status == GSQ_OK;
}

// out32 (T x H) = bf16(silu(xm Wg^T) * xm Wu^T) Wd^T
bool mlp_sublayer(const Dims& D, Gemm& G, const __nv_bfloat16* xm, const __nv_bfloat16* const* W,
                  float* out32) {
  Arena& A = *G.A;
  const int64_t T = D.T, H = D.H, F = D.F;
  float* a32 = A.get<float>(T * F);
  float* b32 = A.get<float>(T * F);
  __nv_bfloat16* hh = A.get<__nv_bfloat16>(T * F);
  if (A.status != GSQ_OK) return false;
  G.run(xm, T, H, W[4], F, H, H, a32, F, false);
  G.run(xm, T, H, W[5], F, H, H, b32, F, false);
  A.ok(launch_swiglu_fwd(a32, b32, T * F, hh, G.sms, A.st));
  G.run(hh, T, F, W[6], H, F, F, out32, H, false);
  for (void* p : {(void*)a32, (void*)b32, (void*)hh}) A.release(p);
  return A.status == GSQ_OK;
}

bool residual_rmsnorm(const Dims& D, Arena& A, const float* x, const float* a, float* h_out,
                      __nv_bfloat16* xn, const float* yfp = nullptr, float* r_out = nullptr) {
  if (A.status != GSQ_OK) return false;
  k_residual_rmsnorm<<<(unsigned)D.T, kBlkThreads, 0, A.st>>>(x, a, D.H, D.eps, h_out, xn, yfp,
                                                             r_out);
  return A.ok(cudaGetLastError());
}

bool add(const Dims& D, Arena& A, int sms, const float* h, const float* m, float* y) {
  if (A.status != GSQ_OK) return false;
  const int64_t n = D.T * D.H;
  k_add<<<grid_cap(n / 4, 256, sms * 8), 256, 0, A.st>>>(h, m, n, y);
  return A.ok(cudaGetLastError());
}

// y (and h) of the block with bf16 device weights W[7] on device x
bool block_forward(const Dims& D, Gemm& G, const float* x, const __nv_bfloat16* const* W,
                   float* h, float* y) {
  Arena& A = *G.A;
  const int64_t TH = D.T * D.H;
  __nv_bfloat16* xa = A.get<__nv_bfloat16>(TH);
  float* t32 = A.get<float>(TH);
  if (!residual_rmsnorm(D, A, x, nullptr, nullptr, xa)) return false;
  if (!attn_sublayer(D, G, xa, W, t32)) return false;
  residual_rmsnorm(D, A, x, t32, h, xa);  // h = x + attn, xa <- xm
  if (!mlp_sublayer(D, G, xa, W, t32)) return false;
  add(D, A, G.sms, h, t32, y);
  A.release(xa);
  A.release(t32);
  return A.status == GSQ_OK;
}

bool gemm_setup(Arena& A, Gemm& G, int sms) {
  G.A = &A;
  G.sms = sms;
  G.partials = A.get<double>(kStagePartials);
  G.ticket = A.get<unsigned>(4);
  G.err = A.get<int>(4);
  if (A.status != GSQ_OK) return false;
  A.ok(cudaMemsetAsync(G.ticket, 0, 16, A.st));
  A.ok(cudaMemsetAsync(G.err, 0, 16, A.st));
  return A.status == GSQ_OK;
}

// device error word of the GEMMs -> status (syncs)
int gemm_error(Arena& A, Gemm& G) {
  if (A.status != GSQ_OK) return A.status;
  if (!A.ok(cudaStreamSynchronize(A.st))) return A.status;
  int h = 0;
  if (!A.ok(cudaMemcpy(&h, G.err, sizeof(int), cudaMemcpyDeviceToHost))) return A.status;
  if (h == DEV_ERR_TIMEOUT) A.ok_status(GSQ_ERR_TIMEOUT);
  else if (h != DEV_OK) A.ok_status(GSQ_ERR_CUDA);
  return A.status;
}

}  // namespace

extern "C" {

int gsq_dequant(int grid_mode, const void* packed, const float* scales_f32, int64_t N,
                int64_t K, int group, void* W_bf16, void* stream) {
  if (!packed || !scales_f32 || !W_bf16 || N <= 0 || K <= 0 || group <= 0 || K % group != 0 ||
      stage_num_logits(grid_mode) < 0)
    return GSQ_ERR_INVALID_ARG;
  if (group != kStageGroup) return GSQ_ERR_UNSUPPORTED;
  int sms = 0;
  int rc = sm100_sms(&sms);
  if (rc != GSQ_OK) return rc;
  size_t pbytes = 0;
  gsq_packed_bytes(grid_mode, N, K, &pbytes);
  Arena A;
  A.st = static_cast<cudaStream_t>(stream);
  const void* pd = device_view(A, packed, pbytes);
  const void* sd = device_view(A, scales_f32, (size_t)N * (K / group) * 4);
  void* wd = W_bf16;
  const bool out_dev = stage_is_device_ptr(W_bf16) && aligned16(W_bf16);
  if (!out_dev) wd = A.get<__nv_bfloat16>(N * K);
  if (A.status != GSQ_OK) return A.status;
  A.ok(launch_dequant(grid_mode, static_cast<const uint32_t*>(pd), static_cast<const float*>(sd),
                      N, K, static_cast<__nv_bfloat16*>(wd), sms, A.st));
  if (!out_dev) A.ok(cudaMemcpyAsync(W_bf16, wd, (size_t)N * K * 2, cudaMemcpyDefault, A.st));
  A.ok(cudaStreamSynchronize(A.st));
  return A.status;
}

int gsq_block_forward(const float* x, const void* const* W, int64_t n_seq, int64_t seq_len,
                      int64_t n_heads, int64_t n_kv_heads, int64_t head_dim, int64_t ffn,
                      double rope_theta, float rms_eps, float* h_out, float* y_out,
                      void* stream) {
  if (!x || !W || !y_out) return GSQ_ERR_INVALID_ARG;
  for (int i = 0; i < 7; ++i)
    if (!W[i]) return GSQ_ERR_INVALID_ARG;
  Dims D;
  int rc = check_dims(&D, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn, rope_theta, rms_eps);
  if (rc != GSQ_OK) return rc;
  int sms = 0;
  if ((rc = sm100_sms(&sms)) != GSQ_OK) return rc;
  Arena A;
  A.st = static_cast<cudaStream_t>(stream);
  Gemm G;
  if (!gemm_setup(A, G, sms)) return A.status;
  const int64_t TH = D.T * D.H;
  const float* xd = static_cast<const float*>(device_view(A, x, (size_t)TH * 4));
  const __nv_bfloat16* Wd[7];
  for (int i = 0; i < 7; ++i)
    Wd[i] = static_cast<const __nv_bfloat16*>(
        device_view(A, W[i], (size_t)D.rows(i) * D.cols(i) * 2));
  float* h = A.get<float>(TH);
  float* y = A.get<float>(TH);
  if (A.status != GSQ_OK) return A.status;
  block_forward(D, G, xd, Wd, h, y);
  if (h_out) A.ok(cudaMemcpyAsync(h_out, h, (size_t)TH * 4, cudaMemcpyDefault, A.st));
  A.ok(cudaMemcpyAsync(y_out, y, (size_t)TH * 4, cudaMemcpyDefault, A.st));
  return gemm_error(A, G);
}

int gsq_block_quantize(const float* x_in, const void* const* W, int64_t n_seq, int64_t seq_len,
                       int64_t n_heads, int64_t n_kv_heads, int64_t head_dim, int64_t ffn,
                       double rope_theta, float rms_eps, int group, int grid_mode,
                       const float* const* taus, const int64_t* n_steps, float lr, float beta1,
                       float beta2, uint64_t seed, float* x_out, void* const* packed,
                       uint16_t* const* scales_f16, float* const* scales_f32, double* stats,
                       void* stream) {
  if (!x_in || !W || !taus || !n_steps || !x_out) return GSQ_ERR_INVALID_ARG;
  for (int i = 0; i < 7; ++i)
    if (!W[i]) return GSQ_ERR_INVALID_ARG;
  for (int j = 0; j < 4; ++j) {
    if (n_steps[j] < 0 || (n_steps[j] > 0 && !taus[j])) return GSQ_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n_steps[j]; ++i)
      if (!stage_step_args_ok(taus[j][i], lr, beta1, beta2)) return GSQ_ERR_INVALID_ARG;
  }
  if (stage_num_logits(grid_mode) < 0 || group <= 0) return GSQ_ERR_INVALID_ARG;
  if (group != kStageGroup) return GSQ_ERR_UNSUPPORTED;
  Dims D;
  int rc = check_dims(&D, n_seq, seq_len, n_heads, n_kv_heads, head_dim, ffn, rope_theta, rms_eps);
  if (rc != GSQ_OK) return rc;
  int sms = 0;
  if ((rc = sm100_sms(&sms)) != GSQ_OK) return rc;
  if (stats)
    for (int i = 0; i < 20; ++i) stats[i] = std::nan("");

  Arena A;
  A.st = static_cast<cudaStream_t>(stream);
  Gemm G;
  if (!gemm_setup(A, G, sms)) return A.status;
  const int64_t T = D.T, H = D.H, TH = T * H;
  const float* x = static_cast<const float*>(device_view(A, x_in, (size_t)TH * 4));
  const __nv_bfloat16* Wfp[7];
  for (int i = 0; i < 7; ++i)
    Wfp[i] = static_cast<const __nv_bfloat16*>(
        device_view(A, W[i], (size_t)D.rows(i) * D.cols(i) * 2));
  // hard weights and their packed form, per weight
  __nv_bfloat16* Wq[7];
  uint32_t* pk[7];
  float* sc[7];
  for (int i = 0; i < 7; ++i) {
    size_t pb = 0;
    gsq_packed_bytes(grid_mode, D.rows(i), D.cols(i), &pb);
    Wq[i] = A.get<__nv_bfloat16>(D.rows(i) * D.cols(i));
    pk[i] = A.get<uint32_t>(pb / 4);
    sc[i] = A.get<float>(D.rows(i) * (D.cols(i) / kStageGroup));
  }
  __nv_bfloat16* xa = A.get<__nv_bfloat16>(TH);
  float* attn_fp = A.get<float>(TH);
  float* y_fp = A.get<float>(TH);
  if (A.status != GSQ_OK) return A.status;

  // 1. the full-precision block: xa, attn_fp (the V/O target), y_fp
  {
    float* h = A.get<float>(TH);
    float* m = A.get<float>(TH);
    __nv_bfloat16* xm = A.get<__nv_bfloat16>(TH);
    residual_rmsnorm(D, A, x, nullptr, nullptr, xa);
    attn_sublayer(D, G, xa, Wfp, attn_fp);
    residual_rmsnorm(D, A, x, attn_fp, h, xm);
    mlp_sublayer(D, G, xm, Wfp, m);
    add(D, A, sms, h, m, y_fp);
    if (gemm_error(A, G) != GSQ_OK) return A.status;
    A.release(h);
    A.release(m);
    A.release(xm);
  }
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (!A.ok(cudaEventCreate(&e0)) || !A.ok(cudaEventCreate(&e1))) {
    if (e0) cudaEventDestroy(e0);
    return A.status;
  }
  struct EvGuard {
    cudaEvent_t a, b;
    ~EvGuard() { cudaEventDestroy(a); cudaEventDestroy(b); }
  } evg{e0, e1};
  // harden weight `wi` through the stage's own harden/pack, then dequantize
  auto harden = [&](int wi, int status) {
    if (!A.ok_status(status)) return false;
    A.ok(launch_dequant(grid_mode, pk[wi], sc[wi], D.rows(wi), D.cols(wi), Wq[wi], sms, A.st));
    return A.status == GSQ_OK;
  };
  auto record = [&](int stage, double first, double last, double ab, double rel) {
    float ms = 0.f;
    cudaEventElapsedTime(&ms, e0, e1);
    if (!stats) return;
    double* o = stats + 5 * stage;
    o[0] = first;
    o[1] = last;
    o[2] = ab;
    o[3] = rel;
    o[4] = ms;
  };
  // 2. Q and K, each on its own output
  for (int j = 0; j < 2 && A.status == GSQ_OK; ++j) {
    gsq_ctx* c = nullptr;
    const uint64_t sj = seed ^ ((uint64_t)j << 56);
    if (!A.ok_status(gsq_init(&c, Wfp[j], GSQ_BF16, xa, GSQ_BF16, D.rows(j), H, T, group,
                              grid_mode, nullptr, sj, A.st)))
      break;
    double first = std::nan(""), last = std::nan(""), ab = 0, rel = 0;
    A.ok(cudaEventRecord(e0, A.st));
    if (n_steps[j] > 0 && A.ok_status(gsq_run(c, taus[j], 1, lr, beta1, beta2)) &&
        A.ok_status(gsq_last_loss(c, &first)) && n_steps[j] > 1)
      A.ok_status(gsq_run(c, taus[j] + 1, n_steps[j] - 1, lr, beta1, beta2));
    A.ok(cudaEventRecord(e1, A.st));
    if (A.status == GSQ_OK && n_steps[j] > 0) A.ok_status(gsq_last_loss(c, &last));
    if (A.status == GSQ_OK) A.ok_status(gsq_recon_error(c, GSQ_RECON_HARD, 1.f, &ab, &rel));
    if (A.status == GSQ_OK) harden(j, gsq_harden_pack(c, pk[j], nullptr, sc[j]));
    gsq_destroy(c);
    if (A.status == GSQ_OK) record(j, first, last, ab, rel);
  }
  if (A.status != GSQ_OK) return A.status;

  // 3. V and O jointly, probabilities from the quantized Q, K
  {
    gsq_attn* c = nullptr;
    const uint64_t s2 = seed ^ ((uint64_t)2 << 56);
    if (!A.ok_status(gsq_attn_init(&c, xa, GSQ_BF16, attn_fp, GSQ_F32, Wq[0], Wq[1], Wfp[2],
                                   Wfp[3], GSQ_BF16, D.nseq, D.S, D.nh, D.nkv, D.d, D.theta,
                                   group, grid_mode, s2, A.st)))
      return A.status;
    double first = std::nan(""), last = std::nan(""), ab = 0, rel = 0;
    A.ok(cudaEventRecord(e0, A.st));
    if (n_steps[2] > 0 && A.ok_status(gsq_attn_run(c, taus[2], 1, lr, beta1, beta2)) &&
        A.ok_status(gsq_attn_last_loss(c, &first)) && n_steps[2] > 1)
      A.ok_status(gsq_attn_run(c, taus[2] + 1, n_steps[2] - 1, lr, beta1, beta2));
    A.ok(cudaEventRecord(e1, A.st));
    if (A.status == GSQ_OK && n_steps[2] > 0) A.ok_status(gsq_attn_last_loss(c, &last));
    if (A.status == GSQ_OK) A.ok_status(gsq_attn_recon_error(c, GSQ_RECON_HARD, 1.f, &ab, &rel));
    for (int i = 0; i < 2 && A.status == GSQ_OK; ++i)
      harden(2 + i, gsq_attn_harden_pack(c, i, pk[2 + i], nullptr, sc[2 + i]));
    gsq_attn_destroy(c);
    if (A.status != GSQ_OK) return A.status;
    record(2, first, last, ab, rel);
  }

  // 4. the quantized attention residual, then the MLP on the block output
  float* h_q = A.get<float>(TH);
  float* r_m = A.get<float>(TH);
  __nv_bfloat16* xm_q = A.get<__nv_bfloat16>(TH);
  if (A.status != GSQ_OK) return A.status;
  {
    float* t32 = A.get<float>(TH);
    attn_sublayer(D, G, xa, Wq, t32);
    residual_rmsnorm(D, A, x, t32, h_q, xm_q, y_fp, r_m);  // h_q, xm_q, y_fp - h_q
    if (gemm_error(A, G) != GSQ_OK) return A.status;
    A.release(t32);
    A.release(attn_fp);
    A.release(xa);
  }
  {
    gsq_mlp* c = nullptr;
    const uint64_t s3 = seed ^ ((uint64_t)3 << 56);
    if (!A.ok_status(gsq_mlp_init(&c, xm_q, GSQ_BF16, r_m, GSQ_F32, Wfp[4], Wfp[5], Wfp[6],
                                  GSQ_BF16, T, H, D.F, group, grid_mode, s3, A.st)))
      return A.status;
    double first = std::nan(""), last = std::nan(""), ab = 0, rel = 0;
    A.ok(cudaEventRecord(e0, A.st));
    if (n_steps[3] > 0 && A.ok_status(gsq_mlp_run(c, taus[3], 1, lr, beta1, beta2)) &&
        A.ok_status(gsq_mlp_last_loss(c, &first)) && n_steps[3] > 1)
      A.ok_status(gsq_mlp_run(c, taus[3] + 1, n_steps[3] - 1, lr, beta1, beta2));
    A.ok(cudaEventRecord(e1, A.st));
    if (A.status == GSQ_OK && n_steps[3] > 0) A.ok_status(gsq_mlp_last_loss(c, &last));
    if (A.status == GSQ_OK) A.ok_status(gsq_mlp_recon_error(c, GSQ_RECON_HARD, 1.f, &ab, &rel));
    for (int i = 0; i < 3 && A.status == GSQ_OK; ++i)
      harden(4 + i, gsq_mlp_harden_pack(c, i, pk[4 + i], nullptr, sc[4 + i]));
    gsq_mlp_destroy(c);
    if (A.status != GSQ_OK) return A.status;
    record(3, first, last, ab, rel);
  }

  // 5. x_out = h_q + MLP_q(xm_q)
  {
    float* m = A.get<float>(TH);
    float* y = A.get<float>(TH);
    mlp_sublayer(D, G, xm_q, Wq, m);
    add(D, A, sms, h_q, m, y);
    A.ok(cudaMemcpyAsync(x_out, y, (size_t)TH * 4, cudaMemcpyDefault, A.st));
  }
  // packed codes and scales to the caller
  for (int i = 0; i < 7 && A.status == GSQ_OK; ++i) {
    const int64_t ng = D.rows(i) * (D.cols(i) / kStageGroup);
    size_t pb = 0;
    gsq_packed_bytes(grid_mode, D.rows(i), D.cols(i), &pb);
    if (packed && packed[i])
      A.ok(cudaMemcpyAsync(packed[i], pk[i], pb, cudaMemcpyDefault, A.st));
    if (scales_f32 && scales_f32[i])
      A.ok(cudaMemcpyAsync(scales_f32[i], sc[i], (size_t)ng * 4, cudaMemcpyDefault, A.st));
    if (scales_f16 && scales_f16[i]) {
      uint16_t* h16 = scales_f16[i];
      uint16_t* tmp = stage_is_device_ptr(h16) ? h16 : A.get<uint16_t>(ng);
      if (A.status != GSQ_OK) break;
      A.ok(launch_export_scales(sc[i], ng, tmp, nullptr, A.st));
      if (tmp != h16) A.ok(cudaMemcpyAsync(h16, tmp, (size_t)ng * 2, cudaMemcpyDefault, A.st));
    }
  }
  return gemm_error(A, G);
}

}  // extern "C"
