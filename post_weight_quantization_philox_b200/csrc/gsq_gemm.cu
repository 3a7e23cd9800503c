// gsq_gemm.cu -- the two dense contractions of the GSQ step on the sm_100a
// tensor cores: C[M x N] = A[M x Kc] . B[N x Kc]^T with both operands
// K-major bf16, fp32 accumulation in TMEM.
//
//   forward:          Y^T = What . Xb^T   (M = N_out, N = Tp, Kc = K), fused
//                     epilogue E = Y^T - Yref^T, loss += sum E^2,
//                     dY^T = bf16(2E)
//   weight gradient:  dW = dY^T . Xt^T    (M = N_out, N = K,  Kc = Tp)
//   reference output: Yref^T = W . Xb^T at init (fp32 store)
//
// Design: persistent CTAs (one per SM), 128 x 256 output tiles, 64-wide K
// slabs staged by TMA (128-byte swizzle) in a 4-deep ring of shared-memory
// stages; warp 0 issues TMA, one thread of warp 1 issues tcgen05.mma into
// one of two 256-column TMEM accumulators, warps 2..5 drain the other
// accumulator through tcgen05.ld so the epilogue of tile i overlaps the
// main loop of tile i+1.  No cluster multicast is used.  Every mbarrier
// wait is bounded: on timeout the kernel records DEV_ERR_TIMEOUT, drains
// its in-flight copies and MMAs, frees TMEM and returns.
#include "gsq_device.cuh"
#include "gsq_internal.h"

namespace gsq {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int NUM_THREADS = 192;
constexpr long long WAIT_LIMIT = 4000000000LL;  // clock cycles (~2 s)
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  double red[4];
};

constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + (int)sizeof(Ctl);

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
  const bool ok = mbar_wait_bounded(bar, parity, WAIT_LIMIT);
  return __all_sync(0xffffffffu, ok);
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA,
           const __grid_constant__ CUtensorMap tmB, int64_t M, int64_t N,
           int64_t Kc, EpiParams ep) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (int)((M + BM - 1) / BM);
  const int n_tiles = (int)((N + BN - 1) / BN);
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = (int)((Kc + BK - 1) / BK);
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&ctl->tfull[b]), 1);
      mbar_init(smem_u32(&ctl->tempty[b]), 4);
    }
    mbar_init(smem_u32(&ctl->done), 1);
    ctl->abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mb = tile % m_tiles, nb = tile / m_tiles;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&ctl->empty[stage]), ph ^ 1,
                                 WAIT_LIMIT) ||
              *(volatile int*)&ctl->abort) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&ctl->full[stage]);
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          tma_load_2d(sa, &tmA, fb, kb * BK, mb * BM);
          tma_load_2d(sa + A_BYTES, &tmB, fb, kb * BK, nb * BN);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
        *(volatile int*)&ctl->abort = 1;
      }
      // drain: the last load issued into each stage has landed
      for (int s = 0; s < STAGES; ++s) {
        if (issued <= s) break;
        const long long last = ((issued - 1 - s) / STAGES) * STAGES + s;
        const uint32_t par = (uint32_t)((last / STAGES) & 1);
        if (!mbar_wait_bounded(smem_u32(&ctl->full[s]), par, WAIT_LIMIT))
          atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait_bounded(smem_u32(&ctl->tempty[acc]), aph ^ 1,
                               WAIT_LIMIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait_bounded(smem_u32(&ctl->full[stage]), ph,
                                 WAIT_LIMIT) ||
              *(volatile int*)&ctl->abort) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * STAGE_BYTES;
          const uint64_t ad = sdesc_kmajor_sw128(sa);
          const uint64_t bd = sdesc_kmajor_sw128(sa + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(d_tmem, ad + 2 * k, bd + 2 * k, IDESC,
                      (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(smem_u32(&ctl->empty[stage]));
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(smem_u32(&ctl->tfull[acc]));
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      if (!ok) {
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
        *(volatile int*)&ctl->abort = 1;
      }
      // drain: every MMA this thread issued has completed
      umma_commit(smem_u32(&ctl->done));
      if (!mbar_wait_bounded(smem_u32(&ctl->done), 0, WAIT_LIMIT))
        atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t aph = 0;
    double lsum = 0.0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % m_tiles, nb = tile / m_tiles;
      if (!warp_wait(smem_u32(&ctl->tfull[acc]), aph) ||
          *(volatile int*)&ctl->abort) {
        if (lane == 0) {
          atomicCAS(ep.err, 0, DEV_ERR_TIMEOUT);
          *(volatile int*)&ctl->abort = 1;
        }
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)mb * BM + r;
      const uint32_t tbase =
          tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      float part = 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), v);
        tmem_wait_ld();
        const int64_t col0 = (int64_t)nb * BN + c * 32;
        if (row < M && col0 < N) {
          if (EPI == EPI_STORE_F32) {
            float* dst = ep.out + row * ep.ldo + col0;
            if (col0 + 32 <= N && (ep.ldo & 3) == 0) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                reinterpret_cast<float4*>(dst)[j] =
                    make_float4(u2f(v[4 * j]), u2f(v[4 * j + 1]),
                                u2f(v[4 * j + 2]), u2f(v[4 * j + 3]));
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) dst[j] = u2f(v[j]);
            }
          } else {
            // N (= Tp) is a multiple of 64: whole 32-column chunks
            const float4* yr =
                reinterpret_cast<const float4*>(ep.yref + row * ep.ldy + col0);
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 y4 = __ldg(yr + j);
              const float e0 = u2f(v[4 * j]) - y4.x;
              const float e1 = u2f(v[4 * j + 1]) - y4.y;
              const float e2 = u2f(v[4 * j + 2]) - y4.z;
              const float e3 = u2f(v[4 * j + 3]) - y4.w;
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
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                                    pk[4 * j + 3]);
            }
          }
        }
      }
      lsum += (double)part;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->tempty[acc]));
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
    if (EPI != EPI_STORE_F32) {
      // deterministic loss: CTA partial in fixed order, last CTA sums all
      lsum = warp_sum_d(lsum);
      if (lane == 0) ctl->red[q] = lsum;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (warp == 2 && lane == 0) {
        const double cta = ctl->red[0] + ctl->red[1] + ctl->red[2] + ctl->red[3];
        ep.partials[blockIdx.x] = cta;
        __threadfence();
        const unsigned tk = atomicAdd(ep.ticket, 1u);
        if (tk == gridDim.x - 1) {
          __threadfence();
          double tot = 0.0;
          for (unsigned b = 0; b < gridDim.x; ++b)
            tot += *((volatile double*)ep.partials + b);
          *ep.loss_out = tot;
          if (!isfinite(tot)) atomicCAS(ep.err, 0, DEV_ERR_NONFINITE);
          *ep.ticket = 0u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType,
                                  cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& tmA, const CUtensorMap& tmB,
                       int64_t M, int64_t N, int64_t Kc, const EpiParams& ep,
                       int sm_count, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(
        k_gemm<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sm_count ? tiles : sm_count);
  k_gemm<EPI><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(tmA, tmB, M, N, Kc, ep);
  return cudaGetLastError();
}

}  // namespace

int make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows,
                   int64_t cols, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB,
                        int64_t M, int64_t N, int64_t Kc, int mode,
                        const EpiParams& ep, int sm_count, cudaStream_t st) {
  switch (mode) {
    case EPI_STORE_F32:
      return launch_epi<EPI_STORE_F32>(tmA, tmB, M, N, Kc, ep, sm_count, st);
    case EPI_LOSS_DY:
      return launch_epi<EPI_LOSS_DY>(tmA, tmB, M, N, Kc, ep, sm_count, st);
    default:
      return launch_epi<EPI_LOSS>(tmA, tmB, M, N, Kc, ep, sm_count, st);
  }
}

}  // namespace gsq
