// gsq_gemm.cu -- tensor-map encoding for the GSQ GEMMs and the GEMM entry
// used by the rest of the library.  The contractions themselves
//
//   forward:          Y^T = What . Xb^T   (M = N_out, N = Tp, Kc = K), fused
//                     epilogue E = Y^T - Yref^T, loss += sum E^2,
//                     dY^T = bf16(2E)
//   weight gradient:  dW = dY^T . Xt^T    (M = N_out, N = K,  Kc = Tp)
//   reference output: Yref^T = W . Xb^T at init (fp32 store)
//
// run on the CTA-pair tcgen05 kernel in gsq_gemm_pair.cu.
#include "gsq_device.cuh"
#include "gsq_internal.h"

namespace gsq {

namespace {

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

}  // namespace

static int encode(CUtensorMap* map, CUtensorMapDataType dt, int esize,
                  const void* base, int64_t rows, int64_t cols, int64_t ld,
                  int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * esize)};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

int make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows,
                   int64_t cols, int64_t ld, int box_rows) {
  // 64 bf16 = 128-byte rows, the K slab of one pipeline stage
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, ld,
                64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

int make_tmap_epi_f32(CUtensorMap* map, const void* base, int64_t rows,
                      int64_t cols, int64_t ld) {
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, rows, cols, ld,
                32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
}

int make_tmap_epi_bf16(CUtensorMap* map, const void* base, int64_t rows,
                       int64_t cols, int64_t ld) {
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, rows, cols, ld,
                32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const EpiMaps& maps, int64_t M, int64_t N, int64_t Kc,
                        int mode, const EpiParams& ep, int sm_count,
                        cudaStream_t st) {
  return launch_gemm_pair(tmA, tmB, maps, M, N, Kc, mode, ep, sm_count, st);
}

}  // namespace gsq
