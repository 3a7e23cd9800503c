// gsq_internal.h -- launchers shared by the translation units of libgsq.
#pragma once

#include <atomic>
#include <vector>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace gsq {

// NVTX range around the host-side issue of a step or phase (names such as
// "gsq_step/backward"), so a profiler's timeline shows where each step's
// kernels come from; inert when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// device-side error codes written into the context's error word
enum : int {
  DEV_OK = 0,
  DEV_ERR_TIMEOUT = 1,    // a bounded mbarrier wait gave up
  DEV_ERR_NONFINITE = 2,  // NaN / Inf in an input or a loss
  DEV_ERR_BAD_INIT = 3    // init_idx out of the grid's range
};

// ---------------------------------------------------------------- GEMM
enum EpiMode : int {
  EPI_STORE_F32 = 0,  // C = acc (fp32 store)
  EPI_LOSS_DY = 1,    // E = acc - Yref; loss += sum E^2; dY = bf16(2E)
  EPI_LOSS = 2,       // E = acc - Yref; loss += sum E^2
  EPI_STORE_BF16 = 3,  // C = bf16(acc)
  EPI_MERGED = 4,      // a forward (EPI_LOSS_DY) and a weight-gradient
                       // (EPI_STORE_F32) problem in one launch (MergeArgs)
  EPI_SUB_F32 = 5      // C = C - acc in place (fp32; C read through the
                       // Y_ref map, written through the out map)
};

struct EpiParams {
  double* partials;      // one slot per CTA
  unsigned* ticket;      // zero between launches
  double* loss_out;      // final loss (fp64)
  int* err;              // device error word
  // test hook: before any load or MMA is issued, one thread per CTA waits
  // (bounded, about 10 ms) on a barrier nothing arrives at, records
  // DEV_ERR_TIMEOUT, and the CTA then processes no tile
  int stall_probe = 0;
};

// The epilogue's tensor maps: out = C (EPI_STORE_F32, fp32 map; EPI_STORE_BF16,
// bf16 map) or dY (EPI_LOSS_DY, bf16 map); yref = Y_ref (EPI_LOSS*, fp32 map).
// Unused maps may be any valid map.
struct EpiMaps {
  CUtensorMap out;
  CUtensorMap yref;
};

// Per-phase device time of a block stage's steps: when on, an event is
// recorded on the stage's stream before each launch, tagged with the phase
// of that launch, and one tagged -1 after the step's last launch; the time
// between an event and the next is the tagged launch's.  collect() syncs,
// sums milliseconds and launches per phase, and starts over.  (The events
// keep each kernel from starting before the previous one ends, so timings
// come from a separate run of the same steps.)
struct PhaseClock {
  bool on = false;
  std::vector<cudaEvent_t> ev;
  std::vector<int> tag;
  size_t used = 0;
  cudaError_t mark(cudaStream_t st, int phase) {
    if (!on) return cudaSuccess;
    if (used == ev.size()) {
      cudaEvent_t e;
      const cudaError_t r = cudaEventCreate(&e);
      if (r != cudaSuccess) return r;
      ev.push_back(e);
      tag.push_back(-1);
    }
    tag[used] = phase;
    return cudaEventRecord(ev[used++], st);
  }
  cudaError_t collect(int nphase, double* ms, int64_t* launches) {
    for (int i = 0; i < nphase; ++i) {
      ms[i] = 0.0;
      launches[i] = 0;
    }
    if (used > 0) {
      const cudaError_t r = cudaEventSynchronize(ev[used - 1]);
      if (r != cudaSuccess) return r;
    }
    for (size_t i = 0; i + 1 < used; ++i) {
      if (tag[i] < 0 || tag[i] >= nphase) continue;
      float t = 0.f;
      const cudaError_t r = cudaEventElapsedTime(&t, ev[i], ev[i + 1]);
      if (r != cudaSuccess) return r;
      ms[tag[i]] += t;
      launches[tag[i]] += 1;
    }
    used = 0;
    return cudaSuccess;
  }
  void release() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    ev.clear();
    tag.clear();
    used = 0;
  }
};
// phases of a block stage's step
enum : int { PH_SOFT = 0, PH_GEMM = 1, PH_ELEM = 2, PH_BACKWARD = 3, PH_COUNT = 4 };

// The weight-gradient problem of a merged launch (launch_gemm_merged).  The
// forward problem's tiles [0, TF) come first, then the weight-gradient tiles
// (both in row-band order: every column tile of a band of 256 rows before the
// next band); both problems have the same M (the rows of W).  Every epilogue
// warp adds 1 to band_done[band] once a forward tile's dY stores are complete;
// a weight-gradient tile of a band waits until band_done[band] reaches target,
// i.e. until that band's dY rows (its A operand) are in memory.
struct MergeArgs {
  CUtensorMap tmA2, tmB2, tmO2;  // dY^T rows, X^T rows, dW (fp32 epilogue map)
  int64_t N2 = 0, Kc2 = 0;
  unsigned* band_done = nullptr;  // one counter per row band, never reset
  unsigned target = 0;            // generation x column tiles x 8 epilogue warps
};

// Opts kernel Fn in to `bytes` of dynamic shared memory on the current device,
// once per device (the attribute is per device; a process may drive several).
template <auto Fn>
inline cudaError_t smem_optin(int bytes) {
  static std::atomic<uint64_t> done{0};  // one bit per device ordinal < 64
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(Fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Pool test hook (gsq_debug_fail_alloc): true when this allocation is to fail.
bool pool_fail_injected();

// Device memory of the library (gsq_pool.cu): one pool per device that keeps
// freed memory reserved for the next allocation.  pool_malloc behaves as
// cudaMalloc on the current device (usable on any stream once it returns),
// pool_free as cudaFree (nothing in flight may still use the memory; null is
// ignored).  library_pool gives the pool itself for stream-ordered use.
cudaError_t pool_malloc(void** p, size_t bytes);
template <typename T>
inline cudaError_t pool_malloc(T** p, size_t bytes) {
  return pool_malloc(reinterpret_cast<void**>(p), bytes);
}
void pool_free(void* p);
cudaMemPool_t library_pool(int dev);

// Encodes a 2-D bf16 tensor map (rows x cols, row stride ld elements) with
// a box of box_rows x 64 elements and 128-byte swizzling (GEMM operands).
int make_tmap_bf16(CUtensorMap* map, const void* base, int64_t rows,
                   int64_t cols, int64_t ld, int box_rows);
// Tensor maps of the GEMM epilogue's 32 x 32 tiles: fp32 (128-byte rows,
// 128-byte swizzle) for stored or read fp32 outputs, bf16 (64-byte rows,
// 64-byte swizzle) for the bf16 output gradient.
int make_tmap_epi_f32(CUtensorMap* map, const void* base, int64_t rows,
                      int64_t cols, int64_t ld);
int make_tmap_epi_bf16(CUtensorMap* map, const void* base, int64_t rows,
                       int64_t cols, int64_t ld);

// Box rows of the tensor maps the GEMM expects for A and for B.
constexpr int kGemmBoxRowsA = 128;
constexpr int kGemmBoxRowsB = 128;

// C[M x N] = A[M x Kc] . B[N x Kc]^T with the epilogue selected by `mode`
// (CTA-pair tcgen05 kernel); tmA / tmB made by make_tmap_bf16 with
// kGemmBoxRowsA / kGemmBoxRowsB rows per box.
cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const EpiMaps& maps, int64_t M, int64_t N, int64_t Kc,
                        int mode, const EpiParams& ep, int sm_count,
                        cudaStream_t st);
cudaError_t launch_gemm_pair(const CUtensorMap& tmA, const CUtensorMap& tmB,
                             const EpiMaps& maps, int64_t M, int64_t N,
                             int64_t Kc, int mode, const EpiParams& ep,
                             int sm_count, cudaStream_t st);
// Forward (C = A . B^T with the loss + dY epilogue, maps as launch_gemm) and
// weight gradient (mg) in one persistent launch: the weight-gradient tiles of
// a row band start as soon as that band's forward tiles are done, so the two
// problems share one tail.  mg.band_done: M / 256 counters (rounded up).
cudaError_t launch_gemm_merged(const CUtensorMap& tmA, const CUtensorMap& tmB,
                               const EpiMaps& maps, int64_t M, int64_t N, int64_t Kc,
                               const MergeArgs& mg, const EpiParams& ep, int sm_count,
                               cudaStream_t st);
// Tiles of the two problems of a merged launch (its grid sizing) and the
// forward tiles per row band.
int64_t merged_tiles(int64_t M, int64_t N, int64_t N2);
int64_t merged_band_tiles(int64_t N);

// Many equal GEMMs in one launch.  Problem p = p1 * inner + p2 (p < count)
// is C_p[M x N] = A_p[M x Kc] . B_p[N x Kc]^T, where the operands and the
// output are windows of the tensor maps whose origin is
//   rows: x[0] * p1 + x[1] * p2,   K / columns: likewise
// for x = a_row / a_k (A), b_row / b_k (B), o_row / o_col (output).
// causal = 1 (lower-triangular A): the rows of A repeat in periods of `seg`
// rows, and an output tile whose rows sit at [r0, r0 + 256) of a period
// contracts over K in [0, r0 + 256) only (A is zero beyond).
// nseg > 1: K is `nseg` segments of `seg` columns (Kc = nseg seg); segment i
// of A starts at K column i a_seg_k and row offset i a_seg_row, of B at
// i b_seg_k and i b_seg_row.
// causal = 2 (transposed, with segments): a tile whose rows sit at
// [r0, r0 + 256) of M (M = seg) contracts over [r0, seg) of each segment
// only.  With causal, tiles with the longest K run first.
// o_fold > 0: local output row ly goes to row ly % o_fold, column offset
// (ly / o_fold) o_fold_col (rows of stacked heads placed side by side).
// Store epilogues only; Kc and, with causal, seg are multiples of 64 and seg
// of 256.
struct GemmSched {
  int count = 1, inner = 1;
  int64_t a_row[2] = {0, 0}, a_k[2] = {0, 0};
  int64_t b_row[2] = {0, 0}, b_k[2] = {0, 0};
  int64_t o_row[2] = {0, 0}, o_col[2] = {0, 0};
  int causal = 0;
  int64_t seg = 0;
  int nseg = 1;
  int64_t a_seg_k = 0, a_seg_row = 0, b_seg_k = 0, b_seg_row = 0;
  int64_t o_fold = 0, o_fold_col = 0;
  // tile order of a non-causal schedule: row tiles fastest within bands of
  // group_m row tiles, every column tile of a band before the next band
  // (1: row tiles fastest over all of them; 0: chosen by the launcher)
  int group_m = 0;
};
// Box rows of the B tensor map for the 128-wide output tiles (bn = 128).
constexpr int kGemmBoxRowsBNarrow = 64;
// bn = 256 (B map with kGemmBoxRowsB rows per box) or 128 (B map with
// kGemmBoxRowsBNarrow rows per box, for N = 128 problems).
// mode: EPI_STORE_F32 (tmOut an fp32 epilogue map) or EPI_STORE_BF16 (bf16).
cudaError_t launch_gemm_batched(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmOut, int64_t M, int64_t N,
                                int64_t Kc, int bn, const GemmSched& sc, int mode,
                                const EpiParams& ep, int sm_count, cudaStream_t st);

// GPTQ initial assignment (gsq_gptq.cu) on device inputs: levels (N x K
// int8 level indices) and scales (N x K/128) into device buffers; returns a
// GSQ status and leaves the stream synchronised.
int gptq_run(int mode, const void* Wd, int w_dtype, const void* Xd, int x_dtype, int64_t N,
             int64_t K, int64_t T, float damp, int8_t* levels, float* scales, int sm_count,
             cudaStream_t st);

// ------------------------------------------------------- elementwise
struct StepArgs {
  int mode;
  int state16 = 0;  // logits / momenta planes hold bf16 (reduced-memory state)
  int64_t N, K, G;
  const float* logits;   // L x N x K
  float* logits_w;       // same buffer, written by the backward
  float* mom;
  float* s;
  float* ms;
  const int8_t* i0;
  uint64_t seed;
  uint32_t t;
  int noise;
  float tau;
  // global coordinate of local coordinate 0 (row0 K for a shard of rows
  // [row0, row0 + N) of a larger layer): the Philox counters take global
  // coordinates, so a shard draws the noise the whole layer would
  uint64_t coord0 = 0;
};

cudaError_t launch_convert_x(const void* X, int dtype, int64_t T, int64_t K,
                             int64_t Tp, __nv_bfloat16* Xb, __nv_bfloat16* Xt,
                             __nv_bfloat16* Xcat, int* err, cudaStream_t st);
cudaError_t launch_convert_w(const void* W, int dtype, int64_t N, int64_t K,
                             float* W32, __nv_bfloat16* Wop, int split,
                             int* err, cudaStream_t st);
// state16: the logit planes hold bf16 (the pointers keep their float type;
// the launchers reinterpret them)
cudaError_t launch_init_state(int mode, const float* W32, const int8_t* init_idx,
                              int64_t N, int64_t K, float* s, int8_t* i0,
                              float* logits, int* err, cudaStream_t st, int state16 = 0);
// Soft weight of step a.t into What (and its fp32 values before rounding
// into wsoft32 when not null).
cudaError_t launch_soft_weight(const StepArgs& a, __nv_bfloat16* What, float* wsoft32,
                               int sm_count, cudaStream_t st);
// Backward + Lion of step a.t from dW (the step's probabilities are drawn
// again from the pre-update logits and the step's counters); with
// tau_next > 0 also the soft weight of step a.t + 1 into What.
cudaError_t launch_backward_lion(const StepArgs& a, const float* dW, float lr, float b1,
                                 float b2, float tau_next, __nv_bfloat16* What,
                                 float* dl_dbg, float* ds_dbg, int sm_count,
                                 cudaStream_t st);
cudaError_t launch_hard_weight(int mode, int64_t N, int64_t K,
                               const float* logits, const float* s,
                               const int8_t* i0, __nv_bfloat16* What,
                               cudaStream_t st, int state16 = 0);
cudaError_t launch_harden_pack(int mode, int64_t N, int64_t K,
                               const float* logits, const int8_t* i0,
                               uint32_t* packed, cudaStream_t st, int state16 = 0);
// scale-only step: int8 level codes of the hard choice; w = bf16(s c_code);
// ds_g = sum dW c_code and Lion on s (ds into ds_dbg when not null)
cudaError_t launch_hard_codes(int mode, int64_t N, int64_t K, const float* logits,
                              const int8_t* i0, int8_t* code, cudaStream_t st,
                              int state16 = 0);
cudaError_t launch_code_weight(int mode, int64_t N, int64_t K, const int8_t* code,
                               const float* s, __nv_bfloat16* What, cudaStream_t st);
cudaError_t launch_scale_lion(int mode, int64_t N, int64_t K, const int8_t* code,
                              const float* dW, float* s, float* ms, float lr, float b1,
                              float b2, float* ds_dbg, int sm_count, cudaStream_t st);
cudaError_t launch_export_scales(const float* s, int64_t n, uint16_t* f16,
                                 float* f32, cudaStream_t st);
cudaError_t launch_uniforms(int mode, uint64_t seed, uint32_t t,
                            uint64_t coord0, int64_t count, float* out,
                            cudaStream_t st);
// log2(u) of u = (m + 1/2) 2^-23 for m = m0 .. m0 + count - 1 (the noise's log2_unit)
cudaError_t launch_log2_unit(uint32_t m0, int64_t count, float* out, cudaStream_t st);
cudaError_t launch_sumsq(const float* x, int64_t n, double* partials,
                         unsigned* ticket, double* out, cudaStream_t st);
// SwiGLU MLP stage: h = bf16(silu(a) b); da = bf16(dh b silu'(a)),
// db = bf16(dh silu(a)); n a multiple of 4
cudaError_t launch_swiglu_fwd(const float* a, const float* b, int64_t n,
                              __nv_bfloat16* h, int sm_count, cudaStream_t st);
cudaError_t launch_swiglu_bwd(const float* a, const float* b, const float* dh,
                              int64_t n, __nv_bfloat16* da, __nv_bfloat16* db,
                              int sm_count, cudaStream_t st);
// out (cols x rows) = in (rows x cols)^T
cudaError_t launch_transpose_bf16(const __nv_bfloat16* in, int64_t rows,
                                  int64_t cols, __nv_bfloat16* out,
                                  cudaStream_t st);
cudaError_t launch_transpose_to_f32(const void* in, int in_bf16, int64_t rows,
                                    int64_t cols, float* out, cudaStream_t st);
// attention V/O stage
cudaError_t launch_rope(const float* x, int64_t T, int64_t cols, int64_t S, int d,
                        double theta, __nv_bfloat16* out, int sm_count, cudaStream_t st);
cudaError_t launch_causal_softmax(const float* scores, int64_t S, float scale,
                                  __nv_bfloat16* P, cudaStream_t st);
cudaError_t launch_transpose_ld(const __nv_bfloat16* in, int64_t rows, int64_t cols,
                                int64_t ld_in, __nv_bfloat16* out, int64_t ld_out,
                                cudaStream_t st);
cudaError_t launch_f32_to_bf16(const float* in, int64_t n, __nv_bfloat16* out,
                               int sm_count, cudaStream_t st);

}  // namespace gsq
