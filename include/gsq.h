/*
 * gsq.h -- C ABI of libgsq: the GSQ Gumbel-Softmax layer-reconstruction step
 * on one NVIDIA B200 (sm_100a).
 *
 * Method: "GSQ: Highly-Accurate Low-Precision Scalar Quantization for LLMs via
 * Gumbel-Softmax Sampling" (Dadgarnia et al., arXiv 2604.18556).  The method
 * paragraph of its summary on agihunt.info defines the state (per-coordinate
 * logits over a symmetric, zero-point-free, group-wise scalar grid plus one
 * learnable scale per group of 128), the relaxation (Gumbel-Softmax soft
 * weighted sum of grid points, annealed to a hard choice), the three grids
 * (2-bit: 4 levels, 4 logits; ternary: a mask choice times a sign choice;
 * 3 bits: 5 logits for shifts -2..+2 around the initial level) and the
 * objective (output reconstruction error on calibration inputs); its
 * optimisation paragraph names Lion; the Approach section on atlas.scime.ai
 * restates the same.  Noise comes from Philox4x32-10 (Salmon et al., SC'11).
 *
 * Notation: W (N x K) is the layer weight, X (T x K) the calibration inputs,
 * G = K / group groups per row, L logits per coordinate (4, 2+2, 5),
 * coord = n*K + k.  One step t computes
 *     u   = Philox4x32-10(key = seed, ctr = (coord lo, coord hi, t, 0)), words
 *           0..3; the 3-bit grid's fifth: word coord % 4 of the block of
 *           ctr = (q lo, q hi, t, 1), q = coord - coord % 4
 *     g   = -log(-log u),  y = softmax((l + g) / tau),  v = sum y_k c_k,
 *     What = bf16(s_g * v),
 *     loss = || X What^T - X W^T ||_F^2,   dY = 2 E,   dWhat = dY^T X,
 *     dl, ds from the softmax Jacobian;  Lion on logits and scales.
 *
 * Conventions for every entry point:
 *   - returns GSQ_OK (0) or a negative status; never throws, never aborts;
 *   - a CUDA error or a device-side failure puts the context into a sticky
 *     failed state: later calls return GSQ_ERR_STATE;
 *   - all device work is enqueued on the stream given to gsq_init (NULL =
 *     the legacy default stream); calls documented as "syncs" wait for it;
 *   - pointers documented "host or device" may point to pageable host,
 *     pinned host or device memory (unified addressing decides);
 *   - the context owns all of its device memory; callers own their buffers.
 */
#ifndef GSQ_H
#define GSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GSQ_API __attribute__((visibility("default")))
#else
#define GSQ_API
#endif

typedef struct gsq_ctx gsq_ctx; /* opaque, library-owned */

/* Grids (agihunt.info method paragraph).  Unit levels:
 *   GSQ_GRID_2BIT        {-1.5, -0.5, 0.5, 1.5}, 4 logits, scale absmax/1.5
 *   GSQ_GRID_TERNARY     {-1, 0, +1} as mask (zero, nonzero) x sign (-, +),
 *                        2 + 2 logits, scale absmax
 *   GSQ_GRID_3BIT_LOCAL  {-3.5 .. 3.5}, 5 logits for shifts -2..+2 around the
 *                        initial level, clamped to [0, 7], scale absmax/3.5 */
enum { GSQ_GRID_2BIT = 0, GSQ_GRID_TERNARY = 1, GSQ_GRID_3BIT_LOCAL = 2 };

/* element types of caller inputs */
enum { GSQ_F32 = 0, GSQ_BF16 = 1 };

enum {
    GSQ_OK = 0,
    GSQ_ERR_INVALID_ARG = -1, /* bad size, null pointer, unknown mode, tau <= 0 */
    GSQ_ERR_CUDA = -2,        /* a CUDA runtime call failed */
    GSQ_ERR_OOM = -3,         /* device allocation failed */
    GSQ_ERR_NONFINITE = -4,   /* a loss or an input was NaN / Inf */
    GSQ_ERR_STATE = -5,       /* context already failed or destroyed */
    GSQ_ERR_UNSUPPORTED = -6, /* e.g. group != 128, no sm_100 device */
    GSQ_ERR_TIMEOUT = -7      /* a bounded device-side wait gave up */
};

/* Recon-error modes */
enum { GSQ_RECON_HARD = 0, GSQ_RECON_SOFT = 1 };

/*
 * gsq_init -- A0 of the step: build the state of one layer.
 *   W        N x K row-major, w_dtype GSQ_F32 or GSQ_BF16, host or device.
 *   X        T x K row-major, x_dtype GSQ_F32 or GSQ_BF16, host or device.
 *   group    must be 128 (the pages' group size); K % 128 == 0.
 *   init_idx nullable; N x K int8 initial level index (2-bit 0..3, ternary
 *            0..2 for -1/0/+1, 3-bit 0..7), host or device.  NULL selects
 *            round-to-nearest (first level on ties) of W / s.  (The pages
 *            start from GPTQ; round-to-nearest is the stand-in.)
 *   seed     Philox key.
 *   stream   cudaStream_t (NULL = legacy default stream).
 * Computes bf16 X (and its transpose), Y_ref = bf16(X) W^T with fp32
 * accumulation (W at its own precision), s_g = absmax_g / c_max, the initial
 * levels, logits = +2 on the initial slot and 0 elsewhere, Lion momenta = 0,
 * step counter t = 0.  W, X and init_idx are read only during the call.
 * Syncs once at the end.  On failure *out is NULL.
 */
GSQ_API int gsq_init(gsq_ctx** out, const void* W, int w_dtype, const void* X,
             int x_dtype, int64_t N, int64_t K, int64_t T, int group,
             int grid_mode, const int8_t* init_idx, uint64_t seed,
             void* stream);

/* gsq_init_bf16_state -- gsq_init with the logits and their Lion momenta
 * stored as bf16 instead of fp32: half the state memory (the pages put the
 * logits alone at 2-5x the weight memory, agihunt.info summary, limitations
 * paragraph) and 32 fewer bytes per coordinate moved by every step's fused
 * backward for the 2-bit and ternary grids (40 for 3-bit).  Each step still
 * computes in fp32; after the Lion update the logits are rounded to bf16
 * stochastically (the fp32 bit pattern plus t << 7, truncated to its top 16
 * bits, where the 9-bit threshold t is the low 9 bits of the Philox word
 * that gives the same coordinate and logit its noise at the next step), so
 * a step smaller than half a bf16 unit still moves a logit in expectation;
 * the momenta are rounded to the nearest bf16.  Scales and their momenta
 * stay fp32.  Arguments and errors as gsq_init.  In this mode
 * GSQ_DBG_LOGITS / GSQ_DBG_MOM and the checkpoint's logit and momentum
 * sections hold bf16 (2 bytes per element). */
GSQ_API int gsq_init_bf16_state(gsq_ctx** out, const void* W, int w_dtype, const void* X,
                                int x_dtype, int64_t N, int64_t K, int64_t T, int group,
                                int grid_mode, const int8_t* init_idx, uint64_t seed,
                                void* stream);

/* gsq_init_rows -- gsq_init for the rows [row0, row0 + N) of a larger layer
 * (a shard; state_bf16 = 1 as gsq_init_bf16_state).  W holds those N rows
 * (N x K), X the whole calibration input, init_idx (nullable) the shard's
 * N x K initial levels.  The layer loss is a sum over output rows and every
 * group lies inside one row, so the shards of a layer are independent
 * problems: Y_ref of the shard is X W_shard^T, i.e. the columns row0 ..
 * row0 + N of the whole layer's reference output.  The Philox counters take
 * the global coordinate (row0 + n) K + k, so the shard draws exactly the
 * noise that a context holding the whole layer draws for those rows, and
 * the shards' steps together reproduce the whole layer's step (the sum of
 * the shards' losses is the layer's loss).  This is how a layer is split
 * over GPUs: one shard per GPU, no exchange during the steps.  (agihunt.info
 * summary, cost paragraph: the pages run the search on 8 GPUs.)
 * gsq_debug_uniforms keeps taking global coordinates.
 * Errors: as gsq_init, and GSQ_ERR_INVALID_ARG for row0 < 0, state_bf16
 * other than 0 or 1, or global coordinates beyond 2^62. */
GSQ_API int gsq_init_rows(gsq_ctx** out, const void* W, int w_dtype, const void* X,
                          int x_dtype, int64_t N, int64_t K, int64_t T, int group,
                          int grid_mode, const int8_t* init_idx, uint64_t seed,
                          int64_t row0, int state_bf16, void* stream);

/* GPTQ initial assignment (agihunt.info summary, optimisation paragraph: GSQ
 * starts from GPTQ; the algorithm of Frantar et al., "GPTQ: Accurate
 * Post-Training Quantization for Generative Pre-trained Transformers",
 * ICLR 2023), for the symmetric group-128 grids of grid_mode:
 *   H = bf16(X)^T bf16(X); dead inputs (H_ii = 0): H_ii = 1, W[:, i] = 0;
 *   H += damp mean(diag H) I; U = upper Cholesky factor of H^-1;
 *   columns in input order: at the first column of each group the scale is
 *   absmax / c_max of the (updated) group; the column is rounded to the
 *   nearest level (first on ties) and its error (w - s c) / U_jj is pushed
 *   onto the later columns through row j of U.
 * Computed in fp32 on the GPU (Hessian on the tensor cores).
 * W (N x K) and X (T x K): fp32 or bf16 (w_dtype, x_dtype), host or device,
 * read only.  levels (N x K int8 level indices, the init_idx of gsq_init)
 * and scales (N x K/group fp32): caller-owned, host or device.  damp >= 0
 * (GPTQ's default 0.01).  Synchronises the stream.  Its workspace (about
 * 8 K^2 + 8 N K bytes) comes from the library's memory pool (see
 * gsq_release_cached_memory).
 * Errors: GSQ_ERR_INVALID_ARG for bad sizes / pointers / dtypes / damp or
 * K > 65536; GSQ_ERR_UNSUPPORTED for group != 128 or a non-sm_100 device;
 * GSQ_ERR_NONFINITE if the damped Hessian is not positive definite in fp32
 * or an input is not finite; GSQ_ERR_OOM. */
GSQ_API int gsq_gptq(const void* W, int w_dtype, const void* X, int x_dtype, int64_t N,
                     int64_t K, int64_t T, int group, int grid_mode, float damp,
                     int8_t* levels, float* scales, void* stream);
/* Device memory: every buffer the library allocates (contexts of all kinds,
 * init-time staging, the GPTQ workspace) comes from one memory pool per
 * device that the library owns.  Freed memory stays reserved in the pool --
 * all of it by default -- so that the next context or call of a similar size
 * maps no new pages (mapping costs tens of milliseconds per GB; a block's MLP
 * stage holds about 45 GB).
 * gsq_set_cached_memory_limit: keep at most `bytes` reserved per device
 * (applies to the pools that exist and to later ones; the excess goes back
 * at the next synchronisation).  gsq_release_cached_memory: return what the
 * pools hold in reserve (all devices) to the driver now; memory of live
 * contexts stays.  Call either with no library call running.
 * Errors: GSQ_ERR_CUDA. */
GSQ_API int gsq_set_cached_memory_limit(uint64_t bytes);
GSQ_API int gsq_release_cached_memory(void);
/* Failure-injection hooks for tests (host side; no GPU fault is involved).
 * gsq_debug_fail_alloc(after): the library's device allocation that comes
 * after `after` more successful ones fails as if the device were out of
 * memory (so 0 fails the next one); a negative value switches the hook off.
 * Process-wide, all devices.  gsq_debug_pool_used(device, bytes): the bytes
 * of the device's pool that are handed out (contexts, workspaces) -- 0
 * before the library first allocates on that device; waits for frees the
 * library queued.  Errors: GSQ_ERR_INVALID_ARG (null bytes, bad device),
 * GSQ_ERR_CUDA. */
GSQ_API int gsq_debug_fail_alloc(int64_t after);
GSQ_API int gsq_debug_pool_used(int device, uint64_t* bytes);
/* gsq_init from the GPTQ assignment: the initial levels (init_idx) and the
 * group scales both come from gsq_gptq (instead of round-to-nearest with
 * absmax scales); everything else as gsq_init.  Synchronises the stream. */
GSQ_API int gsq_init_gptq(gsq_ctx** out, const void* W, int w_dtype, const void* X,
                          int x_dtype, int64_t N, int64_t K, int64_t T, int group,
                          int grid_mode, float damp, uint64_t seed, void* stream);

/*
 * gsq_step -- one reconstruction step at temperature tau (asynchronous):
 * soft weight (noise of step t), forward GEMM with fused loss and dY,
 * weight-gradient GEMM, fused logit/scale gradients and Lion update
 * (c = beta1 m + (1-beta1) g; theta -= lr sign(c); m = beta2 m + (1-beta2) g),
 * then t += 1.  tau > 0, lr >= 0, 0 <= beta < 1.  The annealing schedule is
 * the caller's.  Source: agihunt.info summary, method paragraph (the soft
 * weighted sum of grid points under Gumbel-Softmax sampling, trained on the
 * output reconstruction error and annealed towards a hard choice) and
 * optimisation paragraph (Lion, logits trained jointly with the group
 * scales); atlas.scime.ai, Approach.  Lion itself: Chen et al., "Symbolic
 * Discovery of Optimization Algorithms", 2023.
 * Errors: GSQ_ERR_INVALID_ARG for tau <= 0 or not finite, lr < 0 or beta
 * outside [0, 1); GSQ_ERR_UNSUPPORTED once t reaches 2^32 - 2 (the counter
 * word); GSQ_ERR_STATE after an earlier failure (a device-side failure of
 * this step surfaces at the next call that syncs).
 */
GSQ_API int gsq_step(gsq_ctx* ctx, float tau, float lr, float beta1, float beta2);

/*
 * gsq_step_next -- gsq_step at tau whose fused backward also forms the soft
 * weight of the next step at tau_next (its noise and tempered softmax from
 * the updated logits and scales), so that the next gsq_step or
 * gsq_step_next call at that temperature starts at its forward GEMM: a
 * caller-driven loop of gsq_step_next(tau_t, tau_{t+1}) costs what gsq_run
 * costs and gives the same results bit for bit.  A next call at another
 * temperature recomputes its soft weight.  Errors: as gsq_step, and
 * GSQ_ERR_INVALID_ARG for tau_next <= 0 or not finite.
 */
GSQ_API int gsq_step_next(gsq_ctx* ctx, float tau, float tau_next, float lr, float beta1,
                          float beta2);

/*
 * gsq_run -- n consecutive steps at temperatures taus[0..n) (host array),
 * asynchronous.  Same results, bit for bit, as n calls of gsq_step; the
 * backward of each step but the last also builds the next step's soft weight
 * and Gumbel noise, so no step re-reads the logits for its soft weight.
 */
GSQ_API int gsq_run(gsq_ctx* ctx, const float* taus, int64_t n, float lr,
                    float beta1, float beta2);

/* Scale-only step (agihunt.info summary, optimisation paragraph: the 2-bit
 * models get one more round that changes only the group scales), on the
 * layer objective of gsq_step:
 *   codes   = hard choice of the current logits (argmax, first maximum, no
 *             noise; computed once and kept until the logits change),
 *   w       = bf16(s_g c_code)                  (N x K),
 *   loss, dY^T, dW as in gsq_step,
 *   ds_g    = sum over group g of dW_i c_code(i),
 *   Lion on s with momentum ms (as in gsq_step).
 * Logits, their momenta and i0 are left as they are.  The step counter t
 * advances and the loss goes to the same history as gsq_step's.  Enqueued
 * on the context's stream without a host sync.
 * Errors: GSQ_ERR_INVALID_ARG for lr < 0 or beta outside [0, 1);
 * GSQ_ERR_STATE after an earlier failure. */
GSQ_API int gsq_scale_step(gsq_ctx* ctx, float lr, float beta1, float beta2);
/* n scale-only steps (n > 0) */
GSQ_API int gsq_scale_run(gsq_ctx* ctx, int64_t n, float lr, float beta1, float beta2);

/* gsq_last_loss -- loss (sum of squared errors) of the last step.  Syncs.
 * GSQ_ERR_NONFINITE if it was NaN / Inf; GSQ_ERR_STATE before any step. */
GSQ_API int gsq_last_loss(gsq_ctx* ctx, double* loss);

/* gsq_loss_history -- losses of steps [t0, t0 + n) (the last 4096 steps are
 * kept); host output.  Syncs. */
GSQ_API int gsq_loss_history(gsq_ctx* ctx, uint64_t t0, int64_t n, double* host_out);

/* gsq_packed_bytes -- bytes of the packed code stream for an N x K layer:
 * N * K * b / 8 with b = 2 (2-bit, ternary) or 3 (3-bit).  Host only. */
GSQ_API int gsq_packed_bytes(int grid_mode, int64_t N, int64_t K, size_t* bytes);

/*
 * gsq_harden_pack -- A6: hard level = argmax of the logits (first maximum,
 * no noise; 3-bit: clamp(i0 + argmax - 2, 0, 7); ternary: zero if the mask
 * pair prefers zero, else the sign pair's choice), packed as an LSB-first
 * bitstream per row of 32-bit little-endian words (code j of a row at bits
 * [j b, j b + b)); the code is the level index (ternary: v + 1).  Source:
 * agihunt.info summary, method paragraph (as the temperature falls the soft
 * sum collapses to a hard choice of grid point) and its conclusion
 * (symmetric group-128 grids, no zero-point, so one fp16 scale per group is
 * the whole side information: 2.13 bits per weight at 2 bits in the
 * zero-shot table).  The bit layout is this library's.
 *   packed      gsq_packed_bytes() bytes, host or device.
 *   scales_f16  N x G binary16 (round to nearest even), host or device,
 *               nullable.
 *   scales_f32  N x G fp32, host or device, nullable.
 * Syncs.
 */
GSQ_API int gsq_harden_pack(gsq_ctx* ctx, void* packed, uint16_t* scales_f16,
                    float* scales_f32);

/*
 * gsq_recon_error -- A7: abs = || bf16(X) Wq^T - Y_ref ||_F^2 and
 * rel = abs / || Y_ref ||_F^2 with Wq the hard weight (GSQ_RECON_HARD) or
 * the noiseless soft weight at tau (GSQ_RECON_SOFT; tau ignored for hard).
 * Syncs.  Leaves the optimiser state untouched.  Source: the layer's output
 * reconstruction error on the calibration inputs, the objective named in the
 * agihunt.info summary, method paragraph.
 * Errors: GSQ_ERR_INVALID_ARG for a bad mode, a null output or a soft tau
 * that is not positive and finite; GSQ_ERR_STATE after an earlier failure;
 * GSQ_ERR_NONFINITE if the error is NaN / Inf.
 */
GSQ_API int gsq_recon_error(gsq_ctx* ctx, int mode, float tau, double* abs_err,
                    double* rel_err);

/* Checkpoint: logits, momenta, scales, scale momenta, step counter.  The
 * noise is a pure function of (seed, t, coord), so resuming is bit-exact.
 * gsq_state_bytes gives the size; buffers are host memory.  Sync. */
GSQ_API int gsq_state_bytes(gsq_ctx* ctx, size_t* bytes);
GSQ_API int gsq_export_state(gsq_ctx* ctx, void* host_buf, size_t bytes);
GSQ_API int gsq_import_state(gsq_ctx* ctx, const void* host_buf, size_t bytes);

/* step counter t (the Philox counter word of the next step) */
GSQ_API int gsq_get_step(gsq_ctx* ctx, uint64_t* t);

/* gsq_destroy -- frees the context (syncs its stream).  NULL is a no-op. */
GSQ_API int gsq_destroy(gsq_ctx* ctx);

/* static string for a status code */
GSQ_API const char* gsq_error_string(int status);

/* ---------------------------------------------------------- measurement --
 * gsq_set_timing(ctx, on): record CUDA events on the context stream around
 * each phase of every step.  gsq_phase_times(ctx, ms[5], launches[5])
 * returns and resets the accumulated milliseconds and kernel launches of
 * 0 soft weight, 1 forward GEMM + loss, 2 weight-gradient GEMM,
 * 3 backward + Lion, 4 backward + Lion that also built the next step's soft
 * weight (gsq_run).  Syncs. */
GSQ_API int gsq_set_timing(gsq_ctx* ctx, int on);
GSQ_API int gsq_phase_times(gsq_ctx* ctx, double* ms, int64_t* launches);

/* ------------------------------------------------------------- testing --
 * These expose internal buffers and single phases so tests can compare each
 * phase with an independent implementation on identical inputs.
 *
 * gsq_debug_uniforms: the L Philox uniforms of coords [coord0, coord0+count)
 *   at step t, coordinate-major, into host memory.  Syncs.
 * gsq_debug_noise_log2: log2(u) as every step's noise forms it (the
 *   table-driven logarithm of the kernels) for the uniforms
 *   u = (m + 1/2) 2^-23, m = m0 .. m0 + count - 1, into host memory (count
 *   floats); m0 + count <= 2^23, else GSQ_ERR_INVALID_ARG.  Syncs.
 * gsq_debug_get / gsq_debug_set: copy an internal buffer to / from host
 *   memory; bytes must equal the buffer size.  Syncs.  Buffers:          */
enum {
    GSQ_DBG_LOGITS = 0,  /* L x N x K fp32 (planar)            */
    GSQ_DBG_MOM = 1,     /* L x N x K fp32                     */
    GSQ_DBG_SCALES = 2,  /* N x G fp32                         */
    GSQ_DBG_SMOM = 3,    /* N x G fp32                         */
    GSQ_DBG_I0 = 4,      /* N x K int8 initial level           */
    GSQ_DBG_WHAT = 5,    /* N x K bf16 soft weight             */
    GSQ_DBG_WSOFT32 = 6, /* N x K fp32 soft weight before rounding (filled
                            by gsq_debug_soft_weight)           */
    GSQ_DBG_DW = 7,      /* N x K fp32 weight gradient         */
    GSQ_DBG_DYT = 8,     /* N x Tp bf16 output gradient (transposed, Tp =
                            T rounded up to 64)                */
    GSQ_DBG_YREFT = 9,   /* N x Tp fp32 reference output (transposed) */
    GSQ_DBG_DL = 10,     /* L x N x K fp32 logit gradient (filled by
                            gsq_debug_backward)                 */
    GSQ_DBG_DS = 11      /* N x G fp32 scale gradient (ditto)   */
};
GSQ_API int gsq_debug_uniforms(gsq_ctx* ctx, uint32_t t, uint64_t coord0,
                       int64_t count, float* host_out);
GSQ_API int gsq_debug_noise_log2(gsq_ctx* ctx, uint32_t m0, int64_t count,
                                 float* host_out);
GSQ_API int gsq_debug_get(gsq_ctx* ctx, int which, void* host, size_t bytes);
GSQ_API int gsq_debug_set(gsq_ctx* ctx, int which, const void* host, size_t bytes);
/* noise on (default) / off; off sets g = 0 */
GSQ_API int gsq_debug_noise(gsq_ctx* ctx, int on);
/* single phases at the current t (t is not advanced):
 *   soft weight (also fills GSQ_DBG_WSOFT32), forward GEMM + loss (loss
 *   returned, syncs), weight-gradient GEMM, backward + Lion from the
 *   current dW (also fills GSQ_DBG_DL / GSQ_DBG_DS). */
GSQ_API int gsq_debug_soft_weight(gsq_ctx* ctx, float tau);
GSQ_API int gsq_debug_forward(gsq_ctx* ctx, double* loss);
GSQ_API int gsq_debug_weight_grad(gsq_ctx* ctx);
GSQ_API int gsq_debug_backward(gsq_ctx* ctx, float tau, float lr, float beta1,
                       float beta2);
/* scale-only backward + Lion from the current dW (fills GSQ_DBG_DS) */
GSQ_API int gsq_debug_scale_backward(gsq_ctx* ctx, float lr, float beta1, float beta2);
/* gsq_debug_stall_probe -- test hook of the bounded device waits: the next
 * forward GEMM of the context (in the next gsq_step / gsq_run) first lets
 * one thread of every CTA wait, with a short bound (about 10 ms), on a
 * barrier that nothing arrives at, before the CTA issues any load or MMA;
 * the wait runs out, the kernel records a timeout in the context's error
 * word and processes no tile, so no copy or MMA is ever in flight.  The
 * next call that syncs returns GSQ_ERR_TIMEOUT and the context turns
 * sticky-failed (GSQ_ERR_STATE afterwards), as after a real timeout.
 * Errors: GSQ_ERR_STATE after an earlier failure. */
GSQ_API int gsq_debug_stall_probe(gsq_ctx* ctx);

/* ----------------------------------------------- block stage: SwiGLU MLP --
 * The GSQ pages quantize a transformer block in stages; the last stage trains
 * the MLP on the block output (agihunt.info summary, optimisation paragraph).
 * gsq_mlp_* quantize the gate (F x H), up (F x H) and down (H x F)
 * projections jointly against
 *     loss = || D (silu(G Xn^T) * U Xn^T) - R^T ||_F^2
 * where Xn (T x H) is the normalised MLP input and R (T x H) the output the
 * MLP must produce (the full-precision block output minus the residual that
 * enters the MLP).  Each weight has its own logits, scales, Lion state and
 * Philox key (seed with weight index i xored into bits 48.. of the key);
 * soft weights, backward + Lion, harden/pack and the grids are those of the
 * single-layer entry points.  GEMM operands are bf16 with fp32 accumulation;
 * h = silu(a) b, 2E, da and db are rounded to bf16 as GEMM operands.
 *
 * gsq_mlp_init: Xn, R, Wg, Wu, Wd host or device, dtypes GSQ_F32 / GSQ_BF16;
 *   H and F multiples of 128 (the group), T a multiple of 64.  Syncs.
 * gsq_mlp_step / gsq_mlp_run: as gsq_step / gsq_run for the joint loss.
 * gsq_mlp_last_loss, gsq_mlp_recon_error (vs R; hard or noiseless soft),
 * gsq_mlp_harden_pack(which = 0 gate, 1 up, 2 down; host or device outputs)
 * as their single-layer counterparts.
 * gsq_mlp_debug_get / _set: which = 0..2 with a GSQ_DBG_* weight buffer
 *   (LOGITS, MOM, SCALES, SMOM, I0, WHAT, DW), or which = GSQ_MLP_STAGE with
 *   a GSQ_MLP_DBG_* stage buffer (all "T" layouts are transposed: F x T or
 *   H x T).
 */
typedef struct gsq_mlp gsq_mlp;
#define GSQ_MLP_STAGE 3
enum {
    GSQ_MLP_DBG_AT = 0,   /* F x T fp32  a^T = G Xn^T          */
    GSQ_MLP_DBG_BT = 1,   /* F x T fp32  b^T = U Xn^T          */
    GSQ_MLP_DBG_HT = 2,   /* F x T bf16  h^T = silu(a^T) b^T   */
    GSQ_MLP_DBG_DPT = 3,  /* H x T bf16  2 (pred^T - R^T)      */
    GSQ_MLP_DBG_DHT = 4,  /* F x T fp32  dh^T = D^T dp^T       */
    GSQ_MLP_DBG_DAT = 5,  /* F x T bf16  da^T                  */
    GSQ_MLP_DBG_DBT = 6,  /* F x T bf16  db^T                  */
    GSQ_MLP_DBG_RT = 7    /* H x T fp32  R^T                   */
};
GSQ_API int gsq_mlp_init(gsq_mlp** out, const void* Xn, int x_dtype,
                         const void* R, int r_dtype, const void* Wg,
                         const void* Wu, const void* Wd, int w_dtype,
                         int64_t T, int64_t H, int64_t F, int group,
                         int grid_mode, uint64_t seed, void* stream);
GSQ_API int gsq_mlp_step(gsq_mlp* ctx, float tau, float lr, float beta1,
                         float beta2);
GSQ_API int gsq_mlp_run(gsq_mlp* ctx, const float* taus, int64_t n, float lr,
                        float beta1, float beta2);
GSQ_API int gsq_mlp_last_loss(gsq_mlp* ctx, double* loss);
GSQ_API int gsq_mlp_recon_error(gsq_mlp* ctx, int mode, float tau,
                                double* abs_err, double* rel_err);
GSQ_API int gsq_mlp_harden_pack(gsq_mlp* ctx, int which, void* packed,
                                uint16_t* scales_f16, float* scales_f32);
GSQ_API int gsq_mlp_debug_get(gsq_mlp* ctx, int which, int buf, void* host,
                              size_t bytes);
GSQ_API int gsq_mlp_debug_set(gsq_mlp* ctx, int which, int buf,
                              const void* host, size_t bytes);
GSQ_API int gsq_mlp_get_step(gsq_mlp* ctx, uint64_t* t);
GSQ_API int gsq_mlp_destroy(gsq_mlp* ctx);
/* gsq_mlp_set_timing / gsq_mlp_phase_times: per-phase device time of the
 * stage's steps, as gsq_set_timing / gsq_phase_times for a layer: ms[4] and
 * launches[4] for 0 soft weights, 1 GEMMs (the seven contractions of a
 * step), 2 elementwise (SwiGLU forward and backward, transposes), 3 fused
 * backward + Lion of the three weights.  The events between launches keep
 * each kernel from starting early, so time a separate run.  phase_times
 * syncs and starts over.  Errors: GSQ_ERR_INVALID_ARG, GSQ_ERR_STATE. */
GSQ_API int gsq_mlp_set_timing(gsq_mlp* ctx, int on);
GSQ_API int gsq_mlp_phase_times(gsq_mlp* ctx, double* ms, int64_t* launches);

/* ------------------------------------------- block stage: attention V/O --
 * The GSQ pages quantize a block's query and key projections first, then the
 * value and output projections jointly (agihunt.info summary, optimisation
 * paragraph).  gsq_attn_* quantize Wv (nkv d x H) and Wo (H x H) jointly
 * against
 *     loss = || o Wo^T - R ||_F^2,   o_(s,h) = P_(s,h) (Xa Wv^T)_(s, h / grp)
 * with the attention probabilities P fixed: built once at init from the
 * attention input Xa (T x H, T = n_seq seq_len, H = n_heads head_dim) and the
 * given query / key weights Wq (H x H), Wk (nkv d x H) -- the frozen,
 * already quantized ones -- with the rotate-half rotary embedding (pairs
 * (i, i + d/2), angle p theta^(-2i/d) at position p within the sequence),
 * scaled scores Q K^T / sqrt(d), a causal mask and softmax; grouped
 * key/value heads (grp = n_heads / n_kv_heads query heads per value head).
 * R (T x H) is the output the stage must produce (the full-precision
 * attention output).  Q, K, P, V, o, 2E, do and dV are bf16 GEMM operands.
 * head_dim must be 128, seq_len a multiple of 128, group 128.
 * Entry points mirror gsq_mlp_*: which = 0 value, 1 output; stage buffers
 * under which = GSQ_ATTN_STAGE.
 */
typedef struct gsq_attn gsq_attn;
#define GSQ_ATTN_STAGE 2
enum {
    GSQ_ATTN_DBG_P = 0,   /* [s][h][q][key] bf16 attention probabilities */
    GSQ_ATTN_DBG_PT = 1,  /* [s][g][key][hig][q] bf16, same values        */
    GSQ_ATTN_DBG_VT = 2,  /* nkv d x T bf16  V^T = Wv Xa^T                */
    GSQ_ATTN_DBG_O = 3,   /* T x H bf16 attention output o                */
    GSQ_ATTN_DBG_DPT = 4, /* H x T bf16 2 (pred^T - R^T)                  */
    GSQ_ATTN_DBG_DV = 5,  /* T x nkv d bf16 value gradient dV             */
    GSQ_ATTN_DBG_RT = 6   /* H x T fp32 R^T                               */
};
GSQ_API int gsq_attn_init(gsq_attn** out, const void* Xa, int x_dtype,
                          const void* R, int r_dtype, const void* Wq,
                          const void* Wk, const void* Wv, const void* Wo,
                          int w_dtype, int64_t n_seq, int64_t seq_len,
                          int64_t n_heads, int64_t n_kv_heads,
                          int64_t head_dim, double rope_theta, int group,
                          int grid_mode, uint64_t seed, void* stream);
GSQ_API int gsq_attn_step(gsq_attn* ctx, float tau, float lr, float beta1,
                          float beta2);
GSQ_API int gsq_attn_run(gsq_attn* ctx, const float* taus, int64_t n,
                         float lr, float beta1, float beta2);
GSQ_API int gsq_attn_last_loss(gsq_attn* ctx, double* loss);
GSQ_API int gsq_attn_recon_error(gsq_attn* ctx, int mode, float tau,
                                 double* abs_err, double* rel_err);
GSQ_API int gsq_attn_harden_pack(gsq_attn* ctx, int which, void* packed,
                                 uint16_t* scales_f16, float* scales_f32);
GSQ_API int gsq_attn_debug_get(gsq_attn* ctx, int which, int buf, void* host,
                               size_t bytes);
GSQ_API int gsq_attn_debug_set(gsq_attn* ctx, int which, int buf,
                               const void* host, size_t bytes);
GSQ_API int gsq_attn_get_step(gsq_attn* ctx, uint64_t* t);
GSQ_API int gsq_attn_destroy(gsq_attn* ctx);
/* gsq_attn_set_timing / gsq_attn_phase_times: as gsq_mlp_set_timing, for the
 * V/O stage (GEMMs: V, the batched P V, the output projection with the
 * loss, dWo, do, the batched P^T do, dWv; elementwise: transposes). */
GSQ_API int gsq_attn_set_timing(gsq_attn* ctx, int on);
GSQ_API int gsq_attn_phase_times(gsq_attn* ctx, double* ms, int64_t* launches);

/* ------------------------------------------- staged block pipeline ------
 * GSQ quantizes the blocks of a model one after another: every block is
 * reconstructed from the output of the already quantized blocks before it,
 * and inside a block the query and key projections come first (each on its
 * own output), then the value and output projections together, then the MLP
 * on the block output (agihunt.info summary, optimisation paragraph).
 *
 * The block is a pre-norm Llama block on an fp32 residual stream x (T x H,
 * T = n_seq seq_len tokens, H = n_heads head_dim):
 *   xa = bf16(RMSNorm(x)),  h = x + Attn(xa),  xm = bf16(RMSNorm(h)),
 *   y  = h + bf16(silu(xm Wg^T) * (xm Wu^T)) Wd^T,
 * RMSNorm(v) = v / sqrt(mean(v^2) + rms_eps) (unit gain); Attn as in
 * gsq_attn_* (rotate-half rotary embedding with rope_theta, causal softmax of
 * Q K^T / sqrt(d), grouped key/value heads), then the output projection.
 * GEMMs take bf16 operands with fp32 accumulation; V, the attention output o
 * and silu(a) b are rounded to bf16 as GEMM operands.
 *
 * Weights W[7] in the order query (H x H), key (Hk x H), value (Hk x H),
 * output (H x H), gate (ffn x H), up (ffn x H), down (H x ffn), Hk =
 * n_kv_heads head_dim; bf16, row-major, host or device, read only.
 * head_dim must be 128, seq_len a multiple of 128 (at most 65536), ffn a
 * multiple of 128, n_heads a multiple of n_kv_heads.
 *
 * gsq_dequant -- the bf16 weight of a packed code stream (the output of
 *   gsq_harden_pack): W[n][k] = bf16(scales_f32[n][k / 128] c(code)) with c
 *   the grid's unit level of the code (2-bit code - 1.5, ternary code - 1,
 *   3-bit code - 3.5).  packed: gsq_packed_bytes bytes; scales_f32: N x K/128;
 *   W_bf16: N x K; each host or device.  Syncs.
 *
 * gsq_block_forward -- y (and h, nullable) of the block above for input x
 *   (T x H fp32, host or device) and weights W[7]; outputs T x H fp32, host
 *   or device.  Allocates its own scratch.  Syncs.
 *
 * gsq_block_quantize -- GSQ's staged reconstruction of one block:
 *   1. the full-precision block on x_in: the attention output attn_fp and y_fp;
 *   2. stage 0 (query) and stage 1 (key): a gsq_init context on xa with the
 *      full-precision weight's own output as target, gsq_run over taus[j];
 *   3. stage 2: gsq_attn_* with the probabilities of the quantized query and
 *      key weights, target attn_fp, over taus[2];
 *   4. h_q = x_in + Attn_q(xa); stage 3: gsq_mlp_* on bf16(RMSNorm(h_q))
 *      with target y_fp - h_q (the MLP is trained on the block output), over
 *      taus[3];
 *   5. x_out = h_q + MLP_q(bf16(RMSNorm(h_q))), the next block's input.
 *   Each stage's weights are hardened (argmax, packed, dequantized) before
 *   the next stage uses them.  Stage j draws its noise with Philox key
 *   seed ^ (j << 56) (joint stages further ^ (i << 48) for weight i).
 *   taus[j]: n_steps[j] temperatures (host arrays; n_steps[j] >= 0);
 *   lr, beta1, beta2 as gsq_step.  Outputs: x_out (T x H fp32, host or
 *   device); per weight i (arrays and entries nullable) packed[i]
 *   (gsq_packed_bytes bytes), scales_f16[i] / scales_f32[i] (rows x cols/128);
 *   stats (nullable, 4 x 5 doubles): per stage the first and the last step's
 *   loss, the final hard reconstruction error (abs, rel) and the milliseconds
 *   of its steps (CUDA events).  Every context and scratch buffer is freed
 *   before the call returns.  Syncs.
 * Errors: GSQ_ERR_INVALID_ARG, GSQ_ERR_UNSUPPORTED (shape limits above,
 * group != 128), GSQ_ERR_OOM, GSQ_ERR_NONFINITE, GSQ_ERR_TIMEOUT,
 * GSQ_ERR_CUDA, or a stage's own status.
 */
GSQ_API int gsq_dequant(int grid_mode, const void* packed, const float* scales_f32, int64_t N,
                        int64_t K, int group, void* W_bf16, void* stream);
GSQ_API int gsq_block_forward(const float* x, const void* const* W, int64_t n_seq,
                              int64_t seq_len, int64_t n_heads, int64_t n_kv_heads,
                              int64_t head_dim, int64_t ffn, double rope_theta,
                              float rms_eps, float* h_out, float* y_out, void* stream);
GSQ_API int gsq_block_quantize(const float* x_in, const void* const* W, int64_t n_seq,
                               int64_t seq_len, int64_t n_heads, int64_t n_kv_heads,
                               int64_t head_dim, int64_t ffn, double rope_theta,
                               float rms_eps, int group, int grid_mode,
                               const float* const* taus, const int64_t* n_steps, float lr,
                               float beta1, float beta2, uint64_t seed, float* x_out,
                               void* const* packed, uint16_t* const* scales_f16,
                               float* const* scales_f32, double* stats, void* stream);

/* ------------------------------------------------ GGUF K-Quant formats --
 * GSQ on llama.cpp's K-Quant formats: start from an existing K-Quant (e.g. a
 * released GGUF checkpoint), optimise with the GSQ step, and project the
 * result back into the same format (agihunt.info summary, optimisation and
 * results paragraphs: Qwen3-8B Q2_K and Q3_K_M, format unchanged).
 *
 * Formats (super-blocks of 256 consecutive weights of a row, 16 sub-blocks of
 * 16; K % 256 == 0):
 *   GSQ_KQ_Q2_K  w = d sc_j q - dmin m_j, q 0..3, sc_j, m_j 0..15, d, dmin
 *                fp16; 84 bytes per super-block
 *   GSQ_KQ_Q3_K  w = d sc_j q, q -4..3, sc_j -32..31, d fp16; 110 bytes
 * in the GGUF block encodings of Q2_K / Q3_K (blocks in row-major order of
 * the super-blocks).
 * State: per coordinate logits over q (Q2_K: 4; Q3_K: 5 local shifts
 * -2..+2 around the start code, clamped to [-4, 3]), +2 on the start code;
 * per sub-block continuous a_j (and b_j for Q2_K), starting at d sc_j and
 * dmin m_j.  A step: soft weight w = bf16(a_j sum_k y_k c_k - b_j) with
 * Philox Gumbel noise (the 2-bit grid's words for Q2_K, the 3-bit local
 * grid's for Q3_K), the layer loss ||X w^T - X W^T||^2 and dW as gsq_step,
 * dl_k = (a_j dw / tau) y_k sum_m y_m (c_k - c_m), da_j = sum dw v,
 * db_j = -sum dw, Lion on all of them.  Export (the projection back): hard
 * codes by argmax (first maximum); d = fp16(max_j a_j / 15), sc_j =
 * rint(a_j / d) in 0..15 (a_j, b_j clamped at 0), dmin and m_j likewise
 * (Q2_K); d = fp16(max_j |a_j| / 31), sc_j = rint(a_j / d) in -32..31 (Q3_K).
 *
 * gsq_kq_block_bytes: bytes of the N x K weight in the format.
 * gsq_kq_init: W (N x K), X (T x K) fp32/bf16, host or device; start_blocks
 *   (nullable, host or device) the starting K-Quant; NULL starts from the
 *   min-max K-Quant of W: per sub-block a = (max w - min(0, min w)) / 3 and
 *   b = -min(0, min w) (Q2_K) or a = -w_e / 4 with w_e the largest-magnitude
 *   weight (Q3_K), projected as above, each weight's code its nearest level
 *   (first on ties).  Syncs.
 * gsq_kq_step / gsq_kq_run / gsq_kq_last_loss: as gsq_step / gsq_run /
 *   gsq_last_loss.  gsq_kq_run gives the same result as a loop of
 *   gsq_kq_step bit for bit; inside it each step's backward also forms the
 *   next step's soft weight (at the next temperature), so a step is three
 *   launches instead of four.
 * gsq_kq_export: the projected blocks (host or device).  Syncs.
 * gsq_kq_start_blocks: the starting blocks.  Syncs.
 * gsq_kq_recon_error: abs = ||bf16(X) Wq^T - Y_ref||^2 and rel = abs /
 *   ||Y_ref||^2 of the exported (which = 0) or starting (1) blocks.  Syncs.
 * gsq_kq_dequant: bf16 weight (N x K) of blocks, w = bf16((d sc_j) q -
 *   dmin m_j) with each product and the difference rounded in fp32.  Syncs.
 * gsq_kq_debug_get / _set (GSQ_KQ_DBG_*), gsq_kq_debug_soft_weight (fills
 *   GSQ_KQ_DBG_WSOFT32), gsq_kq_debug_backward (backward + Lion from the
 *   current dW, filling DL, DA, DB; the step's probabilities are drawn
 *   again inside, as in a step; What is left as it was),
 *   gsq_kq_debug_noise: test entry points as their single-layer
 *   counterparts.
 * Errors: GSQ_ERR_INVALID_ARG (sizes, K % 256, format, null pointers),
 * GSQ_ERR_UNSUPPORTED (no sm_100 device), GSQ_ERR_OOM, GSQ_ERR_NONFINITE,
 * GSQ_ERR_STATE, GSQ_ERR_CUDA.
 */
enum { GSQ_KQ_Q2_K = 0, GSQ_KQ_Q3_K = 1 };
enum {
  GSQ_KQ_DBG_LOGITS = 0, /* L x N x K fp32 */
  GSQ_KQ_DBG_MOM = 1,    /* L x N x K fp32 */
  GSQ_KQ_DBG_A = 2,      /* N x K/16 fp32 sub-block scale a_j */
  GSQ_KQ_DBG_MA = 3,
  GSQ_KQ_DBG_B = 4,      /* N x K/16 fp32 sub-block offset b_j (Q2_K) */
  GSQ_KQ_DBG_MB = 5,
  GSQ_KQ_DBG_Q0 = 6,     /* N x K int8 start codes */
  GSQ_KQ_DBG_WHAT = 7,   /* N x K bf16 soft weight */
  GSQ_KQ_DBG_DW = 8,     /* N x K fp32 weight gradient */
  GSQ_KQ_DBG_DL = 9,     /* L x N x K fp32 logit gradient */
  GSQ_KQ_DBG_DA = 10,    /* N x K/16 fp32 */
  GSQ_KQ_DBG_DB = 11,    /* N x K/16 fp32 */
  GSQ_KQ_DBG_WSOFT32 = 12 /* N x K fp32 soft weight before rounding */
};
typedef struct gsq_kq gsq_kq;
GSQ_API int gsq_kq_block_bytes(int format, int64_t N, int64_t K, size_t* bytes);
GSQ_API int gsq_kq_init(gsq_kq** out, const void* W, int w_dtype, const void* X, int x_dtype,
                        int64_t N, int64_t K, int64_t T, int format, const void* start_blocks,
                        uint64_t seed, void* stream);
GSQ_API int gsq_kq_step(gsq_kq* ctx, float tau, float lr, float beta1, float beta2);
GSQ_API int gsq_kq_run(gsq_kq* ctx, const float* taus, int64_t n, float lr, float beta1,
                       float beta2);
GSQ_API int gsq_kq_last_loss(gsq_kq* ctx, double* loss);
GSQ_API int gsq_kq_export(gsq_kq* ctx, void* blocks);
GSQ_API int gsq_kq_start_blocks(gsq_kq* ctx, void* blocks);
GSQ_API int gsq_kq_recon_error(gsq_kq* ctx, int which, double* abs_err, double* rel_err);
GSQ_API int gsq_kq_dequant(int format, const void* blocks, int64_t N, int64_t K, void* W_bf16,
                           void* stream);
GSQ_API int gsq_kq_debug_get(gsq_kq* ctx, int which, void* host, size_t bytes);
GSQ_API int gsq_kq_debug_set(gsq_kq* ctx, int which, const void* host, size_t bytes);
GSQ_API int gsq_kq_debug_soft_weight(gsq_kq* ctx, float tau);
GSQ_API int gsq_kq_debug_backward(gsq_kq* ctx, float tau, float lr, float beta1, float beta2);
GSQ_API int gsq_kq_debug_noise(gsq_kq* ctx, int on);
GSQ_API int gsq_kq_get_step(gsq_kq* ctx, uint64_t* t);
GSQ_API int gsq_kq_destroy(gsq_kq* ctx);

/*
 * gsq_uniforms_noalloc -- the L Philox uniforms of coords
 * [coord0, coord0 + count) at step t for grid_mode and seed (the values
 * gsq_debug_uniforms returns for a context with that mode and seed),
 * coordinate-major, into `out` (host or device, count * L floats), without
 * allocating any device memory.  The pages have no counterpart: this is a
 * convenience for callers that cannot call cudaMalloc, for example a process
 * whose device memory is fully reserved by another allocator, or code inside
 * a framework that forbids device allocation on its execution path.
 * Device staging lives in a fixed array inside the library of
 * GSQ_NOALLOC_MAX_COORDS x 5 floats (1.25 MiB), which every GPU that loads
 * the library holds until exit; count above GSQ_NOALLOC_MAX_COORDS returns
 * GSQ_ERR_INVALID_ARG.  The first call on a device looks up that array's
 * device address (once per device, and again if the device's context changed
 * since, e.g. after cudaDeviceReset); make that first call before any stream
 * capture.  All calls share the array: calls whose work overlaps on the GPU
 * (for example on two streams) race and may return each other's values.
 * Enqueued on `stream` (NULL = legacy default stream); syncs.
 */
#define GSQ_NOALLOC_MAX_COORDS 65536
GSQ_API int gsq_uniforms_noalloc(int grid_mode, uint64_t seed, uint32_t t,
                                 uint64_t coord0, int64_t count, float* out,
                                 void* stream);

/*
 * gsq_gemm_bf16_abt -- the library's tcgen05 GEMM on its own:
 * C (M x N fp32, row-major, ldc = N) = A (M x Kc bf16, row-major) .
 * B (N x Kc bf16, row-major)^T with fp32 accumulation; device pointers,
 * 16-byte aligned, Kc % 8 == 0, N % 4 == 0.  Enqueued on `stream`; syncs.
 */
GSQ_API int gsq_gemm_bf16_abt(const void* A, const void* B, float* Cout, int64_t M,
                      int64_t N, int64_t Kc, void* stream);
/*
 * gsq_gemm_bf16_abt_sub -- the same GEMM with the subtracting epilogue that
 * GPTQ's tensor-core updates use: C (M x N fp32, row-major, ldc = N) -=
 * A . B^T, in place (each output tile is read, reduced by the fp32 product
 * and written back by the tile's own CTA).  Same argument rules and errors
 * as gsq_gemm_bf16_abt; C is read and written.  Enqueued on `stream`; syncs.
 */
GSQ_API int gsq_gemm_bf16_abt_sub(const void* A, const void* B, float* C, int64_t M,
                                  int64_t N, int64_t Kc, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* GSQ_H */
