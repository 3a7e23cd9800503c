/*
 * gsq_oracle.h -- plain CPU restatement of the GSQ Gumbel-Softmax
 * layer-reconstruction step (test infrastructure, not product code).
 *
 * Source: "GSQ: Highly-Accurate Low-Precision Scalar Quantization for LLMs via
 * Gumbel-Softmax Sampling" (Dadgarnia et al., arXiv 2604.18556), as summarised
 * on agihunt.info/papers/2604.18556 (method paragraph: per-coordinate logits
 * over a symmetric group-wise grid, Gumbel-Softmax soft weighted sum, ternary
 * mask x sign split, 2-bit 4-logit grid with a shared scale, local shift
 * {-2..+2} for 3 bits and up; optimisation paragraph: Lion) and on
 * atlas.scime.ai (Approach section). The counter-based generator is
 * Philox4x32-10 from Salmon, Moraes, Dror and Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3" (SC'11).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  It shares no code with the CUDA library.
 *
 * Conventions (all arrays row-major, caller-allocated):
 *   W, dW, w    : N x K   (N = out features, K = in features)
 *   X           : T x K   (calibration tokens)
 *   Yref, dY    : T x N
 *   logits, mom : L planes of N x K (plane p at offset p*N*K), fp32
 *   s, ms       : N x G,  G = K / group
 *   i0 / code   : N x K int8 / uint8 grid level index
 * `row0` is the global index of row 0 of the given arrays, so that a slice of
 * rows draws the same Philox noise as the full layer.
 */
#ifndef GSQ_ORACLE_H
#define GSQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { GSQO_GRID_2BIT = 0, GSQO_GRID_TERNARY = 1, GSQO_GRID_3BIT_LOCAL = 2 };

/* number of logits per coordinate: 4, 2+2, 5 */
int gsqo_num_logits(int mode);
/* number of grid levels: 4, 3, 8 */
int gsqo_num_levels(int mode);
/* unit grid value of level j (2-bit: j-1.5; ternary: j-1; 3-bit: j-3.5) */
double gsqo_level_value(int mode, int j);

/* Philox4x32-10 block function (SC'11): out = bijection_key(ctr). */
void gsqo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2],
                        uint32_t out[4]);
/* 32-bit word -> open-interval uniform ((x >> 9) + 0.5) * 2^-23, exact in fp32 */
float gsqo_u01(uint32_t x);
/* L uniforms per coordinate for coords [coord0, coord0+count) at step t,
 * coordinate-major: out[i*L + j] */
void gsqo_uniforms(int mode, uint64_t seed, uint32_t t, uint64_t coord0,
                   int64_t count, float* out);

/* round to nearest-even bfloat16 / binary16, returned as a double */
double gsqo_bf16_round(double x);
double gsqo_f16_round(double x);
/* binary16 bit pattern of gsqo_f16_round(x) */
uint16_t gsqo_f16_bits(double x);

/* A0: scales, initial level index, logits = +2 on the initial slot, zero
 * Lion state.  init_idx (nullable) overrides the round-to-nearest level. */
int gsqo_init(int mode, int64_t N, int64_t K, int group, const float* W,
              const int8_t* init_idx, float* s, int8_t* i0, float* logits,
              float* mom, float* ms);

/* Y_ref = bf16(X) . W^T in fp64 (T x N); W at its given precision */
void gsqo_reference_output(int64_t N, int64_t K, int64_t T, const float* W,
                           const float* X, double* Yref);

/* A1 + A2: probabilities y (L planes, nullable), unit value v (nullable),
 * soft weight w = s*v before rounding (nullable), bf16-rounded w (nullable). */
void gsqo_soft_weight(int mode, int64_t row0, int64_t N, int64_t K, int group,
                      const float* logits, const float* s, const int8_t* i0,
                      uint64_t seed, uint32_t t, float tau, int noise_on,
                      double* y, double* v, double* w, float* w_bf16);

/* A3: E = bf16(X) . Wb^T - Yref (fp64); returns sum E^2; dY = bf16(2E) */
double gsqo_forward(int64_t N, int64_t K, int64_t T, const float* X,
                    const float* Wb, const double* Yref, float* dY);
/* A4: dW = dY^T . bf16(X) in fp64, stored fp32 */
void gsqo_weight_grad(int64_t N, int64_t K, int64_t T, const float* dY,
                      const float* X, float* dW);
/* A5 gradients: dl (L planes, fp32) and ds (N x G, fp32) from dW */
void gsqo_backward(int mode, int64_t N, int64_t K, int group, const double* y,
                   const double* v, const float* s, const int8_t* i0,
                   const float* dW, float tau, float* dl, float* ds);
/* Lion (Chen et al. 2023) in place on n fp32 parameters */
void gsqo_lion(int64_t n, float* theta, float* mom, const float* grad,
               float lr, float beta1, float beta2);

/* One full step t (A1..A5).  Updates logits, mom, s, ms in place and returns
 * the loss through *loss.  Optional dumps (nullable): w (pre-round soft
 * weight), dY, dW, dl, ds. */
int gsqo_step(int mode, int64_t row0, int64_t N, int64_t K, int64_t T,
              int group, float* logits, float* mom, float* s, float* ms,
              const int8_t* i0, const float* X, const double* Yref,
              uint64_t seed, uint32_t t, float tau, float lr, float beta1,
              float beta2, int noise_on, double* loss, double* w_dump,
              float* dY_dump, float* dW_dump, float* dl_dump, float* ds_dump);

/* A5 alone from a given dW (same noise / probabilities as the step) */
int gsqo_backward_lion(int mode, int64_t row0, int64_t N, int64_t K, int group,
                       float* logits, float* mom, float* s, float* ms,
                       const int8_t* i0, const float* dW, uint64_t seed,
                       uint32_t t, float tau, float lr, float beta1,
                       float beta2, int noise_on, float* dl_dump,
                       float* ds_dump);

/* bf16 state (the reduced-memory mode): stochastic rounding with a 9-bit
 * threshold, and the rounding of logits (stochastic, thresholds from the
 * low 9 bits of the step-(t+1) Philox words) and momenta (nearest) after
 * the fp32 Lion update of step t */
float gsqo_bf16_sr(float x, uint32_t r9);
void gsqo_state16_store(int mode, int64_t row0, int64_t N, int64_t K,
                        uint64_t seed, uint32_t t_next, float* logits,
                        float* mom);

/* A6: hard level per coordinate (argmax of logits, first max, no noise) */
void gsqo_harden(int mode, int64_t N, int64_t K, const float* logits,
                 const int8_t* i0, uint8_t* level);
/* the code written to the bitstream is the level index (ternary: v+1) */
/* packed words per row: 2-bit / ternary K/16, 3-bit 3K/32 */
int64_t gsqo_packed_words_per_row(int mode, int64_t K);
void gsqo_pack(int mode, int64_t N, int64_t K, const uint8_t* level,
               uint32_t* packed);
void gsqo_unpack(int mode, int64_t N, int64_t K, const uint32_t* packed,
                 uint8_t* level);

/* A7: hard (mode 0) or noiseless soft at tau (mode 1) reconstruction error,
 * abs = ||bf16(X).Wq^T - Yref||_F^2, rel = abs / ||Yref||_F^2 */
void gsqo_recon_error(int gmode, int emode, int64_t N, int64_t K, int64_t T,
                      int group, const float* logits, const float* s,
                      const int8_t* i0, const float* X, const double* Yref,
                      float tau, double* abs_err, double* rel_err);

/* Scale-only step (the assignments frozen at the hard choice of the logits,
 * only the group scales trained; agihunt.info summary, optimisation
 * paragraph): w = bf16(s c_level); loss, dY, dW as in gsqo_step; ds_g =
 * sum dW_i c_level(i); Lion on s, ms.  The _backward_lion form takes dW. */
void gsqo_scale_backward_lion(int mode, int64_t N, int64_t K, int group,
                              const float* logits, const int8_t* i0, float* s,
                              float* ms, const float* dW, float lr, float beta1,
                              float beta2, float* ds_dump);
int gsqo_scale_step(int mode, int64_t N, int64_t K, int64_t T, int group,
                    const float* logits, const int8_t* i0, float* s, float* ms,
                    const float* X, const double* Yref, float lr, float beta1,
                    float beta2, double* loss, float* w_dump, float* dW_dump,
                    float* ds_dump);

/* SwiGLU MLP joint stage (the block's MLP trained on the block output).
 * Xn (T x H): the normalised MLP input; R (T x H): the output the MLP must
 * produce; Wg, Wu (F x H) and Wd (H x F): the three soft weights.
 *   a = Xn Wg^T, b = Xn Wu^T, h = silu(a) b, pred = h Wd^T,
 *   loss = sum (pred - R)^2, and the weight gradients dWg, dWu (F x H),
 *   dWd (H x F) (nullable).  With round = 1 the GEMM operands that the
 *   library keeps in bf16 (Xn, h, dpred = 2E, da, db) are rounded to bf16
 *   as there; with round = 0 everything is exact fp64 (for the pins). */
double gsqo_mlp_forward_backward(int64_t T, int64_t H, int64_t F,
                                 const float* Xn, const double* R,
                                 const float* Wg, const float* Wu,
                                 const float* Wd, int round, float* dWg,
                                 float* dWu, float* dWd);

/* Attention V/O joint stage (the block's value and output projections
 * trained together with the attention probabilities fixed).
 *
 * gsqo_attn_probs: P of every sequence s and head h from the attention input
 *   Xa (T x H, T = nseq S, H = nh d) and fixed query / key weights Wq (H x H),
 *   Wk (nkv d x H): Q = Xa Wq^T, K = Xa Wk^T, rotary embedding (rotate-half
 *   pairs (i, i + d/2), angle p theta^(-2i/d) at position p of the sequence),
 *   scores Q_h K_g^T / sqrt(d) with g = h / (nh / nkv), causal mask, softmax.
 *   P layout: [s][h][q][key], fp32.  round = 1 rounds Q, K (after rotation)
 *   and P to bf16 as the library's GEMM operands.
 * gsqo_attn_vo_forward_backward: with V = Xa Wv^T (T x nkv d),
 *   o_(s,h) = P_(s,h) V_(s,g), pred = o Wo^T, loss = sum (pred - R)^2, returns
 *   the loss and dWv (nkv d x H), dWo (H x H); round = 1 rounds V, o, 2E,
 *   do and dV to bf16 as the library's GEMM operands. */
void gsqo_attn_probs(int64_t nseq, int64_t S, int64_t nh, int64_t nkv,
                     int64_t d, double theta, const float* Xa, const float* Wq,
                     const float* Wk, int round, float* P);
/* one row P[s][h][q][:] (S entries) computed on its own, as in
 * gsqo_attn_probs, for sampled checks of large layers */
void gsqo_attn_prob_row(int64_t nseq, int64_t S, int64_t nh, int64_t nkv,
                        int64_t d, double theta, const float* Xa,
                        const float* Wq, const float* Wk, int round, int64_t s,
                        int64_t h, int64_t q, float* row);
double gsqo_attn_vo_forward_backward(int64_t nseq, int64_t S, int64_t nh,
                                     int64_t nkv, int64_t d, const float* Xa,
                                     const float* P, const double* R,
                                     const float* Wv, const float* Wo,
                                     int round, float* dWv, float* dWo);

/* plain fp64 C = A . B^T for A (M x Kc), B (N x Kc), both row-major */
void gsqo_gemm_abt(int64_t M, int64_t N, int64_t Kc, const float* A,
                   const float* B, double* C);

#ifdef __cplusplus
}
#endif
#endif
