/*
 * oracle.h -- declarations of the CPU oracle for the DFlash 2 draft -> select
 * -> verify step.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, fp64 restatement of what
 * the method computes, written to check the CUDA library against.  Only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load
 * it.  It shares no code, header, table or helper with the CUDA library
 * (block_draft_verification_b200/csrc), and it includes nothing from there.
 *
 * Conventions shared by every function here:
 *   - Inputs are read in their storage type (dtype 0 = fp32, 1 = bf16 stored
 *     as uint16 bit patterns) and widened exactly to double.
 *   - All arithmetic is double precision, in the plainest loop order
 *     (ascending vocabulary index, ascending position).
 *   - Floating outputs are returned as double, unrounded.
 *   - Return value: 0 on success, -1 on an argument the oracle cannot handle.
 *
 * Source pages (cited by title and section):
 *   [tamsi] "DFlash 2 — 3× plus de tokens sur Qwen3.8-27B, même sortie"
 *           (tamsi.dev/blog/dflash2), sections "L’idée, sans le papier" and
 *           "Les chiffres qui comptent sur Qwen3.8-27B".
 *   [myaiexp] "DFlash 2" (myaiexp.com), section "主な機能" (features).
 *   [latenode] "DFlash 2: un drafter de 3.43× que cae a 1.45× bajo carga",
 *           sections "Un drafter que adivina el bloque entero de una vez",
 *           "El desacuerdo empieza en las propias tablas del proveedor",
 *           "Preguntas frecuentes".
 *   [psi]   "Qwen 3.8 27B + DFlash2: 140 Token/Sec?", section "Résumé".
 *   [philox] Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as
 *           1, 2, 3", SC'11, section 5 (the Philox family).
 */
#ifndef DFLASH2_ORACLE_H
#define DFLASH2_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };
enum { ORC_Q_SOFTMAX = 0, ORC_Q_ONEHOT = 1 };
enum { ORC_K = 16 };

/* ---- Philox4x32-10 and the uniforms drawn from it ([philox] section 5) ---- */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
/* u = (word0 >> 8) * 2^-24 for counter (step, seq_id, pos, purpose) and key
 * (seed low 32 bits, seed high 32 bits). */
double orc_uniform(uint64_t seed, uint32_t step, uint32_t seq_id, uint32_t pos, uint32_t purpose);
void orc_uniforms(uint64_t seed, uint32_t step, const uint32_t* seq_id, int64_t n,
                  uint32_t pos, uint32_t purpose, double* out);

/* ---- softmax + top-16 per drafted position ([tamsi] "L’idée, sans le papier";
 *      [myaiexp] features: keep the 16 best candidates per position) ---- */
int orc_topk_softmax(const void* logits, int dtype, int64_t rows, int64_t V, int64_t row_stride,
                     double inv_temperature, int32_t* idx, double* prob, double* logp,
                     double* logz);

/* ---- bilinear adjacent-pair score and exact best path ([tamsi] "L’idée, sans
 *      le papier"; [myaiexp] features: adjacent pairs scored; [psi] "Résumé":
 *      bilinear attention over candidates) ---- */
double orc_pair(const void* emb, int emb_dtype, int d, const float* W, int32_t a, int32_t b);
int orc_pair_select(const int32_t* idx, const float* logp, const int32_t* anchor,
                    const void* emb, int emb_dtype, int64_t V, int d, const float* W,
                    int B, int G, int32_t* path_tok, int32_t* path_rank, double* path_score);
int orc_path_rescore(const int32_t* idx, const float* logp, const int32_t* anchor,
                     const void* emb, int emb_dtype, int64_t V, int d, const float* W,
                     int B, int G, const int32_t* path_rank, double* score);

/* ---- greedy lossless verify ([tamsi] "Les chiffres qui comptent": greedy
 *      output equals the target exactly) ---- */
int orc_verify_greedy(const void* target, int dtype, int B, int G, int64_t V,
                      const int32_t* draft_tok, int32_t* n_accept, int32_t* out_tok);

/* ---- sampling lossless verify by rejection sampling ([tamsi] same section;
 *      [latenode] "Un drafter que adivina...": sampling preserves the target
 *      distribution) ---- */
int orc_verify_sample_u(const void* target, const void* draft, int dtype, int B, int G,
                        int64_t V, const int32_t* draft_tok, double inv_temperature,
                        int q_mode, const double* u_acc, const double* u_res,
                        int32_t* n_accept, int32_t* out_tok, double* ratio,
                        double* margin_acc, double* margin_res);
int orc_verify_sample(const void* target, const void* draft, int dtype, int B, int G,
                      int64_t V, const int32_t* draft_tok, double inv_temperature,
                      uint64_t seed, uint32_t step, const uint32_t* seq_id, int q_mode,
                      int32_t* n_accept, int32_t* out_tok, double* ratio, double* u,
                      double* margin_acc, double* margin_res);

/* ---- the same verification of distributions truncated by top-k and top-p
 *      ([latenode] "Preguntas frecuentes": temperature 1.0, top-p 0.95,
 *      top-k 20 for the Qwen targets); top_k <= 0 and top_p >= 1 switch
 *      either off.  margin_trunc[b] = the smallest top-p cut margin of the
 *      rows the sequence's decisions and draw used ---- */
int orc_verify_sample_trunc_u(const void* target, const void* draft, int dtype, int B, int G,
                              int64_t V, const int32_t* draft_tok, double inv_temperature,
                              int top_k, double top_p, int q_mode, const double* u_acc,
                              const double* u_res, int32_t* n_accept, int32_t* out_tok,
                              double* ratio, double* margin_acc, double* margin_res,
                              double* margin_trunc);
int orc_verify_sample_trunc(const void* target, const void* draft, int dtype, int B, int G,
                            int64_t V, const int32_t* draft_tok, double inv_temperature,
                            int top_k, double top_p, uint64_t seed, uint32_t step,
                            const uint32_t* seq_id, int q_mode, int32_t* n_accept,
                            int32_t* out_tok, double* ratio, double* u, double* margin_acc,
                            double* margin_res, double* margin_trunc);

/* ---- two-tap dynamic depthwise conv with its tap projection and residual
 *      ([tamsi] "L’idée, sans le papier": two-tap conv before/after each
 *      attention and MLP; [myaiexp] features: 2-tap dynamic convolution) ---- */
int orc_dynconv2(const void* x, const void* x_prev, const void* w_tap, int dtype,
                 int B, int T, int H, double* out);

#ifdef __cplusplus
}
#endif

#endif
