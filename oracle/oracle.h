/*
 * oracle.h -- plain, slow, fp64 CPU model of the ReplaySSM SSM-layer decode
 * step (Mamba-2, Gated DeltaNet, Kimi Delta Attention), used to check the
 * CUDA path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this code: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no source with the CUDA library.
 *
 * Sources (cited by short tag in oracle.c):
 *   [sitech]    sitech.ge blog, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM להאצת
 *               פענוח מודלים היברידיים" (NVIDIA and Dao AI Lab present
 *               ReplaySSM), sections "How ReplaySSM works", "Reducing state
 *               traffic and simplifying rollback", "Bounding quantisation error".
 *   [hamidun]   news.hamidun.com, "NVIDIA تقدّم ReplaySSM: كيف تُسرّع فك ترميز
 *               النماذج الهجينة Mamba وGDN", sections "Why hybrid models became
 *               the norm" (layer types) and "Where the state problem appears".
 *   [felizola]  thiagofelizola.com, "NVIDIA e Princeton detalham ReplaySSM
 *               para acelerar modelos híbridos", body paragraphs 2-3.
 *   [Dao & Gu 2024]  "Transformers are SSMs" -- the Mamba-2 (SSD) recurrence.
 *   [Yang et al. 2025] "Gated Delta Networks" -- the gated delta rule.
 *   [Kimi Linear 2025] Moonshot AI, "Kimi Linear" -- Kimi Delta Attention,
 *                    the gated delta rule with a per-channel decay.
 *   [OCP MX v1.0]    OCP Microscaling Formats spec -- FP8 E4M3 / FP4 E2M1.
 *
 * Layout conventions (all arrays dense, row-major, the last index innermost):
 *   Mamba-2: state [B][H][P][N]; x [T][B][H][P]; dt [T][B][H];
 *            Bm, Cm [T][B][G][N]; A, D [H]; y [T][B][H][P].
 *            Head h belongs to group g = h / (H/G).
 *   GDN:     state [B][H][DK][DV]; q, k [T][B][H][DK]; v [T][B][H][DV];
 *            alpha, beta [T][B][H]; o [T][B][H][DV].
 *   Record buffers (per (sequence, head)): rec_* [B][H][cap][...], len [B][H].
 *
 * Every function returns 0 on success and -1 on a bad argument.
 */
#ifndef REPLAYSSM_ORACLE_H
#define REPLAYSSM_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Checkpoint / read-copy formats. */
#define ORACLE_FMT_NONE 0   /* fp64 checkpoint, no read copy            */
#define ORACLE_FMT_FP8 1    /* FP8 E4M3, round-nearest-even, saturating */
#define ORACLE_FMT_NVFP4 2  /* FP4 E2M1 codes + E4M3 scale per 16 + fp32 tile scale */

/* ---------------------------------------------------------------- Mamba-2 */

int oracle_m2_conventional(int T, int B, int H, int P, int N, int G,
                           double *S, const double *x, const double *dt,
                           const double *Bm, const double *Cm,
                           const double *A, const double *D, double *y,
                           long long *reads, long long *writes);

int oracle_m2_replay(int T, int B, int H, int P, int N, int G, int L, int cap,
                     int read_fmt, int ckpt_fmt,
                     double *h0, double *rec_x, double *rec_dt, double *rec_B,
                     double *rec_C, int *len,
                     const double *x, const double *dt, const double *Bm,
                     const double *Cm, const double *A, const double *D,
                     double *y, int *len_trace, int *flush_trace,
                     long long *reads, long long *writes);

int oracle_m2_flush(int B, int H, int P, int N, int L, int cap, int force,
                    int ckpt_fmt, double *h0, const double *rec_x,
                    const double *rec_dt, const double *rec_B, int *len,
                    const double *A);

int oracle_m2_materialize(int B, int H, int P, int N, int cap,
                          const double *h0, const double *rec_x,
                          const double *rec_dt, const double *rec_B,
                          const int *len, const double *A, double *S_out);

int oracle_m2_verify_replay(int R, int B, int H, int P, int N, int G, int L,
                            int cap, int Dn, double *h0, double *rec_x,
                            double *rec_dt, double *rec_B, double *rec_C,
                            int *len, const double *x, const double *dt,
                            const double *Bm, const double *Cm,
                            const double *A, const double *D,
                            const int *acc, double *y, int *len_trace);

int oracle_m2_verify_snapshot(int R, int B, int H, int P, int N, int G, int Dn,
                              double *S, const double *x, const double *dt,
                              const double *Bm, const double *Cm,
                              const double *A, const double *D,
                              const int *acc, double *y,
                              long long *state_copies);

/* ---------------------------------------------------------- Gated DeltaNet */

int oracle_gdn_conventional(int T, int B, int H, int DK, int DV, double scale,
                            double *S, const double *q, const double *k,
                            const double *v, const double *alpha,
                            const double *beta, double *o,
                            long long *reads, long long *writes);

int oracle_gdn_replay(int T, int B, int H, int DK, int DV, int L, int cap,
                      double scale, double *h0, double *rec_q, double *rec_k,
                      double *rec_v, double *rec_alpha, double *rec_beta,
                      int *len, const double *q, const double *k,
                      const double *v, const double *alpha, const double *beta,
                      double *o, int *len_trace, int *flush_trace,
                      long long *reads, long long *writes);

/* Gated DeltaNet speculative verify: replay form (drafts appended, outputs
 * from h0 + buffer, accepted prefix committed) and the snapshot-and-restore
 * conventional form.  Layouts as for the Mamba-2 rounds, with q, k [DK],
 * v, o [DV], alpha, beta scalars per (round, sequence, draft, head). */
int oracle_gdn_verify_replay(int R, int B, int H, int DK, int DV, int L, int cap,
                             int Dn, double scale, double *h0, double *rec_q,
                             double *rec_k, double *rec_v, double *rec_alpha,
                             double *rec_beta, int *len, const double *q,
                             const double *k, const double *v,
                             const double *alpha, const double *beta,
                             const int *acc, double *o, int *len_trace);

int oracle_gdn_verify_snapshot(int R, int B, int H, int DK, int DV, int Dn, double scale,
                               double *S, const double *q, const double *k,
                               const double *v, const double *alpha,
                               const double *beta, const int *acc, double *o,
                               long long *state_copies);

int oracle_gdn_flush(int B, int H, int DK, int DV, int L, int cap, int force,
                     double *h0, const double *rec_k, const double *rec_v,
                     const double *rec_alpha, const double *rec_beta, int *len);

int oracle_gdn_materialize(int B, int H, int DK, int DV, int cap,
                           const double *h0, const double *rec_k,
                           const double *rec_v, const double *rec_alpha,
                           const double *rec_beta, const int *len,
                           double *S_out);

/* ----------------------------------------------------- Kimi Delta Attention
 * Gated delta rule with a per-key-channel decay: alpha [T][B][H][DK] (and
 * rec_alpha [B][H][cap][DK]); other layouts as for Gated DeltaNet. */

int oracle_kda_conventional(int T, int B, int H, int DK, int DV, double scale,
                            double *S, const double *q, const double *k,
                            const double *v, const double *alpha,
                            const double *beta, double *o,
                            long long *reads, long long *writes);

int oracle_kda_replay(int T, int B, int H, int DK, int DV, int L, int cap,
                      double scale, double *h0, double *rec_q, double *rec_k,
                      double *rec_v, double *rec_alpha, double *rec_beta,
                      int *len, const double *q, const double *k,
                      const double *v, const double *alpha, const double *beta,
                      double *o, int *len_trace, int *flush_trace,
                      long long *reads, long long *writes);

int oracle_kda_flush(int B, int H, int DK, int DV, int L, int cap, int force,
                     double *h0, const double *rec_k, const double *rec_v,
                     const double *rec_alpha, const double *rec_beta, int *len);

int oracle_kda_materialize(int B, int H, int DK, int DV, int cap,
                           const double *h0, const double *rec_k,
                           const double *rec_v, const double *rec_alpha,
                           const double *rec_beta, const int *len,
                           double *S_out);

/* ------------------------------------------------------------------ codecs */

uint8_t oracle_e4m3_encode(float v);
double oracle_e4m3_decode(uint8_t c);
uint8_t oracle_e2m1_encode(float v);
double oracle_e2m1_decode(uint8_t c);

/* FP8 read copy of n fp32 values (no scale). */
int oracle_fp8_quant(long long n, const float *x, uint8_t *codes);
int oracle_fp8_dequant(long long n, const uint8_t *codes, float *out);

/* NVFP4 read copy of ntile tiles of rows x cols fp32 values each; blocks of
 * 16 run along cols.  codes: [ntile][rows][cols/2] (even element in the low
 * nibble); scales: [ntile][rows][cols/16] E4M3; gscale: [ntile] fp32. */
int oracle_nvfp4_quant(int ntile, int rows, int cols, const float *x,
                       uint8_t *codes, uint8_t *scales, float *gscale);
int oracle_nvfp4_dequant(int ntile, int rows, int cols, const uint8_t *codes,
                         const uint8_t *scales, const float *gscale,
                         float *out);

/* h <- deq(Q(fp32(h))) in place for ntile tiles of rows x cols (the
 * "quantised checkpoint" baseline).  fmt is ORACLE_FMT_FP8 or _NVFP4. */
int oracle_quantize_ckpt(int fmt, int ntile, int rows, int cols, double *h);

#ifdef __cplusplus
}
#endif
#endif /* REPLAYSSM_ORACLE_H */
