/*
 * replayssm.h -- C ABI of the ReplaySSM SSM-layer decode library for B200
 * (sm_100a).  Plain pointers and sizes only; no C++ or framework types.
 *
 * The method (sources cited by page title and section):
 *   [sitech]   sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM להאצת פענוח
 *              מודלים היברידיים" (NVIDIA and Dao AI Lab present ReplaySSM),
 *              sections "How ReplaySSM works", "Reducing state traffic and
 *              simplifying rollback", "Bounding quantisation error".
 *   [felizola] thiagofelizola.com, "NVIDIA e Princeton detalham ReplaySSM para
 *              acelerar modelos híbridos", body paragraphs 2-3.
 *   [hamidun]  news.hamidun.com, "NVIDIA تقدّم ReplaySSM: كيف تُسرّع فك ترميز
 *              النماذج الهجينة Mamba وGDN", sections "Why hybrid models became
 *              the norm", "Where the state problem appears".
 * Every (sequence, head) state of an SSM layer is kept as a high-precision
 * checkpoint h0 plus a buffer of the most recent layer-input records.  A
 * non-flush decode step appends the current record and computes the output
 * from h0 and the buffer without writing the state; when the buffer holds
 * `window` records the step folds them into h0, writes h0 once and empties the
 * buffer [sitech §How ReplaySSM works].  Speculative drafts are appended and
 * evaluated output-only; committing advances the buffer over the accepted
 * prefix, with no snapshot or restore [sitech §Reducing state traffic...],
 * [felizola ¶3].  An optional low-precision read copy of h0 serves the output
 * reads while the fp32 checkpoint carries the recurrence [sitech §Bounding
 * quantisation error].  Layer types: Mamba-2 and Gated DeltaNet
 * [hamidun §Why hybrid models became the norm]; the recurrences are the
 * standard Mamba-2 (Dao & Gu 2024) and gated delta rule (Yang et al. 2025).
 *
 * Ownership and threading.  Every buffer is allocated and owned by the caller
 * (device memory unless a parameter says "host").  The library never
 * allocates or frees memory and never synchronises: each call validates its
 * arguments on the host, enqueues its kernels on `stream` (a cudaStream_t
 * handle; NULL = legacy default stream) and returns.  Calls that share a
 * state must be ordered on one stream.  All pointers to device buffers must be
 * 16-byte aligned.
 *
 * Errors.  Host-detectable problems (NULL pointers, shapes the kernels do not
 * support, misalignment, capacity) return an error code before anything is
 * enqueued.  Problems only the device can see (a buffer length out of range,
 * an acceptance count above the draft count, heads of one sequence out of
 * step) are written to the caller's device status word `state->status` with
 * first-error-wins semantics; the affected (sequence, group) item is skipped
 * and left unchanged, the kernel never traps.  Read the word after a
 * synchronisation; zero means no error.
 *
 * Layouts (row-major, last index innermost; B = batch, H = heads):
 *   Mamba-2: P = headdim (state rows), N = dstate (state columns), G groups,
 *            head h uses group h / (H/G).  Checkpoint h0 [B][H][P][N] fp32.
 *            Step inputs: x [B][H][P], dt [B][H] (post-softplus),
 *            Bm, Cm [B][G][N] -- all of dtype in_dtype; A, D [H] fp32.
 *            Output y [B][H][P] fp32.
 *   GDN:     DK = dstate, DV = headdim.  Checkpoint h0 [B][H][DK][DV] fp32.
 *            Step inputs q, k [B][H][DK], v [B][H][DV] of in_dtype (q, k
 *            already L2-normalised); alpha, beta [B][H] fp32.
 *            Output o [B][H][DV] fp32 = scale * S^T q.
 *   KDA:     Kimi Delta Attention [hamidun §Why hybrid models became the
 *            norm], the gated delta rule with one decay per key channel,
 *            S <- (I - beta k k^T) Diag(alpha) S + beta k v^T, o = scale S^T q:
 *            layouts as for GDN except alpha [B][H][DK] fp32.
 *   Buffer capacity per (sequence, head): cap = window + max(draft_max-1, 0).
 */
#ifndef REPLAYSSM_H
#define REPLAYSSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RSSM_OK = 0,
  RSSM_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, bad enum value   */
  RSSM_ERR_SHAPE = 2,       /* a dimension the kernels are not built for     */
  RSSM_ERR_DTYPE = 3,       /* unsupported input dtype                        */
  RSSM_ERR_ALIGNMENT = 4,   /* a device pointer not 16-byte aligned          */
  RSSM_ERR_CAPACITY = 5,    /* window/draft count beyond the buffer capacity */
  RSSM_ERR_CUDA = 6,        /* a CUDA launch failed                          */
  RSSM_ERR_TIMEOUT = 7,     /* a bounded device wait ran out (status word)   */
  RSSM_ERR_UNSUPPORTED = 8, /* valid request this build does not implement   */
  RSSM_ERR_STATE = 9        /* device: buffer state out of range (status)    */
} rssm_status;

typedef enum { RSSM_MAMBA2 = 0, RSSM_GDN = 1, RSSM_KDA = 2 } rssm_kind;
typedef enum { RSSM_F32 = 0, RSSM_BF16 = 1 } rssm_dtype;
typedef enum { RSSM_FMT_NONE = 0, RSSM_FMT_FP8 = 1, RSSM_FMT_NVFP4 = 2 } rssm_fmt;

/* Static description of one SSM layer's decode state. */
typedef struct {
  int32_t kind;      /* rssm_kind                                               */
  int32_t batch;     /* B, sequences (>= 0; 0: every call returns RSSM_OK at once) */
  int32_t nheads;    /* H                                                        */
  int32_t headdim;   /* Mamba-2 P (64 or 128); GDN DV (128)                      */
  int32_t dstate;    /* Mamba-2 N (64 or 128); GDN DK (128)                      */
  int32_t ngroups;   /* Mamba-2 G (H % G == 0, H/G <= 16); GDN: ignored          */
  int32_t window;    /* records per flush, 1..16 (the pages use 16)              */
  int32_t draft_max; /* most drafts per verify round, 0..4 (KDA: 0)             */
  int32_t in_dtype;  /* rssm_dtype of the step inputs                            */
  int32_t read_fmt;  /* rssm_fmt of the read copy (Mamba-2 only)                 */
  int32_t ckpt_fmt;  /* rssm_fmt the checkpoint is rounded to at each fold: the
                        "quantised checkpoint" comparison baseline (Mamba-2)   */
  float scale;       /* GDN output scale (Mamba-2: ignored)                      */
} rssm_desc;

/* Device buffers of a replay state (caller-allocated, sizes from
 * replayssm_state_bytes).  buf[] holds the records, one slot per token:
 *   Mamba-2: buf[0] x  [B][H][cap][P]  in_dtype
 *            buf[1] dt [B][H][cap]     fp32
 *            buf[2] Bm [B][G][cap][N]  in_dtype   (shared by a group's heads)
 *            buf[3] Cm [B][G][cap][N]  in_dtype
 *   GDN:     buf[0] q  [B][H][cap][DK] in_dtype
 *            buf[1] k  [B][H][cap][DK] in_dtype
 *            buf[2] v  [B][H][cap][DV] in_dtype
 *            buf[3] alpha [B][H][cap]  fp32
 *            buf[4] beta  [B][H][cap]  fp32
 *   KDA:     as GDN, with buf[3] alpha [B][H][cap][DK] fp32 (per channel)
 *   GDN/KDA: buf[5] u  [B][H][cap][DV] fp32: per record i, the delta-rule
 *                   correction u_i = beta_i (v_i - (state before i)^T k_i)
 *                   expressed from h0 and records 0..i (see replayssm_decode_step);
 *                   it depends only on h0 and those records, so it is computed
 *                   once, when record i is appended, and read by later steps
 * len [B][H] int32: records buffered per (sequence, head).  Slots >= len are
 * free (they may hold rejected drafts).  rc/rc_scale/rc_gscale are the read
 * copy (read_fmt != NONE): FP8 codes [B][H][P][N]; NVFP4 codes
 * [B][H][P][N/2] (even element in the low nibble), E4M3 block scales
 * [B][H][P][N/16], fp32 tile scales [B][H].  status: one int32. */
typedef struct {
  float *h0;
  void *buf[6];
  int32_t *len;
  uint8_t *rc;
  uint8_t *rc_scale;
  float *rc_gscale;
  int32_t *status;
} rssm_state;

/* Inputs of one decode step (or of a verify round's drafts).  in[] follows the
 * step-input layout above.  For replayssm_verify_commit every in[] tensor has a
 * draft axis after the batch axis: x [B][n][H][P], dt [B][n][H],
 * Bm/Cm [B][n][G][N].  batch_stride[i] is the element distance between
 * consecutive sequences of in[i] (0 = dense); y_batch_stride likewise for the
 * output (0 = dense). */
typedef struct {
  const void *in[5];
  const float *A; /* Mamba-2 per-head decay rate [H] (negative)  */
  const float *D; /* Mamba-2 per-head skip [H]                   */
  int64_t batch_stride[5];
  int64_t y_batch_stride;
} rssm_step_in;

/* Which buffer replayssm_state_bytes sizes. */
typedef enum {
  RSSM_BYTES_H0 = 0,
  RSSM_BYTES_BUF0 = 1, /* .. RSSM_BYTES_BUF0 + 5 for buf[0..5] */
  RSSM_BYTES_LEN = 7,
  RSSM_BYTES_RC = 8,
  RSSM_BYTES_RC_SCALE = 9,
  RSSM_BYTES_RC_GSCALE = 10,
  RSSM_BYTES_STATUS = 11,
  RSSM_BYTES_FULL_STATE = 12, /* conventional state, same layout as h0 */
  RSSM_BYTES_Y = 13           /* one step's output */
} rssm_bytes_which;

/* Host-only helpers (no CUDA calls). */
rssm_status replayssm_validate(const rssm_desc *desc);
int32_t replayssm_capacity(const rssm_desc *desc);
/* Bytes of one buffer; 0 for a buffer the layer kind does not use or for an
 * invalid desc. */
size_t replayssm_state_bytes(const rssm_desc *desc, int32_t which);
const char *replayssm_status_string(rssm_status s);
/* Text of the CUDA error behind the calling thread's most recent
 * RSSM_ERR_CUDA return ("no error" if there was none).  Host only. */
const char *replayssm_last_cuda_error(void);

/* Test hook for the failure path of the kernels' bounded waits; host only,
 * not for production use.  Every wait in the persistent kernels gives up
 * after a time limit and the kernel then writes RSSM_ERR_TIMEOUT to the
 * status word, stops its remaining work items and returns (every bulk copy it
 * issued lands first; nothing traps).  consumer_wait_ns > 0 sets the limit of
 * the compute warps' waits (default 2 s; <= 0 restores the default);
 * withhold_item >= 0 makes the record-staging warp skip that work item, so the
 * compute warps' wait for it runs out (-1: none).  Work items: Mamba-2
 * decode and verify (sequence * G + group) * chunks + chunk, with chunks = 1
 * when a group has at most 8 heads; GDN and KDA decode and GDN verify (bf16
 * inputs) sequence * H + head.  The
 * values apply to every launch made after the call, from any host thread.
 * Returns RSSM_ERR_INVALID_ARG for withhold_item < -1. */
rssm_status replayssm_set_test_hooks(int64_t consumer_wait_ns, int32_t withhold_item);

/* Start a state from a full state S0 (same layout as h0; device pointer):
 * h0 <- S0 (rounded to ckpt_fmt when set), len <- 0, read copy built from h0,
 * status word cleared.  S0 may equal state->h0. */
rssm_status replayssm_init(const rssm_desc *desc, rssm_state *state, const float *S0,
                           void *stream);

/* One decode step [sitech §How ReplaySSM works].  For each (sequence, head):
 * append the step's record at slot len; y from h0 (or its read copy) and the
 * len+1 buffered records; if len+1 == window, fold the records into h0, write
 * h0 (and the read copy) once and set len = 0, else len += 1.  Requires
 * 0 <= len < window on entry (else RSSM_ERR_STATE in the status word).
 * GDN: with gamma/R the products of the record alphas, the step evaluates
 * z = h0^T k and h0^T q once, u = beta (v - gamma z - sum_j R_j (k_j.k) u_j)
 * from the earlier records' cached u_j, and o = scale (gamma h0^T q +
 * sum_i R_i (k_i.q) u_i); u is appended with the record. */
rssm_status replayssm_decode_step(const rssm_desc *desc, rssm_state *state,
                                  const rssm_step_in *in, float *y, void *stream);

/* A decode step whose record was written into the state by its producer:
 * the kernel that computes a step's layer inputs (a projection's epilogue,
 * say) stores them straight into slot len[b][h] of the record buffers instead
 * of a separate step-input tensor, and this call then runs the step exactly
 * like replayssm_decode_step with those inputs, minus their read and append
 * [news.hamidun.com §Where the state problem appears: serving keeps per-
 * sequence state; the record written once, where the replay reads it].
 * Slots (elements; the producer reads len on the device; a sequence's heads
 * share one length):
 *   Mamba-2: x of head h at buf[0] + ((b*H + h)*cap + len)*P, dt (fp32) at
 *            buf[1] + (b*H + h)*cap + len, Bm and Cm of group g at
 *            buf[2|3] + ((b*G + g)*cap + len)*N;
 *   GDN/KDA: q, k at buf[0|1] + ((b*H + h)*cap + len)*DK, v at
 *            buf[2] + ((b*H + h)*cap + len)*DV, alpha at buf[3] +
 *            (b*H + h)*cap + len (KDA: times DK, DK decays), beta at
 *            buf[4] + (b*H + h)*cap + len.
 * A, D: Mamba-2 per-head parameters (ignored for GDN/KDA).  y dense
 * [B][H][P] / [B][H][DV].  Lengths out of range go to the status word, as
 * for replayssm_decode_step. */
rssm_status replayssm_decode_step_inplace(const rssm_desc *desc, rssm_state *state,
                                          const float *A, const float *D, float *y,
                                          void *stream);

/* Fold the buffer into h0 for every (sequence, head) with len >= window, or
 * with len > 0 when force != 0; those get len = 0.  A: Mamba-2 decay rates
 * [H] (NULL for GDN). */
rssm_status replayssm_flush(const rssm_desc *desc, rssm_state *state, const float *A,
                            int32_t force, void *stream);

/* Speculative verify round [sitech §Reducing state traffic...]:
 *   1. if accepted_prev != NULL: len += accepted_prev[b] (the previous round's
 *      accepted drafts are already in their slots) and, when len >= window,
 *      fold all len records into h0 and set len = 0;
 *   2. write the n_draft drafts of `drafts` to slots len .. len+n_draft-1
 *      (len itself is not advanced);
 *   3. y[b][d][h][p] = output of draft d evaluated from h0 and the len+d+1
 *      records, without forming any intermediate state.
 * Mamba-2 drafts: x [B][n][H][P], dt [B][n][H], Bm/Cm [B][n][G][N], y
 * [B][n][H][P].  Gated DeltaNet drafts [hamidun §Why hybrid models became
 * the norm]: q, k [B][n][H][DK], v [B][n][H][DV], alpha, beta [B][n][H], o
 * [B][n][H][DV]; each draft's delta-rule correction u (buf[5]) is stored with
 * it, so an accepted draft leaves exactly the correction sequential decoding
 * would have cached.
 * accepted_prev [B] int32 in 0..draft_max, and at most the n_draft of the
 * previous call (the device checks only the draft_max bound: a count above
 * the previous round's draft count would commit slots that round never
 * wrote).  1 <= n_draft <= draft_max.
 * Mamba-2: the draft rows of x, Bm and Cm are bulk-copied by the kernel:
 * their base pointers and batch strides (in bytes) must be multiples of 16,
 * else RSSM_ERR_ALIGNMENT is returned before any launch; H/G <= 8, else
 * RSSM_ERR_UNSUPPORTED.  Errors found on the device (a length out of range,
 * heads of a group out of step, accepted_prev[b] > draft_max, a round that
 * would overrun the capacity) set *status to RSSM_ERR_STATE and leave that
 * (sequence, group)'s lengths, checkpoint and committed records untouched
 * (when a group's heads are split over several work items, its draft B/C
 * rows may still be written to free slots at or above its length). */
rssm_status replayssm_verify_commit(const rssm_desc *desc, rssm_state *state,
                                    const int32_t *accepted_prev, const rssm_step_in *drafts,
                                    int32_t n_draft, float *y, void *stream);

/* Close a verify round: len += accepted[b]; fold when len >= window.  A:
 * Mamba-2 decay rates [H] (NULL for GDN). */
rssm_status replayssm_commit(const rssm_desc *desc, rssm_state *state, const int32_t *accepted,
                             const float *A, void *stream);

/* Conventional full-state decode step, the in-build comparison [sitech §How
 * ReplaySSM works]: S is read, updated and written in place every step, y is
 * read from the updated S.  S has the h0 layout.  If limit != NULL, sequence
 * b is stepped only when step_index < limit[b] (otherwise S and y of b are
 * not touched). */
rssm_status replayssm_full_decode_step(const rssm_desc *desc, float *S, const rssm_step_in *in,
                                       float *y, const int32_t *limit, int32_t step_index,
                                       void *stream);

/* S_out <- the full state h0 and the buffered records stand for (the fold
 * applied out of place); the replay state is not modified. */
rssm_status replayssm_materialize(const rssm_desc *desc, const rssm_state *state, const float *A,
                                  float *S_out, void *stream);

/* Build a read copy of ntile fp32 tiles of rows x cols (cols % 16 == 0 for
 * NVFP4): codes, block scales and tile scales as in rssm_state. */
rssm_status replayssm_quantize(int32_t fmt, int32_t ntile, int32_t rows, int32_t cols,
                               const float *src, uint8_t *codes, uint8_t *scales,
                               float *gscale, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* REPLAYSSM_H */
