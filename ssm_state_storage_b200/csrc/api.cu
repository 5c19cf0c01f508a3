// api.cu -- the C ABI declared in include/replayssm.h: host-side validation
// of descriptors, pointers and capacities, then kernel launches on the
// caller's stream.  No allocation, no synchronisation.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"

using namespace rssm;

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int cap_of(const rssm_desc *d) {
  return d->window + (d->draft_max > 1 ? d->draft_max - 1 : 0);
}

inline size_t es_of(const rssm_desc *d) { return d->in_dtype == RSSM_BF16 ? 2 : 4; }

rssm_status check_desc(const rssm_desc *d) {
  if (!d) return RSSM_ERR_INVALID_ARG;
  if (d->kind != RSSM_MAMBA2 && d->kind != RSSM_GDN && d->kind != RSSM_KDA)
    return RSSM_ERR_INVALID_ARG;
  if (d->batch < 0 || d->nheads <= 0 || d->headdim <= 0 || d->dstate <= 0)
    return RSSM_ERR_INVALID_ARG;
  if (d->in_dtype != RSSM_F32 && d->in_dtype != RSSM_BF16) return RSSM_ERR_DTYPE;
  if (d->read_fmt < RSSM_FMT_NONE || d->read_fmt > RSSM_FMT_NVFP4) return RSSM_ERR_INVALID_ARG;
  if (d->ckpt_fmt < RSSM_FMT_NONE || d->ckpt_fmt > RSSM_FMT_NVFP4) return RSSM_ERR_INVALID_ARG;
  if (d->read_fmt != RSSM_FMT_NONE && d->ckpt_fmt != RSSM_FMT_NONE) return RSSM_ERR_INVALID_ARG;
  if (d->window < 1 || d->window > 16) return RSSM_ERR_CAPACITY;
  if (d->draft_max < 0 || d->draft_max > 4) return RSSM_ERR_CAPACITY;
  if (cap_of(d) > kMaxCap) return RSSM_ERR_CAPACITY;
  if (d->kind == RSSM_MAMBA2) {
    if (d->ngroups <= 0 || d->nheads % d->ngroups != 0) return RSSM_ERR_SHAPE;
    if (!m2_supported(d->headdim, d->dstate)) return RSSM_ERR_SHAPE;
    if (!m2_heads_supported(d->nheads / d->ngroups)) return RSSM_ERR_SHAPE;
    if ((int64_t)d->batch * d->ngroups > INT32_MAX) return RSSM_ERR_SHAPE;
  } else {
    if (!gdn_supported(d->dstate, d->headdim)) return RSSM_ERR_SHAPE;
    if (d->read_fmt != RSSM_FMT_NONE || d->ckpt_fmt != RSSM_FMT_NONE) return RSSM_ERR_UNSUPPORTED;
    if (d->kind == RSSM_KDA && d->draft_max != 0) return RSSM_ERR_UNSUPPORTED;
    if ((int64_t)d->batch * d->nheads > INT32_MAX) return RSSM_ERR_SHAPE;
  }
  return RSSM_OK;
}

rssm_status check_state(const rssm_desc *d, const rssm_state *s) {
  if (!s || !s->h0 || !s->len || !s->status) return RSSM_ERR_INVALID_ARG;
  const int nbuf = d->kind == RSSM_MAMBA2 ? 4 : 6;
  for (int i = 0; i < nbuf; ++i)
    if (!s->buf[i]) return RSSM_ERR_INVALID_ARG;
  if (!aligned16(s->h0)) return RSSM_ERR_ALIGNMENT;
  for (int i = 0; i < nbuf; ++i)
    if (!aligned16(s->buf[i])) return RSSM_ERR_ALIGNMENT;
  if (d->read_fmt == RSSM_FMT_FP8) {
    if (!s->rc) return RSSM_ERR_INVALID_ARG;
    if (!aligned16(s->rc)) return RSSM_ERR_ALIGNMENT;
  } else if (d->read_fmt == RSSM_FMT_NVFP4) {
    if (!s->rc || !s->rc_scale || !s->rc_gscale) return RSSM_ERR_INVALID_ARG;
    if (!aligned16(s->rc) || !aligned16(s->rc_scale)) return RSSM_ERR_ALIGNMENT;
  }
  return RSSM_OK;
}

inline cudaStream_t to_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

// Test hooks of the bounded waits (replayssm_set_test_hooks).
std::atomic<uint64_t> g_wait_ns{kWaitLimitNs};
std::atomic<int> g_hold_item{-1};

inline rssm_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return RSSM_OK;
  g_last_cuda_error = e;
  return RSSM_ERR_CUDA;
}

inline int64_t stride_or(int64_t s, int64_t dense) { return s != 0 ? s : dense; }

M2Params m2_params(const rssm_desc *d, const rssm_state *s) {
  M2Params p;
  std::memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.H = d->nheads;
  p.G = d->ngroups;
  p.hpg = d->nheads / d->ngroups;
  p.P = d->headdim;
  p.N = d->dstate;
  p.L = d->window;
  p.cap = cap_of(d);
  p.draft_max = d->draft_max;
  p.in_bf16 = d->in_dtype == RSSM_BF16;
  p.qmode = d->read_fmt != RSSM_FMT_NONE ? d->read_fmt : (d->ckpt_fmt != RSSM_FMT_NONE ? 2 + d->ckpt_fmt : 0);
  p.wait_ns = g_wait_ns.load();
  p.hold_item = g_hold_item.load();
  if (s) {
    p.h0 = s->h0;
    p.xbuf = s->buf[0];
    p.dtbuf = static_cast<float *>(s->buf[1]);
    p.Bbuf = s->buf[2];
    p.Cbuf = s->buf[3];
    p.len = s->len;
    p.status = s->status;
    p.rc = s->rc;
    p.rc_scale = s->rc_scale;
    p.rc_gscale = s->rc_gscale;
  }
  return p;
}

void m2_inputs(M2Params &p, const rssm_step_in *in, int nd) {
  p.x = in->in[0];
  p.dt = in->in[1];
  p.Bm = in->in[2];
  p.Cm = in->in[3];
  p.A = in->A;
  p.D = in->D;
  p.bs_x = stride_or(in->batch_stride[0], (int64_t)nd * p.H * p.P);
  p.bs_dt = stride_or(in->batch_stride[1], (int64_t)nd * p.H);
  p.bs_B = stride_or(in->batch_stride[2], (int64_t)nd * p.G * p.N);
  p.bs_C = stride_or(in->batch_stride[3], (int64_t)nd * p.G * p.N);
  p.bs_y = stride_or(in->y_batch_stride, (int64_t)nd * p.H * p.P);
}

rssm_status check_m2_inputs(const rssm_step_in *in, bool need_out) {
  if (!in) return RSSM_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!in->in[i]) return RSSM_ERR_INVALID_ARG;
  if (!in->A || (need_out && !in->D)) return RSSM_ERR_INVALID_ARG;
  return RSSM_OK;
}

GDNParams gdn_params(const rssm_desc *d, const rssm_state *s) {
  GDNParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = d->batch;
  p.H = d->nheads;
  p.DK = d->dstate;
  p.DV = d->headdim;
  p.L = d->window;
  p.cap = cap_of(d);
  p.in_bf16 = d->in_dtype == RSSM_BF16;
  p.scale = d->scale;
  p.kda = d->kind == RSSM_KDA;
  p.draft_max = d->draft_max;
  p.wait_ns = g_wait_ns.load();
  p.hold_item = g_hold_item.load();
  if (s) {
    p.h0 = s->h0;
    p.qbuf = s->buf[0];
    p.kbuf = s->buf[1];
    p.vbuf = s->buf[2];
    p.abuf = static_cast<float *>(s->buf[3]);
    p.bbuf = static_cast<float *>(s->buf[4]);
    p.ubuf = static_cast<float *>(s->buf[5]);
    p.len = s->len;
    p.status = s->status;
  }
  return p;
}

// nd: the length of the draft axis after the batch axis (1 for a decode step)
rssm_status gdn_inputs(GDNParams &p, const rssm_step_in *in, int nd = 1) {
  if (!in) return RSSM_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i)
    if (!in->in[i]) return RSSM_ERR_INVALID_ARG;
  p.q = in->in[0];
  p.k = in->in[1];
  p.v = in->in[2];
  p.alpha = static_cast<const float *>(in->in[3]);
  p.beta = static_cast<const float *>(in->in[4]);
  p.bs_q = stride_or(in->batch_stride[0], (int64_t)nd * p.H * p.DK);
  p.bs_k = stride_or(in->batch_stride[1], (int64_t)nd * p.H * p.DK);
  p.bs_v = stride_or(in->batch_stride[2], (int64_t)nd * p.H * p.DV);
  p.bs_a = stride_or(in->batch_stride[3], (int64_t)nd * p.H * (p.kda ? p.DK : 1));
  p.bs_b = stride_or(in->batch_stride[4], (int64_t)nd * p.H);
  p.bs_y = stride_or(in->y_batch_stride, (int64_t)nd * p.H * p.DV);
  return RSSM_OK;
}

}  // namespace

extern "C" {

rssm_status replayssm_validate(const rssm_desc *desc) { return check_desc(desc); }

int32_t replayssm_capacity(const rssm_desc *desc) {
  if (check_desc(desc) != RSSM_OK) return 0;
  return cap_of(desc);
}

size_t replayssm_state_bytes(const rssm_desc *d, int32_t which) {
  if (check_desc(d) != RSSM_OK) return 0;
  const size_t B = d->batch, H = d->nheads, P = d->headdim, N = d->dstate;
  const size_t cap = cap_of(d), es = es_of(d);
  const bool m2 = d->kind == RSSM_MAMBA2;
  const size_t G = m2 ? (size_t)d->ngroups : H;
  switch (which) {
    case RSSM_BYTES_H0:
    case RSSM_BYTES_FULL_STATE: return B * H * P * N * 4;
    case RSSM_BYTES_BUF0 + 0: return m2 ? B * H * cap * P * es : B * H * cap * N * es;
    case RSSM_BYTES_BUF0 + 1: return m2 ? B * H * cap * 4 : B * H * cap * N * es;
    case RSSM_BYTES_BUF0 + 2: return m2 ? B * G * cap * N * es : B * H * cap * P * es;
    case RSSM_BYTES_BUF0 + 3:
      return m2 ? B * G * cap * N * es : B * H * cap * (d->kind == RSSM_KDA ? N : 1) * 4;
    case RSSM_BYTES_BUF0 + 4: return m2 ? 0 : B * H * cap * 4;
    case RSSM_BYTES_BUF0 + 5: return m2 ? 0 : B * H * cap * P * 4;
    case RSSM_BYTES_LEN: return B * H * 4;
    case RSSM_BYTES_RC:
      return d->read_fmt == RSSM_FMT_FP8 ? B * H * P * N
             : d->read_fmt == RSSM_FMT_NVFP4 ? B * H * P * N / 2 : 0;
    case RSSM_BYTES_RC_SCALE: return d->read_fmt == RSSM_FMT_NVFP4 ? B * H * P * N / 16 : 0;
    case RSSM_BYTES_RC_GSCALE: return d->read_fmt == RSSM_FMT_NVFP4 ? B * H * 4 : 0;
    case RSSM_BYTES_STATUS: return 4;
    case RSSM_BYTES_Y: return B * H * P * 4;
    default: return 0;
  }
}

const char *replayssm_status_string(rssm_status s) {
  switch (s) {
    case RSSM_OK: return "ok";
    case RSSM_ERR_INVALID_ARG: return "invalid argument";
    case RSSM_ERR_SHAPE: return "unsupported shape";
    case RSSM_ERR_DTYPE: return "unsupported dtype";
    case RSSM_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case RSSM_ERR_CAPACITY: return "buffer capacity exceeded";
    case RSSM_ERR_CUDA: return "CUDA launch error";
    case RSSM_ERR_TIMEOUT: return "device wait timed out";
    case RSSM_ERR_UNSUPPORTED: return "unsupported by this build";
    case RSSM_ERR_STATE: return "buffer state out of range";
    default: return "unknown status";
  }
}

const char *replayssm_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

rssm_status replayssm_set_test_hooks(int64_t consumer_wait_ns, int32_t withhold_item) {
  if (withhold_item < -1) return RSSM_ERR_INVALID_ARG;
  g_wait_ns.store(consumer_wait_ns > 0 ? (uint64_t)consumer_wait_ns : kWaitLimitNs);
  g_hold_item.store(withhold_item);
  return RSSM_OK;
}

rssm_status replayssm_init(const rssm_desc *d, rssm_state *s, const float *S0, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (!S0) return RSSM_ERR_INVALID_ARG;
  cudaStream_t cs = to_stream(stream);
  const size_t bytes = replayssm_state_bytes(d, RSSM_BYTES_H0);
  cudaError_t e = cudaSuccess;
  if (S0 != s->h0 && bytes) e = cudaMemcpyAsync(s->h0, S0, bytes, cudaMemcpyDeviceToDevice, cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(s->len, 0, replayssm_state_bytes(d, RSSM_BYTES_LEN), cs);
  if (e == cudaSuccess) e = cudaMemsetAsync(s->status, 0, sizeof(int32_t), cs);
  const int ntile = d->batch * d->nheads;
  if (e == cudaSuccess && d->ckpt_fmt != RSSM_FMT_NONE)
    e = quant_launch(d->ckpt_fmt, ntile, d->headdim, d->dstate, s->h0, nullptr, nullptr, nullptr,
                     1, s->h0, cs);
  if (e == cudaSuccess && d->read_fmt != RSSM_FMT_NONE)
    e = quant_launch(d->read_fmt, ntile, d->headdim, d->dstate, s->h0, s->rc, s->rc_scale,
                     s->rc_gscale, 0, nullptr, cs);
  return from_cuda(e);
}

rssm_status replayssm_decode_step(const rssm_desc *d, rssm_state *s, const rssm_step_in *in,
                                  float *y, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (!y) return RSSM_ERR_INVALID_ARG;
  if (d->kind == RSSM_MAMBA2) {
    if ((st = check_m2_inputs(in, true)) != RSSM_OK) return st;
    M2Params p = m2_params(d, s);
    m2_inputs(p, in, 1);
    p.y = y;
    return from_cuda(m2_launch_decode(p, to_stream(stream)));
  }
  GDNParams p = gdn_params(d, s);
  if ((st = gdn_inputs(p, in)) != RSSM_OK) return st;
  p.y = y;
  if (p.kda) return from_cuda(kda_launch(p, 0, to_stream(stream)));
  return from_cuda(gdn_launch_decode(p, to_stream(stream)));
}

rssm_status replayssm_decode_step_inplace(const rssm_desc *d, rssm_state *s, const float *A,
                                          const float *D, float *y, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (!y) return RSSM_ERR_INVALID_ARG;
  if (d->kind == RSSM_MAMBA2) {
    if (!A || !D) return RSSM_ERR_INVALID_ARG;
    M2Params p = m2_params(d, s);
    // the step-input pointers are never read in place: point them at the buffers
    p.x = s->buf[0];
    p.dt = s->buf[1];
    p.Bm = s->buf[2];
    p.Cm = s->buf[3];
    p.A = A;
    p.D = D;
    p.bs_y = (int64_t)p.H * p.P;
    p.y = y;
    p.inplace = 1;
    return from_cuda(m2_launch_decode(p, to_stream(stream)));
  }
  GDNParams p = gdn_params(d, s);
  p.q = s->buf[0];
  p.k = s->buf[1];
  p.v = s->buf[2];
  p.alpha = static_cast<const float *>(s->buf[3]);
  p.beta = static_cast<const float *>(s->buf[4]);
  p.bs_y = (int64_t)p.H * p.DV;
  p.y = y;
  p.inplace = 1;
  if (p.kda) return from_cuda(kda_launch(p, 0, to_stream(stream)));
  return from_cuda(gdn_launch_decode(p, to_stream(stream)));
}

rssm_status replayssm_flush(const rssm_desc *d, rssm_state *s, const float *A, int32_t force,
                            void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (d->kind == RSSM_MAMBA2) {
    if (!A) return RSSM_ERR_INVALID_ARG;
    M2Params p = m2_params(d, s);
    p.A = A;
    p.force = force != 0;
    return from_cuda(m2_launch_fold(p, kFoldFlush, to_stream(stream)));
  }
  GDNParams p = gdn_params(d, s);
  p.force = force != 0;
  if (p.kda) return from_cuda(kda_launch(p, 1, to_stream(stream)));
  return from_cuda(gdn_launch_fold(p, kFoldFlush, to_stream(stream)));
}

rssm_status replayssm_verify_commit(const rssm_desc *d, rssm_state *s,
                                    const int32_t *accepted_prev, const rssm_step_in *drafts,
                                    int32_t n_draft, float *y, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->read_fmt != RSSM_FMT_NONE || d->ckpt_fmt != RSSM_FMT_NONE) return RSSM_ERR_UNSUPPORTED;
  if (d->kind == RSSM_KDA) return RSSM_ERR_UNSUPPORTED;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (n_draft < 1 || n_draft > d->draft_max) return RSSM_ERR_CAPACITY;
  if (d->kind == RSSM_GDN) {
    if (!y) return RSSM_ERR_INVALID_ARG;
    GDNParams p = gdn_params(d, s);
    if ((st = gdn_inputs(p, drafts, n_draft)) != RSSM_OK) return st;
    p.y = y;
    p.acc = accepted_prev;
    p.n_draft = n_draft;
    return from_cuda(gdn_launch_verify(p, to_stream(stream)));
  }
  // the verify stager maps (draft, head) pairs of a work item onto one warp's lanes
  if (d->nheads / d->ngroups > 8) return RSSM_ERR_UNSUPPORTED;
  if (!y) return RSSM_ERR_INVALID_ARG;
  if ((st = check_m2_inputs(drafts, true)) != RSSM_OK) return st;
  M2Params p = m2_params(d, s);
  m2_inputs(p, drafts, n_draft);
  // the kernel bulk-copies draft rows of x, B and C: each row must start on
  // a 16-byte boundary
  const int64_t es = (int64_t)es_of(d);
  if (!aligned16(drafts->in[0]) || !aligned16(drafts->in[2]) || !aligned16(drafts->in[3]) ||
      (p.bs_x * es) % 16 || (p.bs_B * es) % 16 || (p.bs_C * es) % 16)
    return RSSM_ERR_ALIGNMENT;
  p.y = y;
  p.acc = accepted_prev;
  p.n_draft = n_draft;
  return from_cuda(m2_launch_verify(p, to_stream(stream)));
}

rssm_status replayssm_commit(const rssm_desc *d, rssm_state *s, const int32_t *accepted,
                             const float *A, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->kind == RSSM_KDA) return RSSM_ERR_UNSUPPORTED;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (!accepted) return RSSM_ERR_INVALID_ARG;
  if (d->kind == RSSM_GDN) {
    GDNParams p = gdn_params(d, s);
    p.acc = accepted;
    return from_cuda(gdn_launch_fold(p, kFoldCommit, to_stream(stream)));
  }
  if (!A) return RSSM_ERR_INVALID_ARG;
  M2Params p = m2_params(d, s);
  p.acc = accepted;
  p.A = A;
  return from_cuda(m2_launch_fold(p, kFoldCommit, to_stream(stream)));
}

rssm_status replayssm_full_decode_step(const rssm_desc *d, float *S, const rssm_step_in *in,
                                       float *y, const int32_t *limit, int32_t step_index,
                                       void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if (!S || !y) return RSSM_ERR_INVALID_ARG;
  if (!aligned16(S)) return RSSM_ERR_ALIGNMENT;
  if (d->kind == RSSM_MAMBA2) {
    if ((st = check_m2_inputs(in, true)) != RSSM_OK) return st;
    M2Params p = m2_params(d, nullptr);
    m2_inputs(p, in, 1);
    p.S = S;
    p.y = y;
    p.limit = limit;
    p.step_index = step_index;
    return from_cuda(m2_launch_full(p, to_stream(stream)));
  }
  GDNParams p = gdn_params(d, nullptr);
  if ((st = gdn_inputs(p, in)) != RSSM_OK) return st;
  p.S = S;
  p.y = y;
  p.limit = limit;
  p.step_index = step_index;
  // the delta-rule conventional step (per-channel decays for KDA, one decay
  // broadcast over the channels for GDN)
  return from_cuda(kda_launch(p, 3, to_stream(stream)));
}

rssm_status replayssm_materialize(const rssm_desc *d, const rssm_state *s, const float *A,
                                  float *S_out, void *stream) {
  rssm_status st = check_desc(d);
  if (st != RSSM_OK) return st;
  if (d->batch == 0) return RSSM_OK;  // empty batch: no pointer is read, nothing runs
  if ((st = check_state(d, s)) != RSSM_OK) return st;
  if (!S_out) return RSSM_ERR_INVALID_ARG;
  if (!aligned16(S_out)) return RSSM_ERR_ALIGNMENT;
  if (d->kind == RSSM_MAMBA2) {
    if (!A) return RSSM_ERR_INVALID_ARG;
    M2Params p = m2_params(d, s);
    p.A = A;
    p.S_out = S_out;
    return from_cuda(m2_launch_fold(p, kFoldMaterialize, to_stream(stream)));
  }
  GDNParams p = gdn_params(d, s);
  p.S_out = S_out;
  if (p.kda) return from_cuda(kda_launch(p, 2, to_stream(stream)));
  return from_cuda(gdn_launch_fold(p, kFoldMaterialize, to_stream(stream)));
}

rssm_status replayssm_quantize(int32_t fmt, int32_t ntile, int32_t rows, int32_t cols,
                               const float *src, uint8_t *codes, uint8_t *scales, float *gscale,
                               void *stream) {
  if (fmt != RSSM_FMT_FP8 && fmt != RSSM_FMT_NVFP4) return RSSM_ERR_INVALID_ARG;
  if (ntile < 0 || rows <= 0 || cols <= 0) return RSSM_ERR_INVALID_ARG;
  if (ntile == 0) return RSSM_OK;
  if (!src || !codes) return RSSM_ERR_INVALID_ARG;
  if (fmt == RSSM_FMT_NVFP4 && (cols % 16 != 0 || !scales || !gscale)) return RSSM_ERR_SHAPE;
  return from_cuda(quant_launch(fmt, ntile, rows, cols, src, codes, scales, gscale, 0, nullptr,
                                to_stream(stream)));
}

}  // extern "C"
