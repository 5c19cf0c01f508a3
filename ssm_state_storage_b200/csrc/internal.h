// internal.h -- launcher interface between the C-ABI layer (api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/replayssm.h"

namespace rssm {

// Mamba-2 launch parameters: the descriptor unpacked plus every pointer a
// Mamba-2 kernel may touch.  Strides are in elements.
struct M2Params {
  int B, H, G, hpg, P, N, L, cap, draft_max;
  int in_bf16;
  int qmode;  // 0 none, 1/2 read copy FP8/NVFP4, 3/4 checkpoint rounded to FP8/NVFP4
  float *h0;
  void *xbuf;
  float *dtbuf;
  void *Bbuf, *Cbuf;
  int32_t *len;
  int32_t *status;
  uint8_t *rc, *rc_scale;
  float *rc_gscale;
  // step inputs (decode: [B][H][P] etc.; verify: with a draft axis)
  const void *x, *dt, *Bm, *Cm;
  int64_t bs_x, bs_dt, bs_B, bs_C, bs_y;
  const float *A, *D;
  float *y;
  // fold-only modes
  const int32_t *acc;
  int force;
  float *S_out;
  // conventional step
  float *S;
  const int32_t *limit;
  int step_index;
  // verify
  int n_draft;
  // bounded waits: the limit of every consumer-side wait, and (test hook) a
  // work item whose records the stager withholds, -1 for none
  uint64_t wait_ns;
  int hold_item;
  // the step's record was written to slot len of the buffers by its producer
  int inplace;
};

struct GDNParams {
  int B, H, DK, DV, L, cap;
  int in_bf16;
  int kda;  // Kimi Delta Attention: alpha and its records carry one decay per key channel
  float scale;
  float *h0;
  void *qbuf, *kbuf, *vbuf;
  float *abuf, *bbuf, *ubuf;
  int32_t *len;
  int32_t *status;
  const void *q, *k, *v;
  const float *alpha, *beta;
  int64_t bs_q, bs_k, bs_v, bs_a, bs_b, bs_y;
  float *y;
  int force;
  float *S_out;
  float *S;
  const int32_t *limit;
  int step_index;
  uint64_t wait_ns;  // as in M2Params
  int hold_item;
  // speculative rounds
  const int32_t *acc;
  int draft_max, n_draft;
  int inplace;  // as in M2Params
};

enum FoldMode { kFoldFlush = 0, kFoldCommit = 1, kFoldMaterialize = 2 };

cudaError_t m2_launch_decode(const M2Params &p, cudaStream_t s);
cudaError_t m2_launch_fold(const M2Params &p, int mode, cudaStream_t s);
cudaError_t m2_launch_full(const M2Params &p, cudaStream_t s);
cudaError_t m2_launch_verify(const M2Params &p, cudaStream_t s);
bool m2_supported(int P, int N);
bool m2_heads_supported(int hpg);  // heads per group: <= 8 or a multiple of 8

cudaError_t gdn_launch_decode(const GDNParams &p, cudaStream_t s);
cudaError_t gdn_launch_fold(const GDNParams &p, int mode, cudaStream_t s);
cudaError_t gdn_launch_verify(const GDNParams &p, cudaStream_t s);

// Kimi Delta Attention (GDNParams with alpha and its records per key channel):
// mode 0 decode step, 1 flush, 2 materialise, 3 conventional step; mode 3 with
// kda == 0 is the conventional Gated DeltaNet step (scalar alpha [B][H]).
cudaError_t kda_launch(const GDNParams &p, int mode, cudaStream_t s);
bool gdn_supported(int DK, int DV);

// Read copy of ntile tiles [rows][cols]; fmt 1 = FP8, 2 = NVFP4.  With
// roundtrip != 0 the tiles are replaced in place by deq(Q(tile)) instead.
cudaError_t quant_launch(int fmt, int ntile, int rows, int cols, const float *src,
                         uint8_t *codes, uint8_t *scales, float *gscale, int roundtrip,
                         float *dst, cudaStream_t s);

}  // namespace rssm
