// m2.cu -- Mamba-2 decode kernels for sm_100a: replay decode step with fused
// flush fold, standalone fold (flush / commit / materialise) and the
// conventional full-state step.  The speculative verify round is in
// m2_verify.cu; helpers shared by both are in m2_device.cuh.
//
// Method: every (sequence, head) keeps a checkpoint h0 and a buffer of the
// latest input records; a non-flush step appends the current record and
// produces the output from h0 and the buffer with no state write; when the
// buffer holds `window` records the step folds them into h0 and writes h0
// once.  [sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…", §How ReplaySSM
// works]
//
// Recurrence (Mamba-2, Dao & Gu 2024), per head with decay rate A:
//   dA_t = exp(dt_t A);  S_t = dA_t S_{t-1} + dt_t x_t B_t^T;  y_t = S_t C_t + D x_t.
// Unrolled from h0 over k buffered records (record k-1 is the current one),
// with s_i = sum_{i<m<k} dt_m and w_i = exp(A s_i) dt_i, Lam = exp(A sum_m dt_m):
//   S_k = Lam h0 + sum_i w_i x_i B_i^T                          (fold)
//   y_k = Lam (h0 C_k) + sum_i w_i (B_i . C_k) x_i + D x_k        (replay output)
// The decay factors are evaluated as exp of suffix sums of dt, so no product
// of many small factors is ever formed.
//
// Work item = (sequence b, group g): the heads of a group share B and C, so the
// B_i . C_k dot products are formed once per item.  A CTA of 256 threads walks
// the group's heads; each head tile (P x N fp32, contiguous) is streamed into
// registers with 128-bit loads: lane (rs = lane/8, c8 = lane%8) of warp w holds
// rows w*P/8 + rs + 4*rho and columns 32*s + 4*c8, so each quarter-warp reads
// one 128-byte line and the row sums need only 3 shuffle levels.
#include "m2_device.cuh"
#include "umma.cuh"

namespace rssm {
namespace {

// =============================================================== decode step
// Persistent, warp-specialised kernel: one CTA per SM walks work items
// (sequence, group, head chunk) in a static round-robin.  Warp 8 is the
// producer: for each item it reads the buffer length, bulk-copies the
// item's buffered records (the group's B records, every head's x records)
// into one of two record buffers, then streams the item's checkpoint tiles
// (or read-copy tiles) into a ring of NS shared-memory slots, each slot's
// arrival tracked by an mbarrier.  Warps 0-7 consume: per item they add this
// step's record, form the B_i.C_k dots and every head's decay weights, then
// for each head pull the tile from the ring into registers, release the slot,
// write y and, on the flush step, fold the tile and write it back.
// HBM traffic therefore overlaps all per-item setup work.

// Byte layout of the decode kernel's shared memory (host and device agree).
// Per record buffer rb (NR = 1 to 3 of them): the group's B records
// [L][N] and every head's x records [hc][L][P] (input dtype; slot k-1 holds
// this step's record), plus a small "stage" block of fp32 values written by
// the producer warp: C_k [N], dt records [hc][L], A [hc], D [hc], header.
struct DecodeLayout {
  int NS, NR, hc, L, tile_bytes, tile_stride, stage_floats, scratch_floats;
  int off_bars, off_recB, off_recX, off_stage, off_scr, off_umma, off_ring, total;
  int umma_b_bytes;  // tensor-core fold: bytes of one head group's B operands (3 terms)

  __host__ __device__ static int align128(int v) { return (v + 127) & ~127; }

  // mma: the flush fold runs on the tensor cores (operand areas added, no
  // fp32 copy of the B records); hpq: heads in flight at once.
  __host__ static DecodeLayout make(int P, int N, int hc, int L, int es, int qm, int budget,
                                    bool mma = false, int hpq = 1) {
    DecodeLayout d;
    d.hc = hc;
    d.L = L;
    d.tile_bytes = qm == 1 ? P * N : qm == 2 ? P * N / 2 + P * N / 16 : P * N * 4;
    d.tile_stride = align128(d.tile_bytes);
    d.stage_floats = N + pad4(hc * L) + 2 * pad4(hc) + 4;
    d.scratch_floats = 2 * pad4(L) + pad4(hc * L) + pad4(hc) + 32 + (mma ? 0 : L * N) + hc * P;
    // A operand: the group's B records as a 128 x 16 K-slab; per head group
    // the three split terms of its head's weighted x records, P x 16 each
    d.umma_b_bytes = mma ? 3 * P * 32 : 0;
    const int umma_bytes = mma ? N * 32 + hpq * d.umma_b_bytes : 0;
    const int rec_b = L * N * es, rec_x = hc * L * P * es;
    // Prefer three record buffers (the stager then runs two items ahead, which
    // hides its two dependent memory round trips) as long as the ring keeps
    // at least 3 slots; fall back to fewer buffers for large tiles.
    for (d.NR = 3; d.NR >= 1; --d.NR) {
      int o = 0;
      d.off_bars = o;
      // up to 8 ring slots and 4 record buffers (192 bytes), then two fold-MMA
      // barriers and the tensor-memory base address
      o += align128(8 * (2 * 8 + 2 * 4) + 2 * 8 + 4);
      d.off_recB = o;
      o += align128(d.NR * rec_b);
      d.off_recX = o;
      o += align128(d.NR * rec_x);
      d.off_stage = o;
      o += align128(d.NR * d.stage_floats * 4);
      d.off_scr = o;
      o += align128(2 * d.scratch_floats * 4);
      d.off_umma = o;
      o += align128(umma_bytes);
      d.off_ring = o;
      const int room = budget - o;
      d.NS = room / d.tile_stride;
      if (d.NS > 8) d.NS = 8;
      if (d.NS >= (d.NR == 1 ? 2 : 3)) {
        d.total = o + d.NS * d.tile_stride;
        return d;
      }
    }
    d.NS = 0;
    return d;
  }
};

// Read view of a head tile held in shared memory (fp32, FP8 or NVFP4 codes).
template <int P, int N, int QM>
__device__ __forceinline__ void view_from_smem(const unsigned char *t, float sg, int warp, int rs,
                                               int c8, float4 (&v)[P / 32][N / 32]) {
  using T = Tile<P, N>;
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
    for (int s = 0; s < T::C4; ++s) {
      const int r = T::row(warp, rs, rho), c = T::col(c8, s);
      if constexpr (QM == 1) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(t + r * N + c);
        v[rho][s] = make_float4(e4m3_decode(w & 0xFF), e4m3_decode((w >> 8) & 0xFF),
                                e4m3_decode((w >> 16) & 0xFF), e4m3_decode(w >> 24));
      } else if constexpr (QM == 2) {
        const uint32_t w = *reinterpret_cast<const uint16_t *>(t + r * (N / 2) + c / 2);
        const float sb = e4m3_decode(t[P * N / 2 + r * (N / 16) + c / 16]);
        v[rho][s] = make_float4(nvfp4_value(w & 0xF, sb, sg), nvfp4_value((w >> 4) & 0xF, sb, sg),
                                nvfp4_value((w >> 8) & 0xF, sb, sg),
                                nvfp4_value((w >> 12) & 0xF, sb, sg));
      } else {
        v[rho][s] = *reinterpret_cast<const float4 *>(t + (r * N + c) * 4);
      }
    }
}

struct DecodeSmemPtrs {
  uint64_t *full, *empty, *rfull, *rempty, *mma;
  uint32_t *tmem_slot;
  unsigned char *ring, *umma;
  unsigned char *recB, *recX;
  float *stage, *scr;
  __device__ DecodeSmemPtrs(unsigned char *smem, const DecodeLayout &lay) {
    full = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
    empty = full + 8;
    rfull = empty + 8;
    rempty = rfull + 4;
    mma = rempty + 4;  // one per head group: its fold MMAs completed
    tmem_slot = reinterpret_cast<uint32_t *>(mma + 2);
    umma = smem + lay.off_umma;
    ring = smem + lay.off_ring;
    recB = smem + lay.off_recB;
    recX = smem + lay.off_recX;
    stage = reinterpret_cast<float *>(smem + lay.off_stage);
    scr = reinterpret_cast<float *>(smem + lay.off_scr);
  }
};

// Stage block of record buffer rb: C [N] | dt [hc][L] | A [hc] | D [hc] | hdr [4]
// (hdr: n0, bad, gscale (NVFP4 tile scales are read per head by consumers)).
struct Stage {
  float *C, *dt, *A, *D;
  int *hdr;
  __device__ Stage(float *base, int N, int hc, int L) {
    C = base;
    dt = C + N;
    A = dt + pad4(hc * L);
    D = A + pad4(hc);
    hdr = reinterpret_cast<int *>(D + pad4(hc));
  }
};


// Stager warp: for item `it` wait until its record buffer is free, then stage
// the small per-item inputs.  Every global load of the item is issued first
// into registers (none depends on the buffer length: all `window` dt slots
// are read), so the item costs one memory latency; then the values are
// written to shared memory, and lane 0 bulk-copies the buffered records and
// arrives on the buffer's barrier.
template <int P, int N, typename TI>
__device__ __forceinline__ bool stage_item(const M2Params &p, const DecodeLayout &lay,
                                           const DecodeSmemPtrs &S, int item, int it, int nchunk,
                                           int lane, volatile int *abort_flag) {
  constexpr int NPL = N / 32;          // B and C values per lane
  constexpr int XPL = 8 * P / 32;      // x values per lane (up to 8 heads)
  constexpr int DPL = 8 * 16 / 32;     // dt slots per lane (up to 8 heads x 16)
  const int hc = lay.hc, L = lay.L;
  const int rb = it % lay.NR;
  const uint32_t rphase = (it / lay.NR) & 1;
  bool ok = true;
  if (lane == 0) ok = mbar_wait(&S.rempty[rb], rphase ^ 1, kWaitLimitNs, abort_flag) && !*abort_flag;
  if (!__shfl_sync(0xffffffffu, (int)ok, 0)) return false;
  int b, g, chunk, h_first;
  item_coords(p, item, nchunk, hc, b, g, chunk, h_first);
  const size_t bh0 = (size_t)b * p.H + h_first;
  const TI *__restrict__ Bin = static_cast<const TI *>(p.Bm) + b * p.bs_B + (size_t)g * N;
  const TI *__restrict__ Cin = static_cast<const TI *>(p.Cm) + b * p.bs_C + (size_t)g * N;
  const TI *__restrict__ xin = static_cast<const TI *>(p.x) + b * p.bs_x + (size_t)h_first * P;

  // ---- phase 1: every load of the item, independent of one another (with
  // the record already in its buffer slot, the x/B/C loads wait for the length)
  const int my_len = lane < hc ? __ldcg(&p.len[bh0 + lane]) : 0;
  const float my_A = lane < hc ? p.A[h_first + lane] : 0.f;
  const float my_D = lane < hc ? p.D[h_first + lane] : 0.f;
  const float my_dt = (lane < hc && !p.inplace) ? ld_in<TI>(p.dt, b * p.bs_dt + h_first + lane) : 0.f;
  const TI *xsrc = xin, *bsrc = Bin, *csrc = Cin;
  int xstride = P;  // elements between consecutive heads' x
  if (p.inplace) {
    const int slot = min(max(__shfl_sync(0xffffffffu, my_len, 0), 0), L - 1);  // stays in bounds
    const size_t bg = (size_t)b * p.G + g;
    xsrc = static_cast<const TI *>(p.xbuf) + (bh0 * p.cap + slot) * P;
    xstride = p.cap * P;
    bsrc = static_cast<const TI *>(p.Bbuf) + (bg * p.cap + slot) * N;
    csrc = static_cast<const TI *>(p.Cbuf) + (bg * p.cap + slot) * N;
  }
  TI bv[NPL], cv[NPL], xv[XPL];
  float dtv[DPL];
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    bv[u] = bsrc[lane + 32 * u];
    cv[u] = csrc[lane + 32 * u];
  }
#pragma unroll
  for (int u = 0; u < XPL; ++u) {
    const int e = lane + 32 * u;
    xv[u] = e < hc * P ? xsrc[(e / P) * xstride + e % P] : TI{};
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int e = lane + 32 * u, j = e / L, i = e - j * L;
    dtv[u] = e < hc * L ? __ldcg(&p.dtbuf[(bh0 + j) * p.cap + i]) : 0.f;
  }

  // ---- phase 2: buffer length and its checks
  const int n0 = __shfl_sync(0xffffffffu, my_len, 0);
  const bool bad = __any_sync(0xffffffffu, (lane < hc && my_len != n0) || n0 < 0 || n0 >= L);
  const int k = min(max(n0 + 1, 1), L);  // copies stay in bounds even for a bad length

  // ---- phase 3: shared-memory writes
  Stage st(S.stage + rb * lay.stage_floats, N, hc, L);
  TI *rB = reinterpret_cast<TI *>(S.recB) + (size_t)rb * L * N;
  TI *rX = reinterpret_cast<TI *>(S.recX) + (size_t)rb * hc * L * P;
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    rB[(k - 1) * N + lane + 32 * u] = bv[u];
    st.C[lane + 32 * u] = to_f32(cv[u]);
  }
#pragma unroll
  for (int u = 0; u < XPL; ++u) {
    const int e = lane + 32 * u, j = e / P, q = e - j * P;
    if (e < hc * P) rX[(j * L + k - 1) * P + q] = xv[u];
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int e = lane + 32 * u, j = e / L, i = e - j * L;
    const float cur = __shfl_sync(0xffffffffu, my_dt, j < 32 ? j : 0);
    if (e < hc * L) st.dt[e] = (i == k - 1 && !p.inplace) ? cur : dtv[u];
  }
  if (lane < hc) {
    st.A[lane] = my_A;
    st.D[lane] = my_D;
  }
  if (lane == 0) {
    st.hdr[0] = n0;
    st.hdr[1] = bad;
  }
  fence_proxy_async_smem();  // these generic writes precede later bulk copies into the buffer
  __syncwarp();
  if (lane == 0) {
    const uint32_t bytesB = (k - 1) * N * sizeof(TI), bytesX = (k - 1) * P * sizeof(TI);
    mbar_arrive_expect_tx(&S.rfull[rb], bytesB + hc * bytesX);
    if (k > 1) {
      const size_t bg = (size_t)b * p.G + g;
      bulk_g2s(rB, static_cast<const TI *>(p.Bbuf) + bg * p.cap * N, bytesB, &S.rfull[rb]);
      for (int j = 0; j < hc; ++j)
        bulk_g2s(rX + (size_t)j * L * P, static_cast<const TI *>(p.xbuf) + (bh0 + j) * p.cap * P,
                 bytesX, &S.rfull[rb]);
    }
  }
  return true;
}

template <int P, int N, typename TI>
__device__ __forceinline__ void decode_stager(const M2Params &p, const DecodeLayout &lay,
                                              const DecodeSmemPtrs &S, volatile int *abort_flag,
                                              int nitems, int nchunk, int lane) {
  int it = 0;
  ArmedRecords armed;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
    // warp-uniform view of the abort flag: every lane takes the same branch
    const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
    if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
    if (abort_now || !stage_item<P, N, TI>(p, lay, S, item, it, nchunk, lane, abort_flag)) {
      if (lane == 0 && !*abort_flag) {
        report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      break;
    }
    armed.arm(it % lay.NR, (it / lay.NR) & 1);
  }
  // the items staged ahead may never be consumed if the consumers stop: wait
  // for their record copies before the warp (and possibly the CTA) ends
  if (lane == 0) armed.drain(S.rfull, lay.NR);
  __syncwarp();
}

// Tile producer (one lane): streams the items' checkpoint (or read-copy)
// tiles into a ring of NS slots, hc heads per item, waiting only for free
// slots.  On a failed wait it marks the CTA aborted and waits (bounded) for
// the copies it has in flight before returning.
template <int P, int N, int QM>
__device__ __forceinline__ void decode_tiles(const M2Params &p, const DecodeLayout &lay,
                                             const DecodeSmemPtrs &S, volatile int *abort_flag,
                                             int nitems, int nchunk) {
  stream_tiles<P, N, QM>(p, S.full, S.empty, S.ring, lay.NS, lay.tile_stride, lay.tile_bytes,
                         lay.hc, abort_flag, nitems, nchunk);
}


// ------------------------------------------------- tensor-core flush fold
// On the flush step the fold's rank-k update runs on the tensor cores:
//   D_j[n][r] = sum_i B_i[n] * (w_{j,i} x_{j,i}[r])        (M = N = 128, N' = P, K = 16)
// as a bf16 MMA with an fp32 accumulator in tensor memory.  B_i is bf16
// (exact); the fp32 products w x are split into three bf16 terms (three
// MMAs into the same accumulator), so every partial product is exact and the
// increment keeps fp32 accuracy.  The epilogue then forms
//   h0[r][n] <- Lam_j h0[r][n] + D_j[n][r]
// with tensor-memory lane n (= state column) per thread, so each warp's
// loads of the old tile and stores of the new one cover 32 consecutive
// columns of a row.

// A operand: the group's B records, A[n][i] = B_i[n] (zero for i >= k),
// written by all consumer threads.
template <int N, typename TI>
__device__ __forceinline__ void build_fold_a(unsigned char *dst, const TI *rB, int k, int tid) {
  for (int e = tid; e < N * 8; e += kThreads) {
    const int n = e % N, q = e / N, i0 = 2 * q;
    const TI b0 = i0 < k ? rB[i0 * N + n] : TI{}, b1 = i0 + 1 < k ? rB[(i0 + 1) * N + n] : TI{};
    __nv_bfloat162 v;
    v.x = b0;
    v.y = b1;
    *reinterpret_cast<__nv_bfloat162 *>(dst + umma::kmajor_offset(n, i0)) = v;
  }
}

// B operands of head j: the three bf16 terms of w_i x_i[r] as P x 16
// K-slabs, written by the head group's WPH warps (gt = thread in group).
template <int P, typename TI>
__device__ __forceinline__ void build_fold_b(unsigned char *dst, const TI *xj, const float *wj,
                                             int k, int gt, int gthreads) {
  for (int e = gt; e < P * 8; e += gthreads) {
    const int r = e % P, q = e / P, i0 = 2 * q;
    const float v0 = i0 < k ? wj[i0] * to_f32(xj[i0 * P + r]) : 0.f;
    const float v1 = i0 + 1 < k ? wj[i0 + 1] * to_f32(xj[(i0 + 1) * P + r]) : 0.f;
    __nv_bfloat162 h, m, l;
    umma::split3_bf16(v0, h.x, m.x, l.x);
    umma::split3_bf16(v1, h.y, m.y, l.y);
    const uint32_t o = umma::kmajor_offset(r, i0);
    *reinterpret_cast<__nv_bfloat162 *>(dst + o) = h;
    *reinterpret_cast<__nv_bfloat162 *>(dst + P * 32 + o) = m;
    *reinterpret_cast<__nv_bfloat162 *>(dst + 2 * P * 32 + o) = l;
  }
}

// Epilogue of head bh's fold by the WPH warps of one head group (`sub` = warp
// in group): the new checkpoint, and for a read copy its new codes.  The old
// tile comes from the ring slot (QM 0) or, with a read copy in the slot, from
// the fp32 checkpoint in global memory.  FP8 codes are written with the new
// values; NVFP4 first agrees on the tile maximum over the group (`red` = the
// group's 8 maxima), then forms the codes from the rows the group just stored
// (re-read after named barrier 2 + hq, while they are in L2) in the row
// layout of the output dots, four values per lane, so a 16-column block spans
// four lanes.
template <int P, int N, int QM, int WPH>
__device__ __forceinline__ void fold_epilogue(const M2Params &p, size_t bh, const float *tile,
                                              float lam, uint32_t tcol, int sub, int lane,
                                              float *red, int hq) {
  static_assert(N == 128, "tensor-memory lanes are the 128 state columns");
  constexpr int NW = WPH / 4;  // warps sharing one tensor-memory lane quarter
  constexpr int CW = P / NW;   // checkpoint rows per warp
  const int n = 32 * (sub & 3) + lane, r0 = (sub >> 2) * CW;
  const uint32_t taddr = tcol + ((uint32_t)(32 * (sub & 3)) << 16) + (uint32_t)r0;
  float *hg = p.h0 + bh * (size_t)(P * N);
  float amax = 0.f;
#pragma unroll 1
  for (int c = 0; c < CW; c += 32) {
    // all 32 old values first: the stores below (the byte stores of the copy
    // may alias anything) would otherwise serialise every load behind them
    float t[32], d[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = r0 + c + i;
      t[i] = QM == 0 ? tile[r * N + n] : __ldcs(hg + r * N + n);
    }
    umma::ld32(taddr + c, d);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int r = r0 + c + i;
      const float hn = fmaf(lam, t[i], d[i]);
      __stcs(hg + r * N + n, hn);
      if constexpr (QM == 1) p.rc[bh * (size_t)(P * N) + r * N + n] = (uint8_t)e4m3_encode(hn);
      if constexpr (QM == 2) amax = fmaxf(amax, fabsf(hn));
    }
  }
  if constexpr (QM == 2) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red[sub] = amax;
    bar_sync(2 + hq, WPH * 32);  // also orders the group's h0 stores before the re-reads
    float tmax = red[0];
    for (int w2 = 1; w2 < WPH; ++w2) tmax = fmaxf(tmax, red[w2]);
    const float sg = nvfp4_tile_scale(tmax);
    // codes from the rows just stored (L2-resident), in the row layout of the
    // output dots: lane (rs, c8) takes four consecutive columns of a row, so
    // a 16-column block spans four lanes
    constexpr int RW = P / WPH, RG = RW / 4;
    const int rs = lane >> 3, c8 = lane & 7;
    for (int g4 = 0; g4 < RG; ++g4) {
      const int r = sub * RW + 4 * g4 + rs;
      float4 v[N / 32];
      load_row<N>(hg, r, c8, v);
      nvfp4_row<P, N>(v, sg, false, p.rc + bh * (size_t)(P * N / 2),
                      p.rc_scale + bh * (size_t)(P * N / 16), r, c8);
    }
    if (sub == 0 && lane == 0) p.rc_gscale[bh] = sg;
    bar_sync(2 + hq, WPH * 32);  // red[] is reused by the group's next head
  }
}

constexpr int kDecodeThreads = kThreads + 64;  // 8 consumer warps, tile producer, stager

template <int P, int N, typename TI, int QM, int WPH, bool MMA>
__global__ void __launch_bounds__(kDecodeThreads, 1) m2_decode_kernel(const M2Params p,
                                                                  const DecodeLayout lay) {
  using T = Tile<P, N>;
  constexpr int C4 = T::C4;
  constexpr bool kReadCopy = (QM == 1 || QM == 2);
  static_assert(!MMA || (N == 128 && QM <= 2 && std::is_same<TI, __nv_bfloat16>::value),
                "tensor-core fold: bf16 records, 128 state columns, fp32 or read-copy checkpoint");
  constexpr int HPQ = 8 / WPH;  // heads in flight (one head group each)
  constexpr uint32_t kTmemCols = MMA ? (HPQ * P <= 128 ? 128 : 256) : 0;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  const DecodeSmemPtrs S(smem, lay);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, rs = lane >> 3, c8 = lane & 7;
  const int hc = lay.hc, nchunk = p.hpg / hc;
  const int nitems = p.B * p.G * nchunk;
  const int L = lay.L;

  if (tid == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], WPH);  // consumer warps reading each tile
    }
    for (int r = 0; r < 4; ++r) {
      mbar_init(&S.rfull[r], 1);
      mbar_init(&S.rempty[r], 8);
    }
    mbar_init(&S.mma[0], 1);
    mbar_init(&S.mma[1], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if constexpr (MMA) {
    if (warp == 0) umma::alloc(S.tmem_slot, kTmemCols);
    umma::fence_before_sync();
  }
  __syncthreads();
  if (warp == 8) {
    if (lane == 0) decode_tiles<P, N, QM>(p, lay, S, abort_flag, nitems, nchunk);
    return;
  }
  if (warp == 9) {
    decode_stager<P, N, TI>(p, lay, S, abort_flag, nitems, nchunk, lane);
    return;
  }

  // Consumers.  Control flow stays uniform across the 256 consumer threads:
  // every branch depends only on values read from shared memory after the
  // same barrier or on bar.red.or results, and a thread whose bounded wait
  // ran out keeps going through every barrier (its data is garbage, the
  // status word says so) until the next item boundary, where all consumers
  // leave together.
  //
  // Heads are processed HPQ = 8 / WPH at a time (one ring slot each, the rest
  // of the ring keeps loading ahead), WPH warps per head; a warp owns
  // RW = P / WPH rows of the tile, RG = RW / 4 row groups (quarter-warp rs
  // takes row 4g + rs, lane c8 columns 32s + 4c8).  A warp first pulls its
  // rows into registers (then the slot is released), so the outputs and the
  // fold run while the producer already refills the slot.
  constexpr int RW = P / WPH, RG = RW / 4;
  constexpr int RGC = RG < 4 ? RG : 4;  // row groups held in registers at once
  const int hq = warp / WPH, sub = warp - hq * WPH, gt = tid - hq * WPH * 32;
  uint32_t tmem = 0, n_mma = 0;  // tensor-memory base; fold MMA batches this group committed
  if constexpr (MMA) {
    umma::fence_after_sync();
    tmem = *S.tmem_slot;
  }
  unsigned char *umma_a = S.umma, *umma_b = S.umma + N * 32 + hq * lay.umma_b_bytes;
  int it = 0;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
    const int rb = it % lay.NR;
    const uint32_t rphase = (it / lay.NR) & 1;
    float *scr = S.scr + (it & 1) * lay.scratch_floats;
    double *bc = reinterpret_cast<double *>(scr);  // B_i.C_k, fp64
    float *wdt = scr + 2 * pad4(L);
    float *lam = wdt + pad4(hc * L);
    float *red = lam + pad4(hc);
    float *Bf = red + 32;  // fp32 copy of the group's B records [k][N] (SIMT fold only)
    float *z = Bf + (MMA ? 0 : L * N);  // buffered-record and skip terms of y [hc][P]
    int b, g, chunk, h_first;
    item_coords(p, item, nchunk, hc, b, g, chunk, h_first);
    const size_t bh0 = (size_t)b * p.H + h_first;
    const Stage st(S.stage + rb * lay.stage_floats, N, hc, L);
    const TI *rB = reinterpret_cast<const TI *>(S.recB) + (size_t)rb * L * N;
    const TI *rX = reinterpret_cast<const TI *>(S.recX) + (size_t)rb * hc * L * P;

    const bool got = mbar_wait(&S.rfull[rb], rphase, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(1, kThreads, !got || *abort_flag)) break;  // uniform exit
    const int n0 = st.hdr[0];
    if (st.hdr[1]) {  // uniform: every consumer reads the same staged header
      if (tid == 0) report(p.status, RSSM_ERR_STATE);
      // skip the item, keeping the ring in step with the producer
      for (int q0 = 0; q0 < hc; q0 += HPQ) {
        const uint32_t pos = (uint32_t)it * hc + q0 + hq;
        if (!mbar_wait(&S.full[pos % lay.NS], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
          if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[pos % lay.NS]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.rempty[rb]);
      continue;
    }
    const int k = n0 + 1;
    const bool flush = (k == L);

    // ---- append this step's record to the global buffer (a flush empties
    // the buffer, so its record is not kept; an in-place step's record is
    // already there); one CTA per group writes B, C
    if (!flush && !p.inplace) {
      const size_t bg = (size_t)b * p.G + g;
      if (chunk == 0) {
        for (int n = tid; n < N; n += kThreads) {
          static_cast<TI *>(p.Bbuf)[(bg * p.cap + k - 1) * N + n] = rB[(k - 1) * N + n];
          static_cast<TI *>(p.Cbuf)[(bg * p.cap + k - 1) * N + n] = from_f32<TI>(st.C[n]);
        }
      }
      for (int e = tid; e < hc * P; e += kThreads) {
        const int j = e / P, q = e - j * P;
        static_cast<TI *>(p.xbuf)[((bh0 + j) * p.cap + k - 1) * P + q] = rX[(j * L + k - 1) * P + q];
      }
      if (tid < hc) p.dtbuf[(bh0 + tid) * p.cap + k - 1] = st.dt[tid * L + k - 1];
    }
    // ---- the fold's B operand (fp32 records, or the MMA's A operand), B_i.C_k
    // dots, decay weights
    if constexpr (MMA) {
      if (flush) {
        build_fold_a<N, TI>(umma_a, rB, k, tid);
        fence_proxy_async_smem();  // visible to the tensor cores after the barrier below
      }
    } else if (flush) {
      for (int e = tid; e < k * N; e += kThreads) Bf[e] = to_f32(rB[e]);
    }
    {
      // 16 threads per record, fp64 (these dots of N rounded products would
      // otherwise dominate the output error when the inputs are fp32); the
      // loop bound is the same for every thread so that all 32 lanes of each
      // warp reach the full-mask shuffles
      constexpr int PER = N / 16;
      for (int base = 0; base < k; base += kThreads / 16) {
        const int i = base + (tid >> 4), c0 = (tid & 15) * PER;
        double acc = 0.0;
        if (i < k) {
#pragma unroll
          for (int e = 0; e < PER; ++e)
            acc = fma((double)to_f32(rB[i * N + c0 + e]), (double)st.C[c0 + e], acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        if (i < k && (tid & 15) == 0) bc[i] = acc;
      }
    }
    for (int j = warp; j < hc; j += 8)
      decay_weights_scan(st.dt + j * L, k, st.A[j], wdt + j * L, lam + j, lane);
    bar_sync(1, kThreads);
    // everything of y but the checkpoint term, per row:
    //   z[j][r] = sum_i w_i (B_i . C_k) x_i[r] + D x_k[r]
    // (threads run along r, so the record reads are conflict-free)
    for (int e = tid; e < hc * P; e += kThreads) {
      const int j = e / P, r = e - j * P;
      const TI *xr = rX + j * L * P + r;
      float acc = 0.f;
      for (int i = 0; i < k; ++i)
        acc = fmaf((float)((double)wdt[j * L + i] * bc[i]), to_f32(xr[i * P]), acc);
      z[e] = fmaf(st.D[j], to_f32(xr[(k - 1) * P]), acc);
    }
    bar_sync(1, kThreads);

    float4 c4[C4];
#pragma unroll
    for (int s = 0; s < C4; ++s) c4[s] = *reinterpret_cast<const float4 *>(&st.C[T::col(c8, s)]);

    // ---- heads: HPQ at a time, WPH warps each, row groups of 4 rows
    for (int q0 = 0; q0 < hc; q0 += HPQ) {
      const int j = q0 + hq, h = h_first + j;
      const size_t bh = bh0 + j;
      const uint32_t pos = (uint32_t)it * hc + j;  // producer's issue order
      const int sl = pos % lay.NS;
      const bool mma_fold = MMA && flush;
      if (mma_fold) {
        // this head's fold increment on the tensor cores, issued before its
        // tile arrives; the group's previous epilogue has finished reading
        // the accumulator columns (tensor-memory loads waited, fence, barrier)
        build_fold_b<P, TI>(umma_b, rX + j * L * P, wdt + j * L, k, gt, WPH * 32);
        fence_proxy_async_smem();
        umma::fence_before_sync();
        bar_sync(4 + hq, WPH * 32);
        if (gt == 0) {
          umma::fence_after_sync();
          const uint32_t id = umma::idesc_bf16_f32(128, P);
          const uint64_t ad = umma::smem_desc(umma_a);
#pragma unroll
          for (int t3 = 0; t3 < 3; ++t3)
            umma::mma_bf16(tmem + hq * P, ad, umma::smem_desc(umma_b + t3 * P * 32), id, t3 > 0);
          umma::commit(&S.mma[hq]);
        }
      }
      if (!mbar_wait(&S.full[sl], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      const unsigned char *t = S.ring + sl * lay.tile_stride;
      const float sg = QM == 2 ? p.rc_gscale[bh] : 1.0f;
      const float lm = lam[j];
      const float *wj = wdt + j * L, *zj = z + j * P;
      const TI *xj = rX + j * L * P;
      float *yout = p.y + b * p.bs_y + (size_t)h * P;
      float *tile = p.h0 + bh * (size_t)(P * N);
      float amax = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < RG; c0 += RGC) {
        float4 v[RGC][C4];
#pragma unroll
        for (int u = 0; u < RGC; ++u) view_row<P, N, QM>(t, sub * RW + 4 * (c0 + u) + rs, c8, v[u]);
        // all of this warp's rows are in registers: release the slot (the
        // tensor-core fold of an fp32 tile still reads it in its epilogue)
        if (c0 + RGC == RG && !(mma_fold && QM == 0)) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.empty[sl]);
        }
        int rows[RGC];
#pragma unroll
        for (int u = 0; u < RGC; ++u) rows[u] = sub * RW + 4 * (c0 + u) + rs;
#pragma unroll
        for (int u = 0; u < RGC; ++u) {
          float a = sum8(tree_dot<C4>(v[u], c4));
          if constexpr (QM == 2) a *= sg;  // the NVFP4 view leaves the tile scale out
          if (c8 == 0) yout[rows[u]] = fmaf(lm, a, zj[rows[u]]);
        }
        if (flush && !MMA) {
          if constexpr (kReadCopy) {
#pragma unroll
            for (int u = 0; u < RGC; ++u) load_row<N>(tile, rows[u], c8, v[u]);
          }
          fold_rows<P, N, TI, RGC>(v, lm, k, wj, xj, rows, Bf, c8);
#pragma unroll
          for (int u = 0; u < RGC; ++u) {
            if constexpr (QM == 3) fp8_roundtrip_row<N>(v[u]);
            store_row<N>(tile, rows[u], c8, v[u]);
            if constexpr (QM == 1) fp8_codes_row<N>(p.rc + bh * (size_t)(P * N), rows[u], c8, v[u]);
            if constexpr (QM == 2 || QM == 4) amax = fmaxf(amax, absmax_row<N>(v[u]));
          }
        }
      }
      if constexpr (MMA) {
        if (mma_fold) {
          const bool done = mbar_wait(&S.mma[hq], n_mma & 1u, p.wait_ns, abort_flag);
          ++n_mma;
          if (!done) {
            if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
            *abort_flag = 1;
          }
          umma::fence_after_sync();
          fold_epilogue<P, N, QM, WPH>(p, bh, reinterpret_cast<const float *>(t), lm,
                                       tmem + hq * P, sub, lane, red + 8 * hq, hq);
          umma::fence_before_sync();
          if constexpr (QM == 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[sl]);
          }
        }
      }
      if constexpr ((QM == 2 || QM == 4) && !MMA) {
        if (flush) {
          // NVFP4 needs the whole tile's maximum: combine the WPH warps of
          // this head, then requantise the rows just written (each thread
          // rereads exactly the elements it stored)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
          if (lane == 0) red[hq * 8 + sub] = amax;
          bar_sync(2 + hq, WPH * 32);
          float tmax = 0.f;
          for (int w2 = 0; w2 < WPH; ++w2) tmax = fmaxf(tmax, red[hq * 8 + w2]);
          const float sgn = nvfp4_tile_scale(tmax);
          for (int g4 = 0; g4 < RG; ++g4) {
            const int r = sub * RW + 4 * g4 + rs;
            float4 v[C4];
            load_row<N>(tile, r, c8, v);
            nvfp4_row<P, N>(v, sgn, QM == 4, p.rc + bh * (size_t)(P * N / 2),
                            p.rc_scale + bh * (size_t)(P * N / 16), r, c8);
            if constexpr (QM == 4) store_row<N>(tile, r, c8, v);
          }
          if constexpr (QM == 2)
            if (sub == 0 && lane == 0) p.rc_gscale[bh] = sgn;
          bar_sync(2 + hq, WPH * 32);  // red[] of this head is reused next round
        }
      }
    }
    // the producer refills this record buffer next: order our reads of it
    // (generic proxy) before its bulk copies (async proxy)
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.rempty[rb]);
    if (tid < hc) p.len[bh0 + tid] = flush ? 0 : k;
  }
  if constexpr (MMA) {
    // every fold MMA has completed before the tensor memory is released (a
    // group that stopped early may not have waited for its last batch)
    if (gt == 0 && n_mma > 0) mbar_wait(&S.mma[hq], (n_mma - 1) & 1u);
    umma::fence_before_sync();
    bar_sync(1, kThreads);
    umma::fence_after_sync();
    if (warp == 0) umma::dealloc(tmem, kTmemCols);
  }
}

// ====================================================== fold-only kernels
// MODE kFoldFlush:       fold where len >= L (or len > 0 with force)
// MODE kFoldCommit:      len += acc[b]; fold where len >= L
// MODE kFoldMaterialize: S_out = fold(h0, records), state untouched

template <int P, int N, typename TI, int QM, int MODE>
__global__ void __launch_bounds__(kThreads, 2) m2_fold_kernel(const M2Params p) {
  using T = Tile<P, N>;
  constexpr int RPT = T::RPT, C4 = T::C4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, rs = lane >> 3, c8 = lane & 7;
  const int hc = head_chunk(p.hpg), nchunk = p.hpg / hc;
  const int bg_i = blockIdx.x / nchunk, chunk = blockIdx.x - bg_i * nchunk;
  const int b = bg_i / p.G, g = bg_i - b * p.G;
  const int h_first = g * p.hpg + chunk * hc;
  const size_t bh0 = (size_t)b * p.H + h_first;
  const int LC = p.cap;  // records here may exceed the window after a verify round
  DecodeSmem S(smem_raw, LC, hc, N);
  TI *s_x = static_cast<TI *>(S.x);

  const int n0 = p.len[bh0];
  bool bad = false;
  if (tid > 0 && tid < hc) bad = p.len[bh0 + tid] != n0;
  int n = n0, act = 0;
  if (MODE == kFoldCommit) {
    const int a = p.acc[b];
    if (tid == 0) bad = n0 < 0 || n0 >= p.L || a < 0 || a > p.draft_max || n0 + a > p.cap;
    n = n0 + a;
    act = n >= p.L;
  } else {
    if (tid == 0) bad = n0 < 0 || n0 > p.cap;
    act = MODE == kFoldMaterialize ? 1 : (n0 >= p.L || (p.force && n0 > 0));
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) report(p.status, RSSM_ERR_STATE);
    return;
  }
  if (!act) {
    if (MODE == kFoldCommit && tid < hc) p.len[bh0 + tid] = n;
    return;
  }
  const size_t bg = (size_t)b * p.G + g;
  stage_f32<TI>(S.B, static_cast<const TI *>(p.Bbuf) + bg * p.cap * N, n * N, tid);
  for (int j = 0; j < hc; ++j)
    stage_raw(s_x + j * LC * P, static_cast<const TI *>(p.xbuf) + (bh0 + j) * p.cap * P,
              n * P * (int)sizeof(TI), tid);
  for (int e = tid; e < hc * n; e += kThreads) {
    const int j = e / n, i = e - j * n;
    S.dt[j * LC + i] = p.dtbuf[(bh0 + j) * p.cap + i];
  }
  __syncthreads();
  for (int j = warp; j < hc; j += 8)
    decay_weights(S.dt + j * LC, n, p.A[h_first + j], S.wdt + j * LC, S.lam + j, lane);
  __syncthreads();
  for (int j = 0; j < hc; ++j) {
    const size_t bh = bh0 + j;
    float *tile = p.h0 + bh * (size_t)(P * N);
    float4 hv[RPT][C4];
    load_tile<P, N>(tile, warp, rs, c8, hv);
    fold_regs<P, N, TI>(hv, S.lam[j], n, S.wdt + j * LC, s_x + j * LC * P, S.B, warp, rs, c8);
    if constexpr (MODE == kFoldMaterialize) {
      store_tile<P, N>(p.S_out + bh * (size_t)(P * N), warp, rs, c8, hv);
    } else {
      commit_checkpoint<P, N, QM>(p, bh, tile, hv, S.red + 8 * (j & 1), warp, lane, rs, c8);
    }
  }
  if (MODE != kFoldMaterialize && tid < hc) p.len[bh0 + tid] = 0;
}

// ================================================ conventional full step
// S <- exp(dt A) S + dt x B^T ; y = S C + D x, in place, every step.

template <int P, int N, typename TI>
__global__ void __launch_bounds__(kThreads, 2) m2_full_kernel(const M2Params p) {
  using T = Tile<P, N>;
  constexpr int RPT = T::RPT, C4 = T::C4;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, rs = lane >> 3, c8 = lane & 7;
  const int b = blockIdx.x / p.G, g = blockIdx.x - b * p.G;
  if (p.limit && p.step_index >= p.limit[b]) return;
  const int h_first = g * p.hpg;
  const TI *Bin = static_cast<const TI *>(p.Bm) + b * p.bs_B + (size_t)g * N;
  const TI *Cin = static_cast<const TI *>(p.Cm) + b * p.bs_C + (size_t)g * N;
  float4 b4[C4], c4[C4];
#pragma unroll
  for (int s = 0; s < C4; ++s) {
    const int c = T::col(c8, s);
    b4[s] = make_float4(to_f32(Bin[c]), to_f32(Bin[c + 1]), to_f32(Bin[c + 2]), to_f32(Bin[c + 3]));
    c4[s] = make_float4(to_f32(Cin[c]), to_f32(Cin[c + 1]), to_f32(Cin[c + 2]), to_f32(Cin[c + 3]));
  }
  for (int j = 0; j < p.hpg; ++j) {
    const int h = h_first + j;
    const size_t bh = (size_t)b * p.H + h;
    float *tile = p.S + bh * (size_t)(P * N);
    float4 sv[RPT][C4];
    load_tile<P, N>(tile, warp, rs, c8, sv);
    const float dt = ld_in<TI>(p.dt, b * p.bs_dt + h);
    const float dA = expf(dt * p.A[h]);
    const float Dh = p.D[h];
    const TI *xin = static_cast<const TI *>(p.x) + b * p.bs_x + (size_t)h * P;
    float *yout = p.y + b * p.bs_y + (size_t)h * P;
#pragma unroll
    for (int rho = 0; rho < RPT; ++rho) {
      const int r = T::row(warp, rs, rho);
      const float xr = to_f32(xin[r]);
      const float u = dt * xr;
      float acc = 0.f;
#pragma unroll
      for (int s = 0; s < C4; ++s) {
        float4 &a = sv[rho][s];
        a.x = fmaf(u, b4[s].x, dA * a.x);
        a.y = fmaf(u, b4[s].y, dA * a.y);
        a.z = fmaf(u, b4[s].z, dA * a.z);
        a.w = fmaf(u, b4[s].w, dA * a.w);
        acc += dot4(a, c4[s]);
      }
      acc = sum8(acc);
      if (c8 == 0) yout[r] = fmaf(Dh, xr, acc);
    }
    store_tile<P, N>(tile, warp, rs, c8, sv);
  }
}

// ================================================================= launchers

template <typename K>
cudaError_t launch_dyn(K kernel, unsigned grid, size_t smem, cudaStream_t s, const M2Params &p) {
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  kernel<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}


// Heads per decode work item: the whole group up to 8 heads, else chunks of 8
// (per-item setup is amortised over as many heads as the ring allows).
__host__ __forceinline__ int decode_chunk(int hpg) {
  // a power of two (1, 2, 4 or 8) dividing the group: the consumer warps split
  // evenly over the heads in flight
  for (int c = 8; c > 1; c >>= 1)
    if (hpg % c == 0) return c;
  return 1;
}

template <typename K>
cudaError_t launch_decode(K kernel, const M2Params &p, const DecodeLayout &lay, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
  if (e != cudaSuccess) return e;
  const int nitems = p.B * p.G * (p.hpg / lay.hc);
  const int grid = nitems < sm_count() ? nitems : sm_count();
  kernel<<<grid, kDecodeThreads, lay.total, s>>>(p, lay);
  return cudaGetLastError();
}

template <int P, int N, typename TI, int WPH>
cudaError_t decode_wph(const M2Params &p, const DecodeLayout &lay, bool mma, cudaStream_t s) {
  if constexpr (N == 128 && std::is_same<TI, __nv_bfloat16>::value) {
    if (mma) {
      switch (p.qmode) {
        case 0: return launch_decode(m2_decode_kernel<P, N, TI, 0, WPH, true>, p, lay, s);
        case 1: return launch_decode(m2_decode_kernel<P, N, TI, 1, WPH, true>, p, lay, s);
        case 2: return launch_decode(m2_decode_kernel<P, N, TI, 2, WPH, true>, p, lay, s);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  switch (p.qmode) {
    case 0: return launch_decode(m2_decode_kernel<P, N, TI, 0, WPH, false>, p, lay, s);
    case 1: return launch_decode(m2_decode_kernel<P, N, TI, 1, WPH, false>, p, lay, s);
    case 2: return launch_decode(m2_decode_kernel<P, N, TI, 2, WPH, false>, p, lay, s);
    case 3: return launch_decode(m2_decode_kernel<P, N, TI, 3, WPH, false>, p, lay, s);
    case 4: return launch_decode(m2_decode_kernel<P, N, TI, 4, WPH, false>, p, lay, s);
    default: return cudaErrorInvalidValue;
  }
}

// The flush fold runs on the tensor cores for bf16 records, 128 state
// columns and an fp32 checkpoint (with or without a read copy), when the
// operand areas fit beside the ring; otherwise, and for fp32 inputs (whose
// records are not exact in bf16) or a quantised checkpoint, on the SIMT pipes.
template <int P, int N, typename TI>
cudaError_t decode_qm(const M2Params &p, cudaStream_t s) {
  const int hc = decode_chunk(p.hpg);
  const int hpq = hc >= 2 ? 2 : 1;  // two heads in flight (4 warps each) when possible
  const int es = (int)sizeof(TI);
  DecodeLayout lay{};
  bool mma = N == 128 && std::is_same<TI, __nv_bfloat16>::value && p.qmode <= 2;
  if (mma) {
    lay = DecodeLayout::make(P, N, hc, p.L, es, p.qmode, 220 * 1024, true, hpq);
    if (lay.NS < 2) mma = false;
  }
  if (!mma) lay = DecodeLayout::make(P, N, hc, p.L, es, p.qmode, 220 * 1024);
  if (lay.NS < 2) return cudaErrorInvalidConfiguration;
  return hpq == 2 ? decode_wph<P, N, TI, 4>(p, lay, mma, s) : decode_wph<P, N, TI, 8>(p, lay, mma, s);
}

template <int P, int N, typename TI, int MODE>
cudaError_t fold_qm(const M2Params &p, cudaStream_t s) {
  const int hc = head_chunk(p.hpg);
  const unsigned grid = (unsigned)(p.B * p.G * (p.hpg / hc));
  const size_t smem = DecodeSmem::bytes(p.cap, hc, P, N, sizeof(TI));
  switch (MODE == kFoldMaterialize ? 0 : p.qmode) {
    case 0: return launch_dyn(m2_fold_kernel<P, N, TI, 0, MODE>, grid, smem, s, p);
    case 1: return launch_dyn(m2_fold_kernel<P, N, TI, 1, MODE>, grid, smem, s, p);
    case 2: return launch_dyn(m2_fold_kernel<P, N, TI, 2, MODE>, grid, smem, s, p);
    case 3: return launch_dyn(m2_fold_kernel<P, N, TI, 3, MODE>, grid, smem, s, p);
    case 4: return launch_dyn(m2_fold_kernel<P, N, TI, 4, MODE>, grid, smem, s, p);
    default: return cudaErrorInvalidValue;
  }
}

template <int P, int N, typename TI>
cudaError_t fold_mode(const M2Params &p, int mode, cudaStream_t s) {
  switch (mode) {
    case kFoldFlush: return fold_qm<P, N, TI, kFoldFlush>(p, s);
    case kFoldCommit: return fold_qm<P, N, TI, kFoldCommit>(p, s);
    case kFoldMaterialize: return fold_qm<P, N, TI, kFoldMaterialize>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool m2_supported(int P, int N) { return (P == 64 || P == 128) && (N == 64 || N == 128); }

bool m2_heads_supported(int hpg) { return hpg <= 8 || hpg % 8 == 0; }

cudaError_t m2_launch_decode(const M2Params &p, cudaStream_t s) {
  if (p.B * p.G == 0) return cudaSuccess;
  return dispatch_shape(p.P, p.N, p.in_bf16, [&](auto PP, auto NN, auto ti) {
    return decode_qm<decltype(PP)::value, decltype(NN)::value, decltype(ti)>(p, s);
  });
}

cudaError_t m2_launch_fold(const M2Params &p, int mode, cudaStream_t s) {
  if (p.B * p.G == 0) return cudaSuccess;
  return dispatch_shape(p.P, p.N, p.in_bf16, [&](auto PP, auto NN, auto ti) {
    return fold_mode<decltype(PP)::value, decltype(NN)::value, decltype(ti)>(p, mode, s);
  });
}

cudaError_t m2_launch_full(const M2Params &p, cudaStream_t s) {
  if (p.B * p.G == 0) return cudaSuccess;
  return dispatch_shape(p.P, p.N, p.in_bf16, [&](auto PP, auto NN, auto ti) {
    m2_full_kernel<decltype(PP)::value, decltype(NN)::value, decltype(ti)>
        <<<(unsigned)(p.B * p.G), kThreads, 0, s>>>(p);
    return cudaGetLastError();
  });
}


}  // namespace rssm
