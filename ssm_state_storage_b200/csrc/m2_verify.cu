// m2_verify.cu -- Mamba-2 speculative verify round for sm_100a: commit of the
// previous round's accepted drafts (fold when the buffer reaches the window),
// append of the new drafts, and every draft's output from the checkpoint and
// the buffer with no intermediate state.
// [sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…", §Speculative decoding:
// drafts enter the buffer, their outputs are evaluated with no per-draft state,
// and the accepted prefix is committed]
#include "m2_device.cuh"

namespace rssm {
namespace {

// ============================================================ verify round
// Persistent speculative-verify kernel, structured like the decode kernel.
// Work item = (sequence, group, chunk) with hc = (H/G)/nchunk heads; nchunk
// is 1 unless the staged records of all the group's heads do not fit in
// shared memory beside the tile ring.  Per item:
//   1. commit of the previous round: n1 = len + accepted; when n1 >= window
//      the n1 buffered records are folded into h0 (written once) and the
//      drafts follow an empty buffer (nb = 0), else nb = n1;
//   2. the nd drafts are appended to slots nb .. nb+nd-1 (len stays nb);
//   3. draft d's output from the (possibly folded) checkpoint and records
//      0..nb+d, with no intermediate state:
//        y_d = Lam_d (h C_d) + sum_i w_{d,i} (B_i . C_d) x_i + D x_d.
// The stager (warp 9) reads the lengths and acceptance counts, loads the
// small inputs, and bulk-copies the buffered prefix records and the draft
// rows (x, B, C); warp 8 streams the heads' checkpoint tiles; warps 0-7 form
// the fold weights, every draft's decay weights and B.C dots (fp64) and the
// per-row terms z_d, then take one head at a time (8 warps, 8 rows each):
// rows into registers, slot released, optional fold + write-back, and all
// nd outputs from the same registers.
// With nchunk > 1 the draft B and C rows (one copy per group) are appended
// by m2_verify_append_bc_kernel after this kernel: a chunk that folds would
// otherwise overwrite buffered B records that another chunk's CTA may not
// have copied yet.

constexpr int kMD = 4;  // most drafts per round
// Consumer warps form kVGroups groups that take alternate items (with two
// groups one group's per-item setup overlaps the other's tile streaming; on
// B200 that measured no faster than one group of 16 warps, which is used).
constexpr int kVGroups = 1, kGWarps = 16, kGThreads = 32 * kGWarps;
constexpr int kVWarps = kVGroups * kGWarps, kVThreads = 32 * kVWarps;

struct VerifyLayout {
  int NS, NR, hc, nchunk, cap, L, tile_bytes, tile_stride;
  int rec_floats, db_floats;  // stage floats per record buffer, scratch per item
  int off_bars, off_recB, off_recX, off_dX, off_dB, off_dC, off_rec, off_scr, off_ring, total;
  int db_b, scr_b;  // per consumer group: item scratch bytes, all scratch bytes
  int recB_b, recX_b, dX_b, dBC_b;  // bytes per record buffer of each array
  __host__ static int a128(int v) { return (v + 127) & ~127; }
  __host__ static VerifyLayout make(int P, int N, int hpg, int nchunk, int cap, int L, int es,
                                    int budget) {
    VerifyLayout d;
    d.nchunk = nchunk;
    const int hc = d.hc = hpg / nchunk;
    d.cap = cap;
    d.L = L;
    d.tile_bytes = P * N * 4;
    d.tile_stride = a128(d.tile_bytes);
    d.recB_b = a128(cap * N * es);
    d.recX_b = a128(hc * cap * P * es);
    d.dX_b = a128(kMD * hc * P * es);
    d.dBC_b = a128(kMD * N * es);
    // stage: dt prefix [hc][cap] | dt drafts [4][hc] | A [hc] | D [hc] | hdr [8]
    d.rec_floats = pad4(hc * cap) + kMD * hc + pad4(hc) * 2 + 8;
    // per item: Bf [cap][N] | wf [hc][cap] | lamf [hc] | lamd [4][hc] | z [4][hc][P]
    d.db_floats = cap * N + pad4(hc * cap) + pad4(hc) + kMD * hc + kMD * hc * P;
    for (d.NR = 2; d.NR >= 1; --d.NR) {
      int o = 0;
      d.off_bars = o;
      o += 256;
      d.off_recB = o;
      o += d.NR * d.recB_b;
      d.off_recX = o;
      o += d.NR * d.recX_b;
      d.off_dX = o;
      o += d.NR * d.dX_b;
      d.off_dB = o;
      o += d.NR * d.dBC_b;
      d.off_dC = o;
      o += d.NR * d.dBC_b;
      d.off_rec = o;
      o += a128(d.NR * d.rec_floats * 4);
      // per consumer group: item scratch | bc [4][cap+4] double | wd [4][hc][cap+4] double
      d.off_scr = o;
      d.db_b = a128(d.db_floats * 4);
      d.scr_b = d.db_b + a128(kMD * (cap + kMD) * 8 + kMD * hc * (cap + kMD) * 8);
      o += kVGroups * d.scr_b;
      d.off_ring = o;
      d.NS = (budget - o) / d.tile_stride;
      if (d.NS > 8) d.NS = 8;
      if (d.NS >= 2) {
        d.total = o + d.NS * d.tile_stride;
        return d;
      }
    }
    d.NS = 0;
    return d;
  }
};

template <int P, int N, typename TI>
__device__ __forceinline__ bool verify_stage(const M2Params &p, const VerifyLayout &lay,
                                             unsigned char *smem, uint64_t *rfull,
                                             uint64_t *rempty, int item, int it, int lane,
                                             volatile int *abort_flag) {
  constexpr int DPL = (8 * 20 + 31) / 32;  // prefix dt slots per lane (hc <= 8, cap <= 20)
  const int hc = lay.hc, cap = lay.cap, L = lay.L, nd = p.n_draft;
  const int rb = it % lay.NR;
  const uint32_t rphase = (it / lay.NR) & 1;
  bool ok = true;
  if (lane == 0) ok = mbar_wait(&rempty[rb], rphase ^ 1, kWaitLimitNs, abort_flag) && !*abort_flag;
  if (!__shfl_sync(0xffffffffu, (int)ok, 0)) return false;
  int b, g, chunk, h_first;
  item_coords(p, item, lay.nchunk, hc, b, g, chunk, h_first);
  const size_t bh0 = (size_t)b * p.H + h_first, bg = (size_t)b * p.G + g;

  // ---- loads
  const int my_len = lane < hc ? __ldcg(&p.len[bh0 + lane]) : 0;
  const int a = p.acc ? __ldcg(&p.acc[b]) : 0;
  const float my_A = lane < hc ? p.A[h_first + lane] : 0.f;
  const float my_D = lane < hc ? p.D[h_first + lane] : 0.f;
  float dtv[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int e = lane + 32 * u, j = e / cap, i = e - j * cap;
    dtv[u] = e < hc * cap ? __ldcg(&p.dtbuf[(bh0 + j) * cap + i]) : 0.f;
  }
  const int dd = lane / hc, dj = lane - (lane / hc) * hc;  // draft dt: lane -> (d, j)
  const float my_dtd = lane < nd * hc ? ld_in<TI>(p.dt, b * p.bs_dt + (int64_t)dd * p.H + h_first + dj)
                                      : 0.f;
  // ---- lengths and checks
  const int n0 = __shfl_sync(0xffffffffu, my_len, 0);
  const int n1 = n0 + a;
  const bool fold = n1 >= L;
  const int nb = fold ? 0 : n1;
  const bool bad = __any_sync(0xffffffffu, (lane < hc && my_len != n0)) || n0 < 0 || n0 >= L ||
                   a < 0 || a > p.draft_max || n1 > cap || nb + nd > cap;
  const int n1c = bad ? 0 : n1;  // copies stay in bounds for a bad item
  // ---- shared-memory writes
  float *st = reinterpret_cast<float *>(smem + lay.off_rec) + rb * lay.rec_floats;
  float *dtb = st, *dtd = st + pad4(hc * cap), *As = dtd + kMD * hc, *Ds = As + pad4(hc);
  int *hdr = reinterpret_cast<int *>(Ds + pad4(hc));
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int e = lane + 32 * u;
    if (e < hc * cap) dtb[e] = dtv[u];
  }
  if (lane < nd * hc) dtd[dd * hc + dj] = my_dtd;
  if (lane < hc) {
    As[lane] = my_A;
    Ds[lane] = my_D;
  }
  if (lane == 0) {
    hdr[0] = n0;
    hdr[1] = n1;
    hdr[2] = fold;
    hdr[3] = nb;
    hdr[4] = bad;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    const uint32_t bB = n1c * N * sizeof(TI), bX = n1c * P * sizeof(TI);
    const uint32_t bdX = hc * P * sizeof(TI), bdBC = N * sizeof(TI);
    const uint32_t dcount = bad ? 0 : nd;
    mbar_arrive_expect_tx(&rfull[rb], bB + hc * bX + dcount * (bdX + 2 * bdBC));
    unsigned char *recB = smem + lay.off_recB + rb * lay.recB_b;
    unsigned char *recX = smem + lay.off_recX + rb * lay.recX_b;
    unsigned char *dX = smem + lay.off_dX + rb * lay.dX_b;
    unsigned char *dB = smem + lay.off_dB + rb * lay.dBC_b;
    unsigned char *dC = smem + lay.off_dC + rb * lay.dBC_b;
    if (n1c > 0) {
      bulk_g2s(recB, static_cast<const TI *>(p.Bbuf) + bg * cap * N, bB, &rfull[rb]);
      for (int j = 0; j < hc; ++j)
        bulk_g2s(recX + (size_t)j * cap * P * sizeof(TI),
                 static_cast<const TI *>(p.xbuf) + (bh0 + j) * cap * P, bX, &rfull[rb]);
    }
    for (uint32_t d = 0; d < dcount; ++d) {
      bulk_g2s(dX + d * bdX, static_cast<const TI *>(p.x) + b * p.bs_x + ((size_t)d * p.H + h_first) * P,
               bdX, &rfull[rb]);
      bulk_g2s(dB + d * bdBC, static_cast<const TI *>(p.Bm) + b * p.bs_B + ((size_t)d * p.G + g) * N,
               bdBC, &rfull[rb]);
      bulk_g2s(dC + d * bdBC, static_cast<const TI *>(p.Cm) + b * p.bs_C + ((size_t)d * p.G + g) * N,
               bdBC, &rfull[rb]);
    }
  }
  return true;
}

// Butterfly reduce-scatter over the 16 lanes of a half warp (lane bits 3..0):
// every lane enters with V partial sums, and after log2(16) rounds lane c16
// holds the complete sum of value c16 / (16 / V) (V = 4, 8 or 16).  Each
// round sends half of the remaining values, so V sums cost V - 1 + (4 -
// log2 V) shuffles instead of 4 V.
template <int NV, int M>
struct HalfWarpReduce {
  static __device__ __forceinline__ void run(float *q, int c16) {
    if constexpr (M > 0) {
      if constexpr (NV == 1) {
        q[0] += __shfl_xor_sync(0xffffffffu, q[0], M);
        HalfWarpReduce<1, M / 2>::run(q, c16);
      } else {
        constexpr int H = NV / 2;
        const bool up = c16 & M;
#pragma unroll
        for (int k = 0; k < H; ++k) {
          const float keep = up ? q[H + k] : q[k], send = up ? q[k] : q[H + k];
          q[k] = keep + __shfl_xor_sync(0xffffffffu, send, M);
        }
        HalfWarpReduce<H, M / 2>::run(q, c16);
      }
    }
  }
};

// K consecutive input elements (bf16 or fp32) from shared memory as floats;
// the address is aligned to K elements.
template <typename TI, int K>
__device__ __forceinline__ void ld_vec(const TI *src, float (&out)[K]) {
  if constexpr (std::is_same<TI, float>::value) {
    if constexpr (K == 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src);
      out[0] = v.x, out[1] = v.y, out[2] = v.z, out[3] = v.w;
    } else {
      static_assert(K == 2, "2 or 4 elements");
      const float2 v = *reinterpret_cast<const float2 *>(src);
      out[0] = v.x, out[1] = v.y;
    }
  } else {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(src);
    if constexpr (K == 4) {
      const uint2 u = *reinterpret_cast<const uint2 *>(src);
      const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
      const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
      out[0] = lo.x, out[1] = lo.y, out[2] = hi.x, out[3] = hi.y;
    } else {
      static_assert(K == 2, "2 or 4 elements");
      const float2 v = __bfloat1622float2(h[0]);
      out[0] = v.x, out[1] = v.y;
    }
  }
}

template <typename TI>
__device__ __forceinline__ float4 ld_vec4(const TI *src) {
  float t[4];
  ld_vec<TI, 4>(src, t);
  return make_float4(t[0], t[1], t[2], t[3]);
}


template <int P, int N, typename TI>
__global__ void __maxnreg__(96) m2_verify_kernel(const M2Params p, const VerifyLayout lay) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
  uint64_t *empty = full + 8, *rfull = empty + 8, *rempty = rfull + 4, *turn = rempty + 4;
  unsigned char *ring = smem + lay.off_ring;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hc = lay.hc, cap = lay.cap, nd = p.n_draft, R = cap + kMD;
  const int nitems = p.B * p.G * lay.nchunk;
  const bool own_bc = lay.nchunk == 1;

  if (tid == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGWarps);  // each tile is read by one group
    }
    for (int r = 0; r < 4; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], kGWarps);
    }
    for (int g2 = 0; g2 < kVGroups; ++g2) mbar_init(&turn[g2], kGWarps);
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (warp == kVWarps) {
    if (lane == 0)
      stream_tiles<P, N, 0>(p, full, empty, ring, lay.NS, lay.tile_stride, lay.tile_bytes, hc,
                            abort_flag, nitems, lay.nchunk);
    return;
  }
  if (warp == kVWarps + 1) {
    int it = 0;
    ArmedRecords armed;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
      const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
      if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
      if (abort_now ||
          !verify_stage<P, N, TI>(p, lay, smem, rfull, rempty, item, it, lane, abort_flag)) {
        if (lane == 0 && !*abort_flag) {
          report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      armed.arm(it % lay.NR, (it / lay.NR) & 1);
    }
    if (lane == 0) armed.drain(rfull, lay.NR);  // no record copy outlives the warp
    __syncwarp();
    return;
  }

  // Consumer group grp takes this CTA's items it = grp, grp + 2, ...
  // Head-loop lane layout: a half warp covers one row, lane c16 holds the
  // columns 64 s + 4 c16 .. +3 (s < N/64); a warp owns RW = P/8 rows of
  // every head, taken four at a time (two per half warp).
  constexpr int S4 = N / 64, RW = P / kGWarps, NSP = RW / 4, RZ = P / 32;
  static_assert(NSP >= 1 && S4 >= 1, "headdim and d_state must be at least 64");
  const int grp = warp / kGWarps, gw = warp - grp * kGWarps, gtid = tid - grp * kGThreads;
  const uint32_t gbar = 1 + grp;  // the group's named barrier
  const int h16 = lane >> 4, c16 = lane & 15;
  unsigned char *scr = smem + lay.off_scr + grp * lay.scr_b;
  double *bc = reinterpret_cast<double *>(scr + lay.db_b);  // [4][R]
  double *wd = bc + kMD * R;                                // [4][hc][R] decay weights
  // Ring hand-off: a group starts waiting for its item's first tile only after
  // every warp of the other group has acquired the previous item's last
  // tile (turn[grp]), so a slot is never awaited more than one phase ahead.
  // With a single record buffer the hand-off also precedes the record wait.
  auto take_turn = [&](int it_) -> bool {
    if constexpr (kVGroups == 1) return true;
    if (it_ == 0) return true;
    return mbar_wait(&turn[grp], ((it_ - 1) >> 1) & 1);
  };
  auto pass_turn = [&]() {
    if constexpr (kVGroups > 1) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&turn[grp ^ 1]);
    }
  };
  int it = grp;
  for (int item = blockIdx.x + grp * gridDim.x; item < nitems;
       item += kVGroups * gridDim.x, it += kVGroups) {
    const int rb = it % lay.NR;
    const uint32_t rphase = (it / lay.NR) & 1;
    int b, g, chunk, h_first;
    item_coords(p, item, lay.nchunk, hc, b, g, chunk, h_first);
    const size_t bh0 = (size_t)b * p.H + h_first, bg = (size_t)b * p.G + g;
    const float *st = reinterpret_cast<const float *>(smem + lay.off_rec) + rb * lay.rec_floats;
    const float *dtb = st, *dtd = st + pad4(hc * cap), *As = dtd + kMD * hc, *Ds = As + pad4(hc);
    const int *hdr = reinterpret_cast<const int *>(Ds + pad4(hc));
    const TI *recB = reinterpret_cast<const TI *>(smem + lay.off_recB + rb * lay.recB_b);
    const TI *recX = reinterpret_cast<const TI *>(smem + lay.off_recX + rb * lay.recX_b);
    const TI *dX = reinterpret_cast<const TI *>(smem + lay.off_dX + rb * lay.dX_b);
    const TI *dB = reinterpret_cast<const TI *>(smem + lay.off_dB + rb * lay.dBC_b);
    const TI *dC = reinterpret_cast<const TI *>(smem + lay.off_dC + rb * lay.dBC_b);
    float *db = reinterpret_cast<float *>(scr);
    float *Bf = db, *wf = Bf + cap * N, *lamf = wf + pad4(hc * cap), *lamd = lamf + pad4(hc);
    float *z = lamd + kMD * hc;

    const bool got =
        (lay.NR > 1 || take_turn(it)) && mbar_wait(&rfull[rb], rphase, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(gbar, kGThreads, !got || *abort_flag)) break;
    if (hdr[4]) {
      if (gtid == 0) report(p.status, RSSM_ERR_STATE);
      if (lay.NR > 1 && !take_turn(it)) {
        report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      for (int j = 0; j < hc; ++j) {
        const uint32_t pos = (uint32_t)it * hc + j;
        if (!mbar_wait(&full[pos % lay.NS], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
          if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[pos % lay.NS]);
      }
      pass_turn();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[rb]);
      continue;
    }
    const int n1 = hdr[1], nb = hdr[3], K = nb + nd;
    const bool fold = hdr[2];

    // ---- S1 (warps 8-15): fp32 B for the fold, B_i . C_d in fp64; alongside,
    // S2 (warps 0-7): the decay weights, then the draft appends.
    if (gw >= kGWarps / 2) {
      const int t2 = gtid - kGThreads / 2;
      if (fold)
        for (int e = t2; e < n1 * (N / 4); e += kGThreads / 2)
          reinterpret_cast<float4 *>(Bf)[e] = ld_vec4<TI>(recB + 4 * e);
      const int npair = nd * K;  // (d, i) with i <= nb + d are used
      constexpr int PER = N / 16;
      for (int base = 0; base < npair; base += kGThreads / 32) {
        const int pr = base + (t2 >> 4), c0 = (t2 & 15) * PER;
        const int d = pr / K, i = pr - d * K;
        const bool use = pr < npair && i <= nb + d;
        double acc = 0.0;
        if (use) {
          const TI *Bi = i < nb ? recB + i * N : dB + (i - nb) * N;
#pragma unroll
          for (int e = 0; e < PER; e += 4) {
            const float4 bv = ld_vec4<TI>(Bi + c0 + e), cv = ld_vec4<TI>(dC + d * N + c0 + e);
            acc = fma((double)bv.x, (double)cv.x, acc);
            acc = fma((double)bv.y, (double)cv.y, acc);
            acc = fma((double)bv.z, (double)cv.z, acc);
            acc = fma((double)bv.w, (double)cv.w, acc);
          }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        acc += __shfl_xor_sync(0xffffffffu, acc, 8);
        if (use && (t2 & 15) == 0) bc[d * R + i] = acc;
      }
    } else {
      // ---- S2 (one warp per head): decay weights from fp64 suffix sums.
      // Draft sequence: the nb committed records, then the nd drafts; with
      // S_l = sum_{m >= l} dt_m, draft d (records 0..e, e = nb + d) weighs
      // record i by exp(A (S_{i+1} - S_{e+1})) dt_i and the checkpoint by
      // exp(A (S_0 - S_{e+1})).  Both factor through the reference point
      // S_ref = S_{nb+1}:  exp(A (S_{i+1} - S_ref)) * exp(A (S_ref - S_{e+1})),
      // so one exponential per lane serves every draft: lanes 0..K-1 take
      // E_l = exp(A (S_{l+1} - S_ref)), lanes 27..30 take F_d = exp(A (S_ref -
      // S_{e+1})) and lane 31 takes G = exp(A (S_0 - S_ref)).  No factor can
      // overflow: S_ref - S_{e+1} and the S_{i+1} - S_ref of draft records span
      // at most 4 dt, and every other argument is <= 0.  The fold sequence is
      // the n1 committed records (weights exp(A S'_{l+1}) dt_l, decay
      // exp(A S'_0)); both scans and both exponentials run side by side.
      for (int j = gw; j < hc; j += kGWarps / 2) {
        const double A = As[j];
        const double dts = lane < nb ? (double)dtb[j * cap + lane]
                                     : (lane < K ? (double)dtd[(lane - nb) * hc + j] : 0.0);
        const double dtf = fold && lane < n1 ? (double)dtb[j * cap + lane] : 0.0;
        double Ss = dts, Sf = dtf;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double ts = __shfl_down_sync(0xffffffffu, Ss, o);
          const double tf = __shfl_down_sync(0xffffffffu, Sf, o);
          if (lane + o < 32) {
            Ss += ts;
            Sf += tf;
          }
        }
        const double Ss1 = __shfl_down_sync(0xffffffffu, Ss, 1);  // S_{l+1}; lanes >= K: 0
        const double Sf1 = __shfl_down_sync(0xffffffffu, Sf, 1);
        const double Sref = __shfl_sync(0xffffffffu, Ss, nb + 1);  // nb + 1 <= cap < 27
        const double S0 = __shfl_sync(0xffffffffu, Ss, 0);
        const double Sf0 = __shfl_sync(0xffffffffu, Sf, 0);
        const double SeL = __shfl_sync(0xffffffffu, Ss, (nb + (lane - 27) + 1) & 31);  // lanes 27..30
        double arg = 0.0;
        if (lane < K) arg = A * (Ss1 - Sref);
        else if (lane >= 27 && lane < 31) arg = lane - 27 < nd ? A * (Sref - SeL) : 0.0;
        else if (lane == 31) arg = A * (S0 - Sref);
        const double ex = exp(arg);
        const double exf = exp(A * (lane + 1 < n1 ? Sf1 : (lane == 31 ? Sf0 : 0.0)));  // n1 <= 20
        if (fold) {
          if (lane < n1) wf[j * cap + lane] = (float)(exf * dtf);
          if (lane == 31) lamf[j] = (float)exf;
        }
        const double G = __shfl_sync(0xffffffffu, ex, 31);
#pragma unroll
        for (int d = 0; d < kMD; ++d) {
          const double F = __shfl_sync(0xffffffffu, ex, 27 + d);
          if (d < nd) {
            if (lane <= nb + d) wd[(d * hc + j) * R + lane] = ex * F * dts;
            if (lane == 0) lamd[d * hc + j] = (float)(G * F);
          }
        }
      }
      {
        constexpr int XC = P * (int)sizeof(TI) / 16, BC = N * (int)sizeof(TI) / 16;
        for (int c = gtid; c < nd * hc * XC; c += kGThreads / 2) {
          const int row = c / XC, k = c - row * XC, d = row / hc, j = row - d * hc;
          reinterpret_cast<uint4 *>(static_cast<TI *>(p.xbuf) + ((bh0 + j) * cap + nb + d) * P)[k] =
              reinterpret_cast<const uint4 *>(dX + (size_t)row * P)[k];
        }
        if (own_bc)
          for (int c = gtid; c < 2 * nd * BC; c += kGThreads / 2) {
            const int which = c / (nd * BC), cc = c - which * (nd * BC), d = cc / BC, k = cc - d * BC;
            TI *dst = static_cast<TI *>(which ? p.Cbuf : p.Bbuf) + (bg * cap + nb + d) * N;
            reinterpret_cast<uint4 *>(dst)[k] =
                reinterpret_cast<const uint4 *>((which ? dC : dB) + (size_t)d * N)[k];
          }
        if (gtid < nd * hc) {
          const int d = gtid / hc, j = gtid - (gtid / hc) * hc;
          p.dtbuf[(bh0 + j) * cap + nb + d] = dtd[d * hc + j];
        }
      }
    }
    // draft C rows for this lane's columns, in registers for the whole item
    float4 cr[kMD][S4];
#pragma unroll
    for (int d = 0; d < kMD; ++d)
#pragma unroll
      for (int s4 = 0; s4 < S4; ++s4) cr[d][s4] = ld_vec4<TI>(dC + d * N + 64 * s4 + 4 * c16);
    bar_sync(gbar, kGThreads);
    // ---- S3 (one warp per (draft, head) row, RZ rows of the head per lane):
    // z[d][j][r] = sum_i c_i x_i[r] + D_j x_d[r], with the coefficient
    // c_i = w_{d,i} (B_i . C_d) rounded once by lane i and broadcast
    // When the warp's two rows are the same head's (kGWarps a multiple of hc),
    // one pass over the records serves both: one load of x_i, two chains.
    const bool pair_rows = (kGWarps % hc) == 0 && nd * hc <= 2 * kGWarps;
    if (pair_rows && gw < nd * hc) {
      const int rowB = gw + kGWarps;
      const bool hasB = rowB < nd * hc;
      const int dA = gw / hc, j = gw - dA * hc, dB = dA + kGWarps / hc;
      const float clA = lane <= nb + dA ? (float)(wd[(dA * hc + j) * R + lane] * bc[dA * R + lane]) : 0.f;
      const float clB = hasB && lane <= nb + dB
                            ? (float)(wd[(dB * hc + j) * R + lane] * bc[dB * R + lane]) : 0.f;
      float accA[RZ], accB[RZ], xv[RZ];
#pragma unroll
      for (int k = 0; k < RZ; ++k) accA[k] = accB[k] = 0.f;
      for (int i = 0; i < nb; ++i) {
        ld_vec<TI, RZ>(recX + (j * cap + i) * P + RZ * lane, xv);
        const float ca = __shfl_sync(0xffffffffu, clA, i), cb = __shfl_sync(0xffffffffu, clB, i);
#pragma unroll
        for (int k = 0; k < RZ; ++k) {
          accA[k] = fmaf(ca, xv[k], accA[k]);
          accB[k] = fmaf(cb, xv[k], accB[k]);
        }
      }
      for (int i = nb; i <= nb + (hasB ? dB : dA); ++i) {
        ld_vec<TI, RZ>(dX + ((i - nb) * hc + j) * P + RZ * lane, xv);
        const float ca = __shfl_sync(0xffffffffu, clA, i), cb = __shfl_sync(0xffffffffu, clB, i);
        if (i <= nb + dA) {
#pragma unroll
          for (int k = 0; k < RZ; ++k) accA[k] = fmaf(ca, xv[k], accA[k]);
        }
#pragma unroll
        for (int k = 0; k < RZ; ++k) accB[k] = fmaf(cb, xv[k], accB[k]);
      }
      const float Dj = Ds[j];
      ld_vec<TI, RZ>(dX + (dA * hc + j) * P + RZ * lane, xv);
#pragma unroll
      for (int k = 0; k < RZ; ++k) z[(dA * hc + j) * P + RZ * lane + k] = fmaf(Dj, xv[k], accA[k]);
      if (hasB) {
        ld_vec<TI, RZ>(dX + (dB * hc + j) * P + RZ * lane, xv);
#pragma unroll
        for (int k = 0; k < RZ; ++k) z[(dB * hc + j) * P + RZ * lane + k] = fmaf(Dj, xv[k], accB[k]);
      }
    }
    for (int row = pair_rows ? nd * hc : gw; row < nd * hc; row += kGWarps) {
      const int d = row / hc, j = row - d * hc;
      const float cl = lane <= nb + d ? (float)(wd[(d * hc + j) * R + lane] * bc[d * R + lane]) : 0.f;
      float acc[RZ], xv[RZ];
#pragma unroll
      for (int k = 0; k < RZ; ++k) acc[k] = 0.f;
      for (int i = 0; i < nb; ++i) {
        ld_vec<TI, RZ>(recX + (j * cap + i) * P + RZ * lane, xv);
        const float ci = __shfl_sync(0xffffffffu, cl, i);
#pragma unroll
        for (int k = 0; k < RZ; ++k) acc[k] = fmaf(ci, xv[k], acc[k]);
      }
      for (int i = nb; i <= nb + d; ++i) {
        ld_vec<TI, RZ>(dX + ((i - nb) * hc + j) * P + RZ * lane, xv);
        const float ci = __shfl_sync(0xffffffffu, cl, i);
#pragma unroll
        for (int k = 0; k < RZ; ++k) acc[k] = fmaf(ci, xv[k], acc[k]);
      }
      ld_vec<TI, RZ>(dX + (d * hc + j) * P + RZ * lane, xv);
      const float Dj = Ds[j];
#pragma unroll
      for (int k = 0; k < RZ; ++k) z[(d * hc + j) * P + RZ * lane + k] = fmaf(Dj, xv[k], acc[k]);
    }
    bar_sync(gbar, kGThreads);

    // ---- heads, one at a time: rows into registers, optional fold, outputs
    if (lay.NR > 1 && !take_turn(it)) {
      report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    bool paired = false;
    if constexpr (NSP == 1) {
      if (!fold) {
        paired = true;
        // no fold: heads in pairs, so the two heads' dot products and
        // reductions interleave (independent chains)
        int rows[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) rows[u] = gw * RW + 2 * u + h16;
        for (int j = 0; j < hc; j += 2) {
          const bool two = j + 1 < hc;
          float4 v[2][2][S4];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (hh == 0 || two) {
              const int jj = j + hh;
              const uint32_t pos = (uint32_t)it * hc + jj;
              const int sl = pos % lay.NS;
              if (!mbar_wait(&full[sl], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
                if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
                *abort_flag = 1;
              }
              if (jj == hc - 1) pass_turn();
              const float *tl = reinterpret_cast<const float *>(ring + sl * lay.tile_stride);
#pragma unroll
              for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int s4 = 0; s4 < S4; ++s4)
                  v[hh][u][s4] = *reinterpret_cast<const float4 *>(tl + rows[u] * N + 64 * s4 + 4 * c16);
              __syncwarp();
              if (lane == 0) mbar_arrive(&empty[sl]);
            } else {  // no second head: its (unused) sums run on a copy of the first
#pragma unroll
              for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int s4 = 0; s4 < S4; ++s4) v[1][u][s4] = v[0][u][s4];
            }
          }
          float q[2][2 * kMD];  // paired fp32 FMAs over this lane's 4 S4 columns
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
              for (int d = 0; d < kMD; ++d) {
                float2 a = __fmul2_rn(make_float2(v[hh][u][0].x, v[hh][u][0].y),
                                      make_float2(cr[d][0].x, cr[d][0].y));
                a = __ffma2_rn(make_float2(v[hh][u][0].z, v[hh][u][0].w),
                               make_float2(cr[d][0].z, cr[d][0].w), a);
#pragma unroll
                for (int s4 = 1; s4 < S4; ++s4) {
                  a = __ffma2_rn(make_float2(v[hh][u][s4].x, v[hh][u][s4].y),
                                 make_float2(cr[d][s4].x, cr[d][s4].y), a);
                  a = __ffma2_rn(make_float2(v[hh][u][s4].z, v[hh][u][s4].w),
                                 make_float2(cr[d][s4].z, cr[d][s4].w), a);
                }
                q[hh][u * kMD + d] = a.x + a.y;
              }
          HalfWarpReduce<2 * kMD, 8>::run(q[0], c16);  // every lane shuffles
          HalfWarpReduce<2 * kMD, 8>::run(q[1], c16);
          const int idx = c16 >> 1, u = idx / kMD, d = idx - u * kMD;
          if ((c16 & 1) == 0 && d < nd) {
            const int r = rows[u];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
              if (hh == 0 || two)
                p.y[b * p.bs_y + ((size_t)d * p.H + h_first + j + hh) * P + r] =
                    fmaf(lamd[d * hc + j + hh], q[hh][0], z[(d * hc + j + hh) * P + r]);
          }
        }
      }
    }
    for (int j = 0; j < (paired ? 0 : hc); ++j) {
      const int h = h_first + j;
      const size_t bh = bh0 + j;
      const uint32_t pos = (uint32_t)it * hc + j;
      const int sl = pos % lay.NS;
      if (!mbar_wait(&full[sl], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      if (j == hc - 1) pass_turn();
      const float *tl = reinterpret_cast<const float *>(ring + sl * lay.tile_stride);
      const float lf = fold ? lamf[j] : 0.f;
#pragma unroll
      for (int sp = 0; sp < NSP; ++sp) {
        int rows[2];
        float4 v[2][S4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          rows[u] = gw * RW + 4 * sp + 2 * u + h16;
#pragma unroll
          for (int s4 = 0; s4 < S4; ++s4)
            v[u][s4] = *reinterpret_cast<const float4 *>(tl + rows[u] * N + 64 * s4 + 4 * c16);
        }
        if (sp == NSP - 1) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[sl]);
        }
        if (fold) {  // v <- lam v + sum_i (w_i x_i[row]) B_i[cols], written back once
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int s4 = 0; s4 < S4; ++s4) v[u][s4] = mul4x(lf, v[u][s4]);
          const float *wj = wf + j * cap;
          const TI *xj = recX + j * cap * P;
          for (int i = 0; i < n1; ++i) {
            float4 bb[S4];
#pragma unroll
            for (int s4 = 0; s4 < S4; ++s4)
              bb[s4] = *reinterpret_cast<const float4 *>(&Bf[i * N + 64 * s4 + 4 * c16]);
            const float wi = wj[i];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float xw = wi * to_f32(xj[i * P + rows[u]]);
#pragma unroll
              for (int s4 = 0; s4 < S4; ++s4) v[u][s4] = fma4x(xw, bb[s4], v[u][s4]);
            }
          }
          float *tile = p.h0 + bh * (size_t)(P * N);
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int s4 = 0; s4 < S4; ++s4)
              st_stream(tile + (size_t)rows[u] * N + 64 * s4 + 4 * c16, v[u][s4]);
        }
        float q[2 * kMD];  // paired fp32 FMAs over this lane's 4 S4 columns
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
          for (int d = 0; d < kMD; ++d) {
            float2 a = __fmul2_rn(make_float2(v[u][0].x, v[u][0].y), make_float2(cr[d][0].x, cr[d][0].y));
            a = __ffma2_rn(make_float2(v[u][0].z, v[u][0].w), make_float2(cr[d][0].z, cr[d][0].w), a);
#pragma unroll
            for (int s4 = 1; s4 < S4; ++s4) {
              a = __ffma2_rn(make_float2(v[u][s4].x, v[u][s4].y), make_float2(cr[d][s4].x, cr[d][s4].y), a);
              a = __ffma2_rn(make_float2(v[u][s4].z, v[u][s4].w), make_float2(cr[d][s4].z, cr[d][s4].w), a);
            }
            q[u * kMD + d] = a.x + a.y;
          }
        HalfWarpReduce<2 * kMD, 8>::run(q, c16);  // every lane shuffles
        const int idx = c16 >> 1, u = idx / kMD, d = idx - u * kMD;
        if ((c16 & 1) == 0 && d < nd) {
          const int r = rows[u];
          p.y[b * p.bs_y + ((size_t)d * p.H + h) * P + r] =
              fmaf(lamd[d * hc + j], q[0], z[(d * hc + j) * P + r]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&rempty[rb]);
    if (gtid < hc) p.len[bh0 + gtid] = nb;
  }
}

// Chunked verify only: append the draft B and C rows of group (b, g) at the
// group's committed length, read back from the lengths the verify kernel just
// wrote.  A group whose heads are not all at the same length (the verify
// kernel rejected some of its chunks and reported it in the status word) is
// skipped, so no buffered record another head still uses is overwritten; for
// a rejected group whose heads agree the rows land in free slots (>= len).
template <typename TI>
__global__ void __launch_bounds__(128) m2_verify_append_bc_kernel(const M2Params p) {
  const int b = blockIdx.x / p.G, g = blockIdx.x - (blockIdx.x / p.G) * p.G;
  const size_t bg = (size_t)b * p.G + g;
  const int32_t *lg = p.len + (size_t)b * p.H + (size_t)g * p.hpg;
  const int nb = lg[0];
  if (__syncthreads_or(threadIdx.x < p.hpg && lg[threadIdx.x] != nb)) return;
  if (nb < 0 || nb + p.n_draft > p.cap) return;
  const TI *Bin = static_cast<const TI *>(p.Bm) + b * p.bs_B;
  const TI *Cin = static_cast<const TI *>(p.Cm) + b * p.bs_C;
  for (int e = threadIdx.x; e < p.n_draft * p.N; e += blockDim.x) {
    const int d = e / p.N, c = e - d * p.N;
    static_cast<TI *>(p.Bbuf)[(bg * p.cap + nb + d) * p.N + c] = Bin[((size_t)d * p.G + g) * p.N + c];
    static_cast<TI *>(p.Cbuf)[(bg * p.cap + nb + d) * p.N + c] = Cin[((size_t)d * p.G + g) * p.N + c];
  }
}

}  // namespace

cudaError_t m2_launch_verify(const M2Params &p, cudaStream_t s) {
  if (p.B * p.G == 0) return cudaSuccess;
  return dispatch_shape(p.P, p.N, p.in_bf16, [&](auto PP, auto NN, auto ti) {
    using TI = decltype(ti);
    constexpr int P_ = decltype(PP)::value, N_ = decltype(NN)::value;
    VerifyLayout lay;
    lay.NS = 0;
    for (int nc = 1; nc <= p.hpg && lay.NS < 2; ++nc)
      if (p.hpg % nc == 0)
        lay = VerifyLayout::make(P_, N_, p.hpg, nc, p.cap, p.L, (int)sizeof(TI), 220 * 1024);
    if (lay.NS < 2) return cudaErrorInvalidConfiguration;
    auto kernel = m2_verify_kernel<P_, N_, TI>;
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
    if (e != cudaSuccess) return e;
    const int nitems = p.B * p.G * lay.nchunk;
    const int grid = nitems < sm_count() ? nitems : sm_count();
    kernel<<<grid, kVThreads + 64, lay.total, s>>>(p, lay);
    if (lay.nchunk > 1) {
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      m2_verify_append_bc_kernel<TI><<<p.B * p.G, 128, 0, s>>>(p);
    }
    return cudaGetLastError();
  });
}

}  // namespace rssm
