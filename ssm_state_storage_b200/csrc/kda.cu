// kda.cu -- Kimi Delta Attention decode kernels for sm_100a: replay decode
// step with fused flush fold, standalone fold (flush / materialise) and the
// conventional full-state step.
//
// Layer type named in [news.hamidun.com, "NVIDIA تقدّم ReplaySSM…", §Why
// hybrid models became the norm]; the ReplaySSM state (checkpoint h0 plus a
// buffer of recent records, outputs without any state write, one checkpoint
// write per window) as in [sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…",
// §How ReplaySSM works].
//
// Recurrence (Kimi Linear, Moonshot AI 2025): the gated delta rule with one
// decay per key channel, state S [DK][DV], alpha_t in (0,1)^DK:
//   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,  o_t = scale S_t^T q_t.
// Writing S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T with the correction
//   u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t),
// and unrolling from h0 over records 0..t (Gamma_i = alpha_0 o .. o alpha_i,
// R_i = alpha_{i+1} o .. o alpha_t, elementwise over the key channels):
//   S_t = Gamma_t o h0 + sum_{i<=t} (R_i o k_i) u_i^T          (fold; o scales rows)
//   u_t = beta_t (v_t - h0^T (Gamma_t o k_t) - sum_{j<t} (k_j . (R_j o k_t)) u_j)
//   o_t = scale (h0^T (Gamma_t o q_t) + sum_{i<=t} (k_i . (R_i o q_t)) u_i)
// Each record's correction depends only on h0 and the records up to it, so
// it is computed once, when the record is appended, and cached in the buffer
// (buf[5]); a step then needs two products with h0 (Gamma o k, Gamma o q)
// and O(t) decay-weighted key dots.  The conventional step is the same
// algebra with one record and the state written back; it also serves as the
// conventional step of Gated DeltaNet (a scalar decay is the all-equal case).
//
// kda_kernel: one CTA of 256 threads per (sequence, head); lane l of warp w
// holds rows 16w..16w+15 and columns 4l..4l+3 of the 128 x 128 tile in
// registers (conventional step, standalone folds).  kda_decode2_kernel: the
// persistent replay decode step with two consumer groups (below).  The
// per-channel decay products are taken in fp64 (one thread per channel).
#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"

namespace rssm {
namespace {

constexpr int KDc = 128, KVc = 128, kKRows = KDc / 8, kKRec = kMaxCap;

enum KdaMode { kKdaDecode = 0, kKdaFlush = 1, kKdaMaterialize = 2, kKdaFull = 3 };

struct KdaSmem {
  float K[kKRec][KDc];  // keys
  float U[kKRec][KVc];  // corrections (cached ones; the current record's is formed here)
  float A[kKRec][KDc];  // per-channel decays
  float R[kKRec][KDc];  // R_i = product of the decays of the records after i
  float gam[KDc];       // Gamma of the last record
  float kg[KDc], qg[KDc];
  float q[KDc], v[KVc];
  float part[8][2][KVc];
  float G[kKRec], KQ[kKRec];
  float beta;
  int n, act, fold;
};

template <typename TI, int MODE>
__global__ void __launch_bounds__(kThreads, 2) kda_kernel(const GDNParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  KdaSmem &S = *reinterpret_cast<KdaSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / p.H, h = blockIdx.x - (blockIdx.x / p.H) * p.H;
  const size_t bh = blockIdx.x;
  constexpr bool kOut = (MODE == kKdaDecode || MODE == kKdaFull);

  // ---- record count n (records 0..n-1), whether to fold
  if (tid == 0) {
    int n = 1, act = 1, ok = 1, fold = 1;
    if (MODE == kKdaFull) {
      act = !(p.limit && p.step_index >= p.limit[b]);
    } else {
      const int n0 = p.len[bh];
      if (MODE == kKdaDecode) {
        ok = n0 >= 0 && n0 < p.L;
        n = n0 + 1;
        fold = n == p.L;
      } else {
        ok = n0 >= 0 && n0 <= p.cap;
        n = n0;
        act = MODE == kKdaMaterialize ? 1 : (n0 >= p.L || (p.force && n0 > 0));
      }
      if (!ok) report(p.status, RSSM_ERR_STATE);
    }
    S.n = ok ? n : -1;
    S.act = act;
    S.fold = fold;
  }
  __syncthreads();
  const int n = S.n;
  if (n < 0 || !S.act) return;
  const bool fold = S.fold;
  const int last = n - 1;

  float *state = (MODE == kKdaFull) ? p.S + bh * (KDc * KVc) : p.h0 + bh * (KDc * KVc);
  float4 hv[kKRows];
#pragma unroll
  for (int rho = 0; rho < kKRows; ++rho)
    hv[rho] = ld_stream(state + (size_t)(kKRows * warp + rho) * KVc + 4 * lane);

  // ---- stage the buffered records, then this step's
  const int nbuf = kOut ? n - 1 : n;
  const TI *kb = static_cast<const TI *>(p.kbuf) + bh * p.cap * KDc;
  const float *ab = p.abuf + bh * p.cap * KDc;
  const float *ub = p.ubuf + bh * p.cap * KVc;
  // every load first (one memory latency for the buffered records and this
  // step's), then the shared-memory stores
  constexpr int PER = kKRec * KDc / kThreads;
  float kv[PER], av[PER], uv[PER];
  if (MODE != kKdaFull) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kThreads;
      if (e < nbuf * KDc) {
        kv[u] = to_f32(kb[e]);
        av[u] = ab[e];
        uv[u] = ub[e];
      }
    }
  }
  float cur0 = 0.f, cur1 = 0.f, cur2 = 0.f, beta = 0.f;
  if (kOut) {
    const TI *qin = static_cast<const TI *>(p.q) + b * p.bs_q + (size_t)h * KDc;
    const TI *kin = static_cast<const TI *>(p.k) + b * p.bs_k + (size_t)h * KDc;
    const TI *vin = static_cast<const TI *>(p.v) + b * p.bs_v + (size_t)h * KVc;
    const float *ain = p.alpha + b * p.bs_a + (size_t)h * KDc;
    const float *bin = p.beta + b * p.bs_b + h;
    if (MODE == kKdaDecode && p.inplace) {  // the record is already in slot len
      const size_t slot = bh * p.cap + last;
      qin = static_cast<const TI *>(p.qbuf) + slot * KDc;
      kin = static_cast<const TI *>(p.kbuf) + slot * KDc;
      vin = static_cast<const TI *>(p.vbuf) + slot * KVc;
      ain = p.abuf + slot * KDc;
      bin = p.bbuf + slot;
    }
    if (tid < KDc) {
      cur0 = to_f32(kin[tid]);
      // Gated DeltaNet's conventional step runs here too: one decay for every
      // channel, alpha [B][H] (Diag(alpha) = alpha I commutes with the rule)
      cur1 = p.kda ? ain[tid] : p.alpha[b * p.bs_a + h];
      cur2 = to_f32(qin[tid]);
    } else {
      cur0 = to_f32(vin[tid - KDc]);
    }
    if (tid == 0) beta = *bin;
  }
  if (MODE != kKdaFull) {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kThreads;
      if (e < nbuf * KDc) {
        const int i = e / KDc, c = e - i * KDc;
        S.K[i][c] = kv[u];
        S.A[i][c] = av[u];
        S.U[i][c] = uv[u];
      }
    }
  }
  if (kOut) {
    if (tid < KDc) {
      S.K[last][tid] = cur0;
      S.A[last][tid] = cur1;
      S.q[tid] = cur2;
    } else {
      S.v[tid - KDc] = cur0;
    }
    if (tid == 0) S.beta = beta;
  }
  __syncthreads();

  // ---- per-channel decay products (fp64, one thread per key channel)
  if (tid < KDc) {
    const int c = tid;
    double pr = 1.0;
    for (int i = last; i >= 0; --i) {
      S.R[i][c] = (float)pr;
      pr *= (double)S.A[i][c];
    }
    S.gam[c] = (float)pr;
    if (kOut) {
      S.kg[c] = (float)(pr * (double)S.K[last][c]);
      S.qg[c] = (float)(pr * (double)S.q[c]);
    }
  }
  __syncthreads();

  const int row0 = kKRows * warp;
  if constexpr (kOut) {
    // decay-weighted key dots, fp64 sums:
    // G_j = k_j . (R_j o k_last) (j < last), KQ_i = k_i . (R_i o q) (i <= last)
    const int ndot = 2 * n - 1;
    if constexpr (MODE == kKdaFull) {  // one dot (n = 1): 16 threads
      const int c0 = (tid & 15) * 8;
      double acc = 0.0;
      if (tid < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          acc += (double)(S.K[0][c0 + e] * S.R[0][c0 + e]) * (double)S.q[c0 + e];
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      acc += __shfl_xor_sync(0xffffffffu, acc, 8);
      if (tid == 0) S.KQ[0] = (float)acc;
    } else
    // 8 threads per dot (one pass for up to 32 dots), thread j of a dot
    // taking the 4-element chunks j + 8m
    for (int base = 0; base < ndot; base += kThreads / 8) {
      const int d = base + (tid >> 3), j = tid & 7;
      double acc = 0.0, acc1 = 0.0;
      if (d < ndot) {
        const int i = d < last ? d : d - last;
        const float *other = d < last ? S.K[last] : S.q;
#pragma unroll
        for (int m = 0; m < KDc / 32; ++m) {
          const int c0 = 4 * (j + 8 * m);
          const float4 kv = *reinterpret_cast<const float4 *>(&S.K[i][c0]);
          const float4 rv = *reinterpret_cast<const float4 *>(&S.R[i][c0]);
          const float4 ov = *reinterpret_cast<const float4 *>(&other[c0]);
          acc += (double)(kv.x * rv.x) * (double)ov.x;
          acc1 += (double)(kv.y * rv.y) * (double)ov.y;
          acc += (double)(kv.z * rv.z) * (double)ov.z;
          acc1 += (double)(kv.w * rv.w) * (double)ov.w;
        }
        acc += acc1;
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (d < ndot && j == 0) {
        if (d < last) S.G[d] = (float)acc;
        else S.KQ[d - last] = (float)acc;
      }
    }
    // h0^T (Gamma o k_last) and h0^T (Gamma o q): partial sums over this warp's rows
    float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
    for (int rho = 0; rho < kKRows; ++rho) {
      pk = fma4x(S.kg[row0 + rho], hv[rho], pk);
      pq = fma4x(S.qg[row0 + rho], hv[rho], pq);
    }
    *reinterpret_cast<float4 *>(&S.part[warp][0][4 * lane]) = pk;
    *reinterpret_cast<float4 *>(&S.part[warp][1][4 * lane]) = pq;
    __syncthreads();
    {
      // thread pair (2c, 2c+1) owns column c: the even thread sums the
      // partials of z, the odd one those of zq, and they swap; each runs over
      // the older records of its parity (one load of u_j for both sums) and
      // the pair adds the two halves
      const int c = tid >> 1, par = tid & 1;
      float zc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) zc += S.part[w][par][c];
      const float zo = __shfl_xor_sync(0xffffffffu, zc, 1);
      const float z = par ? zo : zc, zq = par ? zc : zo;
      float su = 0.f, so = 0.f;
      for (int j = par; j < last; j += 2) {
        const float uj = S.U[j][c];
        su = fmaf(S.G[j], uj, su);
        so = fmaf(S.KQ[j], uj, so);
      }
      su += __shfl_xor_sync(0xffffffffu, su, 1);
      so += __shfl_xor_sync(0xffffffffu, so, 1);
      const float u = S.beta * ((S.v[c] - z) - su);
      if (par == 0) {
        S.U[last][c] = u;
        if (MODE == kKdaDecode && !fold) p.ubuf[(bh * p.cap + last) * KVc + c] = u;
      } else {
        const float o = fmaf(S.KQ[last], u, zq + so);
        p.y[b * p.bs_y + (size_t)h * KVc + c] = p.scale * o;
      }
    }
    if (MODE == kKdaDecode && !fold && !p.inplace) {
      // append this step's record (input values, unrounded)
      const size_t slot = bh * p.cap + last;
      if (tid < KDc) {
        static_cast<TI *>(p.qbuf)[slot * KDc + tid] =
            static_cast<const TI *>(p.q)[b * p.bs_q + (size_t)h * KDc + tid];
        static_cast<TI *>(p.kbuf)[slot * KDc + tid] =
            static_cast<const TI *>(p.k)[b * p.bs_k + (size_t)h * KDc + tid];
        p.abuf[slot * KDc + tid] = S.A[last][tid];
      } else {
        static_cast<TI *>(p.vbuf)[slot * KVc + tid - KDc] =
            static_cast<const TI *>(p.v)[b * p.bs_v + (size_t)h * KVc + tid - KDc];
      }
      if (tid == 0) p.bbuf[slot] = S.beta;
    }
    if (fold) __syncthreads();  // the current correction is read by every thread
  }

  // ---- fold: h <- Gamma o h + sum_i (R_i o k_i) u_i^T, written once
  if (fold) {
#pragma unroll
    for (int rho = 0; rho < kKRows; ++rho) hv[rho] = mul4x(S.gam[row0 + rho], hv[rho]);
    for (int i = 0; i < n; ++i) {
      const float4 ui = *reinterpret_cast<const float4 *>(&S.U[i][4 * lane]);
#pragma unroll
      for (int rho = 0; rho < kKRows; ++rho)
        hv[rho] = fma4x(S.R[i][row0 + rho] * S.K[i][row0 + rho], ui, hv[rho]);
    }
    float *dst = (MODE == kKdaMaterialize) ? p.S_out + bh * (KDc * KVc) : state;
#pragma unroll
    for (int rho = 0; rho < kKRows; ++rho)
      st_stream(dst + (size_t)(row0 + rho) * KVc + 4 * lane, hv[rho]);
  }
  if (tid == 0 && (MODE == kKdaDecode || MODE == kKdaFlush)) p.len[bh] = fold ? 0 : n;
}

// ============================================================ persistent decode step
// Persistent replay decode step (one CTA of 320 threads per SM), structured as
// the two-group Gated DeltaNet kernel: warp 8 streams each item's checkpoint
// as two 32 KiB half-tiles into a ring of exactly 4 slots, warp 9 stages the
// item's inputs and bulk-copies its buffered keys, corrections and decay
// vectors, and two consumer groups of 4 warps take alternate items (item it
// uses slots 2(it%2), 2(it%2)+1 and record buffer it % NR with NR even, so
// each group owns its slots and buffers).  Per item, in a group:
//   * thread c (one key channel) runs the fp64 suffix products of the decays
//     over the records and overwrites each staged decay with the record's
//     weighted key w_i[c] = k_i[c] * R_i[c] (the fp32 product both the dots
//     and the fold use), and forms Gamma o k and Gamma o q;
//   * 4 threads per key dot: G_j = w_j . k_last, KQ_i = w_i . q (fp64 sums);
//   * warp w: partial h0^T (Gamma o k), h0^T (Gamma o q) over rows 32w.. from
//     the slot; thread c: u and the output of column c;
//   * flush: h0[r] <- Gamma[r] h0[r] + sum_i w_i[r] u_i, rows read from the
//     slot, written once.
constexpr int kKHalfRows = KDc / 2, kKHalfBytes = kKHalfRows * KVc * 4;  // 32 KiB

struct KdaLayout {
  int NR, L, stage_floats, db_floats;
  int off_bars, off_recK, off_recU, off_recW, off_stage, off_db, off_single, off_ring, total;
  __host__ static int a128(int v) { return (v + 127) & ~127; }
  // stage: q, v [128] fp32 | beta, n0, bad, pad; per group: Gamma, kg, qg
  // [128] | G, KQ [L]; per group: partial sums [4][2][128] | u [128]
  __host__ static KdaLayout make(int L, int es, int budget) {
    KdaLayout d;
    d.L = L;
    d.stage_floats = 2 * 128 + 4;
    d.db_floats = 3 * 128 + 2 * ((L + 3) & ~3);
    for (d.NR = 4; d.NR >= 2; d.NR -= 2) {
      int o = 0;
      d.off_bars = o;
      o += a128(8 * (2 * 8 + 2 * 4));
      d.off_recK = o;
      o += a128(d.NR * L * KDc * es);
      d.off_recU = o;
      o += a128(d.NR * L * KVc * 4);
      d.off_recW = o;
      o += a128(d.NR * L * KDc * 4);
      d.off_stage = o;
      o += a128(d.NR * d.stage_floats * 4);
      d.off_db = o;
      o += a128(2 * d.db_floats * 4);
      d.off_single = o;
      o += a128(2 * (4 * 2 * 128 + 128) * 4);
      d.off_ring = o;
      d.total = o + 4 * kKHalfBytes;
      if (d.total <= budget) return d;
    }
    d.NR = 0;
    return d;
  }
};

template <typename TI>
__device__ __forceinline__ float4 ld4_in(const TI *p) {
  if constexpr (sizeof(TI) == 4) {
    return *reinterpret_cast<const float4 *>(p);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const TI *e = reinterpret_cast<const TI *>(&raw);
    return make_float4(to_f32(e[0]), to_f32(e[1]), to_f32(e[2]), to_f32(e[3]));
  }
}

template <typename TI>
__global__ void __launch_bounds__(kThreads + 64, 1) kda_decode2_kernel(const GDNParams p,
                                                                    const KdaLayout lay) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
  uint64_t *empty = full + 8, *rfull = empty + 8, *rempty = rfull + 4;
  unsigned char *ring = smem + lay.off_ring;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nitems = p.B * p.H;
  const int L = lay.L, NR = lay.NR;

  if (tid == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);  // the 4 warps of the group that owns the slot
    }
    for (int r = 0; r < 4; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], 4);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == 8) {  // tile producer: half-tiles in (item, half) order, 4 slots
    if (lane != 0) return;
    int slot = 0;
    uint32_t sphase = 0, issued = 0, parity = 0;
    bool failed = false;
    for (int item = blockIdx.x; item < nitems && !failed; item += gridDim.x) {
      for (int half = 0; half < 2; ++half) {
        if (*abort_flag || !mbar_wait(&empty[slot], sphase ^ 1, kWaitLimitNs, abort_flag) ||
            *abort_flag) {
          failed = true;
          break;
        }
        mbar_arrive_expect_tx(&full[slot], kKHalfBytes);
        bulk_g2s(ring + slot * kKHalfBytes,
                 p.h0 + (size_t)item * KDc * KVc + (size_t)half * kKHalfRows * KVc, kKHalfBytes,
                 &full[slot]);
        issued |= 1u << slot;
        parity = (parity & ~(1u << slot)) | (sphase << slot);
        if (++slot == 4) {
          slot = 0;
          sphase ^= 1;
        }
      }
    }
    if (failed) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    for (int s2 = 0; s2 < 4; ++s2)  // every copy issued here lands before the warp returns
      if (issued & (1u << s2)) mbar_wait(&full[s2], (parity >> s2) & 1u);
    return;
  }

  if (warp == 9) {  // stager: all loads of an item first, then shared-memory writes and copies
    int it = 0;
    ArmedRecords armed;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
      const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
      if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
      const int rb = it % NR;
      bool ok = !abort_now;
      if (ok && lane == 0)
        ok = mbar_wait(&rempty[rb], ((it / NR) & 1) ^ 1, kWaitLimitNs, abort_flag) && !*abort_flag;
      if (!__shfl_sync(0xffffffffu, (int)ok, 0)) {
        if (lane == 0 && !*abort_flag) {
          report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      const int b = item / p.H, h = item - (item / p.H) * p.H;
      const size_t bh = (size_t)item;
      const int n0 = __ldcg(&p.len[bh]);
      const TI *qin = static_cast<const TI *>(p.q) + b * p.bs_q + (size_t)h * KDc;
      const TI *kin = static_cast<const TI *>(p.k) + b * p.bs_k + (size_t)h * KDc;
      const TI *vin = static_cast<const TI *>(p.v) + b * p.bs_v + (size_t)h * KVc;
      const float *ain = p.alpha + b * p.bs_a + (size_t)h * KDc;
      const float *bin = p.beta + b * p.bs_b + h;
      if (p.inplace) {  // the record is already in slot len: read it from there
        const size_t slot = bh * p.cap + min(max(n0, 0), L - 1);  // stays in bounds
        qin = static_cast<const TI *>(p.qbuf) + slot * KDc;
        kin = static_cast<const TI *>(p.kbuf) + slot * KDc;
        vin = static_cast<const TI *>(p.vbuf) + slot * KVc;
        ain = p.abuf + slot * KDc;
        bin = p.bbuf + slot;
      }
      TI qv[4], kv[4], vv[4];
      float av[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qv[u] = qin[lane + 32 * u];
        kv[u] = kin[lane + 32 * u];
        vv[u] = vin[lane + 32 * u];
        av[u] = ain[lane + 32 * u];
      }
      const float b_cur = *bin;
      const bool bad = n0 < 0 || n0 >= L;
      const int k = min(max(n0 + 1, 1), L);  // copies stay in bounds even for a bad length
      float *st = reinterpret_cast<float *>(smem + lay.off_stage) + rb * lay.stage_floats;
      TI *rK = reinterpret_cast<TI *>(smem + lay.off_recK) + (size_t)rb * L * KDc;
      float *rW = reinterpret_cast<float *>(smem + lay.off_recW) + (size_t)rb * L * KDc;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = lane + 32 * u;
        st[c] = to_f32(qv[u]);
        st[128 + c] = to_f32(vv[u]);
        rK[(k - 1) * KDc + c] = kv[u];
        rW[(k - 1) * KDc + c] = av[u];
      }
      if (lane == 0) {
        st[256] = b_cur;
        reinterpret_cast<int *>(st)[257] = n0;
        reinterpret_cast<int *>(st)[258] = bad;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t bK = (k - 1) * KDc * sizeof(TI), bU = (k - 1) * KVc * 4, bW = (k - 1) * KDc * 4;
        mbar_arrive_expect_tx(&rfull[rb], bK + bU + bW);
        if (k > 1) {
          bulk_g2s(rK, static_cast<const TI *>(p.kbuf) + bh * p.cap * KDc, bK, &rfull[rb]);
          bulk_g2s(reinterpret_cast<float *>(smem + lay.off_recU) + (size_t)rb * L * KVc,
                   p.ubuf + bh * p.cap * KVc, bU, &rfull[rb]);
          bulk_g2s(rW, p.abuf + bh * p.cap * KDc, bW, &rfull[rb]);
        }
      }
      armed.arm(rb, (it / NR) & 1);
    }
    if (lane == 0) armed.drain(rfull, NR);  // no record copy outlives the warp
    __syncwarp();
    return;
  }

  // Consumer group grp (warps 4grp .. 4grp+3), thread gt = key channel / column.
  constexpr int kG = 128;
  const int grp = warp >> 2, gw = warp & 3, gt = tid & (kG - 1);
  const uint32_t gbar = 1 + grp;
  float *db = reinterpret_cast<float *>(smem + lay.off_db) + grp * lay.db_floats;
  float *gamv = db, *kg = db + 128, *qg = db + 256, *G = db + 384, *KQ = G + ((L + 3) & ~3);
  float *part = reinterpret_cast<float *>(smem + lay.off_single) + grp * (4 * 2 * 128 + 128);
  float *ucur = part + 4 * 2 * 128;

  int it = grp;
  for (int item = blockIdx.x + grp * gridDim.x; item < nitems; item += 2 * gridDim.x, it += 2) {
    const int rb = it % NR;
    const int b = item / p.H, h = item - (item / p.H) * p.H;
    const size_t bh = (size_t)item;
    const float *st = reinterpret_cast<const float *>(smem + lay.off_stage) + rb * lay.stage_floats;
    const float *qs = st, *vs = st + 128;
    const TI *rK = reinterpret_cast<const TI *>(smem + lay.off_recK) + (size_t)rb * L * KDc;
    const float *rU = reinterpret_cast<const float *>(smem + lay.off_recU) + (size_t)rb * L * KVc;
    float *rW = reinterpret_cast<float *>(smem + lay.off_recW) + (size_t)rb * L * KDc;
    const int sl0 = 2 * (it & 1), sl1 = sl0 + 1;
    const uint32_t tphase = (it >> 1) & 1;

    const bool got = mbar_wait(&rfull[rb], (it / NR) & 1, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(gbar, kG, !got || *abort_flag)) break;
    const int n0 = reinterpret_cast<const int *>(st)[257];
    if (reinterpret_cast<const int *>(st)[258]) {
      if (gt == 0) report(p.status, RSSM_ERR_STATE);
      if (!mbar_wait(&full[gw < 2 ? sl0 : sl1], tphase, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[sl0]);
        mbar_arrive(&empty[sl1]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rempty[rb]);
      continue;
    }
    const int k = n0 + 1, last = n0;
    const bool fold = (k == L);
    const float beta = st[256];

    // ---- appends (an in-place step's record is in its slot already)
    if (!fold && !p.inplace) {
      const size_t slot = bh * p.cap + last;
      static_cast<TI *>(p.qbuf)[slot * KDc + gt] = from_f32<TI>(qs[gt]);
      static_cast<TI *>(p.kbuf)[slot * KDc + gt] = rK[last * KDc + gt];
      static_cast<TI *>(p.vbuf)[slot * KVc + gt] = from_f32<TI>(vs[gt]);
      p.abuf[slot * KDc + gt] = rW[last * KDc + gt];
      if (gt == 0) p.bbuf[slot] = beta;
    }
    // ---- channel c: decay suffix products in fp64; each staged decay is
    // replaced by the record's weighted key w_i[c] = k_i[c] * R_i[c]
    {
      const int c = gt;
      double pr = 1.0;
      for (int i = last; i >= 0; --i) {
        const float a = rW[i * KDc + c];
        rW[i * KDc + c] = to_f32(rK[i * KDc + c]) * (float)pr;
        pr *= (double)a;
      }
      gamv[c] = (float)pr;
      kg[c] = (float)(pr * (double)to_f32(rK[last * KDc + c]));
      qg[c] = (float)(pr * (double)qs[c]);
    }
    bar_sync(gbar, kG);
    // ---- 2k-1 <= 31 decay-weighted key dots (the window is at most 16):
    // G_j = w_j . k_last (j < last), KQ_i = w_i . q (i <= last); 4 threads per
    // dot, thread j4 takes the 4-element chunks j4 + 4m; fp64 sums
    {
      const int ndot = 2 * k - 1, d = gt >> 2, j4 = gt & 3;
      double acc = 0.0, acc1 = 0.0;
      if (d < ndot) {
        const int i = d < last ? d : d - last;
#pragma unroll
        for (int m = 0; m < KDc / 16; ++m) {
          const int c0 = 4 * (j4 + 4 * m);
          const float4 w4 = *reinterpret_cast<const float4 *>(&rW[i * KDc + c0]);
          const float4 o4 = d < last ? ld4_in<TI>(rK + last * KDc + c0)
                                     : *reinterpret_cast<const float4 *>(&qs[c0]);
          acc += (double)w4.x * (double)o4.x;
          acc1 += (double)w4.y * (double)o4.y;
          acc += (double)w4.z * (double)o4.z;
          acc1 += (double)w4.w * (double)o4.w;
        }
        acc += acc1;
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (d < ndot && j4 == 0) {
        if (d < last) G[d] = (float)acc;
        else KQ[d - last] = (float)acc;
      }
    }
    // ---- partial h0^T (Gamma o k) and h0^T (Gamma o q) over this warp's 32
    // rows, read from the slot
    const int half = gw >> 1, sl = half ? sl1 : sl0;
    if (!mbar_wait(&full[sl], tphase, p.wait_ns, abort_flag)) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    {
      const float *tile = reinterpret_cast<const float *>(ring + sl * kKHalfBytes) +
                          (size_t)(32 * (gw & 1)) * KVc + 4 * lane;
      const int row0 = 32 * gw;
      float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll 2
      for (int t = 0; t < 8; ++t) {
        const float4 k4 = *reinterpret_cast<const float4 *>(&kg[row0 + 4 * t]);
        const float4 q4 = *reinterpret_cast<const float4 *>(&qg[row0 + 4 * t]);
        const float kr[4] = {k4.x, k4.y, k4.z, k4.w}, qr[4] = {q4.x, q4.y, q4.z, q4.w};
        float4 x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = *reinterpret_cast<const float4 *>(tile + (4 * t + e) * KVc);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pk = fma4x(kr[e], x[e], pk);
          pq = fma4x(qr[e], x[e], pq);
        }
      }
      *reinterpret_cast<float4 *>(&part[(gw * 2 + 0) * 128 + 4 * lane]) = pk;
      *reinterpret_cast<float4 *>(&part[(gw * 2 + 1) * 128 + 4 * lane]) = pq;
    }
    if (!fold) {  // the fold reads both half-tiles again
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[sl0]);
        mbar_arrive(&empty[sl1]);
      }
    }
    bar_sync(gbar, kG);
    // ---- column c: u and the output (one pass over the older records)
    {
      const int c = gt;
      float z = 0.f, zq = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        z += part[(w * 2 + 0) * 128 + c];
        zq += part[(w * 2 + 1) * 128 + c];
      }
      float su0 = 0.f, su1 = 0.f, so0 = 0.f, so1 = 0.f;
      int j = 0;
      for (; j + 1 < last; j += 2) {
        const float u0 = rU[j * KVc + c], u1 = rU[(j + 1) * KVc + c];
        su0 = fmaf(G[j], u0, su0);
        so0 = fmaf(KQ[j], u0, so0);
        su1 = fmaf(G[j + 1], u1, su1);
        so1 = fmaf(KQ[j + 1], u1, so1);
      }
      if (j < last) {
        const float u0 = rU[j * KVc + c];
        su0 = fmaf(G[j], u0, su0);
        so0 = fmaf(KQ[j], u0, so0);
      }
      const float u = beta * ((vs[c] - z) - (su0 + su1));
      const float o = fmaf(KQ[last], u, zq + (so0 + so1));
      if (!fold) p.ubuf[(bh * p.cap + last) * KVc + c] = u;
      else ucur[c] = u;
      p.y[b * p.bs_y + (size_t)h * KVc + c] = p.scale * o;
    }
    // ---- fold: h0[r] <- Gamma[r] h0[r] + sum_i w_i[r] u_i over this warp's
    // rows 32gw.. (its half-tile's slot is still held), written once
    if (fold) {
      bar_sync(gbar, kG);  // every column's u
      const float *tile = reinterpret_cast<const float *>(ring + sl * kKHalfBytes) +
                          (size_t)(32 * (gw & 1)) * KVc + 4 * lane;
      float *dst = p.h0 + bh * (KDc * KVc) + (size_t)(32 * gw) * KVc + 4 * lane;
#pragma unroll 1
      for (int r0 = 0; r0 < 32; r0 += 8) {
        float4 acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          acc[e] = mul4x(gamv[32 * gw + r0 + e], *reinterpret_cast<const float4 *>(tile + (r0 + e) * KVc));
        for (int i = 0; i <= last; ++i) {
          const float4 ui = *reinterpret_cast<const float4 *>(i < last ? &rU[i * KVc + 4 * lane]
                                                                        : &ucur[4 * lane]);
          const float4 wa = *reinterpret_cast<const float4 *>(&rW[i * KDc + 32 * gw + r0]);
          const float4 wb = *reinterpret_cast<const float4 *>(&rW[i * KDc + 32 * gw + r0 + 4]);
          const float wr[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fma4x(wr[e], ui, acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) st_stream(dst + (size_t)(r0 + e) * KVc, acc[e]);
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[sl0]);
        mbar_arrive(&empty[sl1]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&rempty[rb]);
    if (gt == 0) p.len[bh] = fold ? 0 : k;
  }
}

int kda_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

// The persistent decode step when its layout fits (window <= 16), else none.
template <typename TI>
bool kda_launch_persistent(const GDNParams &p, cudaStream_t s, cudaError_t &err) {
  const KdaLayout lay = KdaLayout::make(p.L, (int)sizeof(TI), 227 * 1024);
  if (lay.NR < 2 || p.L > 16) return false;
  err = cudaFuncSetAttribute(kda_decode2_kernel<TI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             lay.total);
  if (err != cudaSuccess) return true;
  const int nitems = p.B * p.H;
  const int grid = nitems < kda_sm_count() ? nitems : kda_sm_count();
  kda_decode2_kernel<TI><<<grid, kThreads + 64, lay.total, s>>>(p, lay);
  err = cudaGetLastError();
  return true;
}

template <typename TI, int MODE>
cudaError_t kda_launch_mode(const GDNParams &p, cudaStream_t s) {
  const size_t smem = sizeof(KdaSmem);
  cudaError_t e = cudaFuncSetAttribute(kda_kernel<TI, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kda_kernel<TI, MODE><<<(unsigned)(p.B * p.H), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t kda_launch_dt(const GDNParams &p, cudaStream_t s) {
  return p.in_bf16 ? kda_launch_mode<__nv_bfloat16, MODE>(p, s) : kda_launch_mode<float, MODE>(p, s);
}

}  // namespace

cudaError_t kda_launch(const GDNParams &p, int mode, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  switch (mode) {
    case 0: {
      cudaError_t e = cudaSuccess;
      if (p.kda && (p.in_bf16 ? kda_launch_persistent<__nv_bfloat16>(p, s, e)
                              : kda_launch_persistent<float>(p, s, e)))
        return e;
      return kda_launch_dt<kKdaDecode>(p, s);
    }
    case 1: return kda_launch_dt<kKdaFlush>(p, s);
    case 2: return kda_launch_dt<kKdaMaterialize>(p, s);
    case 3: return kda_launch_dt<kKdaFull>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rssm
