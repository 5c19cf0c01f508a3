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
// One CTA of 256 threads per (sequence, head); lane l of warp w holds rows
// 16w..16w+15 and columns 4l..4l+3 of the 128 x 128 tile in registers.  The
// per-channel decay products are taken in fp64 (one thread per channel).
#include "common.cuh"
#include "internal.h"

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
    case 0: return kda_launch_dt<kKdaDecode>(p, s);
    case 1: return kda_launch_dt<kKdaFlush>(p, s);
    case 2: return kda_launch_dt<kKdaMaterialize>(p, s);
    case 3: return kda_launch_dt<kKdaFull>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rssm
