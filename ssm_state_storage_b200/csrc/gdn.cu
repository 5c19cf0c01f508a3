// gdn.cu -- Gated DeltaNet decode kernels for sm_100a: replay decode step with
// fused flush fold, standalone fold (flush / materialise), and the conventional
// full-state step.
//
// Method: checkpoint h0 plus a buffer of the latest (q, k, v, alpha, beta)
// records per (sequence, head); outputs are evaluated from h0 and the buffer
// without forming any state, and the buffer is folded into h0 once per window
// [sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…", §How ReplaySSM works,
// §Reducing state traffic and simplifying rollback].  Layer type named in
// [news.hamidun.com, "NVIDIA تقدّم ReplaySSM…", §Why hybrid models became the norm].
//
// Recurrence (gated delta rule, Yang et al. 2025), state S [DK][DV]:
//   S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,  o_t = scale S_t^T q_t.
// Unrolled from h0 over records 0..k-1 with gamma_i = prod_{m<=i} alpha_m and
// R(i,j) = prod_{j<m<=i} alpha_m (= gamma_i/gamma_j, formed as a product):
//   S_i = gamma_i h0 + sum_{j<=i} R(i,j) k_j u_j^T
//   u_i = beta_i (v_i - gamma_i h0^T k_i - sum_{j<i} R(i,j) (k_j.k_i) u_j)
//   o   = scale (gamma_{k-1} h0^T q + sum_i R(k-1,i) (k_i.q) u_i)
//   fold: h0 <- S_{k-1}.
// The only contraction with h0 is Z = [k_0 .. k_{k-1}, q]^T h0 ((k+1) x DV);
// everything else is O(k^2 DV).  The conventional step is the same algebra
// with one record and the state written back every step.
//
// CTA of 256 threads per (sequence, head); lane l of warp w holds rows
// 16w..16w+15 and columns 4l..4l+3 of the 128 x 128 tile in registers (each
// warp load reads one full 512-byte row).  Z is reduced across the 8 warps
// through shared memory in a fixed order.
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace rssm {
namespace {

constexpr int DKc = 128, DVc = 128;
constexpr int kMaxRec = 16;          // GDN buffers hold at most one window
constexpr int kRows = DKc / 8;       // rows per warp
constexpr int kZ = kMaxRec + 1;      // records + q

enum GdnMode { kGdnDecode = 0, kGdnFlush = 1, kGdnMaterialize = 2, kGdnFull = 3 };

struct GdnSmem {
  float k[kZ][DKc];       // k_0..k_{n-1}, then q
  float u[kMaxRec][DVc];  // v_i, overwritten by u_i
  float part[8][kZ][DVc];
  float z[kZ][DVc];
  float alpha[kMaxRec], beta[kMaxRec], gamma[kMaxRec];
  float ratio[kMaxRec][kMaxRec];
  float gram[kMaxRec][kMaxRec];
  float kq[kMaxRec];
  int n, act;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename TI, int MODE>
__global__ void __launch_bounds__(kThreads, 2) gdn_kernel(const GDNParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GdnSmem &S = *reinterpret_cast<GdnSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh_i = blockIdx.x;
  const int b = bh_i / p.H, h = bh_i - b * p.H;
  const size_t bh = (size_t)bh_i;

  // ---- record count n (records 0..n-1), whether to fold, whether to output
  if (tid == 0) {
    int n = 1, act = 1, ok = 1;
    if (MODE == kGdnFull) {
      ok = 1;
      act = !(p.limit && p.step_index >= p.limit[b]);
    } else {
      const int n0 = p.len[bh];
      if (MODE == kGdnDecode) {
        ok = n0 >= 0 && n0 < p.L;
        n = n0 + 1;
        act = 1;
      } else {
        ok = n0 >= 0 && n0 <= p.cap;
        n = n0;
        act = MODE == kGdnMaterialize ? 1 : (n0 >= p.L || (p.force && n0 > 0));
      }
      if (!ok) report(p.status, RSSM_ERR_STATE);
    }
    S.n = ok ? n : -1;
    S.act = act;
  }
  __syncthreads();
  const int n = S.n;
  if (n < 0 || !S.act) return;
  constexpr bool kOut = (MODE == kGdnDecode || MODE == kGdnFull);
  const bool fold = (MODE == kGdnDecode) ? (n == p.L) : true;
  const int nz = kOut ? n + 1 : n;  // rows of Z: records (+ q)

  // ---- checkpoint tile into registers (rows 16w+rho, cols 4l..4l+3)
  float *state = (MODE == kGdnFull) ? p.S + bh * (DKc * DVc) : p.h0 + bh * (DKc * DVc);
  float4 hv[kRows];
#pragma unroll
  for (int rho = 0; rho < kRows; ++rho)
    hv[rho] = ld_stream(state + (size_t)(kRows * warp + rho) * DVc + 4 * lane);

  // ---- stage records (fp32) and append this step's
  const TI *qin = static_cast<const TI *>(p.q) + b * p.bs_q + (size_t)h * DKc;
  const TI *kin = static_cast<const TI *>(p.k) + b * p.bs_k + (size_t)h * DKc;
  const TI *vin = static_cast<const TI *>(p.v) + b * p.bs_v + (size_t)h * DVc;
  TI *qb = static_cast<TI *>(p.qbuf) + bh * p.cap * DKc;
  TI *kb = static_cast<TI *>(p.kbuf) + bh * p.cap * DKc;
  TI *vb = static_cast<TI *>(p.vbuf) + bh * p.cap * DVc;
  const bool append = (MODE == kGdnDecode) && !fold;
  for (int idx = tid; idx < n * DKc; idx += kThreads) {
    const int i = idx / DKc, c = idx - i * DKc;
    const bool cur = kOut && i == n - 1;
    if (cur) {
      const TI kv = kin[c], vv = vin[c];
      S.k[i][c] = to_f32(kv);
      S.u[i][c] = to_f32(vv);
      if (append) {
        kb[(size_t)i * DKc + c] = kv;
        vb[(size_t)i * DVc + c] = vv;
        qb[(size_t)i * DKc + c] = qin[c];
      }
    } else {
      S.k[i][c] = to_f32(kb[(size_t)i * DKc + c]);
      S.u[i][c] = to_f32(vb[(size_t)i * DVc + c]);
    }
  }
  if (kOut)
    for (int c = tid; c < DKc; c += kThreads) S.k[n][c] = to_f32(qin[c]);
  if (tid < n) {
    float a, be;
    if (kOut && tid == n - 1) {
      a = p.alpha[b * p.bs_a + h];
      be = p.beta[b * p.bs_b + h];
      if (append) {
        p.abuf[bh * p.cap + tid] = a;
        p.bbuf[bh * p.cap + tid] = be;
      }
    } else {
      a = p.abuf[bh * p.cap + tid];
      be = p.bbuf[bh * p.cap + tid];
    }
    S.alpha[tid] = a;
    S.beta[tid] = be;
  }
  __syncthreads();

  // ---- partial Z over this warp's 16 rows; key Gram matrix, k.q, decays
  for (int i = 0; i < nz; ++i) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t = 0; t < kRows / 4; ++t) {
      const float4 kr = *reinterpret_cast<const float4 *>(&S.k[i][kRows * warp + 4 * t]);
      const float kk[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 hr = hv[4 * t + e];
        acc.x = fmaf(kk[e], hr.x, acc.x);
        acc.y = fmaf(kk[e], hr.y, acc.y);
        acc.z = fmaf(kk[e], hr.z, acc.z);
        acc.w = fmaf(kk[e], hr.w, acc.w);
      }
    }
    *reinterpret_cast<float4 *>(&S.part[warp][i][4 * lane]) = acc;
  }
  // pairs (j, i), j < i < n: k_j.k_i ; and (i, q): k_i.q
  const int npair = n * (n - 1) / 2 + (kOut ? n : 0);
  for (int pr = warp; pr < npair; pr += 8) {
    int i, j;
    bool isq = false;
    if (pr < n * (n - 1) / 2) {  // row-major over the strict lower triangle
      i = 1;
      int rem = pr;
      while (rem >= i) { rem -= i; ++i; }
      j = rem;
    } else {
      i = pr - n * (n - 1) / 2;
      j = n;  // q
      isq = true;
    }
    float acc = 0.f;
    for (int c = lane; c < DKc; c += 32) acc = fmaf(S.k[j][c], S.k[i][c], acc);
    acc = warp_sum(acc);
    if (lane == 0) {
      if (isq) S.kq[i] = acc;
      else S.gram[i][j] = acc;
    }
  }
  if (tid < n * n) {
    const int i = tid / n, j = tid - (tid / n) * n;
    if (j <= i) {
      float r = 1.f;
      for (int m = j + 1; m <= i; ++m) r *= S.alpha[m];
      S.ratio[i][j] = r;
    }
  }
  if (tid < n) {
    float g = 1.f;
    for (int m = 0; m <= tid; ++m) g *= S.alpha[m];
    S.gamma[tid] = g;
  }
  __syncthreads();

  // ---- Z = sum of the 8 warp partials (fixed order)
  for (int idx = tid; idx < nz * DVc; idx += kThreads) {
    const int i = idx / DVc, c = idx - i * DVc;
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) z += S.part[w][i][c];
    S.z[i][c] = z;
  }
  __syncthreads();

  // ---- u by forward substitution, one column per thread; then the output
  if (tid < DVc) {
    const int c = tid;
    for (int i = 0; i < n; ++i) {
      float u = S.u[i][c] - S.gamma[i] * S.z[i][c];
      for (int j = 0; j < i; ++j) u -= S.ratio[i][j] * S.gram[i][j] * S.u[j][c];
      S.u[i][c] = S.beta[i] * u;
    }
    if (kOut) {
      float o = S.gamma[n - 1] * S.z[n][c];
      for (int i = 0; i < n; ++i) o = fmaf(S.ratio[n - 1][i] * S.kq[i], S.u[i][c], o);
      p.y[b * p.bs_y + (size_t)h * DVc + c] = p.scale * o;
    }
  }

  if (fold) {
    __syncthreads();
    // h0 <- gamma_{n-1} h0 + sum_i R(n-1,i) k_i u_i^T
    const float gl = n > 0 ? S.gamma[n - 1] : 1.f;
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho) {
      hv[rho].x *= gl;
      hv[rho].y *= gl;
      hv[rho].z *= gl;
      hv[rho].w *= gl;
    }
    for (int i = 0; i < n; ++i) {
      const float r = S.ratio[n - 1][i];
      const float4 ui = *reinterpret_cast<const float4 *>(&S.u[i][4 * lane]);
#pragma unroll
      for (int rho = 0; rho < kRows; ++rho) {
        const float kr = r * S.k[i][kRows * warp + rho];
        hv[rho].x = fmaf(kr, ui.x, hv[rho].x);
        hv[rho].y = fmaf(kr, ui.y, hv[rho].y);
        hv[rho].z = fmaf(kr, ui.z, hv[rho].z);
        hv[rho].w = fmaf(kr, ui.w, hv[rho].w);
      }
    }
    float *dst = (MODE == kGdnMaterialize) ? p.S_out + bh * (DKc * DVc) : state;
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho)
      st_stream(dst + (size_t)(kRows * warp + rho) * DVc + 4 * lane, hv[rho]);
  }
  if (tid == 0 && (MODE == kGdnDecode || MODE == kGdnFlush)) p.len[bh] = fold ? 0 : n;
}

template <typename TI, int MODE>
cudaError_t launch(const GDNParams &p, cudaStream_t s) {
  const size_t smem = sizeof(GdnSmem);
  cudaError_t e = cudaFuncSetAttribute(gdn_kernel<TI, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gdn_kernel<TI, MODE><<<(unsigned)(p.B * p.H), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_dt(const GDNParams &p, cudaStream_t s) {
  return p.in_bf16 ? launch<__nv_bfloat16, MODE>(p, s) : launch<float, MODE>(p, s);
}

}  // namespace

bool gdn_supported(int DK, int DV) { return DK == DKc && DV == DVc; }

cudaError_t gdn_launch_decode(const GDNParams &p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  return launch_dt<kGdnDecode>(p, s);
}

cudaError_t gdn_launch_fold(const GDNParams &p, int mode, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  if (mode == kFoldFlush) return launch_dt<kGdnFlush>(p, s);
  if (mode == kFoldMaterialize) return launch_dt<kGdnMaterialize>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t gdn_launch_full(const GDNParams &p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  return launch_dt<kGdnFull>(p, s);
}

}  // namespace rssm
