// gdn.cu -- Gated DeltaNet kernels for sm_100a: replay decode step with fused
// flush fold, standalone fold (flush / materialise / commit), and the
// speculative verify round.  (The conventional full-state step is the
// one-decay case of the delta-rule step in kda.cu.)
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
#include "pipeline.cuh"
#include "umma.cuh"

namespace rssm {
namespace {

constexpr int DKc = 128, DVc = 128;
constexpr int kMaxRec = kMaxCap;     // a window plus the tail of a speculative round
constexpr int kRows = DKc / 8;       // rows per warp

enum GdnMode { kGdnFlush = 1, kGdnMaterialize = 2, kGdnCommit = 4 };

// Eight consecutive shared-memory elements (16-byte aligned for bf16, 32 for
// fp32) as fp32.
template <typename T>
__device__ __forceinline__ void ld8_smem(const T *p, float (&v)[8]) {
  if constexpr (sizeof(T) == 4) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 4);
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w;
    v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
  } else {
    const uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = to_f32(e[i]);
  }
}

// Shared memory of the fold-only kernel: up to kMaxRec records.
struct GdnSmem {
  float k[kMaxRec][DKc];  // keys
  float u[kMaxRec][DVc];  // v_i, overwritten by u_i
  float part[8][kMaxRec][DVc];
  float z[kMaxRec][DVc];
  float alpha[kMaxRec], beta[kMaxRec], gamma[kMaxRec];
  float ratio[kMaxRec][kMaxRec];
  float gram[kMaxRec][kMaxRec];
  int n, act;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Fold-only kernel, one CTA of 256 threads per (sequence, head): the buffered
// records' corrections u_i by forward substitution from h0, then the fold
// h0 <- gamma h0 + sum_i R(n-1,i) k_i u_i^T.  MODE kGdnFlush: where len >= L
// (or len > 0 with force); kGdnCommit: len += accepted, fold where it reaches
// L; kGdnMaterialize: S_out = the fold, state untouched.
template <typename TI, int MODE>
__global__ void __launch_bounds__(kThreads, 2) gdn_kernel(const GDNParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GdnSmem &S = *reinterpret_cast<GdnSmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh_i = blockIdx.x;
  const int b = bh_i / p.H;
  const size_t bh = (size_t)bh_i;

  // ---- record count n (records 0..n-1), whether to fold
  if (tid == 0) {
    int n, act, ok;
    const int n0 = p.len[bh];
    if (MODE == kGdnCommit) {  // len += accepted; fold when it reaches the window
      const int a = p.acc[b];
      ok = n0 >= 0 && n0 < p.L && a >= 0 && a <= p.draft_max && n0 + a <= p.cap;
      n = n0 + a;
      act = n >= p.L;
      if (ok && !act) p.len[bh] = n;
    } else {
      ok = n0 >= 0 && n0 <= p.cap;
      n = n0;
      act = MODE == kGdnMaterialize ? 1 : (n0 >= p.L || (p.force && n0 > 0));
    }
    if (!ok) report(p.status, RSSM_ERR_STATE);
    S.n = ok ? n : -1;
    S.act = act;
  }
  __syncthreads();
  const int n = S.n;
  if (n < 0 || !S.act) return;

  // ---- checkpoint tile into registers (rows 16w+rho, cols 4l..4l+3)
  float *state = p.h0 + bh * (DKc * DVc);
  float4 hv[kRows];
#pragma unroll
  for (int rho = 0; rho < kRows; ++rho)
    hv[rho] = ld_stream(state + (size_t)(kRows * warp + rho) * DVc + 4 * lane);

  // ---- stage the records (fp32)
  const TI *kb = static_cast<const TI *>(p.kbuf) + bh * p.cap * DKc;
  const TI *vb = static_cast<const TI *>(p.vbuf) + bh * p.cap * DVc;
  for (int idx = tid; idx < n * DKc; idx += kThreads) {
    const int i = idx / DKc, c = idx - i * DKc;
    S.k[i][c] = to_f32(kb[(size_t)i * DKc + c]);
    S.u[i][c] = to_f32(vb[(size_t)i * DVc + c]);
  }
  if (tid < n) {
    S.alpha[tid] = p.abuf[bh * p.cap + tid];
    S.beta[tid] = p.bbuf[bh * p.cap + tid];
  }
  __syncthreads();

  // ---- partial Z = [k_0..k_{n-1}]^T h0 over this warp's 16 rows; key Gram
  // matrix and decay ratios
  for (int i = 0; i < n; ++i) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int t = 0; t < kRows / 4; ++t) {
      const float4 kr = *reinterpret_cast<const float4 *>(&S.k[i][kRows * warp + 4 * t]);
      const float kk[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) acc = fma4x(kk[e], hv[4 * t + e], acc);
    }
    *reinterpret_cast<float4 *>(&S.part[warp][i][4 * lane]) = acc;
  }
  // pairs (j, i), j < i < n, row-major over the strict lower triangle
  const int npair = n * (n - 1) / 2;
  for (int pr = warp; pr < npair; pr += 8) {
    int i = 1, rem = pr;
    while (rem >= i) {
      rem -= i;
      ++i;
    }
    const int j = rem;
    float acc = 0.f;
    for (int c = lane; c < DKc; c += 32) acc = fmaf(S.k[j][c], S.k[i][c], acc);
    acc = warp_sum(acc);
    if (lane == 0) S.gram[i][j] = acc;
  }
  for (int e = tid; e < n * n; e += kThreads) {
    const int i = e / n, j = e - (e / n) * n;
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
  for (int idx = tid; idx < n * DVc; idx += kThreads) {
    const int i = idx / DVc, c = idx - i * DVc;
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) z += S.part[w][i][c];
    S.z[i][c] = z;
  }
  __syncthreads();

  // ---- u by forward substitution, one column per thread
  if (tid < DVc) {
    const int c = tid;
    for (int i = 0; i < n; ++i) {
      float u = S.u[i][c] - S.gamma[i] * S.z[i][c];
      for (int j = 0; j < i; ++j) u -= S.ratio[i][j] * S.gram[i][j] * S.u[j][c];
      S.u[i][c] = S.beta[i] * u;
    }
  }
  __syncthreads();

  // ---- h0 <- gamma_{n-1} h0 + sum_i R(n-1,i) k_i u_i^T
  const float gl = n > 0 ? S.gamma[n - 1] : 1.f;
#pragma unroll
  for (int rho = 0; rho < kRows; ++rho) hv[rho] = mul4x(gl, hv[rho]);
  for (int i = 0; i < n; ++i) {
    const float r = S.ratio[n - 1][i];
    const float4 ui = *reinterpret_cast<const float4 *>(&S.u[i][4 * lane]);
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho) hv[rho] = fma4x(r * S.k[i][kRows * warp + rho], ui, hv[rho]);
  }
  float *dst = (MODE == kGdnMaterialize) ? p.S_out + bh * (DKc * DVc) : state;
#pragma unroll
  for (int rho = 0; rho < kRows; ++rho)
    st_stream(dst + (size_t)(kRows * warp + rho) * DVc + 4 * lane, hv[rho]);
  if (tid == 0 && (MODE == kGdnFlush || MODE == kGdnCommit)) p.len[bh] = 0;
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

// ============================================================ decode step
// Persistent, warp-specialised replay decode step (one CTA of 320 threads
// per SM).  Work item = one (sequence, head).  Warp 8 streams the item's
// checkpoint as two 32 KiB half-tiles (rows 0-63, 64-127) with bulk copies
// into a ring of shared-memory slots; warp 9 stages the item's small inputs
// and bulk-copies its buffered k and u records, up to NR items ahead; warps
// 0-3 consume half-tile 0 and warps 4-7 half-tile 1 (16 rows x 4 columns per
// thread, held in registers so the slot is freed at once).
//
// With R_i = prod_{i<m<k} alpha_m, gamma = prod_{m<k} alpha_m (records
// 0..k-1, record k-1 = this step's) and the cached u_0..u_{k-2}:
//   z  = h0^T k_{k-1},   zq = h0^T q
//   u_{k-1} = beta_{k-1} (v_{k-1} - gamma z - sum_{j<k-1} R_j (k_j.k_{k-1}) u_j)
//   o  = scale (gamma zq + sum_{i<k} R_i (k_i.q) u_i)
//   flush (k = window): h0 <- gamma h0 + sum_{i<k} R_i k_i u_i^T.

namespace {

constexpr int kHalfRows = DKc / 2;                       // rows per half-tile
constexpr int kHalfBytes = kHalfRows * DVc * 4;          // 32 KiB

struct GdnLayout {
  int NS, NR, L;
  int off_bars, off_recK, off_recU, off_stage, off_db, off_single, off_umma, off_ring, total;
  int stage_floats, db_floats;
  __host__ static int a128(int v) { return (v + 127) & ~127; }
  // mma: the flush fold's operands (three split terms of the weighted
  // corrections, 128 x 16 bf16 each, and the keys, 128 x 16) get an area
  __host__ static GdnLayout make(int L, int es, int budget, bool mma = false) {
    GdnLayout d;
    d.L = L;
    // stage: q, kc, v [128] fp32 | alpha [L] | beta | hdr(2 ints)
    d.stage_floats = 3 * 128 + ((L + 3) & ~3) + 4;
    // per item, double-buffered: R [L] | kk [L] | kq [L] | gamma,pad [4] | Kf [L][128]
    d.db_floats = 3 * ((L + 3) & ~3) + 4 + L * 128;
    for (d.NR = 3; d.NR >= 1; --d.NR) {
      int o = 0;
      d.off_bars = o;
      o += a128(8 * (2 * 8 + 2 * 4) + 8 + 4);  // ring, records, fold MMA, tensor-memory base
      d.off_recK = o;
      o += a128(d.NR * L * DKc * es);
      d.off_recU = o;
      o += a128(d.NR * L * DVc * 4);
      d.off_stage = o;
      o += a128(d.NR * d.stage_floats * 4);
      d.off_db = o;
      o += a128(2 * d.db_floats * 4);
      d.off_single = o;  // part [8][2][128] | ucur [128]
      o += a128((8 * 2 * 128 + 128) * 4);
      d.off_umma = o;
      o += mma ? 4 * 128 * 32 : 0;
      d.off_ring = o;
      d.NS = (budget - o) / kHalfBytes;
      if (d.NS > 8) d.NS = 8;
      if (d.NS >= 4) {
        d.total = o + d.NS * kHalfBytes;
        return d;
      }
    }
    d.NS = 0;
    return d;
  }
  // Two consumer groups (bf16 keys, tensor-core fold): per group the decay
  // ratios and key dots R | kk | kq | gamma, the partial sums [4][2][128] and
  // the current correction [128], and a fold operand area; a ring of exactly
  // 4 half-tiles and an even number of record buffers (4, else 2), so that
  // each group owns its slots and buffers and waits on them in its own order.
  __host__ static GdnLayout make2(int L, int budget) {
    GdnLayout d;
    d.L = L;
    d.stage_floats = 3 * 128 + ((L + 3) & ~3) + 4;
    d.db_floats = 3 * ((L + 3) & ~3) + 4;
    for (d.NR = 4; d.NR >= 2; d.NR -= 2) {
      int o = 0;
      d.off_bars = o;
      o += a128(8 * (2 * 8 + 2 * 4) + 2 * 8 + 4);  // ring, records, two fold MMAs, TMEM base
      d.off_recK = o;
      o += a128(d.NR * L * DKc * 2);
      d.off_recU = o;
      o += a128(d.NR * L * DVc * 4);
      d.off_stage = o;
      o += a128(d.NR * d.stage_floats * 4);
      d.off_db = o;
      o += a128(2 * d.db_floats * 4);
      d.off_single = o;
      o += a128(2 * (4 * 2 * 128 + 128) * 4);
      d.off_umma = o;
      o += 2 * 4 * 128 * 32;
      d.off_ring = o;
      d.NS = 4;
      d.total = o + d.NS * kHalfBytes;
      if (d.total <= budget) return d;
    }
    d.NS = 0;
    return d;
  }
};

struct GdnPtrs {
  uint64_t *full, *empty, *rfull, *rempty, *mma;
  uint32_t *tmem_slot;
  unsigned char *recK, *ring, *umma;
  float *recU, *stage, *db, *part, *ucur;
  __device__ GdnPtrs(unsigned char *smem, const GdnLayout &l) {
    full = reinterpret_cast<uint64_t *>(smem + l.off_bars);
    empty = full + 8;
    rfull = empty + 8;
    rempty = rfull + 4;
    mma = rempty + 4;
    tmem_slot = reinterpret_cast<uint32_t *>(mma + 1);
    umma = smem + l.off_umma;
    recK = smem + l.off_recK;
    recU = reinterpret_cast<float *>(smem + l.off_recU);
    stage = reinterpret_cast<float *>(smem + l.off_stage);
    db = reinterpret_cast<float *>(smem + l.off_db);
    part = reinterpret_cast<float *>(smem + l.off_single);
    ucur = part + 8 * 2 * 128;
    ring = smem + l.off_ring;
  }
};

// Shared memory of the two-group decode kernel (GdnLayout::make2).
struct Gdn2Ptrs {
  uint64_t *full, *empty, *rfull, *rempty, *mma;  // mma[2]: one per group
  uint32_t *tmem_slot;
  unsigned char *recK, *ring, *umma;
  float *recU, *stage, *db, *part, *ucur;
  __device__ Gdn2Ptrs(unsigned char *smem, const GdnLayout &l) {
    full = reinterpret_cast<uint64_t *>(smem + l.off_bars);
    empty = full + 8;
    rfull = empty + 8;
    rempty = rfull + 4;
    mma = rempty + 4;
    tmem_slot = reinterpret_cast<uint32_t *>(mma + 2);
    umma = smem + l.off_umma;
    recK = smem + l.off_recK;
    recU = reinterpret_cast<float *>(smem + l.off_recU);
    stage = reinterpret_cast<float *>(smem + l.off_stage);
    db = reinterpret_cast<float *>(smem + l.off_db);
    part = reinterpret_cast<float *>(smem + l.off_single);  // [2][4][2][128]
    ucur = part + 2 * 4 * 2 * 128;                           // [2][128]
    ring = smem + l.off_ring;
  }
};

// Stager warp: all loads of item `it` first (none depends on the length:
// every alpha slot of the window is read), then shared-memory writes, then
// (lane 0) the bulk copies of the buffered k and u records.
template <typename TI, typename Ptrs>
__device__ __forceinline__ bool gdn_stage(const GDNParams &p, const GdnLayout &lay,
                                          const Ptrs &S, int item, int it, int lane,
                                          volatile int *abort_flag) {
  const int L = lay.L;
  const int rb = it % lay.NR;
  const uint32_t rphase = (it / lay.NR) & 1;
  bool ok = true;
  if (lane == 0) ok = mbar_wait(&S.rempty[rb], rphase ^ 1, kWaitLimitNs, abort_flag) && !*abort_flag;
  if (!__shfl_sync(0xffffffffu, (int)ok, 0)) return false;
  const int b = item / p.H, h = item - (item / p.H) * p.H;
  const size_t bh = (size_t)item;
  const TI *qin = static_cast<const TI *>(p.q) + b * p.bs_q + (size_t)h * DKc;
  const TI *kin = static_cast<const TI *>(p.k) + b * p.bs_k + (size_t)h * DKc;
  const TI *vin = static_cast<const TI *>(p.v) + b * p.bs_v + (size_t)h * DVc;
  const int n0 = __ldcg(&p.len[bh]);
  float a_cur, b_cur;
  if (p.inplace) {  // the record is already in slot len: read it from there
    const size_t slot = bh * p.cap + min(max(n0, 0), L - 1);  // stays in bounds
    qin = static_cast<const TI *>(p.qbuf) + slot * DKc;
    kin = static_cast<const TI *>(p.kbuf) + slot * DKc;
    vin = static_cast<const TI *>(p.vbuf) + slot * DVc;
    a_cur = __ldcg(&p.abuf[slot]);
    b_cur = __ldcg(&p.bbuf[slot]);
  } else {
    a_cur = p.alpha[b * p.bs_a + h];
    b_cur = p.beta[b * p.bs_b + h];
  }
  const float a_rec = lane < L ? __ldcg(&p.abuf[bh * p.cap + lane]) : 0.f;
  TI qv[4], kv[4], vv[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    qv[u] = qin[lane + 32 * u];
    kv[u] = kin[lane + 32 * u];
    vv[u] = vin[lane + 32 * u];
  }
  const bool bad = n0 < 0 || n0 >= L;
  const int k = min(max(n0 + 1, 1), L);  // copies stay in bounds even for a bad length
  float *st = S.stage + rb * lay.stage_floats;
  TI *rK = reinterpret_cast<TI *>(S.recK) + (size_t)rb * L * DKc;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane + 32 * u;
    st[c] = to_f32(qv[u]);
    st[128 + c] = to_f32(kv[u]);
    st[256 + c] = to_f32(vv[u]);
    rK[(k - 1) * DKc + c] = kv[u];
  }
  float *alpha = st + 384;
  if (lane < k) alpha[lane] = lane == k - 1 ? a_cur : a_rec;
  float *tail = alpha + ((L + 3) & ~3);
  if (lane == 0) {
    tail[0] = b_cur;
    reinterpret_cast<int *>(tail)[1] = n0;
    reinterpret_cast<int *>(tail)[2] = bad;
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    const uint32_t bytesK = (k - 1) * DKc * sizeof(TI), bytesU = (k - 1) * DVc * 4;
    mbar_arrive_expect_tx(&S.rfull[rb], bytesK + bytesU);
    if (k > 1) {
      bulk_g2s(rK, static_cast<const TI *>(p.kbuf) + bh * p.cap * DKc, bytesK, &S.rfull[rb]);
      bulk_g2s(S.recU + (size_t)rb * L * DVc, p.ubuf + bh * p.cap * DVc, bytesU, &S.rfull[rb]);
    }
  }
  return true;
}

// Tensor-core flush fold (bf16 keys): the rank-k increment
//   D[c][row] = sum_i (R_i u_i[c]) k_i[row]          (M = DV = 128, N' = DK = 128, K = 16)
// as a bf16 MMA with an fp32 accumulator in tensor memory; the fp32 products
// R_i u_i are split into three bf16 terms (three MMAs), the keys are exact in
// bf16.  Epilogue h0[row][c] <- gamma h0[row][c] + D[c][row] with lane c per
// thread: warps 0-3 take rows 0-63 (half-tile 0), warps 4-7 rows 64-127.
template <typename TI>
__device__ __forceinline__ void gdn_build_fold_operands(unsigned char *ua, const float *rU,
                                                        const float *ucur, const float *R,
                                                        const TI *rK, int k, int tid,
                                                        int nthr = kThreads) {
  unsigned char *ub = ua + 3 * 128 * 32;
  for (int e = tid; e < 128 * 8; e += nthr) {
    const int c = e % 128, q = e / 128, i0 = 2 * q, i1 = i0 + 1;
    auto uval = [&](int i) -> float {
      return i < k - 1 ? rU[i * DVc + c] : (i == k - 1 ? ucur[c] : 0.f);
    };
    const float v0 = i0 < k ? R[i0] * uval(i0) : 0.f, v1 = i1 < k ? R[i1] * uval(i1) : 0.f;
    __nv_bfloat162 h, m, l, kb;
    umma::split3_bf16(v0, h.x, m.x, l.x);
    umma::split3_bf16(v1, h.y, m.y, l.y);
    const uint32_t o = umma::kmajor_offset(c, i0);
    *reinterpret_cast<__nv_bfloat162 *>(ua + o) = h;
    *reinterpret_cast<__nv_bfloat162 *>(ua + 128 * 32 + o) = m;
    *reinterpret_cast<__nv_bfloat162 *>(ua + 2 * 128 * 32 + o) = l;
    // keys: row index c here runs over d_k
    kb.x = i0 < k ? rK[i0 * DKc + c] : TI{};
    kb.y = i1 < k ? rK[i1 * DKc + c] : TI{};
    *reinterpret_cast<__nv_bfloat162 *>(ub + o) = kb;
  }
}

template <typename TI, bool MMA>
__global__ void __launch_bounds__(kThreads + 64, 1) gdn_decode_kernel(const GDNParams p,
                                                                   const GdnLayout lay) {
  static_assert(!MMA || std::is_same<TI, __nv_bfloat16>::value, "tensor-core fold: bf16 keys");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  const GdnPtrs S(smem, lay);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nitems = p.B * p.H;
  const int L = lay.L;

  if (tid == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 4);  // the 4 consumer warps of a half-tile
    }
    for (int r = 0; r < 4; ++r) {
      mbar_init(&S.rfull[r], 1);
      mbar_init(&S.rempty[r], 8);
    }
    mbar_init(S.mma, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if constexpr (MMA) {
    if (warp == 0) umma::alloc(S.tmem_slot, 128);
    umma::fence_before_sync();
  }
  __syncthreads();

  if (warp == 8) {  // tile producer: half-tiles in (item, half) order
    if (lane != 0) return;
    int slot = 0;
    uint32_t sphase = 0, issued = 0, parity = 0;
    bool failed = false;
    for (int item = blockIdx.x; item < nitems && !failed; item += gridDim.x) {
      for (int half = 0; half < 2; ++half) {
        if (*abort_flag || !mbar_wait(&S.empty[slot], sphase ^ 1, kWaitLimitNs, abort_flag) ||
            *abort_flag) {
          failed = true;
          break;
        }
        mbar_arrive_expect_tx(&S.full[slot], kHalfBytes);
        bulk_g2s(S.ring + slot * kHalfBytes,
                 p.h0 + (size_t)item * DKc * DVc + (size_t)half * kHalfRows * DVc, kHalfBytes,
                 &S.full[slot]);
        issued |= 1u << slot;
        parity = (parity & ~(1u << slot)) | (sphase << slot);
        if (++slot == lay.NS) {
          slot = 0;
          sphase ^= 1;
        }
      }
    }
    if (failed) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // every copy issued here lands before the warp returns (see stream_tiles)
    for (int s = 0; s < lay.NS; ++s)
      if (issued & (1u << s)) mbar_wait(&S.full[s], (parity >> s) & 1u);
    return;
  }
  if (warp == 9) {  // stager
    int it = 0;
    ArmedRecords armed;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
      const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
      if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
      if (abort_now || !gdn_stage<TI>(p, lay, S, item, it, lane, abort_flag)) {
        if (lane == 0 && !*abort_flag) {
          report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      armed.arm(it % lay.NR, (it / lay.NR) & 1);
    }
    if (lane == 0) armed.drain(S.rfull, lay.NR);  // no record copy outlives the warp
    __syncwarp();
    return;
  }

  // Consumers (uniform control flow, as in the Mamba-2 kernel).  Warp w
  // holds rows 16w..16w+15 (local rows 16(w%4).. of half-tile w/4) and
  // columns 4*lane..4*lane+3.
  const int half = warp >> 2, row0 = 16 * warp;
  uint32_t tmem = 0, n_mma = 0;
  if constexpr (MMA) {
    umma::fence_after_sync();
    tmem = *S.tmem_slot;
  }
  int it = 0;
  for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
    const int rb = it % lay.NR;
    const uint32_t rphase = (it / lay.NR) & 1;
    const int b = item / p.H, h = item - (item / p.H) * p.H;
    const size_t bh = (size_t)item;
    const float *st = S.stage + rb * lay.stage_floats;
    const float *qs = st, *ks = st + 128, *vs = st + 256, *alpha = st + 384;
    const float *tail = alpha + ((L + 3) & ~3);
    const TI *rK = reinterpret_cast<const TI *>(S.recK) + (size_t)rb * L * DKc;
    const float *rU = S.recU + (size_t)rb * L * DVc;
    float *db = S.db + (it & 1) * lay.db_floats;
    float *R = db, *kk = db + ((L + 3) & ~3), *kq = kk + ((L + 3) & ~3);
    float *gam = kq + ((L + 3) & ~3);
    float *Kf = gam + 4;

    const bool got = mbar_wait(&S.rfull[rb], rphase, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(1, kThreads, !got || *abort_flag)) break;
    const int n0 = reinterpret_cast<const int *>(tail)[1];
    const int pos = 2 * it + half;  // this warp's half-tile in the producer's order
    if (reinterpret_cast<const int *>(tail)[2]) {
      if (tid == 0) report(p.status, RSSM_ERR_STATE);
      if (!mbar_wait(&S.full[pos % lay.NS], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[pos % lay.NS]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.rempty[rb]);
      continue;
    }
    const int k = n0 + 1;
    const bool flush = (k == L);
    const float beta = tail[0];

    // ---- P1: appends (an in-place step's record is in its slot already),
    // decay ratios, k_j.k and k_i.q, fp32 keys for the fold
    if (!flush && !p.inplace) {
      TI *qb = static_cast<TI *>(p.qbuf) + (bh * p.cap + k - 1) * DKc;
      TI *kb = static_cast<TI *>(p.kbuf) + (bh * p.cap + k - 1) * DKc;
      TI *vb = static_cast<TI *>(p.vbuf) + (bh * p.cap + k - 1) * DVc;
      if (tid < 128) {
        qb[tid] = from_f32<TI>(qs[tid]);
        kb[tid] = rK[(k - 1) * DKc + tid];
      } else {
        vb[tid - 128] = from_f32<TI>(vs[tid - 128]);
      }
      if (tid == 0) {
        p.abuf[bh * p.cap + k - 1] = alpha[k - 1];
        p.bbuf[bh * p.cap + k - 1] = beta;
      }
    }
    if (warp == 7) {  // R_i = prod_{i<m<k} alpha_m (lane i), gamma: fp64 suffix-product scan
      double pr = lane < k ? (double)alpha[lane] : 1.0;  // inclusive: prod_{m >= lane}
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_down_sync(0xffffffffu, pr, o);
        if (lane + o < 32) pr *= t;
      }
      const double nxt = __shfl_down_sync(0xffffffffu, pr, 1);  // prod_{m > lane}
      if (lane < k) R[lane] = (float)(lane + 1 < 32 ? nxt : 1.0);
      if (lane == 0) gam[0] = (float)pr;
    }
    {
      // 2k-1 dot products of 128: k_j.k_{k-1} (j < k-1) then k_i.q (i < k);
      // 8 threads per dot (one pass for up to 32 dots), thread j of a dot
      // takes the 8-element chunks j and j + 8 with 16-byte key loads
      const int ndot = 2 * k - 1;
      for (int base = 0; base < ndot; base += kThreads / 8) {
        const int d = base + (tid >> 3), j = tid & 7;
        // products in fp32 (exact for bf16 inputs: 8 x 8 significant bits),
        // sums in fp64 over two independent chains
        double acc = 0.0, acc1 = 0.0;
        if (d < ndot) {
          const int i = d < k - 1 ? d : d - (k - 1);
          const float *other = d < k - 1 ? ks : qs;
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            const int c0 = 8 * (j + 8 * m);
            float kv[8], ov[8];
            ld8_smem(rK + i * DKc + c0, kv);
            ld8_smem(other + c0, ov);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              acc += (double)(kv[e] * ov[e]);
              acc1 += (double)(kv[e + 1] * ov[e + 1]);
            }
          }
          acc += acc1;
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
        if (d < ndot && j == 0) {
          if (d < k - 1) kk[d] = (float)acc;
          else kq[d - (k - 1)] = (float)acc;
        }
      }
    }
    if (flush && !MMA)
      for (int e = tid; e < k * DKc; e += kThreads) Kf[e] = to_f32(rK[e]);

    // ---- P2: this warp's 16 rows into registers; partial h0^T k and h0^T q
    const int sl = pos % lay.NS;
    if (!mbar_wait(&S.full[sl], (pos / lay.NS) & 1, p.wait_ns, abort_flag)) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    float4 hv[16];
    const float *tile = reinterpret_cast<const float *>(S.ring + sl * kHalfBytes);
#pragma unroll
    for (int rho = 0; rho < 16; ++rho)
      hv[rho] = *reinterpret_cast<const float4 *>(tile + (16 * (warp & 3) + rho) * DVc + 4 * lane);
    const bool mma_fold = MMA && flush;
    if (!mma_fold) {  // the tensor-core fold reads the half-tile again in its epilogue
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[sl]);
    }
    {
      float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 k4 = *reinterpret_cast<const float4 *>(&ks[row0 + 4 * t]);
        const float4 q4 = *reinterpret_cast<const float4 *>(&qs[row0 + 4 * t]);
        const float kr[4] = {k4.x, k4.y, k4.z, k4.w}, qr[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float4 x = hv[4 * t + e];
          pk.x = fmaf(kr[e], x.x, pk.x);
          pk.y = fmaf(kr[e], x.y, pk.y);
          pk.z = fmaf(kr[e], x.z, pk.z);
          pk.w = fmaf(kr[e], x.w, pk.w);
          pq.x = fmaf(qr[e], x.x, pq.x);
          pq.y = fmaf(qr[e], x.y, pq.y);
          pq.z = fmaf(qr[e], x.z, pq.z);
          pq.w = fmaf(qr[e], x.w, pq.w);
        }
      }
      *reinterpret_cast<float4 *>(&S.part[(warp * 2 + 0) * 128 + 4 * lane]) = pk;
      *reinterpret_cast<float4 *>(&S.part[(warp * 2 + 1) * 128 + 4 * lane]) = pq;
    }
    bar_sync(1, kThreads);
    // ---- P3 + P4: thread pair (2c, 2c+1) owns column c.  The even thread
    // sums the 8 warps' partials of z = h0^T k, the odd one those of
    // zq = h0^T q (fixed order), and they swap; each then runs over the
    // older records of its parity, one load of u_j serving both the
    // correction's and the output's sum, and the pair adds the two halves.
    // Both threads hold u and o; no barrier is needed (the next item starts
    // with one).
    {
      const int c = tid >> 1, par = tid & 1;
      const float g = gam[0];
      float zc = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) zc += S.part[(w * 2 + par) * 128 + c];
      const float zo = __shfl_xor_sync(0xffffffffu, zc, 1);
      const float z = par ? zo : zc, zq = par ? zc : zo;
      float su = 0.f, so = 0.f;
      for (int j = par; j < k - 1; j += 2) {
        const float uj = rU[j * DVc + c], rj = R[j];
        su = fmaf(rj * kk[j], uj, su);
        so = fmaf(rj * kq[j], uj, so);
      }
      su += __shfl_xor_sync(0xffffffffu, su, 1);
      so += __shfl_xor_sync(0xffffffffu, so, 1);
      const float u = beta * ((vs[c] - g * z) - su);
      const float o = fmaf(kq[k - 1], u, fmaf(g, zq, so));  // R_{k-1} = 1
      if (par == 0) {
        if (!flush) p.ubuf[(bh * p.cap + k - 1) * DVc + c] = u;
        S.ucur[c] = u;
      } else {
        p.y[b * p.bs_y + (size_t)h * DVc + c] = p.scale * o;
      }
    }
    if (flush) bar_sync(1, kThreads);  // the fold reads every column's u
    if constexpr (MMA) {
      if (mma_fold) {
        // ---- P5 on the tensor cores: the previous fold's accumulator reads
        // finished before the barrier (wait::ld, fence)
        gdn_build_fold_operands<TI>(S.umma, rU, S.ucur, R, rK, k, tid);
        fence_proxy_async_smem();
        umma::fence_before_sync();
        bar_sync(1, kThreads);
        if (tid == 0) {
          umma::fence_after_sync();
          const uint32_t id = umma::idesc_bf16_f32(128, 128);
          const uint64_t bd = umma::smem_desc(S.umma + 3 * 128 * 32);
#pragma unroll
          for (int t3 = 0; t3 < 3; ++t3)
            umma::mma_bf16(tmem, umma::smem_desc(S.umma + t3 * 128 * 32), bd, id, t3 > 0);
          umma::commit(S.mma);
        }
        const bool done = mbar_wait(S.mma, n_mma & 1u, p.wait_ns, abort_flag);
        ++n_mma;
        if (!done) {
          if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        umma::fence_after_sync();
        const int c = 32 * (warp & 3) + lane, rbase = 64 * half;
        const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)rbase;
        const float g = gam[0];
        float *dst = p.h0 + bh * (DKc * DVc);
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          float d[32];
          umma::ld32(taddr + c0, d);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int r = c0 + i;  // row within the half-tile
            dst[(size_t)(rbase + r) * DVc + c] = fmaf(g, tile[r * DVc + c], d[i]);
          }
        }
        umma::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[sl]);
      }
    }
    // ---- P5 (flush): h0 <- gamma h0 + sum_i R_i k_i u_i^T, written once
    if (flush && !MMA) {
      const float g = gam[0];
#pragma unroll
      for (int rho = 0; rho < 16; ++rho) hv[rho] = mul4x(g, hv[rho]);
      for (int i = 0; i < k; ++i) {
        const float4 ui = *reinterpret_cast<const float4 *>(
            i < k - 1 ? &rU[i * DVc + 4 * lane] : &S.ucur[4 * lane]);
        const float ri = R[i];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float4 k4 = *reinterpret_cast<const float4 *>(&Kf[i * DKc + row0 + 4 * t]);
          const float kr[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) hv[4 * t + e] = fma4x(ri * kr[e], ui, hv[4 * t + e]);
        }
      }
      float *dst = p.h0 + bh * (DKc * DVc);
#pragma unroll
      for (int rho = 0; rho < 16; ++rho)
        st_stream(dst + (size_t)(row0 + rho) * DVc + 4 * lane, hv[rho]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.rempty[rb]);
    if (tid == 0) p.len[bh] = flush ? 0 : k;
  }
  if constexpr (MMA) {
    if (tid == 0 && n_mma > 0) mbar_wait(S.mma, (n_mma - 1) & 1u);  // no MMA outlives the memory
    umma::fence_before_sync();
    bar_sync(1, kThreads);
    umma::fence_after_sync();
    if (warp == 0) umma::dealloc(tmem, 128);
  }
}


// Two consumer groups (bf16 keys, tensor-core fold).  Warps 0-3 and 4-7 take
// alternate work items of this CTA (group g: items it = g, g + 2, ...), so one
// item's latency chain (key dots, partial products, u and output, fold)
// overlaps the other group's.  Same producer, stager and ring as the kernel
// above with exactly 4 half-tile slots: item it fills slots 2(it%2) and
// 2(it%2)+1, so each group owns one pair; with an even number of record
// buffers each group also owns its buffers.  A group therefore never waits on
// a barrier phase beyond the next one of its own slots and buffers.  Within a
// group warp w (0-3) reads rows 32w..32w+31 of the tile straight from its slot
// (no register copy: the tile is used once on non-flush steps, and the fold
// epilogue reads it again from the slot); thread c of the group forms u and
// the output of column c; the fold's accumulator is this group's 128 of 256
// tensor-memory columns.
template <typename TI>
__global__ void __launch_bounds__(kThreads + 64, 1) gdn_decode2_kernel(const GDNParams p,
                                                                    const GdnLayout lay) {
  static_assert(std::is_same<TI, __nv_bfloat16>::value, "tensor-core fold: bf16 keys");
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  const Gdn2Ptrs S(smem, lay);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nitems = p.B * p.H;
  const int L = lay.L;

  if (tid == 0) {
    for (int s = 0; s < 8; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 4);  // the 4 warps of the group that owns the slot
    }
    for (int r = 0; r < 4; ++r) {
      mbar_init(&S.rfull[r], 1);
      mbar_init(&S.rempty[r], 4);
    }
    mbar_init(&S.mma[0], 1);
    mbar_init(&S.mma[1], 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) umma::alloc(S.tmem_slot, 256);
  umma::fence_before_sync();
  __syncthreads();

  if (warp == 8) {  // tile producer: half-tiles in (item, half) order, 4 slots
    if (lane != 0) return;
    int slot = 0;
    uint32_t sphase = 0, issued = 0, parity = 0;
    bool failed = false;
    for (int item = blockIdx.x; item < nitems && !failed; item += gridDim.x) {
      for (int half = 0; half < 2; ++half) {
        if (*abort_flag || !mbar_wait(&S.empty[slot], sphase ^ 1, kWaitLimitNs, abort_flag) ||
            *abort_flag) {
          failed = true;
          break;
        }
        mbar_arrive_expect_tx(&S.full[slot], kHalfBytes);
        bulk_g2s(S.ring + slot * kHalfBytes,
                 p.h0 + (size_t)item * DKc * DVc + (size_t)half * kHalfRows * DVc, kHalfBytes,
                 &S.full[slot]);
        issued |= 1u << slot;
        parity = (parity & ~(1u << slot)) | (sphase << slot);
        if (++slot == lay.NS) {
          slot = 0;
          sphase ^= 1;
        }
      }
    }
    if (failed) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    // every copy issued here lands before the warp returns
    for (int s2 = 0; s2 < lay.NS; ++s2)
      if (issued & (1u << s2)) mbar_wait(&S.full[s2], (parity >> s2) & 1u);
    return;
  }
  if (warp == 9) {  // stager
    int it = 0;
    ArmedRecords armed;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
      const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
      if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
      if (abort_now || !gdn_stage<TI>(p, lay, S, item, it, lane, abort_flag)) {
        if (lane == 0 && !*abort_flag) {
          report(p.status, RSSM_ERR_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      armed.arm(it % lay.NR, (it / lay.NR) & 1);
    }
    if (lane == 0) armed.drain(S.rfull, lay.NR);  // no record copy outlives the warp
    __syncwarp();
    return;
  }

  // Consumer group grp (warps 4grp .. 4grp+3), thread gt = column c.
  constexpr int kG = 128;  // threads per group
  const int grp = warp >> 2, gw = warp & 3, gt = tid & (kG - 1);
  const uint32_t gbar = 1 + grp;  // the group's named barrier
  umma::fence_after_sync();
  const uint32_t tmem_base = *S.tmem_slot;
  const uint32_t tmem = tmem_base + 128u * grp;  // this group's accumulator columns
  uint32_t n_mma = 0;
  float *part = S.part + grp * (4 * 2 * 128);
  float *ucur = S.ucur + grp * 128;
  unsigned char *ua = S.umma + grp * (4 * 128 * 32);
  uint64_t *mbar_mma = &S.mma[grp];
  float *db = S.db + grp * lay.db_floats;
  float *R = db, *kk = db + ((L + 3) & ~3), *kq = kk + ((L + 3) & ~3);
  float *gam = kq + ((L + 3) & ~3);

  int it = grp;
  for (int item = blockIdx.x + grp * gridDim.x; item < nitems; item += 2 * gridDim.x, it += 2) {
    const int rb = it % lay.NR;
    const uint32_t rphase = (it / lay.NR) & 1;
    const int b = item / p.H, h = item - (item / p.H) * p.H;
    const size_t bh = (size_t)item;
    const float *st = S.stage + rb * lay.stage_floats;
    const float *qs = st, *ks = st + 128, *vs = st + 256, *alpha = st + 384;
    const float *tail = alpha + ((L + 3) & ~3);
    const TI *rK = reinterpret_cast<const TI *>(S.recK) + (size_t)rb * L * DKc;
    const float *rU = S.recU + (size_t)rb * L * DVc;
    // this item's two half-tiles: slots 2 (it % 2) and 2 (it % 2) + 1, phase it / 2
    const int sl0 = 2 * (it & 1), sl1 = sl0 + 1;
    const uint32_t tphase = (it >> 1) & 1;

    const bool got = mbar_wait(&S.rfull[rb], rphase, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(gbar, kG, !got || *abort_flag)) break;
    const int n0 = reinterpret_cast<const int *>(tail)[1];
    if (reinterpret_cast<const int *>(tail)[2]) {
      if (gt == 0) report(p.status, RSSM_ERR_STATE);
      const int sl = gw < 2 ? sl0 : sl1;
      if (!mbar_wait(&S.full[sl], tphase, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.empty[sl0]);
        mbar_arrive(&S.empty[sl1]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.rempty[rb]);
      continue;
    }
    const int k = n0 + 1;
    const bool flush = (k == L);
    const float beta = tail[0];

    // ---- P1: appends (an in-place step's record is in its slot already),
    // decay ratios, k_j.k and k_i.q
    if (!flush && !p.inplace) {
      const size_t slot = bh * p.cap + k - 1;
      static_cast<TI *>(p.qbuf)[slot * DKc + gt] = from_f32<TI>(qs[gt]);
      static_cast<TI *>(p.kbuf)[slot * DKc + gt] = rK[(k - 1) * DKc + gt];
      static_cast<TI *>(p.vbuf)[slot * DVc + gt] = from_f32<TI>(vs[gt]);
      if (gt == 0) {
        p.abuf[slot] = alpha[k - 1];
        p.bbuf[slot] = beta;
      }
    }
    if (gw == 3) {  // R_i = prod_{i<m<k} alpha_m (lane i), gamma: fp64 suffix-product scan
      double pr = lane < k ? (double)alpha[lane] : 1.0;  // inclusive: prod_{m >= lane}
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_down_sync(0xffffffffu, pr, o);
        if (lane + o < 32) pr *= t;
      }
      const double nxt = __shfl_down_sync(0xffffffffu, pr, 1);  // prod_{m > lane}
      if (lane < k) R[lane] = (float)(lane + 1 < 32 ? nxt : 1.0);
      if (lane == 0) gam[0] = (float)pr;
    }
    {
      // 2k-1 <= 31 dot products of 128 (the window is at most 16):
      // k_j.k_{k-1} (j < k-1) then k_i.q (i < k); 4 threads per dot, thread j
      // of a dot takes the 8-element chunks j + 4m (16-byte key loads);
      // products in fp32 (exact for bf16 inputs), sums in fp64 over two chains
      const int ndot = 2 * k - 1, d = gt >> 2, j = gt & 3;
      double acc = 0.0, acc1 = 0.0;
      if (d < ndot) {
        const int i = d < k - 1 ? d : d - (k - 1);
        const float *other = d < k - 1 ? ks : qs;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int c0 = 8 * (j + 4 * m);
          float kv[8], ov[8];
          ld8_smem(rK + i * DKc + c0, kv);
          ld8_smem(other + c0, ov);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            acc += (double)(kv[e] * ov[e]);
            acc1 += (double)(kv[e + 1] * ov[e + 1]);
          }
        }
        acc += acc1;
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      if (d < ndot && j == 0) {
        if (d < k - 1) kk[d] = (float)acc;
        else kq[d - (k - 1)] = (float)acc;
      }
    }

    // ---- P2: partial h0^T k and h0^T q over this warp's 32 rows, read from
    // the slot (rows 64 half + 32 (gw % 2) ..)
    const int half = gw >> 1, sl = half ? sl1 : sl0;
    if (!mbar_wait(&S.full[sl], tphase, p.wait_ns, abort_flag)) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    {
      const float *tile = reinterpret_cast<const float *>(S.ring + sl * kHalfBytes) +
                          (size_t)(32 * (gw & 1)) * DVc + 4 * lane;
      const int row0 = 32 * gw;  // = 64 half + 32 (gw % 2)
      float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
#pragma unroll 2
      for (int t = 0; t < 8; ++t) {
        const float4 k4 = *reinterpret_cast<const float4 *>(&ks[row0 + 4 * t]);
        const float4 q4 = *reinterpret_cast<const float4 *>(&qs[row0 + 4 * t]);
        const float kr[4] = {k4.x, k4.y, k4.z, k4.w}, qr[4] = {q4.x, q4.y, q4.z, q4.w};
        float4 x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = *reinterpret_cast<const float4 *>(tile + (4 * t + e) * DVc);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pk = fma4x(kr[e], x[e], pk);
          pq = fma4x(qr[e], x[e], pq);
        }
      }
      *reinterpret_cast<float4 *>(&part[(gw * 2 + 0) * 128 + 4 * lane]) = pk;
      *reinterpret_cast<float4 *>(&part[(gw * 2 + 1) * 128 + 4 * lane]) = pq;
    }
    if (!flush) {  // the fold epilogue reads both half-tiles again
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.empty[sl0]);
        mbar_arrive(&S.empty[sl1]);
      }
    }
    bar_sync(gbar, kG);

    // ---- P3 + P4: thread c sums the 4 warps' partials of z = h0^T k and
    // zq = h0^T q for column c (fixed order), then one pass over the older
    // records gives both the correction's and the output's sums (one load of
    // u_j each, even and odd records in separate accumulators)
    {
      const int c = gt;
      const float g = gam[0];
      float z = 0.f, zq = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        z += part[(w * 2 + 0) * 128 + c];
        zq += part[(w * 2 + 1) * 128 + c];
      }
      float su0 = 0.f, su1 = 0.f, so0 = 0.f, so1 = 0.f;
      int jj = 0;
      for (; jj + 1 < k - 1; jj += 2) {
        const float u0 = rU[jj * DVc + c], u1 = rU[(jj + 1) * DVc + c];
        const float r0 = R[jj], r1 = R[jj + 1];
        su0 = fmaf(r0 * kk[jj], u0, su0);
        so0 = fmaf(r0 * kq[jj], u0, so0);
        su1 = fmaf(r1 * kk[jj + 1], u1, su1);
        so1 = fmaf(r1 * kq[jj + 1], u1, so1);
      }
      if (jj < k - 1) {
        const float u0 = rU[jj * DVc + c], r0 = R[jj];
        su0 = fmaf(r0 * kk[jj], u0, su0);
        so0 = fmaf(r0 * kq[jj], u0, so0);
      }
      const float u = beta * ((vs[c] - g * z) - (su0 + su1));
      const float o = fmaf(kq[k - 1], u, fmaf(g, zq, so0 + so1));  // R_{k-1} = 1
      if (!flush) p.ubuf[(bh * p.cap + k - 1) * DVc + c] = u;
      else ucur[c] = u;
      p.y[b * p.bs_y + (size_t)h * DVc + c] = p.scale * o;
    }

    if (flush) {
      // ---- P5 on the tensor cores: h0 <- gamma h0 + sum_i R_i k_i u_i^T
      bar_sync(gbar, kG);  // every column's u; the previous fold's reads are done
      gdn_build_fold_operands<TI>(ua, rU, ucur, R, rK, k, gt, kG);
      fence_proxy_async_smem();
      umma::fence_before_sync();
      bar_sync(gbar, kG);
      if (gt == 0) {
        umma::fence_after_sync();
        const uint32_t id = umma::idesc_bf16_f32(128, 128);
        const uint64_t bd = umma::smem_desc(ua + 3 * 128 * 32);
#pragma unroll
        for (int t3 = 0; t3 < 3; ++t3)
          umma::mma_bf16(tmem, umma::smem_desc(ua + t3 * 128 * 32), bd, id, t3 > 0);
        umma::commit(mbar_mma);
      }
      const bool done = mbar_wait(mbar_mma, n_mma & 1u, p.wait_ns, abort_flag);
      ++n_mma;
      if (!done) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
        *abort_flag = 1;
      }
      umma::fence_after_sync();
      // epilogue: lane = column c = 32 gw + lane, all 128 rows, 32 at a time
      if (!mbar_wait(&S.full[half ? sl0 : sl1], tphase, p.wait_ns, abort_flag)) {
        if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);  // the other half-tile
        *abort_flag = 1;
      }
      const int c = 32 * gw + lane;
      const uint32_t taddr = tmem + ((uint32_t)(32 * gw) << 16);
      const float g = gam[0];
      float *dst = p.h0 + bh * (DKc * DVc);
#pragma unroll 1
      for (int r0 = 0; r0 < DKc; r0 += 32) {
        const float *tile = reinterpret_cast<const float *>(S.ring + (r0 < 64 ? sl0 : sl1) * kHalfBytes);
        float dv[32];
        umma::ld32(taddr + (uint32_t)r0, dv);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = r0 + i;
          dst[(size_t)r * DVc + c] = fmaf(g, tile[(r & 63) * DVc + c], dv[i]);
        }
      }
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.empty[sl0]);
        mbar_arrive(&S.empty[sl1]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.rempty[rb]);
    if (gt == 0) p.len[bh] = flush ? 0 : k;
  }
  if (gt == 0 && n_mma > 0) mbar_wait(mbar_mma, (n_mma - 1) & 1u);  // no MMA outlives the memory
  umma::fence_before_sync();
  bar_sync(3, kThreads);
  umma::fence_after_sync();
  if (warp == 0) umma::dealloc(tmem_base, 256);
}

// ============================================================ verify round
// Speculative verify round of Gated DeltaNet [sitech.ge, "NVIDIA ו-Dao AI Lab
// הציגו ReplaySSM…", §Reducing state traffic and simplifying rollback], one
// CTA of 256 threads per (sequence, head):
//   1. commit of the previous round: n1 = len + accepted; when n1 reaches the
//      window the n1 buffered records are folded into h0 with their cached
//      corrections u_i (h0 <- gamma h0 + sum_i R_i k_i u_i^T, written once) and
//      the drafts follow an empty buffer (nb = 0), else nb = n1;
//   2. draft d becomes record e = nb + d.  One pass over the checkpoint tile
//      gives every draft's h0^T k_d and h0^T q_d (2 nd columns); then, draft
//      by draft (each needs the corrections of the earlier ones),
//        u_e = beta_e (v_e - gamma_e h0^T k_e - sum_{j<e} R(e,j) (k_j.k_e) u_j)
//        o_d = scale (gamma_e h0^T q_d + sum_{i<=e} R(e,i) (k_i.q_d) u_i)
//      with gamma_e = prod_{m<=e} alpha_m and R(e,j) = prod_{j<m<=e} alpha_m over
//      the committed records followed by the drafts;
//   3. the drafts and their u_e are appended at slots nb .. nb+nd-1 and len =
//      nb: the u_e of a draft that is accepted later is exactly the correction
//      sequential decoding would have cached for it.
// Decay products are prefix products in fp64 (R(e,j) = Q_e / Q_j with all
// alpha > 0); the key dots are fp32 products summed in fp64.
constexpr int kVD = 4;               // most drafts per round
constexpr int kVSeq = kMaxRec + kVD;  // records a draft sequence can reach (with slack)

struct GdnVerifySmem {
  float Kc[kMaxRec][DKc];     // committed keys (records 0..n1-1)
  float U[kVSeq][DVc];        // cached corrections, then this round's drafts'
  float Kd[kVD][DKc], Qd[kVD][DKc], Vd[kVD][DVc];
  float part[8][2 * kVD][DVc];
  float z[2 * kVD][DVc];      // h0^T k_d, then h0^T q_d
  float G[kVD][kVSeq];        // k_j . k_{e_d}
  float KQ[kVD][kVSeq];       // k_i . q_d
  float R[kVD][kVSeq];        // R(e_d, j)
  float gam[kVD];
  float af[kMaxRec], Rf[kMaxRec];  // committed alphas; fold weights
  float ad[kVD], bd[kVD];          // draft alpha, beta
  float gf;
  int n1, nb, fold, bad;
};

template <typename TI>
__global__ void __launch_bounds__(kThreads, 2) gdn_verify_kernel(const GDNParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GdnVerifySmem &S = *reinterpret_cast<GdnVerifySmem *>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / p.H, h = blockIdx.x - (blockIdx.x / p.H) * p.H;
  const size_t bh = blockIdx.x;
  const int nd = p.n_draft;

  if (tid == 0) {
    const int n0 = p.len[bh];
    const int a = p.acc ? p.acc[b] : 0;
    const int n1 = n0 + a, fold = n1 >= p.L, nb = fold ? 0 : n1;
    const int bad = n0 < 0 || n0 >= p.L || a < 0 || a > p.draft_max || n1 > p.cap ||
                    nb + nd > p.cap;
    if (bad) report(p.status, RSSM_ERR_STATE);
    S.n1 = n1;
    S.nb = nb;
    S.fold = fold;
    S.bad = bad;
  }
  __syncthreads();
  if (S.bad) return;
  const int n1 = S.n1, nb = S.nb, ne = nb + nd;  // draft sequence: records 0..ne-1
  const bool fold = S.fold;

  // ---- checkpoint tile into registers (rows 16w + rho, columns 4 lane ..)
  float *tile = p.h0 + bh * (DKc * DVc);
  float4 hv[kRows];
#pragma unroll
  for (int rho = 0; rho < kRows; ++rho)
    hv[rho] = ld_stream(tile + (size_t)(kRows * warp + rho) * DVc + 4 * lane);

  // ---- stage committed records and the drafts (fp32)
  const TI *kb = static_cast<const TI *>(p.kbuf) + bh * p.cap * DKc;
  const float *ub = p.ubuf + bh * p.cap * DVc;
  {
    // every load first (one memory latency for all committed records), then the
    // shared-memory stores
    constexpr int PER = kMaxRec * DKc / kThreads;
    float kv[PER], uv[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kThreads;
      if (e < n1 * DKc) {
        kv[u] = to_f32(kb[e]);
        uv[u] = ub[e];
      }
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int e = tid + u * kThreads;
      if (e < n1 * DKc) {
        S.Kc[e / DKc][e % DKc] = kv[u];
        S.U[e / DVc][e % DVc] = uv[u];
      }
    }
  }
  for (int e = tid; e < nd * DKc; e += kThreads) {
    const int d = e / DKc, c = e % DKc;
    const int64_t o = (int64_t)(d * p.H + h) * DKc + c;
    S.Qd[d][c] = ld_in<TI>(p.q, b * p.bs_q + o);
    S.Kd[d][c] = ld_in<TI>(p.k, b * p.bs_k + o);
    S.Vd[d][c] = ld_in<TI>(p.v, b * p.bs_v + (int64_t)(d * p.H + h) * DVc + c);
  }
  if (tid < n1) S.af[tid] = p.abuf[bh * p.cap + tid];
  if (tid < nd) {
    S.ad[tid] = p.alpha[b * p.bs_a + tid * p.H + h];
    S.bd[tid] = p.beta[b * p.bs_b + tid * p.H + h];
  }
  __syncthreads();

  // ---- append the drafts at slots nb .. nb+nd-1 (input values: the fp32
  // copies convert back exactly); every committed record is in shared memory
  for (int e = tid; e < nd * DKc; e += kThreads) {
    const int d = e / DKc, c = e % DKc;
    const size_t slot = (bh * p.cap + nb + d) * DKc + c;
    static_cast<TI *>(p.qbuf)[slot] = from_f32<TI>(S.Qd[d][c]);
    static_cast<TI *>(p.kbuf)[slot] = from_f32<TI>(S.Kd[d][c]);
    static_cast<TI *>(p.vbuf)[(bh * p.cap + nb + d) * DVc + c] = from_f32<TI>(S.Vd[d][c]);
  }
  if (tid < nd) {
    p.abuf[bh * p.cap + nb + tid] = S.ad[tid];
    p.bbuf[bh * p.cap + nb + tid] = S.bd[tid];
  }

  // ---- decay factors (warps 0, 1) and key dots (16 threads per dot)
  if (warp == 0) {  // fold: R_i = prod_{i<m<n1} alpha_m, gamma = prod_{m<n1} alpha_m
    double pr = lane < n1 ? (double)S.af[lane] : 1.0;  // inclusive prefix product
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double t = __shfl_up_sync(0xffffffffu, pr, o);
      if (lane >= o) pr *= t;
    }
    const double last = __shfl_sync(0xffffffffu, pr, (n1 > 0 ? n1 : 1) - 1);
    if (fold && lane < n1) S.Rf[lane] = (float)(last / pr);
    if (lane == 0) S.gf = (float)last;
  } else if (warp == 1) {  // drafts: Q_m over the draft sequence, R(e,j) = Q_e / Q_j
    const float am = lane < nb ? S.af[lane] : (lane < ne ? S.ad[lane - nb] : 1.f);
    double pr = am;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double t = __shfl_up_sync(0xffffffffu, pr, o);
      if (lane >= o) pr *= t;
    }
#pragma unroll
    for (int d = 0; d < kVD; ++d) {
      const double qe = __shfl_sync(0xffffffffu, pr, (nb + d) & 31);
      if (d < nd) {
        if (lane <= nb + d) S.R[d][lane] = (float)(qe / pr);
        if (lane == 0) S.gam[d] = (float)qe;
      }
    }
  }
  {
    // dots: (d, j < e_d) keys . k_d, then (d, i <= e_d) keys . q_d
    const int nkk = nd * nb + nd * (nd - 1) / 2, nkq = nd * nb + nd * (nd + 1) / 2;
    const int ndot = nkk + nkq;
    // 8 threads per dot, thread jt of a dot taking the 4-element chunks jt + 8m
    for (int base = 0; base < ndot; base += kThreads / 8) {
      const int t = base + (tid >> 3), jt = tid & 7;
      double acc = 0.0, acc1 = 0.0;
      int d = 0, j = 0;
      bool isq = false;
      if (t < ndot) {
        int r = t < nkk ? t : t - nkk;
        isq = t >= nkk;
        // enumerate (d, j): draft d has nb + d (keys) or nb + d + 1 (queries) partners
        for (d = 0; d < nd; ++d) {
          const int cnt = nb + d + (isq ? 1 : 0);
          if (r < cnt) break;
          r -= cnt;
        }
        j = r;
        const float *kj = j < nb ? S.Kc[j] : S.Kd[j - nb];
        const float *other = isq ? S.Qd[d] : S.Kd[d];
#pragma unroll
        for (int m = 0; m < DKc / 32; ++m) {
          const int c0 = 4 * (jt + 8 * m);
          const float4 a4 = *reinterpret_cast<const float4 *>(kj + c0);
          const float4 o4 = *reinterpret_cast<const float4 *>(other + c0);
          acc += (double)(a4.x * o4.x);
          acc1 += (double)(a4.y * o4.y);
          acc += (double)(a4.z * o4.z);
          acc1 += (double)(a4.w * o4.w);
        }
        acc += acc1;
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      if (t < ndot && jt == 0) {
        if (isq) S.KQ[d][j] = (float)acc;
        else S.G[d][j] = (float)acc;
      }
    }
  }
  __syncthreads();

  // ---- commit fold in registers, written once
  const int row0 = kRows * warp;
  if (fold) {
    const float g = S.gf;
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho) hv[rho] = mul4x(g, hv[rho]);
    for (int i = 0; i < n1; ++i) {
      const float4 ui = *reinterpret_cast<const float4 *>(&S.U[i][4 * lane]);
      const float ri = S.Rf[i];
#pragma unroll
      for (int rho = 0; rho < kRows; ++rho) hv[rho] = fma4x(ri * S.Kc[i][row0 + rho], ui, hv[rho]);
    }
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho)
      st_stream(tile + (size_t)(row0 + rho) * DVc + 4 * lane, hv[rho]);
  }

  // ---- h^T k_d and h^T q_d: partial sums over this warp's 16 rows
  for (int v = 0; v < 2 * nd; ++v) {
    const float *vec = v < nd ? S.Kd[v] : S.Qd[v - nd];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int rho = 0; rho < kRows; ++rho) acc = fma4x(vec[row0 + rho], hv[rho], acc);
    *reinterpret_cast<float4 *>(&S.part[warp][v][4 * lane]) = acc;
  }
  __syncthreads();
  for (int e = tid; e < 2 * nd * DVc; e += kThreads) {
    const int v = e / DVc, c = e % DVc;
    float zc = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) zc += S.part[w][v][c];
    S.z[v][c] = zc;
  }
  __syncthreads();

  // ---- drafts in order: correction u_e, output o_d.  Thread pair (2c, 2c+1)
  // owns column c and splits the older records by parity (one load of u_j for
  // both sums); the pair adds the two halves, so both hold u_e and o_d.
  {
    const int c = tid >> 1, par = tid & 1;
    for (int d = 0; d < nd; ++d) {
      const int e = nb + d;
      float su = 0.f, so = 0.f;
      for (int j = par; j < e; j += 2) {
        const float uj = S.U[j][c], rj = S.R[d][j];
        su = fmaf(rj * S.G[d][j], uj, su);
        so = fmaf(rj * S.KQ[d][j], uj, so);
      }
      su += __shfl_xor_sync(0xffffffffu, su, 1);
      so += __shfl_xor_sync(0xffffffffu, so, 1);
      const float g = S.gam[d];
      const float u = S.bd[d] * ((S.Vd[d][c] - g * S.z[d][c]) - su);
      if (par == 0) {
        S.U[e][c] = u;
        p.ubuf[(bh * p.cap + e) * DVc + c] = u;
      } else {
        const float o = fmaf(S.R[d][e] * S.KQ[d][e], u, fmaf(g, S.z[nd + d][c], so));
        p.y[b * p.bs_y + (size_t)(d * p.H + h) * DVc + c] = p.scale * o;
      }
      __syncwarp();  // u_e is read by both threads of the pair for later drafts
    }
  }
  if (tid == 0) p.len[bh] = nb;
}

// Persistent verify round with two consumer groups on alternate items, on the
// structure of gdn_decode2_kernel: warp 8 streams each item's checkpoint as
// two half-tiles into a ring of exactly 4 slots, warp 9 stages the item (the
// draft inputs, the committed alphas) and bulk-copies its committed keys and
// corrections into record buffer it % 4 (two per group, so the next item of a
// group is staged while it works on this one).  Per item, in a group of 4 warps:
//   * warp 0: fold factors (prefix products of the committed alphas); warp 1:
//     the draft sequence's factors R(e, j) = Q_e / Q_j; 4 threads per key dot
//     (k_j . k_e and k_i . q_d, fp32 products, fp64 sums);
//   * commit fold (n1 reaches the window): warp w folds its 32 rows in its
//     slot, writes them to h0 and leaves them in the slot for the products;
//   * warp w: partial h^T k_d and h^T q_d over its 32 rows in one pass (the
//     sums go through one partial-sum buffer in two halves);
//   * thread c: the drafts in order, u_e and o_d of column c (the earlier
//     drafts' corrections of column c stay in its registers), then the
//     drafts are appended.
struct GdnV2Layout {
  int L, off_bars, off_rec, rec_bytes, off_scr, scr_bytes, off_ring, total;
  // record buffer: Kc [20][128] (input dtype) | Uc [20][128] | Qd, Kd, Vd [4][128]
  // (input dtype) | af [20 -> 32] | ad, bd [4] | hdr [8]
  int o_uc, o_qd, o_kd, o_vd, o_af, o_ad, o_bd, o_hdr;
  // group scratch: part [4][4][128] | G, KQ, R [4][24] | gam [4] | Rf [20 -> 32] | gf
  int s_part, s_g, s_kq, s_r, s_gam, s_rf, s_gf;
  __host__ static int a128(int v) { return (v + 127) & ~127; }
  __host__ static GdnV2Layout make(int L, int es, int budget) {
    GdnV2Layout d;
    d.L = L;
    int o = 0;
    d.o_uc = a128(kMaxRec * DKc * es);
    d.o_qd = d.o_uc + kMaxRec * DVc * 4;
    d.o_kd = d.o_qd + kVD * DKc * es;
    d.o_vd = d.o_kd + kVD * DKc * es;
    d.o_af = d.o_vd + kVD * DVc * es;
    d.o_ad = d.o_af + 32 * 4;
    d.o_bd = d.o_ad + kVD * 4;
    d.o_hdr = d.o_bd + kVD * 4;
    d.rec_bytes = a128(d.o_hdr + 8 * 4);
    d.s_part = 0;
    d.s_g = 4 * kVD * DVc * 4;
    d.s_kq = d.s_g + kVD * kVSeq * 4;
    d.s_r = d.s_kq + kVD * kVSeq * 4;
    d.s_gam = d.s_r + kVD * kVSeq * 4;
    d.s_rf = d.s_gam + kVD * 4;
    d.s_gf = d.s_rf + 32 * 4;
    d.scr_bytes = a128(d.s_gf + 4 * 4);
    d.off_bars = o;
    o += a128(8 * (2 * 8 + 2 * 4));
    d.off_rec = o;
    o += 4 * d.rec_bytes;
    d.off_scr = o;
    o += 2 * d.scr_bytes;
    d.off_ring = o;
    d.total = o + 4 * kHalfBytes;
    if (d.total > budget) d.total = 0;
    return d;
  }
};

// Four consecutive shared-memory elements (8-byte aligned for bf16, 16 for
// fp32) as fp32.
template <typename T>
__device__ __forceinline__ float4 ld4_smem(const T *p) {
  if constexpr (sizeof(T) == 4) {
    return *reinterpret_cast<const float4 *>(p);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const T *e = reinterpret_cast<const T *>(&raw);
    return make_float4(to_f32(e[0]), to_f32(e[1]), to_f32(e[2]), to_f32(e[3]));
  }
}

template <typename TI>
__global__ void __launch_bounds__(kThreads + 64, 1) gdn_verify2_kernel(const GDNParams p,
                                                                    const GdnV2Layout lay) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int abort_word;
  volatile int *abort_flag = &abort_word;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + lay.off_bars);
  uint64_t *empty = full + 8, *rfull = empty + 8, *rempty = rfull + 4;
  unsigned char *ring = smem + lay.off_ring;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nitems = p.B * p.H;
  const int L = lay.L, nd = p.n_draft;

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
        mbar_arrive_expect_tx(&full[slot], kHalfBytes);
        bulk_g2s(ring + slot * kHalfBytes,
                 p.h0 + (size_t)item * DKc * DVc + (size_t)half * kHalfRows * DVc, kHalfBytes,
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

  if (warp == 9) {  // stager: the item's loads first, then shared-memory writes and copies
    int it = 0;
    ArmedRecords armed;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++it) {
      const bool abort_now = __any_sync(0xffffffffu, *abort_flag != 0);
      if (!abort_now && item == p.hold_item) continue;  // test hook: never staged
      const int rb = it & 3;
      bool ok = !abort_now;
      if (ok && lane == 0)
        ok = mbar_wait(&rempty[rb], ((it >> 2) & 1) ^ 1, kWaitLimitNs, abort_flag) && !*abort_flag;
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
      const int a = p.acc ? __ldcg(&p.acc[b]) : 0;
      const int n1 = n0 + a, fold = n1 >= L, nb = fold ? 0 : n1;
      const int bad = n0 < 0 || n0 >= L || a < 0 || a > p.draft_max || n1 > p.cap ||
                      nb + nd > p.cap;
      const int n1c = min(max(n1, 0), p.cap);  // copies stay in this item's slots even when bad
      const float af = lane < n1c ? __ldcg(&p.abuf[bh * p.cap + lane]) : 0.f;
      TI qv[kVD][4], kv[kVD][4], vv[kVD][4];
      float adv = 0.f, bdv = 0.f;
#pragma unroll
      for (int d = 0; d < kVD; ++d) {
        if (d < nd) {
          const int64_t o = (int64_t)(d * p.H + h) * DKc;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            qv[d][u] = static_cast<const TI *>(p.q)[b * p.bs_q + o + lane + 32 * u];
            kv[d][u] = static_cast<const TI *>(p.k)[b * p.bs_k + o + lane + 32 * u];
            vv[d][u] = static_cast<const TI *>(p.v)[b * p.bs_v + (int64_t)(d * p.H + h) * DVc + lane + 32 * u];
          }
        }
      }
      if (lane < nd) {
        adv = p.alpha[b * p.bs_a + lane * p.H + h];
        bdv = p.beta[b * p.bs_b + lane * p.H + h];
      }
      unsigned char *rec = smem + lay.off_rec + rb * lay.rec_bytes;
      TI *Qd = reinterpret_cast<TI *>(rec + lay.o_qd), *Kd = reinterpret_cast<TI *>(rec + lay.o_kd);
      TI *Vd = reinterpret_cast<TI *>(rec + lay.o_vd);
#pragma unroll
      for (int d = 0; d < kVD; ++d) {
        if (d < nd) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            Qd[d * DKc + lane + 32 * u] = qv[d][u];
            Kd[d * DKc + lane + 32 * u] = kv[d][u];
            Vd[d * DVc + lane + 32 * u] = vv[d][u];
          }
        }
      }
      reinterpret_cast<float *>(rec + lay.o_af)[lane] = af;
      if (lane < kVD) {
        reinterpret_cast<float *>(rec + lay.o_ad)[lane] = adv;
        reinterpret_cast<float *>(rec + lay.o_bd)[lane] = bdv;
      }
      if (lane == 0) {
        int *hdr = reinterpret_cast<int *>(rec + lay.o_hdr);
        hdr[0] = n1;
        hdr[1] = nb;
        hdr[2] = fold;
        hdr[3] = bad;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const uint32_t bK = n1c * DKc * sizeof(TI), bU = n1c * DVc * 4;
        mbar_arrive_expect_tx(&rfull[rb], bK + bU);
        if (n1c > 0) {
          bulk_g2s(rec, static_cast<const TI *>(p.kbuf) + bh * p.cap * DKc, bK, &rfull[rb]);
          bulk_g2s(rec + lay.o_uc, p.ubuf + bh * p.cap * DVc, bU, &rfull[rb]);
        }
      }
      armed.arm(rb, (it >> 2) & 1);
    }
    if (lane == 0) armed.drain(rfull, 4);  // no record copy outlives the warp
    __syncwarp();
    return;
  }

  // Consumer group grp (warps 4grp .. 4grp+3), thread gt = column c.
  constexpr int kG = 128;
  const int grp = warp >> 2, gw = warp & 3, gt = tid & (kG - 1);
  const uint32_t gbar = 1 + grp;
  unsigned char *scr = smem + lay.off_scr + grp * lay.scr_bytes;
  float *part = reinterpret_cast<float *>(scr + lay.s_part);
  float *G = reinterpret_cast<float *>(scr + lay.s_g), *KQ = reinterpret_cast<float *>(scr + lay.s_kq);
  float *Rd = reinterpret_cast<float *>(scr + lay.s_r), *gam = reinterpret_cast<float *>(scr + lay.s_gam);
  float *Rf = reinterpret_cast<float *>(scr + lay.s_rf), *gf = reinterpret_cast<float *>(scr + lay.s_gf);
  int it = grp;
  for (int item = blockIdx.x + grp * gridDim.x; item < nitems; item += 2 * gridDim.x, it += 2) {
    const int rb = it & 3;  // this group's buffers: grp and grp + 2
    const unsigned char *rec = smem + lay.off_rec + rb * lay.rec_bytes;
    const TI *Kc = reinterpret_cast<const TI *>(rec);
    const float *Uc = reinterpret_cast<const float *>(rec + lay.o_uc);
    const TI *Qd = reinterpret_cast<const TI *>(rec + lay.o_qd);
    const TI *Kd = reinterpret_cast<const TI *>(rec + lay.o_kd);
    const TI *Vd = reinterpret_cast<const TI *>(rec + lay.o_vd);
    const float *afs = reinterpret_cast<const float *>(rec + lay.o_af);
    const float *ads = reinterpret_cast<const float *>(rec + lay.o_ad);
    const float *bds = reinterpret_cast<const float *>(rec + lay.o_bd);
    const int *hdr = reinterpret_cast<const int *>(rec + lay.o_hdr);
    const int b = item / p.H, h = item - (item / p.H) * p.H;
    const size_t bh = (size_t)item;
    const int sl0 = 2 * (it & 1), sl1 = sl0 + 1;
    const uint32_t tphase = (it >> 1) & 1;
    const int half = gw >> 1, sl = half ? sl1 : sl0;

    const bool got = mbar_wait(&rfull[rb], (it >> 2) & 1, p.wait_ns, abort_flag);
    if (!got) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    if (bar_or(gbar, kG, !got || *abort_flag)) break;
    if (hdr[3]) {
      if (gt == 0) report(p.status, RSSM_ERR_STATE);
      if (!mbar_wait(&full[sl], tphase, p.wait_ns, abort_flag)) {
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
    const int n1 = hdr[0], nb = hdr[1], ne = nb + nd;  // draft sequence: records 0..ne-1
    const bool fold = hdr[2];

    // ---- decay factors (warps 0, 1) and key dots (4 threads per dot)
    if (gw == 0) {  // fold: R_i = prod_{i<m<n1} alpha_m, gamma = prod_{m<n1} alpha_m
      double pr = lane < n1 ? (double)afs[lane] : 1.0;  // inclusive prefix product
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, pr, o);
        if (lane >= o) pr *= t;
      }
      const double lastp = __shfl_sync(0xffffffffu, pr, (n1 > 0 ? n1 : 1) - 1);
      if (fold && lane < n1) Rf[lane] = (float)(lastp / pr);
      if (lane == 0) gf[0] = (float)lastp;
    } else if (gw == 1) {  // drafts: Q_m over the draft sequence, R(e,j) = Q_e / Q_j
      const float am = lane < nb ? afs[lane] : (lane < ne ? ads[lane - nb] : 1.f);
      double pr = am;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, pr, o);
        if (lane >= o) pr *= t;
      }
#pragma unroll
      for (int d = 0; d < kVD; ++d) {
        const double qe = __shfl_sync(0xffffffffu, pr, (nb + d) & 31);
        if (d < nd) {
          if (lane <= nb + d) Rd[d * kVSeq + lane] = (float)(qe / pr);
          if (lane == 0) gam[d] = (float)qe;
        }
      }
    }
    {
      // dots: (d, j < e_d) keys . k_d, then (d, i <= e_d) keys . q_d
      const int nkk = nd * nb + nd * (nd - 1) / 2, nkq = nd * nb + nd * (nd + 1) / 2;
      const int ndot = nkk + nkq;
      for (int base = 0; base < ndot; base += kG / 4) {
        const int t = base + (gt >> 2), j4 = gt & 3;
        double acc = 0.0, acc1 = 0.0;
        int d = 0, j = 0;
        bool isq = false;
        if (t < ndot) {
          int r = t < nkk ? t : t - nkk;
          isq = t >= nkk;
          // enumerate (d, j): draft d has nb + d (keys) or nb + d + 1 (queries) partners
          for (d = 0; d < nd; ++d) {
            const int cnt = nb + d + (isq ? 1 : 0);
            if (r < cnt) break;
            r -= cnt;
          }
          j = r;
          const TI *other = isq ? Qd + d * DKc : Kd + d * DKc;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int c0 = 8 * (j4 + 4 * m);
            float kv[8], ov[8];
            if (j < nb) ld8_smem(Kc + j * DKc + c0, kv);
            else ld8_smem(Kd + (j - nb) * DKc + c0, kv);
            ld8_smem(other + c0, ov);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              acc += (double)(kv[e] * ov[e]);
              acc1 += (double)(kv[e + 1] * ov[e + 1]);
            }
          }
          acc += acc1;
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        if (t < ndot && j4 == 0) {
          if (isq) KQ[d * kVSeq + j] = (float)acc;
          else G[d * kVSeq + j] = (float)acc;
        }
      }
    }
    bar_sync(gbar, kG);

    // ---- this warp's 32 rows: commit fold in the slot, then partial products
    if (!mbar_wait(&full[sl], tphase, p.wait_ns, abort_flag)) {
      if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
      *abort_flag = 1;
    }
    float *tile = reinterpret_cast<float *>(ring + sl * kHalfBytes) +
                  (size_t)(32 * (gw & 1)) * DVc + 4 * lane;
    const int row0 = 32 * gw;
    if (fold) {  // h <- gamma h0 + sum_i R_i k_i u_i^T, written to h0 and to the slot
      const float g = gf[0];
      float *dst = p.h0 + bh * (DKc * DVc) + (size_t)row0 * DVc + 4 * lane;
#pragma unroll 1
      for (int r0 = 0; r0 < 32; r0 += 8) {
        float4 acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = mul4x(g, *reinterpret_cast<const float4 *>(tile + (r0 + e) * DVc));
        for (int i = 0; i < n1; ++i) {
          const float4 ui = *reinterpret_cast<const float4 *>(&Uc[i * DVc + 4 * lane]);
          const float ri = Rf[i];
          float kr[8];
          ld8_smem(Kc + i * DKc + row0 + r0, kr);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = fma4x(ri * kr[e], ui, acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          *reinterpret_cast<float4 *>(tile + (r0 + e) * DVc) = acc[e];
          st_stream(dst + (size_t)(r0 + e) * DVc, acc[e]);
        }
      }
      __syncwarp();
    }
    // one pass over the rows for all 2 nd products; the partial sums go
    // through one buffer in two halves (h^T k_d, then h^T q_d), thread c
    // keeping its column's sums in registers
    float zk[kVD], zq[kVD];
    {
      float4 pa[2][kVD];
#pragma unroll
      for (int pass = 0; pass < 2; ++pass)
#pragma unroll
        for (int v = 0; v < kVD; ++v) pa[pass][v] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
      for (int t = 0; t < 8; ++t) {
        float4 x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = *reinterpret_cast<const float4 *>(tile + (4 * t + e) * DVc);
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const TI *vecs = pass ? Qd : Kd;
#pragma unroll
          for (int v = 0; v < kVD; ++v) {
            if (v < nd) {
              const float4 w4 = ld4_smem(vecs + v * DKc + row0 + 4 * t);
              pa[pass][v] = fma4x(w4.x, x[0], pa[pass][v]);
              pa[pass][v] = fma4x(w4.y, x[1], pa[pass][v]);
              pa[pass][v] = fma4x(w4.z, x[2], pa[pass][v]);
              pa[pass][v] = fma4x(w4.w, x[3], pa[pass][v]);
            }
          }
        }
      }
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        if (pass) bar_sync(gbar, kG);  // the first half's sums have been read
#pragma unroll
        for (int v = 0; v < kVD; ++v)
          *reinterpret_cast<float4 *>(&part[(gw * kVD + v) * DVc + 4 * lane]) = pa[pass][v];
        bar_sync(gbar, kG);
#pragma unroll
        for (int d = 0; d < kVD; ++d) {
          float zs = 0.f;
          if (d < nd) {
#pragma unroll
            for (int w = 0; w < 4; ++w) zs += part[(w * kVD + d) * DVc + gt];
          }
          if (pass) zq[d] = zs;
          else zk[d] = zs;
        }
      }
    }
    fence_proxy_async_smem();  // the fold's slot writes before the slot's next bulk copy
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[sl0]);
      mbar_arrive(&empty[sl1]);
    }

    // ---- column c: the drafts in order (each needs the earlier ones' u)
    {
      const int c = gt;
      float su[kVD], so[kVD], ud[kVD];
#pragma unroll
      for (int d = 0; d < kVD; ++d) su[d] = so[d] = ud[d] = 0.f;
      // the committed records' terms, one load of u_j for every draft
      for (int j = 0; j < nb; ++j) {
        const float uj = Uc[j * DVc + c];
#pragma unroll
        for (int d = 0; d < kVD; ++d) {
          if (d < nd) {
            const float rj = Rd[d * kVSeq + j];
            su[d] = fmaf(-rj * G[d * kVSeq + j], uj, su[d]);
            so[d] = fmaf(rj * KQ[d * kVSeq + j], uj, so[d]);
          }
        }
      }
#pragma unroll
      for (int d = 0; d < kVD; ++d) {
        if (d < nd) {
          const int e = nb + d;
          float a0 = to_f32(Vd[d * DVc + c]) - gam[d] * zk[d] + su[d];
#pragma unroll
          for (int q = 0; q < kVD; ++q)  // earlier drafts' records
            if (q < d) a0 = fmaf(-Rd[d * kVSeq + nb + q] * G[d * kVSeq + nb + q], ud[q], a0);
          const float u = bds[d] * a0;
          ud[d] = u;
          float o0 = gam[d] * zq[d] + so[d];
#pragma unroll
          for (int q = 0; q < kVD; ++q)
            if (q <= d) o0 = fmaf(Rd[d * kVSeq + nb + q] * KQ[d * kVSeq + nb + q], ud[q], o0);
          p.ubuf[(bh * p.cap + e) * DVc + c] = u;
          p.y[b * p.bs_y + (size_t)(d * p.H + h) * DVc + c] = p.scale * o0;
        }
      }
      // ---- append the drafts at slots nb .. nb+nd-1 (their staged input values)
#pragma unroll
      for (int d = 0; d < kVD; ++d) {
        if (d < nd) {
          const size_t slot = bh * p.cap + nb + d;
          static_cast<TI *>(p.qbuf)[slot * DKc + c] = Qd[d * DKc + c];
          static_cast<TI *>(p.kbuf)[slot * DKc + c] = Kd[d * DKc + c];
          static_cast<TI *>(p.vbuf)[slot * DVc + c] = Vd[d * DVc + c];
        }
      }
      if (c < nd) {
        p.abuf[bh * p.cap + nb + c] = ads[c];
        p.bbuf[bh * p.cap + nb + c] = bds[c];
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&rempty[rb]);
    if (gt == 0) p.len[bh] = nb;
  }
}

int gdn_sm_count();

template <typename TI>
cudaError_t gdn_verify_launch(const GDNParams &p, cudaStream_t s) {
  if (p.L <= 16) {  // two consumer groups when their layout fits
    const GdnV2Layout lay = GdnV2Layout::make(p.L, (int)sizeof(TI), 227 * 1024);
    if (lay.total > 0) {
      cudaError_t e = cudaFuncSetAttribute(gdn_verify2_kernel<TI>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
      if (e != cudaSuccess) return e;
      const int nitems = p.B * p.H;
      const int grid = nitems < gdn_sm_count() ? nitems : gdn_sm_count();
      gdn_verify2_kernel<TI><<<grid, kThreads + 64, lay.total, s>>>(p, lay);
      return cudaGetLastError();
    }
  }
  const size_t smem = sizeof(GdnVerifySmem);
  cudaError_t e = cudaFuncSetAttribute(gdn_verify_kernel<TI>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gdn_verify_kernel<TI><<<(unsigned)(p.B * p.H), kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

int gdn_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

// bf16 keys fold on the tensor cores (when the operand area fits beside a
// ring of at least 4 half-tiles); fp32 keys, which are not exact in bf16, on
// the SIMT pipes.
template <typename TI>
cudaError_t gdn_launch_persistent(const GDNParams &p, cudaStream_t s) {
  constexpr bool kMma = std::is_same<TI, __nv_bfloat16>::value;
  if constexpr (kMma) {  // two consumer groups when their layout fits
    const GdnLayout lay2 = GdnLayout::make2(p.L, 227 * 1024);
    if (lay2.NS == 4) {
      cudaError_t e = cudaFuncSetAttribute(gdn_decode2_kernel<TI>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, lay2.total);
      if (e != cudaSuccess) return e;
      const int nitems = p.B * p.H;
      const int grid = nitems < gdn_sm_count() ? nitems : gdn_sm_count();
      gdn_decode2_kernel<TI><<<grid, kThreads + 64, lay2.total, s>>>(p, lay2);
      return cudaGetLastError();
    }
  }
  GdnLayout lay = GdnLayout::make(p.L, (int)sizeof(TI), 220 * 1024, kMma);
  const bool mma = kMma && lay.NS >= 4;
  if (!mma) lay = GdnLayout::make(p.L, (int)sizeof(TI), 220 * 1024);
  if (lay.NS < 4) return cudaErrorInvalidConfiguration;
  auto kernel = mma ? gdn_decode_kernel<TI, kMma> : gdn_decode_kernel<TI, false>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.total);
  if (e != cudaSuccess) return e;
  const int nitems = p.B * p.H;
  const int grid = nitems < gdn_sm_count() ? nitems : gdn_sm_count();
  kernel<<<grid, kThreads + 64, lay.total, s>>>(p, lay);
  return cudaGetLastError();
}

}  // namespace

bool gdn_supported(int DK, int DV) { return DK == DKc && DV == DVc; }

cudaError_t gdn_launch_decode(const GDNParams &p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  return p.in_bf16 ? gdn_launch_persistent<__nv_bfloat16>(p, s) : gdn_launch_persistent<float>(p, s);
}

cudaError_t gdn_launch_fold(const GDNParams &p, int mode, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  if (mode == kFoldFlush) return launch_dt<kGdnFlush>(p, s);
  if (mode == kFoldMaterialize) return launch_dt<kGdnMaterialize>(p, s);
  if (mode == kFoldCommit) return launch_dt<kGdnCommit>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t gdn_launch_verify(const GDNParams &p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  return p.in_bf16 ? gdn_verify_launch<__nv_bfloat16>(p, s) : gdn_verify_launch<float>(p, s);
}

}  // namespace rssm
