// m2_device.cuh -- device helpers shared by the Mamba-2 kernels (m2.cu:
// decode step, folds, conventional step; m2_verify.cu: speculative verify):
// head-tile register layouts and row views, decay weights, the register
// fold, read-copy codecs on rows, the item -> (sequence, group, chunk) map,
// the tile producer, and the host-side shape dispatch.
#pragma once
#include <type_traits>

#include "codec.cuh"
#include "common.cuh"
#include "internal.h"
#include "pipeline.cuh"

namespace rssm {
namespace {


__device__ __forceinline__ float sum8(float v) {  // over the 8 lanes of a quarter-warp
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  return v;
}

// Dot product of C4 float4 pairs summed as a balanced tree.
template <int C4>
__device__ __forceinline__ float tree_dot(const float4 (&a)[C4], const float4 (&b)[C4]) {
  float d[C4];
#pragma unroll
  for (int s = 0; s < C4; ++s) d[s] = (a[s].x * b[s].x + a[s].y * b[s].y) + (a[s].z * b[s].z + a[s].w * b[s].w);
#pragma unroll
  for (int w = 1; w < C4; w <<= 1)
#pragma unroll
    for (int s = 0; s + w < C4; s += 2 * w) d[s] += d[s + w];
  return d[0];
}

template <int P, int N>
struct Tile {
  static constexpr int RPT = P / 32;  // rows per thread
  static constexpr int C4 = N / 32;   // float4 column segments per thread
  static __device__ __forceinline__ int row(int warp, int rs, int rho) {
    return warp * (P / 8) + rs + 4 * rho;
  }
  static __device__ __forceinline__ int col(int c8, int s) { return 32 * s + 4 * c8; }
};

// ---------------------------------------------------------------- read copy

// Quantise a register tile after a fold.  fmt 1 = FP8, 2 = NVFP4.  With
// roundtrip the values are replaced by deq(Q(v)) (quantised checkpoint);
// otherwise the codes are written to the read copy.  Must be called by every
// thread of the CTA (NVFP4 needs the tile maximum).
template <int P, int N>
__device__ __forceinline__ void quantize_tile(const M2Params &p, size_t bh, int fmt, bool roundtrip,
                                              float4 (&v)[P / 32][N / 32], float *s_red, int warp,
                                              int lane, int rs, int c8, int bar_threads = 0) {
  using T = Tile<P, N>;
  if (fmt == 1) {
    uint8_t *rc = p.rc + bh * (size_t)(P * N);
#pragma unroll
    for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
      for (int s = 0; s < T::C4; ++s) {
        const int r = T::row(warp, rs, rho), c = T::col(c8, s);
        float4 &a = v[rho][s];
        const uint32_t b0 = e4m3_encode(a.x), b1 = e4m3_encode(a.y), b2 = e4m3_encode(a.z),
                       b3 = e4m3_encode(a.w);
        if (roundtrip) {
          a = make_float4(e4m3_decode(b0), e4m3_decode(b1), e4m3_decode(b2), e4m3_decode(b3));
        } else {
          *reinterpret_cast<uint32_t *>(rc + (size_t)r * N + c) = b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
        }
      }
    return;
  }
  // NVFP4: tile maximum first
  float m = 0.f;
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
    for (int s = 0; s < T::C4; ++s) {
      const float4 a = v[rho][s];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  if (bar_threads) bar_sync(2, bar_threads);  // the consumer warps only
  else __syncthreads();
  float amax = s_red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, s_red[w]);
  const float sg = nvfp4_tile_scale(amax);
  uint8_t *rc = p.rc + bh * (size_t)(P * N / 2);
  uint8_t *sc = p.rc_scale + bh * (size_t)(P * N / 16);
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
    for (int s = 0; s < T::C4; ++s) {
      const int r = T::row(warp, rs, rho), c = T::col(c8, s);
      float4 &a = v[rho][s];
      float bm = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w)));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
      bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
      const uint32_t scode = nvfp4_block_code(bm, sg);
      const float d = nvfp4_step(scode, sg);
      const uint32_t lo = nvfp4_pack2(a.x, a.y, d), hi = nvfp4_pack2(a.z, a.w, d);
      if (roundtrip) {
        const float sb = e4m3_decode(scode);
        a = make_float4(nvfp4_value(lo & 0xF, sb, sg), nvfp4_value(lo >> 4, sb, sg),
                        nvfp4_value(hi & 0xF, sb, sg), nvfp4_value(hi >> 4, sb, sg));
      } else {
        *reinterpret_cast<uint16_t *>(rc + (size_t)r * (N / 2) + c / 2) = (uint16_t)(lo | (hi << 8));
        if ((c8 & 3) == 0) sc[(size_t)r * (N / 16) + c / 16] = (uint8_t)scode;
      }
    }
  if (!roundtrip && warp == 0 && lane == 0) p.rc_gscale[bh] = sg;
}

template <int P, int N>
__device__ __forceinline__ void load_tile(const float *tile, int warp, int rs, int c8,
                                          float4 (&v)[P / 32][N / 32]) {
  using T = Tile<P, N>;
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
    for (int s = 0; s < T::C4; ++s)
      v[rho][s] = ld_stream(tile + (size_t)T::row(warp, rs, rho) * N + T::col(c8, s));
}

template <int P, int N>
__device__ __forceinline__ void store_tile(float *tile, int warp, int rs, int c8,
                                           const float4 (&v)[P / 32][N / 32]) {
  using T = Tile<P, N>;
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho)
#pragma unroll
    for (int s = 0; s < T::C4; ++s)
      st_stream(tile + (size_t)T::row(warp, rs, rho) * N + T::col(c8, s), v[rho][s]);
}

// Decay weights of k records for one head, by one warp (lane i owns record i):
//   wdt[i] = exp(A * sum_{i<m<k} dt_m) * dt_i,   *lam = exp(A * sum_{m<k} dt_m).
// The suffix sums come from a shuffle scan (fixed association order, so the
// result does not depend on timing); every dt term is non-negative, so no
// cancellation occurs.  Sums, products and exponentials are taken in fp64 (a
// handful per head; B200 runs fp64 at half the fp32 rate): an fp32 exp(A s)
// would carry a relative error of about |A s| * 2^-24 into every weight.
__device__ __forceinline__ void decay_weights_scan(const float *dt, int k, float A, float *wdt,
                                                   float *lam, int lane) {
  const double mine = lane < k ? (double)dt[lane] : 0.0;
  double s = lane + 1 < k ? (double)dt[lane + 1] : 0.0;  // suffix of the records after this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_down_sync(0xffffffffu, s, o);
    if (lane + o < 32) s += t;
  }
  const double a = A;
  if (lane < k) wdt[lane] = (float)(exp(a * s) * mine);
  if (lane == 0) *lam = (float)exp(a * (s + mine));
}

__device__ __forceinline__ void decay_weights(const float *dt, int k, float A, float *wdt,
                                              float *lam, int lane) {
  const double a = A;
  if (lane < k) {
    double s = 0.0;
    for (int m = lane + 1; m < k; ++m) s += dt[m];
    wdt[lane] = (float)(exp(a * s) * (double)dt[lane]);
  }
  if (lane == 0) {
    double t = 0.0;
    for (int m = 0; m < k; ++m) t += dt[m];
    *lam = (float)exp(a * t);
  }
}

// h <- lam * h + sum_{i<k} (wdt_i x_i[r]) B_i[cols]  -- the fold, in registers.
// x: the head's records [k][P] (input dtype); B: the group's records [k][N] fp32.
template <typename TB>
__device__ __forceinline__ float4 ld4_smem(const TB *p) {
  if constexpr (sizeof(TB) == 4) {
    return *reinterpret_cast<const float4 *>(p);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    const TB *e = reinterpret_cast<const TB *>(&raw);
    return make_float4(to_f32(e[0]), to_f32(e[1]), to_f32(e[2]), to_f32(e[3]));
  }
}

template <int P, int N, typename TI, typename TB = float>
__device__ __forceinline__ void fold_regs(float4 (&hv)[P / 32][N / 32], float lam, int k,
                                          const float *wdt, const TI *x, const TB *Bs,
                                          int warp, int rs, int c8) {
  using T = Tile<P, N>;
#pragma unroll
  for (int rho = 0; rho < T::RPT; ++rho) {
    const int r = T::row(warp, rs, rho);
#pragma unroll
    for (int s = 0; s < T::C4; ++s) {
      hv[rho][s].x *= lam;
      hv[rho][s].y *= lam;
      hv[rho][s].z *= lam;
      hv[rho][s].w *= lam;
    }
    for (int i = 0; i < k; ++i) {
      const float xw = wdt[i] * to_f32(x[i * P + r]);
#pragma unroll
      for (int s = 0; s < T::C4; ++s) {
        const float4 bb = ld4_smem<TB>(&Bs[i * N + T::col(c8, s)]);
        hv[rho][s].x = fmaf(xw, bb.x, hv[rho][s].x);
        hv[rho][s].y = fmaf(xw, bb.y, hv[rho][s].y);
        hv[rho][s].z = fmaf(xw, bb.z, hv[rho][s].z);
        hv[rho][s].w = fmaf(xw, bb.w, hv[rho][s].w);
      }
    }
  }
}

// After a fold: round the checkpoint (qmode 3/4), store it, refresh the read
// copy (qmode 1/2).  NVFP4 variants synchronise the CTA.
template <int P, int N, int QM>
__device__ __forceinline__ void commit_checkpoint(const M2Params &p, size_t bh, float *dst,
                                                  float4 (&hv)[P / 32][N / 32], float *s_red,
                                                  int warp, int lane, int rs, int c8,
                                                  int bar_threads = 0) {
  if constexpr (QM >= 3)
    quantize_tile<P, N>(p, bh, QM - 2, true, hv, s_red, warp, lane, rs, c8, bar_threads);
  store_tile<P, N>(dst, warp, rs, c8, hv);
  if constexpr (QM == 1 || QM == 2)
    quantize_tile<P, N>(p, bh, QM, false, hv, s_red, warp, lane, rs, c8, bar_threads);
}

// Heads handled by one CTA: the whole group when it has at most 8 heads,
// otherwise chunks of 8 (the host requires H/G <= 8 or a multiple of 8).
__host__ __device__ __forceinline__ int head_chunk(int hpg) { return hpg <= 8 ? hpg : 8; }

// Copy `count` elements of T from global to shared memory as fp32, 16 bytes
// per load (both ends 16-byte aligned, count a multiple of 16 / sizeof(T)).
template <typename T>
__device__ __forceinline__ void stage_f32(float *dst, const T *src, int count, int tid) {
  constexpr int V = 16 / sizeof(T);
  const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
  for (int v = tid; v < count / V; v += kThreads) {
    const uint4 raw = s4[v];
    const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
    for (int j = 0; j < V; ++j) dst[v * V + j] = to_f32(e[j]);
  }
}

// Copy `bytes` (multiple of 16) from global to shared memory unchanged.
__device__ __forceinline__ void stage_raw(void *dst, const void *src, int bytes, int tid) {
  const uint4 *s4 = static_cast<const uint4 *>(src);
  uint4 *d4 = static_cast<uint4 *>(dst);
  for (int v = tid; v < bytes / 16; v += kThreads) d4[v] = s4[v];
}

__host__ __device__ __forceinline__ int pad4(int n) { return (n + 3) & ~3; }

// Shared-memory layout of the decode / fold kernels (floats unless noted):
//   B [L][N] | C [N] | bc [pad4(L)] | dt [hc][L] | wdt [hc][L] | lam [pad4(hc)]
//   | red [2][8] (tile maxima, alternating between consecutive heads) | x [hc][L][P] (input dtype)
struct DecodeSmem {
  float *B, *C, *bc, *dt, *wdt, *lam, *red;
  void *x;
  __host__ __device__ static size_t bytes(int L, int hc, int P, int N, int es) {
    const size_t f = (size_t)L * N + N + pad4(L) + 2 * pad4(hc * L) + pad4(hc) + 16;
    return f * 4 + (size_t)hc * L * P * es;
  }
  __device__ DecodeSmem(unsigned char *base, int L, int hc, int N) {
    float *f = reinterpret_cast<float *>(base);
    B = f;
    C = B + L * N;
    bc = C + N;
    dt = bc + pad4(L);
    wdt = dt + pad4(hc * L);
    lam = wdt + pad4(hc * L);
    red = lam + pad4(hc);
    x = red + 16;
  }
};

// ------------------------------------------------------------- row helpers
// One row of a P x N head tile as seen by one lane of the decode kernel:
// columns 32 s + 4 c8 (s < N/32), four values each (for an NVFP4 copy
// without its per-tile scale).

template <int P, int N, int QM>
__device__ __forceinline__ void view_row(const unsigned char *t, int r, int c8,
                                         float4 (&v)[N / 32]) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s) {
    const int c = 32 * s + 4 * c8;
    if constexpr (QM == 1) {
      const uint32_t w = *reinterpret_cast<const uint32_t *>(t + r * N + c);
      const float2 lo = e4m3x2_decode(w & 0xFFFFu), hi = e4m3x2_decode(w >> 16);
      v[s] = make_float4(lo.x, lo.y, hi.x, hi.y);
    } else if constexpr (QM == 2) {
      // E2M1 * s_b (exact in fp32); the per-tile scale s_g is left to the
      // caller, which applies it once to each row's dot product
      const uint32_t w = *reinterpret_cast<const uint16_t *>(t + r * (N / 2) + c / 2);
      const float sb = e4m3_decode(t[P * N / 2 + r * (N / 16) + c / 16]);
      const float2 lo = e2m1x2_decode(w & 0xFFu), hi = e2m1x2_decode(w >> 8);
      v[s] = make_float4(lo.x * sb, lo.y * sb, hi.x * sb, hi.y * sb);
    } else {
      v[s] = *reinterpret_cast<const float4 *>(t + (r * N + c) * 4);
    }
  }
}

template <int N>
__device__ __forceinline__ void load_row(const float *tile, int r, int c8, float4 (&v)[N / 32]) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s) v[s] = ld_stream(tile + (size_t)r * N + 32 * s + 4 * c8);
}

template <int N>
__device__ __forceinline__ void store_row(float *tile, int r, int c8, const float4 (&v)[N / 32]) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s) st_stream(tile + (size_t)r * N + 32 * s + 4 * c8, v[s]);
}

// The fold of RGC register-held rows of one head:
//   v[u] <- lam v[u] + sum_{i<k} (w_i x_i[rows[u]]) B_i[cols],
// record loop outermost so that each B_i fragment (fp32 in shared memory) is
// loaded once and feeds 4 * RGC * (N/32) independent FMAs (issued in pairs).
template <int P, int N, typename TI, int RGC>
__device__ __forceinline__ void fold_rows(float4 (&v)[RGC][N / 32], float lam, int k,
                                          const float *w, const TI *x, const int (&rows)[RGC],
                                          const float *Bf, int c8) {
#pragma unroll
  for (int u = 0; u < RGC; ++u)
#pragma unroll
    for (int s = 0; s < N / 32; ++s) v[u][s] = mul4x(lam, v[u][s]);
  for (int i = 0; i < k; ++i) {
    float4 bb[N / 32];
#pragma unroll
    for (int s = 0; s < N / 32; ++s)
      bb[s] = *reinterpret_cast<const float4 *>(&Bf[i * N + 32 * s + 4 * c8]);
    const float wi = w[i];
#pragma unroll
    for (int u = 0; u < RGC; ++u) {
      const float xw = wi * to_f32(x[i * P + rows[u]]);
#pragma unroll
      for (int s = 0; s < N / 32; ++s) v[u][s] = fma4x(xw, bb[s], v[u][s]);
    }
  }
}

template <int N>
__device__ __forceinline__ void fp8_roundtrip_row(float4 (&v)[N / 32]) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s)
    v[s] = make_float4(e4m3_decode(e4m3_encode(v[s].x)), e4m3_decode(e4m3_encode(v[s].y)),
                       e4m3_decode(e4m3_encode(v[s].z)), e4m3_decode(e4m3_encode(v[s].w)));
}

template <int N>
__device__ __forceinline__ void fp8_codes_row(uint8_t *rc_tile, int r, int c8,
                                              const float4 (&v)[N / 32]) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s) {
    const uint32_t w = e4m3_encode(v[s].x) | (e4m3_encode(v[s].y) << 8) |
                       (e4m3_encode(v[s].z) << 16) | (e4m3_encode(v[s].w) << 24);
    *reinterpret_cast<uint32_t *>(rc_tile + (size_t)r * N + 32 * s + 4 * c8) = w;
  }
}

template <int N>
__device__ __forceinline__ float absmax_row(const float4 (&v)[N / 32]) {
  float m = 0.f;
#pragma unroll
  for (int s = 0; s < N / 32; ++s)
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[s].x), fabsf(v[s].y)), fmaxf(fabsf(v[s].z), fabsf(v[s].w))));
  return m;
}

// NVFP4 of one row given the tile scale: block maxima over the 4 lanes that
// share a 16-column block, then codes (written) or deq(Q(v)) (roundtrip).
template <int P, int N>
__device__ __forceinline__ void nvfp4_row(float4 (&v)[N / 32], float sg, bool roundtrip,
                                          uint8_t *rc_tile, uint8_t *sc_tile, int r, int c8) {
#pragma unroll
  for (int s = 0; s < N / 32; ++s) {
    const int c = 32 * s + 4 * c8;
    float bm = fmaxf(fmaxf(fabsf(v[s].x), fabsf(v[s].y)), fmaxf(fabsf(v[s].z), fabsf(v[s].w)));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
    const uint32_t scode = nvfp4_block_code(bm, sg);
    const float d = nvfp4_step(scode, sg);
    const uint32_t lo = nvfp4_pack2(v[s].x, v[s].y, d), hi = nvfp4_pack2(v[s].z, v[s].w, d);
    if (roundtrip) {
      const float sb = e4m3_decode(scode);
      v[s] = make_float4(nvfp4_value(lo & 0xF, sb, sg), nvfp4_value(lo >> 4, sb, sg),
                         nvfp4_value(hi & 0xF, sb, sg), nvfp4_value(hi >> 4, sb, sg));
    } else {
      *reinterpret_cast<uint16_t *>(rc_tile + (size_t)r * (N / 2) + c / 2) = (uint16_t)(lo | (hi << 8));
      if ((c8 & 3) == 0) sc_tile[(size_t)r * (N / 16) + c / 16] = (uint8_t)scode;
    }
  }
}

__device__ __forceinline__ void item_coords(const M2Params &p, int item, int nchunk, int hc, int &b,
                                            int &g, int &chunk, int &h_first) {
  const int bg_i = item / nchunk;
  chunk = item - bg_i * nchunk;
  b = bg_i / p.G;
  g = bg_i - b * p.G;
  h_first = g * p.hpg + chunk * hc;
}

// Tile producer (one thread): streams the checkpoint tiles (or their read
// copies) of this CTA's items, in item order, into the NS-slot ring.  (An L2
// bulk prefetch running one or two items ahead of the ring made the verify
// round 4-8% slower on B200, so there is none.)
template <int P, int N, int QM>
__device__ __forceinline__ void stream_tiles(const M2Params &p, uint64_t *full, uint64_t *empty,
                                             unsigned char *ring, int NS, int tile_stride,
                                             int tile_bytes, int hc, volatile int *abort_flag,
                                             int nitems, int nchunk) {
  auto src_of = [&](int item, int j) -> size_t {
    int b, g, chunk, h_first;
    item_coords(p, item, nchunk, hc, b, g, chunk, h_first);
    return (size_t)b * p.H + h_first + j;
  };
  int slot = 0;
  uint32_t sphase = 0;
  uint32_t issued = 0, parity = 0;  // per slot: a copy was issued / its phase parity
  bool failed = false;
  for (int item = blockIdx.x; item < nitems && !failed; item += gridDim.x) {
    for (int j = 0; j < hc; ++j) {
      // re-check the flag after the wait: a consumer that gave up sets it
      // before releasing its slot, and no copy may follow an abort
      if (*abort_flag || !mbar_wait(&empty[slot], sphase ^ 1, kWaitLimitNs, abort_flag) ||
          *abort_flag) {
        failed = true;
        break;
      }
      mbar_arrive_expect_tx(&full[slot], tile_bytes);
      unsigned char *dst = ring + slot * tile_stride;
      const size_t bh = src_of(item, j);
      if constexpr (QM == 1) {
        bulk_g2s(dst, p.rc + bh * (size_t)(P * N), P * N, &full[slot]);
      } else if constexpr (QM == 2) {
        bulk_g2s(dst, p.rc + bh * (size_t)(P * N / 2), P * N / 2, &full[slot]);
        bulk_g2s(dst + P * N / 2, p.rc_scale + bh * (size_t)(P * N / 16), P * N / 16, &full[slot]);
      } else {
        bulk_g2s(dst, p.h0 + bh * (size_t)(P * N), P * N * 4, &full[slot]);
      }
      issued |= 1u << slot;
      parity = (parity & ~(1u << slot)) | (sphase << slot);
      if (++slot == NS) {
        slot = 0;
        sphase ^= 1;
      }
    }
  }
  if (failed) {
    if (!*abort_flag) report(p.status, RSSM_ERR_TIMEOUT);
    *abort_flag = 1;
  }
  // Whether or not the run aborted, return only once every copy issued here
  // has landed: consumers that give up later must not leave the CTA exiting
  // with a copy still writing its shared memory.
  for (int s = 0; s < NS; ++s)
    if (issued & (1u << s)) mbar_wait(&full[s], (parity >> s) & 1u);
}



int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

template <typename F>
cudaError_t dispatch_shape(int P, int N, int bf16, F &&f) {
#define RSSM_M2_CASE(PP, NN)                                                                    \
  if (P == PP && N == NN)                                                                       \
    return bf16 ? f(std::integral_constant<int, PP>{}, std::integral_constant<int, NN>{},       \
                    __nv_bfloat16{})                                                            \
                : f(std::integral_constant<int, PP>{}, std::integral_constant<int, NN>{}, 0.0f);
  RSSM_M2_CASE(64, 64)
  RSSM_M2_CASE(64, 128)
  RSSM_M2_CASE(128, 64)
  RSSM_M2_CASE(128, 128)
#undef RSSM_M2_CASE
  return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace rssm
