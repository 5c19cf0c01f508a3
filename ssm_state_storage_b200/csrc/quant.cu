// quant.cu -- read copy of checkpoint tiles (FP8 E4M3, or NVFP4: E2M1 codes,
// an E4M3 scale per 16 elements and an fp32 scale per tile), and the in-place
// deq(Q(.)) rounding used by the quantised-checkpoint comparison baseline.
// The arithmetic is the one of codec.cuh, shared with the fused fold epilogue
// of the decode kernels, so both produce identical codes for identical input.
#include "codec.cuh"
#include "common.cuh"
#include "internal.h"

namespace rssm {
namespace {

__global__ void __launch_bounds__(kThreads) fp8_tiles_kernel(int64_t n_per_tile, const float *src,
                                                             uint8_t *codes, int roundtrip,
                                                             float *dst) {
  const int64_t base = (int64_t)blockIdx.x * n_per_tile;
  for (int64_t i = threadIdx.x; i < n_per_tile; i += kThreads) {
    const float v = src[base + i];
    const uint32_t c = e4m3_encode(v);
    if (roundtrip) dst[base + i] = e4m3_decode(c);
    else codes[base + i] = (uint8_t)c;
  }
}

__global__ void __launch_bounds__(kThreads) nvfp4_tiles_kernel(int rows, int cols, const float *src,
                                                               uint8_t *codes, uint8_t *scales,
                                                               float *gscale, int roundtrip,
                                                               float *dst) {
  __shared__ float s_red[kThreads / 32];
  const int64_t tile = blockIdx.x;
  const int64_t n = (int64_t)rows * cols;
  const float *x = src + tile * n;
  float m = 0.f;
  for (int64_t i = threadIdx.x; i < n; i += kThreads) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = s_red[0];
  for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, s_red[w]);
  const float sg = nvfp4_tile_scale(amax);
  const int nb = cols / 16;
  for (int64_t blk = threadIdx.x; blk < (int64_t)rows * nb; blk += kThreads) {
    const int64_t r = blk / nb, j = blk - r * nb;
    const float *xb = x + r * cols + j * 16;
    float bm = 0.f;
    for (int e = 0; e < 16; ++e) bm = fmaxf(bm, fabsf(xb[e]));
    const uint32_t sc = nvfp4_block_code(bm, sg);
    const float d = nvfp4_step(sc, sg);
    const float sb = e4m3_decode(sc);
    for (int e = 0; e < 16; e += 2) {
      const uint32_t byte = nvfp4_pack2(xb[e], xb[e + 1], d);
      if (roundtrip) {
        float *db = dst + tile * n + r * cols + j * 16;
        db[e] = nvfp4_value(byte & 0xF, sb, sg);
        db[e + 1] = nvfp4_value(byte >> 4, sb, sg);
      } else {
        codes[tile * (n / 2) + r * (cols / 2) + j * 8 + e / 2] = (uint8_t)byte;
      }
    }
    if (!roundtrip) scales[tile * (rows * nb) + blk] = (uint8_t)sc;
  }
  if (!roundtrip && threadIdx.x == 0) gscale[tile] = sg;
}

}  // namespace

cudaError_t quant_launch(int fmt, int ntile, int rows, int cols, const float *src, uint8_t *codes,
                         uint8_t *scales, float *gscale, int roundtrip, float *dst,
                         cudaStream_t s) {
  if (ntile == 0) return cudaSuccess;
  if (fmt == 1) {
    fp8_tiles_kernel<<<ntile, kThreads, 0, s>>>((int64_t)rows * cols, src, codes, roundtrip, dst);
  } else if (fmt == 2) {
    nvfp4_tiles_kernel<<<ntile, kThreads, 0, s>>>(rows, cols, src, codes, scales, gscale,
                                                  roundtrip, dst);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rssm
