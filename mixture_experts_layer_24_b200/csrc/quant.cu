// quant.cu -- FP8 (OCP E4M3) block quantiser.
//
// Per block of block_rows x 128 elements: s = amax / 448 (IEEE fp32 divide;
// s = 1 for an all-zero block), q = e4m3(v / s) rounded to nearest even with
// saturation to +-448 (cvt.rn.satfinite). Weights use 128 x 128 blocks,
// activations 1 x 128 (per token per 128 columns), the FP8 layout of
// DeepSeek-class checkpoints served by vLLM-Moet (topairepos.com page, model
// table; the Qwen3.8 FP8 MoE GEMV row). amax is a max (order-free) and every
// other step is one correctly-rounded operation, so the codes and scales are
// bit-exact against any implementation of the same rule.
#include "common.cuh"
#include "internal.h"

namespace moe {

__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// One CTA (256 threads) per 128 x 128 block.
__global__ void __launch_bounds__(256) quant_block128_kernel(const uint16_t* __restrict__ src, int rows, int cols,
                                                              uint8_t* __restrict__ q, float* __restrict__ scales) {
  __shared__ float red[8];
  const int rb = blockIdx.y, cb = blockIdx.x;
  const int c = cb * 128 + (threadIdx.x & 15) * 8;
  const int r0 = rb * 128 + (threadIdx.x >> 4);
  float amax = 0.0f;
  for (int r = r0; r < min(rows, rb * 128 + 128); r += 16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * cols + c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xffff0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
  if (threadIdx.x == 0) scales[(size_t)rb * (cols / 128) + cb] = s;
  for (int r = r0; r < min(rows, rb * 128 + 128); r += 16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (size_t)r * cols + c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t a = to_e4m3(__uint_as_float(w[i] << 16) / s);
      const uint32_t b = to_e4m3(__uint_as_float(w[i] & 0xffff0000u) / s);
      out[i >> 1] |= (a | (b << 8)) << ((i & 1) * 16);
    }
    *reinterpret_cast<uint2*>(q + (size_t)r * cols + c) = make_uint2(out[0], out[1]);
  }
}

// One warp per (row, 128-column group); lane l owns columns 4l..4l+3.
// Optional row gather (src row = perm_src[row]) and row limit (offsets[E]).
__global__ void __launch_bounds__(256) quant_rows_kernel(const uint16_t* __restrict__ src,
                                                          const int32_t* __restrict__ perm_src,
                                                          const int32_t* __restrict__ offsets, int E, int rows,
                                                          int cols, uint8_t* __restrict__ q,
                                                          float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int groups = cols / 128;
  const int row = (int)(wid / groups), g = (int)(wid - (int64_t)row * groups);
  if (row >= rows) return;
  if (offsets && row >= offsets[E]) return;
  const int srow = perm_src ? perm_src[row] : row;
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + (size_t)srow * cols + g * 128 + lane * 4));
  const float f0 = __uint_as_float(v.x << 16), f1 = __uint_as_float(v.x & 0xffff0000u);
  const float f2 = __uint_as_float(v.y << 16), f3 = __uint_as_float(v.y & 0xffff0000u);
  float amax = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
  const uint32_t packed = (uint32_t)to_e4m3(f0 / s) | ((uint32_t)to_e4m3(f1 / s) << 8) |
                          ((uint32_t)to_e4m3(f2 / s) << 16) | ((uint32_t)to_e4m3(f3 / s) << 24);
  *reinterpret_cast<uint32_t*>(q + (size_t)row * cols + g * 128 + lane * 4) = packed;
  if (lane == 0) scales[(size_t)row * groups + g] = s;
}

// One warp per (token, 128-column group), lane l owns columns 4l..4l+3: the
// same codes and scale as quant_rows_kernel on each gathered row, computed
// once per token and stored to the token's K pair rows (inv[t*K+k] = its
// sorted row; -1: a dropped pair, skipped).
__global__ void __launch_bounds__(256) quant_scatter_rows_kernel(const uint16_t* __restrict__ src,
                                                                  const int32_t* __restrict__ inv, int T, int K,
                                                                  int cols, uint8_t* __restrict__ q,
                                                                  float* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int groups = cols / 128;
  const int t = (int)(wid / groups), g = (int)(wid - (int64_t)t * groups);
  if (t >= T) return;
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(src + (size_t)t * cols + g * 128 + lane * 4));
  const float f0 = __uint_as_float(v.x << 16), f1 = __uint_as_float(v.x & 0xffff0000u);
  const float f2 = __uint_as_float(v.y << 16), f3 = __uint_as_float(v.y & 0xffff0000u);
  float amax = fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float sc = (amax == 0.0f) ? 1.0f : amax / 448.0f;
  const uint32_t packed = (uint32_t)to_e4m3(f0 / sc) | ((uint32_t)to_e4m3(f1 / sc) << 8) |
                          ((uint32_t)to_e4m3(f2 / sc) << 16) | ((uint32_t)to_e4m3(f3 / sc) << 24);
  for (int k = 0; k < K; ++k) {
    const int p = __ldg(inv + (size_t)t * K + k);
    if (p < 0) continue;
    *reinterpret_cast<uint32_t*>(q + (size_t)p * cols + g * 128 + lane * 4) = packed;
    if (lane == 0) scales[(size_t)p * groups + g] = sc;
  }
}

cudaError_t launch_quant_scatter_rows(const void* x, const int32_t* inv, int T, int K, int H, uint8_t* xq, float* xs,
                                      cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  const int64_t warps = (int64_t)T * (H / 128);
  return launch_ex(quant_scatter_rows_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, pdl,
                   static_cast<const uint16_t*>(x), inv, T, K, H, xq, xs);
}

cudaError_t launch_quant_e4m3(const void* src, int rows, int cols, int block_rows, uint8_t* q, float* scales,
                              cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const uint16_t* sb = static_cast<const uint16_t*>(src);
  if (block_rows == 128) {
    dim3 grid(cols / 128, (rows + 127) / 128);
    quant_block128_kernel<<<grid, 256, 0, s>>>(sb, rows, cols, q, scales);
  } else {
    const int64_t warps = (int64_t)rows * (cols / 128);
    quant_rows_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, s>>>(sb, nullptr, nullptr, 0, rows, cols, q, scales);
  }
  return cudaGetLastError();
}

cudaError_t launch_gather_quant_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E, int P,
                                     int H, uint8_t* xq, float* xs, cudaStream_t s, bool pdl) {
  if (P <= 0) return cudaSuccess;
  const int64_t warps = (int64_t)P * (H / 128);
  return launch_ex(quant_rows_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, pdl,
                   static_cast<const uint16_t*>(x), perm_src, offsets, E, P, H, xq, xs);
}

cudaError_t launch_quant_rows_e4m3_count(const void* src, const int32_t* offsets, int E, int rows, int cols,
                                         uint8_t* q, float* scales, cudaStream_t s, bool pdl) {
  if (rows <= 0) return cudaSuccess;
  const int64_t warps = (int64_t)rows * (cols / 128);
  return launch_ex(quant_rows_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, s, pdl,
                   static_cast<const uint16_t*>(src), static_cast<const int32_t*>(nullptr), offsets, E, rows, cols,
                   q, scales);
}

}  // namespace moe
