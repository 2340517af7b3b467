// mx.cu -- OCP Microscaling (MX) quantisers for the FP4 expert path.
//
// The pages' checkpoint serves its experts in FP4 (vLLM-Moet, topairepos.com
// page, hybrid results table, row "quality, paired against the native FP4
// reference"); they give no block size or scale type, and this library reads
// them as the open MX formats: MXFP4 weights (E2M1 elements) and MX e4m3
// activations, one E8M0 scale (a power of two, stored as exponent + 127) per
// 32 consecutive elements along K:
//   X = 2^(floor(log2 amax) - emax), emax = 2 (E2M1, max 6) or 8 (E4M3, max
//   448), clamped to 2^-127 .. 2^127 (2^-127 for an all-zero block);
//   q = encode(v / X), round to nearest even, saturating.
// amax is a max (order-free), v / X is an exact power-of-two scaling (one
// correctly rounded multiply), and the encoders are exact tables of
// comparisons, so codes and scales are bit-exact against any implementation
// of the same rule.
//
// Layouts:
//   - e2m1 codes are packed two per byte, element 2i in the low nibble;
//   - plain scales are [rows, cols/32] bytes;
//   - the tensor cores take scales as 512-byte blocks, one per 128 rows x 4
//     scales (128 K elements): byte 16*(r%32) + 4*(r/32) + j holds row r's
//     scale j. Down-projection scales are kept as [H/128][I/128][512]; gate/up
//     scales as [I/128][H/128][2][512], the gate block of row tile mt beside
//     the up block of the same tile (rows I + 128 mt ..), so that one copy
//     brings both for several K blocks; activation scales as
//     [N tile][K/128][512], row r of the block being the tile's r-th pair.
#include "common.cuh"
#include "internal.h"

namespace moe {

// floor(log2 amax) - emax, clamped to [-127, 127]; amax >= 0 and finite.
__device__ __forceinline__ int mx_scale_exp(float amax, int emax) {
  if (amax == 0.0f) return -127;
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xffu);
  const int fl = ex ? ex - 127 : (31 - __clz((int)(b & 0x7fffffu))) - 149;
  const int s = fl - emax;
  return s < -127 ? -127 : (s > 127 ? 127 : s);
}

// 2^-sexp as fp32 (exact; sexp <= 125 for bf16 inputs, so the result is normal).
__device__ __forceinline__ float mx_inv_scale(int sexp) { return __int_as_float((127 - sexp) << 23); }

// fp32 -> E2M1 code (sign bit 3), round to nearest even, saturating at 6.
__device__ __forceinline__ uint32_t to_e2m1(float v) {
  const uint32_t sign = (__float_as_uint(v) >> 31) << 3;
  const float a = fabsf(v);
  uint32_t c;
  if (a <= 0.25f) c = 0;        // ties to 0 (even)
  else if (a < 0.75f) c = 1;    // 0.5
  else if (a <= 1.25f) c = 2;   // 1.0 (0.75 and 1.25 tie to the even 1.0)
  else if (a < 1.75f) c = 3;    // 1.5
  else if (a <= 2.5f) c = 4;    // 2.0
  else if (a < 3.5f) c = 5;     // 3.0
  else if (a <= 5.0f) c = 6;    // 4.0
  else c = 7;                   // 6.0 (and everything above)
  return sign | c;
}

__device__ __forceinline__ uint32_t to_e4m3_bits(float v) {
  return static_cast<uint32_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// 32 bf16 values (64 bytes at p) -> their amax.
__device__ __forceinline__ void load32_bf16(const uint16_t* p, float (&f)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(q + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
      f[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
}

__device__ __forceinline__ float amax32(const float (&f)[32]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(f[i]));
  return m;
}

// Quantises one 32-element block: e4m3 codes to q (32 bytes) or packed e2m1
// codes (16 bytes); returns the E8M0 scale byte.
__device__ __forceinline__ uint32_t quant_block32(const float (&f)[32], int elem_e4m3, uint8_t* q) {
  const int sexp = mx_scale_exp(amax32(f), elem_e4m3 ? 8 : 2);
  const float inv = mx_inv_scale(sexp);
  if (elem_e4m3) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = to_e4m3_bits(f[4 * i] * inv) | (to_e4m3_bits(f[4 * i + 1] * inv) << 8) |
             (to_e4m3_bits(f[4 * i + 2] * inv) << 16) | (to_e4m3_bits(f[4 * i + 3] * inv) << 24);
    uint4* d = reinterpret_cast<uint4*>(q);
    d[0] = make_uint4(w[0], w[1], w[2], w[3]);
    d[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t v = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) v |= to_e2m1(f[8 * i + k] * inv) << (4 * k);
      w[i] = v;
    }
    *reinterpret_cast<uint4*>(q) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return (uint32_t)(sexp + 127);
}

// Plain quantiser: one thread per 32-element block of a [rows, cols] bf16 matrix.
__global__ void __launch_bounds__(256) quant_mx_kernel(const uint16_t* __restrict__ src, int rows, int cols,
                                                        int elem_e4m3, uint8_t* __restrict__ q,
                                                        uint8_t* __restrict__ scales) {
  const int nb = cols / 32;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)rows * nb) return;
  const int r = (int)(i / nb), b = (int)(i - (int64_t)r * nb);
  float f[32];
  load32_bf16(src + (size_t)r * cols + (size_t)b * 32, f);
  uint8_t* qd = elem_e4m3 ? q + (size_t)r * cols + (size_t)b * 32 : q + (size_t)r * (cols / 2) + (size_t)b * 16;
  scales[(size_t)r * nb + b] = (uint8_t)quant_block32(f, elem_e4m3, qd);
}

cudaError_t launch_quant_mx(const void* src, int rows, int cols, int elem_e4m3, uint8_t* q, uint8_t* scales,
                            cudaStream_t s) {
  const int64_t n = (int64_t)rows * (cols / 32);
  if (n <= 0) return cudaSuccess;
  quant_mx_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(static_cast<const uint16_t*>(src), rows, cols,
                                                              elem_e4m3, q, scales);
  return cudaGetLastError();
}

// Plain weight scales [rows, K/32] -> blocked; one thread per (row, 4-scale
// word). split_rows = 0: [rows/128][K/128][512]; split_rows = I (gate/up,
// rows = 2I): [I/128][K/128][2][512], rows >= I going to the second block.
__global__ void __launch_bounds__(256) mx_block_scales_kernel(const uint8_t* __restrict__ s, int rows, int K,
                                                               int split_rows, uint8_t* __restrict__ blk) {
  const int nkb = K / 128;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)rows * nkb) return;
  const int r = (int)(i / nkb), kb = (int)(i - (int64_t)r * nkb);
  const uint32_t w = *reinterpret_cast<const uint32_t*>(s + (size_t)r * (K / 32) + 4 * kb);
  const int rr = r % 128;
  size_t block;
  if (split_rows > 0) {
    const int which = r >= split_rows ? 1 : 0;
    const int mt = (r - which * split_rows) / 128;
    block = ((size_t)mt * nkb + kb) * 2 + which;
  } else {
    block = (size_t)(r / 128) * nkb + kb;
  }
  *reinterpret_cast<uint32_t*>(blk + block * 512 + 16 * (rr % 32) + 4 * (rr / 32)) = w;
}

cudaError_t launch_mx_block_scales(const uint8_t* scales, int rows, int K, int split_rows, uint8_t* blocked,
                                   cudaStream_t s) {
  const int64_t n = (int64_t)rows * (K / 128);
  if (n <= 0) return cudaSuccess;
  mx_block_scales_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(scales, rows, K, split_rows, blocked);
  return cudaGetLastError();
}

// Activation rows of the sorted pairs: row p (< offsets[E]) is token
// perm_src[p] quantised to MX e4m3 (codes [P, H]); its scales go to the
// blocked layout of its N tile: tile nt_prefix[e] + (p - offsets[e]) / bn,
// block row (p - offsets[e]) % bn. Rows of an expert with no tiles (no
// registered weights) are skipped. One warp per row, lanes over the blocks.
__global__ void __launch_bounds__(256) quant_mx_pairs_kernel(const uint16_t* __restrict__ x,
                                                              const int32_t* __restrict__ perm_src,
                                                              const int32_t* __restrict__ offsets,
                                                              const int32_t* __restrict__ nt_prefix, int E, int bn,
                                                              int P, int H, uint8_t* __restrict__ xq,
                                                              uint8_t* __restrict__ sfb) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= P || p >= offsets[E]) return;
  int lo = 0, hi = E;  // expert e with offsets[e] <= p < offsets[e + 1] (the last such e)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (offsets[mid] <= p) lo = mid;
    else hi = mid;
  }
  const int e = lo;
  if (nt_prefix[e + 1] == nt_prefix[e]) return;  // no tiles: the pair is dropped
  const int local = p - offsets[e];
  const int ng = nt_prefix[e] + local / bn, n = local % bn;
  const int t = perm_src[p];
  const int nkb = H / 128;
  for (int b = lane; b < H / 32; b += 32) {
    float f[32];
    load32_bf16(x + (size_t)t * H + (size_t)b * 32, f);
    const uint32_t sb = quant_block32(f, 1, xq + (size_t)p * H + (size_t)b * 32);
    const int kb = b >> 2, j = b & 3;
    sfb[((size_t)ng * nkb + kb) * 512 + 16 * (n % 32) + 4 * (n / 32) + j] = (uint8_t)sb;
  }
}

cudaError_t launch_quant_mx_pairs(const void* x, const int32_t* perm_src, const int32_t* offsets,
                                  const int32_t* nt_prefix, int E, int bn, int P, int H, uint8_t* xq, uint8_t* sfb,
                                  cudaStream_t s, bool pdl) {
  if (P <= 0) return cudaSuccess;
  return launch_ex(quant_mx_pairs_kernel, dim3((P + 7) / 8), dim3(256), 0, s, pdl, static_cast<const uint16_t*>(x),
                   perm_src, offsets, nt_prefix, E, bn, P, H, xq, sfb);
}

}  // namespace moe
