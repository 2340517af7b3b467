// combine.cu -- weighted scatter-combine back to token order:
// out[t, :] = bf16_rne(((y[inv[t,0]] + y[inv[t,1]]) + ...) + y[inv[t,K-1]]).
// The sum starts from the k = 0 term and runs k ascending in fp32, one
// rounding to bf16 at the end, so the result is bit-exact against any
// implementation of the same order. The routing weight is already inside
// y_pair (applied in the down-projection epilogue).
#include "common.cuh"
#include "internal.h"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y,
                                                       const int32_t* __restrict__ inv, int K, int H4,
                                                       uint2* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int v = blockIdx.y * blockDim.x + threadIdx.x;
  if (v >= H4) return;
  const int32_t* iv = inv + (size_t)t * K;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  bool have = false;
  // eight pairs at a time: their inv entries, then their rows, are loaded
  // before any is added; the adds run k ascending as before
  for (int k0 = 0; k0 < K; k0 += 8) {
    int pk[8];
    float4 a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) pk[u] = k0 + u < K ? __ldg(iv + k0 + u) : -1;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (pk[u] >= 0) a[u] = __ldg(y + (size_t)pk[u] * H4 + v);  // p < 0: a dropped pair contributes nothing
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (pk[u] < 0) continue;
      if (!have) {
        acc = a[u];
        have = true;
      } else {
        acc.x = acc.x + a[u].x;
        acc.y = acc.y + a[u].y;
        acc.z = acc.z + a[u].z;
        acc.w = acc.w + a[u].w;
      }
    }
  }
  const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 o;
  o.x = *reinterpret_cast<const uint32_t*>(&lo);
  o.y = *reinterpret_cast<const uint32_t*>(&hi);
  out[(size_t)t * H4 + v] = o;
}

cudaError_t launch_combine(const float* y, const int32_t* inv, int T, int K, int H, void* out, cudaStream_t s,
                           bool pdl) {
  if (T <= 0) return cudaSuccess;
  const int H4 = H / 4;
  dim3 grid(T, (H4 + 255) / 256);
  return launch_ex(combine_kernel, grid, dim3(256), 0, s, pdl, reinterpret_cast<const float4*>(y), inv, K, H4,
                   static_cast<uint2*>(out));
}

}  // namespace moe
