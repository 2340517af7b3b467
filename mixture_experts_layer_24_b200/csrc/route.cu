// route.cu -- router logits and top-k selection.
//
// Router of a routed MoE layer (vLLM-Moet, topairepos.com page: DeepSeek-V4.1
// layers of 384 routed experts, top-k routing; "identical requests return
// identical logits at any batch size" is the results-table "quality" row).
//
// Logit order (the contract both this kernel and the CPU oracle follow):
// H is cut into 16 contiguous segments of L = H/16; segment s accumulates
// fmaf(x[h], Wr[e][h], acc) from +0 over its h in increasing order; the 16
// partials are summed by the pairwise tree p[s] += p[s+o], o = 8, 4, 2, 1,
// which is exactly what an xor-butterfly over 16 lanes leaves in every lane;
// then one fp32 add of bias[e]. A token's logits therefore depend on that
// token alone, whatever the batch.
#include "common.cuh"
#include "internal.h"

namespace moe {

// One 16-lane group per (expert, token group); lane s owns segment s.
// EPC experts per CTA, TG tokens per thread.
template <int EPC, int TG>
__global__ void __launch_bounds__(EPC * 16) router_logits_kernel(const uint16_t* __restrict__ x,
                                                                  const float* __restrict__ wr,
                                                                  const float* __restrict__ bias, int T, int H,
                                                                  int E, float* __restrict__ logits) {
  const int s = threadIdx.x & 15;
  const int e = blockIdx.x * EPC + (threadIdx.x >> 4);
  const int t0 = blockIdx.y * TG;
  const int L = H >> 4;
  float acc[TG];
#pragma unroll
  for (int i = 0; i < TG; ++i) acc[i] = 0.0f;

  if (e < E) {
    const float* w = wr + (size_t)e * H + (size_t)s * L;
    const uint16_t* xs = x + (size_t)t0 * H + (size_t)s * L;
    const int ntok = min(TG, T - t0);
#pragma unroll 2
    for (int h = 0; h < L; h += 8) {
      const float4 wa = __ldg(reinterpret_cast<const float4*>(w + h));
      const float4 wb = __ldg(reinterpret_cast<const float4*>(w + h + 4));
#pragma unroll
      for (int i = 0; i < TG; ++i) {
        if (i < ntok) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xs + (size_t)i * H + h));
          float a = acc[i];
          a = fmaf(__uint_as_float(xv.x << 16), wa.x, a);
          a = fmaf(__uint_as_float(xv.x & 0xffff0000u), wa.y, a);
          a = fmaf(__uint_as_float(xv.y << 16), wa.z, a);
          a = fmaf(__uint_as_float(xv.y & 0xffff0000u), wa.w, a);
          a = fmaf(__uint_as_float(xv.z << 16), wb.x, a);
          a = fmaf(__uint_as_float(xv.z & 0xffff0000u), wb.y, a);
          a = fmaf(__uint_as_float(xv.w << 16), wb.z, a);
          a = fmaf(__uint_as_float(xv.w & 0xffff0000u), wb.w, a);
          acc[i] = a;
        }
      }
    }
  }
  // pairwise tree over the 16 segments (xor offsets stay inside the 16-lane group)
#pragma unroll
  for (int i = 0; i < TG; ++i) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) acc[i] = acc[i] + __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (s == 0 && e < E) {
    const float b = bias ? bias[e] : 0.0f;
#pragma unroll
    for (int i = 0; i < TG; ++i) {
      if (t0 + i < T) logits[(size_t)(t0 + i) * E + e] = bias ? acc[i] + b : acc[i];
    }
  }
}

cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  if (T <= 4) {
    dim3 grid((E + 3) / 4, (T + 3) / 4);
    router_logits_kernel<4, 4><<<grid, 64, 0, s>>>(xb, wr, bias, T, H, E, logits);
  } else if (T <= 64) {
    dim3 grid((E + 7) / 8, (T + 7) / 8);
    router_logits_kernel<8, 8><<<grid, 128, 0, s>>>(xb, wr, bias, T, H, E, logits);
  } else {
    dim3 grid((E + 15) / 16, (T + 15) / 16);
    router_logits_kernel<16, 16><<<grid, 256, 0, s>>>(xb, wr, bias, T, H, E, logits);
  }
  return cudaGetLastError();
}

// ----------------------------------------------------------------- top-k --
// One warp per token. Round r picks the best expert strictly after round r-1's
// pick in the total order (logit desc, expert asc), so nothing is marked and
// ties (including +0 == -0) resolve to the lower index. Weights:
// expf(l_k - l_0), summed k = 0..K-1 in order, one IEEE divide each.

__device__ __forceinline__ bool ranks_before(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                    int32_t* __restrict__ idx, float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* l = logits + (size_t)t * E;

  float prev_v = __int_as_float(0x7f800000);  // +inf
  int prev_e = -1;
  float my_v = 0.0f;
  int my_e = 0;
  for (int r = 0; r < K; ++r) {
    float best_v = 0.0f;
    int best_e = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = __ldg(l + e);
      const bool after_prev = ranks_before(prev_v, prev_e, v, e);
      if (after_prev && (best_e == 0x7fffffff || ranks_before(v, e, best_v, best_e))) {
        best_v = v;
        best_e = e;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best_v, o);
      const int oe = __shfl_xor_sync(0xffffffffu, best_e, o);
      if (oe != 0x7fffffff && (best_e == 0x7fffffff || ranks_before(ov, oe, best_v, best_e))) {
        best_v = ov;
        best_e = oe;
      }
    }
    prev_v = best_v;
    prev_e = best_e;
    if (lane == r) {
      my_v = best_v;
      my_e = best_e;
    }
  }
  const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = (lane < K) ? expf(my_v - l0) : 0.0f;
  float sum = 0.0f;
  for (int k = 0; k < K; ++k) sum = sum + __shfl_sync(0xffffffffu, ex, k);
  if (lane < K) {
    idx[(size_t)t * K + lane] = my_e;
    w[(size_t)t * K + lane] = ex / sum;
  }
}

cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w, int* status,
                        cudaStream_t s) {
  (void)status;
  if (T <= 0) return cudaSuccess;
  const int warps = 8;
  topk_kernel<<<(T + warps - 1) / warps, warps * 32, 0, s>>>(logits, T, E, K, idx, w);
  return cudaGetLastError();
}

}  // namespace moe
