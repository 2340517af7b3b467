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

// ------------------------------------------------- warp top-k (registers) --
// The token's logits sit in registers, NJ = ceil(E/32) per lane (expert
// lane + 32 j). Each of the K rounds takes the lane's best expert not yet
// taken (a tree over its NJ slots), then a warp arg-max; all comparisons use
// the same total order (logit desc, expert asc), so ties (+0 == -0 included)
// go to the lower index. Weights as in topk_kernel. Logits are read through L2
// (ld.global.cg): other CTAs wrote them.
struct Cand {
  float v;
  int e;  // INT_MAX = none
};

__device__ __forceinline__ Cand better(Cand a, Cand b) {
  if (b.e == 0x7fffffff) return a;
  if (a.e == 0x7fffffff) return b;
  return ranks_before(a.v, a.e, b.v, b.e) ? a : b;
}

template <int NJ>
__device__ __forceinline__ void topk_warp(const float* l, int E, int K, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float v[NJ];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int e = lane + 32 * j;
    v[j] = e < E ? __ldcg(l + e) : 0.0f;
    if (e >= E) taken |= 1u << j;
  }
  float my_v = 0.0f;
  int my_e = 0;
  for (int r = 0; r < K; ++r) {
    Cand c[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) c[j] = Cand{v[j], ((taken >> j) & 1u) ? 0x7fffffff : lane + 32 * j};
#pragma unroll
    for (int step = 1; step < NJ; step <<= 1) {
#pragma unroll
      for (int j = 0; j + step < NJ; j += 2 * step) c[j] = better(c[j], c[j + step]);
    }
    Cand b = c[0];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      Cand other{__shfl_xor_sync(0xffffffffu, b.v, o), __shfl_xor_sync(0xffffffffu, b.e, o)};
      b = better(b, other);
    }
    if (b.e != 0x7fffffff && (b.e & 31) == lane) taken |= 1u << (b.e >> 5);
    if (lane == r) {
      my_v = b.v;
      my_e = b.e;
    }
  }
  const float l0 = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = (lane < K) ? expf(my_v - l0) : 0.0f;
  float sum = 0.0f;
  for (int k = 0; k < K; ++k) sum = sum + __shfl_sync(0xffffffffu, ex, k);
  if (lane < K) {
    idx[lane] = my_e;
    w[lane] = ex / sum;
  }
}

__device__ __forceinline__ void topk_warp_any(const float* l, int E, int K, int32_t* idx, float* w) {
  const int nj = (E + 31) >> 5;
  if (nj <= 1) topk_warp<1>(l, E, K, idx, w);
  else if (nj <= 4) topk_warp<4>(l, E, K, idx, w);
  else if (nj <= 8) topk_warp<8>(l, E, K, idx, w);
  else if (nj <= 12) topk_warp<12>(l, E, K, idx, w);
  else if (nj <= 16) topk_warp<16>(l, E, K, idx, w);
  else topk_warp<32>(l, E, K, idx, w);
}

__global__ void __launch_bounds__(256) topk_warp_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                         int32_t* __restrict__ idx, float* __restrict__ w) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_warp_any(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
}

cudaError_t launch_topk_warp(const float* logits, int T, int E, int K, int32_t* idx, float* w, cudaStream_t s,
                             bool pdl) {
  if (T <= 0) return cudaSuccess;
  return launch_ex(topk_warp_kernel, dim3((T + 7) / 8), dim3(256), 0, s, pdl, logits, T, E, K, idx, w);
}

// ------------------------------------------------- decode-regime router --
// One CTA per (EPC experts, TG tokens). The CTA's Wr segments (1 KB each at
// H = 4096) and token segments are staged in padded shared memory by TMA bulk
// copies -- one request per segment, all in flight at once -- then thread
// (expert el, segment s) runs the segment's fma chain for every token of the
// group and the 16-lane tree sums the partials (the same order as
// router_logits_kernel). With fuse_topk, the last CTA of a token group (an
// arrival counter) selects the group's top-k, one warp per token, and returns
// the counter to zero; otherwise a top-k kernel follows.
template <int EPC, int TG>
__global__ void __launch_bounds__(EPC * 16) route_small_kernel(const uint16_t* __restrict__ x,
                                                                const float* __restrict__ wr,
                                                                const float* __restrict__ bias, int T, int H,
                                                                int E, int K, float* __restrict__ logits,
                                                                int32_t* __restrict__ idx, float* __restrict__ w,
                                                                unsigned int* __restrict__ counters, int fuse_topk,
                                                                int* status) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_last;
  pdl_trigger();  // first kernel of a forward: the next one may launch (it waits for us)
  const int L = H >> 4;
  const int wst = L + 4;  // padded floats per Wr segment row
  const int xst = L + 8;  // padded bf16 per x segment row
  float* sw = reinterpret_cast<float*>(sm);
  uint16_t* sx = reinterpret_cast<uint16_t*>(sm + (size_t)EPC * 16 * wst * 4);
  const int s = threadIdx.x & 15, el = threadIdx.x >> 4;
  const int e0 = blockIdx.x * EPC;
  const int e = e0 + el;
  const int t0 = blockIdx.y * TG;
  const int ntok = min(TG, T - t0);
  const int nexp = min(EPC, E - e0);
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(b, (uint32_t)(nexp * 16 * L * 4 + ntok * 16 * L * 2));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < (nexp + ntok) * 16; i += blockDim.x) {
    if (i < nexp * 16) {
      const int ee = i >> 4, ss = i & 15;
      bulk_load(smem_u32(sw + (size_t)i * wst), wr + (size_t)(e0 + ee) * H + (size_t)ss * L, L * 4, b);
    } else {
      const int j = i - nexp * 16, tt = j >> 4, ss = j & 15;
      bulk_load(smem_u32(sx + (size_t)j * xst), x + (size_t)(t0 + tt) * H + (size_t)ss * L, L * 2, b);
    }
  }
  if (!mbar_wait(b, 0)) flag_status(status, MOE_DEV_TIMEOUT);

  float acc[TG];
#pragma unroll
  for (int i = 0; i < TG; ++i) acc[i] = 0.0f;
  if (el < nexp) {
    const float* wseg = sw + (size_t)(el * 16 + s) * wst;
#pragma unroll 2
    for (int h = 0; h < L; h += 8) {
      const float4 wa = *reinterpret_cast<const float4*>(wseg + h);
      const float4 wb = *reinterpret_cast<const float4*>(wseg + h + 4);
#pragma unroll
      for (int i = 0; i < TG; ++i) {
        if (i < ntok) {
          const uint4 xv = *reinterpret_cast<const uint4*>(sx + (size_t)(i * 16 + s) * xst + h);
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
#pragma unroll
  for (int i = 0; i < TG; ++i) {
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) acc[i] = acc[i] + __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
  if (s == 0 && e < E) {
    const float bv = bias ? bias[e] : 0.0f;
#pragma unroll
    for (int i = 0; i < TG; ++i)
      if (i < ntok) logits[(size_t)(t0 + i) * E + e] = bias ? acc[i] + bv : acc[i];
  }
  if (!fuse_topk) return;
  // ---- arrival: the last CTA of this token group runs the group's top-k
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(counters + blockIdx.y, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int i = warp; i < ntok; i += nw) {
    const int t = t0 + i;
    topk_warp_any(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
  }
  if (threadIdx.x == 0) counters[blockIdx.y] = 0u;
}

template <int EPC, int TG>
static cudaError_t launch_rs(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                             float* logits, int32_t* idx, float* w, unsigned int* counters, int fuse, int* status,
                             cudaStream_t s) {
  const int L = H >> 4;
  const size_t smem = (size_t)EPC * 16 * (L + 4) * 4 + (size_t)TG * 16 * (L + 8) * 2;
  auto kern = route_small_kernel<EPC, TG>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((E + EPC - 1) / EPC, (T + TG - 1) / TG);
  return launch_ex(kern, grid, dim3(EPC * 16), smem, s, false, static_cast<const uint16_t*>(x), wr, bias, T, H, E,
                   K, logits, idx, w, counters, fuse, status);
}

// ------------------------------------------------ prefill-regime router --
// Logits as a register-tiled fp32 GEMM in the same order. CTA tile: 32 tokens
// x 32 experts, 256 threads. Lane s = segment (two 16-lane groups per warp);
// group g = 2 warp + lane/16 owns an 8-token x 8-expert tile of segment-s
// partials (64 accumulators). Each stage brings RC consecutive h of every
// segment, for the CTA's 32 tokens and 32 experts, into padded shared memory
// (cp.async, two buffers); the h loop runs in increasing order inside each
// segment, so every partial is the same fma chain as in router_logits_kernel,
// and the 16-lane tree at the end sums them the same way.
constexpr int kRgT = 32, kRgE = 32, kRgC = 16;
constexpr int kRgXs = kRgC + 8;  // bf16 per padded (token, segment) row
constexpr int kRgWs = kRgC + 4;  // floats per padded (expert, segment) row
constexpr size_t kRgStageBytes = (size_t)kRgT * 16 * kRgXs * 2 + (size_t)kRgE * 16 * kRgWs * 4;

__global__ void __launch_bounds__(256, 1) route_gemm_kernel(const uint16_t* __restrict__ x,
                                                             const float* __restrict__ wr,
                                                             const float* __restrict__ bias, int T, int H, int E,
                                                             float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t sm[];
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = lane & 15, g = warp * 2 + (lane >> 4);
  const int tt0 = (g >> 2) * 8, ee0 = (g & 3) * 8;
  const int tb = blockIdx.y * kRgT, eb = blockIdx.x * kRgE;
  const int L = H >> 4, nsteps = L / kRgC;
  auto xs = [&](int buf) { return reinterpret_cast<uint16_t*>(sm + buf * kRgStageBytes); };
  auto ws = [&](int buf) {
    return reinterpret_cast<float*>(sm + buf * kRgStageBytes + (size_t)kRgT * 16 * kRgXs * 2);
  };
  auto load_stage = [&](int st, int buf) {
    const int h0 = st * kRgC;
    uint16_t* xd = xs(buf);
    float* wd = ws(buf);
    // x: (token, segment, 2 x 16-byte parts); rows past T re-read row T-1 (results discarded)
    for (int c = tid; c < kRgT * 16 * 2; c += 256) {
      const int part = c & 1, ts = c >> 1, ss = ts & 15, t = ts >> 4;
      const int row = min(tb + t, T - 1);
      cp_async16(xd + (size_t)ts * kRgXs + part * 8, x + (size_t)row * H + (size_t)ss * L + h0 + part * 8);
    }
    // Wr: (expert, segment, 4 x 16-byte parts)
    for (int c = tid; c < kRgE * 16 * 4; c += 256) {
      const int part = c & 3, es = c >> 2, ss = es & 15, e = es >> 4;
      const int row = min(eb + e, E - 1);
      cp_async16(wd + (size_t)es * kRgWs + part * 4, wr + (size_t)row * H + (size_t)ss * L + h0 + part * 4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  load_stage(0, 0);
  for (int st = 0; st < nsteps; ++st) {
    const int buf = st & 1;
    if (st + 1 < nsteps) {
      load_stage(st + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint16_t* xb = xs(buf);
    const float* wb = ws(buf);
#pragma unroll
    for (int hh = 0; hh < kRgC; hh += 4) {
      uint2 xv[8];
      float4 wv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) xv[i] = *reinterpret_cast<const uint2*>(xb + (size_t)((tt0 + i) * 16 + s) * kRgXs + hh);
#pragma unroll
      for (int j = 0; j < 8; ++j) wv[j] = *reinterpret_cast<const float4*>(wb + (size_t)((ee0 + j) * 16 + s) * kRgWs + hh);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x0 = __uint_as_float(xv[i].x << 16), x1 = __uint_as_float(xv[i].x & 0xffff0000u);
        const float x2 = __uint_as_float(xv[i].y << 16), x3 = __uint_as_float(xv[i].y & 0xffff0000u);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float a = acc[i][j];
          a = fmaf(x0, wv[j].x, a);
          a = fmaf(x1, wv[j].y, a);
          a = fmaf(x2, wv[j].z, a);
          a = fmaf(x3, wv[j].w, a);
          acc[i][j] = a;
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) acc[i][j] = acc[i][j] + __shfl_xor_sync(0xffffffffu, acc[i][j], o);
  if (s == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = tb + tt0 + i;
      if (t >= T) continue;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = eb + ee0 + j;
        if (e < E) logits[(size_t)t * E + e] = bias ? acc[i][j] + bias[e] : acc[i][j];
      }
    }
  }
}

cudaError_t launch_route_gemm(const void* x, const float* wr, const float* bias, int T, int H, int E,
                              float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if ((H >> 4) % kRgC != 0) return launch_router_logits(x, wr, bias, T, H, E, logits, s);
  const size_t smem = 2 * kRgStageBytes;
  cudaError_t err = cudaFuncSetAttribute(route_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((E + kRgE - 1) / kRgE, (T + kRgT - 1) / kRgT);
  return launch_ex(route_gemm_kernel, grid, dim3(256), smem, s, false, static_cast<const uint16_t*>(x), wr, bias, T,
                   H, E, logits);
}

// T <= 4: logits + fused top-k in one launch; up to 64 tokens: logits in
// 16-token groups, then the warp top-k kernel (programmatic launch).
cudaError_t launch_route_small(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                               float* logits, int32_t* idx, float* w, unsigned int* counters, int* status,
                               cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  if (T <= 2) return launch_rs<2, 2>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, status, s);
  if (T <= 4) return launch_rs<4, 4>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, status, s);
  cudaError_t err;
  if (T <= 8) err = launch_rs<4, 8>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 0, status, s);
  else err = launch_rs<4, 16>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 0, status, s);
  if (err != cudaSuccess) return err;
  return launch_topk_warp(logits, T, E, K, idx, w, s, pdl);
}

}  // namespace moe
