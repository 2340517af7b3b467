// route.cu -- router logits and top-k selection.
//
// Router of a routed MoE layer (vLLM-Moet, topairepos.com page: DeepSeek-V4.1
// layers of 384 routed experts, top-k routing; "identical requests return
// identical logits at any batch size" is the results-table "quality" row).
//
// Logit order (the contract both these kernels and the CPU oracle follow):
// h is cut into chunks of 8 (chunk c = h 8c..8c+7); lane j of a warp owns the
// chunks c = j, j+32, j+64, ... and runs fmaf(x[h], Wr[e][h], acc) from +0
// over them in increasing c (h increasing inside a chunk); the 32 lane
// partials are then summed by the xor butterfly (offsets 16, 8, 4, 2, 1),
// which leaves p[j] += p[j+o] (o = 16 .. 1) in every lane; then one fp32 add
// of bias[e]. Every warp load of Wr or x is 32 consecutive 16-byte pieces,
// and a token's logits depend on that token alone, whatever the batch.
#include "common.cuh"
#include "internal.h"

namespace moe {

// One warp per expert, TG tokens per warp; lane j owns chunks j, j+32, ...
// U chunks per lane are loaded before any is used, so a warp keeps
// U x (32 + 16 TG) bytes per lane in flight. Wr streams once per token
// group with coalesced 512-byte warp loads; x comes through L1 (shared by
// the CTA's warps, which all read the same tokens).
template <int TG, int U>
__device__ __forceinline__ void logits_warp(const uint16_t* __restrict__ x, const float* __restrict__ wrow, int T,
                                            int H, int t0, float (&acc)[TG]) {
  const int lane = threadIdx.x & 31;
  const int ntok = min(TG, T - t0);
#pragma unroll
  for (int i = 0; i < TG; ++i) acc[i] = 0.0f;
  for (int hb = lane * 8; hb < H; hb += 256 * U) {
    float4 wa[U], wb[U];
    uint4 xv[U][TG];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int h = hb + 256 * u;
      if (h < H) {
        wa[u] = __ldg(reinterpret_cast<const float4*>(wrow + h));
        wb[u] = __ldg(reinterpret_cast<const float4*>(wrow + h + 4));
#pragma unroll
        for (int i = 0; i < TG; ++i)
          if (i < ntok) xv[u][i] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + i) * H + h));
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (hb + 256 * u < H) {
#pragma unroll
        for (int i = 0; i < TG; ++i) {
          if (i < ntok) {
            const uint4 v = xv[u][i];
            float a = acc[i];
            a = fmaf(__uint_as_float(v.x << 16), wa[u].x, a);
            a = fmaf(__uint_as_float(v.x & 0xffff0000u), wa[u].y, a);
            a = fmaf(__uint_as_float(v.y << 16), wa[u].z, a);
            a = fmaf(__uint_as_float(v.y & 0xffff0000u), wa[u].w, a);
            a = fmaf(__uint_as_float(v.z << 16), wb[u].x, a);
            a = fmaf(__uint_as_float(v.z & 0xffff0000u), wb[u].y, a);
            a = fmaf(__uint_as_float(v.w << 16), wb[u].z, a);
            a = fmaf(__uint_as_float(v.w & 0xffff0000u), wb[u].w, a);
            acc[i] = a;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TG; ++i) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc[i] = acc[i] + __shfl_xor_sync(0xffffffffu, acc[i], o);
  }
}

// Loads in flight per lane for a token group of TG (registers: U (8 + 4 TG)).
template <int TG>
struct LogitsUnroll {
  static constexpr int value = TG <= 2 ? 8 : (TG <= 4 ? 4 : 2);
};

template <int TG>
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                             const float* __restrict__ wr,
                                                             const float* __restrict__ bias, int T, int H, int E,
                                                             float* __restrict__ logits) {
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int t0 = blockIdx.y * TG;
  if (e >= E) return;  // warp-uniform
  float acc[TG];
  logits_warp<TG, LogitsUnroll<TG>::value>(x, wr + (size_t)e * H, T, H, t0, acc);
  if ((threadIdx.x & 31) == 0) {
    const float b = bias ? bias[e] : 0.0f;
#pragma unroll
    for (int i = 0; i < TG; ++i)
      if (t0 + i < T) logits[(size_t)(t0 + i) * E + e] = bias ? acc[i] + b : acc[i];
  }
}

cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  const dim3 block(256);
  if (T <= 4) {
    router_logits_kernel<4><<<dim3((E + 7) / 8, (T + 3) / 4), block, 0, s>>>(xb, wr, bias, T, H, E, logits);
  } else {
    router_logits_kernel<8><<<dim3((E + 7) / 8, (T + 7) / 8), block, 0, s>>>(xb, wr, bias, T, H, E, logits);
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
// Same warp-per-expert logits (WPC experts per CTA, TG tokens per group); with
// fuse_topk, the last CTA of each token group (an arrival counter) selects the
// group's top-k, one warp per token, and returns the counter to zero;
// otherwise a top-k kernel follows.
template <int TG, int WPC>
__global__ void __launch_bounds__(WPC * 32) route_small_kernel(const uint16_t* __restrict__ x,
                                                           const float* __restrict__ wr,
                                                           const float* __restrict__ bias, int T, int H, int E, int K,
                                                           float* __restrict__ logits, int32_t* __restrict__ idx,
                                                           float* __restrict__ w, unsigned int* __restrict__ counters,
                                                           int fuse_topk) {
  __shared__ int s_last;
  pdl_trigger();  // first kernel of a forward: the next one may launch (it waits for us)
  const int warp = threadIdx.x >> 5;
  const int e = blockIdx.x * WPC + warp;
  const int t0 = blockIdx.y * TG;
  const int ntok = min(TG, T - t0);
  if (e < E) {
    float acc[TG];
    logits_warp<TG, LogitsUnroll<TG>::value>(x, wr + (size_t)e * H, T, H, t0, acc);
    if ((threadIdx.x & 31) == 0) {
      const float b = bias ? bias[e] : 0.0f;
#pragma unroll
      for (int i = 0; i < TG; ++i)
        if (i < ntok) logits[(size_t)(t0 + i) * E + e] = bias ? acc[i] + b : acc[i];
    }
  }
  if (!fuse_topk) return;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(counters + blockIdx.y, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = warp; i < ntok; i += WPC) {
    const int t = t0 + i;
    topk_warp_any(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
  }
  if (threadIdx.x == 0) counters[blockIdx.y] = 0u;
}

// Four warps per CTA: a 384-expert router spreads over 96 SMs.
constexpr int kRsWarps = 4;

template <int TG>
static cudaError_t launch_rs(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                             float* logits, int32_t* idx, float* w, unsigned int* counters, int fuse, cudaStream_t s) {
  dim3 grid((E + kRsWarps - 1) / kRsWarps, (T + TG - 1) / TG);
  return launch_ex(route_small_kernel<TG, kRsWarps>, grid, dim3(kRsWarps * 32), 0, s, false, static_cast<const uint16_t*>(x), wr, bias,
                   T, H, E, K, logits, idx, w, counters, fuse);
}

// T <= 8: logits + fused top-k in one launch; up to 64 tokens: logits in
// 8-token groups, then the warp top-k kernel (programmatic launch).
cudaError_t launch_route_small(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                               float* logits, int32_t* idx, float* w, unsigned int* counters, int* status,
                               cudaStream_t s, bool pdl) {
  (void)status;
  if (T <= 0) return cudaSuccess;
  if (T <= 1) return launch_rs<1>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, s);
  if (T <= 2) return launch_rs<2>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, s);
  if (T <= 4) return launch_rs<4>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, s);
  if (T <= 8) return launch_rs<8>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, s);
  cudaError_t err = launch_rs<8>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 0, s);
  if (err != cudaSuccess) return err;
  return launch_topk_warp(logits, T, E, K, idx, w, s, pdl);
}

// ------------------------------------------------ prefill-regime router --
// Register-tiled fp32 GEMM in the same order. CTA tile: 48 tokens x 16
// experts, 12 warps as 6 token groups x 2 expert groups; a warp owns 8 tokens
// x 8 experts and its lane j keeps the 64 lane-j partials (chunks j, j+32,
// ...). Each stage holds 256 consecutive h of the tile's tokens and experts
// in shared memory (cp.async, kRgStages buffers, kRgStages - 1 in flight):
// token rows as stored, each Wr row
// split into its chunks' first halves then second halves so that the 32
// lanes' 16-byte reads are consecutive.
constexpr int kRgT = 48, kRgE = 16, kRgStages = 3, kRgThreads = 384;
constexpr size_t kRgStageBytes = (size_t)kRgT * 256 * 2 + (size_t)kRgE * 256 * 4;

__global__ void __launch_bounds__(kRgThreads, 1) route_gemm_kernel(const uint16_t* __restrict__ x,
                                                             const float* __restrict__ wr,
                                                             const float* __restrict__ bias, int T, int H, int E,
                                                             float* __restrict__ logits) {
  extern __shared__ __align__(16) uint8_t sm[];
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tt0 = (warp >> 1) * 8, ee0 = (warp & 1) * 8;
  const int tb = blockIdx.y * kRgT, eb = blockIdx.x * kRgE;
  const int nsteps = H / 256;
  auto xs = [&](int buf) { return reinterpret_cast<uint16_t*>(sm + buf * kRgStageBytes); };
  auto ws = [&](int buf) { return reinterpret_cast<float*>(sm + buf * kRgStageBytes + (size_t)kRgT * 256 * 2); };
  auto load_stage = [&](int st, int buf) {
    const int h0 = st * 256;
    uint16_t* xd = xs(buf);
    float* wd = ws(buf);
    for (int c = tid; c < kRgT * 32; c += kRgThreads) {  // token row: 32 x 16 B
      const int t = c >> 5, part = c & 31;
      const int row = min(tb + t, T - 1);  // rows past T re-read row T-1 (results discarded)
      cp_async16(xd + (size_t)t * 256 + part * 8, x + (size_t)row * H + h0 + part * 8);
    }
    for (int c = tid; c < kRgE * 64; c += kRgThreads) {  // expert row: 64 x 16 B (32 chunks x 2 halves)
      const int e = c >> 6, q = c & 63, chunk = q >> 1, half = q & 1;
      const int row = min(eb + e, E - 1);
      cp_async16(wd + (size_t)e * 256 + half * 128 + chunk * 4, wr + (size_t)row * H + h0 + q * 4);
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

#pragma unroll
  for (int st = 0; st < kRgStages - 1; ++st) {
    if (st < nsteps) load_stage(st, st);
    asm volatile("cp.async.commit_group;" ::: "memory");  // empty groups keep the count uniform
  }
  for (int st = 0; st < nsteps; ++st) {
    const int buf = st % kRgStages;
    {
      const int nx = st + kRgStages - 1;  // its buffer was last read in iteration st - 1
      if (nx < nsteps) load_stage(nx, nx % kRgStages);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.wait_group %0;" ::"n"(kRgStages - 1) : "memory");
    __syncthreads();
    const uint16_t* xb = xs(buf);
    const float* wb = ws(buf);
    float xf[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = *reinterpret_cast<const uint4*>(xb + (size_t)(tt0 + i) * 256 + lane * 8);
      xf[i][0] = __uint_as_float(v.x << 16);
      xf[i][1] = __uint_as_float(v.x & 0xffff0000u);
      xf[i][2] = __uint_as_float(v.y << 16);
      xf[i][3] = __uint_as_float(v.y & 0xffff0000u);
      xf[i][4] = __uint_as_float(v.z << 16);
      xf[i][5] = __uint_as_float(v.z & 0xffff0000u);
      xf[i][6] = __uint_as_float(v.w << 16);
      xf[i][7] = __uint_as_float(v.w & 0xffff0000u);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float* wrow = wb + (size_t)(ee0 + j) * 256;
      const float4 wa = *reinterpret_cast<const float4*>(wrow + lane * 4);
      const float4 wc = *reinterpret_cast<const float4*>(wrow + 128 + lane * 4);
      const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wc.x, wc.y, wc.z, wc.w};
      // h-element outer, token inner: eight independent chains between two
      // dependent FMAs (each acc still takes its eight FMAs in h order)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][j] = fmaf(xf[i][q], wv[q], acc[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc[i][j] = acc[i][j] + __shfl_xor_sync(0xffffffffu, acc[i][j], o);
  if (lane == 0) {
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
  if (H % 256 != 0) return launch_router_logits(x, wr, bias, T, H, E, logits, s);
  const size_t smem = kRgStages * kRgStageBytes;
  cudaError_t err = cudaFuncSetAttribute(route_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((E + kRgE - 1) / kRgE, (T + kRgT - 1) / kRgT);
  return launch_ex(route_gemm_kernel, grid, dim3(kRgThreads), smem, s, false, static_cast<const uint16_t*>(x), wr, bias, T,
                   H, E, logits);
}

}  // namespace moe
