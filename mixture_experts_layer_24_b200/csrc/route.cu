// route.cu -- router logits and top-k selection.
//
// Router of a routed MoE layer (vLLM-Moet, topairepos.com page: DeepSeek-V4.1
// layers of 384 routed experts, top-k routing; "identical requests return
// identical logits at any batch size" is the results-table "quality" row).
//
// Logit order (the contract both these kernels and the CPU oracle follow):
// lane j of a warp runs fmaf(x[h], Wr[e][h], acc) from +0 over h = j, j+32,
// j+64, ... in increasing h; the 32 lane partials are then summed by the xor
// butterfly (offsets 16, 8, 4, 2, 1), which leaves p[j] += p[j+o]
// (o = 16 .. 1) in lane 0; then one fp32 add of bias[e]. A warp's loads of
// one h step are 32 consecutive elements, and a token's logits depend on that
// token alone, whatever the batch.
#include "common.cuh"
#include "internal.h"
#include "residency.cuh"
#include "topk.cuh"

namespace moe {

__device__ __forceinline__ float bf16_lo(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Two fp32 values in one 64-bit register, and the paired fused multiply-add
// (two independent IEEE fmaf with round-to-nearest, one instruction).
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ void fma2(uint64_t& c, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(c) : "l"(a), "l"(b));
}

__device__ __forceinline__ void butterfly_sum(float& v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = v + __shfl_xor_sync(0xffffffffu, v, o);
}

// ------------------------------------------------ direct (global) router --
// One warp per expert, TG tokens per warp, operands straight from global
// memory: per h step a warp reads 128 contiguous bytes of Wr and 64 of each x
// row. U steps are loaded before any is used.
template <int TG, int U>
__device__ __forceinline__ void logits_warp_direct(const uint16_t* __restrict__ x, const float* __restrict__ wrow,
                                                   int T, int H, int t0, float (&acc)[TG]) {
  const int lane = threadIdx.x & 31;
  const int ntok = min(TG, T - t0);
#pragma unroll
  for (int i = 0; i < TG; ++i) acc[i] = 0.0f;
  for (int hb = lane; hb < H; hb += 32 * U) {
    float w[U];
    uint32_t xv[U][TG];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int h = hb + 32 * u;
      if (h < H) {
        w[u] = __ldg(wrow + h);
#pragma unroll
        for (int i = 0; i < TG; ++i)
          if (i < ntok) xv[u][i] = __ldg(x + (size_t)(t0 + i) * H + h);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (hb + 32 * u < H) {
#pragma unroll
        for (int i = 0; i < TG; ++i)
          if (i < ntok) acc[i] = fmaf(bf16_lo(xv[u][i]), w[u], acc[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TG; ++i) butterfly_sum(acc[i]);
}

template <int TG>
struct DirectUnroll {
  static constexpr int value = TG == 1 ? 32 : (TG <= 2 ? 16 : (TG <= 4 ? 8 : 4));
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
  logits_warp_direct<TG, DirectUnroll<TG>::value>(x, wr + (size_t)e * H, T, H, t0, acc);
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
// One warp per token (topk.cuh: redux arg-max over order-preserving keys).
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

// --------------------------------------------- register-tiled router GEMM --
// fp32 GEMM in the same order. A warp owns WT tokens x WE experts; NWT x NWE
// warps make the CTA tile (TT = WT*NWT tokens, TE = WE*NWE experts). Each
// stage holds 256 consecutive h of the tile's tokens and experts in shared
// memory as stored (cp.async, kRgStages buffers, kRgStages - 1 in flight).
// Each thread copies the same 16-byte parts of the same rows in every stage,
// so their offsets are computed once.
//
// Lane (half, i) = (lane / 16, lane % 16) runs the two order chains 2i and
// 2i+1 of the tokens 2m + half (m = 0 .. WT/2-1) against all WE experts: one
// 32-bit load brings x[h], x[h+1] (h = h0 + 32q + 2i) of a token, one 64-bit
// load the matching pair of Wr[e], and one paired FMA advances both chains.
// The chains keep the order above (chain c runs h = c, c+32, ... in
// increasing h); at the end the 32 chains of each output meet in shared
// memory and one lane sums them by the xor butterfly's pairwise tree. Token
// rows are staged 576 bytes apart, so the two halves' rows (even and odd
// tokens) fall in different banks.
//   prefill:          WT = 8, WE = 8, 4 x 2 warps (32 tokens x 16 experts; two
//                     CTAs per SM: each hides the other's stage barriers)
//   16 < T <= 64:     WT = 4, WE = 8, 2 x 2 warps (8 x 16)
//   8 < T <= 16:      WT = 4, WE = 4, 2 x 2 warps (8 x 8)
constexpr int kRgStages = 3;
constexpr int kRgXPitch = 256 * 2 + 64;  // bytes per staged token row

template <int WT, int WE, int NWT, int NWE>
struct RgCfg {
  static constexpr int TT = WT * NWT, TE = WE * NWE, kThreads = 32 * NWT * NWE;
  static constexpr size_t kXBytes = (size_t)TT * kRgXPitch;
  static constexpr size_t kStageBytes = kXBytes + (size_t)TE * 256 * 4;
  static constexpr size_t kSmem = kRgStages * kStageBytes;
  static constexpr int kXCopies = TT * 32 / kThreads, kWCopies = TE * 64 / kThreads;  // 16-byte parts per thread
  static_assert(TT * 32 % kThreads == 0 && TE * 64 % kThreads == 0, "whole parts per thread");
  static_assert(kXBytes % 16 == 0, "Wr tile stays 16-byte aligned");
};

template <int WT, int WE, int NWT, int NWE>
__global__ void __launch_bounds__(32 * NWT * NWE, 2) route_gemm_kernel(const uint16_t* __restrict__ x,
                                                                        const float* __restrict__ wr,
                                                                        const float* __restrict__ bias, int T, int H,
                                                                        int E, float* __restrict__ logits,
                                                                        int* __restrict__ sched, int sched_n) {
  using C = RgCfg<WT, WE, NWT, NWE>;
  constexpr int TT = C::TT, TE = C::TE, NT = C::kThreads;
  static_assert(WT % 2 == 0, "each half-warp takes half of a warp's tokens");
  extern __shared__ __align__(16) uint8_t sm[];
  pdl_wait();  // x may come from the previous kernel
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = lane >> 4, li = lane & 15;
  if (blockIdx.x == 0 && blockIdx.y == 0)  // counters of the decode FFN that follows (first kernel of the forward)
    for (int i = tid; i < sched_n; i += NT) sched[i] = 0;
  const int tt0 = (warp / NWE) * WT, ee0 = (warp % NWE) * WE;
  const int tb = blockIdx.y * TT, eb = blockIdx.x * TE;
  const int nsteps = H / 256;
  // this thread's parts: token row tid/32 + k*NT/32, part tid%32 (8 bf16);
  // expert row tid/64 + k*NT/64, part tid%64 (4 fp32). Rows past T or E
  // re-read the last row (results discarded). Offsets in elements (< 2^29).
  uint32_t xoff[C::kXCopies], woff[C::kWCopies];
#pragma unroll
  for (int k = 0; k < C::kXCopies; ++k)
    xoff[k] = (uint32_t)min(tb + (tid >> 5) + k * (NT / 32), T - 1) * (uint32_t)H + (uint32_t)(tid & 31) * 8u;
#pragma unroll
  for (int k = 0; k < C::kWCopies; ++k)
    woff[k] = (uint32_t)min(eb + (tid >> 6) + k * (NT / 64), E - 1) * (uint32_t)H + (uint32_t)(tid & 63) * 4u;
  const uint32_t xdst0 = (uint32_t)((tid >> 5) * kRgXPitch + (tid & 31) * 16);
  const uint32_t wdst0 = (uint32_t)(C::kXBytes + (tid >> 6) * 1024 + (tid & 63) * 16);
  const uint32_t sbase = smem_u32(sm);
  auto load_stage = [&](int st, int buf) {
    const uint16_t* xs0 = x + (size_t)st * 256;
    const float* ws0 = wr + (size_t)st * 256;
    const uint32_t d = sbase + (uint32_t)(buf * C::kStageBytes);
#pragma unroll
    for (int k = 0; k < C::kXCopies; ++k)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + xdst0 + k * (NT / 32) * kRgXPitch),
                   "l"(xs0 + xoff[k])
                   : "memory");
#pragma unroll
    for (int k = 0; k < C::kWCopies; ++k)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d + wdst0 + k * (NT / 64) * 1024),
                   "l"(ws0 + woff[k])
                   : "memory");
  };

  uint64_t acc2[WT / 2][WE];  // (chain 2i, chain 2i+1) of token tt0 + 2m + half, expert ee0 + j
#pragma unroll
  for (int m = 0; m < WT / 2; ++m)
#pragma unroll
    for (int j = 0; j < WE; ++j) acc2[m][j] = 0ull;

#pragma unroll
  for (int st = 0; st < kRgStages - 1; ++st) {
    if (st < nsteps) load_stage(st, st);
    asm volatile("cp.async.commit_group;" ::: "memory");  // empty groups keep the count uniform
  }
  int buf = 0;
  for (int st = 0; st < nsteps; ++st) {
    {
      const int nx = st + kRgStages - 1;  // its buffer was last read in iteration st - 1
      int nbuf = buf + kRgStages - 1;
      if (nbuf >= kRgStages) nbuf -= kRgStages;
      if (nx < nsteps) load_stage(nx, nbuf);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.wait_group %0;" ::"n"(kRgStages - 1) : "memory");
    __syncthreads();
    const uint8_t* xb = sm + buf * C::kStageBytes + (size_t)(tt0 + half) * kRgXPitch + 4 * li;
    const float* wb = reinterpret_cast<const float*>(sm + buf * C::kStageBytes + C::kXBytes) + (size_t)ee0 * 256 + 2 * li;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint64_t xp[WT / 2];
#pragma unroll
      for (int m = 0; m < WT / 2; ++m) {
        const uint32_t v = *reinterpret_cast<const uint32_t*>(xb + (size_t)(2 * m) * kRgXPitch + 64 * q);
        xp[m] = ((uint64_t)(v & 0xffff0000u) << 32) | (uint64_t)(v << 16);  // fp32 of bf16 x[h] (low), x[h+1]
      }
#pragma unroll
      for (int j = 0; j < WE; ++j) {
        const uint64_t wp = *reinterpret_cast<const uint64_t*>(wb + (size_t)j * 256 + 32 * q);
#pragma unroll
        for (int m = 0; m < WT / 2; ++m) fma2(acc2[m][j], xp[m], wp);
      }
    }
    __syncthreads();
    if (++buf == kRgStages) buf = 0;
  }
  // The 32 chain partials of each of the warp's WT x WE outputs go through shared memory (the stage buffers are
  // free: every copy has landed and the last barrier has passed): row (token i, expert j) holds chain c at
  // 16-byte chunk (c / 4) ^ (row % 8), so a lane's 16-byte reads of its own row and the other lanes' rows fall
  // in different banks. Lane l then sums rows l, l + 32, ... by the xor butterfly's tree in registers: offsets
  // 16, 8, 4, 2, 1, each partial added to its partner, as the shuffles would.
  static_assert((size_t)NWT * NWE * WT * WE * 32 * 4 <= C::kSmem, "the partials fit the stage buffers");
  float* red = reinterpret_cast<float*>(sm) + (size_t)warp * WT * WE * 32;
#pragma unroll
  for (int m = 0; m < WT / 2; ++m)
#pragma unroll
    for (int j = 0; j < WE; ++j) {
      const int row = (2 * m + half) * WE + j;
      const int chunk = (li >> 1) ^ (row & 7);  // chains 2li, 2li+1 sit in chunk li / 2, at (2li) % 4
      float lo, hi;
      unpack2(acc2[m][j], lo, hi);
      *reinterpret_cast<float2*>(red + row * 32 + chunk * 4 + ((2 * li) & 3)) = make_float2(lo, hi);
    }
  __syncwarp();
#pragma unroll
  for (int rr = 0; rr < (WT * WE + 31) / 32; ++rr) {
    const int row = lane + 32 * rr;
    if (row >= WT * WE) break;
    float c[32];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 v = *reinterpret_cast<const float4*>(red + row * 32 + (k ^ (row & 7)) * 4);
      c[4 * k] = v.x;
      c[4 * k + 1] = v.y;
      c[4 * k + 2] = v.z;
      c[4 * k + 3] = v.w;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
      for (int q = 0; q < o; ++q) c[q] = c[q] + c[q + o];
    const int t = tb + tt0 + row / WE, e = eb + ee0 + row % WE;
    if (t < T && e < E) logits[(size_t)t * E + e] = bias ? c[0] + bias[e] : c[0];
  }
}

template <int WT, int WE, int NWT, int NWE>
static cudaError_t launch_rg(const void* x, const float* wr, const float* bias, int T, int H, int E, float* logits,
                             cudaStream_t s, bool pdl, int* sched = nullptr, int sched_n = 0) {
  using C = RgCfg<WT, WE, NWT, NWE>;
  auto kern = route_gemm_kernel<WT, WE, NWT, NWE>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (err != cudaSuccess) return err;
  dim3 grid((E + C::TE - 1) / C::TE, (T + C::TT - 1) / C::TT);
  return launch_ex(kern, grid, dim3(C::kThreads), C::kSmem, s, pdl, static_cast<const uint16_t*>(x), wr, bias, T, H,
                   E, logits, sched, sched ? sched_n : 0);
}

static bool rg_tile_ok(const void* x, const float* wr, int H) {
  return ((uintptr_t)x % 16 == 0) && ((uintptr_t)wr % 16 == 0) && (H % 256 == 0);
}

cudaError_t launch_route_gemm(const void* x, const float* wr, const float* bias, int T, int H, int E,
                              float* logits, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  if (!rg_tile_ok(x, wr, H)) return launch_router_logits(x, wr, bias, T, H, E, logits, s);
  return launch_rg<8, 8, 4, 2>(x, wr, bias, T, H, E, logits, s, false);
}

// ------------------------------------------------- decode-regime router --
// WPC warps per CTA, one expert each, TG tokens per CTA. The CTA's x rows and
// its warps' Wr rows arrive in shared memory by bulk copies (one per row, all
// in flight together: a single DRAM round trip), then each lane reads its h
// steps from there (consecutive lanes, consecutive words: no bank conflict).
// With fuse_topk, the last CTA of each token group (an arrival counter) picks
// the group's top-k, one warp per token, and returns the counter to zero;
// otherwise a top-k kernel follows.
constexpr int kRsWarps = 4;

__host__ __device__ constexpr size_t route_small_smem(int tg, int H) {
  return 16 + (size_t)kRsWarps * H * 4 + (size_t)tg * H * 2;
}

template <int TG>
__global__ void __launch_bounds__(kRsWarps * 32) route_small_kernel(const uint16_t* __restrict__ x,
                                                                     const float* __restrict__ wr,
                                                                     const float* __restrict__ bias, int T, int H,
                                                                     int E, int K, float* __restrict__ logits,
                                                                     int32_t* __restrict__ idx, float* __restrict__ w,
                                                                     unsigned int* __restrict__ counters,
                                                                     int fuse_topk, int* status,
                                                                     int* __restrict__ sched, int sched_n,
                                                                     ResidencyDev rd, int32_t* map_of, int res_plan) {
  extern __shared__ __align__(16) uint8_t sm[];
  __shared__ int s_last;
  __shared__ ResidencyPlanSmem s_plan;
  pdl_trigger();  // first kernel of a forward: the next one may launch (it waits for us)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && blockIdx.y == 0)  // counters of the decode FFN that follows
    for (int i = threadIdx.x; i < sched_n; i += blockDim.x) sched[i] = 0;
  const int e0 = blockIdx.x * kRsWarps, e = e0 + warp;
  const int t0 = blockIdx.y * TG;
  const int ntok = min(TG, T - t0), nexp = min(kRsWarps, E - e0);
  const uint32_t bar = smem_u32(sm);
  float* ws = reinterpret_cast<float*>(sm + 16);                              // [kRsWarps][H]
  const uint16_t* xs = reinterpret_cast<const uint16_t*>(sm + 16 + (size_t)kRsWarps * H * 4);  // [TG][H]
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, (uint32_t)(nexp * H * 4 + ntok * H * 2));
    for (int i = 0; i < nexp; ++i)
      bulk_load(smem_u32(ws + (size_t)i * H), wr + (size_t)(e0 + i) * H, (uint32_t)H * 4, bar);
    for (int i = 0; i < ntok; ++i)
      bulk_load(smem_u32(xs + (size_t)i * H), x + (size_t)(t0 + i) * H, (uint32_t)H * 2, bar);
  }
  __syncthreads();
  bool ok = mbar_wait(bar, 0);
  ok = __syncthreads_and(ok);
  if (!ok && threadIdx.x == 0) {
    // the copies did not land in time: flag it. They write this CTA's shared
    // memory, so they must land before the CTA exits: keep waiting, in bounded
    // rounds of the same limit (a few more at most). The CTA then skips its
    // logits but still takes part in the top-k arrival count, which must
    // return to zero.
    flag_status(status, MOE_DEV_TIMEOUT);
    for (int round = 0; round < 4 && !mbar_wait(bar, 0); ++round) {
    }
  }
  if (ok && e < E) {
    const float* wrow = ws + (size_t)warp * H;
    float acc[TG];
#pragma unroll
    for (int i = 0; i < TG; ++i) acc[i] = 0.0f;
#pragma unroll 4
    for (int h = lane; h < H; h += 32) {
      const float wv = wrow[h];
#pragma unroll
      for (int i = 0; i < TG; ++i)
        if (i < ntok) acc[i] = fmaf(bf16_lo(xs[(size_t)i * H + h]), wv, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < TG; ++i) butterfly_sum(acc[i]);
    if (lane == 0) {
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
  for (int i = warp; i < ntok; i += kRsWarps) {
    const int t = t0 + i;
    topk_warp_any(logits + (size_t)t * E, E, K, idx + (size_t)t * K, w + (size_t)t * K);
  }
  if (res_plan) {
    // one CTA holds every token (T <= TG): the LRU plan of the spare slots follows the top-k here instead of
    // in a launch of its own
    __syncthreads();
    residency_plan_block(idx, T * K, E, rd, map_of, s_plan);
  }
  if (threadIdx.x == 0) counters[blockIdx.y] = 0u;
}

template <int TG>
static cudaError_t launch_rs(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                             float* logits, int32_t* idx, float* w, unsigned int* counters, int fuse, int* status,
                             cudaStream_t s, int* sched, int sched_n, const ResidencyDev* rd = nullptr,
                             int32_t* map_of = nullptr) {
  const size_t smem = route_small_smem(TG, H);
  cudaError_t err = cudaFuncSetAttribute(route_small_kernel<TG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  dim3 grid((E + kRsWarps - 1) / kRsWarps, (T + TG - 1) / TG);
  return launch_ex(route_small_kernel<TG>, grid, dim3(kRsWarps * 32), smem, s, false,
                   static_cast<const uint16_t*>(x), wr, bias, T, H, E, K, logits, idx, w, counters, fuse, status,
                   sched, sched ? sched_n : 0, rd ? *rd : ResidencyDev{}, map_of, rd ? 1 : 0);
}

// T <= 4: logits + fused top-k in one launch; up to 64 tokens: logits, then
// the warp top-k kernel (programmatic launch), which measured faster from 8
// tokens on (the fused top-k runs in the last CTA's four warps, two tokens
// each at T = 8: 299.0 vs 293.5 us per layer) and slower below (by 0.7-1.9
// us). The fused form was also slower for the register-tiled kernel at 16 and
// 64 tokens. Rows that a bulk copy cannot take (not 16-byte aligned, or too
// large for shared memory) go through the direct kernel.
cudaError_t launch_route_small(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                               float* logits, int32_t* idx, float* w, unsigned int* counters, int* status,
                               cudaStream_t s, bool pdl, int* sched, int sched_n, const ResidencyDev* rd,
                               int32_t* map_of, bool* planned) {
  if (planned) *planned = false;
  if (T <= 0) return cudaSuccess;
  const bool bulk_ok = ((uintptr_t)x % 16 == 0) && ((uintptr_t)wr % 16 == 0) && (H % 8 == 0) &&
                       route_small_smem(8, H) <= 200 * 1024;
  if (!bulk_ok) {
    if (sched) cudaMemsetAsync(sched, 0, sizeof(int) * sched_n, s);
    cudaError_t err = launch_router_logits(x, wr, bias, T, H, E, logits, s);
    if (err != cudaSuccess) return err;
    return launch_topk_warp(logits, T, E, K, idx, w, s, false);
  }
  // the fused last CTA runs the residency plan when the caller asks for it (and learns it through *planned)
  const ResidencyDev* rdp = (T <= 4 && planned) ? rd : nullptr;
  if (rdp) *planned = true;
  if (T <= 1)
    return launch_rs<1>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, status, s, sched, sched_n, rdp, map_of);
  if (T <= 2)
    return launch_rs<2>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, status, s, sched, sched_n, rdp, map_of);
  if (T <= 4)
    return launch_rs<4>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 1, status, s, sched, sched_n, rdp, map_of);
  if (T <= 8) {
    const cudaError_t err = launch_rs<8>(x, wr, bias, T, H, E, K, logits, idx, w, counters, 0, status, s, sched,
                                         sched_n);
    if (err != cudaSuccess) return err;
    return launch_topk_warp(logits, T, E, K, idx, w, s, pdl);
  }
  // more tokens: W rows would be staged once per 8-token group; register
  // tiles reuse each loaded element across 4 tokens and 4 or 8 experts
  cudaError_t err;
  if (!rg_tile_ok(x, wr, H)) {
    if (sched) cudaMemsetAsync(sched, 0, sizeof(int) * sched_n, s);
    err = launch_router_logits(x, wr, bias, T, H, E, logits, s);
  } else if (T <= 16) {
    err = launch_rg<4, 4, 2, 2>(x, wr, bias, T, H, E, logits, s, false, sched, sched_n);
  } else {
    err = launch_rg<4, 8, 2, 2>(x, wr, bias, T, H, E, logits, s, false, sched, sched_n);
  }
  if (err != cudaSuccess) return err;
  return launch_topk_warp(logits, T, E, K, idx, w, s, pdl);
}

}  // namespace moe
