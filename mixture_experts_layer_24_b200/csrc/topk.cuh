// topk.cuh -- one warp's top-k of one token's router logits (the top-k
// kernels and the decode router's fused last-CTA top-k in route.cu).
//
// Top-k routing (vLLM-Moet, topairepos.com page: DeepSeek-V4.1 layers of 384
// routed experts, top-8 of the router's softmax, weights renormalised over the
// chosen experts). The experts are taken in the total order (logit
// descending, expert ascending): ties, +0 == -0 included, go to the lower
// index. A NaN logit (finite inputs never produce one) ranks below every
// number. Weights: expf(l_k - l_0), summed over k = 0..K-1 in order, one IEEE
// divide each.
#pragma once

#include "common.cuh"

namespace moe {

// Order-preserving key: a > b as logits (-0 == +0) iff key(a) > key(b); NaN -> 0,
// below every number (the smallest number, -inf, has key 0x007fffff).
__device__ __forceinline__ uint32_t logit_key(float v) {
  const uint32_t u = __float_as_uint(v + 0.0f);  // -0 + 0 = +0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return v == v ? k : 0u;  // selects, no branch on the loaded value
}
__device__ __forceinline__ float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Lane l holds the keys of experts l + 32 j (j < NJ) and ranks them once in
// the same order (key descending, j ascending: all comparisons independent).
// Each round takes the warp's largest head key (redux max), then the lowest
// expert holding it (redux min); the lane that gave it up moves its head to
// its next rank. A round is a short dependent chain, which matters here: one
// warp does this alone. Logits are read through L2 (ld.global.cg): another
// CTA or kernel wrote them. Lane k < K writes idx[k] and w[k].
template <int NJ>
__device__ __forceinline__ void topk_warp(const float* l, int E, int K, int32_t* idx, float* w) {
  const int lane = threadIdx.x & 31;
  // every load first (the index clamped, so none waits on a branch), then the keys
  float v[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) v[j] = __ldcg(l + min(lane + 32 * j, E - 1));
  uint32_t key[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) key[j] = lane + 32 * j < E ? logit_key(v[j]) : 0u;
  const int nv = lane < E ? min(NJ, (E - 1 - lane) / 32 + 1) : 0;  // slots holding an expert: j < nv
  int rank[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    int r = 0;
#pragma unroll
    for (int i = 0; i < NJ; ++i)
      if (i != j) r += (key[i] > key[j] || (key[i] == key[j] && i < j)) ? 1 : 0;
    rank[j] = r;  // empty slots (j >= nv, key 0, highest j) rank after every expert
  }
  int wins = 0;  // slots of this lane taken so far: its head has rank `wins`
  uint32_t hk = 0;
  int hj = 0;
  auto head = [&]() {
#pragma unroll
    for (int j = 0; j < NJ; ++j)
      if (rank[j] == wins) {
        hk = key[j];
        hj = j;
      }
  };
  head();
  float my_v = 0.0f;
  int my_e = 0;
  for (int r = 0; r < K; ++r) {
    const bool has = wins < nv;
    const uint32_t gk = __reduce_max_sync(0xffffffffu, has ? hk : 0u);
    const uint32_t ge = __reduce_min_sync(0xffffffffu, (has && hk == gk) ? (uint32_t)(lane + 32 * hj) : 0xffffffffu);
    if (lane == r) {
      my_v = key_logit(gk);
      my_e = (int)ge;
    }
    if ((int)(ge & 31u) == lane) {
      ++wins;
      head();
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

}  // namespace moe
