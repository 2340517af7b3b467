// permute.cu -- token-to-expert permutation ("compact MoE calls": the pairs
// routed to one expert made contiguous; vLLM-Moet, topairepos.com page, hybrid
// results table, row "identity") as a deterministic counting sort by
// (expert asc, token asc), plus the FFN tile plan and the row gathers that
// feed the grouped GEMMs.
//
//   rank:    one warp per chunk of tokens; the warp walks its chunk in token
//            order, 32/K tokens per step, and gives each pair its rank among
//            the chunk's earlier pairs of the same expert (match_any for
//            pairs of one step, a per-warp shared counter across steps).
//   scan:    one CTA: per-expert exclusive scan over chunks, counts, and the
//            exclusive scan over experts (offsets).
//   scatter: p = offsets[e] + chunk_base[c][e] + rank.
// Integer arithmetic only: the result is bit-exact and run-to-run identical.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kRankWarps = 4;
constexpr int kMaxChunks = 64;

int permute_chunk_tokens(int T, int K) {
  const int tps = 32 / K;
  int c = (T + kMaxChunks - 1) / kMaxChunks;
  if (c < 32) c = 32;
  c = (c + tps - 1) / tps * tps;
  return c;
}

__global__ void __launch_bounds__(kRankWarps * 32) permute_rank_kernel(const int32_t* __restrict__ idx, int T,
                                                                        int K, int E, int chunk,
                                                                        int32_t* __restrict__ rank,
                                                                        int32_t* __restrict__ chunk_counts,
                                                                        int* status) {
  extern __shared__ int32_t cnt_all[];
  pdl_wait();
  pdl_trigger();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x * kRankWarps + w;
  const int n_chunks = (T + chunk - 1) / chunk;
  if (c >= n_chunks) return;  // warp-uniform
  int32_t* cnt = cnt_all + (size_t)w * E;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const int tps = 32 / K;
  const int tl = lane / K, k = lane - tl * K;
  const unsigned lt_mask = (1u << lane) - 1u;
  const int t_end = min(T, (c + 1) * chunk);
  for (int t0 = c * chunk; t0 < t_end; t0 += tps) {
    const int t = t0 + tl;
    const bool active = tl < tps && t < t_end;
    const int e = active ? idx[(size_t)t * K + k] : -1;
    const bool valid = active && e >= 0 && e < E;
    if (active && !valid) flag_status(status, MOE_DEV_BAD_EXPERT);
    const int key = valid ? e : E + lane;  // invalid lanes match nobody
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    int r = -1;
    if (valid) r = cnt[e] + __popc(peers & lt_mask);
    __syncwarp();
    if (valid && (peers >> lane) == 1u) cnt[e] += __popc(peers);  // highest peer lane updates
    __syncwarp();
    if (active) rank[(size_t)t * K + k] = r;
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) chunk_counts[(size_t)c * E + e] = cnt[e];
}

cudaError_t launch_permute_rank(const int32_t* idx, int T, int K, int E, int chunk, int32_t* rank,
                                int32_t* chunk_counts, int* status, cudaStream_t s, bool pdl) {
  if (T <= 0) return cudaSuccess;
  const int n_chunks = (T + chunk - 1) / chunk;
  const int blocks = (n_chunks + kRankWarps - 1) / kRankWarps;
  const size_t smem = sizeof(int32_t) * (size_t)E * kRankWarps;
  return launch_ex(permute_rank_kernel, dim3(blocks), dim3(kRankWarps * 32), smem, s, pdl, idx, T, K, E, chunk,
                   rank, chunk_counts, status);
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ chunk_counts, int n_chunks,
                                                             int E, int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ offsets) {
  __shared__ int sh[33];
  pdl_wait();
  pdl_trigger();
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
    // 16 independent loads in flight per round, then the running sum
    for (int c0 = 0; c0 < n_chunks; c0 += 16) {
      int v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = c0 + j < n_chunks ? chunk_counts[(size_t)(c0 + j) * E + e] : 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (c0 + j < n_chunks) chunk_counts[(size_t)(c0 + j) * E + e] = run;  // chunk's base within expert e
        run += v[j];
      }
    }
    counts[e] = run;
  }
  int total;
  const int off = block_exclusive_scan_1024(e < E ? run : 0, sh, &total);
  if (e < E) offsets[e] = off;
  if (e == 0) offsets[E] = total;
}

cudaError_t launch_permute_scan(int32_t* chunk_counts, int n_chunks, int E, int32_t* counts, int32_t* offsets,
                                cudaStream_t s, bool pdl) {
  return launch_ex(permute_scan_kernel, dim3(1), dim3(1024), 0, s, pdl, chunk_counts, n_chunks, E, counts, offsets);
}

__global__ void __launch_bounds__(256) permute_scatter_kernel(const int32_t* __restrict__ idx,
                                                               const int32_t* __restrict__ rank,
                                                               const int32_t* __restrict__ chunk_base,
                                                               const int32_t* __restrict__ offsets, int T, int K,
                                                               int E, int chunk, int32_t* __restrict__ perm_src,
                                                               int32_t* __restrict__ perm_k,
                                                               int32_t* __restrict__ inv) {
  pdl_wait();
  pdl_trigger();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)T * K) return;
  const int t = (int)(i / K), k = (int)(i - (int64_t)t * K);
  const int e = idx[i];
  const int r = rank[i];
  if (e < 0 || e >= E || r < 0) {
    inv[i] = -1;
    return;
  }
  const int c = t / chunk;
  const int p = offsets[e] + chunk_base[(size_t)c * E + e] + r;
  perm_src[p] = t;
  perm_k[p] = k;
  inv[i] = p;
}

cudaError_t launch_permute_scatter(const int32_t* idx, const int32_t* rank, const int32_t* chunk_base,
                                   const int32_t* offsets, int T, int K, int E, int chunk, int32_t* perm_src,
                                   int32_t* perm_k, int32_t* inv, cudaStream_t s, bool pdl) {
  const int64_t n = (int64_t)T * K;
  if (n <= 0) return cudaSuccess;
  return launch_ex(permute_scatter_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, pdl, idx, rank,
                   chunk_base, offsets, T, K, E, chunk, perm_src, perm_k, inv);
}

// --------------------------------------------------------------- FFN plan --
// List = every expert in index order; experts with pairs but no registered
// weights are flagged and given no tiles. Their pairs are dropped: their
// y_pair rows are written as zeros and, when inv is given (the forward), their
// inv entries become -1 so the combine leaves them out, as for a bad expert id.
__device__ void drop_pair_range(int p0, int p1, const int32_t* __restrict__ perm_src,
                                const int32_t* __restrict__ perm_k, int K, int32_t* __restrict__ inv,
                                float4* __restrict__ y_pair, int H4) {
  const int64_t n = (int64_t)(p1 - p0) * H4;
  for (int64_t q = threadIdx.x; q < n; q += blockDim.x)
    y_pair[(size_t)p0 * H4 + q] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (inv)
    for (int p = p0 + (int)threadIdx.x; p < p1; p += blockDim.x) inv[(size_t)perm_src[p] * K + perm_k[p]] = -1;
}

__global__ void __launch_bounds__(1024) ffn_plan_kernel(const int32_t* __restrict__ offsets,
                                                         const int32_t* __restrict__ map_of, int E, int bn,
                                                         int32_t* __restrict__ list_expert,
                                                         int32_t* __restrict__ list_map,
                                                         int32_t* __restrict__ nt_prefix, int* status,
                                                         int* __restrict__ sched, int sched_n, DropArgs drop, int bn2,
                                                         int32_t* __restrict__ nt_prefix2) {
  __shared__ int sh[33];
  __shared__ int s_missing;
  pdl_wait();
  pdl_trigger();
  const int e = threadIdx.x;
  if (e == 0) s_missing = 0;
  __syncthreads();
  for (int i = e; i < sched_n; i += blockDim.x) sched[i] = 0;  // counters of the fused decode FFN
  int nt = 0;
  if (e < E) {
    const int cnt = offsets[e + 1] - offsets[e];
    const int m = map_of[e];
    nt = (cnt + bn - 1) / bn;
    if (cnt > 0 && m < 0) {
      flag_status(status, MOE_DEV_NO_SLOT);
      s_missing = 1;
      nt = 0;
    }
    list_expert[e] = e;
    list_map[e] = m < 0 ? 0 : m;
  }
  int total;
  const int pre = block_exclusive_scan_1024(nt, sh, &total);  // its barriers also publish s_missing
  if (e < E) nt_prefix[e] = pre;
  if (e == 0) nt_prefix[E] = total;
  if (nt_prefix2) {  // block-uniform
    const int nt2 = (e < E && nt > 0) ? (offsets[e + 1] - offsets[e] + bn2 - 1) / bn2 : 0;
    int total2;
    const int pre2 = block_exclusive_scan_1024(nt2, sh, &total2);
    if (e < E) nt_prefix2[e] = pre2;
    if (e == 0) nt_prefix2[E] = total2;
  }
  if (!s_missing || !drop.y_pair) return;  // block-uniform
  for (int x = 0; x < E; ++x) {
    const int p0 = offsets[x], p1 = offsets[x + 1];
    if (p1 > p0 && map_of[x] < 0)
      drop_pair_range(p0, p1, drop.perm_src, drop.perm_k, drop.K, drop.inv, reinterpret_cast<float4*>(drop.y_pair),
                      drop.H / 4);
  }
}

cudaError_t launch_ffn_plan(const int32_t* offsets, const int32_t* map_of, int E, int bn, int32_t* list_expert,
                            int32_t* list_map, int32_t* nt_prefix, int* status, cudaStream_t s, bool pdl, int* sched,
                            int sched_n, const DropArgs& drop, int bn2, int32_t* nt_prefix2) {
  return launch_ex(ffn_plan_kernel, dim3(1), dim3(1024), 0, s, pdl, offsets, map_of, E, bn, list_expert, list_map,
                   nt_prefix, status, sched, sched ? sched_n : 0, drop, bn2, nt_prefix2);
}

// Pairs [p0, p1) of one unregistered expert on the host-synchronised path:
// dropped as above.
__global__ void __launch_bounds__(1024) drop_pairs_kernel(int p0, int p1, DropArgs drop) {
  drop_pair_range(p0, p1, drop.perm_src, drop.perm_k, drop.K, drop.inv, reinterpret_cast<float4*>(drop.y_pair),
                  drop.H / 4);
}

cudaError_t launch_drop_pairs(int p0, int p1, const DropArgs& drop, cudaStream_t s) {
  if (p1 <= p0) return cudaSuccess;
  drop_pairs_kernel<<<1, 1024, 0, s>>>(p0, p1, drop);
  return cudaGetLastError();
}

// ----------------------------------------------------------------- gather --
// x_perm[p, :] = x[perm_src[p], :] for the offsets[E] valid pairs; one warp per
// row, 16-byte vectors.
// Copies one row of n 16-byte vectors with a warp, eight loads in flight per
// lane before the stores.
__device__ __forceinline__ void copy_row_warp(const uint4* __restrict__ src, uint4* __restrict__ dst, int n,
                                              int lane) {
  for (int v0 = lane; v0 < n; v0 += 32 * 8) {
    uint4 tmp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (v0 + 32 * u < n) tmp[u] = __ldg(src + v0 + 32 * u);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (v0 + 32 * u < n) dst[v0 + 32 * u] = tmp[u];
  }
}

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                           const int32_t* __restrict__ perm_src,
                                                           const int32_t* __restrict__ offsets, int E, int P,
                                                           int vec_per_row, uint4* __restrict__ xp) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= P || p >= offsets[E]) return;
  const int t = perm_src[p];
  copy_row_warp(x + (size_t)t * vec_per_row, xp + (size_t)p * vec_per_row, vec_per_row, lane);
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E, int P,
                               int H, void* x_perm, cudaStream_t s, bool pdl) {
  if (P <= 0) return cudaSuccess;
  return launch_ex(gather_rows_kernel, dim3((P + 7) / 8), dim3(256), 0, s, pdl, static_cast<const uint4*>(x),
                   perm_src, offsets, E, P, H * 2 / 16, static_cast<uint4*>(x_perm));
}

// ------------------------------------------------------ small batches --
// Whole permutation of T*K <= 1024 pairs in one launch: every CTA builds it in
// shared memory (a counting sort: order-free counts, one block scan, then each
// pair's rank among earlier pairs of its expert), CTA 0 writes counts,
// offsets, the sorted pairs and (optionally) the FFN tile plan, and all CTAs
// copy their share of the sorted x rows. Same result as rank/scan/scatter.
__global__ void __launch_bounds__(1024) permute_small_kernel(
    const int32_t* __restrict__ idx, int T, int K, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_src, int32_t* __restrict__ perm_k,
    int32_t* __restrict__ inv, const int32_t* __restrict__ map_of, int bn, int32_t* __restrict__ list_expert,
    int32_t* __restrict__ list_map, int32_t* __restrict__ nt_prefix, const uint4* __restrict__ x, int vec_per_row,
    uint4* __restrict__ x_perm, int* status, int* __restrict__ sched, int sched_n, int bn2,
    int32_t* __restrict__ nt_prefix2) {
  __shared__ __align__(16) int s_e[kPermuteSmallMaxPairs];
  __shared__ int s_cnt[1024];
  __shared__ int s_off[1024];
  __shared__ int s_src[kPermuteSmallMaxPairs];
  __shared__ int sh[33];
  pdl_wait();
  pdl_trigger();
  const int P = T * K;
  const int i = threadIdx.x;
  int e = -1;
  if (i < P) {
    e = idx[i];
    if (e < 0 || e >= E) {
      if (blockIdx.x == 0) flag_status(status, MOE_DEV_BAD_EXPERT);
      e = -1;
    }
  }
  s_e[i] = e;
  s_cnt[i] = 0;
  __syncthreads();
  if (e >= 0) atomicAdd(&s_cnt[e], 1);
  __syncthreads();
  const int cnt = i < E ? s_cnt[i] : 0;
  int total;
  const int off = block_exclusive_scan_1024(cnt, sh, &total);
  s_off[i] = off;
  __syncthreads();
  int p = -1;
  if (e >= 0) {
    int r = 0;
    const int4* e4 = reinterpret_cast<const int4*>(s_e);
    const int n4 = i >> 2;
    for (int j = 0; j < n4; ++j) {
      const int4 v = e4[j];
      r += (v.x == e) + (v.y == e) + (v.z == e) + (v.w == e);
    }
    for (int j = n4 << 2; j < i; ++j) r += s_e[j] == e;
    p = s_off[e] + r;
    s_src[p] = i;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    if (i < E) {
      counts[i] = cnt;
      offsets[i] = off;
    }
    if (i == 0) offsets[E] = total;
    if (i < P) {
      // with a plan (the forward), a pair of an unregistered expert is dropped: the combine skips inv = -1
      inv[i] = (map_of && e >= 0 && map_of[e] < 0) ? -1 : p;
      if (p >= 0) {
        perm_src[p] = i / K;
        perm_k[p] = i - (i / K) * K;
      }
    }
    for (int j = i; j < sched_n; j += blockDim.x) sched[j] = 0;  // counters of the fused decode FFN
    if (map_of) {
      int nt = 0;
      if (i < E) {
        const int m = map_of[i];
        nt = (cnt + bn - 1) / bn;
        if (cnt > 0 && m < 0) {
          flag_status(status, MOE_DEV_NO_SLOT);
          nt = 0;
        }
        list_expert[i] = i;
        list_map[i] = m < 0 ? 0 : m;
      }
      int nt_total;
      const int pre = block_exclusive_scan_1024(nt, sh, &nt_total);
      if (i < E) nt_prefix[i] = pre;
      if (i == 0) nt_prefix[E] = nt_total;
      if (nt_prefix2) {  // N tiles of the wider down GEMM (block-uniform)
        const int nt2 = nt > 0 ? (cnt + bn2 - 1) / bn2 : 0;
        int nt2_total;
        const int pre2 = block_exclusive_scan_1024(nt2, sh, &nt2_total);
        if (i < E) nt_prefix2[i] = pre2;
        if (i == 0) nt_prefix2[E] = nt2_total;
      }
    }
  }
  if (x_perm) {
    const int warp = i >> 5, lane = i & 31, nw = blockDim.x >> 5;
    for (int row = blockIdx.x * nw + warp; row < total; row += gridDim.x * nw) {
      const int t = s_src[row] / K;
      copy_row_warp(x + (size_t)t * vec_per_row, x_perm + (size_t)row * vec_per_row, vec_per_row, lane);
    }
  }
}

cudaError_t launch_permute_small(const int32_t* idx, int T, int K, int E, int32_t* counts, int32_t* offsets,
                                 int32_t* perm_src, int32_t* perm_k, int32_t* inv, const int32_t* map_of, int bn,
                                 int32_t* list_expert, int32_t* list_map, int32_t* nt_prefix, const void* x, int H,
                                 void* x_perm, int* status, cudaStream_t s, bool pdl, int* sched,
                                 int sched_n, int bn2, int32_t* nt_prefix2) {
  const int P = T * K;
  int ctas = 1;
  if (x_perm) ctas = std::max(1, std::min(64, (P + 31) / 32));
  return launch_ex(permute_small_kernel, dim3(ctas), dim3(1024), 0, s, pdl, idx, T, K, E, counts, offsets, perm_src,
                   perm_k, inv, map_of, bn, list_expert, list_map, nt_prefix, static_cast<const uint4*>(x), H / 8,
                   static_cast<uint4*>(x_perm), status, sched, sched ? sched_n : 0, bn2, nt_prefix2);
}

}  // namespace moe
