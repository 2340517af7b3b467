// ep.cu -- the data movement of expert parallelism: experts are split into G
// contiguous ranges, one per GPU; each pair goes to the GPU that holds its
// expert and its result comes back to the token's GPU. The collective between
// the steps (an all-to-all of rows) is the caller's (NCCL); these kernels only
// lay the rows out for it and take them back.
//
// The pages run their GPUs as tensor-parallel slices of each expert with an
// all-reduce ("NCCL 0.8-1.0 ms" of the step; vLLM-Moet, topairepos.com page,
// hybrid results table, row "the step"). A cross-GPU sum would change the
// order of a token's additions; moving whole pairs instead keeps every
// token's sum on its own GPU, in the same order, so the output bits do not
// depend on G.
//
//   pack:   x_send[p] = x[perm_src[p]], w_send[p] = w[perm_src[p], perm_k[p]]
//           for the valid sorted pairs p < offsets[E]. The sort is by expert,
//           so the rows for GPU g are the contiguous range of g's experts.
//   plan:   on an expert GPU, the received rows arrive grouped by source GPU
//           and, inside each source, by expert. The plan orders them by
//           (local expert, source, arrival): offsets per local expert,
//           perm (sorted place -> received row), inv (received row -> sorted
//           place), and a zero top-k slot per row (each row is one pair).
//   gather: y_back[i] = y_sorted[inv[i]]: the expert FFN's rows put back in
//           arrival order, ready to be sent home.
// Integer bookkeeping and copies only: bit-exact.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

// Copies one row of n 16-byte vectors with a warp, eight loads in flight per lane.
__device__ __forceinline__ void warp_copy_row(const uint4* __restrict__ src, uint4* __restrict__ dst, int n,
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

__global__ void __launch_bounds__(256) ep_pack_kernel(const uint4* __restrict__ x, const float* __restrict__ topk_w,
                                                       const int32_t* __restrict__ perm_src,
                                                       const int32_t* __restrict__ perm_k,
                                                       const int32_t* __restrict__ offsets, int E, int K, int P,
                                                       int vec_per_row, uint4* __restrict__ x_send,
                                                       float* __restrict__ w_send) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (p >= P || p >= offsets[E]) return;
  const int t = perm_src[p];
  if (lane == 0) w_send[p] = topk_w[(size_t)t * K + perm_k[p]];
  warp_copy_row(x + (size_t)t * vec_per_row, x_send + (size_t)p * vec_per_row, vec_per_row, lane);
}

// One CTA. recv_counts [G][E_loc] (row g: the rows source g sent for each
// local expert, in the order they arrive). G * E_loc <= 1024. Block (g, e) of
// the received buffer starts at the arrival-order scan of the counts; in the
// sorted order block (e, g) starts at the (expert, source)-order scan. Each
// sorted row q then finds its block by binary search over the sorted starts.
__global__ void __launch_bounds__(1024) ep_recv_plan_kernel(const int32_t* __restrict__ recv_counts, int G,
                                                             int E_loc, int32_t* __restrict__ offsets_loc,
                                                             int32_t* __restrict__ perm, int32_t* __restrict__ perm_k,
                                                             int32_t* __restrict__ inv) {
  __shared__ int sh[33];
  __shared__ int s_rbase[1024];   // arrival-order start of block b = g * E_loc + e
  __shared__ int s_sstart[1025];  // sorted-order start of sorted block k = e * G + g
  const int n = G * E_loc;
  const int i = threadIdx.x;
  int total;
  const int rbase = block_exclusive_scan_1024(i < n ? recv_counts[i] : 0, sh, &total);
  if (i < n) s_rbase[i] = rbase;
  const int e_s = i / G, g_s = i - (i / G) * G;  // sorted block k = i
  int total2;
  const int sbase = block_exclusive_scan_1024(i < n ? recv_counts[g_s * E_loc + e_s] : 0, sh, &total2);
  if (i < n) s_sstart[i] = sbase;
  if (i == 0) s_sstart[n] = total2;
  if (i < n && g_s == 0) offsets_loc[e_s] = sbase;
  if (i == 0) offsets_loc[E_loc] = total2;
  __syncthreads();
  for (int q = i; q < total2; q += blockDim.x) {
    int lo = 0, hi = n;  // largest k with s_sstart[k] <= q (empty blocks share a start: take the last)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_sstart[mid] <= q) lo = mid;
      else hi = mid;
    }
    const int e = lo / G, g = lo - (lo / G) * G;
    const int r = s_rbase[g * E_loc + e] + (q - s_sstart[lo]);
    perm[q] = r;
    perm_k[q] = 0;
    inv[r] = q;
  }
}

__global__ void __launch_bounds__(256) ep_gather_rows_f32_kernel(const uint4* __restrict__ src,
                                                                  const int32_t* __restrict__ idx, int n_rows,
                                                                  int vec_per_row, uint4* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= n_rows) return;
  warp_copy_row(src + (size_t)idx[r] * vec_per_row, dst + (size_t)r * vec_per_row, vec_per_row, lane);
}

}  // namespace

cudaError_t launch_ep_pack(const void* x, const float* topk_w, const int32_t* perm_src, const int32_t* perm_k,
                           const int32_t* offsets, int E, int K, int P, int H, void* x_send, float* w_send,
                           cudaStream_t s) {
  if (P <= 0) return cudaSuccess;
  ep_pack_kernel<<<(P + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(x), topk_w, perm_src, perm_k, offsets, E, K,
                                              P, H * 2 / 16, static_cast<uint4*>(x_send), w_send);
  return cudaGetLastError();
}

cudaError_t launch_ep_recv_plan(const int32_t* recv_counts, int G, int E_loc, int32_t* offsets_loc, int32_t* perm,
                                int32_t* perm_k, int32_t* inv, cudaStream_t s) {
  ep_recv_plan_kernel<<<1, 1024, 0, s>>>(recv_counts, G, E_loc, offsets_loc, perm, perm_k, inv);
  return cudaGetLastError();
}

cudaError_t launch_ep_gather_rows_f32(const float* src, const int32_t* idx, int n_rows, int H, float* dst,
                                      cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  ep_gather_rows_f32_kernel<<<(n_rows + 7) / 8, 256, 0, s>>>(reinterpret_cast<const uint4*>(src), idx, n_rows,
                                                             H * 4 / 16, reinterpret_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace moe
