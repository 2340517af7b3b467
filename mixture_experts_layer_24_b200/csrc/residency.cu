// residency.cu -- host-resident experts without a host round trip.
//
// The "hotsplit" recipes wiki (Home page) keeps the hot experts on the GPU and
// reads the cold ones from pinned host memory on demand; the vLLM-Moet page's
// cache variant (hybrid results, "hit rate 0.88 vs 0.87") keeps the most
// recently used ones. Here the spare HBM slots are an LRU cache of the
// host-resident experts, and for a decode batch whose pairs can route to no
// more host experts than there are slots, the whole bookkeeping runs on the
// device, in the forward's launch chain:
//
//   plan (one CTA): the experts the top-k routes to; a host expert already in
//     a slot is a hit (its slot's tick is refreshed); each miss, in expert
//     order, takes the least recently used slot this call does not need (ties
//     to the lowest slot), the evicted expert loses its slot, and the expert
//     -> map-entry table the FFN reads points the new one at its slot; the
//     misses are listed for the copy.
//   copy (grid): the listed experts' records are read from pinned host memory
//     (mapped into the device's address space) over PCIe and written to their
//     slots; with nothing listed the kernel returns at once.
//
// The FFN kernel then computes cached experts from their slots with the same
// tiles and K order as resident ones, so the outputs are bit-identical to the
// all-resident run (vLLM-Moet, hybrid results table, row "identity"). No
// stream synchronisation, so the forward can be captured in a CUDA graph.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

__global__ void __launch_bounds__(1024) residency_plan_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                               ResidencyDev rd, int32_t* __restrict__ map_of) {
  __shared__ uint8_t s_touched[1024];
  __shared__ int s_miss[1024];
  __shared__ int s_nmiss;
  __shared__ long long s_tick;
  pdl_wait();  // the top-k comes from the router
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) s_touched[e] = 0;
  __syncthreads();
  for (int i = tid; i < P; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) s_touched[e] = 1;
  }
  __syncthreads();
  if (tid >= 32) return;
  // one warp from here: hits first, misses listed in expert order
  if (lane == 0) {
    s_tick = *rd.tick + 1;
    *rd.tick = s_tick;
    s_nmiss = 0;
  }
  __syncwarp();
  const long long tick = s_tick;
  int touched = 0, routed = 0, hits = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const bool t = e < E && s_touched[e];
    const bool host = t && rd.loc[e] == MOE_LOC_HOST_PINNED;
    const int slot = host ? rd.expert_slot[e] : -1;
    if (host && slot >= 0) rd.slot_tick[slot] = tick;
    const unsigned miss = __ballot_sync(0xffffffffu, host && slot < 0);
    if (host && slot < 0) s_miss[s_nmiss + __popc(miss & ((1u << lane) - 1u))] = e;
    touched += __popc(__ballot_sync(0xffffffffu, t));
    routed += __popc(__ballot_sync(0xffffffffu, host));
    hits += __popc(__ballot_sync(0xffffffffu, host && slot >= 0));
    __syncwarp();
    if (lane == 0) s_nmiss += __popc(miss);
    __syncwarp();
  }
  const int nmiss = s_nmiss;
  for (int m = 0; m < nmiss; ++m) {
    // least recently used slot that this call does not need; ties to the lowest slot index
    long long best_t = 0x7fffffffffffffffll;
    int best_s = 0x7fffffff;
    for (int sidx = lane; sidx < rd.n_spare; sidx += 32) {
      const long long st = rd.slot_tick[sidx];
      if (st != tick && (st < best_t || (st == best_t && sidx < best_s))) {
        best_t = st;
        best_s = sidx;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const long long ot = __shfl_xor_sync(0xffffffffu, best_t, o);
      const int os = __shfl_xor_sync(0xffffffffu, best_s, o);
      if (ot < best_t || (ot == best_t && os < best_s)) {
        best_t = ot;
        best_s = os;
      }
    }
    if (lane == 0) {
      const int e = s_miss[m];
      if (best_s >= rd.n_spare) {  // cannot happen: the host takes this path only when the slots suffice
        flag_status(rd.status_word, MOE_DEV_NO_SLOT);
      } else {
        const int old = rd.slot_expert[best_s];
        if (old >= 0) {
          rd.expert_slot[old] = -1;
          map_of[old] = -1;
        }
        rd.slot_expert[best_s] = e;
        rd.expert_slot[e] = best_s;
        rd.slot_tick[best_s] = tick;
        map_of[e] = E + best_s;
        rd.copy_e[m] = e;
        rd.copy_slot[m] = best_s;
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    *rd.copy_n = nmiss;
    long long* st = rd.stats;
    st[0] = touched;
    st[1] = routed;
    st[2] = hits;
    st[3] = nmiss;
    st[4] += hits;
    st[5] += nmiss;
    st[6] += 1;
  }
}

// Copies the listed experts' records (gate/up, down, and FP8 scales) from
// pinned host memory into their spare slots: 16-byte vectors, four loads in
// flight per thread, grid-stride over every listed record.
__global__ void __launch_bounds__(512) residency_copy_kernel(ResidencyDev rd, uint8_t* __restrict__ spare) {
  pdl_wait();  // the copy list comes from the plan
  pdl_trigger();
  const int n = *rd.copy_n;
  if (n == 0) return;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (int i = 0; i < n; ++i) {
    const int e = rd.copy_e[i];
    uint8_t* slot = spare + (size_t)rd.copy_slot[i] * rd.slot_bytes;
    for (int part = 0; part < 4; ++part) {
      const uint4* src = static_cast<const uint4*>(rd.host[e].p[part]);
      if (!src || rd.part_bytes[part] == 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(slot + rd.part_off[part]);
      const size_t nv = rd.part_bytes[part] / 16;
      size_t v = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
      for (; v + 3 * stride < nv; v += 4 * stride) {
        const uint4 a = src[v], b = src[v + stride], c = src[v + 2 * stride], d = src[v + 3 * stride];
        dst[v] = a;
        dst[v + stride] = b;
        dst[v + 2 * stride] = c;
        dst[v + 3 * stride] = d;
      }
      for (; v < nv; v += stride) dst[v] = src[v];
    }
  }
}

}  // namespace

cudaError_t launch_residency_plan(const int32_t* idx, int P, int E, const ResidencyDev& rd, int32_t* map_of,
                                  cudaStream_t s, bool pdl) {
  return launch_ex(residency_plan_kernel, dim3(1), dim3(1024), 0, s, pdl, idx, P, E, rd, map_of);
}

cudaError_t launch_residency_copy(const ResidencyDev& rd, uint8_t* spare, int num_sms, cudaStream_t s, bool pdl) {
  return launch_ex(residency_copy_kernel, dim3(2 * num_sms), dim3(512), 0, s, pdl, rd, spare);
}

}  // namespace moe
