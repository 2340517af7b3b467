// residency.cuh -- the device-side LRU plan of one forward over the spare HBM
// slots (residency.cu's plan kernel, and the decode router's fused last CTA,
// which runs it right after the top-k so that no launch sits between them).
//
// The "hotsplit" recipes wiki (Home page) keeps the hot experts on the GPU and
// reads the cold ones from pinned host memory on demand; the vLLM-Moet page's
// cache variant (hybrid results, "hit rate 0.88 vs 0.87") keeps the most
// recently used ones. The experts the top-k routes to are marked; a host
// expert already in a slot is a hit (its slot's tick is refreshed); each miss,
// in expert order, takes the least recently used slot this call does not need
// (ties to the lowest slot), the evicted expert loses its slot, and the
// expert -> map-entry table the FFN reads points the new one at its slot; the
// misses are listed for the copy.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

// Shared memory of the plan, in the calling kernel.
struct ResidencyPlanSmem {
  uint8_t touched[1024];
  int miss[1024];
  int nmiss;
  long long tick;
};

// Run by every thread of one CTA (any blockDim that is a multiple of 32);
// idx [P] must be complete and visible to the CTA.
__device__ __forceinline__ void residency_plan_block(const int32_t* idx, int P, int E, const ResidencyDev& rd,
                                                     int32_t* map_of, ResidencyPlanSmem& sp) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int e = tid; e < E; e += blockDim.x) sp.touched[e] = 0;
  __syncthreads();
  for (int i = tid; i < P; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) sp.touched[e] = 1;
  }
  __syncthreads();
  if (tid >= 32) return;
  // one warp from here: hits first, misses listed in expert order
  if (lane == 0) {
    sp.tick = *rd.tick + 1;
    *rd.tick = sp.tick;
    sp.nmiss = 0;
  }
  __syncwarp();
  const long long tick = sp.tick;
  int touched = 0, routed = 0, hits = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    const bool t = e < E && sp.touched[e];
    const bool host = t && rd.loc[e] == MOE_LOC_HOST_PINNED;
    const int slot = host ? rd.expert_slot[e] : -1;
    if (host && slot >= 0) rd.slot_tick[slot] = tick;
    const unsigned miss = __ballot_sync(0xffffffffu, host && slot < 0);
    if (host && slot < 0) sp.miss[sp.nmiss + __popc(miss & ((1u << lane) - 1u))] = e;
    touched += __popc(__ballot_sync(0xffffffffu, t));
    routed += __popc(__ballot_sync(0xffffffffu, host));
    hits += __popc(__ballot_sync(0xffffffffu, host && slot >= 0));
    __syncwarp();
    if (lane == 0) sp.nmiss += __popc(miss);
    __syncwarp();
  }
  const int nmiss = sp.nmiss;
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
      const int e = sp.miss[m];
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

}  // namespace moe
