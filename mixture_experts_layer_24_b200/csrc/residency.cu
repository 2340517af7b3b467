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
//   plan (one CTA, residency.cuh): the experts the top-k routes to; a host
//     expert already in a slot is a hit (its slot's tick is refreshed); each
//     miss, in expert order, takes the least recently used slot this call
//     does not need (ties to the lowest slot), the evicted expert loses its
//     slot, and the expert -> map-entry table the FFN reads points the new one
//     at its slot; the misses are listed for the copy. Up to 4 tokens the
//     router's fused last CTA runs it after the top-k, and this kernel is not
//     launched.
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
#include "residency.cuh"

namespace moe {

namespace {

__global__ void __launch_bounds__(1024) residency_plan_kernel(const int32_t* __restrict__ idx, int P, int E,
                                                               ResidencyDev rd, int32_t* __restrict__ map_of) {
  __shared__ ResidencyPlanSmem sp;
  pdl_wait();  // the top-k comes from the router
  pdl_trigger();
  residency_plan_block(idx, P, E, rd, map_of, sp);
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
