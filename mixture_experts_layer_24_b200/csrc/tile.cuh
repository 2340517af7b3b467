// tile.cuh -- tile bookkeeping shared by the grouped expert GEMMs
// (ffn_gemm.cu, ffn_mxfp4.cu): which (expert, 128-row weight tile, N tile of
// pairs) a persistent CTA's tile index names, and the per-tile MMA width.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr uint32_t kABytes = 128 * 128;  // one 128-row x 128-byte operand tile

__host__ __device__ constexpr uint32_t tmem_cols_for(int cols) {
  return cols <= 32 ? 32 : cols <= 64 ? 64 : cols <= 128 ? 128 : cols <= 256 ? 256 : 512;
}

struct TileInfo {
  int e, mapi, mt, row0, nvalid, nti;  // nti: N tiles of this expert (readers of each weight tile)
  int ng;                              // global index of the tile's N tile (nt_prefix[expert slot] + nt)
  int li;                              // the expert's index in the launch's list
};

// The (expert, 128-row tile, N tile) of tile index `tile` (no range or status checks).
__device__ __forceinline__ void decode_tile_at(const GemmArgs& a, int m_tiles, int bn, int tile, TileInfo& ti) {
  int lo = 0, hi = a.L;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.nt_prefix[mid] * m_tiles <= tile) lo = mid;
    else hi = mid;
  }
  const int nti = a.nt_prefix[lo + 1] - a.nt_prefix[lo];
  const int local = tile - a.nt_prefix[lo] * m_tiles;
  const int mt = local / nti, nt = local - mt * nti;
  ti.e = a.list_expert[lo];
  ti.mapi = a.list_map[lo];
  ti.mt = mt;
  ti.row0 = a.offsets[ti.e] + nt * bn;
  ti.nvalid = min(bn, a.offsets[ti.e + 1] - ti.row0);
  ti.nti = nti;
  ti.ng = a.nt_prefix[lo] + nt;
  ti.li = lo;
}

__device__ __forceinline__ void tensormap_acquire(const void* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(map) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Per-tile MMA width: the smallest of 16, 32, 64, 128 (<= BN) that holds
// the tile's pairs; its index selects the activation map of that box height.
__device__ __forceinline__ int tile_width_index(int nvalid, int bn) {
  int w = 16, i = 0;
  while (w < nvalid && w < bn) {
    w <<= 1;
    ++i;
  }
  return i;
}

}  // namespace moe
