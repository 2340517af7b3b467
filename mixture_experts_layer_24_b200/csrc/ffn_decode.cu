// ffn_decode.cu -- the decode forward's whole expert FFN in one persistent
// launch (bf16 weights, up to 64 tokens), planned from the router's top-k.
//
// Per routed pair (token t, expert e, slot k), as in ffn_gemm.cu:
//   g = Wg[e] x_t, u = Wu[e] x_t, h = bf16(silu(g) * u), y_pair = w[t,k] * (Wd[e] h)
// with the same swap-AB tiles, K order and per-column results as the grouped
// GEMMs, so its outputs equal theirs bit for bit.
#include "common.cuh"
#include "internal.h"
#include "tile.cuh"

namespace moe {

// ============================================================ decode (planned here)
// The decode forward's FFN straight from the router's top-k: no permutation
// kernel and no gathered copy of x. After its programmatic wait every CTA
// builds the permutation (a counting sort of the T*K pairs by expert, then
// token) and the tile plan in shared memory; CTA 0 also writes counts,
// offsets, perm_src, perm_k and inv for the combine. The gate/up B operand is
// x itself, all TP = T rounded up to 16 tokens (rows past T read as zeros), so
// a gate/up tile covers every pair of its expert and writes h row p from
// token column perm_src[p]; a down tile reads its expert's h rows. Per-column
// MMA results do not depend on the tile width, so every value equals the one
// the separate kernels compute. Tile queue, dependency counters (one per
// touched expert; zeroed by the router, the first kernel of the forward) and
// pipelines are those of ffn_bf16_fused_kernel.

template <int TP>
struct DecodeCfg {
  static constexpr uint32_t kStageBytes = 2 * kABytes + 2 * TP * 128;  // down: 2 chunks; gate/up: 1 chunk
  static constexpr int kStagesFit = (196 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kRing = 8;
  static constexpr uint32_t kAcc = 2 * TP;
  static constexpr uint32_t kTmemCols = tmem_cols_for(2 * kAcc);
  static constexpr int kMaxPairs = 512;
  // plan: s_e, s_psrc, s_pk [kMaxPairs]; s_cnt[E], s_off[E+1], s_list[E]; s_t2p[TP]; scan[8]; s_run[E]; s_inv[kMaxPairs]
  static size_t plan_bytes(int E) { return 4 * (4 * (size_t)kMaxPairs + 4 * (size_t)E + 1 + TP + 8); }
  static size_t smem(int E) {
    return 1024 + (size_t)kStages * kStageBytes + 8 * (2 * kStages + 4 + 2 * kRing) + 4 * kRing + 16 + 4 * TP +
           plan_bytes(E);
  }
  static_assert(kStages >= 2, "a pipeline needs two stages");
};

// Exclusive scan over 192 threads (6 warps), one value per thread.
__device__ __forceinline__ int scan192(int v, int* sh /* >= 8 ints */, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) sh[w] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < 6; ++i) {
      const int t = sh[i];
      sh[i] = run;
      run += t;
    }
    sh[6] = run;
  }
  __syncthreads();
  const int res = sh[w] + incl - v;
  *total = sh[6];
  __syncthreads();
  return res;
}

template <int TP>
__global__ void __launch_bounds__(192, 1) ffn_bf16_decode_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                 const __grid_constant__ ActMaps hact,
                                                                 const GemmArgs a, DecodeArgs d) {
  using C = DecodeCfg<TP>;
  constexpr int S = C::kStages, R = C::kRing;
  constexpr uint32_t STAGE = C::kStageBytes, ACC = C::kAcc, B_OFF = 2 * kABytes;
  const int mg = a.I / 128, md = a.H / 128;
  const int KBg = a.H / 64, KBd = a.I / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int E = d.E, K = a.K, P = d.T * K;

  pdl_wait();  // the router's top-k (and the zeroed counters) come from the previous kernel
  pdl_trigger();

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + S * STAGE;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto tfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  auto rfull = [&](int r) { return bars + 8u * (2 * S + 4 + r); };
  auto rempty = [&](int r) { return bars + 8u * (2 * S + 4 + R + r); };
  uint8_t* after_bars = gbase + S * STAGE + 8 * (2 * S + 4 + 2 * R);
  volatile int* ring = reinterpret_cast<volatile int*>(after_bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(after_bars + 4 * R);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* wcol = reinterpret_cast<float*>(tmem_slot + 4);  // [TP]
  int* s_e = reinterpret_cast<int*>(wcol + TP);           // [kMaxPairs] expert of pair i (-1: invalid)
  int* s_psrc = s_e + C::kMaxPairs;                       // [kMaxPairs] token of sorted pair p
  int* s_pk = s_psrc + C::kMaxPairs;                      // [kMaxPairs] top-k slot of sorted pair p
  int* s_cnt = s_pk + C::kMaxPairs;                       // [E]
  int* s_off = s_cnt + E;                                 // [E + 1]
  int* s_list = s_off + E + 1;                            // [E] touched experts, ascending
  int* s_t2p = s_list + E;                                // [TP] gate/up epilogue: token -> pair of the tile's expert
  int* s_scan = s_t2p + TP;                               // [8]
  int* s_run = s_scan + 8;                                // [E] running count per expert (ranks)
  int* s_inv = s_run + E;                                 // [kMaxPairs] sorted place of pair i

  // ---------------------------------------------------------------- plan
  for (int i = tid; i < E; i += 192) s_cnt[i] = 0;
  __syncthreads();
  for (int i = tid; i < P; i += 192) {
    int e = d.topk_idx[i];
    if (e < 0 || e >= E) {
      if (blockIdx.x == 0) flag_status(a.status, MOE_DEV_BAD_EXPERT);
      e = -1;
    } else if (d.map_of[e] < 0) {
      if (blockIdx.x == 0) flag_status(a.status, MOE_DEV_NO_SLOT);
    }
    s_e[i] = e;
    if (e >= 0) atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  // one scan of (count | touched << 16) gives both the pair offsets and the touched list
  const int per = (E + 191) / 192;
  const int e0 = tid * per;
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int c = s_cnt[e];
    local += c + ((c > 0 && d.map_of[e] >= 0) ? (1 << 16) : 0);
  }
  int tot;
  int run = scan192(local, s_scan, &tot);
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int c = s_cnt[e];
    s_off[e] = run & 0xffff;
    if (c > 0 && d.map_of[e] >= 0) s_list[run >> 16] = e;
    run += c + ((c > 0 && d.map_of[e] >= 0) ? (1 << 16) : 0);
  }
  if (tid == 0) s_off[E] = tot & 0xffff;
  const int L = tot >> 16;
  __syncthreads();
  // ranks: warp 0 walks the pairs in chunks of 32 in pair order; a pair's
  // place is its expert's running count plus the same-expert lanes before it
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) s_run[e] = s_off[e];
    __syncwarp();
    for (int i0 = 0; i0 < P; i0 += 32) {
      const int i = i0 + lane;
      const int e = i < P ? s_e[i] : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int before = __popc(peers & ((1u << lane) - 1u));
      int p = -1;
      if (e >= 0) {
        p = s_run[e] + before;
        s_psrc[p] = i / K;
        s_pk[p] = i - (i / K) * K;
      }
      if (i < P) s_inv[i] = p;
      __syncwarp();
      if (e >= 0 && before == 0) s_run[e] += __popc(peers);  // the group's first lane advances the count
      __syncwarp();
    }
  }
  __syncthreads();
  if (blockIdx.x == 0)  // a pair of an unregistered expert is dropped: the combine skips inv = -1
    for (int i = tid; i < P; i += 192) d.inv[i] = (s_e[i] >= 0 && d.map_of[s_e[i]] < 0) ? -1 : s_inv[i];
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += 192) {
      d.counts[e] = s_cnt[e];
      d.offsets[e] = s_off[e];
    }
    if (tid == 0) d.offsets[E] = s_off[E];
    for (int p = tid; p < s_off[E]; p += 192) {
      d.perm_src[p] = s_psrc[p];
      d.perm_k[p] = s_pk[p];
    }
  }

  const int Gt = L * mg, total = Gt + L * md;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) return;

  // tile -> (gate/up?, expert, 128-row tile)
  auto decode = [&](int tile, bool& gu, int& l, int& mt) {
    gu = tile < Gt;
    const int t2 = gu ? tile : tile - Gt;
    const int m = gu ? mg : md;
    l = t2 / m;
    mt = t2 - l * m;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), 4);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(rfull(r), 1);
      mbar_init(rempty(r), 5);
    }
    *abort_flag = 0;
    *ep_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const uint32_t gu_tx = 2 * kABytes + TP * 128u;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();  // one tile per expert and row block: sole reader
      int issued = 0;
      int tile = blockIdx.x;
      auto fail = [&]() {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      };
      tensormap_acquire(&xmap);
      for (int j = 0;; ++j) {
        const int slot = j % R;
        if (j >= R && !mbar_wait(rempty(slot), ((j / R) - 1) & 1)) {
          fail();
          break;
        }
        const int pub = (tile < total && !*abort_flag) ? tile : -1;
        ring[slot] = pub;
        mbar_arrive(rfull(slot));
        if (pub < 0) break;
        bool gu;
        int l, mt;
        decode(tile, gu, l, mt);
        const int e = s_list[l];
        const MapEntry* me = a.maps + d.map_of[e];
        bool ok = true;
        if (gu) {
          const void* wmap = &me->gu;
          tensormap_acquire(wmap);
          for (int kb = 0; kb < KBg; ++kb, ++issued) {
            const int s = issued % S;
            if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
              ok = false;
              break;
            }
            const uint32_t st = base + s * STAGE;
            mbar_arrive_expect_tx(full(s), gu_tx);
            tma_load_3d_hint(st, wmap, full(s), 0, mt * 128, kb, pol_w);
            tma_load_3d_hint(st + kABytes, wmap, full(s), 0, a.I + mt * 128, kb, pol_w);
            tma_load_3d(st + B_OFF, &xmap, full(s), 0, 0, kb);
          }
        } else {
          const int cnt = s_cnt[e], row0 = s_off[e];
          const int wi = tile_width_index(cnt, TP);
          const void* wmap = &me->dn2;
          const void* amap = &hact.m[wi];
          const uint32_t tx = 2 * kABytes + 2 * (16u << wi) * 128u;
          tensormap_acquire(wmap);
          const int npre = KBd < S ? KBd : S;
          int kb = 0;
          for (; kb < npre; ++kb) {
            const int n = issued + kb, s = n % S;
            if (n >= S && !mbar_wait(empty(s), ((n / S) - 1) & 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full(s), tx);
            tma_load_3d_hint(base + s * STAGE, wmap, full(s), 0, mt * 128, 2 * kb, pol_w);
          }
          if (ok) {
            const int* dep = a.sched + 1 + l;  // gate/up tiles of this expert that stored their h
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_gpu(dep) < mg) {
              if (global_timer_ns() - t0 > kWaitLimitNs) {
                ok = false;
                break;
              }
              __nanosleep(64);
            }
          }
          if (ok) {
            fence_proxy_async_global();
            for (int j2 = 0; j2 < npre; ++j2) {
              const int s = (issued + j2) % S;
              tma_load_3d(base + s * STAGE + B_OFF, amap, full(s), 0, row0, 2 * j2);
            }
            issued += npre;
            for (; kb < KBd; ++kb, ++issued) {
              const int s = issued % S;
              if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
                ok = false;
                break;
              }
              const uint32_t st = base + s * STAGE;
              mbar_arrive_expect_tx(full(s), tx);
              tma_load_3d_hint(st, wmap, full(s), 0, mt * 128, 2 * kb, pol_w);
              tma_load_3d(st + B_OFF, amap, full(s), 0, row0, 2 * kb);
            }
          } else {
            issued += kb;
          }
        }
        if (!ok) {
          fail();
          tile = total;
          continue;
        }
        tile = (int)gridDim.x + atomicAdd(a.sched, 1);
      }
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int consumed = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int slot = j % R;
        if (!mbar_wait(rfull(slot), (j / R) & 1)) {
          ok = false;
          break;
        }
        const int tile = ring[slot];
        mbar_arrive(rempty(slot));
        if (tile < 0) break;
        bool gu;
        int l, mt;
        decode(tile, gu, l, mt);
        const int width = gu ? TP : 16 << tile_width_index(s_cnt[s_list[l]], TP);
        const uint32_t idesc = instr_desc(128, width, 1u);
        const int buf = j & 1;
        if (j >= 2 && !mbar_wait(tempty(buf), ((j >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dd = tmem + buf * ACC;
        const int KB = gu ? KBg : KBd;
        for (int kb = 0; kb < KB; ++kb, ++consumed) {
          const int s = consumed % S;
          if (!mbar_wait(full(s), (consumed / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * STAGE;
          if (gu) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t bdesc = sw128_kmajor_desc(st + B_OFF + k * 32);
              const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
              tc_mma_bf16(dd, sw128_kmajor_desc(st + k * 32), bdesc, idesc, acc);
              tc_mma_bf16(dd + TP, sw128_kmajor_desc(st + kABytes + k * 32), bdesc, idesc, acc);
            }
          } else {
            const uint32_t chunk_b = (uint32_t)width * 128u;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t bdesc = sw128_kmajor_desc(st + B_OFF + c * chunk_b + k * 32);
                const uint32_t acc = (kb | c | k) != 0 ? 1u : 0u;
                tc_mma_bf16(dd, sw128_kmajor_desc(st + c * kABytes + k * 32), bdesc, idesc, acc);
              }
            }
          }
          tc_commit(empty(s));
        }
        tc_commit(tfull(buf));
      }
      if (!ok) {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0..3)
    const int r = warp * 32 + lane;
    for (int j = 0;; ++j) {
      const int slot = j % R;
      int tile = -1;
      if (lane == 0) {
        if (!*abort_flag && mbar_wait(rfull(slot), (j / R) & 1)) {
          tile = ring[slot];
          mbar_arrive(rempty(slot));
        } else {
          *ep_abort = 1;
        }
      }
      tile = __shfl_sync(0xffffffffu, tile, 0);
      named_bar_sync(2, 128);
      if (*ep_abort) {
        flag_status(a.status, MOE_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      if (tile < 0) break;
      bool gu;
      int l, mt;
      decode(tile, gu, l, mt);
      const int e = s_list[l], cnt = s_cnt[e], row0 = s_off[e];
      named_bar_sync(1, 128);  // previous tile's readers are done with s_t2p / wcol
      if (gu) {
        for (int c = r; c < TP; c += 128) s_t2p[c] = -1;
        named_bar_sync(1, 128);
        for (int n = r; n < cnt; n += 128) s_t2p[s_psrc[row0 + n]] = row0 + n;
      } else {
        for (int n = r; n < TP; n += 128)
          wcol[n] = n < cnt ? __ldg(a.topk_w + (size_t)s_psrc[row0 + n] * K + s_pk[row0 + n]) : 0.0f;
      }
      named_bar_sync(1, 128);
      const int buf = j & 1;
      if (lane == 0 && (*abort_flag || !mbar_wait(tfull(buf), (j >> 1) & 1))) *ep_abort = 1;
      named_bar_sync(2, 128);
      if (*ep_abort) {
        flag_status(a.status, MOE_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem + buf * ACC + (static_cast<uint32_t>(warp * 32) << 16);
      if (gu) {
        const int jj = mt * 128 + r;
        __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(a.h_out);
#pragma unroll 1
        for (int c = 0; c < TP; c += 16) {
          if (c >= d.T) break;
          uint32_t g[16], u[16];
          tmem_ld16(tl + c, g);
          tmem_ld16(tl + TP + c, u);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int pp = s_t2p[c + q];  // token c + q's pair with this expert, if any
            if (pp >= 0) {
              const float gv = __uint_as_float(g[q]);
              const float uv = __uint_as_float(u[q]);
              const float hv = gv / (1.0f + expf(-gv)) * uv;
              hout[(size_t)pp * a.I + jj] = __float2bfloat16_rn(hv);
            }
          }
        }
      } else {
        const int o = mt * 128 + r;
#pragma unroll 1
        for (int c = 0; c < TP; c += 16) {
          if (c >= cnt) break;
          uint32_t v[16];
          tmem_ld16(tl + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            if (c + q < cnt) a.y_out[(size_t)(row0 + c + q) * a.H + o] = wcol[c + q] * __uint_as_float(v[q]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(buf));
      if (gu) {
        __threadfence();
        named_bar_sync(1, 128);
        if (r == 0) atomicAdd(a.sched + 1 + l, 1);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int TP>
static cudaError_t launch_decode(const CUtensorMap& xmap, const ActMaps& hmaps, const GemmArgs& a,
                                 const DecodeArgs& d, int grid, cudaStream_t s, bool pdl) {
  using C = DecodeCfg<TP>;
  const size_t smem = C::smem(d.E);
  if (smem > 232448) return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(ffn_bf16_decode_kernel<TP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;
  if (persistent <= 0) return cudaSuccess;
  return launch_ex(ffn_bf16_decode_kernel<TP>, dim3(persistent), dim3(192), smem, s, pdl, xmap, hmaps, a, d);
}

size_t ffn_decode_smem_bytes(int T, int E) {
  const int tp = (T + 15) / 16 * 16;
  if (tp <= 16) return DecodeCfg<16>::smem(E);
  if (tp <= 32) return DecodeCfg<32>::smem(E);
  return DecodeCfg<64>::smem(E);
}

cudaError_t launch_ffn_decode(const CUtensorMap& xmap, const ActMaps& hmaps, const GemmArgs& a, const DecodeArgs& d,
                              int max_tiles, cudaStream_t s, bool pdl) {
  const int tp = (d.T + 15) / 16 * 16;
  switch (tp) {
    case 16: return launch_decode<16>(xmap, hmaps, a, d, max_tiles, s, pdl);
    case 32: return launch_decode<32>(xmap, hmaps, a, d, max_tiles, s, pdl);
    case 48:
    case 64: return launch_decode<64>(xmap, hmaps, a, d, max_tiles, s, pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
