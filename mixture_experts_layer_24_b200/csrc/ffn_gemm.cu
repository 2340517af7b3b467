// ffn_gemm.cu -- grouped expert FFN on the 5th-generation tensor cores.
//
// Per routed pair (token t, expert e, slot k) of a DeepSeek-class MoE layer
// (vLLM-Moet, topairepos.com page, model table: the "b12x" MoE GPU kernels of
// the hybrid's step breakdown are this step):
//   gate/up:  g = Wg[e] x_t, u = Wu[e] x_t (fp32 accumulate), h = bf16(silu(g) * u)
//   down:     y_pair = w[t,k] * (Wd[e] h)                     (fp32)
//
// Orientation ("swap AB"): the expert's weight rows are the MMA M operand
// (128 rows per CTA) and the pairs routed to the expert are the N operand
// (BN columns), both K-major in shared memory with the 128-byte swizzle and
// fed by TMA. Each CTA computes one (expert, 128-row tile, BN-pair tile) over
// the full K, K-blocks in increasing order, with no split-K, so the fp32 sum
// behind any output element is the same whatever BN, the batch or the set of
// resident experts; only the columns a CTA owns differ.
//
// Warp roles (one CTA per tile):
//   warps 0..3 (bf16) / 0..7 (fp8): epilogue (TMEM -> registers -> global)
//   next warp: TMA producer (one elected lane)
//   last warp: TMEM allocator + MMA issuer (one elected lane)
// Gate/up CTAs hold two accumulators, gate rows [j, j+128) and up rows
// [I+j, I+j+128), so one thread owns g and u of the same (j, pair) and SwiGLU
// happens in the epilogue without any exchange.
//
// FP8 (e4m3 operands, kind::f8f6f4): one stage is one 128-wide K block, which
// is one scale block of both operands. The MMA writes each block's partial
// sum P_kb into one of two TMEM buffers; the epilogue promotes it in fp32
// registers, acc = fmaf(P_kb, s_act[pair, kb] * s_w[rowblock, kb], acc),
// K blocks in increasing order.
#include "common.cuh"
#include "internal.h"
#include "tile.cuh"

namespace moe {

// bf16: one pipeline stage holds kKC consecutive 64-wide K chunks, fetched by
// one 3-D TMA copy per operand (the per-copy cost of the TMA unit, not the
// bytes, bounds a single SM's streaming rate for small boxes).
template <int MODE, int BN>
struct Bf16Cfg {
  static constexpr int NA = MODE == kGateUp ? 2 : 1;
  static constexpr int KC = kBf16KChunks;
  static constexpr uint32_t kChunkA = kABytes;     // 128 rows x 128 B
  static constexpr uint32_t kChunkB = BN * 128;    // BN rows x 128 B
  static constexpr uint32_t kStageBytes = KC * (NA * kChunkA + kChunkB);
  // up to 220 KB of stages (227 KB per CTA at most; one CTA per SM): three
  // two-chunk stages at BN <= 32
  static constexpr int kStagesFit = (220 * 1024) / kStageBytes;
  static constexpr int kStagesMax = kStagesFit > 8 ? 8 : kStagesFit;
  // two accumulator buffers whenever both fit in TMEM's 512 columns
  static constexpr int NBUF = 2 * NA * BN <= 512 ? 2 : 1;
  static constexpr uint32_t kTmemCols = tmem_cols_for(NBUF * NA * BN);
  static constexpr size_t smem(int stages) { return 1024 + (size_t)stages * kStageBytes + 256 + 4 * BN; }
  static_assert(kStagesMax >= 2, "a pipeline needs two stages");
};

template <int MODE, int BN>
struct Fp8Cfg {
  static constexpr int NA = MODE == kGateUp ? 2 : 1;
  static constexpr uint32_t kStageBytes = NA * kABytes + BN * 128;  // one 128-wide K block
  static constexpr int kMaxKB = 64;                                   // K / 128 <= 64 (K <= 8192)
  // activation scales [BN][KB], weight scales [2][KB], routing weights [BN]
  static constexpr uint32_t kScaleBytes = BN * kMaxKB * 4 + 2 * kMaxKB * 4 + BN * 4;
  static constexpr int kStagesRaw = (220 * 1024 - (int)kScaleBytes) / (int)kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  // TMEM buffers of per-K-block partial sums (the MMA runs up to NP blocks ahead of the promotion)
  static constexpr int kNpRaw = 512 / (NA * BN);
  static constexpr int NP = kNpRaw > 8 ? 8 : kNpRaw;
  static constexpr uint32_t kTmemCols = tmem_cols_for(NP * NA * BN);
  static constexpr size_t kSmem = 1024 + kStages * kStageBytes + kScaleBytes + 8 * (2 * kStages + 2 * NP) + 64;
  // epilogue warps (4 TMEM lane quarters x EW/4 column groups); 16 at BN = 64
  // measured no faster than 8
  static constexpr int EW = 8;
  static_assert(kStages >= 2 && NP >= 2, "FP8 pipeline needs two stages and two partial buffers");
};

// ====================================================================== bf16
// Persistent: one CTA per SM walks tiles blockIdx.x, +gridDim.x, ... The
// shared-memory pipeline runs on across tile boundaries (stage and phase come
// from one running K-step count), and the accumulator lives in one of NBUF
// TMEM buffers so that the epilogue of tile j overlaps the MMAs of tile j+1.

template <int MODE, int BN>
__global__ void __launch_bounds__(192, 1) ffn_bf16_kernel(const __grid_constant__ ActMaps act,
                                                          const GemmArgs a) {
  using C = Bf16Cfg<MODE, BN>;
  constexpr int NA = C::NA, kKC = C::KC, NBUF = C::NBUF;
  constexpr uint32_t STAGE = C::kStageBytes;
  constexpr uint32_t A_OP = kKC * C::kChunkA;  // bytes of one A operand per stage
  constexpr uint32_t B_OFF = NA * A_OP;        // stage: [A gate][A up][B], kKC chunks each
  constexpr uint32_t ACC = NA * BN;            // TMEM columns of one accumulator buffer
  const int S = a.stages;
  const int m_tiles = (MODE == kGateUp ? a.I : a.H) / 128;
  const int KB = (MODE == kGateUp ? a.H : a.I) / (64 * kKC);  // K steps per tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (!a.plan_ready) {
    pdl_wait();
    pdl_trigger();
  }
  const int total = a.nt_prefix[a.L] * m_tiles;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) {
    pdl_wait();
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + S * STAGE;  // full[S], empty[S], tfull[2], tempty[2]
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto tfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * STAGE + 8 * (2 * S + 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);  // written by epilogue warps only
  float* wcol = reinterpret_cast<float*>(tmem_slot + 4);  // [BN] routing weights of the tile's pairs (down)

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), 4);
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

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // Weights: evict-first when the tile is the weight rows' only reader;
      // an expert with several N tiles has each weight tile read by all of
      // them (close together in time), so there the lines keep the normal
      // policy and the later readers hit L2.
      const uint64_t pol_once = l2_policy_evict_first(), pol_shared = l2_policy_evict_normal();
      int issued = 0;  // K steps issued so far (all tiles)
      bool first = true;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int wi = tile_width_index(ti.nvalid, BN);
        const void* amap = &act.m[wi];
        const uint32_t stage_tx = NA * A_OP + kKC * ((16u << wi) * 128u);
        const uint64_t pol_w = ti.nti > 1 ? pol_shared : pol_once;
        const MapEntry* me = a.maps + ti.mapi;
        const void* wmap = MODE == kGateUp ? static_cast<const void*>(kKC == 1 ? &me->gu : &me->gu2)
                                           : static_cast<const void*>(kKC == 1 ? &me->dn : &me->dn2);
        tensormap_acquire(wmap);
        int kb = 0;
        if (first) {
          first = false;
          // the plan is complete: the first weight stages go out before waiting
          // for the kernel that writes the activations
          const int npre = a.plan_ready ? (KB < S ? KB : S) : 0;
          for (int j = 0; j < npre; ++j) {
            const uint32_t st = base + j * STAGE;
            mbar_arrive_expect_tx(full(j), stage_tx);
            tma_load_3d_hint(st, wmap, full(j), 0, ti.mt * 128, j * kKC, pol_w);
            if (MODE == kGateUp) tma_load_3d_hint(st + A_OP, wmap, full(j), 0, a.I + ti.mt * 128, j * kKC, pol_w);
          }
          if (a.plan_ready) {
            pdl_wait();
            pdl_trigger();
          }
          for (int j = 0; j < npre; ++j) tma_load_3d(base + j * STAGE + B_OFF, amap, full(j), 0, ti.row0, j * kKC);
          kb = npre;
          issued = npre;
        }
        for (; kb < KB; ++kb, ++issued) {
          const int s = issued % S;
          if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
            *abort_flag = 1;
            flag_status(a.status, MOE_DEV_TIMEOUT);
            break;
          }
          const uint32_t st = base + s * STAGE;
          mbar_arrive_expect_tx(full(s), stage_tx);
          tma_load_3d_hint(st, wmap, full(s), 0, ti.mt * 128, kb * kKC, pol_w);
          if (MODE == kGateUp) tma_load_3d_hint(st + A_OP, wmap, full(s), 0, a.I + ti.mt * 128, kb * kKC, pol_w);
          tma_load_3d(st + B_OFF, amap, full(s), 0, ti.row0, kb * kKC);
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    if (lane == 0) {
      int consumed = 0, j = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
        const int buf = j % NBUF;
        if (j >= NBUF && !mbar_wait(tempty(buf), ((j / NBUF) - 1) & 1)) {
          *abort_flag = 1;
          flag_status(a.status, MOE_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + buf * ACC;
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int width = 16 << tile_width_index(ti.nvalid, BN);
        const uint32_t idesc = instr_desc(128, width, 1u);
        const uint32_t chunk_b = (uint32_t)width * 128u;  // a 3-D box lands its K chunks densely
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++consumed) {
          const int s = consumed % S;
          if (!mbar_wait(full(s), (consumed / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * STAGE;
#pragma unroll
          for (int c = 0; c < kKC; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t bdesc = sw128_kmajor_desc(st + B_OFF + c * chunk_b + k * 32);
              const uint32_t acc = (kb | c | k) != 0 ? 1u : 0u;
              tc_mma_bf16(d, sw128_kmajor_desc(st + c * C::kChunkA + k * 32), bdesc, idesc, acc);
              if (MODE == kGateUp)
                tc_mma_bf16(d + BN, sw128_kmajor_desc(st + A_OP + c * C::kChunkA + k * 32), bdesc, idesc, acc);
            }
          }
          tc_commit(empty(s));
        }
        tc_commit(tfull(buf));
        if (!ok) {
          *abort_flag = 1;
          flag_status(a.status, MOE_DEV_TIMEOUT);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0..3)
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    const int r = warp * 32 + lane;
    int j = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
      const int buf = j % NBUF;
      TileInfo ti;
      decode_tile_at(a, m_tiles, BN, tile, ti);
      if (MODE == kDown) {
        // routing weights of this tile's pairs, once per tile
        named_bar_sync(1, 128);  // previous tile's readers are done with wcol
        for (int n = r; n < BN; n += 128) {
          float wv = 0.0f;
          if (n < ti.nvalid) {
            const int p = ti.row0 + n;
            wv = __ldg(a.topk_w + (size_t)__ldg(a.perm_src + p) * a.K + __ldg(a.perm_k + p));
          }
          wcol[n] = wv;
        }
        named_bar_sync(1, 128);
      }
      int okv = 1;
      if (lane == 0) okv = mbar_wait(tfull(buf), (j / NBUF) & 1) ? 1 : 0;
      if (lane == 0 && !okv) *ep_abort = 1;
      named_bar_sync(2, 128);  // the four epilogue warps leave the loop together or not at all
      if (*ep_abort) {
        flag_status(a.status, MOE_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int skip = __shfl_sync(0xffffffffu, *abort_flag ? 1 : 0, 0);  // warp-uniform around tcgen05.ld
      if (!skip) {
        const uint32_t tl = tmem + buf * ACC + (static_cast<uint32_t>(warp * 32) << 16);
        if (MODE == kGateUp) {
          const int jj = ti.mt * 128 + r;
          __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(a.h_out);
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t g[16], u[16];
            tmem_ld16(tl + c, g);
            tmem_ld16(tl + BN + c, u);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              if (c + q < ti.nvalid) {
                const float gv = __uint_as_float(g[q]);
                const float uv = __uint_as_float(u[q]);
                const float hv = gv / (1.0f + expf(-gv)) * uv;
                hout[(size_t)(ti.row0 + c + q) * a.I + jj] = __float2bfloat16_rn(hv);
              }
            }
          }
        } else {
          const int o = ti.mt * 128 + r;
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t v[16];
            tmem_ld16(tl + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              if (c + q < ti.nvalid) a.y_out[(size_t)(ti.row0 + c + q) * a.H + o] = wcol[c + q] * __uint_as_float(v[q]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(buf));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ======================================================================= fp8
// Persistent, like the bf16 kernel: one CTA per SM walks tiles blockIdx.x,
// +gridDim.x, ...; the shared-memory pipeline and a ring of NP TMEM buffers
// for the per-K-block partial sums run on across tile boundaries. Per tile the
// epilogue warps stage the tile's activation and weight scales (and, for down,
// the routing weights) in shared memory, then promote every K block's partial
// sum in registers, K blocks in increasing order. The MMA width adapts per
// tile (16 .. BN). After a failed (timed-out) wait a warp stops working but
// keeps its control flow, so the epilogue warps always meet at the same named
// barriers.

template <int MODE, int BN>
__global__ void __launch_bounds__(32 * (Fp8Cfg<MODE, BN>::EW + 2), 1)
    ffn_fp8_kernel(const __grid_constant__ ActMaps act, const GemmArgs a) {
  using C = Fp8Cfg<MODE, BN>;
  constexpr int NA = C::NA, S = C::kStages, NP = C::NP;
  constexpr uint32_t STAGE = C::kStageBytes;
  constexpr int EW = C::EW;            // epilogue warps: 4 TMEM lane quarters x EW/4 column groups
  constexpr int EPT = 32 * EW;         // epilogue threads
  constexpr int PW = EW, MW = EW + 1;  // producer warp, MMA warp
  constexpr int HALF = BN * 4 / EW;    // columns per epilogue warp
  constexpr int NCH = HALF >= 16 ? HALF / 16 : 1;
  constexpr int CW = HALF >= 16 ? 16 : HALF;  // columns used per TMEM load

  const int m_tiles = (MODE == kGateUp ? a.I : a.H) / 128;
  const int KD = MODE == kGateUp ? a.H : a.I;  // reduction length
  const int KB = KD / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (!a.plan_ready) {
    pdl_wait();
    pdl_trigger();
  }
  const int total = a.nt_prefix[a.L] * m_tiles;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) {
    pdl_wait();
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  float* s_act = reinterpret_cast<float*>(gbase + S * STAGE);  // [BN][KB] activation scales of the tile's pairs
  float* s_w = s_act + BN * C::kMaxKB;                         // [NA][KB] weight scales of the tile's row blocks
  float* wcol = s_w + 2 * C::kMaxKB;                           // [BN] routing weights (down)
  const uint32_t bars = base + S * STAGE + C::kScaleBytes;     // full[S], empty[S], pfull[NP], pempty[NP]
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto pfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto pempty = [&](int b) { return bars + 8u * (2 * S + NP + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * STAGE + C::kScaleBytes + 8 * (2 * S + 2 * NP));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < NP; ++b) {
      mbar_init(pfull(b), 1);
      mbar_init(pempty(b), EW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == MW) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == PW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_once = l2_policy_evict_first(), pol_shared = l2_policy_evict_normal();
      int issued = 0;
      bool first = true;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int wi = tile_width_index(ti.nvalid, BN);
        const void* amap = &act.m[wi];
        const uint32_t stage_tx = NA * kABytes + (16u << wi) * 128u;
        const uint64_t pol_w = ti.nti > 1 ? pol_shared : pol_once;  // evict-first only for a sole reader
        const MapEntry* me = a.maps + ti.mapi;
        const void* wmap = MODE == kGateUp ? static_cast<const void*>(&me->gu) : static_cast<const void*>(&me->dn);
        tensormap_acquire(wmap);
        int kb = 0;
        if (first) {
          first = false;
          const int npre = a.plan_ready ? (KB < S ? KB : S) : 0;
          for (int j = 0; j < npre; ++j) {
            const uint32_t st = base + j * STAGE;
            mbar_arrive_expect_tx(full(j), stage_tx);
            tma_load_2d_hint(st, wmap, full(j), j * 128, ti.mt * 128, pol_w);
            if (MODE == kGateUp) tma_load_2d_hint(st + kABytes, wmap, full(j), j * 128, a.I + ti.mt * 128, pol_w);
          }
          if (a.plan_ready) {
            pdl_wait();
            pdl_trigger();
          }
          for (int j = 0; j < npre; ++j) tma_load_2d(base + j * STAGE + NA * kABytes, amap, full(j), j * 128, ti.row0);
          kb = npre;
          issued = npre;
        }
        for (; kb < KB; ++kb, ++issued) {
          const int s = issued % S;
          if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
            *abort_flag = 1;
            flag_status(a.status, MOE_DEV_TIMEOUT);
            break;
          }
          const uint32_t st = base + s * STAGE;
          mbar_arrive_expect_tx(full(s), stage_tx);
          tma_load_2d_hint(st, wmap, full(s), kb * 128, ti.mt * 128, pol_w);
          if (MODE == kGateUp) tma_load_2d_hint(st + kABytes, wmap, full(s), kb * 128, a.I + ti.mt * 128, pol_w);
          tma_load_2d(st + NA * kABytes, amap, full(s), kb * 128, ti.row0);
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp == MW) {
    // ------------------------------------------------------------ MMA issuer
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    if (lane == 0) {
      int consumed = 0, kp = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int width = 16 << tile_width_index(ti.nvalid, BN);
        const uint32_t idesc = instr_desc(128, width, 0u);
        for (int kb = 0; kb < KB; ++kb, ++consumed, ++kp) {
          const int s = consumed % S, pb = kp % NP;
          ok = mbar_wait(full(s), (consumed / S) & 1);
          if (ok && kp >= NP) ok = mbar_wait(pempty(pb), ((kp / NP) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = base + s * STAGE;
          const uint32_t d = tmem + static_cast<uint32_t>(pb * NA * BN);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = sw128_kmajor_desc(st + NA * kABytes + k * 32);
            const uint32_t acc = k != 0 ? 1u : 0u;
            tc_mma_e4m3(d, sw128_kmajor_desc(st + k * 32), bdesc, idesc, acc);
            if (MODE == kGateUp) tc_mma_e4m3(d + BN, sw128_kmajor_desc(st + kABytes + k * 32), bdesc, idesc, acc);
          }
          tc_commit(empty(s));
          tc_commit(pfull(pb));
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0..EW-1)
    // warp w owns TMEM lanes [32(w%4), +32) and columns [HALF*(w/4), +HALF)
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    const int q4 = warp & 3, hf = warp >> 2;
    const int r = q4 * 32 + lane;
    const int et = threadIdx.x;  // 0..EPT-1
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int c0 = hf * HALF;
    bool aborted = false;  // warp-uniform
    int kp = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      TileInfo ti;
      decode_tile_at(a, m_tiles, BN, tile, ti);
      const int width = 16 << tile_width_index(ti.nvalid, BN);
      const MapEntry* me = a.maps + ti.mapi;
      const float* sw = MODE == kGateUp ? me->s_gu : me->s_dn;
      named_bar_sync(1, EPT);  // the previous tile's readers are done with the scale tables
      for (int i = et; i < BN * KB; i += EPT) {
        const int n = i / KB, kb = i - n * KB;
        s_act[n * KB + kb] = n < ti.nvalid ? a.act_scale[(size_t)(ti.row0 + n) * KB + kb] : 0.0f;
      }
      for (int i = et; i < NA * KB; i += EPT) {
        const int which = i / KB, kb = i - which * KB;
        const int rb = which == 0 ? ti.mt : a.I / 128 + ti.mt;  // gate (or down) row block, then up
        s_w[which * KB + kb] = sw[(size_t)rb * KB + kb];
      }
      if (MODE == kDown) {
        for (int n = et; n < BN; n += EPT) {
          float wv = 0.0f;
          if (n < ti.nvalid) {
            const int p = ti.row0 + n;
            wv = __ldg(a.topk_w + (size_t)__ldg(a.perm_src + p) * a.K + __ldg(a.perm_k + p));
          }
          wcol[n] = wv;
        }
      }
      named_bar_sync(1, EPT);

      float accg[HALF], accu[MODE == kGateUp ? HALF : 1];
#pragma unroll
      for (int i = 0; i < HALF; ++i) accg[i] = 0.0f;
#pragma unroll
      for (int i = 0; i < (MODE == kGateUp ? HALF : 1); ++i) accu[i] = 0.0f;
      for (int kb = 0; kb < KB; ++kb, ++kp) {
        const int pb = kp % NP;
        if (!aborted) {
          bool ok = !*abort_flag && mbar_wait(pfull(pb), (kp / NP) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            aborted = true;
            if (lane == 0) {
              *abort_flag = 1;
              flag_status(a.status, MOE_DEV_TIMEOUT);
            }
          }
        }
        if (!aborted) {
          tc_fence_after();
          const float swg = s_w[kb];
          const float swu = MODE == kGateUp ? s_w[KB + kb] : 0.0f;
          const uint32_t pbase = tl + static_cast<uint32_t>(pb * NA * BN);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const int cstart = CW == 16 ? c0 + ch * 16 : 0;  // first TMEM column of this load
            if (cstart < width) {                             // warp-uniform
              uint32_t pg[16], pu[16];
              tmem_ld16(pbase + cstart, pg);
              if (MODE == kGateUp) tmem_ld16(pbase + BN + cstart, pu);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < CW; ++q) {
                const int col = ch * CW + q;  // index within this warp's half
                const int n = c0 + col;       // tile column
                // register holding column n (HALF < 16: the load holds both halves)
                const uint32_t gb = CW == 16 ? pg[q] : (hf ? pg[(CW + q) & 15] : pg[q]);
                const float sa = s_act[n * KB + kb];
                accg[col] = fmaf(__uint_as_float(gb), sa * swg, accg[col]);
                if (MODE == kGateUp) {
                  const uint32_t ub = CW == 16 ? pu[q] : (hf ? pu[(CW + q) & 15] : pu[q]);
                  accu[col] = fmaf(__uint_as_float(ub), sa * swu, accu[col]);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pempty(pb));
      }
      if (!aborted) {
        if (MODE == kGateUp) {
          const int j = ti.mt * 128 + r;
          __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(a.h_out);
#pragma unroll
          for (int col = 0; col < HALF; ++col) {
            const int n = c0 + col;
            if (n < ti.nvalid) {
              const float gv = accg[col], uv = accu[col];
              const float hv = gv / (1.0f + expf(-gv)) * uv;
              hout[(size_t)(ti.row0 + n) * a.I + j] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          const int o = ti.mt * 128 + r;
#pragma unroll
          for (int col = 0; col < HALF; ++col) {
            const int n = c0 + col;
            if (n < ti.nvalid) a.y_out[(size_t)(ti.row0 + n) * a.H + o] = wcol[n] * accg[col];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MW) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ================================================================ fused decode
// Gate/up and down tiles of one forward in one persistent launch (bf16,
// BN <= 64). The tile queue is all gate/up tiles (expert, 128-row tile, N
// tile), then all down tiles; a CTA starts at blockIdx.x and takes further
// tiles from a global counter, so every gate/up tile is claimed before any
// down tile and CTAs that run out of gate/up work move on to down tiles while
// others finish, instead of waiting for a kernel boundary. A down tile needs
// the h rows of its N tile, which the 16 (I/128) gate/up tiles of the same
// expert and N tile write: each of those increments a counter after its
// stores; the down tile's producer streams its first weight stages, waits
// (acquire, bounded) for the count, and only then loads h. Each tile runs the
// same MMAs in the same K order as the separate kernels, so results are
// identical to them bit for bit.
//   stage: gate/up = [A gate][A up][B] (one 64-wide K chunk),
//          down    = [A c0][A c1][B c0][B c1] (two chunks); A always at 0, B at 32 KB.

template <int BN>
struct FusedCfg {
  static constexpr uint32_t kGuStage = 2 * kABytes + BN * 128;
  static constexpr uint32_t kDnStage = 2 * kABytes + 2 * BN * 128;
  static constexpr uint32_t kStageBytes = kDnStage;
  static constexpr int kStagesFit = (220 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr int kRing = 8;                             // tile indices in flight producer -> consumers
  static constexpr uint32_t kAcc = 2 * BN;                    // TMEM columns of one accumulator (gate + up)
  static constexpr uint32_t kTmemCols = tmem_cols_for(2 * kAcc);
  static constexpr size_t smem() {
    return 1024 + (size_t)kStages * kStageBytes + 8 * (2 * kStages + 4 + 2 * kRing) + 4 * kRing + 16 + 4 * BN;
  }
  static_assert(kStages >= 2, "a pipeline needs two stages");
  static_assert(kGuStage <= kStageBytes, "gate/up stage must fit the slot");
};

template <int BN>
__global__ void __launch_bounds__(192, 1) ffn_bf16_fused_kernel(const __grid_constant__ ActMaps xact,
                                                                const __grid_constant__ ActMaps hact,
                                                                const GemmArgs a) {
  using C = FusedCfg<BN>;
  constexpr int S = C::kStages, R = C::kRing;
  constexpr uint32_t STAGE = C::kStageBytes, ACC = C::kAcc, B_OFF = 2 * kABytes;
  const int mg = a.I / 128, md = a.H / 128;   // 128-row tiles per expert: gate/up, down
  const int KBg = a.H / 64, KBd = a.I / 128;  // K steps per tile: gate/up (1 chunk), down (2 chunks)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_wait();  // the plan and the counters come from the immediately preceding kernel
  pdl_trigger();
  const int NT = a.nt_prefix[a.L];
  const int Gt = NT * mg, total = Gt + NT * md;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + S * STAGE;  // full[S], empty[S], tfull[2], tempty[2], rfull[R], rempty[R]
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto tfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto tempty = [&](int b) { return bars + 8u * (2 * S + 2 + b); };
  auto rfull = [&](int r) { return bars + 8u * (2 * S + 4 + r); };
  auto rempty = [&](int r) { return bars + 8u * (2 * S + 4 + R + r); };
  volatile int* ring = reinterpret_cast<volatile int*>(gbase + S * STAGE + 8 * (2 * S + 4 + 2 * R));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * STAGE + 8 * (2 * S + 4 + 2 * R) + 4 * R);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);  // written by epilogue warps only
  float* wcol = reinterpret_cast<float*>(tmem_slot + 4);                     // [BN] routing weights (down)

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
      mbar_init(rempty(r), 5);  // the MMA issuer and the four epilogue warps
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

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_once = l2_policy_evict_first(), pol_shared = l2_policy_evict_normal();
      int issued = 0;  // K steps issued so far (all tiles)
      int tile = blockIdx.x;
      auto fail = [&]() {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      };
      for (int j = 0;; ++j) {
        const int slot = j % R;
        if (j >= R && !mbar_wait(rempty(slot), ((j / R) - 1) & 1)) {
          fail();
          break;
        }
        const int pub = (tile < total && !*abort_flag) ? tile : -1;
        ring[slot] = pub;
        mbar_arrive(rfull(slot));  // releases the ring entry to the MMA issuer and the epilogue
        if (pub < 0) break;
        const bool gu = tile < Gt;
        TileInfo ti;
        decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
        const int wi = tile_width_index(ti.nvalid, BN);
        const uint64_t pol_w = ti.nti > 1 ? pol_shared : pol_once;
        const MapEntry* me = a.maps + ti.mapi;
        bool ok = true;
        if (gu) {
          const void* wmap = &me->gu;
          const void* amap = &xact.m[wi];
          const uint32_t tx = 2 * kABytes + (16u << wi) * 128u;
          tensormap_acquire(wmap);
          for (int kb = 0; kb < KBg; ++kb, ++issued) {
            const int s = issued % S;
            if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
              ok = false;
              break;
            }
            const uint32_t st = base + s * STAGE;
            mbar_arrive_expect_tx(full(s), tx);
            tma_load_3d_hint(st, wmap, full(s), 0, ti.mt * 128, kb, pol_w);
            tma_load_3d_hint(st + kABytes, wmap, full(s), 0, a.I + ti.mt * 128, kb, pol_w);
            tma_load_3d(st + B_OFF, amap, full(s), 0, ti.row0, kb);
          }
        } else {
          const void* wmap = &me->dn2;
          const void* amap = &hact.m[wi];
          const uint32_t tx = 2 * kABytes + 2 * (16u << wi) * 128u;
          tensormap_acquire(wmap);
          // weights of the first stages first: they do not depend on h
          const int npre = KBd < S ? KBd : S;
          int kb = 0;
          for (; kb < npre; ++kb) {
            const int n = issued + kb, s = n % S;
            if (n >= S && !mbar_wait(empty(s), ((n / S) - 1) & 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full(s), tx);
            tma_load_3d_hint(base + s * STAGE, wmap, full(s), 0, ti.mt * 128, 2 * kb, pol_w);
          }
          if (ok) {
            // h rows of this N tile: written by the mg gate/up tiles of the same N tile
            const int* dep = a.sched + 1 + ti.ng;
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
            fence_proxy_async_global();  // the acquire above, before the TMA reads of h
            for (int j2 = 0; j2 < npre; ++j2) {
              const int s = (issued + j2) % S;
              tma_load_3d(base + s * STAGE + B_OFF, amap, full(s), 0, ti.row0, 2 * j2);
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
              tma_load_3d_hint(st, wmap, full(s), 0, ti.mt * 128, 2 * kb, pol_w);
              tma_load_3d(st + B_OFF, amap, full(s), 0, ti.row0, 2 * kb);
            }
          } else {
            issued += kb;  // the weight stages already armed (their copies are in flight)
          }
        }
        if (!ok) {
          fail();
          tile = total;  // publish the end marker next
          continue;
        }
        tile = (int)gridDim.x + atomicAdd(a.sched, 1);
      }
      // every copy this thread issued has landed before the CTA may exit
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
        const bool gu = tile < Gt;
        TileInfo ti;
        decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
        const int width = 16 << tile_width_index(ti.nvalid, BN);
        const uint32_t idesc = instr_desc(128, width, 1u);
        const int buf = j & 1;
        if (j >= 2 && !mbar_wait(tempty(buf), ((j >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + buf * ACC;
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
              tc_mma_bf16(d, sw128_kmajor_desc(st + k * 32), bdesc, idesc, acc);
              tc_mma_bf16(d + BN, sw128_kmajor_desc(st + kABytes + k * 32), bdesc, idesc, acc);
            }
          } else {
            const uint32_t chunk_b = (uint32_t)width * 128u;  // a 3-D box lands its K chunks densely
#pragma unroll
            for (int c = 0; c < 2; ++c) {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t bdesc = sw128_kmajor_desc(st + B_OFF + c * chunk_b + k * 32);
                const uint32_t acc = (kb | c | k) != 0 ? 1u : 0u;
                tc_mma_bf16(d, sw128_kmajor_desc(st + c * kABytes + k * 32), bdesc, idesc, acc);
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
      // the four warps take every decision together: lane 0 of each waits,
      // a failure is shared through ep_abort before anyone acts on it
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
      const bool gu = tile < Gt;
      TileInfo ti;
      decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
      if (!gu) {
        named_bar_sync(1, 128);  // previous tile's readers are done with wcol
        for (int n = r; n < BN; n += 128) {
          float wv = 0.0f;
          if (n < ti.nvalid) {
            const int p = ti.row0 + n;
            wv = __ldg(a.topk_w + (size_t)__ldg(a.perm_src + p) * a.K + __ldg(a.perm_k + p));
          }
          wcol[n] = wv;
        }
        named_bar_sync(1, 128);
      }
      const int buf = j & 1;
      if (lane == 0 && (*abort_flag || !mbar_wait(tfull(buf), (j >> 1) & 1))) *ep_abort = 1;
      named_bar_sync(2, 128);  // past this point no warp reads the abort flags until the next tile
      if (*ep_abort) {
        flag_status(a.status, MOE_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tl = tmem + buf * ACC + (static_cast<uint32_t>(warp * 32) << 16);
      {
        if (gu) {
          const int jj = ti.mt * 128 + r;
          __nv_bfloat16* hout = static_cast<__nv_bfloat16*>(a.h_out);
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t g[16], u[16];
            tmem_ld16(tl + c, g);
            tmem_ld16(tl + BN + c, u);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              if (c + q < ti.nvalid) {
                const float gv = __uint_as_float(g[q]);
                const float uv = __uint_as_float(u[q]);
                const float hv = gv / (1.0f + expf(-gv)) * uv;
                hout[(size_t)(ti.row0 + c + q) * a.I + jj] = __float2bfloat16_rn(hv);
              }
            }
          }
        } else {
          const int o = ti.mt * 128 + r;
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t v[16];
            tmem_ld16(tl + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              if (c + q < ti.nvalid) a.y_out[(size_t)(ti.row0 + c + q) * a.H + o] = wcol[c + q] * __uint_as_float(v[q]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(buf));
      if (gu) {
        // this tile's h rows are stored: count it for the down tiles of its N tile
        __threadfence();
        named_bar_sync(1, 128);
        if (r == 0) atomicAdd(a.sched + 1 + ti.ng, 1);
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

// ============================================================== fused fp8 decode
// FP8 counterpart of ffn_bf16_fused_kernel: gate/up and down tiles of one
// forward in one persistent launch with the same dynamic queue and per-N-tile
// dependency counters. The gate/up epilogue also does the activation
// quantisation of h: for each pair its 128 h values of the tile are one
// 128-column scale block, so amax (a max over the 4 row-quarter warps), the
// scale s = amax / 448 (1 for an all-zero block) and the e4m3 codes of the
// bf16-rounded h are formed right there, with the arithmetic of
// quant_rows_kernel, and written to hq and h_scale; the bf16 h is not stored.
// Per-K-block promotion as in ffn_fp8_kernel.

template <int BN>
struct Fp8FusedCfg {
  static constexpr uint32_t kStageBytes = 2 * kABytes + BN * 128;  // gate/up; down uses kABytes + BN * 128
  static constexpr int kMaxKB = 64;
  // activation scales [BN][64], weight scales [2][64], routing weights [BN], amax partials [4][BN]
  static constexpr uint32_t kScaleBytes = BN * kMaxKB * 4 + 2 * kMaxKB * 4 + BN * 4 + 4 * BN * 4;
  static constexpr int kStagesRaw = (212 * 1024 - (int)kScaleBytes) / (int)kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kRing = 8;
  static constexpr int kNpRaw = 512 / (2 * BN);
  static constexpr int NP = kNpRaw > 8 ? 8 : kNpRaw;
  static constexpr uint32_t kTmemCols = tmem_cols_for(NP * 2 * BN);
  static constexpr size_t kSmem =
      1024 + (size_t)kStages * kStageBytes + kScaleBytes + 8 * (2 * kStages + 2 * NP + 2 * kRing) + 4 * kRing + 64;
  static_assert(kStages >= 2 && NP >= 2, "FP8 pipeline needs two stages and two partial buffers");
};

template <int BN>
__global__ void __launch_bounds__(320, 1) ffn_fp8_fused_kernel(const __grid_constant__ ActMaps xact,
                                                               const __grid_constant__ ActMaps hact,
                                                               const GemmArgs a) {
  using C = Fp8FusedCfg<BN>;
  constexpr int S = C::kStages, NP = C::NP, R = C::kRing;
  constexpr uint32_t STAGE = C::kStageBytes;
  constexpr int HALF = BN / 2;
  constexpr int NCH = HALF >= 16 ? HALF / 16 : 1;
  constexpr int CW = HALF >= 16 ? 16 : HALF;
  const int mg = a.I / 128, md = a.H / 128;
  const int KBg = a.H / 128, KBd = a.I / 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  pdl_wait();  // the plan, the quantised x and the counters come from earlier kernels of the forward
  pdl_trigger();
  const int NT = a.nt_prefix[a.L];
  const int Gt = NT * mg, total = Gt + NT * md;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  float* s_act = reinterpret_cast<float*>(gbase + S * STAGE);  // [BN][KB]
  float* s_w = s_act + BN * C::kMaxKB;                         // [2][KB]
  float* wcol = s_w + 2 * C::kMaxKB;                           // [BN]
  float* s_amax = wcol + BN;                                   // [4][BN]
  const uint32_t bars = base + S * STAGE + C::kScaleBytes;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto pfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto pempty = [&](int b) { return bars + 8u * (2 * S + NP + b); };
  auto rfull = [&](int r) { return bars + 8u * (2 * S + 2 * NP + r); };
  auto rempty = [&](int r) { return bars + 8u * (2 * S + 2 * NP + R + r); };
  uint8_t* after = gbase + S * STAGE + C::kScaleBytes + 8 * (2 * S + 2 * NP + 2 * R);
  volatile int* ring = reinterpret_cast<volatile int*>(after);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(after + 4 * R);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* ep_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < NP; ++b) {
      mbar_init(pfull(b), 1);
      mbar_init(pempty(b), 8);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(rfull(r), 1);
      mbar_init(rempty(r), 9);  // the MMA issuer and the eight epilogue warps
    }
    *abort_flag = 0;
    *ep_abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_once = l2_policy_evict_first(), pol_shared = l2_policy_evict_normal();
      int issued = 0;
      int tile = blockIdx.x;
      auto fail = [&]() {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      };
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
        const bool gu = tile < Gt;
        TileInfo ti;
        decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
        const int wi = tile_width_index(ti.nvalid, BN);
        const uint64_t pol_w = ti.nti > 1 ? pol_shared : pol_once;
        const MapEntry* me = a.maps + ti.mapi;
        bool ok = true;
        if (gu) {
          const void* wmap = &me->gu;
          const void* amap = &xact.m[wi];
          const uint32_t tx = 2 * kABytes + (16u << wi) * 128u;
          tensormap_acquire(wmap);
          for (int kb = 0; kb < KBg; ++kb, ++issued) {
            const int s = issued % S;
            if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
              ok = false;
              break;
            }
            const uint32_t st = base + s * STAGE;
            mbar_arrive_expect_tx(full(s), tx);
            tma_load_2d_hint(st, wmap, full(s), kb * 128, ti.mt * 128, pol_w);
            tma_load_2d_hint(st + kABytes, wmap, full(s), kb * 128, a.I + ti.mt * 128, pol_w);
            tma_load_2d(st + 2 * kABytes, amap, full(s), kb * 128, ti.row0);
          }
        } else {
          const void* wmap = &me->dn;
          const void* amap = &hact.m[wi];
          const uint32_t tx = kABytes + (16u << wi) * 128u;
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
            tma_load_2d_hint(base + s * STAGE, wmap, full(s), kb * 128, ti.mt * 128, pol_w);
          }
          if (ok) {
            const int* dep = a.sched + 1 + ti.ng;
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
              tma_load_2d(base + s * STAGE + kABytes, amap, full(s), j2 * 128, ti.row0);
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
              tma_load_2d_hint(st, wmap, full(s), kb * 128, ti.mt * 128, pol_w);
              tma_load_2d(st + kABytes, amap, full(s), kb * 128, ti.row0);
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
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int consumed = 0, kp = 0;
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
        const bool gu = tile < Gt;
        TileInfo ti;
        decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
        const int width = 16 << tile_width_index(ti.nvalid, BN);
        const uint32_t idesc = instr_desc(128, width, 0u);
        const uint32_t b_off = gu ? 2 * kABytes : kABytes;
        const int KB = gu ? KBg : KBd;
        for (int kb = 0; kb < KB; ++kb, ++consumed, ++kp) {
          const int s = consumed % S, pb = kp % NP;
          ok = mbar_wait(full(s), (consumed / S) & 1);
          if (ok && kp >= NP) ok = mbar_wait(pempty(pb), ((kp / NP) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = base + s * STAGE;
          const uint32_t dd = tmem + static_cast<uint32_t>(pb * 2 * BN);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = sw128_kmajor_desc(st + b_off + k * 32);
            const uint32_t acc = k != 0 ? 1u : 0u;
            tc_mma_e4m3(dd, sw128_kmajor_desc(st + k * 32), bdesc, idesc, acc);
            if (gu) tc_mma_e4m3(dd + BN, sw128_kmajor_desc(st + kABytes + k * 32), bdesc, idesc, acc);
          }
          tc_commit(empty(s));
          tc_commit(pfull(pb));
        }
      }
      if (!ok) {
        *abort_flag = 1;
        flag_status(a.status, MOE_DEV_TIMEOUT);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0..7)
    // warp w owns TMEM lanes [32(w%4), +32) and columns [HALF*(w/4), +HALF)
    const int q4 = warp & 3, hf = warp >> 2;
    const int r = q4 * 32 + lane;
    const int et = threadIdx.x;  // 0..255
    const uint32_t tl = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int c0 = hf * HALF;
    bool aborted = false;  // warp-uniform
    int kp = 0;
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
      named_bar_sync(2, 256);  // the eight warps leave together or not at all
      if (*ep_abort) {
        flag_status(a.status, MOE_DEV_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      if (tile < 0) break;
      const bool gu = tile < Gt;
      TileInfo ti;
      decode_tile_at(a, gu ? mg : md, BN, gu ? tile : tile - Gt, ti);
      const int width = 16 << tile_width_index(ti.nvalid, BN);
      const int KB = gu ? KBg : KBd;
      const MapEntry* me = a.maps + ti.mapi;
      const float* sw = gu ? me->s_gu : me->s_dn;
      named_bar_sync(1, 256);  // the previous tile's readers are done with the tables
      if (!gu && et == 0) {
        // h scales of this N tile come from its gate/up tiles (the producer waited for their h codes)
        const int* dep = a.sched + 1 + ti.ng;
        const uint64_t t0 = global_timer_ns();
        while (ld_acquire_gpu(dep) < mg) {
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort_flag = 1;
            flag_status(a.status, MOE_DEV_TIMEOUT);
            break;
          }
          __nanosleep(64);
        }
      }
      named_bar_sync(1, 256);
      const float* act_scale = gu ? a.act_scale : a.h_scale;
      for (int i = et; i < BN * KB; i += 256) {  // through L2: h scales are written during this launch
        const int n = i / KB, kb = i - n * KB;
        s_act[n * KB + kb] = n < ti.nvalid ? __ldcg(act_scale + (size_t)(ti.row0 + n) * KB + kb) : 0.0f;
      }
      for (int i = et; i < (gu ? 2 : 1) * KB; i += 256) {
        const int which = i / KB, kb = i - which * KB;
        const int rb = which == 0 ? ti.mt : a.I / 128 + ti.mt;
        s_w[which * KB + kb] = sw[(size_t)rb * KB + kb];
      }
      if (!gu) {
        for (int n = et; n < BN; n += 256) {
          float wv = 0.0f;
          if (n < ti.nvalid) {
            const int p = ti.row0 + n;
            wv = __ldg(a.topk_w + (size_t)__ldg(a.perm_src + p) * a.K + __ldg(a.perm_k + p));
          }
          wcol[n] = wv;
        }
      }
      named_bar_sync(1, 256);

      float accg[HALF], accu[HALF];
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        accg[i] = 0.0f;
        accu[i] = 0.0f;
      }
      if constexpr (HALF <= 16) {
        // Narrow tiles (decode): each warp loads only its own HALF columns, for G K blocks at once, then
        // promotes them in K order; one TMEM round trip per G blocks instead of per block. A warp whose
        // columns are all past the tile's pairs loads nothing.
        constexpr int G = HALF <= 8 ? 4 : 2;
        const bool mine = c0 < ti.nvalid;  // warp-uniform
        for (int kb0 = 0; kb0 < KB; kb0 += G) {
          const int ng = KB - kb0 < G ? KB - kb0 : G;
          if (!aborted) {
            bool ok = !*abort_flag;
            for (int g = 0; g < ng && ok; ++g) ok = mbar_wait(pfull((kp + g) % NP), ((kp + g) / NP) & 1);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
              aborted = true;
              if (lane == 0) {
                *abort_flag = 1;
                flag_status(a.status, MOE_DEV_TIMEOUT);
              }
            }
          }
          if (!aborted && mine) {
            tc_fence_after();
            uint32_t pg[G][HALF], pu[G][HALF];
#pragma unroll
            for (int g = 0; g < G; ++g) {
              if (g < ng) {
                const uint32_t pbase = tl + static_cast<uint32_t>(((kp + g) % NP) * 2 * BN) + c0;
                if constexpr (HALF == 8) {
                  tmem_ld8(pbase, pg[g]);
                  if (gu) tmem_ld8(pbase + BN, pu[g]);
                } else {
                  tmem_ld16(pbase, pg[g]);
                  if (gu) tmem_ld16(pbase + BN, pu[g]);
                }
              }
            }
            tmem_wait_ld();
#pragma unroll
            for (int g = 0; g < G; ++g) {
              if (g < ng) {
                const int kb = kb0 + g;
                const float swg = s_w[kb];
                const float swu = gu ? s_w[KB + kb] : 0.0f;
#pragma unroll
                for (int q = 0; q < HALF; ++q) {
                  const float sa = s_act[(c0 + q) * KB + kb];
                  accg[q] = fmaf(__uint_as_float(pg[g][q]), sa * swg, accg[q]);
                  if (gu) accu[q] = fmaf(__uint_as_float(pu[g][q]), sa * swu, accu[q]);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0)
            for (int g = 0; g < ng; ++g) mbar_arrive(pempty((kp + g) % NP));
          kp += ng;
        }
      } else {
      for (int kb = 0; kb < KB; ++kb, ++kp) {
        const int pb = kp % NP;
        if (!aborted) {
          bool ok = !*abort_flag && mbar_wait(pfull(pb), (kp / NP) & 1);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) {
            aborted = true;
            if (lane == 0) {
              *abort_flag = 1;
              flag_status(a.status, MOE_DEV_TIMEOUT);
            }
          }
        }
        if (!aborted) {
          tc_fence_after();
          const float swg = s_w[kb];
          const float swu = gu ? s_w[KB + kb] : 0.0f;
          const uint32_t pbase = tl + static_cast<uint32_t>(pb * 2 * BN);
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const int cstart = CW == 16 ? c0 + ch * 16 : 0;
            if (cstart < width) {
              uint32_t pg[16], pu[16];
              tmem_ld16(pbase + cstart, pg);
              if (gu) tmem_ld16(pbase + BN + cstart, pu);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < CW; ++q) {
                const int col = ch * CW + q;
                const int n = c0 + col;
                const uint32_t gb = CW == 16 ? pg[q] : (hf ? pg[(CW + q) & 15] : pg[q]);
                const float sa = s_act[n * KB + kb];
                accg[col] = fmaf(__uint_as_float(gb), sa * swg, accg[col]);
                if (gu) {
                  const uint32_t ub = CW == 16 ? pu[q] : (hf ? pu[(CW + q) & 15] : pu[q]);
                  accu[col] = fmaf(__uint_as_float(ub), sa * swu, accu[col]);
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pempty(pb));
      }
      }
      if (gu) {
        // h = bf16(silu(g) * u), then its e4m3 block code: amax over the tile's 128 rows per pair
        const int jj = ti.mt * 128 + r;
        float hv[HALF];
#pragma unroll
        for (int col = 0; col < HALF; ++col) {
          const int n = c0 + col;
          float h = 0.0f;
          if (n < ti.nvalid) {
            const float gv = accg[col], uv = accu[col];
            h = __bfloat162float(__float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv));
          }
          hv[col] = h;
          float m = fabsf(h);
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) s_amax[q4 * BN + n] = m;
        }
        named_bar_sync(1, 256);
        uint8_t* hq = static_cast<uint8_t*>(a.h_out);
#pragma unroll
        for (int col = 0; col < HALF; ++col) {
          const int n = c0 + col;
          if (n < ti.nvalid && !aborted) {
            const float amax = fmaxf(fmaxf(s_amax[n], s_amax[BN + n]), fmaxf(s_amax[2 * BN + n], s_amax[3 * BN + n]));
            const float sc = (amax == 0.0f) ? 1.0f : amax / 448.0f;
            const int p = ti.row0 + n;
            hq[(size_t)p * a.I + jj] =
                static_cast<uint8_t>(__nv_cvt_float_to_fp8(hv[col] / sc, __NV_SATFINITE, __NV_E4M3));
            if (r == 0) a.h_scale[(size_t)p * KBd + ti.mt] = sc;
          }
        }
        __threadfence();
        named_bar_sync(1, 256);
        if (et == 0 && !*abort_flag) atomicAdd(a.sched + 1 + ti.ng, 1);
      } else if (!aborted) {
        const int o = ti.mt * 128 + r;
#pragma unroll
        for (int col = 0; col < HALF; ++col) {
          const int n = c0 + col;
          if (n < ti.nvalid) a.y_out[(size_t)(ti.row0 + n) * a.H + o] = wcol[n] * accg[col];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN>
static cudaError_t launch_fp8_fused(const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a, int grid,
                                    cudaStream_t s, bool pdl) {
  using C = Fp8FusedCfg<BN>;
  cudaError_t err = cudaFuncSetAttribute(ffn_fp8_fused_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmem);
  if (err != cudaSuccess) return err;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;
  if (persistent <= 0) return cudaSuccess;
  return launch_ex(ffn_fp8_fused_kernel<BN>, dim3(persistent), dim3(320), C::kSmem, s, pdl, xmaps, hmaps, a);
}

cudaError_t launch_ffn_fp8_fused(int bn, const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a,
                                 int max_tiles, cudaStream_t s, bool pdl) {
  switch (bn) {
    case 16: return launch_fp8_fused<16>(xmaps, hmaps, a, max_tiles, s, pdl);
    case 32: return launch_fp8_fused<32>(xmaps, hmaps, a, max_tiles, s, pdl);
    case 64: return launch_fp8_fused<64>(xmaps, hmaps, a, max_tiles, s, pdl);
  }
  return cudaErrorInvalidValue;
}

template <int BN>
static cudaError_t launch_fused(const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a, int grid,
                                cudaStream_t s, bool pdl) {
  using C = FusedCfg<BN>;
  cudaError_t err = cudaFuncSetAttribute(ffn_bf16_fused_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::smem());
  if (err != cudaSuccess) return err;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;
  if (persistent <= 0) return cudaSuccess;
  return launch_ex(ffn_bf16_fused_kernel<BN>, dim3(persistent), dim3(192), C::smem(), s, pdl, xmaps, hmaps, a);
}

cudaError_t launch_ffn_fused(int bn, const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a, int max_tiles,
                             cudaStream_t s, bool pdl) {
  switch (bn) {
    case 16: return launch_fused<16>(xmaps, hmaps, a, max_tiles, s, pdl);
    case 32: return launch_fused<32>(xmaps, hmaps, a, max_tiles, s, pdl);
    case 64: return launch_fused<64>(xmaps, hmaps, a, max_tiles, s, pdl);
  }
  return cudaErrorInvalidValue;
}

// ==================================================================== launch

template <typename Kern, typename MapT>
static cudaError_t launch_kernel(Kern kern, size_t smem, int threads, int grid, const MapT& map, const GemmArgs& a,
                                 cudaStream_t s, bool pdl) {
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (grid <= 0) return cudaSuccess;
  return launch_ex(kern, dim3(grid), dim3(threads), smem, s, pdl, map, a);
}

template <int MODE, int BN>
static cudaError_t launch_bf16(const ActMaps& maps, GemmArgs a, int grid, cudaStream_t s, bool pdl) {
  using C = Bf16Cfg<MODE, BN>;
  a.stages = C::kStagesMax;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;  // one CTA per SM walks the tiles
  return launch_kernel(ffn_bf16_kernel<MODE, BN>, C::smem(a.stages), 192, persistent, maps, a, s, pdl);
}

template <int MODE, int BN>
static cudaError_t launch_fp8(const ActMaps& maps, const GemmArgs& a, int grid, cudaStream_t s, bool pdl) {
  const int persistent = grid < a.num_sms ? grid : a.num_sms;  // one CTA per SM walks the tiles
  return launch_kernel(ffn_fp8_kernel<MODE, BN>, Fp8Cfg<MODE, BN>::kSmem, 32 * (Fp8Cfg<MODE, BN>::EW + 2), persistent,
                       maps, a, s, pdl);
}

template <int MODE>
static cudaError_t launch_mode(int wdtype, int bn, const CUtensorMap& map, const ActMaps* maps, const GemmArgs& a,
                               int grid, cudaStream_t s, bool pdl) {
  if (wdtype == MOE_BF16) {
    switch (bn) {
      case 16: return launch_bf16<MODE, 16>(*maps, a, grid, s, pdl);
      case 32: return launch_bf16<MODE, 32>(*maps, a, grid, s, pdl);
      case 64: return launch_bf16<MODE, 64>(*maps, a, grid, s, pdl);
      case 128: return launch_bf16<MODE, 128>(*maps, a, grid, s, pdl);
    }
  } else {
    switch (bn) {
      case 16: return launch_fp8<MODE, 16>(*maps, a, grid, s, pdl);
      case 32: return launch_fp8<MODE, 32>(*maps, a, grid, s, pdl);
      case 64: return launch_fp8<MODE, 64>(*maps, a, grid, s, pdl);
    }
  }
  return cudaErrorInvalidValue;
}

int ffn_block_n(int T, int wdtype) {
  // 128 at most: gate/up at 128 keeps two TMEM accumulators (the epilogue of
  // one tile overlaps the next tile's MMAs) and two stages of two 64-deep K
  // chunks; at 256 one accumulator leaves the epilogue exposed (measured 12%
  // slower on a 4096-token chunk).
  int bn = T <= 16 ? 16 : T <= 32 ? 32 : T <= 64 ? 64 : 128;
  if (wdtype == MOE_FP8_E4M3_B128 && bn > 64) bn = 64;
  if (wdtype == MOE_MXFP4 && bn > kMxfp4MaxBn) bn = kMxfp4MaxBn;
  return bn;
}


cudaError_t launch_ffn_gemm(int mode, int wdtype, int bn, const CUtensorMap& act_map, const ActMaps* act_maps,
                            const GemmArgs& a, int max_tiles, cudaStream_t s, bool pdl) {
  if (mode == kGateUp) return launch_mode<kGateUp>(wdtype, bn, act_map, act_maps, a, max_tiles, s, pdl);
  return launch_mode<kDown>(wdtype, bn, act_map, act_maps, a, max_tiles, s, pdl);
}

}  // namespace moe
