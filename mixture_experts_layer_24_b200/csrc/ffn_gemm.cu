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
// Warp roles of the GEMM (one CTA per SM, persistent over tiles):
//   warps 0..3: epilogue (TMEM -> registers -> global)
//   warp 4: TMA producer (one elected lane)
//   warp 5: TMEM allocator + MMA issuer of gate (or down); warp 6: MMA issuer
//   of up (one elected lane each; the fused kernels keep one issuer)
// Gate/up CTAs hold two accumulators, gate rows [j, j+128) and up rows
// [I+j, I+j+128), so one thread owns g and u of the same (j, pair) and SwiGLU
// happens in the epilogue without any exchange.
//
// FP8 weights: ffn_fp8.cu; MXFP4 weights: ffn_mxfp4.cu; the one-launch decode
// FFN: ffn_decode.cu.
#include "common.cuh"
#include "internal.h"
#include "tile.cuh"

namespace moe {

// bf16: one pipeline stage holds kKC consecutive 64-wide K chunks, fetched by
// one 3-D TMA copy per operand. NA weight operands share each staged
// activation tile, each with its own accumulator: gate/up stages the gate and
// up rows of the same 128 rows; down, up to BN = 128, stages two consecutive
// 128-row blocks of the output, so each h tile comes from L2 once per 256
// output rows (at BN = 256 one operand: two accumulators of 256 columns would
// not fit twice in TMEM). Two-operand stages hold one chunk, one-operand
// stages two (the depths measured fastest).
template <int MODE, int BN>
struct Bf16Cfg {
  static constexpr int KC = MODE == kGateUp ? kBf16GateUpChunks : bf16_down_gemm_chunks(BN);
  static constexpr int NA = (MODE == kGateUp || KC == 1) ? 2 : 1;
  static constexpr uint32_t kChunkA = kABytes;     // 128 rows x 128 B
  static constexpr uint32_t kChunkB = BN * 128;    // BN rows x 128 B
  static constexpr uint32_t kStageBytes = KC * (NA * kChunkA + kChunkB);
  // up to 220 KB of stages (227 KB per CTA at most; one CTA per SM)
  static constexpr int kStagesFit = (220 * 1024) / kStageBytes;
  static constexpr int kStagesMax = kStagesFit > 8 ? 8 : kStagesFit;
  // two accumulator buffers whenever both fit in TMEM's 512 columns
  static constexpr int NBUF = 2 * NA * BN <= 512 ? 2 : 1;
  static constexpr uint32_t kTmemCols = tmem_cols_for(NBUF * NA * BN);
  static constexpr size_t smem(int stages) { return 1024 + (size_t)stages * kStageBytes + 256 + 4 * BN; }
  static_assert(kStagesMax >= 2, "a pipeline needs two stages");
};

// ====================================================================== bf16
// Persistent: one CTA per SM walks tiles blockIdx.x, +gridDim.x, ... The
// shared-memory pipeline runs on across tile boundaries (stage and phase come
// from one running K-step count), and the accumulator lives in one of NBUF
// TMEM buffers so that the epilogue of tile j overlaps the MMAs of tile j+1.

template <int MODE, int BN>
__global__ void __launch_bounds__(224, 1) ffn_bf16_kernel(const __grid_constant__ ActMaps act,
                                                          const GemmArgs a) {
  using C = Bf16Cfg<MODE, BN>;
  constexpr int NA = C::NA, kKC = C::KC, NBUF = C::NBUF;
  constexpr uint32_t STAGE = C::kStageBytes;
  constexpr uint32_t A_OP = kKC * C::kChunkA;  // bytes of one A operand per stage
  constexpr uint32_t B_OFF = NA * A_OP;        // stage: [A gate][A up][B], kKC chunks each
  constexpr uint32_t ACC = NA * BN;            // TMEM columns of one accumulator buffer
  constexpr int S = C::kStagesMax;  // compile-time depth: no division by a launch value in the K loops
  // weight tiles of NA operands; with an odd number of 128-row blocks in H the last down tile's second block lies
  // past the weight rows: its TMA box reads the zero fill and its results are not stored
  const int m_tiles = MODE == kGateUp ? a.I / 128 : (a.H + 128 * NA - 1) / (128 * NA);
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
      mbar_init(empty(s), NA);  // one commit per MMA issuer
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), NA);
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
        // weight rows of the two operands: gate and up rows of the same 128 rows, or (down) two consecutive blocks
        const int ra0 = MODE == kGateUp ? ti.mt * 128 : ti.mt * 128 * NA;
        const int ra1 = MODE == kGateUp ? a.I + ti.mt * 128 : ra0 + 128;
        int kb = 0;
        if (first) {
          first = false;
          // the plan is complete: the first weight stages go out before waiting
          // for the kernel that writes the activations
          const int npre = a.plan_ready ? (KB < S ? KB : S) : 0;
          for (int j = 0; j < npre; ++j) {
            const uint32_t st = base + j * STAGE;
            mbar_arrive_expect_tx(full(j), stage_tx);
            tma_load_3d_hint(st, wmap, full(j), 0, ra0, j * kKC, pol_w);
            if (NA == 2) tma_load_3d_hint(st + A_OP, wmap, full(j), 0, ra1, j * kKC, pol_w);
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
          tma_load_3d_hint(st, wmap, full(s), 0, ra0, kb * kKC, pol_w);
          if (NA == 2) tma_load_3d_hint(st + A_OP, wmap, full(s), 0, ra1, kb * kKC, pol_w);
          tma_load_3d(st + B_OFF, amap, full(s), 0, ti.row0, kb * kKC);
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp == 5 || warp == 6) {
    // ------------------------------------------------------------ MMA issuers: warp 5 gate (or the first down
    // block), warp 6 up (or the second)
    // (each tcgen05 instruction holds its issuing thread for tens of cycles, about as long as a 128 x 128 x 16
    // MMA computes, so two threads issue the two accumulators' MMAs)
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    const int who = warp - 5;
    if (lane == 0 && who < NA) {
      int consumed = 0, j = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++j) {
        const int buf = j % NBUF;
        if (j >= NBUF && !mbar_wait(tempty(buf), ((j / NBUF) - 1) & 1)) {
          *abort_flag = 1;
          flag_status(a.status, MOE_DEV_TIMEOUT);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + buf * ACC + who * BN;
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
          const uint32_t st = base + s * STAGE + who * A_OP;
          const uint32_t sb = base + s * STAGE + B_OFF;
#pragma unroll
          for (int c = 0; c < kKC; ++c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t bdesc = sw128_kmajor_desc(sb + c * chunk_b + k * 32);
              const uint32_t acc = (kb | c | k) != 0 ? 1u : 0u;
              tc_mma_bf16(d, sw128_kmajor_desc(st + c * C::kChunkA + k * 32), bdesc, idesc, acc);
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
          const int o = ti.mt * 128 * NA + r;  // output column of accumulator 0; accumulator 1 is 128 further
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t v[16], v1[16];
            tmem_ld16(tl + c, v);
            if (NA == 2) tmem_ld16(tl + BN + c, v1);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              if (c + q < ti.nvalid) {
                float* yrow = a.y_out + (size_t)(ti.row0 + c + q) * a.H;
                yrow[o] = wcol[c + q] * __uint_as_float(v[q]);
                if (NA == 2 && o + 128 < a.H) yrow[o + 128] = wcol[c + q] * __uint_as_float(v1[q]);
              }
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
  return launch_kernel(ffn_bf16_kernel<MODE, BN>, C::smem(a.stages), 224, persistent, maps, a, s, pdl);
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
      case 256:
        if constexpr (MODE == kDown) return launch_bf16<MODE, 256>(*maps, a, grid, s, pdl);  // wide down tiles
        break;
    }
    return cudaErrorInvalidValue;
  }
  return launch_ffn_fp8(MODE, bn, *maps, a, grid, s, pdl);
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
