// ffn_fp8.cu -- the grouped expert FFN with FP8 weights (e4m3, one fp32 scale
// per 128 x 128 weight block and per 1 x 128 activation block) on the
// tensor cores (tcgen05.mma kind::f8f6f4).
//
// Same per-pair computation, orientation (swap-AB: 128 weight rows x BN pairs
// per tile), persistent schedule and K order as the bf16 GEMM (ffn_gemm.cu).
// One stage is one 128-wide K block, which is one scale block of both
// operands. The MMA writes each block's partial sum P_kb into one of NP TMEM
// buffers; the epilogue promotes it in fp32 registers,
//   acc = fmaf(P_kb, s_act[pair, kb] * s_w[rowblock, kb], acc),
// K blocks in increasing order (DeepSeek-V3-style fine-grained FP8; the
// pages' model table lists DeepSeek-class layers).
//
// Warp roles: warps 0..7 epilogue (4 TMEM lane quarters x 2 column groups),
// warp 8 TMA producer, warp 9 TMEM allocator + MMA issuer.
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "tile.cuh"

namespace moe {

// One TMEM load of N consecutive fp32 columns of the thread's own lane (N = 8, 16 or 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 32) tmem_ld32(taddr, r);
  else if constexpr (N == 16) tmem_ld16(taddr, r);
  else tmem_ld8(taddr, r);
}

template <int MODE, int BN>
struct Fp8Cfg {
  static constexpr int NA = MODE == kGateUp ? 2 : 1;
  static constexpr uint32_t kStageBytes = NA * kABytes + BN * 128;  // one 128-wide K block
  static constexpr int kMaxKB = 64;                                   // K / 128 <= 64 (K <= 8192)
  // per tile: the combined scales s_act[pair, kb] * s_w[row block, kb] as [NA][KB][BN] (a warp's columns of one
  // K block are consecutive, so they load as 16-byte vectors), then the routing weights [BN]
  __host__ __device__ static constexpr uint32_t scale_bytes(int KB) { return (uint32_t)(NA * KB * BN * 4 + BN * 4); }
  static int stages(int KB) {
    const int s = (int)((220 * 1024 - scale_bytes(KB)) / kStageBytes);
    return s > 8 ? 8 : s;
  }
  // TMEM buffers of per-K-block partial sums (the MMA runs up to NP blocks ahead of the promotion)
  static constexpr int kNpRaw = 512 / (NA * BN);
  static constexpr int NP = kNpRaw > 8 ? 8 : kNpRaw;
  static constexpr uint32_t kTmemCols = tmem_cols_for(NP * NA * BN);
  static size_t smem(int KB) { return 1024 + stages(KB) * kStageBytes + scale_bytes(KB) + 8 * (2 * stages(KB) + 2 * NP) + 64; }
  // epilogue warps (4 TMEM lane quarters x EW/4 column groups); 16 at BN = 64
  // measured no faster than 8
  static constexpr int EW = 8;
  static constexpr int kThreads = 32 * (EW + 1 + NA);  // + producer + one MMA issuer per accumulator
  static constexpr int HALF = BN * 4 / EW;             // columns per epilogue warp: 8, 16 or 32
  static_assert(NP >= 2, "FP8 pipeline needs two partial buffers");
};

// ======================================================================= fp8
// Persistent, like the bf16 kernel: one CTA per SM walks tiles blockIdx.x,
// +gridDim.x, ...; the shared-memory pipeline and a ring of NP TMEM buffers
// for the per-K-block partial sums run on across tile boundaries. Per tile the
// epilogue warps build the tile's table of combined scales s_act * s_w (and,
// for down, the routing weights) in shared memory, then promote every K
// block's partial sum in registers, K blocks in increasing order: one TMEM
// load of the warp's columns per operand, one wait, then per column one fma
// with the table's scale (the same fp32 product the promotion always used,
// so the results do not change). Gate and up MMAs are issued by two threads
// (warps EW+1 and EW+2), each committing to the stage and partial barriers
// (which count both): every tcgen05 instruction holds its issuing thread for
// tens of cycles, and at BN = 64 the eight MMAs of a K block took about as
// long to issue as the promotion took. The MMA width adapts per tile
// (16 .. BN). After a failed (timed-out) wait a warp stops working but keeps
// its control flow, so the epilogue warps always meet at the same named
// barriers.

template <int MODE, int BN>
__global__ void __launch_bounds__(Fp8Cfg<MODE, BN>::kThreads, 1)
    ffn_fp8_kernel(const __grid_constant__ ActMaps act, const GemmArgs a) {
  using C = Fp8Cfg<MODE, BN>;
  constexpr int NA = C::NA, NP = C::NP;
  constexpr uint32_t STAGE = C::kStageBytes;
  constexpr int EW = C::EW;            // epilogue warps: 4 TMEM lane quarters x EW/4 column groups
  constexpr int EPT = 32 * EW;         // epilogue threads
  constexpr int PW = EW, MW = EW + 1;  // producer warp, first MMA warp
  constexpr int HALF = C::HALF;        // columns per epilogue warp

  const int m_tiles = (MODE == kGateUp ? a.I : a.H) / 128;
  const int KD = MODE == kGateUp ? a.H : a.I;  // reduction length
  const int KB = KD / 128;
  const int S = a.stages;
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
  float* cs = reinterpret_cast<float*>(gbase + S * STAGE);  // [NA][KB][BN] combined scales of the tile
  float* wcol = cs + NA * KB * BN;                          // [BN] routing weights (down)
  const uint32_t bars = base + S * STAGE + C::scale_bytes(KB);  // full[S], empty[S], pfull[NP], pempty[NP]
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (S + s); };
  auto pfull = [&](int b) { return bars + 8u * (2 * S + b); };
  auto pempty = [&](int b) { return bars + 8u * (2 * S + NP + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + S * STAGE + C::scale_bytes(KB) + 8 * (2 * S + 2 * NP));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), NA);
    }
    for (int b = 0; b < NP; ++b) {
      mbar_init(pfull(b), NA);
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
      int issued = 0, ps = 0;
      uint32_t pphase = 0;
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
          ps = npre == S ? 0 : npre;
          pphase = npre == S ? 1u : 0u;
        }
        for (; kb < KB; ++kb, ++issued) {
          // slot ps = issued % S; its previous fill was round issued / S - 1 (S is a launch value: running
          // counters instead of divisions)
          if (issued >= S && !mbar_wait(empty(ps), pphase ^ 1u)) {
            *abort_flag = 1;
            flag_status(a.status, MOE_DEV_TIMEOUT);
            break;
          }
          const uint32_t st = base + ps * STAGE;
          mbar_arrive_expect_tx(full(ps), stage_tx);
          tma_load_2d_hint(st, wmap, full(ps), kb * 128, ti.mt * 128, pol_w);
          if (MODE == kGateUp) tma_load_2d_hint(st + kABytes, wmap, full(ps), kb * 128, a.I + ti.mt * 128, pol_w);
          tma_load_2d(st + NA * kABytes, amap, full(ps), kb * 128, ti.row0);
          if (++ps == S) {
            ps = 0;
            pphase ^= 1u;
          }
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp >= MW) {
    // ------------------------------------------------------------ MMA issuers (gate or down; up)
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    const int who = warp - MW;
    if (lane == 0 && who < NA) {
      int cslot = 0, kp = 0;  // consumed stage slot (running), K blocks consumed
      uint32_t cphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int width = 16 << tile_width_index(ti.nvalid, BN);
        const uint32_t idesc = instr_desc(128, width, 0u);
        for (int kb = 0; kb < KB; ++kb, ++kp) {
          const int pb = kp % NP;
          ok = mbar_wait(full(cslot), cphase);
          if (ok && kp >= NP) ok = mbar_wait(pempty(pb), ((kp / NP) - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = base + cslot * STAGE;
          const int s = cslot;
          if (++cslot == S) {
            cslot = 0;
            cphase ^= 1u;
          }
          const uint32_t d = tmem + static_cast<uint32_t>(pb * NA * BN + who * BN);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t bdesc = sw128_kmajor_desc(st + NA * kABytes + k * 32);
            tc_mma_e4m3(d, sw128_kmajor_desc(st + who * kABytes + k * 32), bdesc, idesc, k != 0 ? 1u : 0u);
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
      named_bar_sync(1, EPT);  // the previous tile's readers are done with the tables
      // combined scales [which][kb][n] of the tile's pairs, n fastest (each pair's row of activation scales
      // stays in L1); columns n >= nvalid keep stale values: their sums are never stored
      const int nv = ti.nvalid;
      for (int i = et; i < NA * KB * nv; i += EPT) {
        const int n = i % nv, t = i / nv;
        const int kb = t % KB, which = t / KB;
        const int rb = which == 0 ? ti.mt : a.I / 128 + ti.mt;  // gate (or down) row block, then up
        cs[(which * KB + kb) * BN + n] =
            __ldg(a.act_scale + (size_t)(ti.row0 + n) * KB + kb) * __ldg(sw + (size_t)rb * KB + kb);
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
      const bool live = c0 < width;  // warp-uniform: the MMA wrote this warp's columns
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
        if (!aborted && live) {
          tc_fence_after();
          const uint32_t pbase = tl + static_cast<uint32_t>(pb * NA * BN + c0);
          // NC columns from c0: all HALF, or 16 when the MMA width leaves no more for this warp
          auto promote = [&](auto nc) {
            constexpr int NC = decltype(nc)::value;
            uint32_t pg[NC];
            [[maybe_unused]] uint32_t pu[MODE == kGateUp ? NC : 1];
            tmem_ld_cols<NC>(pbase, pg);
            if constexpr (MODE == kGateUp) tmem_ld_cols<NC>(pbase + BN, pu);
            tmem_wait_ld();
            const float4* cg = reinterpret_cast<const float4*>(cs + kb * BN + c0);
#pragma unroll
            for (int q = 0; q < NC / 4; ++q) {
              const float4 g4 = cg[q];
              accg[4 * q + 0] = fmaf(__uint_as_float(pg[4 * q + 0]), g4.x, accg[4 * q + 0]);
              accg[4 * q + 1] = fmaf(__uint_as_float(pg[4 * q + 1]), g4.y, accg[4 * q + 1]);
              accg[4 * q + 2] = fmaf(__uint_as_float(pg[4 * q + 2]), g4.z, accg[4 * q + 2]);
              accg[4 * q + 3] = fmaf(__uint_as_float(pg[4 * q + 3]), g4.w, accg[4 * q + 3]);
            }
            if constexpr (MODE == kGateUp) {
              const float4* cu = reinterpret_cast<const float4*>(cs + (KB + kb) * BN + c0);
#pragma unroll
              for (int q = 0; q < NC / 4; ++q) {
                const float4 u4 = cu[q];
                accu[4 * q + 0] = fmaf(__uint_as_float(pu[4 * q + 0]), u4.x, accu[4 * q + 0]);
                accu[4 * q + 1] = fmaf(__uint_as_float(pu[4 * q + 1]), u4.y, accu[4 * q + 1]);
                accu[4 * q + 2] = fmaf(__uint_as_float(pu[4 * q + 2]), u4.z, accu[4 * q + 2]);
                accu[4 * q + 3] = fmaf(__uint_as_float(pu[4 * q + 3]), u4.w, accu[4 * q + 3]);
              }
            }
          };
          if constexpr (HALF == 32) {
            if (width - c0 <= 16) promote(std::integral_constant<int, 16>{});
            else promote(std::integral_constant<int, 32>{});
          } else {
            promote(std::integral_constant<int, HALF>{});
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pempty(pb));
      }
      if (!aborted && live) {
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

  // The plan and the counters come from a kernel two or more launches back when a.plan_ready is set (the
  // quantised x from the one just before): then the first weight stages go out before the programmatic wait.
  if (!a.plan_ready) {
    pdl_wait();
    pdl_trigger();
  }
  const int NT = a.nt_prefix[a.L];
  const int Gt = NT * mg, total = Gt + NT * md;
  const bool stand_down = a.status && (*reinterpret_cast<volatile int*>(a.status) & MOE_DEV_TIMEOUT);
  if ((int)blockIdx.x >= total || stand_down) {
    if (a.plan_ready) pdl_wait();
    return;
  }

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
      bool waited = !a.plan_ready;  // programmatic wait done
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
          int kb = 0;
          if (!waited) {
            // first tile: its weight stages before the wait, x (from the previous kernel) after it
            const int npre = KBg < S ? KBg : S;
            for (; kb < npre; ++kb) {
              const uint32_t st = base + kb * STAGE;
              mbar_arrive_expect_tx(full(kb), tx);
              tma_load_2d_hint(st, wmap, full(kb), kb * 128, ti.mt * 128, pol_w);
              tma_load_2d_hint(st + kABytes, wmap, full(kb), kb * 128, a.I + ti.mt * 128, pol_w);
            }
            pdl_wait();
            pdl_trigger();
            waited = true;
            for (int q = 0; q < npre; ++q) tma_load_2d(base + q * STAGE + 2 * kABytes, amap, full(q), q * 128, ti.row0);
            issued = npre;
          }
          for (; kb < KBg; ++kb, ++issued) {
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
          if (!waited) {
            pdl_wait();
            pdl_trigger();
            waited = true;
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
      if (!waited) {
        pdl_wait();
        pdl_trigger();
      }
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
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
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
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

// ==================================================================== launch

template <int MODE, int BN>
static cudaError_t launch_fp8(const ActMaps& maps, GemmArgs a, int grid, cudaStream_t s, bool pdl) {
  using C = Fp8Cfg<MODE, BN>;
  const int KB = (MODE == kGateUp ? a.H : a.I) / 128;
  if (KB > C::kMaxKB || C::stages(KB) < 2) return cudaErrorInvalidValue;
  a.stages = C::stages(KB);
  const size_t smem = C::smem(KB);
  auto kern = ffn_fp8_kernel<MODE, BN>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;  // one CTA per SM walks the tiles
  if (persistent <= 0) return cudaSuccess;
  return launch_ex(kern, dim3(persistent), dim3(C::kThreads), smem, s, pdl, maps, a);
}

cudaError_t launch_ffn_fp8(int mode, int bn, const ActMaps& maps, const GemmArgs& a, int max_tiles, cudaStream_t s,
                           bool pdl) {
  if (mode == kGateUp) {
    switch (bn) {
      case 16: return launch_fp8<kGateUp, 16>(maps, a, max_tiles, s, pdl);
      case 32: return launch_fp8<kGateUp, 32>(maps, a, max_tiles, s, pdl);
      case 64: return launch_fp8<kGateUp, 64>(maps, a, max_tiles, s, pdl);
    }
  } else {
    switch (bn) {
      case 16: return launch_fp8<kDown, 16>(maps, a, max_tiles, s, pdl);
      case 32: return launch_fp8<kDown, 32>(maps, a, max_tiles, s, pdl);
      case 64: return launch_fp8<kDown, 64>(maps, a, max_tiles, s, pdl);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
