// ffn_mxfp4.cu -- the grouped expert FFN with MXFP4 weights on the block-scaled
// tensor cores (tcgen05.mma kind::mxf8f6f4.block_scale).
//
// The pages' checkpoint keeps its experts in FP4 (vLLM-Moet, topairepos.com
// page, hybrid results table, row "quality, paired against the native FP4
// reference"); read here as OCP MXFP4: E2M1 weights and MX e4m3 activations,
// one E8M0 scale per 32 K elements of each operand (mx.cu). Per pair:
//   gate/up: g, u = sum over 32-blocks b of 2^(sw_b + sx_b) * <w_b, x_b>;
//            h = bf16(silu(g) * u), then h quantised to MX e4m3 (per pair,
//            per 32 columns) for the down GEMM;
//   down:    y_pair = w[t,k] * sum_b 2^(sw_b + sh_b) * <w_b, h_b>.
// The tensor core applies both scales inside the MMA (the scale is a power of
// two, so each block's contribution is exact before accumulation) and keeps
// the whole sum in TMEM: unlike the FP8 path there is no promotion in
// registers.
//
// Same orientation and schedule as the bf16 GEMM (ffn_gemm.cu): swap-AB (128
// weight rows x BN pairs per tile), persistent CTAs over (expert, row tile,
// N tile), K blocks in increasing order, no split-K, per-tile MMA width
// 16..BN, two TMEM accumulators so one tile's epilogue overlaps the next
// tile's MMAs. One stage is kMxKC (2) consecutive 128-deep K blocks:
//   [A gate: KC x 16 KB][A up: KC x 16 KB (gate/up only)][B: KC x W x 128 B]
//   [scales A: KC x (gate 512 B, up 512 B)][scales B: KC x 512 B]
// fetched by five copies (four for down): one 3-D TMA copy per operand brings
// all KC blocks, and the weight scales of gate and up for KC blocks sit
// together in global memory (mx.cu), as do the activation scales, so one bulk
// copy each brings them (one K block and six copies per stage measured
// 2.5-3.1 TB/s; the copies alone, without the MMAs, stream these stages at
// 6.9-7.0 TB/s, so they are not the bound). A (E2M1) arrives in the tensor
// cores' unpacked layout (16 codes per 16 bytes, the 128-byte swizzle); HBM
// moves 4 bits per weight. Before the four 32-deep MMAs of each K block its
// scale blocks go to TMEM with tcgen05.cp (32x128b, copied to all four lane
// quarters); the MMAs read scale byte j = 0..3 of each row's word.
//
// What bounds it: a 32-deep MMA of this kind covers 16 bytes of E2M1 per
// weight row, half of what a bf16 or e4m3 MMA covers, so a stage of 32 KB of
// weights takes 16 MMAs and 6 scale copies, and each tcgen05 instruction
// held its issuing thread about 60 SM cycles whatever the MMA width (clock64
// stamps around the issue loop: 8 MMAs 470 cycles, 3 copies 160-200). Gate
// and up are therefore issued by two threads (warps 5 and 6), each with its
// own scale columns and its own commits (the stage and accumulator barriers
// count both); that measured 7-11% faster than one issuer.
//
// Warp roles: warps 0..3 epilogue (TMEM lane quarters), warp 4 TMA producer,
// warp 5 MMA issuer (gate, or down), warp 6 MMA issuer (up), warp 5 also
// allocates TMEM.
#include "common.cuh"
#include "internal.h"
#include "tile.cuh"

namespace moe {

namespace {

// D[tmem] (+)= (A * 2^sfa) (B * 2^sfb)^T over 32 K: A E2M1, B E4M3, E8M0 scales in TMEM.
__device__ __forceinline__ void tc_mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 lanes x 16 bytes of shared memory (one 512-byte scale block) to TMEM
// columns [taddr, taddr + 4) of all 128 lanes (each lane quarter gets a copy).
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a 512-byte scale block: K-major, no swizzle,
// 16-byte rows, 8-row core matrices 128 bytes apart (stride byte offset),
// descriptor version 1.
__device__ __forceinline__ uint64_t sf_block_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46);
}

// Instruction descriptor of the block-scaled MMA: A E2M1 (5), B E4M3 (0),
// K-major both, E8M0 scales (bit 23), M = 128, N = n, scale byte sf_id of
// both operands' TMEM words.
__device__ __forceinline__ uint32_t mx_instr_desc(int n, uint32_t sf_id) {
  return (sf_id << 4) | (5u << 7) | (0u << 10) | (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(128 >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ int mx_scale_exp8(float amax) {
  if (amax == 0.0f) return -127;
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xffu);
  const int fl = ex ? ex - 127 : (31 - __clz((int)(b & 0x7fffffu))) - 149;
  const int s = fl - 8;  // E4M3: emax 8
  return s < -127 ? -127 : (s > 127 ? 127 : s);
}

}  // namespace

template <int MODE, int BN>
struct MxCfg {
  static constexpr int NA = MODE == kGateUp ? 2 : 1;
  static constexpr int KC = kMxKC;
  static constexpr uint32_t kAOp = KC * kABytes;           // KC blocks of 128 rows x 128 K, unpacked E2M1
  static constexpr uint32_t kBOff = NA * kAOp;
  static constexpr uint32_t kSfOff = kBOff + KC * BN * 128;  // weight scales (KC x NA blocks), then activation
  static constexpr uint32_t kSfBOff = kSfOff + KC * NA * 512;
  static constexpr uint32_t kStageRaw = kSfBOff + KC * 512;
  static constexpr uint32_t kStageBytes = (kStageRaw + 1023u) & ~1023u;  // next stage's A stays 1024-aligned
  static constexpr int kStagesFit = (220 * 1024) / kStageBytes;
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  // two accumulator buffers (the epilogue of one tile overlaps the next tile's MMAs) while they and the scale
  // columns fit TMEM's 512 columns: every width but gate/up at 128, which is why gate/up stays at 64 or less
  static constexpr int NBUF = 2 * NA * BN + 8 * NA <= 512 ? 2 : 1;
  static constexpr uint32_t kAcc = NA * BN;                 // TMEM columns of one accumulator buffer
  static constexpr uint32_t kSfCol = NBUF * kAcc;           // scale columns after the accumulators:
  static constexpr uint32_t kTmemCols = tmem_cols_for(kSfCol + 8 * NA);  // per issuer 4 weight + 4 activation
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + 256 + 4 * BN;
  static_assert(kStages >= 2, "a pipeline needs two stages");
  static_assert(NBUF * NA * BN + 8 * NA <= 512, "accumulators plus scale columns in 512 TMEM columns");
};

template <int MODE, int BN>
__global__ void __launch_bounds__(224, 1) ffn_mxfp4_kernel(const __grid_constant__ ActMaps act, const GemmArgs a) {
  using C = MxCfg<MODE, BN>;
  constexpr int NA = C::NA, NBUF = C::NBUF, S = C::kStages;
  constexpr uint32_t STAGE = C::kStageBytes, ACC = C::kAcc;
  constexpr int KC = C::KC;
  const int m_tiles = (MODE == kGateUp ? a.I : a.H) / 128;
  const int Kdim = MODE == kGateUp ? a.H : a.I;
  const int KB = Kdim / 128;  // 128-deep K blocks per tile
  const int KS = KB / KC;     // stages per tile
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
  volatile int* ep_abort = reinterpret_cast<volatile int*>(tmem_slot + 2);
  float* wcol = reinterpret_cast<float*>(tmem_slot + 4);  // [BN] routing weights of the tile's pairs (down)

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), NA);
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
      // weights: evict-first when the tile is its weight rows' only reader
      const uint64_t pol_once = l2_policy_evict_first(), pol_shared = l2_policy_evict_normal();
      int issued = 0;
      bool first = true;
      for (int tile = blockIdx.x; tile < total && !*abort_flag; tile += gridDim.x) {
        TileInfo ti;
        decode_tile_at(a, m_tiles, BN, tile, ti);
        const int wi = tile_width_index(ti.nvalid, BN);
        const void* amap = &act.m[wi];
        // per stage: KC blocks of A (128 x 128 x 4 bits each), of B and of the scales
        const uint32_t stage_tx = KC * (NA * 8192u + (16u << wi) * 128u + NA * 512u + 512u);
        const uint64_t pol_w = ti.nti > 1 ? pol_shared : pol_once;
        const MapEntry* me = a.maps + ti.mapi;
        const void* wmap = MODE == kGateUp ? static_cast<const void*>(&me->gu) : static_cast<const void*>(&me->dn);
        // weight scales: [m tile][K block][NA][512] (gate and up of a K block side by side)
        const uint8_t* sfa = reinterpret_cast<const uint8_t*>(MODE == kGateUp ? me->s_gu : me->s_dn) +
                             (size_t)ti.mt * KB * NA * 512;
        const uint8_t* sfb = a.act_sfb + (size_t)ti.ng * KB * 512;
        tensormap_acquire(wmap);
        auto issue_w = [&](uint32_t st, int ks) {
          tma_load_3d_hint(st, wmap, full(issued % S), 0, ti.mt * 128, ks * KC, pol_w);
          if (MODE == kGateUp) tma_load_3d_hint(st + C::kAOp, wmap, full(issued % S), 0, a.I + ti.mt * 128, ks * KC, pol_w);
          bulk_load(st + C::kSfOff, sfa + (size_t)ks * KC * NA * 512, KC * NA * 512, full(issued % S));
        };
        auto issue_x = [&](uint32_t st, int ks, uint32_t bar) {
          tma_load_3d(st + C::kBOff, amap, bar, 0, ti.row0, ks * KC);
          bulk_load(st + C::kSfBOff, sfb + (size_t)ks * KC * 512, KC * 512, bar);
        };
        int ks = 0;
        if (first) {
          first = false;
          // the plan is complete: the first stages' weights and weight scales go out before waiting for the
          // kernel that writes the activations and their scales
          const int npre = a.plan_ready ? (KS < S ? KS : S) : 0;
          for (int j = 0; j < npre; ++j, ++issued) {
            mbar_arrive_expect_tx(full(j), stage_tx);
            issue_w(base + j * STAGE, j);
          }
          if (a.plan_ready) {
            pdl_wait();
            pdl_trigger();
          }
          for (int j = 0; j < npre; ++j) issue_x(base + j * STAGE, j, full(j));
          ks = npre;
        }
        for (; ks < KS; ++ks, ++issued) {
          const int s = issued % S;
          if (issued >= S && !mbar_wait(empty(s), ((issued / S) - 1) & 1)) {
            *abort_flag = 1;
            flag_status(a.status, MOE_DEV_TIMEOUT);
            break;
          }
          const uint32_t st = base + s * STAGE;
          mbar_arrive_expect_tx(full(s), stage_tx);
          issue_w(st, ks);
          issue_x(st, ks, full(s));
        }
      }
      // every copy this thread issued has landed before the CTA may exit
      for (int g = issued - S < 0 ? 0 : issued - S; g < issued; ++g) mbar_wait(full(g % S), (g / S) & 1);
    } else if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
  } else if (warp == 5 || warp == 6) {
    // ------------------------------------------------------------ MMA issuers: warp 5 gate (or down), warp 6 up
    if (a.plan_ready) {
      pdl_wait();
      pdl_trigger();
    }
    const int who = warp - 5;
    if (lane == 0 && who < NA) {
      const uint32_t sf_a = tmem + C::kSfCol + 8 * who, sf_b = sf_a + 4;
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
        bool ok = true;
        const uint32_t chunk_b = (uint32_t)width * 128u;
        for (int ks = 0; ks < KS; ++ks, ++consumed) {
          const int s = consumed % S;
          if (!mbar_wait(full(s), (consumed / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * STAGE;
#pragma unroll
          for (int c = 0; c < KC; ++c) {
            tc_cp_sf(sf_a, sf_block_desc(st + C::kSfOff + c * NA * 512 + who * 512));
            tc_cp_sf(sf_b, sf_block_desc(st + C::kSfBOff + c * 512));
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
              const uint32_t idesc = mx_instr_desc(width, k);
              const uint64_t bdesc = sw128_kmajor_desc(st + C::kBOff + c * chunk_b + k * 32);
              const uint32_t acc = (ks | c | (int)k) != 0 ? 1u : 0u;
              tc_mma_mx(d, sw128_kmajor_desc(st + who * C::kAOp + c * kABytes + k * 32), bdesc, idesc,
                        sf_a | (k << 30), sf_b | (k << 30), acc);
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
          // h column jj of each pair, then MX e4m3 per 32 columns: the warp's 32 lanes are one block
          const int jj = ti.mt * 128 + r;
          uint8_t* hq = static_cast<uint8_t*>(a.h_out);
          const int KBd = a.I / 128;
          // h's scale blocks are laid out in the down GEMM's N tiles (width a.h_bn, a multiple of BN): pair
          // `local` of the expert is row local % h_bn of block (N tile, K block mt); scale byte = warp
          const int local0 = ti.row0 - a.offsets[ti.e];
          const int ngd = a.h_nt_prefix[ti.li] + local0 / a.h_bn, n0d = local0 % a.h_bn;
          uint8_t* hs = a.h_sfb + ((size_t)ngd * KBd + ti.mt) * 512 + warp;
#pragma unroll 1
          for (int c = 0; c < BN; c += 16) {
            if (c >= ti.nvalid) break;
            uint32_t g[16], u[16];
            tmem_ld16(tl + c, g);
            tmem_ld16(tl + BN + c, u);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int n = c + q;
              if (n < ti.nvalid) {  // warp-uniform
                const float gv = __uint_as_float(g[q]);
                const float uv = __uint_as_float(u[q]);
                const float hv = __bfloat162float(__float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv));
                float amax = fabsf(hv);
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                const int sexp = mx_scale_exp8(amax);
                const float inv = __int_as_float((127 - sexp) << 23);
                hq[(size_t)(ti.row0 + n) * a.I + jj] =
                    static_cast<uint8_t>(__nv_cvt_float_to_fp8(hv * inv, __NV_SATFINITE, __NV_E4M3));
                if (lane == 0) hs[16 * ((n0d + n) % 32) + 4 * ((n0d + n) / 32)] = static_cast<uint8_t>(sexp + 127);
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

template <int MODE, int BN>
static cudaError_t launch_mx(const ActMaps& maps, const GemmArgs& a, int grid, cudaStream_t s, bool pdl) {
  using C = MxCfg<MODE, BN>;
  auto kern = ffn_mxfp4_kernel<MODE, BN>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
  if (err != cudaSuccess) return err;
  if (grid <= 0) return cudaSuccess;
  const int persistent = grid < a.num_sms ? grid : a.num_sms;  // one CTA per SM walks the tiles
  return launch_ex(kern, dim3(persistent), dim3(224), C::kSmem, s, pdl, maps, a);
}

cudaError_t launch_ffn_mxfp4(int mode, int bn, const ActMaps& act_maps, const GemmArgs& a, int max_tiles,
                             cudaStream_t s, bool pdl) {
  if (mode == kGateUp) {
    switch (bn) {
      case 16: return launch_mx<kGateUp, 16>(act_maps, a, max_tiles, s, pdl);
      case 32: return launch_mx<kGateUp, 32>(act_maps, a, max_tiles, s, pdl);
      case 64: return launch_mx<kGateUp, 64>(act_maps, a, max_tiles, s, pdl);
    }
  } else {
    switch (bn) {
      case 16: return launch_mx<kDown, 16>(act_maps, a, max_tiles, s, pdl);
      case 32: return launch_mx<kDown, 32>(act_maps, a, max_tiles, s, pdl);
      case 64: return launch_mx<kDown, 64>(act_maps, a, max_tiles, s, pdl);
      case 128: return launch_mx<kDown, 128>(act_maps, a, max_tiles, s, pdl);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
