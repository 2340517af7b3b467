// api.cu -- the C ABI of libmoe: context, workspace layout, the expert-slot
// table (residency + cold-expert staging), and the entry points that chain
// the kernels of route.cu, permute.cu, ffn_gemm.cu, quant.cu and combine.cu.
//
// Residency follows the "hotsplit" recipes wiki (Home page): hot experts stay
// in HBM, cold experts live in pinned host memory and are brought in on
// demand. Here a cold expert routed to by the batch is copied by the copy
// engine into a spare HBM slot and computed by the SAME kernels, tile shapes
// and K order as a resident one, so outputs are bit-identical to the
// all-resident run (vLLM-Moet, topairepos.com page, hybrid results table,
// row "identity").
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe.h"
#include "internal.h"

using namespace moe;

namespace moe {
// debug.cu: the bounded-wait test hook behind moe_debug_wait_flag
cudaError_t launch_debug_wait_flag(const int* flag, uint64_t limit_ns, int* status, cudaStream_t s);
}  // namespace moe

namespace {

thread_local std::string g_last_error;

moe_status_t fail(moe_status_t st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

#define MOE_CUDA(call)                                                                              \
  do {                                                                                              \
    cudaError_t err_ = (call);                                                                      \
    if (err_ != cudaSuccess)                                                                        \
      return fail(MOE_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(err_));             \
  } while (0)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

void moe::record_error(const char* msg) { g_last_error = msg ? msg : ""; }

struct moe_ctx {
  moe_config_t cfg;
  int device = 0;
  int* d_status = nullptr;
  int num_sms = 148;
  bool chain = true;  // programmatic dependent launch between this library's kernels
  unsigned int* d_counters = nullptr;  // arrival counters of the decode router (self-resetting)
  int host_status = 0;
  EncodeTiledFn encode = nullptr;
  std::atomic<int64_t> launches{0};
  // kernel timing (moe_profile_*)
  bool prof_on = false;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Rec> prof_pending;
  std::vector<cudaEvent_t> ev_pool;
  double prof_ms[MOE_PROF_KINDS] = {};
  int64_t prof_n[MOE_PROF_KINDS] = {};
  std::mutex prof_mu;

  cudaEvent_t take_event() {
    if (!ev_pool.empty()) {
      cudaEvent_t e = ev_pool.back();
      ev_pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};

namespace {
// Step names of the MOE_PROF_* kinds, for the NVTX ranges below.
static const char* const kStepNames[MOE_PROF_KINDS] = {"moe.router",  "moe.topk", "moe.permute",
                                                       "moe.gather",  "moe.gate_up", "moe.down",
                                                       "moe.quant",   "moe.combine", "moe.ffn_fused"};

// Counts one kernel launch, names it with an NVTX range on the host timeline
// (free unless a profiler is attached), and, when timing is on, brackets it
// with events on the launching stream.
struct Prof {
  moe_ctx* c;
  int kind;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  Prof(moe_ctx* c_, int kind_, cudaStream_t s_) : c(c_), kind(kind_), s(s_) {
    nvtxRangePushA(kStepNames[kind]);
    if (c->prof_on) {
      std::lock_guard<std::mutex> g(c->prof_mu);
      a = c->take_event();
      cudaEventRecord(a, s);
    }
  }
  ~Prof() {
    nvtxRangePop();
    c->launches.fetch_add(1, std::memory_order_relaxed);
    if (a) {
      std::lock_guard<std::mutex> g(c->prof_mu);
      cudaEvent_t b = c->take_event();
      cudaEventRecord(b, s);
      c->prof_pending.push_back({kind, a, b});
    }
  }
};
}  // namespace

struct moe_slots {
  moe_ctx* ctx = nullptr;
  int E = 0, n_spare = 0;
  std::vector<int> loc;  // -1 unregistered, MOE_LOC_*
  std::vector<const void*> gu, dn;
  std::vector<const float*> sgu, sdn;
  std::vector<MapEntry> h_maps;  // [E + n_spare]
  std::vector<int32_t> h_map_of; // [E]
  MapEntry* d_maps = nullptr;
  int32_t* d_map_of = nullptr;
  uint8_t* spare = nullptr;
  size_t off_dn = 0, off_sgu = 0, off_sdn = 0, slot_bytes = 0;
  size_t bytes_gu = 0, bytes_dn = 0, bytes_sgu = 0, bytes_sdn = 0;
  cudaStream_t copy_stream = nullptr;
  cudaEvent_t ev_ready[2] = {nullptr, nullptr};
  cudaEvent_t ev_free[2] = {nullptr, nullptr};
  int32_t* h_pinned = nullptr;  // offsets readback + list staging
  size_t h_pinned_ints = 0;
  int n_host = 0;
  moe_slots_stats_t stats{};
  // spare slots as an LRU cache of host-resident experts (MOE_SLOTS_LRU)
  int policy = MOE_SLOTS_LRU;
  std::vector<int> slot_expert;     // [n_spare] expert held, -1 empty
  std::vector<int> expert_slot;     // [E] its spare slot, -1 not cached
  std::vector<int64_t> slot_tick;   // [n_spare] call that last used the slot
  int64_t tick = 0;
  cudaEvent_t ev_done = nullptr;    // after the most recent call's GEMMs (they may read the slots)
  bool ev_done_valid = false;
  std::vector<uint8_t*> sf_blk;     // [E] MXFP4: the expert's E8M0 scales in the block layout (owned here)
  // The LRU state lives on the device (decode batches run it there, residency.cu); the vectors above
  // mirror it for the host-synchronised path, which pulls it before and pushes it after its own use.
  void* d_res = nullptr;
  ResidencyDev rdev{};
  std::vector<HostRec> h_host;      // [E] device-visible addresses of host records
  std::vector<char> unmapped;       // [E] host record without a device address
  int n_unmapped = 0;
  bool last_dev = false;            // the most recent call ran the device-side path
  int64_t* h_lru = nullptr;         // pinned staging: pull half, push half
  size_t h_lru_words = 0;           // int64 words per half
  std::mutex mu;
};

namespace {

// ----------------------------------------------------------- workspace --

struct WsLayout {
  size_t logits, rank, chunk_counts, topk_idx, topk_w, counts, offsets, perm_src, perm_k, inv;
  size_t list_expert, list_map, nt_prefix, sched, x_perm, x_scale, h, hq, h_scale, y_pair, total;
  size_t x_sfb, h_sfb;  // MXFP4: activation scales in the tensor cores' block layout, per N tile
  size_t nt_prefix2;    // MXFP4: N tiles of the (wider) down GEMM per listed expert
};

// MXFP4 down GEMM tile width for a gate/up width bn: 128 once gate/up is at its 64 (a 128-wide down tile keeps two
// accumulators and ran 28% faster at 4096 tokens; a 128-wide gate/up tile has one and ran 42% slower).
inline int mx_down_bn(int bn) { return bn >= 64 ? 128 : bn; }

// bf16 down GEMM tile width on the all-resident path: 256 for chunks of at least kBf16WideDownMinT tokens (down
// measured 8% faster at 16384 tokens and unchanged at 4096; gate/up stays at 128: at 256 it keeps one accumulator
// and ran 27% slower).
constexpr int kBf16WideDownMinT = 8192;
inline int bf16_down_bn(int bn, int T) { return (bn == 128 && T >= kBf16WideDownMinT) ? 256 : bn; }

WsLayout ws_layout(const moe_config_t& c, int T) {
  WsLayout L{};
  const size_t P = (size_t)T * c.top_k, E = c.n_experts, H = c.hidden, I = c.intermediate;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  const bool mx = c.wdtype == MOE_MXFP4;
  const size_t bn = (size_t)ffn_block_n(T, c.wdtype);
  const size_t n_tiles = (P + bn - 1) / bn + std::min(E, P);  // N tiles of a plan, at most
  size_t o = 0;
  auto take = [&](size_t bytes) {
    size_t at = o;
    o += align256(bytes);
    return at;
  };
  L.logits = take((size_t)T * E * 4);
  L.rank = take(P * 4);
  L.chunk_counts = take(64 * E * 4);
  L.topk_idx = take(P * 4);
  L.topk_w = take(P * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.perm_src = take(P * 4);
  L.perm_k = take(P * 4);
  L.inv = take(P * 4);
  L.list_expert = take((2 * E + 64) * 4);
  L.list_map = take((2 * E + 64) * 4);
  L.nt_prefix = take((2 * E + 64) * 4);
  L.nt_prefix2 = take((E + 1) * 4);
  L.sched = take((size_t)fused_sched_entries((int)E) * 4);
  L.x_perm = take(P * H * ((fp8 || mx) ? 1 : 2));
  L.x_scale = take(fp8 ? P * (H / 128) * 4 : 0);
  L.h = take(mx ? 0 : P * I * 2);
  L.hq = take((fp8 || mx) ? P * I : 0);
  L.h_scale = take(fp8 ? P * (I / 128) * 4 : 0);
  L.x_sfb = take(mx ? n_tiles * (H / 128) * 512 : 0);
  L.h_sfb = take(mx ? n_tiles * (I / 128) * 512 : 0);
  L.y_pair = take(P * H * 4);
  L.total = o;
  return L;
}

moe_status_t check_cfg(const moe_config_t& c) {
  if (c.hidden <= 0 || c.n_experts <= 0 || c.top_k <= 0 || c.intermediate <= 0)
    return fail(MOE_ERR_INVALID_ARG, "config sizes must be positive");
  if (c.wdtype != MOE_BF16 && c.wdtype != MOE_FP8_E4M3_B128 && c.wdtype != MOE_MXFP4)
    return fail(MOE_ERR_INVALID_ARG, "unknown wdtype");
  if (c.flags & ~MOE_FLAG_NO_PDL) return fail(MOE_ERR_INVALID_ARG, "unknown flag bits");
  if (c.hidden % 128 || c.intermediate % 128) return fail(MOE_ERR_UNSUPPORTED, "H and I must be multiples of 128");
  if (c.hidden > 8192 || c.intermediate > 8192) return fail(MOE_ERR_UNSUPPORTED, "H and I must be <= 8192");
  if (c.wdtype == MOE_MXFP4 && ((c.hidden % (128 * kMxKC)) || (c.intermediate % (128 * kMxKC))))
    return fail(MOE_ERR_UNSUPPORTED, "MXFP4 needs H and I multiples of 256 (two 128-deep K blocks per stage)");
  if (c.top_k > 32 || c.top_k > c.n_experts || c.n_experts > 1024)
    return fail(MOE_ERR_UNSUPPORTED, "need 1 <= K <= 32 and K <= E <= 1024");
  return MOE_OK;
}

moe_status_t check_T(const moe_ctx_t* ctx, int T) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (T > 65536) return fail(MOE_ERR_UNSUPPORTED, "T must be <= 65536");
  (void)ctx;
  return MOE_OK;
}

moe_status_t check_ws(const moe_ctx_t* ctx, int T, const void* ws, size_t ws_bytes) {
  const WsLayout L = ws_layout(ctx->cfg, T);
  if (!ws && L.total > 0) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (ws_bytes < L.total) return fail(MOE_ERR_INVALID_ARG, "workspace too small (see moe_workspace_size)");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(MOE_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t encode_2d(moe_ctx_t* ctx, CUtensorMap* m, const void* ptr, bool fp8, uint64_t inner, uint64_t rows,
                       uint32_t box_rows) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = ctx->encode(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                 const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return MOE_OK;
}

// bf16 operand as (64 elements, rows, K/64 chunks): one copy of box
// {64, box_rows, kc} brings kc K chunks, each a swizzled box_rows x 128 B block.
moe_status_t encode_3d_bf16(moe_ctx_t* ctx, CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                            uint32_t box_rows, uint32_t kc) {
  const cuuint64_t dims[3] = {64, rows, inner / 64};
  const cuuint64_t strides[2] = {inner * 2, 128};
  const cuuint32_t box[3] = {64u, box_rows, kc};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                                 estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (3-D) failed: " + std::to_string((int)r));
  return MOE_OK;
}

// Packed E2M1 codes [rows, inner] (two per byte) as (128 elements, rows,
// inner/128 blocks), box {128, 128, kMxKC}: one copy brings kMxKC K blocks of a
// 128-row tile, each landing unpacked (16 codes per 16 bytes) with the
// 128-byte swizzle.
moe_status_t encode_3d_fp4(moe_ctx_t* ctx, CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows) {
  const cuuint64_t dims[3] = {128, rows, inner / 128};
  const cuuint64_t strides[2] = {inner / 2, 64};
  const cuuint32_t box[3] = {128u, 128u, (cuuint32_t)kMxKC};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void*>(ptr), dims, strides,
                                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (E2M1) failed: " + std::to_string((int)r));
  return MOE_OK;
}

// Byte rows [rows, inner] (e4m3 codes) as (128 bytes, rows, inner/128 blocks),
// box {128, box_rows, kMxKC}: kMxKC K blocks per copy, each a swizzled
// box_rows x 128 B block.
moe_status_t encode_3d_u8(moe_ctx_t* ctx, CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                          uint32_t box_rows) {
  const cuuint64_t dims[3] = {128, rows, inner / 128};
  const cuuint64_t strides[2] = {inner, 128};
  const cuuint32_t box[3] = {128u, box_rows, (cuuint32_t)kMxKC};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = ctx->encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
                                 estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (3-D bytes) failed: " + std::to_string((int)r));
  return MOE_OK;
}

moe_status_t make_entry(moe_ctx_t* ctx, MapEntry* me, const void* gu, const void* dn, const float* sgu,
                        const float* sdn) {
  const moe_config_t& c = ctx->cfg;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  std::memset(me, 0, sizeof(*me));
  if (c.wdtype == MOE_MXFP4) {  // sgu / sdn: the blocked E8M0 scales
    moe_status_t st = encode_3d_fp4(ctx, &me->gu, gu, c.hidden, 2ull * c.intermediate);
    if (st != MOE_OK) return st;
    st = encode_3d_fp4(ctx, &me->dn, dn, c.intermediate, c.hidden);
    if (st != MOE_OK) return st;
    me->s_gu = sgu;
    me->s_dn = sdn;
    return MOE_OK;
  }
  if (!fp8) {
    for (int kc = 1; kc <= 2; ++kc) {
      moe_status_t st = encode_3d_bf16(ctx, kc == 1 ? &me->gu : &me->gu2, gu, c.hidden, 2ull * c.intermediate, 128, kc);
      if (st != MOE_OK) return st;
      st = encode_3d_bf16(ctx, kc == 1 ? &me->dn : &me->dn2, dn, c.intermediate, c.hidden, 128, kc);
      if (st != MOE_OK) return st;
    }
    return MOE_OK;
  }
  moe_status_t st = encode_2d(ctx, &me->gu, gu, fp8, c.hidden, 2ull * c.intermediate, 128);
  if (st != MOE_OK) return st;
  st = encode_2d(ctx, &me->dn, dn, fp8, c.intermediate, c.hidden, 128);
  if (st != MOE_OK) return st;
  me->s_gu = sgu;
  me->s_dn = sdn;
  return MOE_OK;
}


// ---- the slot table's LRU state between host and device. Staging half (words): [0] tick, [1..8] stats,
// [9 .. 9+n_spare) slot ticks, then int32 slot_expert [n_spare], expert_slot [E], map_of [E].
int64_t* lru_half(moe_slots_t* sl, int half) { return sl->h_lru + (size_t)half * sl->h_lru_words; }

// Queues the device state's copy into the pull half (the caller synchronises before lru_unpack).
moe_status_t lru_pull_async(moe_slots_t* sl, cudaStream_t s) {
  if (!sl->d_res) return MOE_OK;
  int64_t* h = lru_half(sl, 0);
  int32_t* h32 = reinterpret_cast<int32_t*>(h + 9 + sl->n_spare);
  MOE_CUDA(cudaMemcpyAsync(h, sl->rdev.tick, sizeof(int64_t), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaMemcpyAsync(h + 1, sl->rdev.stats, 8 * sizeof(int64_t), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaMemcpyAsync(h + 9, sl->rdev.slot_tick, sl->n_spare * sizeof(int64_t), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaMemcpyAsync(h32, sl->rdev.slot_expert, sl->n_spare * sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaMemcpyAsync(h32 + sl->n_spare, sl->rdev.expert_slot, sl->E * sizeof(int32_t), cudaMemcpyDeviceToHost,
                           s));
  return MOE_OK;
}

void lru_unpack(moe_slots_t* sl) {
  if (!sl->d_res) return;
  const int64_t* h = lru_half(sl, 0);
  const int32_t* h32 = reinterpret_cast<const int32_t*>(h + 9 + sl->n_spare);
  sl->tick = h[0];
  for (int i = 0; i < sl->n_spare; ++i) {
    sl->slot_tick[i] = h[9 + i];
    sl->slot_expert[i] = h32[i];
  }
  for (int e = 0; e < sl->E; ++e) sl->expert_slot[e] = h32[sl->n_spare + e];
}

// Queues the host mirror's copy to the device, with the expert -> map-entry table it implies.
moe_status_t lru_push_async(moe_slots_t* sl, cudaStream_t s) {
  if (!sl->d_res) return MOE_OK;
  int64_t* h = lru_half(sl, 1);
  int32_t* h32 = reinterpret_cast<int32_t*>(h + 9 + sl->n_spare);
  h[0] = sl->tick;
  for (int i = 0; i < sl->n_spare; ++i) {
    h[9 + i] = sl->slot_tick[i];
    h32[i] = sl->slot_expert[i];
  }
  for (int e = 0; e < sl->E; ++e) {
    h32[sl->n_spare + e] = sl->expert_slot[e];
    const int m = sl->loc[e] == MOE_LOC_HBM ? e
                  : (sl->loc[e] == MOE_LOC_HOST_PINNED && sl->expert_slot[e] >= 0) ? sl->E + sl->expert_slot[e]
                                                                                   : -1;
    h32[sl->n_spare + sl->E + e] = m;
    sl->h_map_of[e] = m;
  }
  MOE_CUDA(cudaMemcpyAsync(sl->rdev.tick, h, sizeof(int64_t), cudaMemcpyHostToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(sl->rdev.slot_tick, h + 9, sl->n_spare * sizeof(int64_t), cudaMemcpyHostToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(sl->rdev.slot_expert, h32, sl->n_spare * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(sl->rdev.expert_slot, h32 + sl->n_spare, sl->E * sizeof(int32_t), cudaMemcpyHostToDevice,
                           s));
  MOE_CUDA(cudaMemcpyAsync(sl->d_map_of, h32 + sl->n_spare + sl->E, sl->E * sizeof(int32_t), cudaMemcpyHostToDevice,
                           s));
  return MOE_OK;
}

// Runs the two GEMMs (and, for FP8, the quantiser of h between them) for one
// expert list whose arrays live in the workspace at list offset `lo`.
// nt_prefix_dn / bn_dn (bf16): the down GEMM's own, wider N tiling (from the plan kernel), or null for bn.
moe_status_t run_gemms(moe_ctx_t* ctx, moe_slots_t* sl, const WsLayout& W, void* ws, int T, int bn,
                       const int32_t* perm_src, const int32_t* perm_k, const int32_t* offsets, const float* topk_w,
                       float* y_pair, const int32_t* list_expert, const int32_t* list_map, const int32_t* nt_prefix,
                       int L, int max_ntiles, cudaStream_t s, bool pdl, bool plan_ready_gu,
                       int* sched = nullptr, const int32_t* nt_prefix_dn = nullptr, int bn_dn = 0) {
  const moe_config_t& c = ctx->cfg;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  const int P = T * c.top_k;
  if (c.wdtype == MOE_MXFP4) {
    // both GEMMs on the block-scaled tensor cores; gate/up writes h as MX e4m3 codes and blocked scales
    // the down GEMM runs on wider N tiles (bn_dn; its prefix from the plan), and gate/up writes h's scale blocks
    // in that tiling
    const int bn_dn = mx_down_bn(bn);
    const int32_t* np_dn = at<int32_t>(ws, W.nt_prefix2);
    const int max_ntiles_dn = (P + bn_dn - 1) / bn_dn + std::min(c.n_experts, P);
    ActMaps xm, hm;
    std::memset(&xm, 0, sizeof(xm));
    std::memset(&hm, 0, sizeof(hm));
    for (int i = 0, rows = 16; rows <= bn; ++i, rows <<= 1) {
      moe_status_t st = encode_3d_u8(ctx, &xm.m[i], at<void>(ws, W.x_perm), c.hidden, P, rows);
      if (st != MOE_OK) return st;
    }
    for (int i = 0, rows = 16; rows <= bn_dn; ++i, rows <<= 1) {
      moe_status_t st = encode_3d_u8(ctx, &hm.m[i], at<void>(ws, W.hq), c.intermediate, P, rows);
      if (st != MOE_OK) return st;
    }
    GemmArgs a{};
    a.maps = sl->d_maps;
    a.list_expert = list_expert;
    a.list_map = list_map;
    a.nt_prefix = nt_prefix;
    a.offsets = offsets;
    a.L = L;
    a.H = c.hidden;
    a.I = c.intermediate;
    a.K = c.top_k;
    a.h_out = at<void>(ws, W.hq);
    a.h_sfb = at<uint8_t>(ws, W.h_sfb);
    a.h_nt_prefix = np_dn;
    a.h_bn = bn_dn;
    a.act_sfb = at<uint8_t>(ws, W.x_sfb);
    a.y_out = y_pair;
    a.topk_w = topk_w;
    a.perm_src = perm_src;
    a.perm_k = perm_k;
    a.status = ctx->d_status;
    a.plan_ready = (pdl && plan_ready_gu) ? 1 : 0;
    a.num_sms = ctx->num_sms;
    {
      Prof p(ctx, MOE_PROF_GATE_UP, s);
      MOE_CUDA(launch_ffn_mxfp4(kGateUp, bn, xm, a, (c.intermediate / 128) * max_ntiles, s, pdl));
    }
    a.act_sfb = at<uint8_t>(ws, W.h_sfb);
    a.nt_prefix = np_dn;
    a.plan_ready = pdl ? 1 : 0;  // the plan is at least two launches back from the down GEMM
    {
      Prof p(ctx, MOE_PROF_DOWN, s);
      MOE_CUDA(launch_ffn_mxfp4(kDown, bn_dn, hm, a, (c.hidden / 128) * max_ntiles_dn, s, pdl));
    }
    return MOE_OK;
  }
  CUtensorMap xmap, hmap;
  ActMaps xmaps, hmaps;  // one activation map per tile box height 16 .. bn
  std::memset(&xmaps, 0, sizeof(xmaps));
  std::memset(&hmaps, 0, sizeof(hmaps));
  moe_status_t st = MOE_OK;
  if (fp8) {
    for (int i = 0, rows = 16; rows <= bn; ++i, rows <<= 1) {
      st = encode_2d(ctx, &xmaps.m[i], at<void>(ws, W.x_perm), true, c.hidden, P, rows);
      if (st != MOE_OK) return st;
      st = encode_2d(ctx, &hmaps.m[i], at<void>(ws, W.hq), true, c.intermediate, P, rows);
      if (st != MOE_OK) return st;
    }
    xmap = xmaps.m[0];
    hmap = hmaps.m[0];
  } else {
    for (int i = 0, rows = 16; rows <= bn; ++i, rows <<= 1) {
      st = encode_3d_bf16(ctx, &xmaps.m[i], at<void>(ws, W.x_perm), c.hidden, P, rows, kBf16GateUpChunks);
      if (st != MOE_OK) return st;
    }
    const int bn_down = (nt_prefix_dn && bn_dn > bn) ? bn_dn : bn;  // the down GEMM's N tile width
    for (int i = 0, rows = 16; rows <= bn_down; ++i, rows <<= 1) {
      st = encode_3d_bf16(ctx, &hmaps.m[i], at<void>(ws, W.h), c.intermediate, P, rows, bf16_down_gemm_chunks(bn_down));
      if (st != MOE_OK) return st;
    }
    xmap = xmaps.m[0];
    hmap = hmaps.m[0];
  }
  if (st != MOE_OK) return st;
  // the fused launches' counters: [0] + one per N tile, all inside the range the plan kernel zeroes
  const bool fused_ok = sched && T <= kDecodeMaxT && bn <= kFusedMaxBn && max_ntiles + 1 <= fused_sched_entries(L);
  if (fused_ok && fp8 && bn <= 32) {
    // decode, FP8, up to 32 tokens: both GEMMs and the quantisation of h in one launch (at 64 tokens the
    // in-epilogue quantisation costs more than the launch it saves: measured 442 vs 559 us per layer)
    GemmArgs a{};
    a.maps = sl->d_maps;
    a.list_expert = list_expert;
    a.list_map = list_map;
    a.nt_prefix = nt_prefix;
    a.offsets = offsets;
    a.L = L;
    a.H = c.hidden;
    a.I = c.intermediate;
    a.K = c.top_k;
    a.h_out = at<void>(ws, W.hq);
    a.h_scale = at<float>(ws, W.h_scale);
    a.y_out = y_pair;
    a.topk_w = topk_w;
    a.perm_src = perm_src;
    a.perm_k = perm_k;
    a.act_scale = at<float>(ws, W.x_scale);
    a.status = ctx->d_status;
    a.sched = sched;
    a.num_sms = ctx->num_sms;
    a.plan_ready = (pdl && plan_ready_gu) ? 1 : 0;  // plan -> quantiser -> this launch
    Prof p(ctx, MOE_PROF_FFN_FUSED, s);
    MOE_CUDA(launch_ffn_fp8_fused(bn, xmaps, hmaps, a, (c.intermediate / 128 + c.hidden / 128) * max_ntiles, s, pdl));
    return MOE_OK;
  }
  if (fused_ok && !fp8) {
    // decode: both GEMMs in one launch (x with one K chunk per box, h with two)
    ActMaps x1, h2;
    std::memset(&x1, 0, sizeof(x1));
    std::memset(&h2, 0, sizeof(h2));
    for (int i = 0, rows = 16; rows <= bn; ++i, rows <<= 1) {
      st = encode_3d_bf16(ctx, &x1.m[i], at<void>(ws, W.x_perm), c.hidden, P, rows, 1);
      if (st != MOE_OK) return st;
      st = encode_3d_bf16(ctx, &h2.m[i], at<void>(ws, W.h), c.intermediate, P, rows, 2);
      if (st != MOE_OK) return st;
    }
    GemmArgs a{};
    a.maps = sl->d_maps;
    a.list_expert = list_expert;
    a.list_map = list_map;
    a.nt_prefix = nt_prefix;
    a.offsets = offsets;
    a.L = L;
    a.H = c.hidden;
    a.I = c.intermediate;
    a.K = c.top_k;
    a.h_out = at<void>(ws, W.h);
    a.y_out = y_pair;
    a.topk_w = topk_w;
    a.perm_src = perm_src;
    a.perm_k = perm_k;
    a.status = ctx->d_status;
    a.sched = sched;
    a.num_sms = ctx->num_sms;
    Prof p(ctx, MOE_PROF_FFN_FUSED, s);
    MOE_CUDA(launch_ffn_fused(bn, x1, h2, a, (c.intermediate / 128 + c.hidden / 128) * max_ntiles, s, pdl));
    return MOE_OK;
  }
  GemmArgs a{};
  a.maps = sl->d_maps;
  a.list_expert = list_expert;
  a.list_map = list_map;
  a.nt_prefix = nt_prefix;
  a.offsets = offsets;
  a.L = L;
  a.H = c.hidden;
  a.I = c.intermediate;
  a.K = c.top_k;
  a.h_out = at<void>(ws, W.h);
  a.y_out = y_pair;
  a.topk_w = topk_w;
  a.perm_src = perm_src;
  a.perm_k = perm_k;
  a.status = ctx->d_status;
  a.act_scale = fp8 ? at<float>(ws, W.x_scale) : nullptr;
  a.plan_ready = (pdl && plan_ready_gu) ? 1 : 0;
  a.num_sms = ctx->num_sms;
  const int max_experts = std::min(L, P);  // experts that can hold a pair
  a.est_tiles = (c.intermediate / 128) * std::min(max_ntiles, max_experts * ((P + bn - 1) / bn));
  {
    Prof p(ctx, MOE_PROF_GATE_UP, s);
    MOE_CUDA(launch_ffn_gemm(kGateUp, c.wdtype, bn, xmap, &xmaps, a, (c.intermediate / 128) * max_ntiles, s, pdl));
  }
  if (fp8) {
    {
      Prof p(ctx, MOE_PROF_QUANT, s);
      MOE_CUDA(launch_quant_rows_e4m3_count(at<void>(ws, W.h), offsets, c.n_experts, P, c.intermediate,
                                            at<uint8_t>(ws, W.hq), at<float>(ws, W.h_scale), s, pdl));
    }
    a.act_scale = at<float>(ws, W.h_scale);
  }
  a.plan_ready = pdl ? 1 : 0;  // the plan is at least two launches back from the down GEMM
  int bnd = bn, max_ntiles_d = max_ntiles;  // bnd: as the h maps above were encoded
  if (nt_prefix_dn && bn_dn > bn) {
    bnd = bn_dn;
    a.nt_prefix = nt_prefix_dn;
    max_ntiles_d = (P + bnd - 1) / bnd + std::min(L, P);
  }
  a.est_tiles = (c.hidden / 128) * std::min(max_ntiles_d, max_experts * ((P + bnd - 1) / bnd));
  {
    Prof p(ctx, MOE_PROF_DOWN, s);
    MOE_CUDA(launch_ffn_gemm(kDown, c.wdtype, bnd, hmap, &hmaps, a, (c.hidden / 128) * max_ntiles_d, s, pdl));
  }
  return MOE_OK;
}

}  // namespace

// ---------------------------------------------------- allocation hook --
// Every allocation the library makes goes through lib_malloc / lib_host_alloc,
// so that moe_debug_fail_allocs can make chosen ones fail as an exhausted
// device or host would.
namespace {
std::mutex g_fail_mu;
int g_fail_kind = MOE_ALLOC_ANY, g_fail_skip = 0, g_fail_n = 0;

bool injected_alloc_failure(int kind) {
  std::lock_guard<std::mutex> lock(g_fail_mu);
  if (g_fail_n <= 0 || (g_fail_kind != MOE_ALLOC_ANY && g_fail_kind != kind)) return false;
  if (g_fail_skip > 0) {
    --g_fail_skip;
    return false;
  }
  --g_fail_n;
  return true;
}

template <typename P>
cudaError_t lib_malloc(P** p, size_t bytes) {
  if (injected_alloc_failure(MOE_ALLOC_DEVICE)) return cudaErrorMemoryAllocation;
  return cudaMalloc(reinterpret_cast<void**>(p), bytes);
}

template <typename P>
cudaError_t lib_host_alloc(P** p, size_t bytes) {
  if (injected_alloc_failure(MOE_ALLOC_PINNED)) return cudaErrorMemoryAllocation;
  return cudaHostAlloc(reinterpret_cast<void**>(p), bytes, cudaHostAllocDefault);
}
}  // namespace

// =================================================================== ABI ==

extern "C" {

const char* moe_last_error(void) { return g_last_error.c_str(); }

moe_status_t moe_debug_fail_allocs(int kind, int skip, int n) {
  if (kind < MOE_ALLOC_ANY || kind > MOE_ALLOC_PINNED || skip < 0 || n < 0)
    return fail(MOE_ERR_INVALID_ARG, "moe_debug_fail_allocs: unknown kind or negative count");
  std::lock_guard<std::mutex> lock(g_fail_mu);
  g_fail_kind = kind;
  g_fail_skip = skip;
  g_fail_n = n;
  return MOE_OK;
}

moe_status_t moe_ctx_create(moe_ctx_t** out, const moe_config_t* cfg) {
  if (!out || !cfg) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  *out = nullptr;
  moe_status_t st = check_cfg(*cfg);
  if (st != MOE_OK) return st;
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  MOE_CUDA(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10) return fail(MOE_ERR_UNSUPPORTED, "libmoe needs an sm_100 (B200-class) device");
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  MOE_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
  if (!fn || q != cudaDriverEntryPointSuccess) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled not found");
  moe_ctx_t* ctx = new moe_ctx_t();
  ctx->cfg = *cfg;
  ctx->device = dev;
  ctx->num_sms = prop.multiProcessorCount;
  ctx->chain = !(cfg->flags & MOE_FLAG_NO_PDL);
  ctx->encode = reinterpret_cast<EncodeTiledFn>(fn);
  if (lib_malloc(&ctx->d_status, sizeof(int)) != cudaSuccess ||
      lib_malloc(&ctx->d_counters, sizeof(unsigned int) * kRouteSmallMaxT) != cudaSuccess) {
    cudaFree(ctx->d_status);
    delete ctx;
    return fail(MOE_ERR_OOM, "cudaMalloc of the context's device words failed");
  }
  cudaMemset(ctx->d_status, 0, sizeof(int));
  cudaMemset(ctx->d_counters, 0, sizeof(unsigned int) * kRouteSmallMaxT);
  cudaDeviceSynchronize();
  *out = ctx;
  return MOE_OK;
}

moe_status_t moe_ctx_destroy(moe_ctx_t* ctx) {
  if (!ctx) return MOE_OK;
  for (auto& r : ctx->prof_pending) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : ctx->ev_pool) cudaEventDestroy(e);
  cudaFree(ctx->d_status);
  cudaFree(ctx->d_counters);
  delete ctx;
  return MOE_OK;
}

size_t moe_workspace_size(const moe_ctx_t* ctx, int T) {
  if (!ctx || T < 0) return 0;
  return ws_layout(ctx->cfg, T).total;
}

int64_t moe_launch_count(const moe_ctx_t* ctx) { return ctx ? ctx->launches.load() : 0; }

moe_status_t moe_profile_enable(moe_ctx_t* ctx, int enable) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  std::lock_guard<std::mutex> g(ctx->prof_mu);
  ctx->prof_on = enable != 0;
  return MOE_OK;
}

moe_status_t moe_profile_read(moe_ctx_t* ctx, int kind, double* total_ms, int64_t* launches, int reset) {
  if (!ctx || !total_ms || !launches) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  if (kind < 0 || kind >= MOE_PROF_KINDS) return fail(MOE_ERR_INVALID_ARG, "unknown kernel kind");
  std::lock_guard<std::mutex> g(ctx->prof_mu);
  for (auto& r : ctx->prof_pending) {
    MOE_CUDA(cudaEventSynchronize(r.b));
    float ms = 0.f;
    MOE_CUDA(cudaEventElapsedTime(&ms, r.a, r.b));
    ctx->prof_ms[r.kind] += ms;
    ctx->prof_n[r.kind] += 1;
    ctx->ev_pool.push_back(r.a);
    ctx->ev_pool.push_back(r.b);
  }
  ctx->prof_pending.clear();
  *total_ms = ctx->prof_ms[kind];
  *launches = ctx->prof_n[kind];
  if (reset) {
    ctx->prof_ms[kind] = 0.0;
    ctx->prof_n[kind] = 0;
  }
  return MOE_OK;
}

moe_status_t moe_debug_wait_flag(moe_ctx_t* ctx, const int32_t* flag, int64_t limit_ns, moe_stream_t stream) {
  if (!ctx || !flag) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  if (limit_ns <= 0 || limit_ns > 2000000000LL) return fail(MOE_ERR_INVALID_ARG, "limit_ns must be in (0, 2 s]");
  MOE_CUDA(moe::launch_debug_wait_flag(flag, static_cast<uint64_t>(limit_ns), ctx->d_status,
                                       static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status_t moe_get_device_status(moe_ctx_t* ctx, int32_t* status, int reset) {
  if (!ctx || !status) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  MOE_CUDA(cudaDeviceSynchronize());
  int v = 0;
  MOE_CUDA(cudaMemcpy(&v, ctx->d_status, sizeof(int), cudaMemcpyDeviceToHost));
  *status = v | ctx->host_status;
  if (reset) {
    MOE_CUDA(cudaMemset(ctx->d_status, 0, sizeof(int)));
    ctx->host_status = 0;
  }
  return MOE_OK;
}

}  // extern "C"

namespace {

// ---- step implementations; `pdl` = launch the first kernel with programmatic
// stream serialisation (only when the preceding launch is this library's own
// kernel of the same forward).

// rd / map_of / planned: the device-side residency plan, which the decode router's last CTA runs after the top-k
// when it can (*planned = true); otherwise the caller launches it.
moe_status_t route_impl(moe_ctx_t* ctx, const void* x, const float* w_router, const float* logit_bias, int T,
                        int32_t* topk_idx, float* topk_w, void* ws, cudaStream_t s, int* sched = nullptr,
                        int sched_n = 0, const ResidencyDev* rd = nullptr, int32_t* map_of = nullptr,
                        bool* planned = nullptr) {
  if (planned) *planned = false;
  const moe_config_t& c = ctx->cfg;
  const WsLayout W = ws_layout(c, T);
  float* logits = at<float>(ws, W.logits);
  if (T <= kRouteSmallMaxT) {
    Prof p(ctx, MOE_PROF_ROUTER, s);
    MOE_CUDA(launch_route_small(x, w_router, logit_bias, T, c.hidden, c.n_experts, c.top_k, logits, topk_idx,
                                topk_w, ctx->d_counters, ctx->d_status, s, ctx->chain, sched, sched_n, rd, map_of,
                                planned));
    return MOE_OK;
  }
  {
    Prof p(ctx, MOE_PROF_ROUTER, s);
    MOE_CUDA(launch_route_gemm(x, w_router, logit_bias, T, c.hidden, c.n_experts, logits, s));
  }
  {
    Prof p(ctx, MOE_PROF_TOPK, s);
    MOE_CUDA(launch_topk_warp(logits, T, c.n_experts, c.top_k, topk_idx, topk_w, s, ctx->chain));
  }
  return MOE_OK;
}

// Small batches: one launch (plus, with map_of, the FFN tile plan and, with
// x_perm, the sorted activation rows). Otherwise rank -> scan -> scatter.
moe_status_t permute_impl(moe_ctx_t* ctx, const int32_t* topk_idx, int T, int32_t* counts, int32_t* offsets,
                          int32_t* perm_src, int32_t* perm_k, int32_t* inv, void* ws, cudaStream_t s, bool pdl,
                          const int32_t* map_of = nullptr, int bn = 0, const void* x = nullptr,
                          void* x_perm = nullptr, bool* planned = nullptr) {
  const moe_config_t& c = ctx->cfg;
  const WsLayout W = ws_layout(c, T);
  if (planned) *planned = false;
  if ((long long)T * c.top_k <= kPermuteSmallMaxPairs) {
    Prof p(ctx, MOE_PROF_PERMUTE, s);
    const bool mx2 = map_of && c.wdtype == MOE_MXFP4;  // also the down GEMM's wider N tiles
    MOE_CUDA(launch_permute_small(topk_idx, T, c.top_k, c.n_experts, counts, offsets, perm_src, perm_k, inv, map_of,
                                  bn, at<int32_t>(ws, W.list_expert), at<int32_t>(ws, W.list_map),
                                  at<int32_t>(ws, W.nt_prefix), x, c.hidden, x_perm, ctx->d_status, s, pdl,
                                  map_of ? at<int>(ws, W.sched) : nullptr, fused_sched_entries(c.n_experts),
                                  mx2 ? mx_down_bn(bn) : 0, mx2 ? at<int32_t>(ws, W.nt_prefix2) : nullptr));
    if (planned) *planned = map_of != nullptr;
    return MOE_OK;
  }
  const int chunk = permute_chunk_tokens(T, c.top_k);
  const int n_chunks = T > 0 ? (T + chunk - 1) / chunk : 0;
  int32_t* cc = at<int32_t>(ws, W.chunk_counts);
  if (T > 0) {
    Prof p(ctx, MOE_PROF_PERMUTE, s);
    MOE_CUDA(launch_permute_rank(topk_idx, T, c.top_k, c.n_experts, chunk, at<int32_t>(ws, W.rank), cc,
                                 ctx->d_status, s, pdl));
    pdl = ctx->chain;
  }
  {
    Prof p(ctx, MOE_PROF_PERMUTE, s);
    MOE_CUDA(launch_permute_scan(cc, n_chunks, c.n_experts, counts, offsets, s, pdl));
  }
  if (T > 0) {
    Prof p(ctx, MOE_PROF_PERMUTE, s);
    MOE_CUDA(launch_permute_scatter(topk_idx, at<int32_t>(ws, W.rank), cc, offsets, T, c.top_k, c.n_experts, chunk,
                                    perm_src, perm_k, inv, s, ctx->chain));
  }
  return MOE_OK;
}

// Decode FFN planned inside the kernel from the router's top-k (no permutation
// kernel, no gathered x). The caller checked decode_path_ok().
moe_status_t ffn_decode_impl(moe_ctx_t* ctx, moe_slots_t* sl, const void* x, const int32_t* idx, const float* topk_w,
                             int T, float* y_pair, void* ws, cudaStream_t s, int* sched) {
  const moe_config_t& c = ctx->cfg;
  const WsLayout W = ws_layout(c, T);
  const int E = c.n_experts, P = T * c.top_k;
  const int tp = std::min(64, (T + 15) / 16 * 16 == 48 ? 64 : (T + 15) / 16 * 16);
  std::lock_guard<std::mutex> lock(sl->mu);
  sl->stats.calls++;
  sl->stats.last_cold = 0;
  sl->stats.last_touched = -1;
  CUtensorMap xmap;
  moe_status_t st = encode_3d_bf16(ctx, &xmap, x, c.hidden, T, tp, 1);
  if (st != MOE_OK) return st;
  ActMaps hmaps;
  std::memset(&hmaps, 0, sizeof(hmaps));
  for (int i = 0, rows = 16; rows <= tp; ++i, rows <<= 1) {
    st = encode_3d_bf16(ctx, &hmaps.m[i], at<void>(ws, W.h), c.intermediate, P, rows, 2);
    if (st != MOE_OK) return st;
  }
  GemmArgs a{};
  a.maps = sl->d_maps;
  a.H = c.hidden;
  a.I = c.intermediate;
  a.K = c.top_k;
  a.h_out = at<void>(ws, W.h);
  a.y_out = y_pair;
  a.topk_w = topk_w;
  a.status = ctx->d_status;
  a.sched = sched;
  a.num_sms = ctx->num_sms;
  DecodeArgs d{};
  d.topk_idx = idx;
  d.map_of = sl->d_map_of;
  d.T = T;
  d.E = E;
  d.counts = at<int32_t>(ws, W.counts);
  d.offsets = at<int32_t>(ws, W.offsets);
  d.perm_src = at<int32_t>(ws, W.perm_src);
  d.perm_k = at<int32_t>(ws, W.perm_k);
  d.inv = at<int32_t>(ws, W.inv);
  Prof p(ctx, MOE_PROF_FFN_FUSED, s);
  MOE_CUDA(launch_ffn_decode(xmap, hmaps, a, d, (c.intermediate / 128 + c.hidden / 128) * std::min(E, P), s,
                             ctx->chain));
  return MOE_OK;
}

// Decode batches with host-resident experts whose pairs cannot route to more host experts than there are
// spare slots: the cache bookkeeping and the copies run on the device (residency.cu), no host round trip.
// Decode batches with host-resident experts whose pairs fit the spare slots: the LRU plan and the copies run on
// the device. bf16 then takes the one-launch decode FFN; FP8 the one-launch permutation and plan, the quantiser and
// its GEMMs, which read the cached experts through the same slot table.
bool residency_device_path_ok(const moe_ctx_t* ctx, const moe_slots_t* sl, const void* x, int T) {
  const moe_config_t& c = ctx->cfg;
  const long long P = (long long)T * c.top_k;
  if (sl->n_host <= 0 || !sl->d_res || sl->policy != MOE_SLOTS_LRU || sl->n_unmapped != 0 || T < 1 ||
      P > sl->n_spare)
    return false;
  if (c.wdtype == MOE_FP8_E4M3_B128) return P <= kPermuteSmallMaxPairs;
  return c.wdtype == MOE_BF16 && T <= kDecodeMaxT && P <= kDecodeMaxPairs && ((uintptr_t)x % 16) == 0 &&
         ffn_decode_smem_bytes(T, c.n_experts) <= 232448;
}

bool decode_path_ok(const moe_ctx_t* ctx, const moe_slots_t* sl, const void* x, int T) {
  const moe_config_t& c = ctx->cfg;
  return c.wdtype == MOE_BF16 && sl->n_host == 0 && T >= 1 && T <= kDecodeMaxT &&
         (long long)T * c.top_k <= kDecodeMaxPairs && ((uintptr_t)x % 16) == 0 &&
         ffn_decode_smem_bytes(T, c.n_experts) <= 232448;
}

// Expert FFN. `planned`: the permutation step already wrote the tile plan and
// (bf16) the sorted rows; `pdl`: the previous launch is this forward's own.
moe_status_t ffn_impl(moe_ctx_t* ctx, moe_slots_t* sl, const void* x, const int32_t* perm_src,
                      const int32_t* perm_k, const int32_t* offsets, const float* topk_w, int T, float* y_pair,
                      void* ws, cudaStream_t s, bool pdl, bool planned, const int32_t* inv = nullptr,
                      bool cached_on_device = false) {
  const moe_config_t& c = ctx->cfg;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  const WsLayout W = ws_layout(c, T);
  const int E = c.n_experts, P = T * c.top_k;
  // FP8 activation rows in sorted-pair order: with inv each token is quantised once and stored to its K rows
  auto quant_x = [&](bool chain_pdl) -> cudaError_t {
    if (inv)
      return launch_quant_scatter_rows(x, inv, T, c.top_k, c.hidden, at<uint8_t>(ws, W.x_perm),
                                       at<float>(ws, W.x_scale), s, chain_pdl);
    return launch_gather_quant_rows(x, perm_src, offsets, E, P, c.hidden, at<uint8_t>(ws, W.x_perm),
                                    at<float>(ws, W.x_scale), s, chain_pdl);
  };
  const int bn = ffn_block_n(T, c.wdtype);
  moe_status_t st = MOE_OK;
  std::lock_guard<std::mutex> lock(sl->mu);
  sl->stats.calls++;

  int32_t* le = at<int32_t>(ws, W.list_expert);
  int32_t* lm = at<int32_t>(ws, W.list_map);
  int32_t* np = at<int32_t>(ws, W.nt_prefix);
  const int ntile_bound = (P + bn - 1) / bn + std::min(E, P);
  // pairs routed to an expert with no registered weights: zero rows, and inv = -1 in the forward
  const DropArgs drop{perm_src, perm_k, c.top_k, const_cast<int32_t*>(inv), y_pair, c.hidden};

  if (sl->n_host == 0 && c.wdtype == MOE_MXFP4) {
    sl->stats.last_cold = 0;
    sl->stats.last_touched = -1;
    if (!planned) {
      Prof p(ctx, MOE_PROF_PERMUTE, s);
      MOE_CUDA(launch_ffn_plan(offsets, sl->d_map_of, E, bn, le, lm, np, ctx->d_status, s, pdl,
                               at<int>(ws, W.sched), fused_sched_entries(E), drop, mx_down_bn(bn),
                               at<int32_t>(ws, W.nt_prefix2)));
    }
    {
      // MX e4m3 activation rows in sorted-pair order, scales in the block layout of their N tile
      Prof pg(ctx, MOE_PROF_GATHER, s);
      MOE_CUDA(launch_quant_mx_pairs(x, perm_src, offsets, np, E, bn, P, c.hidden, at<uint8_t>(ws, W.x_perm),
                                     at<uint8_t>(ws, W.x_sfb), s, planned ? pdl : ctx->chain));
    }
    return run_gemms(ctx, sl, W, ws, T, bn, perm_src, perm_k, offsets, topk_w, y_pair, le, lm, np, E, ntile_bound,
                     s, ctx->chain, planned ? pdl : true);
  }
  if (sl->n_host == 0 || cached_on_device) {
    // every routed expert is in HBM: resident, or (cached_on_device) put in a spare slot by the device-side plan
    // earlier in this forward, which also wrote the counts the stats report
    if (!cached_on_device) {
      sl->stats.last_cold = 0;
      sl->stats.last_touched = -1;
    }
    bool plan_ready_gu = false;
    const int bn_dn = c.wdtype == MOE_BF16 && !planned ? bf16_down_bn(bn, T) : bn;
    if (!planned) {
      {
        Prof p(ctx, MOE_PROF_PERMUTE, s);
        MOE_CUDA(launch_ffn_plan(offsets, sl->d_map_of, E, bn, le, lm, np, ctx->d_status, s, pdl,
                                 at<int>(ws, W.sched), fused_sched_entries(E), drop, bn_dn,
                                 bn_dn != bn ? at<int32_t>(ws, W.nt_prefix2) : nullptr));
      }
      Prof pg(ctx, MOE_PROF_GATHER, s);
      if (fp8) {
        MOE_CUDA(quant_x(ctx->chain));
      } else {
        MOE_CUDA(launch_gather_rows(x, perm_src, offsets, E, P, c.hidden, at<void>(ws, W.x_perm), s, ctx->chain));
      }
      plan_ready_gu = true;  // plan -> gather -> gate/up
    } else if (fp8) {
      Prof pg(ctx, MOE_PROF_GATHER, s);
      MOE_CUDA(quant_x(pdl));
      plan_ready_gu = pdl;  // permutation+plan -> quantiser -> gate/up
    }
    return run_gemms(ctx, sl, W, ws, T, bn, perm_src, perm_k, offsets, topk_w, y_pair, le, lm, np, E, ntile_bound,
                     s, ctx->chain, plan_ready_gu, at<int>(ws, W.sched),
                     bn_dn != bn ? at<int32_t>(ws, W.nt_prefix2) : nullptr, bn_dn);
  }

  // activation rows in sorted-pair order (quantised for FP8); no PDL on the host-synchronised path
  {
    Prof pg(ctx, MOE_PROF_GATHER, s);
    if (fp8) {
      MOE_CUDA(quant_x(false));
    } else {
      MOE_CUDA(launch_gather_rows(x, perm_src, offsets, E, P, c.hidden, at<void>(ws, W.x_perm), s, false));
    }
  }

  // ---- hot/cold: read the per-expert offsets back, stage the routed cold experts
  int32_t* hoff = sl->h_pinned;
  MOE_CUDA(cudaMemcpyAsync(hoff, offsets, sizeof(int32_t) * (E + 1), cudaMemcpyDeviceToHost, s));
  if ((st = lru_pull_async(sl, s)) != MOE_OK) return st;  // the cache state the device-side path left
  MOE_CUDA(cudaStreamSynchronize(s));
  lru_unpack(sl);
  sl->last_dev = false;
  std::vector<int> hot, cold;
  int touched = 0;
  for (int e = 0; e < E; ++e) {
    const int cnt = hoff[e + 1] - hoff[e];
    if (cnt <= 0) continue;
    ++touched;
    if (sl->loc[e] == MOE_LOC_HBM) hot.push_back(e);
    else if (sl->loc[e] == MOE_LOC_HOST_PINNED) cold.push_back(e);
    else {
      ctx->host_status |= MOE_DEV_NO_SLOT;
      MOE_CUDA(launch_drop_pairs(hoff[e], hoff[e + 1], drop, s));
    }
  }
  sl->stats.last_touched = touched;
  sl->stats.last_cold = (int32_t)cold.size();
  sl->stats.last_hits = 0;
  sl->stats.last_routed_cold = (int32_t)cold.size();
  if (!cold.empty() && sl->n_spare <= 0) return fail(MOE_ERR_SLOT, "cold experts routed but no spare slots");

  if (sl->policy == MOE_SLOTS_LRU && (int)cold.size() <= sl->n_spare) {
    // ---- LRU: hits keep their slot; each miss takes the least recently used slot this call does not need
    const int64_t tick = ++sl->tick;
    std::vector<int> miss;
    int hits = 0;
    for (int e : cold) {
      const int sidx = sl->expert_slot[e];
      if (sidx >= 0) {
        sl->slot_tick[sidx] = tick;
        ++hits;
      } else {
        miss.push_back(e);
      }
    }
    bool waited = false;
    for (int e : miss) {
      int victim = -1;
      for (int i = 0; i < sl->n_spare; ++i) {
        if (sl->slot_tick[i] == tick) continue;  // holds an expert of this call
        if (victim < 0 || sl->slot_tick[i] < sl->slot_tick[victim]) victim = i;
      }
      if (victim < 0) return fail(MOE_ERR_SLOT, "no free spare slot");  // cannot happen: cold.size() <= n_spare
      if (sl->slot_expert[victim] >= 0) sl->expert_slot[sl->slot_expert[victim]] = -1;
      sl->slot_expert[victim] = e;
      sl->expert_slot[e] = victim;
      sl->slot_tick[victim] = tick;
      if (!waited && sl->ev_done_valid) {
        // the previous call's GEMMs may still read the slot being overwritten
        MOE_CUDA(cudaStreamWaitEvent(sl->copy_stream, sl->ev_done, 0));
        waited = true;
      }
      uint8_t* slot = sl->spare + (size_t)victim * sl->slot_bytes;
      MOE_CUDA(cudaMemcpyAsync(slot, sl->gu[e], sl->bytes_gu, cudaMemcpyHostToDevice, sl->copy_stream));
      MOE_CUDA(cudaMemcpyAsync(slot + sl->off_dn, sl->dn[e], sl->bytes_dn, cudaMemcpyHostToDevice, sl->copy_stream));
      if (fp8) {
        MOE_CUDA(cudaMemcpyAsync(slot + sl->off_sgu, sl->sgu[e], sl->bytes_sgu, cudaMemcpyHostToDevice,
                                 sl->copy_stream));
        MOE_CUDA(cudaMemcpyAsync(slot + sl->off_sdn, sl->sdn[e], sl->bytes_sdn, cudaMemcpyHostToDevice,
                                 sl->copy_stream));
      }
      sl->stats.cold_staged++;
      sl->stats.bytes_staged += (int64_t)(sl->bytes_gu + sl->bytes_dn + (fp8 ? sl->bytes_sgu + sl->bytes_sdn : 0));
    }
    sl->stats.last_cold = (int32_t)miss.size();
    sl->stats.last_hits = hits;
    sl->stats.cache_hits += hits;
    // one list over every touched expert, ascending: resident ones by their own map, cached ones by their slot's
    std::vector<int32_t> he, hm, hp;
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      const int cnt = hoff[e + 1] - hoff[e];
      if (cnt <= 0) continue;
      int m;
      if (sl->loc[e] == MOE_LOC_HBM) m = e;
      else if (sl->loc[e] == MOE_LOC_HOST_PINNED) m = E + sl->expert_slot[e];
      else continue;
      he.push_back(e);
      hm.push_back(m);
      hp.push_back(acc);
      acc += (cnt + bn - 1) / bn;
    }
    hp.push_back(acc);
    int32_t* stage = sl->h_pinned + (E + 1);
    const size_t n_e = he.size(), n_p = hp.size();
    std::memcpy(stage, he.data(), n_e * 4);
    std::memcpy(stage + n_e, hm.data(), n_e * 4);
    std::memcpy(stage + 2 * n_e, hp.data(), n_p * 4);
    MOE_CUDA(cudaMemcpyAsync(le, stage, n_e * 4, cudaMemcpyHostToDevice, s));
    MOE_CUDA(cudaMemcpyAsync(lm, stage + n_e, n_e * 4, cudaMemcpyHostToDevice, s));
    MOE_CUDA(cudaMemcpyAsync(np, stage + 2 * n_e, n_p * 4, cudaMemcpyHostToDevice, s));
    if (!miss.empty()) {
      MOE_CUDA(cudaEventRecord(sl->ev_ready[0], sl->copy_stream));
      MOE_CUDA(cudaStreamWaitEvent(s, sl->ev_ready[0], 0));
    }
    if (n_e > 0) {
      st = run_gemms(ctx, sl, W, ws, T, bn, perm_src, perm_k, offsets, topk_w, y_pair, le, lm, np, (int)n_e,
                     ntile_bound, s, false, false);
      if (st != MOE_OK) return st;
    }
    MOE_CUDA(cudaEventRecord(sl->ev_done, s));
    sl->ev_done_valid = true;
    return lru_push_async(sl, s);
  }
  // per-call staging (or more routed host experts than slots): every slot is overwritten, the cache empties
  std::fill(sl->slot_expert.begin(), sl->slot_expert.end(), -1);
  std::fill(sl->expert_slot.begin(), sl->expert_slot.end(), -1);
  std::fill(sl->slot_tick.begin(), sl->slot_tick.end(), -1);
  if (sl->ev_done_valid) MOE_CUDA(cudaStreamWaitEvent(sl->copy_stream, sl->ev_done, 0));
  const bool two_buf = (int)cold.size() > sl->n_spare && sl->n_spare >= 2;
  const int bsz = two_buf ? sl->n_spare / 2 : sl->n_spare;

  // list staging: [hot][batch0][batch1]...; each list: experts, maps, prefix (L+1)
  struct ListRef {
    int L, e_off, p_off;
  };
  std::vector<ListRef> lists;
  int32_t* stage = sl->h_pinned + (E + 1);
  std::vector<int32_t> he, hm, hp;
  auto add_list = [&](const std::vector<int>& ex, int map_base) {
    ListRef r{(int)ex.size(), (int)he.size(), (int)hp.size()};
    int acc = 0;
    for (size_t i = 0; i < ex.size(); ++i) {
      const int e = ex[i];
      he.push_back(e);
      hm.push_back(map_base < 0 ? e : map_base + (int)i);
      hp.push_back(acc);
      acc += (hoff[e + 1] - hoff[e] + bn - 1) / bn;
    }
    hp.push_back(acc);
    lists.push_back(r);
  };
  if (!hot.empty()) add_list(hot, -1);
  const int n_batches = cold.empty() ? 0 : ((int)cold.size() + bsz - 1) / bsz;
  for (int b = 0; b < n_batches; ++b) {
    std::vector<int> part(cold.begin() + (size_t)b * bsz,
                          cold.begin() + std::min(cold.size(), (size_t)(b + 1) * bsz));
    add_list(part, E + (two_buf ? (b & 1) * bsz : 0));
  }
  const size_t n_e = he.size(), n_p = hp.size();
  std::memcpy(stage, he.data(), n_e * 4);
  std::memcpy(stage + n_e, hm.data(), n_e * 4);
  std::memcpy(stage + 2 * n_e, hp.data(), n_p * 4);
  // three device arrays from one staging block (lists region holds 2E+64 ints each)
  MOE_CUDA(cudaMemcpyAsync(le, stage, n_e * 4, cudaMemcpyHostToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(lm, stage + n_e, n_e * 4, cudaMemcpyHostToDevice, s));
  MOE_CUDA(cudaMemcpyAsync(np, stage + 2 * n_e, n_p * 4, cudaMemcpyHostToDevice, s));

  size_t li = 0;
  if (!hot.empty()) {
    const ListRef& r = lists[li++];
    st = run_gemms(ctx, sl, W, ws, T, bn, perm_src, perm_k, offsets, topk_w, y_pair, le + r.e_off, lm + r.e_off,
                   np + r.p_off, r.L, ntile_bound, s, false, false);
    if (st != MOE_OK) return st;
  }
  for (int b = 0; b < n_batches; ++b) {
    const ListRef& r = lists[li++];
    const int buf = two_buf ? (b & 1) : 0;
    MOE_CUDA(cudaStreamWaitEvent(sl->copy_stream, sl->ev_free[buf], 0));
    for (int i = 0; i < r.L; ++i) {
      const int e = he[r.e_off + i];
      uint8_t* slot = sl->spare + (size_t)(buf * bsz + i) * sl->slot_bytes;
      MOE_CUDA(cudaMemcpyAsync(slot, sl->gu[e], sl->bytes_gu, cudaMemcpyHostToDevice, sl->copy_stream));
      MOE_CUDA(cudaMemcpyAsync(slot + sl->off_dn, sl->dn[e], sl->bytes_dn, cudaMemcpyHostToDevice, sl->copy_stream));
      if (fp8) {
        MOE_CUDA(cudaMemcpyAsync(slot + sl->off_sgu, sl->sgu[e], sl->bytes_sgu, cudaMemcpyHostToDevice,
                                 sl->copy_stream));
        MOE_CUDA(cudaMemcpyAsync(slot + sl->off_sdn, sl->sdn[e], sl->bytes_sdn, cudaMemcpyHostToDevice,
                                 sl->copy_stream));
      }
      sl->stats.cold_staged++;
      sl->stats.bytes_staged += (int64_t)(sl->bytes_gu + sl->bytes_dn + (fp8 ? sl->bytes_sgu + sl->bytes_sdn : 0));
    }
    MOE_CUDA(cudaEventRecord(sl->ev_ready[buf], sl->copy_stream));
    MOE_CUDA(cudaStreamWaitEvent(s, sl->ev_ready[buf], 0));
    st = run_gemms(ctx, sl, W, ws, T, bn, perm_src, perm_k, offsets, topk_w, y_pair, le + r.e_off, lm + r.e_off,
                   np + r.p_off, r.L, ntile_bound, s, false, false);
    if (st != MOE_OK) return st;
    MOE_CUDA(cudaEventRecord(sl->ev_free[buf], s));
  }
  MOE_CUDA(cudaEventRecord(sl->ev_done, s));
  sl->ev_done_valid = true;
  return lru_push_async(sl, s);
}

}  // namespace

extern "C" {

moe_status_t moe_route(moe_ctx_t* ctx, const void* x, const float* w_router, const float* logit_bias, int T,
                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((st = check_ws(ctx, T, ws, ws_bytes)) != MOE_OK) return st;
  return route_impl(ctx, x, w_router, logit_bias, T, topk_idx, topk_w, ws, static_cast<cudaStream_t>(stream));
}

moe_status_t moe_permute(moe_ctx_t* ctx, const int32_t* topk_idx, int T, int32_t* counts, int32_t* offsets,
                         int32_t* perm_src, int32_t* perm_k, int32_t* inv, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (!counts || !offsets) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if (T > 0 && (!topk_idx || !perm_src || !perm_k || !inv)) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((st = check_ws(ctx, T, ws, ws_bytes)) != MOE_OK) return st;
  return permute_impl(ctx, topk_idx, T, counts, offsets, perm_src, perm_k, inv, ws, static_cast<cudaStream_t>(stream),
                      false);
}

moe_status_t moe_expert_ffn(moe_ctx_t* ctx, moe_slots_t* sl, const void* x, const int32_t* perm_src,
                            const int32_t* perm_k, const int32_t* offsets, const float* topk_w, int T,
                            float* y_pair, void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ctx || !sl) return fail(MOE_ERR_INVALID_ARG, "NULL context or slot table");
  if (sl->ctx != ctx) return fail(MOE_ERR_SLOT, "slot table belongs to another context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !perm_src || !perm_k || !offsets || !topk_w || !y_pair) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((st = check_ws(ctx, T, ws, ws_bytes)) != MOE_OK) return st;
  return ffn_impl(ctx, sl, x, perm_src, perm_k, offsets, topk_w, T, y_pair, ws, static_cast<cudaStream_t>(stream),
                  false, false);
}

moe_status_t moe_combine(moe_ctx_t* ctx, const float* y_pair, const int32_t* inv, int T, void* out,
                         moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!y_pair || !inv || !out) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  Prof p(ctx, MOE_PROF_COMBINE, static_cast<cudaStream_t>(stream));
  MOE_CUDA(launch_combine(y_pair, inv, T, ctx->cfg.top_k, ctx->cfg.hidden, out, static_cast<cudaStream_t>(stream),
                          false));
  return MOE_OK;
}

moe_status_t moe_forward(moe_ctx_t* ctx, moe_slots_t* sl, const void* x, const float* w_router,
                         const float* logit_bias, int T, void* out, void* ws, size_t ws_bytes,
                         moe_stream_t stream) {
  if (!ctx || !sl) return fail(MOE_ERR_INVALID_ARG, "NULL context or slot table");
  if (sl->ctx != ctx) return fail(MOE_ERR_SLOT, "slot table belongs to another context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !out) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((st = check_ws(ctx, T, ws, ws_bytes)) != MOE_OK) return st;
  const moe_config_t& c = ctx->cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const WsLayout W = ws_layout(c, T);
  int32_t* idx = at<int32_t>(ws, W.topk_idx);
  float* w = at<float>(ws, W.topk_w);
  int32_t* counts = at<int32_t>(ws, W.counts);
  int32_t* offsets = at<int32_t>(ws, W.offsets);
  int32_t* ps = at<int32_t>(ws, W.perm_src);
  int32_t* pk = at<int32_t>(ws, W.perm_k);
  int32_t* inv = at<int32_t>(ws, W.inv);
  float* y = at<float>(ws, W.y_pair);
  const bool resident = sl->n_host == 0;
  const bool chain = ctx->chain;
  if (residency_device_path_ok(ctx, sl, x, T)) {
    // decode with host-resident experts: router -> cache plan -> copies of the missed experts (none when
    // every routed expert is resident or cached) -> FFN planned from the top-k -> combine
    int* sched = at<int>(ws, W.sched);
    const int sched_n = 1 + std::min(c.n_experts, T * c.top_k);
    bool planned = false;  // up to 4 tokens the router's last CTA runs the cache plan after the top-k
    if ((st = route_impl(ctx, x, w_router, logit_bias, T, idx, w, ws, s, sched, sched_n, &sl->rdev, sl->d_map_of,
                         &planned)) != MOE_OK)
      return st;
    if (!planned) {
      Prof p(ctx, MOE_PROF_PERMUTE, s);
      MOE_CUDA(launch_residency_plan(idx, T * c.top_k, c.n_experts, sl->rdev, sl->d_map_of, s, chain));
    }
    {
      Prof p(ctx, MOE_PROF_GATHER, s);
      MOE_CUDA(launch_residency_copy(sl->rdev, sl->spare, ctx->num_sms, s, chain));
    }
    if (c.wdtype == MOE_BF16) {
      if ((st = ffn_decode_impl(ctx, sl, x, idx, w, T, y, ws, s, sched)) != MOE_OK) return st;
    } else {
      // FP8: the permutation and tile plan read the expert -> map table the cache plan just updated
      bool planned = false;
      if ((st = permute_impl(ctx, idx, T, counts, offsets, ps, pk, inv, ws, s, chain, sl->d_map_of,
                             ffn_block_n(T, c.wdtype), x, nullptr, &planned)) != MOE_OK)
        return st;
      if ((st = ffn_impl(ctx, sl, x, ps, pk, offsets, w, T, y, ws, s, chain, planned, inv, true)) != MOE_OK)
        return st;
    }
    sl->last_dev = true;
    Prof p(ctx, MOE_PROF_COMBINE, s);
    MOE_CUDA(launch_combine(y, inv, T, c.top_k, c.hidden, out, s, chain));
    return MOE_OK;
  }
  if (decode_path_ok(ctx, sl, x, T)) {
    // decode: router (which also zeroes the FFN's counters) -> FFN planned from the top-k -> combine
    int* sched = at<int>(ws, W.sched);
    const int sched_n = 1 + std::min(c.n_experts, T * c.top_k);
    if ((st = route_impl(ctx, x, w_router, logit_bias, T, idx, w, ws, s, sched, sched_n)) != MOE_OK) return st;
    if ((st = ffn_decode_impl(ctx, sl, x, idx, w, T, y, ws, s, sched)) != MOE_OK) return st;
    Prof p(ctx, MOE_PROF_COMBINE, s);
    MOE_CUDA(launch_combine(y, inv, T, c.top_k, c.hidden, out, s, chain));
    return MOE_OK;
  }
  // route (first kernel: ordinary stream order with whatever came before)
  if ((st = route_impl(ctx, x, w_router, logit_bias, T, idx, w, ws, s)) != MOE_OK) return st;
  // permutation (+ tile plan + sorted bf16 rows when the batch is small)
  bool planned = false;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  if ((st = permute_impl(ctx, idx, T, counts, offsets, ps, pk, inv, ws, s, chain, resident ? sl->d_map_of : nullptr,
                         ffn_block_n(T, c.wdtype), x, (resident && c.wdtype == MOE_BF16) ? at<void>(ws, W.x_perm) : nullptr,
                         &planned)) != MOE_OK)
    return st;
  if ((st = ffn_impl(ctx, sl, x, ps, pk, offsets, w, T, y, ws, s, chain, planned, inv)) != MOE_OK) return st;
  Prof p(ctx, MOE_PROF_COMBINE, s);
  MOE_CUDA(launch_combine(y, inv, T, c.top_k, c.hidden, out, s, resident && chain));
  return MOE_OK;
}

// ---------------------------------------------------- expert parallelism --

moe_status_t moe_ep_pack(moe_ctx_t* ctx, const void* x, const float* topk_w, const int32_t* perm_src,
                         const int32_t* perm_k, const int32_t* offsets, int T, void* x_send, float* w_send,
                         moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  moe_status_t st = check_T(ctx, T);
  if (st != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  if (!x || !topk_w || !perm_src || !perm_k || !offsets || !x_send || !w_send)
    return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(x_send)) % 16)
    return fail(MOE_ERR_INVALID_ARG, "x and x_send must be 16-byte aligned");
  const moe_config_t& c = ctx->cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Prof p(ctx, MOE_PROF_GATHER, s);
  MOE_CUDA(launch_ep_pack(x, topk_w, perm_src, perm_k, offsets, c.n_experts, c.top_k, T * c.top_k, c.hidden, x_send,
                          w_send, s));
  return MOE_OK;
}

moe_status_t moe_ep_recv_plan(moe_ctx_t* ctx, const int32_t* recv_counts, int n_src, int32_t* offsets,
                              int32_t* perm_src, int32_t* perm_k, int32_t* inv, moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  if (!recv_counts || !offsets || !perm_src || !perm_k || !inv) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if (n_src <= 0) return fail(MOE_ERR_INVALID_ARG, "n_src must be positive");
  if ((long long)n_src * ctx->cfg.n_experts > 1024)
    return fail(MOE_ERR_UNSUPPORTED, "n_src * E must be <= 1024 (E = this context's experts)");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Prof p(ctx, MOE_PROF_PERMUTE, s);
  MOE_CUDA(launch_ep_recv_plan(recv_counts, n_src, ctx->cfg.n_experts, offsets, perm_src, perm_k, inv, s));
  return MOE_OK;
}

moe_status_t moe_ep_gather_rows(moe_ctx_t* ctx, const float* src, const int32_t* idx, int n_rows, float* dst,
                                moe_stream_t stream) {
  if (!ctx) return fail(MOE_ERR_INVALID_ARG, "NULL context");
  if (n_rows < 0) return fail(MOE_ERR_INVALID_ARG, "n_rows must be >= 0");
  if (n_rows == 0) return MOE_OK;
  if (!src || !idx || !dst) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) % 16)
    return fail(MOE_ERR_INVALID_ARG, "src and dst must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Prof p(ctx, MOE_PROF_GATHER, s);
  MOE_CUDA(launch_ep_gather_rows_f32(src, idx, n_rows, ctx->cfg.hidden, dst, s));
  return MOE_OK;
}

moe_status_t moe_quantize_e4m3(const void* src, int rows, int cols, int block_rows, uint8_t* q, float* scales,
                               moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 128) return fail(MOE_ERR_INVALID_ARG, "need rows >= 0 and cols % 128 == 0");
  if (block_rows != 1 && block_rows != 128) return fail(MOE_ERR_UNSUPPORTED, "block_rows must be 1 or 128");
  if (rows == 0) return MOE_OK;
  if (!src || !q || !scales) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  MOE_CUDA(launch_quant_e4m3(src, rows, cols, block_rows, q, scales, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status_t moe_quantize_mx(const void* src, int rows, int cols, int elem, uint8_t* q, uint8_t* scales,
                             moe_stream_t stream) {
  if (rows < 0 || cols <= 0 || cols % 32) return fail(MOE_ERR_INVALID_ARG, "need rows >= 0 and cols % 32 == 0");
  if (elem != 0 && elem != 1) return fail(MOE_ERR_INVALID_ARG, "elem must be 0 (E2M1) or 1 (E4M3)");
  if (rows == 0) return MOE_OK;
  if (!src || !q || !scales) return fail(MOE_ERR_INVALID_ARG, "NULL tensor");
  if ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(q)) % 16)
    return fail(MOE_ERR_INVALID_ARG, "src and q must be 16-byte aligned");
  MOE_CUDA(launch_quant_mx(src, rows, cols, elem, q, scales, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

// ----------------------------------------------------------------- slots --

moe_status_t moe_slots_create(moe_slots_t** out, moe_ctx_t* ctx, int n_spare) {
  if (!out || !ctx || n_spare < 0) return fail(MOE_ERR_INVALID_ARG, "bad argument");
  *out = nullptr;
  if (ctx->cfg.wdtype == MOE_MXFP4 && n_spare > 0)
    return fail(MOE_ERR_UNSUPPORTED, "MXFP4 experts are HBM-resident only (no spare slots)");
  const moe_config_t& c = ctx->cfg;
  const bool fp8 = c.wdtype == MOE_FP8_E4M3_B128;
  moe_slots_t* sl = new moe_slots_t();
  sl->ctx = ctx;
  sl->E = c.n_experts;
  sl->n_spare = n_spare;
  sl->loc.assign(sl->E, -1);
  sl->gu.assign(sl->E, nullptr);
  sl->dn.assign(sl->E, nullptr);
  sl->sgu.assign(sl->E, nullptr);
  sl->sdn.assign(sl->E, nullptr);
  sl->sf_blk.assign(sl->E, nullptr);
  sl->h_maps.assign(sl->E + n_spare, MapEntry{});
  sl->h_map_of.assign(sl->E, -1);
  const size_t esz = fp8 ? 1 : 2;
  sl->bytes_gu = 2ull * c.intermediate * c.hidden * esz;
  sl->bytes_dn = (size_t)c.hidden * c.intermediate * esz;
  sl->bytes_sgu = fp8 ? (2ull * c.intermediate / 128) * (c.hidden / 128) * 4 : 0;
  sl->bytes_sdn = fp8 ? ((size_t)c.hidden / 128) * (c.intermediate / 128) * 4 : 0;
  sl->off_dn = align256(sl->bytes_gu);
  sl->off_sgu = sl->off_dn + align256(sl->bytes_dn);
  sl->off_sdn = sl->off_sgu + align256(sl->bytes_sgu);
  sl->slot_bytes = sl->off_sdn + align256(sl->bytes_sdn);
  auto cleanup = [&](moe_status_t st, const std::string& msg) {
    moe_slots_destroy(sl);
    return fail(st, msg);
  };
  if (lib_malloc(&sl->d_maps, sizeof(MapEntry) * (sl->E + n_spare)) != cudaSuccess)
    return cleanup(MOE_ERR_OOM, "cudaMalloc of the map table failed");
  if (lib_malloc(&sl->d_map_of, sizeof(int32_t) * sl->E) != cudaSuccess)
    return cleanup(MOE_ERR_OOM, "cudaMalloc of the slot index failed");
  if (n_spare > 0 && lib_malloc(&sl->spare, sl->slot_bytes * n_spare) != cudaSuccess)
    return cleanup(MOE_ERR_OOM, "cudaMalloc of the spare slots failed");
  sl->h_pinned_ints = (size_t)(sl->E + 1) + 4 * (size_t)sl->E + 256;
  if (lib_host_alloc(&sl->h_pinned, sizeof(int32_t) * sl->h_pinned_ints) != cudaSuccess)
    return cleanup(MOE_ERR_OOM, "cudaHostAlloc failed");
  if (cudaStreamCreateWithFlags(&sl->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
    return cleanup(MOE_ERR_CUDA, "cudaStreamCreate failed");
  for (int i = 0; i < 2; ++i) {
    if (cudaEventCreateWithFlags(&sl->ev_ready[i], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&sl->ev_free[i], cudaEventDisableTiming) != cudaSuccess)
      return cleanup(MOE_ERR_CUDA, "cudaEventCreate failed");
  }
  if (cudaEventCreateWithFlags(&sl->ev_done, cudaEventDisableTiming) != cudaSuccess)
    return cleanup(MOE_ERR_CUDA, "cudaEventCreate failed");
  sl->slot_expert.assign(n_spare, -1);
  sl->expert_slot.assign(sl->E, -1);
  sl->slot_tick.assign(n_spare, -1);
  sl->h_host.assign(sl->E, HostRec{});
  sl->unmapped.assign(sl->E, 0);
  if (n_spare > 0) {
    // the LRU state on the device: loc, host records, slot_expert, slot_tick, expert_slot, tick, copy list, stats
    const size_t E_ = sl->E;
    size_t o = 0;
    auto take = [&](size_t bytes) {
      const size_t at = o;
      o += align256(bytes);
      return at;
    };
    const size_t o_loc = take(E_ * 4), o_host = take(E_ * sizeof(HostRec)), o_se = take(n_spare * 4),
                 o_st = take(n_spare * 8), o_es = take(E_ * 4), o_tick = take(8), o_cn = take(4),
                 o_ce = take(n_spare * 4), o_cs = take(n_spare * 4), o_stats = take(8 * 8);
    uint8_t* d = nullptr;
    if (lib_malloc(&d, o) != cudaSuccess) return cleanup(MOE_ERR_OOM, "cudaMalloc of the residency state failed");
    sl->d_res = d;
    ResidencyDev& r = sl->rdev;
    r.loc = reinterpret_cast<const int32_t*>(d + o_loc);
    r.host = reinterpret_cast<const HostRec*>(d + o_host);
    r.slot_expert = reinterpret_cast<int32_t*>(d + o_se);
    r.slot_tick = reinterpret_cast<long long*>(d + o_st);
    r.expert_slot = reinterpret_cast<int32_t*>(d + o_es);
    r.tick = reinterpret_cast<long long*>(d + o_tick);
    r.copy_n = reinterpret_cast<int32_t*>(d + o_cn);
    r.copy_e = reinterpret_cast<int32_t*>(d + o_ce);
    r.copy_slot = reinterpret_cast<int32_t*>(d + o_cs);
    r.stats = reinterpret_cast<long long*>(d + o_stats);
    r.status_word = ctx->d_status;
    r.n_spare = n_spare;
    r.slot_bytes = sl->slot_bytes;
    r.part_off[0] = 0;
    r.part_off[1] = sl->off_dn;
    r.part_off[2] = sl->off_sgu;
    r.part_off[3] = sl->off_sdn;
    r.part_bytes[0] = sl->bytes_gu;
    r.part_bytes[1] = sl->bytes_dn;
    r.part_bytes[2] = sl->bytes_sgu;
    r.part_bytes[3] = sl->bytes_sdn;
    if (cudaMemset(d, 0xff, o) != cudaSuccess ||  // -1 everywhere ...
        cudaMemset(d + o_host, 0, E_ * sizeof(HostRec)) != cudaSuccess ||
        cudaMemset(d + o_tick, 0, 8) != cudaSuccess || cudaMemset(d + o_cn, 0, 4) != cudaSuccess ||
        cudaMemset(d + o_stats, 0, 64) != cudaSuccess)  // ... except the records, tick, copy count, stats
      return cleanup(MOE_ERR_CUDA, "cudaMemset of the residency state failed");
    sl->h_lru_words = 9 + (size_t)n_spare + (2 * (size_t)n_spare + 2 * E_ + 1) / 2 + 1;
    if (lib_host_alloc(&sl->h_lru, 2 * sl->h_lru_words * sizeof(int64_t)) != cudaSuccess)
      return cleanup(MOE_ERR_OOM, "cudaHostAlloc of the residency staging failed");
  }
  for (int i = 0; i < n_spare; ++i) {
    uint8_t* slot = sl->spare + (size_t)i * sl->slot_bytes;
    moe_status_t st = make_entry(ctx, &sl->h_maps[sl->E + i], slot, slot + sl->off_dn,
                                 fp8 ? reinterpret_cast<const float*>(slot + sl->off_sgu) : nullptr,
                                 fp8 ? reinterpret_cast<const float*>(slot + sl->off_sdn) : nullptr);
    if (st != MOE_OK) {
      std::string m = g_last_error;
      return cleanup(st, m);
    }
  }
  if (cudaMemcpy(sl->d_maps, sl->h_maps.data(), sizeof(MapEntry) * (sl->E + n_spare), cudaMemcpyHostToDevice) !=
          cudaSuccess ||
      cudaMemcpy(sl->d_map_of, sl->h_map_of.data(), sizeof(int32_t) * sl->E, cudaMemcpyHostToDevice) != cudaSuccess)
    return cleanup(MOE_ERR_CUDA, "cudaMemcpy of the slot table failed");
  *out = sl;
  return MOE_OK;
}

moe_status_t moe_slots_destroy(moe_slots_t* sl) {
  if (!sl) return MOE_OK;
  if (sl->copy_stream) cudaStreamSynchronize(sl->copy_stream);
  for (int i = 0; i < 2; ++i) {
    if (sl->ev_ready[i]) cudaEventDestroy(sl->ev_ready[i]);
    if (sl->ev_free[i]) cudaEventDestroy(sl->ev_free[i]);
  }
  if (sl->ev_done) cudaEventDestroy(sl->ev_done);
  if (sl->copy_stream) cudaStreamDestroy(sl->copy_stream);
  if (sl->h_pinned) cudaFreeHost(sl->h_pinned);
  if (sl->spare) cudaFree(sl->spare);
  if (sl->d_maps) cudaFree(sl->d_maps);
  if (sl->d_map_of) cudaFree(sl->d_map_of);
  if (sl->d_res) cudaFree(sl->d_res);
  if (sl->h_lru) cudaFreeHost(sl->h_lru);
  for (uint8_t* b : sl->sf_blk)
    if (b) cudaFree(b);
  delete sl;
  return MOE_OK;
}

moe_status_t moe_slots_register(moe_slots_t* sl, int expert, const void* w_gu, const void* w_dn, const void* s_gu_,
                                const void* s_dn_, int location) {
  if (!sl) return fail(MOE_ERR_INVALID_ARG, "NULL slot table");
  if (expert < 0 || expert >= sl->E) return fail(MOE_ERR_SLOT, "expert index out of range");
  if (!w_gu || !w_dn) return fail(MOE_ERR_INVALID_ARG, "NULL weights");
  const moe_config_t& c = sl->ctx->cfg;
  const bool scaled = c.wdtype != MOE_BF16;
  if (scaled != (s_gu_ != nullptr) || scaled != (s_dn_ != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "scales must be given for FP8 and MXFP4 weights and only for them");
  if (location != MOE_LOC_HBM && location != MOE_LOC_HOST_PINNED) return fail(MOE_ERR_INVALID_ARG, "bad location");
  if (c.wdtype == MOE_MXFP4 && location != MOE_LOC_HBM)
    return fail(MOE_ERR_UNSUPPORTED, "MXFP4 experts are HBM-resident only");
  const float* s_gu = static_cast<const float*>(s_gu_);
  const float* s_dn = static_cast<const float*>(s_dn_);
  std::lock_guard<std::mutex> lock(sl->mu);
  if (sl->d_res) {  // the cache state as the device-side path left it
    MOE_CUDA(cudaDeviceSynchronize());
    moe_status_t st = lru_pull_async(sl, nullptr);
    if (st != MOE_OK) return st;
    MOE_CUDA(cudaDeviceSynchronize());
    lru_unpack(sl);
  }
  if (location == MOE_LOC_HBM) {
    const uintptr_t align = c.wdtype == MOE_MXFP4 ? 32 : 16;  // packed E2M1 tensor maps need 32-byte bases
    if ((reinterpret_cast<uintptr_t>(w_gu) | reinterpret_cast<uintptr_t>(w_dn)) % align)
      return fail(MOE_ERR_INVALID_ARG, c.wdtype == MOE_MXFP4 ? "MXFP4 weights must be 32-byte aligned"
                                                             : "device weights must be 16-byte aligned");
    if (c.wdtype == MOE_MXFP4) {
      // the scales, rearranged once into the block layout the tensor cores read (owned by the table)
      const int H = c.hidden, I = c.intermediate;
      const size_t gu_blk = (size_t)(2 * I / 128) * (H / 128) * 512, dn_blk = (size_t)(H / 128) * (I / 128) * 512;
      uint8_t* blk = nullptr;
      if (lib_malloc(&blk, gu_blk + dn_blk) != cudaSuccess) return fail(MOE_ERR_OOM, "cudaMalloc of MXFP4 scales failed");
      cudaError_t err = launch_mx_block_scales(static_cast<const uint8_t*>(s_gu_), 2 * I, H, I, blk, nullptr);
      if (err == cudaSuccess)
        err = launch_mx_block_scales(static_cast<const uint8_t*>(s_dn_), H, I, 0, blk + gu_blk, nullptr);
      if (err == cudaSuccess) err = cudaStreamSynchronize(nullptr);
      if (err != cudaSuccess) {
        cudaFree(blk);
        return fail(MOE_ERR_CUDA, std::string("MXFP4 scale layout: ") + cudaGetErrorString(err));
      }
      if (sl->sf_blk[expert]) cudaFree(sl->sf_blk[expert]);
      sl->sf_blk[expert] = blk;
      s_gu = reinterpret_cast<const float*>(blk);
      s_dn = reinterpret_cast<const float*>(blk + gu_blk);
    }
    MapEntry me;
    moe_status_t st = make_entry(sl->ctx, &me, w_gu, w_dn, s_gu, s_dn);
    if (st != MOE_OK) return st;
    sl->h_maps[expert] = me;
    sl->h_map_of[expert] = expert;
    MOE_CUDA(cudaMemcpy(sl->d_maps + expert, &me, sizeof(MapEntry), cudaMemcpyHostToDevice));
  } else {
    sl->h_map_of[expert] = -1;
  }
  if (sl->expert_slot[expert] >= 0) {  // its cached copy no longer matches
    sl->slot_expert[sl->expert_slot[expert]] = -1;
    sl->slot_tick[sl->expert_slot[expert]] = -1;
    sl->expert_slot[expert] = -1;
  }
  const int prev = sl->loc[expert];
  if (prev == MOE_LOC_HOST_PINNED) sl->n_host--;
  if (location == MOE_LOC_HOST_PINNED) sl->n_host++;
  sl->loc[expert] = location;
  sl->gu[expert] = w_gu;
  sl->dn[expert] = w_dn;
  sl->sgu[expert] = s_gu;
  sl->sdn[expert] = s_dn;
  MOE_CUDA(cudaMemcpy(sl->d_map_of + expert, &sl->h_map_of[expert], sizeof(int32_t), cudaMemcpyHostToDevice));
  if (sl->d_res) {
    // device side: where the expert lives, its record's device-visible addresses (pinned host memory is
    // mapped into the device's address space), and the cache state
    HostRec hr{};
    char unm = 0;
    if (location == MOE_LOC_HOST_PINNED) {
      const void* parts[4] = {w_gu, w_dn, s_gu, s_dn};
      for (int i = 0; i < 4; ++i) {
        if (!parts[i]) continue;
        void* dp = nullptr;
        if (cudaHostGetDevicePointer(&dp, const_cast<void*>(parts[i]), 0) != cudaSuccess || !dp) {
          cudaGetLastError();  // not mapped: this expert keeps the host-synchronised path
          unm = 1;
          break;
        }
        hr.p[i] = dp;
      }
    }
    sl->n_unmapped += (int)unm - (int)sl->unmapped[expert];
    sl->unmapped[expert] = unm;
    sl->h_host[expert] = hr;
    MOE_CUDA(cudaMemcpy(const_cast<int32_t*>(sl->rdev.loc) + expert, &location, sizeof(int32_t),
                        cudaMemcpyHostToDevice));
    MOE_CUDA(cudaMemcpy(const_cast<HostRec*>(sl->rdev.host) + expert, &hr, sizeof(HostRec), cudaMemcpyHostToDevice));
    moe_status_t st = lru_push_async(sl, nullptr);
    if (st != MOE_OK) return st;
    MOE_CUDA(cudaDeviceSynchronize());
  }
  return MOE_OK;
}

moe_status_t moe_slots_query(const moe_slots_t* sl, int expert, int* location, int* slot) {
  if (!sl || !location || !slot) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  if (expert < 0 || expert >= sl->E) return fail(MOE_ERR_SLOT, "expert index out of range");
  *location = sl->loc[expert];
  *slot = sl->loc[expert] == MOE_LOC_HBM ? sl->h_map_of[expert] : -1;
  return MOE_OK;
}

moe_status_t moe_slots_set_policy(moe_slots_t* sl, int policy) {
  if (!sl) return fail(MOE_ERR_INVALID_ARG, "NULL slot table");
  if (policy != MOE_SLOTS_LRU && policy != MOE_SLOTS_PER_CALL) return fail(MOE_ERR_INVALID_ARG, "bad policy");
  std::lock_guard<std::mutex> lock(sl->mu);
  sl->policy = policy;
  if (sl->d_res) {
    MOE_CUDA(cudaDeviceSynchronize());
    moe_status_t st = lru_pull_async(sl, nullptr);  // keeps the tick
    if (st != MOE_OK) return st;
    MOE_CUDA(cudaDeviceSynchronize());
    lru_unpack(sl);
  }
  std::fill(sl->slot_expert.begin(), sl->slot_expert.end(), -1);
  std::fill(sl->expert_slot.begin(), sl->expert_slot.end(), -1);
  std::fill(sl->slot_tick.begin(), sl->slot_tick.end(), -1);
  if (sl->d_res) {
    moe_status_t st = lru_push_async(sl, nullptr);
    if (st != MOE_OK) return st;
    MOE_CUDA(cudaDeviceSynchronize());
  }
  return MOE_OK;
}

moe_status_t moe_slots_stats(const moe_slots_t* sl, moe_slots_stats_t* stats) {
  if (!sl || !stats) return fail(MOE_ERR_INVALID_ARG, "NULL argument");
  *stats = sl->stats;
  if (sl->d_res) {
    // counts of the device-side path: [0] last touched, [1] last routed host, [2] last hits, [3] last misses,
    // [4] hits, [5] misses (cumulative)
    int64_t dst[8];
    MOE_CUDA(cudaDeviceSynchronize());
    MOE_CUDA(cudaMemcpy(dst, sl->rdev.stats, sizeof(dst), cudaMemcpyDeviceToHost));
    if (sl->last_dev) {
      stats->last_touched = (int32_t)dst[0];
      stats->last_routed_cold = (int32_t)dst[1];
      stats->last_hits = (int32_t)dst[2];
      stats->last_cold = (int32_t)dst[3];
    }
    stats->cache_hits += dst[4];
    stats->cold_staged += dst[5];
    stats->bytes_staged += dst[5] * (int64_t)(sl->bytes_gu + sl->bytes_dn + sl->bytes_sgu + sl->bytes_sdn);
  }
  return MOE_OK;
}

moe_status_t moe_plan_hot_set(const int64_t* hist, int E, int n_hot, int32_t* hot) {
  if (!hist || !hot || E <= 0 || n_hot < 0 || n_hot > E) return fail(MOE_ERR_INVALID_ARG, "bad argument");
  std::vector<int> order(E);
  for (int e = 0; e < E; ++e) order[e] = e;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return hist[a] > hist[b]; });
  for (int i = 0; i < n_hot; ++i) hot[i] = order[i];
  return MOE_OK;
}

}  // extern "C"
