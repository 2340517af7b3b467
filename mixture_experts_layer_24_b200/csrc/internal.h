// internal.h -- declarations shared between the .cu files of libmoe (not part
// of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

// Per-slot TMA descriptors of one expert's weights (and FP8 / MXFP4 scales),
// kept in a device array that the FFN kernels index by slot.
struct alignas(64) MapEntry {
  // bf16:  3-D maps (64 elements, rows, K/64 chunks), box {64, 128, kc} with
  //        kc = 1 (gu, dn) and kc = 2 (gu2, dn2);
  // FP8:   2-D maps in gu / dn, box {128 B of K, 128 rows};
  // MXFP4: 3-D maps in gu / dn over the packed E2M1 codes (two per byte),
  //        (128 elements, rows, K/128 blocks), box {128, 128, kMxKC}, each
  //        block landing unpacked (16 codes per 16 B); s_gu / s_dn point at the
  //        E8M0 scales in the tensor cores' 512-byte block layout (mx.cu).
  CUtensorMap gu;   // w_gu [2I, H]
  CUtensorMap dn;   // w_dn [H, I]
  CUtensorMap gu2;
  CUtensorMap dn2;
  const float* s_gu;
  const float* s_dn;
};

enum FfnMode { kGateUp = 0, kDown = 1 };

// 64-wide K chunks per pipeline stage (one 3-D TMA copy per operand) of the
// bf16 GEMMs, measured at BN = 128 (4096 and 16384 tokens): gate/up streams
// two weight operands per chunk, and one-chunk stages (4 of 48 KB in flight
// instead of 2 of 96 KB) ran 4-10% faster. A down GEMM with one weight
// operand has stages half that size, where two-chunk stages (3 of 64 KB) ran
// 7-24% faster than one-chunk ones; with two weight operands (two output
// blocks per h tile) it takes the gate/up depth.
constexpr int kBf16GateUpChunks = 1;
constexpr int kBf16DownChunks = 2;
// Chunks per stage of the separate bf16 down GEMM at N tile width bn: up to
// 128 it stages two weight operands (two 128-row output blocks) against each
// h tile, one chunk per stage like gate/up; at 256, one operand and two
// chunks. Its h tensor maps carry the same count per box.
constexpr int bf16_down_gemm_chunks(int bn) { return bn <= 128 ? kBf16GateUpChunks : kBf16DownChunks; }

// Launches `kern` on `s`, with programmatic stream serialisation when pdl is
// true (the kernel must then follow the pdl_wait / pdl_trigger rule).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// The token-column tile width the FFN GEMMs use for a batch of T tokens. It
// depends on T only, so the tile that computes a given pair does not depend on
// which experts are resident.
int ffn_block_n(int T, int wdtype);

// Launch arguments common to both FFN GEMMs.
struct GemmArgs {
  const MapEntry* maps;       // [n_maps]
  const int32_t* list_expert; // [L]: experts this launch computes
  const int32_t* list_map;    // [L]: map entry of each listed expert
  const int32_t* nt_prefix;   // [L+1]: exclusive prefix of token tiles per listed expert
  const int32_t* offsets;     // [E+1]: pair offsets per expert (sorted order)
  int L;
  int H, I, K;
  void* h_out;                // gate/up output: [P, I] bf16 (or e4m3 for FP8) ...
  float* h_scale;             // ... and its per-128-column scales [P, I/128] (FP8)
  float* y_out;               // down output: [P, H] fp32
  const float* topk_w;        // [T*K]
  const int32_t* perm_src;    // [P]
  const int32_t* perm_k;      // [P]
  const float* act_scale;     // FP8: scales of the activation operand [P, Kdim/128]
  int* status;
  int plan_ready;             // 1: the tile plan was written two or more launches back
                              // (read it, and start streaming weights, before pdl_wait)
  int* sched;                 // fused decode FFN: [0] tile counter, [1 + n] finished gate/up
                              // tiles of global N tile n (zeroed by the plan kernel)
  const uint8_t* act_sfb;     // MXFP4: the activation operand's E8M0 scales, blocked per N tile
  uint8_t* h_sfb;             // MXFP4 gate/up: h's scales, written blocked per N tile for the down GEMM
  const int32_t* h_nt_prefix; // MXFP4 gate/up: [L+1] N tiles of the down GEMM per listed expert ...
  int h_bn;                   // ... of this width (the blocks h_sfb is written in)
  int stages;                 // pipeline depth (set by the launcher)
  int est_tiles;              // host-side bound on the tiles of this launch
  int num_sms;
};

// Activation-operand TMA descriptors for box heights 16 .. 256 rows (the GEMMs
// pick, per tile, the smallest that holds its pairs).
struct alignas(64) ActMaps {
  CUtensorMap m[5];  // 16, 32, 64, 128, 256 (the bf16 down GEMM's widest tile)
};

// Launches one FFN GEMM (gate/up+SwiGLU or down*weight) over the tile list.
// act_map is the TMA descriptor of the activation operand (x_perm or h);
// max_tiles bounds the grid (CTAs past the real tile count exit at once).
cudaError_t launch_ffn_gemm(int mode, int wdtype, int bn, const CUtensorMap& act_map, const ActMaps* act_maps,
                            const GemmArgs& a, int max_tiles, cudaStream_t s, bool pdl);
// The FP8 GEMMs behind launch_ffn_gemm (bn 16, 32 or 64).
cudaError_t launch_ffn_fp8(int mode, int bn, const ActMaps& maps, const GemmArgs& a, int max_tiles, cudaStream_t s,
                           bool pdl);

// Fused decode FFN (bf16, bn <= 64): gate/up and down tiles of one forward in
// one persistent launch with a dynamic tile queue. xmaps: x_perm with one K
// chunk per box; hmaps: h with two. a.sched must be zeroed by the plan kernel.
cudaError_t launch_ffn_fused(int bn, const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a, int max_tiles,
                             cudaStream_t s, bool pdl);
constexpr int kFusedMaxBn = 64;
// FP8 counterpart (the gate/up epilogue also quantises h into a.h_out (e4m3
// codes [P, I]) and a.h_scale): xmaps over the e4m3 x rows, hmaps over hq.
cudaError_t launch_ffn_fp8_fused(int bn, const ActMaps& xmaps, const ActMaps& hmaps, const GemmArgs& a,
                                 int max_tiles, cudaStream_t s, bool pdl);

// The decode forward's FFN planned from the router's top-k inside the kernel
// (no permutation kernel, no gathered x): T <= 64 tokens, T*K <= 512 pairs,
// bf16, every expert resident, x 16-byte aligned. xmap: x [T, H] with box
// {64, TP, 1}, TP = T rounded up to 16 (48 -> 64); hmaps: h, two K chunks.
// a.sched: [0] tile counter, [1 + l] per touched expert, zeroed by the router.
struct DecodeArgs {
  const int32_t* topk_idx;  // [T*K] from the router
  const int32_t* map_of;    // [E] expert -> slot (map entry), -1 if not registered
  int T, E;
  int32_t* counts;          // [E]    written by CTA 0
  int32_t* offsets;         // [E+1]
  int32_t* perm_src;        // [P]
  int32_t* perm_k;          // [P]
  int32_t* inv;             // [P]
};
cudaError_t launch_ffn_decode(const CUtensorMap& xmap, const ActMaps& hmaps, const GemmArgs& a, const DecodeArgs& d,
                              int max_tiles, cudaStream_t s, bool pdl);
size_t ffn_decode_smem_bytes(int T, int E);
constexpr int kDecodeMaxT = 64, kDecodeMaxPairs = 512;
// entries of the fused kernel's counter array for a plan of up to n_list experts
inline int fused_sched_entries(int n_list) { return 1 + 2 * n_list + 64; }

cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t s);
cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w, int* status,
                        cudaStream_t s);

// Decode-regime router (T <= kRouteSmallMaxT): logits and top-k in one launch.
// counters: >= kRouteSmallMaxT zero-initialised words owned by the caller's
// context (each is returned to zero by the kernel that uses it).
constexpr int kRouteSmallMaxT = 64;
// rd / map_of: up to 4 tokens (one CTA then holds every token's top-k) the
// fused last CTA also runs the residency plan; *planned says whether it did.
struct ResidencyDev;
cudaError_t launch_route_small(const void* x, const float* wr, const float* bias, int T, int H, int E, int K,
                               float* logits, int32_t* idx, float* w, unsigned int* counters, int* status,
                               cudaStream_t s, bool pdl, int* sched = nullptr, int sched_n = 0,
                               const ResidencyDev* rd = nullptr, int32_t* map_of = nullptr, bool* planned = nullptr);
// Prefill-regime router logits (register-tiled fp32 GEMM in the same order).
cudaError_t launch_route_gemm(const void* x, const float* wr, const float* bias, int T, int H, int E,
                              float* logits, cudaStream_t s);
// Top-k + weights for any T, one warp per token (logits read through L2).
cudaError_t launch_topk_warp(const float* logits, int T, int E, int K, int32_t* idx, float* w, cudaStream_t s,
                             bool pdl);

// Small-batch permutation (T*K <= kPermuteSmallMaxPairs): counts, offsets, the
// sorted pairs, optionally the FFN tile plan (map_of != nullptr) and the row
// gather of x (x_perm != nullptr), in one launch of n_ctas CTAs.
constexpr int kPermuteSmallMaxPairs = 1024;
cudaError_t launch_permute_small(const int32_t* idx, int T, int K, int E, int32_t* counts, int32_t* offsets,
                                 int32_t* perm_src, int32_t* perm_k, int32_t* inv, const int32_t* map_of, int bn,
                                 int32_t* list_expert, int32_t* list_map, int32_t* nt_prefix, const void* x, int H,
                                 void* x_perm, int* status, cudaStream_t s, bool pdl, int* sched = nullptr,
                                 int sched_n = 0, int bn2 = 0, int32_t* nt_prefix2 = nullptr);

// Permutation: rank -> scan -> scatter. chunk = tokens per warp-chunk.
int permute_chunk_tokens(int T, int K);
cudaError_t launch_permute_rank(const int32_t* idx, int T, int K, int E, int chunk, int32_t* rank,
                                int32_t* chunk_counts, int* status, cudaStream_t s, bool pdl);
cudaError_t launch_permute_scan(int32_t* chunk_counts, int n_chunks, int E, int32_t* counts, int32_t* offsets,
                                cudaStream_t s, bool pdl);
cudaError_t launch_permute_scatter(const int32_t* idx, const int32_t* rank, const int32_t* chunk_base,
                                   const int32_t* offsets, int T, int K, int E, int chunk, int32_t* perm_src,
                                   int32_t* perm_k, int32_t* inv, cudaStream_t s, bool pdl);

// Pairs routed to an expert with no registered weights are dropped: their
// y_pair rows are zeroed and, with inv (the forward), their inv entries set to
// -1 so the combine skips them. y_pair == nullptr: nothing is dropped.
struct DropArgs {
  const int32_t* perm_src;
  const int32_t* perm_k;
  int K;
  int32_t* inv;     // nullable
  float* y_pair;    // [P, H]
  int H;
};

// FFN tile plan for the all-resident case: every expert with pairs, in order.
// With nt_prefix2, also the prefix of N tiles of width bn2 (a down GEMM tiled
// wider than gate/up; MXFP4).
cudaError_t launch_ffn_plan(const int32_t* offsets, const int32_t* map_of, int E, int bn, int32_t* list_expert,
                            int32_t* list_map, int32_t* nt_prefix, int* status, cudaStream_t s, bool pdl, int* sched,
                            int sched_n, const DropArgs& drop, int bn2 = 0, int32_t* nt_prefix2 = nullptr);
// Drops the sorted pairs [p0, p1) (one unregistered expert) as above.
cudaError_t launch_drop_pairs(int p0, int p1, const DropArgs& drop, cudaStream_t s);

cudaError_t launch_gather_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E, int P,
                               int H, void* x_perm, cudaStream_t s, bool pdl);
// FP8 activation rows of the forward: each token's row quantised once (per 128
// columns) and stored to its K sorted pair rows through inv.
cudaError_t launch_quant_scatter_rows(const void* x, const int32_t* inv, int T, int K, int H, uint8_t* xq, float* xs,
                                      cudaStream_t s, bool pdl);
cudaError_t launch_gather_quant_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E,
                                     int P, int H, uint8_t* xq, float* xs, cudaStream_t s, bool pdl);
cudaError_t launch_combine(const float* y, const int32_t* inv, int T, int K, int H, void* out, cudaStream_t s,
                           bool pdl);
cudaError_t launch_quant_e4m3(const void* src, int rows, int cols, int block_rows, uint8_t* q, float* scales,
                              cudaStream_t s);
// Expert parallelism (ep.cu): rows in sorted order for the all-to-all, the
// plan of the rows an expert GPU receives, and the fp32 row gather that puts
// results back in arrival order.
cudaError_t launch_ep_pack(const void* x, const float* topk_w, const int32_t* perm_src, const int32_t* perm_k,
                           const int32_t* offsets, int E, int K, int P, int H, void* x_send, float* w_send,
                           cudaStream_t s);
cudaError_t launch_ep_recv_plan(const int32_t* recv_counts, int G, int E_loc, int32_t* offsets_loc, int32_t* perm,
                                int32_t* perm_k, int32_t* inv, cudaStream_t s);
cudaError_t launch_ep_gather_rows_f32(const float* src, const int32_t* idx, int n_rows, int H, float* dst,
                                      cudaStream_t s);

// MXFP4 (mx.cu, ffn_mxfp4.cu).
cudaError_t launch_quant_mx(const void* src, int rows, int cols, int elem_e4m3, uint8_t* q, uint8_t* scales,
                            cudaStream_t s);
cudaError_t launch_mx_block_scales(const uint8_t* scales, int rows, int K, int split_rows, uint8_t* blocked,
                                   cudaStream_t s);
// K blocks (128 deep) per pipeline stage of the MXFP4 GEMMs: one 3-D copy per operand brings them all.
constexpr int kMxKC = 2;
cudaError_t launch_quant_mx_pairs(const void* x, const int32_t* perm_src, const int32_t* offsets,
                                  const int32_t* nt_prefix, int E, int bn, int P, int H, uint8_t* xq, uint8_t* sfb,
                                  cudaStream_t s, bool pdl);
// One MXFP4 GEMM (gate/up + SwiGLU + MX quantisation of h, or down * weight)
// over the tile list; act_maps: e4m3 activation maps of box heights 16..bn.
cudaError_t launch_ffn_mxfp4(int mode, int bn, const ActMaps& act_maps, const GemmArgs& a, int max_tiles,
                             cudaStream_t s, bool pdl);
constexpr int kMxfp4MaxBn = 64;

// Host-resident experts on the device path (residency.cu): the slot table's
// LRU state in device memory, and the device-visible addresses of every host
// expert's pinned record (gate/up, down, FP8 scales).
struct HostRec {
  const void* p[4];
};
struct ResidencyDev {
  const int32_t* loc;      // [E] MOE_LOC_* or -1
  const HostRec* host;     // [E]
  int32_t* slot_expert;    // [n_spare] expert held, -1 empty
  long long* slot_tick;    // [n_spare] call that last used the slot, -1 never
  int32_t* expert_slot;    // [E] its spare slot, -1 not cached
  long long* tick;         // calls so far (shared with the host-synchronised path)
  int32_t* copy_n;         // misses of the current call ...
  int32_t* copy_e;         // [n_spare] ... their experts ...
  int32_t* copy_slot;      // [n_spare] ... and slots
  long long* stats;        // [8] last touched, last routed host, last hits, last misses, hits, misses
  int* status_word;
  int n_spare;
  size_t slot_bytes;
  size_t part_off[4], part_bytes[4];
};
cudaError_t launch_residency_plan(const int32_t* idx, int P, int E, const ResidencyDev& rd, int32_t* map_of,
                                  cudaStream_t s, bool pdl);
cudaError_t launch_residency_copy(const ResidencyDev& rd, uint8_t* spare, int num_sms, cudaStream_t s, bool pdl);

// Sets the text moe_last_error() returns on this thread.
void record_error(const char* msg);

cudaError_t launch_quant_rows_e4m3_count(const void* src, const int32_t* offsets, int E, int rows, int cols,
                                         uint8_t* q, float* scales, cudaStream_t s, bool pdl);

}  // namespace moe
