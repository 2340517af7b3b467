// internal.h -- declarations shared between the .cu files of libmoe (not part
// of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Per-slot TMA descriptors of one expert's weights (and FP8 scales), kept in
// a device array that the FFN kernels index by slot.
struct alignas(64) MapEntry {
  CUtensorMap gu;  // w_gu [2I, H]: box {128 B of K, 128 rows}
  CUtensorMap dn;  // w_dn [H, I]:  box {128 B of K, 128 rows}
  const float* s_gu;
  const float* s_dn;
};

enum FfnMode { kGateUp = 0, kDown = 1 };

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
};

// Launches one FFN GEMM (gate/up+SwiGLU or down*weight) over the tile list.
// act_map is the TMA descriptor of the activation operand (x_perm or h);
// max_tiles bounds the grid (CTAs past the real tile count exit at once).
cudaError_t launch_ffn_gemm(int mode, int wdtype, int bn, const CUtensorMap& act_map, const GemmArgs& a,
                            int max_tiles, cudaStream_t s);
size_t ffn_gemm_smem_bytes(int mode, int wdtype, int bn);

cudaError_t launch_router_logits(const void* x, const float* wr, const float* bias, int T, int H, int E,
                                 float* logits, cudaStream_t s);
cudaError_t launch_topk(const float* logits, int T, int E, int K, int32_t* idx, float* w, int* status,
                        cudaStream_t s);

// Permutation: rank -> scan -> scatter. chunk = tokens per warp-chunk.
int permute_chunk_tokens(int T, int K);
cudaError_t launch_permute_rank(const int32_t* idx, int T, int K, int E, int chunk, int32_t* rank,
                                int32_t* chunk_counts, int* status, cudaStream_t s);
cudaError_t launch_permute_scan(int32_t* chunk_counts, int n_chunks, int E, int32_t* counts, int32_t* offsets,
                                cudaStream_t s);
cudaError_t launch_permute_scatter(const int32_t* idx, const int32_t* rank, const int32_t* chunk_base,
                                   const int32_t* offsets, int T, int K, int E, int chunk, int32_t* perm_src,
                                   int32_t* perm_k, int32_t* inv, cudaStream_t s);

// FFN tile plan for the all-resident case: every expert with pairs, in order.
cudaError_t launch_ffn_plan(const int32_t* offsets, const int32_t* map_of, int E, int bn, int32_t* list_expert,
                            int32_t* list_map, int32_t* nt_prefix, int* status, cudaStream_t s);

cudaError_t launch_gather_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E, int P,
                               int H, void* x_perm, cudaStream_t s);
cudaError_t launch_gather_quant_rows(const void* x, const int32_t* perm_src, const int32_t* offsets, int E,
                                     int P, int H, uint8_t* xq, float* xs, cudaStream_t s);
cudaError_t launch_combine(const float* y, const int32_t* inv, int T, int K, int H, void* out, cudaStream_t s);
cudaError_t launch_quant_e4m3(const void* src, int rows, int cols, int block_rows, uint8_t* q, float* scales,
                              cudaStream_t s);
// Sets the text moe_last_error() returns on this thread.
void record_error(const char* msg);

cudaError_t launch_quant_rows_e4m3_count(const void* src, const int32_t* offsets, int E, int rows, int cols,
                                         uint8_t* q, float* scales, cudaStream_t s);

}  // namespace moe
