/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts layer forward.
 *
 * The layer (DeepSeek-class routed MoE, as served by vLLM-Moet: topairepos.com
 * page, model table row "DeepSeek-V4.1-Flash ... MoET hybrid" -- 384 routed
 * experts per layer, top-k routing -- and the hybrid results table, rows
 * "identity" and "the step"):
 *
 *   moe_route       router logits l[t,e] = <x[t,:], Wr[e,:]> (+ bias[e]) in a
 *                   fixed fp32 order, top-k by (logit desc, expert asc),
 *                   weights w[t,k] = exp(l_k - l_0) / sum_j exp(l_j - l_0)
 *   moe_permute     per-expert counts, exclusive offsets, and the pairs (t,k)
 *                   sorted by (expert asc, token asc) ("compact MoE calls",
 *                   same page, hybrid results table, row "identity")
 *   moe_expert_ffn  per pair: h = bf16(silu(Wg x) * (Wu x)),
 *                   y_pair = w[t,k] * (Wd h)   (tcgen05 tensor-core GEMMs)
 *   moe_combine     out[t] = bf16(sum_k y_pair[inv[t,k]]), k ascending
 *   moe_forward     the four steps in one call
 *   moe_slots_*     expert residency: each expert lives in HBM or in pinned
 *                   host memory and is staged into a spare HBM slot when a
 *                   batch routes to it (the "hotsplit" recipes wiki, Home page:
 *                   hot experts resident, cold experts read from pinned host
 *                   memory on demand); results are bit-identical to the
 *                   all-resident run (vLLM-Moet page, hybrid results table,
 *                   row "identity").
 *
 * Conventions (all entry points):
 *   - Layout is row-major. x, out: [T, H] bf16. Router weight Wr: [E, H] fp32.
 *     Expert weights use the [out, in] convention: w_gu [2I, H] (rows 0..I-1
 *     gate, rows I..2I-1 up), w_dn [H, I]. bf16 data are passed as void*.
 *   - Pointers are DEVICE pointers unless stated. The caller owns every
 *     tensor, the workspace and the stream; the library owns only the
 *     context, the slot table and the slot table's spare HBM slots.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) unless its comment says it synchronises.
 *     Argument and shape checks are synchronous and return an error code
 *     without launching anything.
 *   - Errors the device detects (an expert id outside [0, E), an expert that
 *     is routed to but not registered, a bounded wait that ran out) set bits
 *     in the context's device status word (moe_get_device_status) and never
 *     trap. A pair with a bad expert id or an unregistered expert is dropped:
 *     moe_forward leaves it out of the token's sum (as if the token had one
 *     pair fewer), moe_expert_ffn writes its y_pair row as zeros. Outputs after
 *     a time-out are unspecified.
 *   - There is no CPU fallback: every step runs in this library's kernels.
 *
 * Size limits: H and I multiples of 128; 1 <= K <= 32; K <= E <= 1024;
 * 0 <= T <= 65536 (T * K < 2^31).
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_ctx moe_ctx_t;
typedef struct moe_slots moe_slots_t;
typedef void* moe_stream_t; /* cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, wrong enum, workspace too small */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside the size limits above, or no sm_100 device */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (see moe_last_error) */
  MOE_ERR_SLOT = 4,        /* slot-table misuse: unknown expert, slot table of another context */
  MOE_ERR_TIMEOUT = 5,     /* reported through the device status word */
  MOE_ERR_OOM = 6          /* the library could not allocate its own memory */
} moe_status_t;

typedef enum {
  MOE_BF16 = 0,          /* bf16 expert weights */
  MOE_FP8_E4M3_B128 = 1, /* e4m3 expert weights with fp32 scales per 128x128 block;
                            activations quantised to e4m3 per token per 128 columns */
  MOE_MXFP4 = 2          /* OCP MXFP4 expert weights: E2M1 codes packed two per byte
                            (element 2i in the low nibble) with one E8M0 scale byte
                            per 32 elements along K; activations and h quantised to
                            MX e4m3 (per token per 32 columns) inside the layer; the
                            tensor cores apply both scales (kind::mxf8f6f4.block_scale).
                            The pages' checkpoint ships FP4 experts (vLLM-Moet,
                            topairepos.com page, hybrid results table, row "quality,
                            paired against the native FP4 reference"); they name no
                            block format, and this is the open one. HBM-resident only;
                            H and I multiples of 256. */
} moe_wdtype_t;

enum { MOE_LOC_HBM = 0, MOE_LOC_HOST_PINNED = 1 };

/* Bits of the device status word. */
enum {
  MOE_DEV_BAD_EXPERT = 1, /* a top-k index outside [0, E) reached moe_permute */
  MOE_DEV_NO_SLOT = 2,    /* a pair was routed to an expert with no registered weights (pair dropped) */
  MOE_DEV_TIMEOUT = 4     /* a bounded wait inside a kernel gave up (~2 s) */
};

typedef struct {
  int hidden;       /* H */
  int n_experts;    /* E */
  int top_k;        /* K */
  int intermediate; /* I */
  int wdtype;       /* moe_wdtype_t */
  int flags;        /* MOE_FLAG_* bits, 0 = defaults */
} moe_config_t;

/* Config flags. */
enum {
  /* Launch every kernel in plain stream order instead of chaining the
   * kernels of one call with programmatic dependent launch. */
  MOE_FLAG_NO_PDL = 1
};

/* Creates a context on the CURRENT CUDA device (which must be sm_100).
 * Allocates the device status word. Synchronous. */
moe_status_t moe_ctx_create(moe_ctx_t** ctx, const moe_config_t* cfg);
moe_status_t moe_ctx_destroy(moe_ctx_t* ctx);

/* Bytes of workspace moe_forward / moe_expert_ffn / moe_route / moe_permute
 * need for T tokens. The caller allocates it on the context's device
 * (256-byte aligned) and may reuse it between calls on the same stream. */
size_t moe_workspace_size(const moe_ctx_t* ctx, int T);

/* Router: logits in the fixed order below, top-k, renormalised weights.
 *   x [T, H] bf16, w_router [E, H] fp32, logit_bias [E] fp32 or NULL.
 *   topk_idx [T, K] int32 out (by logit desc, expert asc), topk_w [T, K] fp32 out.
 * Logit order: partial j (j = 0..31) accumulates fmaf(x[h], Wr[e][h], acc)
 * from +0 over h = j, j+32, j+64, ... in increasing h; the 32 partials are
 * summed pairwise (p[j] += p[j+o], o = 16, 8, 4, 2, 1: an xor butterfly's
 * lane 0); then + bias[e] (one fp32 add). Ties between equal logits
 * (+0 == -0) go to the lower expert index.
 * Weights: fp32 expf(l_k - l_0), summed k ascending, then one IEEE divide. */
moe_status_t moe_route(moe_ctx_t* ctx, const void* x, const float* w_router, const float* logit_bias, int T,
                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Permutation (counting sort of the T*K pairs by expert, then token).
 *   counts [E], offsets [E+1] (exclusive scan of counts), perm_src [T*K]
 *   (token of each sorted pair), perm_k [T*K] (its top-k slot), inv [T*K]
 *   (inv[t*K+k] = sorted position of pair (t,k)). Bit-exact, deterministic.
 * A top-k index outside [0, E) sets MOE_DEV_BAD_EXPERT; that pair is left out
 * (inv = -1) and offsets[E] counts only the valid pairs. */
moe_status_t moe_permute(moe_ctx_t* ctx, const int32_t* topk_idx, int T, int32_t* counts, int32_t* offsets,
                         int32_t* perm_src, int32_t* perm_k, int32_t* inv, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* Grouped expert FFN over the sorted pairs.
 *   x [T, H] bf16; perm_src/perm_k/offsets from moe_permute; topk_w [T, K];
 *   y_pair [T*K, H] fp32 out, row p = w * (Wd h) for sorted pair p.
 * Expert weights come from `slots` (moe_slots_register). If any registered
 * expert lives in pinned host memory, this call reads offsets back to the host
 * (it synchronises `stream` once), stages the routed cold experts into spare
 * HBM slots on an internal copy stream, and computes them with the same
 * kernels as resident experts (bit-identical results). The slot table's
 * pinned staging buffer, its cache state and its spare slots are shared by
 * every call that uses the table: such calls must run on one stream, or the
 * caller must order them (an event), as with the workspace. */
moe_status_t moe_expert_ffn(moe_ctx_t* ctx, moe_slots_t* slots, const void* x, const int32_t* perm_src,
                            const int32_t* perm_k, const int32_t* offsets, const float* topk_w, int T,
                            float* y_pair, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Combine: out[t, :] = bf16_rne(((y[inv[t,0]] + y[inv[t,1]]) + ...) + y[inv[t,K-1]]).
 *   y_pair [T*K, H] fp32, inv [T*K] int32, out [T, H] bf16. Bit-exact. */
moe_status_t moe_combine(moe_ctx_t* ctx, const float* y_pair, const int32_t* inv, int T, void* out,
                         moe_stream_t stream);

/* The whole layer: route -> permute -> expert FFN -> combine.
 *   x [T, H] bf16, w_router [E, H] fp32, logit_bias [E] or NULL, out [T, H] bf16.
 * A token's output bits do not depend on the other tokens of the batch or on T. */
moe_status_t moe_forward(moe_ctx_t* ctx, moe_slots_t* slots, const void* x, const float* w_router,
                         const float* logit_bias, int T, void* out, void* ws, size_t ws_bytes,
                         moe_stream_t stream);

/* ---- expert parallelism ------------------------------------------------
 * Experts split into G contiguous ranges, one per GPU (GPU g holds experts
 * [g*E/G, (g+1)*E/G)); every pair is computed on the GPU that holds its
 * expert and its y_pair row comes back to the token's GPU, where the combine
 * runs in the usual order. The pages split each expert across their GPUs and
 * sum the slices over NCCL (vLLM-Moet, topairepos.com page, hybrid results
 * table, row "the step"; model table, "one expert as its 576-row slices"); a
 * cross-GPU sum would change the order of a token's additions, so here whole
 * pairs move instead and a token's output bits do not depend on G. The
 * exchange itself (two all-to-alls of rows, one of counts) is the caller's:
 * NCCL through torch.distributed in the Python binding (ep.py).
 *
 * Token GPU, after moe_route and moe_permute (context with all E experts):
 *   moe_ep_pack: x_send[p] = x[perm_src[p]] (bf16 [T*K, H]) and
 *   w_send[p] = topk_w[perm_src[p], perm_k[p]] (fp32 [T*K]) for the valid
 *   sorted pairs p < offsets[E]. Rows for GPU g are the range
 *   offsets[g*E/G] .. offsets[(g+1)*E/G]. x, x_send 16-byte aligned. */
moe_status_t moe_ep_pack(moe_ctx_t* ctx, const void* x, const float* topk_w, const int32_t* perm_src,
                         const int32_t* perm_k, const int32_t* offsets, int T, void* x_send, float* w_send,
                         moe_stream_t stream);

/* Expert GPU (a context with its E_loc = E/G experts and top_k = 1): the
 * received rows arrive grouped by source GPU (n_src of them) and, within a
 * source, by local expert; recv_counts [n_src][E_loc] gives each group's rows.
 * Writes the plan that sorts them by (local expert, source, arrival):
 * offsets [E_loc+1], perm_src [R] (sorted place -> received row), perm_k [R]
 * (zeros: each received row is one pair) and inv [R] (received row -> sorted
 * place), R = the sum of recv_counts. Feed x_recv, perm_src, perm_k, offsets
 * and w_recv (as topk_w [R, 1]) to moe_expert_ffn with T = R.
 * n_src * E_loc <= 1024. */
moe_status_t moe_ep_recv_plan(moe_ctx_t* ctx, const int32_t* recv_counts, int n_src, int32_t* offsets,
                              int32_t* perm_src, int32_t* perm_k, int32_t* inv, moe_stream_t stream);

/* fp32 row gather, dst[i, :] = src[idx[i], :] for i < n_rows, rows of H
 * (the context's hidden size) floats: on the expert GPU, with idx = inv from
 * moe_ep_recv_plan, it puts moe_expert_ffn's rows back in arrival order for
 * the return all-to-all. src, dst 16-byte aligned. */
moe_status_t moe_ep_gather_rows(moe_ctx_t* ctx, const float* src, const int32_t* idx, int n_rows, float* dst,
                                moe_stream_t stream);

/* FP8 block quantiser (used for weights with block_rows = 128 and for
 * activations with block_rows = 1): per block of block_rows x 128 elements,
 * s = amax / 448 (IEEE fp32 divide; 1 if the block is all zero) and
 * q = e4m3_rne_satfinite(v / s).
 *   src [rows, cols] bf16, cols % 128 == 0; q [rows, cols] e4m3 (uint8);
 *   scales [ceil(rows / block_rows), cols / 128] fp32. Bit-exact. */
moe_status_t moe_quantize_e4m3(const void* src, int rows, int cols, int block_rows, uint8_t* q, float* scales,
                               moe_stream_t stream);

/* MX quantiser (OCP Microscaling; the MXFP4 path's weights and activations):
 * per 32 consecutive elements of a row, X = 2^(floor(log2 amax) - emax)
 * (emax 2 for E2M1, 8 for E4M3; clamped to 2^-127 .. 2^127, 2^-127 for an
 * all-zero block) and q = encode(v / X), round to nearest even, saturating.
 *   src [rows, cols] bf16, cols % 32 == 0 (16-byte aligned rows);
 *   elem 0 (E2M1): q [rows, cols/2] packed, element 2i in the low nibble;
 *   elem 1 (E4M3): q [rows, cols];
 *   scales [rows, cols/32] E8M0 bytes (exponent + 127). Bit-exact. */
moe_status_t moe_quantize_mx(const void* src, int rows, int cols, int elem, uint8_t* q, uint8_t* scales,
                             moe_stream_t stream);

/* moe_route_noalloc -- the router (logits, top-k, weights; same kernels, same
 * order and results as moe_route) for callers that cannot allocate device
 * memory: engines that reserve HBM up front and hand it out only through
 * their own pool, latency-critical paths that cannot take cudaMalloc's
 * device-wide synchronisation, and plug-ins whose host process owns the
 * device allocator. There is no counterpart on the pages this library
 * follows; it is an interface convenience.
 *   x [T, H] bf16, w_router [E, H] fp32, logit_bias [E] or NULL (device),
 *   topk_idx [T, K] int32 out, topk_w [T, K] fp32 out (device).
 * Needs no context and allocates nothing: its only scratch, the [T, E] fp32
 * logits, is a fixed array of MOE_ROUTE_NOALLOC_MAX_LOGITS floats (256 KiB)
 * compiled into the library, present on every GPU that loads it until the
 * process exits. T * E above that limit returns MOE_ERR_UNSUPPORTED. The
 * first call on each device looks up the array's device address and keeps it
 * for that device's CUDA context; the first call in a new context (after
 * cudaDeviceReset) looks it up again. Make those calls before any stream
 * capture: a lookup during capture is refused with MOE_ERR_UNSUPPORTED. All
 * calls share the array: calls that overlap on the GPU (two streams, two host
 * threads) race and must be serialised by the caller. Size limits otherwise as
 * above; errors do not set a status word (there is no context). */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS 65536
moe_status_t moe_route_noalloc(const void* x, const float* w_router, const float* logit_bias, int T, int H, int E,
                               int K, int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* ---- expert-slot table (residency) ------------------------------------ */

/* Creates the slot table of `ctx` with n_spare_slots spare HBM slots
 * (allocated here, one expert each) for staging cold experts. Synchronous. */
moe_status_t moe_slots_create(moe_slots_t** slots, moe_ctx_t* ctx, int n_spare_slots);
moe_status_t moe_slots_destroy(moe_slots_t* slots);

/* Registers expert `expert`. location MOE_LOC_HBM: w_gu/w_dn (and s_gu/s_dn
 * for FP8) are device pointers, borrowed for the table's lifetime.
 * MOE_LOC_HOST_PINNED: they are page-locked host pointers (cudaHostAlloc or
 * cudaHostRegister), borrowed and kept pinned by the caller.
 * bf16: w_gu [2I, H], w_dn [H, I] bf16; s_gu, s_dn must be NULL.
 * FP8: w_gu [2I, H], w_dn [H, I] e4m3; s_gu [2I/128, H/128], s_dn [H/128, I/128] fp32.
 * MXFP4 (HBM only): w_gu [2I, H/2], w_dn [H, I/2] packed E2M1 bytes, 32-byte
 * aligned; s_gu [2I, H/32], s_dn [H, I/32] E8M0 bytes (uint8). The table
 * copies the scales into the tensor cores' block layout (memory it owns);
 * the codes are borrowed.
 * Device pointers must be 16-byte aligned. Synchronous. */
moe_status_t moe_slots_register(moe_slots_t* slots, int expert, const void* w_gu, const void* w_dn,
                                const void* s_gu, const void* s_dn, int location);

/* Reports where `expert` lives: *location = MOE_LOC_* or -1 if unregistered;
 * *slot = its resident index, or -1 for host-resident experts. */
moe_status_t moe_slots_query(const moe_slots_t* slots, int expert, int* location, int* slot);

typedef struct {
  int64_t calls;          /* moe_expert_ffn calls that used this table */
  int64_t cold_staged;    /* cold experts copied host -> HBM (cache misses), cumulative */
  int64_t bytes_staged;   /* bytes copied host -> HBM, cumulative */
  int32_t last_cold;      /* cold experts staged (copied) by the most recent call */
  int32_t last_touched;   /* experts with at least one pair in the most recent call */
  int64_t cache_hits;     /* routed host-resident experts found in a spare slot, cumulative */
  int32_t last_hits;      /* ... in the most recent call */
  int32_t last_routed_cold; /* routed host-resident experts in the most recent call */
} moe_slots_stats_t;

moe_status_t moe_slots_stats(const moe_slots_t* slots, moe_slots_stats_t* stats);

/* What the spare slots hold between calls (the pages' hybrid keeps a subset of
 * the experts on the cards and serves the rest from host memory; the recipes
 * wiki's cache variant keeps recently used experts resident).
 *   MOE_SLOTS_LRU (default): the spare slots are an LRU cache of host-resident
 *     experts. A routed host expert already in a slot is a hit (no copy); a
 *     miss takes the least recently used slot that the call does not need.
 *     Registering every expert as MOE_LOC_HOST_PINNED sends every expert
 *     through the cache. A call that routes more host experts than there are
 *     spare slots falls back to per-call staging and empties the cache.
 *   MOE_SLOTS_PER_CALL: every call copies its routed host experts again.
 * Results are bit-identical under either policy (the same kernels read the
 * same bytes). Synchronous with respect to the host; call between forwards. */
enum { MOE_SLOTS_LRU = 0, MOE_SLOTS_PER_CALL = 1 };
moe_status_t moe_slots_set_policy(moe_slots_t* slots, int policy);

/* Greedy hot set (the "hotsplit" recipes wiki, Home page: the planner picks
 * the experts with the largest routing share per byte from routing
 * histograms). All experts here have the same size, so this is the n_hot
 * experts with the largest counts, ties to the lower index. Host function.
 *   hist [E] counts (host), hot [n_hot] out (host), listed best first. */
moe_status_t moe_plan_hot_set(const int64_t* hist, int E, int n_hot, int32_t* hot);

/* ---- diagnostics ------------------------------------------------------ */

/* Test hook for failure detection: launches one thread on `stream` that
 * waits, with the library's bounded acquire-load loop, until *flag (a device
 * int32) is nonzero or limit_ns nanoseconds pass (%globaltimer). On time-out it
 * sets MOE_DEV_TIMEOUT in the device status word and returns; nothing traps,
 * and the context stays usable. limit_ns must be in (0, 2e9]: larger or
 * non-positive limits return MOE_ERR_INVALID_ARG without launching. */
moe_status_t moe_debug_wait_flag(moe_ctx_t* ctx, const int32_t* flag, int64_t limit_ns, moe_stream_t stream);

/* Test hook for failure detection on the host: the library's own allocations
 * of the given kind -- MOE_ALLOC_DEVICE (cudaMalloc: context words, slot
 * tables, spare slots, residency state, MXFP4 scale blocks), MOE_ALLOC_PINNED
 * (cudaHostAlloc: the slot tables' pinned staging words) or MOE_ALLOC_ANY --
 * let `skip` succeed and then fail the next n as if the memory were exhausted.
 * The calls that make them return MOE_ERR_OOM and release what they had
 * allocated. Process-wide; n = 0 disarms it. Negative counts or an unknown
 * kind return MOE_ERR_INVALID_ARG. The hook itself touches no device. */
enum { MOE_ALLOC_ANY = 0, MOE_ALLOC_DEVICE = 1, MOE_ALLOC_PINNED = 2 };
moe_status_t moe_debug_fail_allocs(int kind, int skip, int n);

/* Copies the device status word to *status (synchronises the context's
 * device); reset != 0 clears it afterwards. */
moe_status_t moe_get_device_status(moe_ctx_t* ctx, int32_t* status, int reset);

/* Text of the most recent error on this thread (empty if none). */
const char* moe_last_error(void);

/* Number of kernel launches this context has issued so far. */
int64_t moe_launch_count(const moe_ctx_t* ctx);

/* ---- kernel timing (tracing) ------------------------------------------ */
/* When enabled, every launch of this context is bracketed by a pair of CUDA
 * events recorded on the launching stream; moe_profile_read synchronises on
 * them and returns, per kernel kind, the summed device time and the launch
 * count since the last reset. Off by default (no events are recorded). */
typedef enum {
  MOE_PROF_ROUTER = 0,  /* router logits */
  MOE_PROF_TOPK = 1,    /* top-k + weights */
  MOE_PROF_PERMUTE = 2, /* rank + scan + scatter + tile plan */
  MOE_PROF_GATHER = 3,  /* activation rows in sorted order (+ FP8 quantiser) */
  MOE_PROF_GATE_UP = 4, /* gate/up GEMM + SwiGLU */
  MOE_PROF_DOWN = 5,    /* down GEMM * routing weight */
  MOE_PROF_QUANT = 6,   /* FP8 quantiser of h */
  MOE_PROF_COMBINE = 7, /* weighted combine */
  MOE_PROF_FFN_FUSED = 8, /* decode: gate/up + SwiGLU and down * weight in one launch */
  MOE_PROF_KINDS = 9
} moe_prof_kind_t;

moe_status_t moe_profile_enable(moe_ctx_t* ctx, int enable);
moe_status_t moe_profile_read(moe_ctx_t* ctx, int kind, double* total_ms, int64_t* launches, int reset);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_MOE_H */
