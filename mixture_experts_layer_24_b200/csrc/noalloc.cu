// noalloc.cu -- moe_route_noalloc: the router (logits + top-k) for callers
// that cannot allocate device memory.
//
// Who cannot allocate: a serving engine that reserves its share of HBM at
// start-up and hands memory out only through its own pool (a kernel library
// calling cudaMalloc behind its back would break that budget); code on a
// latency-critical path where cudaMalloc's implicit device-wide
// synchronisation is not acceptable; and plug-ins loaded into a host process
// whose allocator owns the device and offers them no allocation hook. None of
// them can create a moe_ctx_t (which allocates its status word) or hand this
// library a workspace, so this entry point takes sizes directly and keeps its
// only scratch -- the [T, E] fp32 logits between the two kernels -- in a
// fixed array compiled into the library.
//
// The array lives in device global memory of every GPU that loads the
// library, until the process exits. In host code its name is only a host-side
// stand-in, never a device address: the first call on each device (with that
// device current) looks the real address up with cudaGetSymbolAddress and
// keeps it, together with the id of the device's current CUDA context; later
// calls reuse it while that context is still the current one. A new context
// (after cudaDeviceReset, say) gets its address looked up again. Make the
// first call on a device, and the first after a reset, before any stream
// capture: a lookup that would happen while the stream is capturing is refused
// with MOE_ERR_UNSUPPORTED. All calls share the one array, which keeps the
// last call's contents; nothing in it needs to start at zero (every logit a
// call reads is written by that call first). Calls that overlap on the GPU --
// on two streams, or from two host threads -- race on the array and must be
// serialised by the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "internal.h"

namespace {

constexpr int kMaxLogits = MOE_ROUTE_NOALLOC_MAX_LOGITS;  // T * E limit
constexpr int kMaxDevices = 64;

__device__ __align__(256) float g_route_scratch[kMaxLogits];

std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

// The driver's context calls, resolved through the runtime (the library does
// not link libcuda directly).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Id of the calling thread's current CUDA context (0 if it cannot be read).
unsigned long long current_ctx_id() {
  if (!g_ctx_get_current || !g_ctx_get_id) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
      return 0;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS || !c || g_ctx_get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

moe_status_t bad(moe_status_t st, const std::string& msg) {
  moe::record_error(msg.c_str());
  return st;
}

}  // namespace

extern "C" moe_status_t moe_route_noalloc(const void* x, const float* w_router, const float* logit_bias, int T,
                                          int H, int E, int K, int32_t* topk_idx, float* topk_w,
                                          moe_stream_t stream) {
  if (T < 0 || H <= 0 || E <= 0 || K <= 0) return bad(MOE_ERR_INVALID_ARG, "sizes must be positive (T >= 0)");
  if (H % 128 || H > 8192) return bad(MOE_ERR_UNSUPPORTED, "H must be a multiple of 128 and <= 8192");
  if (K > 32 || K > E || E > 1024) return bad(MOE_ERR_UNSUPPORTED, "need 1 <= K <= 32 and K <= E <= 1024");
  if ((long long)T * E > kMaxLogits)
    return bad(MOE_ERR_UNSUPPORTED, "T * E = " + std::to_string((long long)T * E) +
                                        " exceeds the static scratch of moe_route_noalloc (" +
                                        std::to_string(kMaxLogits) + " logits); use moe_route with a workspace");
  if (T == 0) return MOE_OK;
  if (!x || !w_router || !topk_idx || !topk_w) return bad(MOE_ERR_INVALID_ARG, "NULL tensor");
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return bad(MOE_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices) return bad(MOE_ERR_UNSUPPORTED, "device ordinal out of range");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const unsigned long long ctx_id = current_ctx_id();  // 0: none current yet (the lookup below creates it)
    if (!g_scratch_ptr[dev] || ctx_id == 0 || ctx_id != g_scratch_ctx[dev]) {
      cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
      err = cudaStreamIsCapturing(s, &cap);
      if (err != cudaSuccess)
        return bad(MOE_ERR_CUDA, std::string("cudaStreamIsCapturing: ") + cudaGetErrorString(err));
      if (cap != cudaStreamCaptureStatusNone)
        return bad(MOE_ERR_UNSUPPORTED,
                   "moe_route_noalloc: the first call on a device (or after a device reset) looks up the static "
                   "scratch's address and cannot run during stream capture; call it once before capturing");
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_route_scratch);
      if (err != cudaSuccess || !p)
        return bad(MOE_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(err));
      g_scratch_ptr[dev] = static_cast<float*>(p);
      g_scratch_ctx[dev] = current_ctx_id();
    }
    scratch = g_scratch_ptr[dev];
  }
  err = moe::launch_router_logits(x, w_router, logit_bias, T, H, E, scratch, s);
  if (err != cudaSuccess) return bad(MOE_ERR_CUDA, std::string("router launch: ") + cudaGetErrorString(err));
  err = moe::launch_topk(scratch, T, E, K, topk_idx, topk_w, nullptr, s);
  if (err != cudaSuccess) return bad(MOE_ERR_CUDA, std::string("top-k launch: ") + cudaGetErrorString(err));
  return MOE_OK;
}
