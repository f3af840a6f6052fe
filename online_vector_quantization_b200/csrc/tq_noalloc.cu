// Decode attention for callers that cannot allocate device memory.
//
// tq_decode_attn needs a caller-provided workspace (query fragments and split
// partials).  Some callers cannot obtain one: an inference engine that
// reserves all device memory up front for its own pool and runs our call from
// plugin code that has no handle on that pool, or a latency-critical decode
// loop where cudaMalloc's implicit device synchronization is not acceptable.
// This entry point runs the same kernels with the workspace taken from a fixed
// array in device memory that the library defines once (kStaticScratchBytes
// per GPU that loads the library, held until the process exits).  It never
// calls cudaMalloc, cudaFree or any allocating routine.

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "tq_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

// The shared scratch.  In host code this name is only a stand-in: the device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

// Driver calls that name the current context, looked up once through the
// runtime (no link-time dependency on the driver library).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

struct ScratchRecord {
  unsigned long long ctx_id = 0;  // context the address belongs to (0: none yet)
  void* ptr = nullptr;
};

std::mutex g_scratch_mu;
ScratchRecord g_scratch[kMaxDevices];

// Unique id of the calling thread's current context (ids are never reused
// within a process, unlike context handles); 0 when no context is current.
tq_status current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  static bool found = false;
  std::call_once(once, [] {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1{}, q2{};
    found = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  });
  if (!found) return tq::fail(TQ_ERR_CUDA, "tq_decode_attn_noalloc: driver entry points cuCtxGetCurrent/cuCtxGetId");
  CUcontext ctx = nullptr;
  *id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS) return tq::fail(TQ_ERR_CUDA, "tq_decode_attn_noalloc: cuCtxGetCurrent");
  if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return tq::fail(TQ_ERR_CUDA, "tq_decode_attn_noalloc: cuCtxGetId");
  return TQ_OK;
}

// Device address of the scratch array on the current device.  It is looked up
// once per device, by the first call there (with that device current), and
// again when the device's context was replaced since (after cudaDeviceReset
// the array lives at a new address).
tq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::cuda_fail(e, "tq_decode_attn_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return tq::fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn_noalloc: device index too large");
  unsigned long long ctx_id = 0;
  tq_status st = current_context_id(&ctx_id);
  if (st != TQ_OK) return st;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchRecord& rec = g_scratch[dev];
  if (!rec.ptr || ctx_id == 0 || rec.ctx_id != ctx_id) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);  // makes the device's context current if none was
    if (e != cudaSuccess || !ptr) return tq::cuda_fail(e, "tq_decode_attn_noalloc: cudaGetSymbolAddress");
    if (ctx_id == 0) {
      st = current_context_id(&ctx_id);
      if (st != TQ_OK) return st;
    }
    rec.ptr = ptr;
    rec.ctx_id = ctx_id;
  }
  *out = rec.ptr;
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_decode_attn_noalloc(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache,
                                            int B, int hq, int max_len, void* out, int out_dtype,
                                            const tq_attn_flags* flags, void* stream) {
  using tq::fail;
  // the same checks as tq_decode_attn (cache planes, sizes, alignment, flags)
  tq::DecodePlan plan;
  float thr = 0.f;
  unsigned long long* sv_stats = nullptr;
  tq_status st = tq::check_decode_call(p, q, q_dtype, cache, B, hq, max_len, out, out_dtype, flags,
                                       "tq_decode_attn_noalloc", &plan, &thr, &sv_stats);
  if (st != TQ_OK) return st;
  if (plan.ws_total_bytes > kStaticScratchBytes)
    return fail(TQ_ERR_CAPACITY, "tq_decode_attn_noalloc: this call needs " + std::to_string(plan.ws_total_bytes) +
                                     " bytes of scratch; the static scratch holds " +
                                     std::to_string(kStaticScratchBytes) + " (use tq_decode_attn with a workspace)");
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != TQ_OK) return st;
  // Nothing in the scratch needs to start at zero: every word a kernel reads
  // was written earlier in the same call.
  return tq::launch_decode(p, q, q_dtype == TQ_BF16, cache, plan, out, out_dtype == TQ_BF16, scratch, thr,
                           sv_stats, static_cast<cudaStream_t>(stream));
}
