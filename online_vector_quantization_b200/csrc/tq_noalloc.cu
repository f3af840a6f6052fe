// Decode attention for callers that cannot allocate device memory.
//
// tq_decode_attn needs a caller-provided workspace (query fragments and split
// partials).  Some callers cannot obtain one: an
// inference engine that reserves all device memory up front for its own pool
// and runs our call from plugin code that has no handle on that pool, or a
// latency-critical decode loop where cudaMalloc's implicit device
// synchronization is not acceptable.  This entry point runs the same kernels
// with the workspace taken from a fixed array in device memory that the
// library defines once (kStaticScratchBytes per GPU that loads the library,
// held until the process exits).  It never calls cudaMalloc, cudaFree or any
// allocating routine.

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

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (the first call on a device does this).
tq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::cuda_fail(e, "tq_decode_attn_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return tq::fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn_noalloc: device index too large");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) return tq::cuda_fail(e, "tq_decode_attn_noalloc: cudaGetSymbolAddress");
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return TQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

extern "C" tq_status tq_decode_attn_noalloc(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache,
                                            int B, int hq, int max_len, void* out, int out_dtype,
                                            const tq_attn_flags* flags, void* stream) {
  using tq::fail;
  if (!p) return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: NULL params");
  if (!cache) return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: NULL cache");
  if (cache->n_seq < 1 || cache->n_kv_heads < 1 || cache->capacity < 0 || cache->capacity % 64 || cache->n_sink < 0 ||
      !cache->lens || !cache->status || !cache->k_norms || !cache->v_norms)
    return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: bad cache");
  if (B < 1 || B > cache->n_seq || hq < 1 || max_len < 0 || (q_dtype != TQ_F32 && q_dtype != TQ_BF16) ||
      (out_dtype != TQ_F32 && out_dtype != TQ_BF16))
    return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: bad B, hq, max_len or dtype");
  const int hkv = cache->n_kv_heads;
  if (hq % hkv) return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: hq must be a multiple of n_kv_heads");
  if (hq / hkv > 8) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn_noalloc: at most 8 query heads per kv-head");
  if (max_len > cache->capacity + cache->n_sink)
    return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: max_len above the cache's capacity");
  if (!q || !out) return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: NULL q or out");
  if (!aligned16(q) || !aligned16(out)) return fail(TQ_ERR_ALIGN, "tq_decode_attn_noalloc: q and out must be 16-byte aligned");
  const float thr = flags ? flags->sparse_v_threshold : 0.f;
  if (!(thr >= 0.f) || thr >= 1.f) return fail(TQ_ERR_ARG, "tq_decode_attn_noalloc: sparse_v_threshold must be in [0, 1)");
  const tq::DecodePlan plan = tq::plan_decode(p, B, hq, hkv, max_len);
  if (plan.ws_total_bytes > kStaticScratchBytes)
    return fail(TQ_ERR_CAPACITY, "tq_decode_attn_noalloc: this call needs " + std::to_string(plan.ws_total_bytes) +
                                     " bytes of scratch; the static scratch holds " +
                                     std::to_string(kStaticScratchBytes) + " (use tq_decode_attn with a workspace)");
  void* scratch = nullptr;
  tq_status st = scratch_address(&scratch);
  if (st != TQ_OK) return st;
  // Nothing in the scratch needs to start at zero: every word a kernel reads
  // was written earlier in the same call.
  return tq::launch_decode(p, q, q_dtype == TQ_BF16, cache, plan, out, out_dtype == TQ_BF16, scratch, thr,
                           static_cast<cudaStream_t>(stream));
}
