// Internal declarations shared by the host code and the CUDA kernels of libtq.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>
#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kDim = 128;       // head dimension handled by the kernels
constexpr int kSketch = 128;    // QJL sketch size m
constexpr int kMaxBits = 4;     // largest MSE width of the small codebook tables
constexpr int kBookSlots = 16;  // centroid slots per width in those tables
constexpr int kWideBits = 8;    // the 8-bit MSE width (256 levels) has tables of its own
constexpr int kSigSlots = kWideBits + 1;  // sigma per width, 0..8
constexpr int kCell8Max = 512;  // code-search cells of the 8-bit codebook (quantize kernels)

// One quantizer format (keys or values).
//   mse_bits: width of the uniform MSE part (bits, or bits-1 in prod mode);
//   mixed:    the first d/2 rotated coordinates use mse_bits+1;
//   prod:     a QJL sign row (m/8 bytes) and a residual norm follow.
// id packs the three into one small integer used to pick kernel variants.
struct FormatSpec {
  int total_bits = 0;
  int mse_bits = 0;
  int mixed = 0;
  int prod = 0;
  int code_bytes = 0;
  int qjl_bytes = 0;
  int id() const { return mse_bits | (mixed << 4) | (prod << 5); }
  int width(int j) const { return (mixed && j < kDim / 2) ? mse_bits + 1 : mse_bits; }
  bool wide() const { return mse_bits == kWideBits; }
};

}  // namespace tq

struct tq_params {
  tq_config cfg;
  tq::FormatSpec fk, fv;
  int device = 0;
  // host copies (fp64)
  std::vector<double> pi, s;
  // device tables, carved from one allocation
  void* block = nullptr;
  float* pi32 = nullptr;   // Pi   [d][d] row-major (y = Pi u)
  float* pit32 = nullptr;  // Pi^T [d][d]
  float* s32 = nullptr;    // S    [m][d]
  float* st32 = nullptr;   // S^T  [d][m]
  float* mt32 = nullptr;   // (S Pi^T)^T [d][m]: sketch of a rotated-domain residual
  double* pi64 = nullptr;  // Pi [d][d] fp64 (dequantize)
  double* s64 = nullptr;   // S  [m][d] fp64 (dequantize)
  float* cb32 = nullptr;   // centroids [kMaxBits+1][16] (row b = width b)
  float* cbs32 = nullptr;  // centroids times sigma_b, the values fed to fp16 MMAs
  float* sig32 = nullptr;  // sigma_b [kSigSlots]: scale making sigma_b*c near-exact in fp16
  float* bd32 = nullptr;   // decision bounds [kMaxBits+1][16]
  double* cb64 = nullptr;  // centroids fp64 [kMaxBits+1][16]
  int32_t* status32 = nullptr;  // device word that plain quantize kernels OR error bits into
  // 8-bit MSE codebook (256 levels): centroids, sigma-scaled centroids (the
  // decode tables), the 255 decision bounds, fp64 centroids (dequantize) and
  // the code-search cells of the positive half: cell c of width 1/cell8_inv_w
  // holds {number of positive bounds at or below its start, the one bound
  // inside it or +inf}.  Pi^T in fp64 for the 8-bit SIMT quantizer.
  float* cb8_32 = nullptr;
  float* cbs8_32 = nullptr;
  float* bd8_32 = nullptr;
  double* cb8_64 = nullptr;
  float2* cell8 = nullptr;
  int cell8_n = 0;
  float cell8_inv_w = 0.f;
  double* pit64 = nullptr;
  // Tensor-core B operands of the quantize kernels, each a 128 x 128 16-bit
  // tile in the 128-byte-swizzled K-major layout (32 KB; see kTcImg*)
  uint8_t* tc_img = nullptr;
  // The decode kernel's shared-memory lookup tables for the (fk, fv) pair,
  // built once on the device (tq_attn.cu) and bulk-copied by every decode
  // CTA at its start; lut_bytes = 0 when the pair has no decode kernel.
  uint8_t* lut_img = nullptr;
  size_t lut_bytes = 0;
};

namespace tq {
constexpr int kTcImgBytes = 128 * 128 * 2;
// images in tq_params::tc_img, in this order
enum { kTcImgPiHi = 0, kTcImgPiLo, kTcImgPiA, kTcImgPiB, kTcImgPiC, kTcImgMHi, kTcImgMLo, kTcImgCount };
}  // namespace tq

namespace tq {

tq_status fail(tq_status st, const std::string& msg);
tq_status cuda_fail(cudaError_t e, const char* what);

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device, calling the runtime only the first time a larger value is
// needed there (the attribute persists; the call costs host time on every
// launch otherwise).  One instantiation, and so one record, per kernel.
template <auto kernel>
cudaError_t ensure_dyn_smem(int bytes) {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> granted[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices)
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (granted[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  int cur = granted[dev].load(std::memory_order_relaxed);
  while (cur < bytes && !granted[dev].compare_exchange_weak(cur, bytes, std::memory_order_release)) {
  }
  return cudaSuccess;
}

// Prefer the largest shared-memory carveout for a small kernel that runs
// right before or after the decode kernel (query rotation, merge): an SM
// whose carveout already fits the decode kernel's 226 KB takes its CTA as
// soon as the small kernel's CTAs leave, without reconfiguring first.
template <auto kernel>
cudaError_t ensure_max_carveout() {
  constexpr int kMaxDevices = 64;
  static std::atomic<bool> done[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return e;
}

// Kernel launchers (defined in the .cu files).
tq_status launch_quantize(const tq_params* p, const FormatSpec& f, const void* x, int x_bf16,
                          int64_t n, const tq_packed* out, cudaStream_t st);
tq_status launch_append(const tq_params* p, const tq_cache* c, const int32_t* seq_ids,
                        const void* k, const void* v, int x_bf16, int n_tok, int n_seq,
                        cudaStream_t st);
tq_status launch_cache_rows(const tq_params* p, const tq_cache* c, int which, int seq, int kv_head, int row0,
                            int64_t n, const tq_packed* rows, int to_cache, cudaStream_t st);
tq_status launch_dequantize(const tq_params* p, const FormatSpec& f, const tq_packed* in,
                            int64_t n, float* out, cudaStream_t st);

struct DecodePlan {
  int B, hq, hkv, group, max_len, ctas, part_floats;
  size_t ws_qfrag_bytes;  // rotated-query fragments, then
  size_t ws_parts_bytes;  // the split partials
  size_t ws_total_bytes;
};
DecodePlan plan_decode(const tq_params* p, int B, int hq, int hkv, int max_len);
// Argument checks of a cache and of a whole decode call (tq_decode_attn and
// tq_decode_attn_noalloc share them): on success *plan and *thr are set.
tq_status check_cache(const tq_params* p, const tq_cache* c, const char* who);
tq_status check_decode_call(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache, int B, int hq,
                            int max_len, const void* out, int out_dtype, const tq_attn_flags* flags,
                            const char* who, DecodePlan* plan, float* thr, unsigned long long** sv_stats);
tq_status launch_decode(const tq_params* p, const void* q, int q_bf16, const tq_cache* c,
                        const DecodePlan& plan, void* out, int out_bf16, void* ws,
                        float sparse_thr, unsigned long long* sv_stats, cudaStream_t st);
// Size of the decode lookup-table image of a format pair (0: no decode
// kernel), and its construction into p->lut_img (legacy stream, synchronized).
size_t decode_lut_bytes(const FormatSpec& fk, const FormatSpec& fv);
tq_status build_decode_luts(tq_params* p);
size_t search_workspace_bytes();
int search_max_k();
tq_status launch_search(const tq_params* p, const FormatSpec& f, const tq_packed* db, int64_t n, const void* q,
                        int q_bf16, int n_queries, int k, float* scores, int64_t* rows, void* ws,
                        cudaStream_t st);

}  // namespace tq
