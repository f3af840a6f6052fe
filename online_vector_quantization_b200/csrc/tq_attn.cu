// Decode attention over the packed TurboQuant cache.
//
// Method: page "TurboQuant-MLX: quantizzare pesi e KV cache per LLM
// open-weight su Mac", section "Il metodo TurboQuant, in breve": a key is
// ||k|| Pi^T c[idx] (+ the QJL correction sqrt(pi/2)/m ||r|| S^T z), so
//   <q, k> = ||k|| ( <Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, z> )
// and the query is rotated once; values are accumulated in the rotated (and
// sketch) domain and Pi^T (S^T) is applied once per output.  Sparse V
// ("Greetings from TurboQuant-MLX", item 3) and the bf16 attention sink
// (same page, item 1) follow the header tq.h.
//
// Kernels of one decode step
//   1. qrot_kernel: q -> Pi q (and S q), scaled by log2(e)/sqrt(d), stored as
//      fp16 MMA B-fragments in the workspace, once per (sequence, kv-head).
//   2. decode_kernel: grid (split, kv-head, sequence) + one sink CTA per
//      (sequence, kv-head).  Each warp walks 16-token tiles of its split:
//        scores S^T[16 tok x 8 heads] = C_k[16 x 128] Q~^T  (mma.sync m16n8k16)
//        online softmax (base 2), sparse-V mask, P' = p * ||v||
//        O^T[128 x 8 heads] += C_v^T[128 x 16 tok] P'^T    (mma.sync m16n8k16)
//      The dequantized codebook values for both MMAs come straight from
//      per-lane-replicated shared-memory tables indexed by packed code bytes
//      (two or four codes per lookup, no bank conflicts), so no fp16 tile is
//      ever written back to memory.  Warps merge in shared memory, the CTA
//      writes (m, l, acc) partials, and the last CTA of a (sequence, kv-head)
//      (atomic ticket, no spin-waits) merges the splits and applies Pi^T/S^T.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTok = 16;       // tokens per warp tile
constexpr int kMaxG = 8;       // query heads per kv-head (MMA N = 8)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQjlScale = 1.2533141373155003f / kSketch;  // sqrt(pi/2)/m
// Query fragments per (sequence, kv-head): [kstep 16][b0,b1][hi,lo][lane 32].
// The rotated query is split as hi = fp16(x), lo = fp16(x - hi), and both
// halves are multiplied with the same code fragment, so the query enters the
// scores with fp32-level accuracy.
constexpr int kQfragWords = 16 * 2 * 2 * 32;

// ---------------------------------------------------------------------------
// Formats (id = mse_bits | mixed << 3 | prod << 4).  Segments of the MSE row:
// one uniform segment of 128 coordinates, or (mixed) 64 coordinates at
// mse+1 bits followed by 64 at mse bits.
// ---------------------------------------------------------------------------
template <int F>
struct Fmt {
  static constexpr int mse = F & 7;
  static constexpr bool mixed = (F >> 3) & 1;
  static constexpr bool prod = (F >> 4) & 1;
  static constexpr int nseg = mixed ? 2 : (mse > 0 ? 1 : 0);
  static constexpr int code_bytes = mixed ? 8 * (2 * mse + 1) : 16 * mse;
  static constexpr int b0 = mixed ? mse + 1 : mse;
  static constexpr int nd0 = mixed ? 64 : 128;
  static constexpr int b1 = mse;
  static constexpr int byte1 = mixed ? 8 * (mse + 1) : 0;
  static constexpr bool uses(int b) { return (nseg > 0 && b0 == b) || (nseg > 1 && b1 == b); }
  __host__ __device__ static constexpr int width(int j) { return (mixed && j < 64) ? mse + 1 : mse; }
};

// Shared-memory lookup tables.  Region A (row stride 256 B): bytes [0,128) of
// row r hold, for each lane, half2(c4[r & 15], c4[r >> 4]); bytes [128, 256)
// of rows r < 64 hold half2(c3[r & 7], c3[r >> 3]).  Region B (row stride
// 256 B, 8 B per lane): four 2-bit centroids of byte r.  Entry (r, lane) sits
// at r*256 + lane*4 (or *8): every lane hits its own bank.
template <int KF, int VF>
struct Lut {
  static constexpr bool t4 = Fmt<KF>::uses(4) || Fmt<VF>::uses(4);
  static constexpr bool t3 = Fmt<KF>::uses(3) || Fmt<VF>::uses(3);
  static constexpr bool t2 = Fmt<KF>::uses(2) || Fmt<VF>::uses(2);
  static constexpr int region_a = t4 ? 65536 : (t3 ? 16384 : 0);
  static constexpr int region_b_off = region_a;
  static constexpr int bytes = region_a + (t2 ? 65536 : 0);
};

__device__ __forceinline__ uint32_t h2bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int N>
struct IntC {
  static constexpr int value = N;
};
template <int N, int I = 0, typename Fn>
__device__ __forceinline__ void static_for(Fn&& fn) {
  if constexpr (I < N) {
    fn(IntC<I>{});
    static_for<N, I + 1>(fn);
  }
}

__device__ __forceinline__ uint32_t lds32(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint32_t*>(smem + off);
}

__device__ __forceinline__ uint2 lds64(const unsigned char* smem, uint32_t off) {
  return *reinterpret_cast<const uint2*>(smem + off);
}

// byte k of w placed at bits 8..15, lane offset `lb` (< 256) at bits 0..7
__device__ __forceinline__ uint32_t byte_addr(uint32_t w, uint32_t lb, int k) {
  return __byte_perm(w, lb, 0x5504 | (k << 4));
}

// half2 of +-c from bits p and p+16 of w (bit set -> +c); c_bits = half2(c, c)
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int p, uint32_t c_bits) {
  const uint32_t x = w << (15 - p);
  return (~x & 0x80008000u) | c_bits;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- TMA bulk copies and mbarriers (PTX) ----------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory (no multicast); both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for a phase with a time limit (~0.5 s of SM clocks); false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > (1ll << 30)) return false;
  return true;
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

// LUT address of the 6-bit field at bit `off` of x: (field << 8) | lb, in a
// shift and one logic op.
template <int OFF>
__device__ __forceinline__ uint32_t addr6(uint64_t x, uint32_t lb) {
  uint32_t v;
  if constexpr (OFF >= 8)
    v = static_cast<uint32_t>(x >> (OFF - 8));
  else
    v = static_cast<uint32_t>(x) << (8 - OFF);
  return (v & 0x3F00u) | lb;
}

template <int N>
__device__ __forceinline__ uint64_t field_mask3() {
  uint64_t m = 0;
#pragma unroll
  for (int k = 0; k < N; ++k) m |= 7ull << (6 * k);
  return m;
}

// ---------------------------------------------------------------------------
// K side.  Thread (g, t) of a warp decodes tokens g and g+8 of a 16-token
// tile; within each segment it owns a contiguous quarter of the coordinates
// (ND/4 of them), consumed 4 per MMA k-step.
// ---------------------------------------------------------------------------
template <int B, int ND, int BYTE0>
struct KChunk {
  static constexpr int BYTES = ND * B / 32;
  static constexpr int WORDS = BYTES > 0 ? (BYTES + 3) / 4 : 1;
  static constexpr int KSTEPS = ND / 16;
  uint32_t w[WORDS];

  __device__ __forceinline__ void load(const uint8_t* row, int t) {
    const int o = BYTE0 + t * BYTES;
    if constexpr (BYTES == 16) {
      const uint4 v = *reinterpret_cast<const uint4*>(row + o);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BYTES == 12) {
      const uint32_t* p = reinterpret_cast<const uint32_t*>(row + o);
      w[0] = p[0]; w[1] = p[1]; w[2] = p[2];
    } else if constexpr (BYTES == 8) {
      const uint2 v = *reinterpret_cast<const uint2*>(row + o);
      w[0] = v.x; w[1] = v.y;
    } else if constexpr (BYTES == 6) {
      const int al = o & ~3;
      const uint32_t* p = reinterpret_cast<const uint32_t*>(row + al);
      const uint32_t lo = p[0], hi = p[1];
      const int sh = (o & 3) * 8;
      w[0] = __funnelshift_r(lo, hi, sh);
      w[1] = hi >> sh;
    } else {
      static_assert(BYTES == 4, "unsupported K chunk");
      w[0] = *reinterpret_cast<const uint32_t*>(row + o);
    }
  }

  // 64-bit window holding the 6-bit field p (3-bit chunks)
  template <int P>
  __device__ __forceinline__ uint32_t pair3(uint32_t lb) const {
    if constexpr (6 * P + 6 <= 64) {
      const uint64_t x = static_cast<uint64_t>(w[0]) | (static_cast<uint64_t>(w[WORDS > 1 ? 1 : 0]) << 32);
      return addr6<6 * P>(x, lb);
    } else {
      const uint64_t x = static_cast<uint64_t>(w[1]) | (static_cast<uint64_t>(w[WORDS > 2 ? 2 : 1]) << 32);
      return addr6<6 * P - 32>(x, lb);
    }
  }

  // k-step S: (lo, hi) = A-fragment registers for k = 2t..2t+1 and 2t+8..2t+9
  template <int S>
  __device__ __forceinline__ void decode(const unsigned char* smem, uint32_t lane4, uint32_t lane8,
                                         uint32_t c_bits, uint32_t& lo, uint32_t& hi) const {
    constexpr int s = S;
    if constexpr (B == 4) {
      const uint32_t ww = w[s >> 1];
      lo = lds32(smem, byte_addr(ww, lane4, 2 * (s & 1)));
      hi = lds32(smem, byte_addr(ww, lane4, 2 * (s & 1) + 1));
    } else if constexpr (B == 3) {
      lo = lds32(smem, pair3<2 * S>(lane4 + 128));
      hi = lds32(smem, pair3<2 * S + 1>(lane4 + 128));
    } else if constexpr (B == 2) {
      const uint2 v = lds64(smem, byte_addr(w[s >> 2], lane8, s & 3));
      lo = v.x;
      hi = v.y;
    } else {
      lo = sign_pair(w[0], 2 * s, c_bits);
      hi = sign_pair(w[0], 2 * s + 1, c_bits);
    }
  }

  // coordinate behind half e (0..3 = lo.x, lo.y, hi.x, hi.y) of k-step s
  __host__ __device__ static constexpr int dim(int dim0, int t, int s, int e) {
    return B == 1 ? dim0 + t * (ND / 4) + 2 * s + (e & 1) * 16 + (e >> 1)
                  : dim0 + t * (ND / 4) + 4 * s + e;
  }
};

// ---------------------------------------------------------------------------
// V side.  Thread (g, t) decodes tokens 2t, 2t+1, 2t+8, 2t+9 of the tile
// and, within each segment, the ND/8 coordinates g*ND/8 ..; A-fragment
// registers pair two tokens at one coordinate.
// ---------------------------------------------------------------------------
template <int B, int ND, int BYTE0>
struct VChunk {
  static constexpr int MT = ND / 16;          // m-tiles of the segment
  uint64_t x;

  __device__ __forceinline__ void load(const uint8_t* row, int g) {
    constexpr int bits = ND * B / 8;
    if constexpr (bits == 64) {
      x = *reinterpret_cast<const uint64_t*>(row + BYTE0 + 8 * g);
    } else if constexpr (bits == 32) {
      x = *reinterpret_cast<const uint32_t*>(row + BYTE0 + 4 * g);
    } else if constexpr (bits == 16) {
      x = *reinterpret_cast<const uint16_t*>(row + BYTE0 + 2 * g);
    } else if constexpr (bits == 48) {
      const int o = BYTE0 + 6 * g, al = o & ~3;
      const uint32_t* p = reinterpret_cast<const uint32_t*>(row + al);
      const uint64_t v = static_cast<uint64_t>(p[0]) | (static_cast<uint64_t>(p[1]) << 32);
      x = (v >> ((o & 3) * 8)) & 0xFFFFFFFFFFFFull;
    } else {
      static_assert(bits == 24, "unsupported V chunk");
      const int o = BYTE0 + 3 * g, al = o & ~3, sh = (o & 3) * 8;
      const uint32_t* p = reinterpret_cast<const uint32_t*>(row + al);
      uint64_t v = p[0];
      if (sh > 8) v |= static_cast<uint64_t>(p[1]) << 32;  // field crosses into the next word
      x = (v >> sh) & 0xFFFFFFull;
    }
  }

  // rows g (coordinate 2mt) and g+8 (2mt+1) for every m-tile, tokens (A, B)
  __device__ __forceinline__ static void decode(const VChunk& a, const VChunk& b, const unsigned char* smem,
                                                uint32_t lane4, uint32_t lane8, uint32_t c_bits,
                                                uint32_t (&rg)[MT], uint32_t (&rg8)[MT]) {
    if constexpr (B == 4) {
#pragma unroll
      for (int wd = 0; wd < MT / 4; ++wd) {
        const uint32_t xa = static_cast<uint32_t>(a.x >> (32 * wd));
        const uint32_t xb = static_cast<uint32_t>(b.x >> (32 * wd));
        const uint32_t ev = (xa & 0x0F0F0F0Fu) | ((xb << 4) & 0xF0F0F0F0u);
        const uint32_t od = ((xa >> 4) & 0x0F0F0F0Fu) | (xb & 0xF0F0F0F0u);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          rg[4 * wd + k] = lds32(smem, byte_addr(ev, lane4, k));
          rg8[4 * wd + k] = lds32(smem, byte_addr(od, lane4, k));
        }
      }
    } else if constexpr (B == 3) {
      const uint64_t m = field_mask3<MT>();
      const uint64_t ev = (a.x & m) | ((b.x & m) << 3);
      const uint64_t od = ((a.x >> 3) & m) | (b.x & (m << 3));
      const uint32_t lb = lane4 + 128;
      static_for<MT>([&](auto kk) {
        constexpr int k = decltype(kk)::value;
        rg[k] = lds32(smem, addr6<6 * k>(ev, lb));
        rg8[k] = lds32(smem, addr6<6 * k>(od, lb));
      });
    } else if constexpr (B == 2) {
      const uint32_t xa = static_cast<uint32_t>(a.x), xb = static_cast<uint32_t>(b.x);
      const uint32_t ev = (xa & 0x33333333u) | ((xb & 0x33333333u) << 2);
      const uint32_t od = ((xa >> 2) & 0x33333333u) | (xb & 0xCCCCCCCCu);
#pragma unroll
      for (int j = 0; j < MT / 2; ++j) {
        const uint2 e = lds64(smem, byte_addr(ev, lane8, j));
        const uint2 o = lds64(smem, byte_addr(od, lane8, j));
        rg[2 * j] = e.x;
        rg[2 * j + 1] = e.y;
        rg8[2 * j] = o.x;
        rg8[2 * j + 1] = o.y;
      }
    } else {
      const uint32_t wv = (static_cast<uint32_t>(a.x) & 0xFFFFu) | (static_cast<uint32_t>(b.x) << 16);
#pragma unroll
      for (int k = 0; k < MT; ++k) {
        rg[k] = sign_pair(wv, 2 * k, c_bits);
        rg8[k] = sign_pair(wv, 2 * k + 1, c_bits);
      }
    }
  }

  __host__ __device__ static constexpr int dim(int dim0, int g, int mt, int r) {
    return dim0 + g * (ND / 8) + 2 * mt + r;
  }
};

template <int F>
struct KRow {
  using S0 = KChunk<Fmt<F>::b0, Fmt<F>::nd0, 0>;
  using S1 = KChunk<(Fmt<F>::nseg > 1 ? Fmt<F>::b1 : 4), 64, Fmt<F>::byte1>;
  using Q = KChunk<1, 128, 0>;
};
template <int F>
struct VRow {
  using S0 = VChunk<Fmt<F>::b0, Fmt<F>::nd0, 0>;
  using S1 = VChunk<(Fmt<F>::nseg > 1 ? Fmt<F>::b1 : 4), 64, Fmt<F>::byte1>;
  using Q = VChunk<1, 128, 0>;
};

struct DecodeArgs {
  const void* q;
  int q_bf16;
  const uint8_t* k_codes;
  const float* k_norms;
  const uint8_t* k_qjl;
  const float* k_res;
  const uint8_t* v_codes;
  const float* v_norms;
  const uint8_t* v_qjl;
  const float* v_res;
  const uint16_t* k_sink;
  const uint16_t* v_sink;
  const int32_t* lens;
  int32_t* status;
  int hkv, group, hq, capacity, n_sink, max_len, n_splits, split_tokens, part_floats;
  float* parts;
  int32_t* tickets;
  const uint32_t* qfrag;
  void* out;
  int out_bf16;
  const float* pit;  // Pi^T
  const float* st;   // S^T
  const float* pi;   // Pi
  const float* s;    // S
  const float* cbs;  // sigma-scaled centroids [5][16] (the values the MMAs see)
  const float* sig;  // sigma per width [5]
  float sparse_thr;
  int pack;          // 1: group <= 4, query hi/lo halves share one MMA (columns g and g+4)
};

__device__ __forceinline__ float load_q(const void* q, int bf16, int64_t i) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]) : reinterpret_cast<const float*>(q)[i];
}

// ---------------------------------------------------------------------------
// 1. query rotation: one CTA per (sequence, kv-head).  Threads 0..127 form
//    Pi q for all heads (one output coordinate each), threads 128..255 form
//    S q (prod keys); then the fp16 B-fragments are written.
// ---------------------------------------------------------------------------
template <int KF>
__global__ void __launch_bounds__(kThreads) qrot_kernel(DecodeArgs a) {
  using KR = KRow<KF>;
  using FK = Fmt<KF>;
  __shared__ float qs[kMaxG][kDim];
  __shared__ float qt[kMaxG][kDim];
  __shared__ float qsk[kMaxG][kSketch];
  const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = a.group;
  for (int i = tid; i < kMaxG * kDim; i += kThreads) {
    const int h = i / kDim, d = i % kDim;
    qs[h][d] = h < G ? load_q(a.q, a.q_bf16, (static_cast<int64_t>(b) * a.hq + kvh * G + h) * kDim + d) : 0.f;
  }
  __syncthreads();
  const float scale = kLog2e * rsqrtf(static_cast<float>(kDim));
  {
    const int j = tid & (kDim - 1);
    const bool sketch = tid >= kDim;
    if (!sketch || FK::prod) {
      const float* mat = sketch ? a.st : a.pit;  // [k][j] layouts, coalesced over j
      float acc[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) acc[h] = 0.f;
#pragma unroll 8
      for (int k = 0; k < kDim; ++k) {
        const float m = __ldg(mat + k * kDim + j);
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) acc[h] = fmaf(m, qs[h][k], acc[h]);
      }
      if (sketch) {
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) qsk[h][j] = acc[h] * scale;
      } else {
        const int wj = FK::width(j);
        const float f = wj > 0 ? scale / a.sig[wj] : 0.f;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) qt[h][j] = acc[h] * f;
      }
    }
  }
  __syncthreads();
  // B fragments: lane (g, t) supplies column g; k-steps 0..7 from the MSE
  // segments, 8..15 from the QJL segment.  Unpacked: column g = head g, halves
  // hi (x = 0) and lo (x = 1).  Packed (group <= 4): column g < 4 = hi of head
  // g, column g >= 4 = lo of head g - 4, in x = 0.
  uint32_t* dst = const_cast<uint32_t*>(a.qfrag) + (static_cast<int64_t>(b) * a.hkv + kvh) * kQfragWords;
  for (int i = tid; i < 16 * 32; i += kThreads) {
    const int ks = i / 32, lane = i % 32, g = lane >> 2, t = lane & 3;
    int dims[4] = {0, 0, 0, 0};
    bool valid = true;
    const bool qjl = ks >= 8;
    if (!qjl) {
      if (FK::nseg == 0) {
        valid = false;
      } else if (FK::nseg == 1 || ks < KR::S0::KSTEPS) {
        for (int e = 0; e < 4; ++e) dims[e] = KR::S0::dim(0, t, ks, e);
      } else {
        for (int e = 0; e < 4; ++e) dims[e] = KR::S1::dim(64, t, ks - KR::S0::KSTEPS, e);
      }
    } else {
      if (!FK::prod) valid = false;
      for (int e = 0; e < 4; ++e) dims[e] = KR::Q::dim(0, t, ks - 8, e);
    }
    const int head = a.pack ? (g & 3) : g;
    const float* src = qjl ? qsk[head] : qt[head];
    uint32_t hi[2] = {0, 0}, lo[2] = {0, 0};
    if (valid) {
      for (int r = 0; r < 2; ++r) {
        const float x0 = src[dims[2 * r]], x1 = src[dims[2 * r + 1]];
        const __half2 h = __floats2half2_rn(x0, x1);
        const float2 hf = __half22float2(h);
        hi[r] = *reinterpret_cast<const uint32_t*>(&h);
        lo[r] = h2bits(x0 - hf.x, x1 - hf.y);
      }
    }
    for (int r = 0; r < 2; ++r) {
      if (a.pack) {
        dst[((ks * 2 + r) * 2 + 0) * 32 + lane] = g < 4 ? hi[r] : lo[r];
        dst[((ks * 2 + r) * 2 + 1) * 32 + lane] = 0;
      } else {
        dst[((ks * 2 + r) * 2 + 0) * 32 + lane] = hi[r];
        dst[((ks * 2 + r) * 2 + 1) * 32 + lane] = lo[r];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Split merge (last CTA of a (sequence, kv-head)): combine the partials and
// apply Pi^T (and S^T) once per output.
// ---------------------------------------------------------------------------
template <int VF>
__device__ void merge_unit(const DecodeArgs& a, int b, int kvh, int n_real, bool has_sink, float* sm) {
  constexpr bool VPROD = Fmt<VF>::prod;
  const int tid = threadIdx.x, G = a.group;
  const int PF = a.part_floats;
  const float* base = a.parts + (static_cast<int64_t>(b) * a.hkv + kvh) * (a.n_splits + 1) * kMaxG * PF;
  float* acc = sm;                         // [kMaxG][2*kDim] rotated | sketch
  float* osk = sm + kMaxG * 2 * kDim;      // [kMaxG][kDim] sink, original domain
  float* mm = osk + kMaxG * kDim;          // [kMaxG]: M
  float* ll = mm + kMaxG;                  // [kMaxG]: L
  if (tid < kMaxG) {
    float M = -INFINITY;
    for (int sp = 0; sp < n_real; ++sp) M = fmaxf(M, __ldcg(base + (sp * kMaxG + tid) * PF));
    if (has_sink) M = fmaxf(M, __ldcg(base + (a.n_splits * kMaxG + tid) * PF));
    float L = 0.f;
    for (int sp = 0; sp < n_real; ++sp) {
      const float* pp = base + (sp * kMaxG + tid) * PF;
      L += __ldcg(pp + 1) * exp2f(__ldcg(pp) - M);
    }
    if (has_sink) {
      const float* pp = base + (a.n_splits * kMaxG + tid) * PF;
      L += __ldcg(pp + 1) * exp2f(__ldcg(pp) - M);
    }
    mm[tid] = M;
    ll[tid] = L;
  }
  __syncthreads();
  const int width = VPROD ? 2 * kDim : kDim;
  for (int i = tid; i < G * width; i += kThreads) {
    const int h = i / width, j = i % width;
    float s = 0.f;
    for (int sp = 0; sp < n_real; ++sp) {
      const float* pp = base + (sp * kMaxG + h) * PF;
      s += __ldcg(pp + 2 + j) * exp2f(__ldcg(pp) - mm[h]);
    }
    if (j < kDim) s = Fmt<VF>::width(j) > 0 ? s / a.sig[Fmt<VF>::width(j)] : 0.f;
    acc[h * 2 * kDim + j] = s;
  }
  for (int i = tid; i < G * kDim; i += kThreads) {
    const int h = i / kDim, j = i % kDim;
    float s = 0.f;
    if (has_sink) {
      const float* pp = base + (a.n_splits * kMaxG + h) * PF;
      s = __ldcg(pp + 2 + j) * exp2f(__ldcg(pp) - mm[h]);
    }
    osk[h * kDim + j] = s;
  }
  __syncthreads();
  for (int i = tid; i < G * kDim; i += kThreads) {
    const int h = i / kDim, o = i % kDim;
    float r = 0.f;
    const float* ah = acc + h * 2 * kDim;
    for (int j = 0; j < kDim; ++j) r = fmaf(a.pi[j * kDim + o], ah[j], r);
    if (VPROD) {
      float z = 0.f;
      for (int l = 0; l < kSketch; ++l) z = fmaf(a.s[l * kDim + o], ah[kDim + l], z);
      r = fmaf(kQjlScale, z, r);
    }
    const float L = ll[h];
    const float val = L > 0.f ? (r + osk[h * kDim + o]) / L : 0.f;
    const int64_t oi = (static_cast<int64_t>(b) * a.hq + kvh * G + h) * kDim + o;
    if (a.out_bf16)
      reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(val);
    else
      reinterpret_cast<float*>(a.out)[oi] = val;
  }
}

// Publish this CTA's partial; the CTA that completes the set merges.
template <int VF>
__device__ void finish_cta(const DecodeArgs& a, int b, int kvh, int expected, int n_real, bool has_sink,
                           float* sm) {
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  int32_t* ticket = a.tickets + static_cast<int64_t>(b) * a.hkv + kvh;
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(ticket, 1);
    s_last = prev == expected - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  merge_unit<VF>(a, b, kvh, n_real, has_sink, sm);
  if (threadIdx.x == 0) *ticket = 0;  // leave the workspace ready for the next call
}

// ---------------------------------------------------------------------------
// One warp tile: 16 tokens, the registers a lane needs from them.
// ---------------------------------------------------------------------------
template <int KF, int VF>
struct Tile {
  typename KRow<KF>::S0 k0A, k0B;
  typename KRow<KF>::S1 k1A, k1B;
  typename KRow<KF>::Q kqA, kqB;
  typename VRow<VF>::S0 v0[4];
  typename VRow<VF>::S1 v1[4];
  typename VRow<VF>::Q vq[4];
  float nkA, nkB, nvA, nvB, gkA, gkB, gvA, gvB;
};

struct UnitPlanes {
  const uint8_t* kcodes;
  const uint8_t* vcodes;
  const float* knorm;
  const float* vnorm;
  const uint8_t* kq;
  const uint8_t* vq;
  const float* kres;
  const float* vres;
};

// One pipeline stage in shared memory: the planes of kChunk consecutive
// tokens, each copied by one bulk copy.
constexpr int kChunk = kTok * kWarps;  // 128 tokens: one tile per warp
template <int KF, int VF>
struct StageLayout {
  static constexpr int kc = 0;
  static constexpr int vc = kc + kChunk * Fmt<KF>::code_bytes;
  static constexpr int kn = vc + kChunk * Fmt<VF>::code_bytes;
  static constexpr int vn = kn + kChunk * 4;
  static constexpr int kq = vn + kChunk * 4;
  static constexpr int kr = kq + (Fmt<KF>::prod ? kChunk * (kSketch / 8) : 0);
  static constexpr int vq = kr + (Fmt<KF>::prod ? kChunk * 4 : 0);
  static constexpr int vr = vq + (Fmt<VF>::prod ? kChunk * (kSketch / 8) : 0);
  static constexpr int bytes = vr + (Fmt<VF>::prod ? kChunk * 4 : 0);
  // bytes of a stage holding `rows` tokens (rows a multiple of 16)
  __host__ __device__ static constexpr uint32_t tx_bytes(int rows) {
    return static_cast<uint32_t>(rows) * (bytes / kChunk);
  }
};

// Pipeline depth: three stages when two CTAs (LUT + stages each, plus the
// 1 KB the driver reserves per CTA) still fit in the SM's 228 KB, else two.
template <int KF, int VF>
__host__ __device__ constexpr int decode_stages() {
  return 2 * (Lut<KF, VF>::bytes + 3 * StageLayout<KF, VF>::bytes + 2048) <= 228 * 1024 ? 3 : 2;
}

// Lane loads of one tile from a staged chunk (or any planes with the same row
// layout); rows row0 .. row0+15 exist in every plane, rows at or past the
// sequence length hold stale data and are masked when used.
template <int KF, int VF>
__device__ __forceinline__ void load_tile(Tile<KF, VF>& T, const UnitPlanes& u, int row0, int g, int t) {
  using FK = Fmt<KF>;
  using FV = Fmt<VF>;
  const int rA = row0 + g, rB = row0 + g + 8;
  const uint8_t* ka = u.kcodes + static_cast<int64_t>(rA) * FK::code_bytes;
  const uint8_t* kb = u.kcodes + static_cast<int64_t>(rB) * FK::code_bytes;
  if constexpr (FK::nseg > 0) { T.k0A.load(ka, t); T.k0B.load(kb, t); }
  if constexpr (FK::nseg > 1) { T.k1A.load(ka, t); T.k1B.load(kb, t); }
  if constexpr (FK::prod) {
    T.kqA.load(u.kq + rA * (kSketch / 8), t);
    T.kqB.load(u.kq + rB * (kSketch / 8), t);
    T.gkA = u.kres[rA];
    T.gkB = u.kres[rB];
  }
  T.nkA = u.knorm[rA];
  T.nkB = u.knorm[rB];
  T.nvA = u.vnorm[rA];
  T.nvB = u.vnorm[rB];
  if constexpr (FV::prod) {
    T.gvA = u.vres[rA];
    T.gvB = u.vres[rB];
  }
  const int v0 = row0 + 2 * t;  // tokens v0, v0+1, v0+8, v0+9
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = v0 + (i & 1) + 8 * (i >> 1);
    const uint8_t* vr = u.vcodes + static_cast<int64_t>(r) * FV::code_bytes;
    if constexpr (FV::nseg > 0) T.v0[i].load(vr, g);
    if constexpr (FV::nseg > 1) T.v1[i].load(vr, g);
    if constexpr (FV::prod) T.vq[i].load(u.vq + r * (kSketch / 8), g);
  }
}

template <int KF, int VF, bool PACK>
struct WarpState {
  static constexpr int VMT = 8 + (Fmt<VF>::prod ? 8 : 0);  // m-tiles of the V accumulator
  float oacc[VMT][4];
  float m0, m1, l0, l1;
};

template <int KF, int VF, bool PACK>
__device__ __forceinline__ void compute_tile(const Tile<KF, VF>& T, WarpState<KF, VF, PACK>& W,
                                             const uint32_t (&bq)[8][2][PACK ? 1 : 2],
                                             const uint32_t (&bqs)[8][2][PACK ? 1 : 2], int row0, int t_end,
                                             int g, const unsigned char* lut_a, const unsigned char* lut_b,
                                             uint32_t lane4, uint32_t lane8, uint32_t c1k, uint32_t c1v,
                                             float thr) {
  using FK = Fmt<KF>;
  using FV = Fmt<VF>;
  using KR = KRow<KF>;
  using VR = VRow<VF>;
  constexpr int NX = PACK ? 1 : 2;
  constexpr int VMT = WarpState<KF, VF, PACK>::VMT;
  const uint32_t one2 = 0x3C003C00u;  // half2(1, 1)
  const bool okA = row0 + g < t_end, okB = row0 + g + 8 < t_end;

  // ---- scores S^T (tokens x columns), four independent MMA accumulator chains
  float ca[4][4], cq[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) ca[i][j] = cq[i][j] = 0.f;
  if constexpr (FK::nseg > 0) {
    const unsigned char* lk = FK::b0 == 2 ? lut_b : lut_a;
    static_for<KR::S0::KSTEPS>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      T.k0A.template decode<s>(lk, lane4, lane8, c1k, la, ha);
      T.k0B.template decode<s>(lk, lane4, lane8, c1k, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x) mma16816(ca[(NX * s + x) & 3], la, lb, ha, hb, bq[s][0][x], bq[s][1][x]);
    });
  }
  if constexpr (FK::nseg > 1) {
    static_for<KR::S1::KSTEPS>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      T.k1A.template decode<s>(lut_a, lane4, lane8, c1k, la, ha);
      T.k1B.template decode<s>(lut_a, lane4, lane8, c1k, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x)
        mma16816(ca[(NX * s + x + 2) & 3], la, lb, ha, hb, bq[KR::S0::KSTEPS + s][0][x], bq[KR::S0::KSTEPS + s][1][x]);
    });
  }
  if constexpr (FK::prod) {
    static_for<8>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      T.kqA.template decode<s>(lut_a, lane4, lane8, one2, la, ha);
      T.kqB.template decode<s>(lut_a, lane4, lane8, one2, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x) mma16816(cq[(NX * s + x) & 3], la, lb, ha, hb, bqs[s][0][x], bqs[s][1][x]);
    });
  }
  float sc[4], sq[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[j] = (ca[0][j] + ca[1][j]) + (ca[2][j] + ca[3][j]);
    sq[j] = (cq[0][j] + cq[1][j]) + (cq[2][j] + cq[3][j]);
  }
  if constexpr (PACK) {
    // columns c and c+4 hold the hi and lo halves of one head: add them
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sc[i] += __shfl_xor_sync(0xffffffffu, sc[i], 2);
      if constexpr (FK::prod) sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], 2);
    }
  }
  // s (base 2): c0,c1 = token g, columns 2t, 2t+1; c2,c3 = token g+8
  const float gkA = FK::prod ? T.gkA : 0.f, gkB = FK::prod ? T.gkB : 0.f;
  float s2[4];
  s2[0] = okA ? T.nkA * (sc[0] + kQjlScale * gkA * sq[0]) : -INFINITY;
  s2[1] = okA ? T.nkA * (sc[1] + kQjlScale * gkA * sq[1]) : -INFINITY;
  s2[2] = okB ? T.nkB * (sc[2] + kQjlScale * gkB * sq[2]) : -INFINITY;
  s2[3] = okB ? T.nkB * (sc[3] + kQjlScale * gkB * sq[3]) : -INFINITY;
  float mx0 = fmaxf(s2[0], s2[2]), mx1 = fmaxf(s2[1], s2[3]);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float mn0 = fmaxf(W.m0, mx0), mn1 = fmaxf(W.m1, mx1);
  const float al0 = exp2f(W.m0 - mn0), al1 = exp2f(W.m1 - mn1);
  float p[4];
  p[0] = exp2f(s2[0] - mn0);
  p[1] = exp2f(s2[1] - mn1);
  p[2] = exp2f(s2[2] - mn0);
  p[3] = exp2f(s2[3] - mn1);
  float rs0 = p[0] + p[2], rs1 = p[1] + p[3];
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    rs0 += __shfl_xor_sync(0xffffffffu, rs0, off);
    rs1 += __shfl_xor_sync(0xffffffffu, rs1, off);
  }
  W.l0 = W.l0 * al0 + rs0;
  W.l1 = W.l1 * al1 + rs1;
  W.m0 = mn0;
  W.m1 = mn1;
  if (__any_sync(0xffffffffu, (al0 != 1.f) | (al1 != 1.f))) {
#pragma unroll
    for (int i = 0; i < VMT; ++i) {
      W.oacc[i][0] *= al0;
      W.oacc[i][1] *= al1;
      W.oacc[i][2] *= al0;
      W.oacc[i][3] *= al1;
    }
  }
  // sparse V: exp(s - m)/l over the tokens seen so far bounds the final weight
  if (thr > 0.f) {
    const float c0 = thr * W.l0, c1 = thr * W.l1;
    p[0] = p[0] >= c0 ? p[0] : 0.f;
    p[1] = p[1] >= c1 ? p[1] : 0.f;
    p[2] = p[2] >= c0 ? p[2] : 0.f;
    p[3] = p[3] >= c1 ? p[3] : 0.f;
    const bool any = (p[0] + p[1] + p[2] + p[3]) > 0.f;
    if (!__any_sync(0xffffffffu, any)) return;
  }

  // ---- P'^T fragments: P' = p * ||v|| (and * ||r_v|| for the sketch part)
  const float wA = okA ? T.nvA : 0.f, wB = okB ? T.nvB : 0.f;
  const uint32_t pb0 = movmatrix_t(h2bits(p[0] * wA, p[1] * wA));
  const uint32_t pb1 = movmatrix_t(h2bits(p[2] * wB, p[3] * wB));
  uint32_t qb0 = 0, qb1 = 0;
  if constexpr (FV::prod) {
    const float uA = okA ? wA * T.gvA : 0.f, uB = okB ? wB * T.gvB : 0.f;
    qb0 = movmatrix_t(h2bits(p[0] * uA, p[1] * uA));
    qb1 = movmatrix_t(h2bits(p[2] * uB, p[3] * uB));
  }
  // ---- O^T += C_v^T P'^T
  if constexpr (FV::nseg > 0) {
    constexpr int MT = VR::S0::MT;
    uint32_t r0[MT], r08[MT], r1[MT], r18[MT];
    const unsigned char* lut = FV::b0 == 2 ? lut_b : lut_a;
    VR::S0::decode(T.v0[0], T.v0[1], lut, lane4, lane8, c1v, r0, r08);
    VR::S0::decode(T.v0[2], T.v0[3], lut, lane4, lane8, c1v, r1, r18);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) mma16816(W.oacc[mt], r0[mt], r08[mt], r1[mt], r18[mt], pb0, pb1);
  }
  if constexpr (FV::nseg > 1) {
    constexpr int MT = VR::S1::MT;
    uint32_t r0[MT], r08[MT], r1[MT], r18[MT];
    VR::S1::decode(T.v1[0], T.v1[1], lut_a, lane4, lane8, c1v, r0, r08);
    VR::S1::decode(T.v1[2], T.v1[3], lut_a, lane4, lane8, c1v, r1, r18);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
      mma16816(W.oacc[VR::S0::MT + mt], r0[mt], r08[mt], r1[mt], r18[mt], pb0, pb1);
  }
  if constexpr (FV::prod) {
    uint32_t r0[8], r08[8], r1[8], r18[8];
    VR::Q::decode(T.vq[0], T.vq[1], lut_a, lane4, lane8, one2, r0, r08);
    VR::Q::decode(T.vq[2], T.vq[3], lut_a, lane4, lane8, one2, r1, r18);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) mma16816(W.oacc[8 + mt], r0[mt], r08[mt], r1[mt], r18[mt], qb0, qb1);
  }
}

// ---------------------------------------------------------------------------
// 2. decode kernel
// ---------------------------------------------------------------------------
template <int KF, int VF, bool PACK>
__global__ void __launch_bounds__(kThreads, (Fmt<KF>::prod || Fmt<VF>::prod) ? 1 : 2) decode_kernel(DecodeArgs a) {
  using FK = Fmt<KF>;
  using FV = Fmt<VF>;
  using KR = KRow<KF>;
  using VR = VRow<VF>;
  using L = Lut<KF, VF>;
  extern __shared__ __align__(16) unsigned char smem[];
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int G = a.group;

  int len = a.lens[b];
  if (len > a.max_len) {
    if (split == 0 && kvh == 0 && tid == 0) atomicOr(a.status, 2);
    len = a.max_len;
  }
  if (len < 0) len = 0;
  const int ns = min(a.n_sink, len);
  const int nq = len - ns;
  const int n_real = (nq + a.split_tokens - 1) / a.split_tokens;
  const bool has_sink = ns > 0;
  const int expected = n_real + (has_sink ? 1 : 0);
  const int PF = a.part_floats;
  float* part_base = a.parts + (static_cast<int64_t>(b) * a.hkv + kvh) * (a.n_splits + 1) * kMaxG * PF;
  float* sm = reinterpret_cast<float*>(smem);

  if (expected == 0) {
    if (split == 0)
      for (int i = tid; i < G * kDim; i += kThreads) {
        const int64_t oi = (static_cast<int64_t>(b) * a.hq + kvh * G) * kDim + i;
        if (a.out_bf16)
          reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(0.f);
        else
          reinterpret_cast<float*>(a.out)[oi] = 0.f;
      }
    return;
  }

  if (split == a.n_splits) {
    // ---- sink CTA: bf16 keys/values of tokens [0, ns), original domain ----
    if (!has_sink) return;
    float* qs = sm;                        // [8][128]
    float* sc = qs + kMaxG * kDim;         // [8][n_sink]
    float* red = sc + kMaxG * a.n_sink;    // [8][2]
    for (int i = tid; i < kMaxG * kDim; i += kThreads) {
      const int h = i / kDim, d = i % kDim;
      qs[i] = h < G ? load_q(a.q, a.q_bf16, (static_cast<int64_t>(b) * a.hq + kvh * G + h) * kDim + d) : 0.f;
    }
    __syncthreads();
    const uint16_t* ks = a.k_sink + (static_cast<int64_t>(b) * a.hkv + kvh) * a.n_sink * kDim;
    const uint16_t* vs = a.v_sink + (static_cast<int64_t>(b) * a.hkv + kvh) * a.n_sink * kDim;
    const float scale = kLog2e * rsqrtf(static_cast<float>(kDim));
    for (int i = tid; i < G * ns; i += kThreads) {
      const int h = i / ns, tok = i % ns;
      float acc = 0.f;
      for (int d = 0; d < kDim; ++d) {
        const uint16_t kb = ks[tok * kDim + d];
        acc = fmaf(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&kb)), qs[h * kDim + d], acc);
      }
      sc[h * a.n_sink + tok] = acc * scale;
    }
    __syncthreads();
    if (tid < G) {
      float m = -INFINITY;
      for (int tok = 0; tok < ns; ++tok) m = fmaxf(m, sc[tid * a.n_sink + tok]);
      float l = 0.f;
      for (int tok = 0; tok < ns; ++tok) {
        const float p = exp2f(sc[tid * a.n_sink + tok] - m);
        sc[tid * a.n_sink + tok] = p;
        l += p;
      }
      red[2 * tid] = m;
      red[2 * tid + 1] = l;
    }
    __syncthreads();
    for (int i = tid; i < G * kDim; i += kThreads) {
      const int h = i / kDim, d = i % kDim;
      float acc = 0.f;
      for (int tok = 0; tok < ns; ++tok) {
        const uint16_t vb = vs[tok * kDim + d];
        acc = fmaf(sc[h * a.n_sink + tok], __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&vb)), acc);
      }
      part_base[(a.n_splits * kMaxG + h) * PF + 2 + d] = acc;
    }
    if (tid < G) {
      part_base[(a.n_splits * kMaxG + tid) * PF + 0] = red[2 * tid];
      part_base[(a.n_splits * kMaxG + tid) * PF + 1] = red[2 * tid + 1];
    }
    __syncthreads();
    finish_cta<VF>(a, b, kvh, expected, n_real, has_sink, sm);
    return;
  }

  if (split >= n_real) return;

  // ---- quantized split ----------------------------------------------------
  // lookup tables
  {
    const float* cb = a.cbs;
    if constexpr (L::t4) {
      for (int i = tid; i < 256 * 32; i += kThreads) {
        const int r = i >> 5, ln = i & 31;
        *reinterpret_cast<uint32_t*>(smem + r * 256 + ln * 4) = h2bits(cb[4 * kBookSlots + (r & 15)], cb[4 * kBookSlots + (r >> 4)]);
      }
    }
    if constexpr (L::t3) {
      for (int i = tid; i < 64 * 32; i += kThreads) {
        const int r = i >> 5, ln = i & 31;
        *reinterpret_cast<uint32_t*>(smem + r * 256 + 128 + ln * 4) = h2bits(cb[3 * kBookSlots + (r & 7)], cb[3 * kBookSlots + (r >> 3)]);
      }
    }
    if constexpr (L::t2) {
      for (int i = tid; i < 256 * 32; i += kThreads) {
        const int r = i >> 5, ln = i & 31;
        uint2 v;
        v.x = h2bits(cb[2 * kBookSlots + (r & 3)], cb[2 * kBookSlots + ((r >> 2) & 3)]);
        v.y = h2bits(cb[2 * kBookSlots + ((r >> 4) & 3)], cb[2 * kBookSlots + (r >> 6)]);
        *reinterpret_cast<uint2*>(smem + L::region_b_off + r * 256 + ln * 8) = v;
      }
    }
  }
  const unsigned char* lut_a = smem;
  const unsigned char* lut_b = smem + L::region_b_off;
  const uint32_t lane4 = lane * 4, lane8 = lane * 8;
  const uint32_t c1k = FK::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const uint32_t c1v = FV::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;

  // query B-fragments
  constexpr int NX = PACK ? 1 : 2;
  const uint32_t* qf = a.qfrag + (static_cast<int64_t>(b) * a.hkv + kvh) * kQfragWords;
  uint32_t bq[8][2][NX], bqs[8][2][NX];  // [kstep][b0,b1][hi,lo]
#pragma unroll
  for (int s = 0; s < 8; ++s)
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int x = 0; x < NX; ++x) {
        bq[s][r][x] = qf[((s * 2 + r) * 2 + x) * 32 + lane];
        if constexpr (FK::prod) bqs[s][r][x] = qf[(((8 + s) * 2 + r) * 2 + x) * 32 + lane];
      }
  __syncthreads();

  WarpState<KF, VF, PACK> wst;
  constexpr int VMT = WarpState<KF, VF, PACK>::VMT;
#pragma unroll
  for (int i = 0; i < VMT; ++i) wst.oacc[i][0] = wst.oacc[i][1] = wst.oacc[i][2] = wst.oacc[i][3] = 0.f;
  wst.m0 = wst.m1 = -INFINITY;
  wst.l0 = wst.l1 = 0.f;

  const int t_begin = split * a.split_tokens;
  const int t_end = min(nq, t_begin + a.split_tokens);
  const int64_t ubase = (static_cast<int64_t>(b) * a.hkv + kvh) * a.capacity;
  UnitPlanes u;
  u.kcodes = a.k_codes + ubase * FK::code_bytes;
  u.vcodes = a.v_codes + ubase * FV::code_bytes;
  u.knorm = a.k_norms + ubase;
  u.vnorm = a.v_norms + ubase;
  u.kq = FK::prod ? a.k_qjl + ubase * (kSketch / 8) : nullptr;
  u.vq = FV::prod ? a.v_qjl + ubase * (kSketch / 8) : nullptr;
  u.kres = FK::prod ? a.k_res + ubase : nullptr;
  u.vres = FV::prod ? a.v_res + ubase : nullptr;
  const float thr = a.sparse_thr;

  // software pipeline: the loads of the warp's next tile are in flight while
  // the current one is decoded (two register buffers, no copies)
  // TMA pipeline: thread 0 streams kChunk-token chunks of the split into a
  // ring of shared-memory stages (one bulk copy per plane); warp w decodes
  // tile w of each chunk.
  using SL = StageLayout<KF, VF>;
  constexpr int kStages = decode_stages<KF, VF>();
  unsigned char* stages = smem + L::bytes;
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ int s_abort;
  const int n_chunks = (t_end - t_begin + kChunk - 1) / kChunk;
  const int t_end16 = (t_end + kTok - 1) / kTok * kTok;  // <= capacity (a multiple of 64)
  auto issue = [&](int c) {
    unsigned char* st = stages + (c % kStages) * SL::bytes;
    const int r0 = t_begin + c * kChunk;
    const int rows = min(kChunk, t_end16 - r0);
    uint64_t* bar = &full_bar[c % kStages];
    mbar_expect_tx(bar, SL::tx_bytes(rows));
    if constexpr (FK::code_bytes > 0)
      bulk_g2s(st + SL::kc, u.kcodes + static_cast<int64_t>(r0) * FK::code_bytes, rows * FK::code_bytes, bar);
    if constexpr (FV::code_bytes > 0)
      bulk_g2s(st + SL::vc, u.vcodes + static_cast<int64_t>(r0) * FV::code_bytes, rows * FV::code_bytes, bar);
    bulk_g2s(st + SL::kn, u.knorm + r0, rows * 4, bar);
    bulk_g2s(st + SL::vn, u.vnorm + r0, rows * 4, bar);
    if constexpr (FK::prod) {
      bulk_g2s(st + SL::kq, u.kq + r0 * (kSketch / 8), rows * (kSketch / 8), bar);
      bulk_g2s(st + SL::kr, u.kres + r0, rows * 4, bar);
    }
    if constexpr (FV::prod) {
      bulk_g2s(st + SL::vq, u.vq + r0 * (kSketch / 8), rows * (kSketch / 8), bar);
      bulk_g2s(st + SL::vr, u.vres + r0, rows * 4, bar);
    }
  };
  if (tid == 0) {
    s_abort = 0;
#pragma unroll
    for (int i = 0; i < kStages; ++i) mbar_init(&full_bar[i], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int c = 0; c < min(kStages, n_chunks); ++c) issue(c);
  int issued = min(kStages, n_chunks);
  for (int c = 0; c < n_chunks; ++c) {
    if (!mbar_wait(&full_bar[c % kStages], (c / kStages) & 1)) s_abort = 1;
    const int row0 = t_begin + c * kChunk + warp * kTok;
    if (row0 < t_end && !s_abort) {
      const unsigned char* st = stages + (c % kStages) * SL::bytes;
      UnitPlanes sp;
      sp.kcodes = st + SL::kc;
      sp.vcodes = st + SL::vc;
      sp.knorm = reinterpret_cast<const float*>(st + SL::kn);
      sp.vnorm = reinterpret_cast<const float*>(st + SL::vn);
      sp.kq = st + SL::kq;
      sp.kres = reinterpret_cast<const float*>(st + SL::kr);
      sp.vq = st + SL::vq;
      sp.vres = reinterpret_cast<const float*>(st + SL::vr);
      Tile<KF, VF> tl;
      load_tile(tl, sp, warp * kTok, g, t);
      compute_tile<KF, VF, PACK>(tl, wst, bq, bqs, row0, t_end, g, lut_a, lut_b, lane4, lane8, c1k, c1v, thr);
    }
    __syncthreads();  // stage c % kStages is free again
    if (s_abort) break;
    if (tid == 0 && issued < n_chunks) {
      fence_proxy_async();
      issue(issued);
      ++issued;
    }
  }
  if (s_abort) {
    // a copy never completed: flag it, drain what was issued (bounded) and
    // leave without publishing a partial
    if (tid == 0) {
      atomicOr(a.status, 4);
      for (int c = 0; c < issued; ++c) mbar_wait(&full_bar[c % kStages], (c / kStages) & 1);
    }
    return;
  }
  float (&oacc)[VMT][4] = wst.oacc;
  const float m0 = wst.m0, m1 = wst.m1, l0 = wst.l0, l1 = wst.l1;

  // ---- merge the warps of this CTA (shared memory reused after the loop)
  __syncthreads();
  constexpr int W = FV::prod ? 2 * kDim : kDim;  // accumulator width per head
  float* wm = sm;                                // [warp][head]
  float* wl = wm + kWarps * kMaxG;
  float* wacc = wl + kWarps * kMaxG;             // [warp][head][W]
  if (g == 0) {
    wm[warp * kMaxG + 2 * t] = m0;
    wm[warp * kMaxG + 2 * t + 1] = m1;
    wl[warp * kMaxG + 2 * t] = l0;
    wl[warp * kMaxG + 2 * t + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < VMT; ++mt) {
    int d0, d1;
    if (mt < 8) {
      if (FV::nseg > 1 && mt >= VR::S0::MT) {
        d0 = VR::S1::dim(64, g, mt - VR::S0::MT, 0);
        d1 = VR::S1::dim(64, g, mt - VR::S0::MT, 1);
      } else {
        d0 = VR::S0::dim(0, g, mt, 0);
        d1 = VR::S0::dim(0, g, mt, 1);
      }
    } else {
      d0 = kDim + VR::Q::dim(0, g, mt - 8, 0);
      d1 = kDim + VR::Q::dim(0, g, mt - 8, 1);
    }
    float* w0 = wacc + (warp * kMaxG + 2 * t) * W;
    float* w1 = wacc + (warp * kMaxG + 2 * t + 1) * W;
    w0[d0] = oacc[mt][0];
    w1[d0] = oacc[mt][1];
    w0[d1] = oacc[mt][2];
    w1[d1] = oacc[mt][3];
  }
  __syncthreads();
  float* mine = part_base + static_cast<int64_t>(split) * kMaxG * PF;
  for (int i = tid; i < kMaxG * W; i += kThreads) {
    const int h = i / W, j = i % W;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wm[w * kMaxG + h]);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = wm[w * kMaxG + h];
      if (mw > -INFINITY) s += wacc[(w * kMaxG + h) * W + j] * exp2f(mw - M);
    }
    mine[h * PF + 2 + j] = s;
    if (j == 0) {
      float l = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = wm[w * kMaxG + h];
        if (mw > -INFINITY) l += wl[w * kMaxG + h] * exp2f(mw - M);
      }
      mine[h * PF + 0] = M;
      mine[h * PF + 1] = l;
    }
  }
  __syncthreads();
  finish_cta<VF>(a, b, kvh, expected, n_real, has_sink, sm);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int KF, int VF>
size_t decode_smem_bytes() {
  using L = Lut<KF, VF>;
  const size_t pipeline = static_cast<size_t>(L::bytes) + decode_stages<KF, VF>() * StageLayout<KF, VF>::bytes;
  const size_t W = Fmt<VF>::prod ? 2 * kDim : kDim;
  const size_t combine = (2 * kWarps * kMaxG + kWarps * kMaxG * W) * sizeof(float);
  const size_t merge = (kMaxG * 2 * kDim + kMaxG * kDim + 2 * kMaxG) * sizeof(float);
  return std::max<size_t>({pipeline, combine, merge, 24 * 1024});
}

template <int KF, int VF, bool PACK>
tq_status run_decode_v(DecodeArgs& a, const DecodePlan& plan, size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<KF, VF, PACK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel attribute");
  qrot_kernel<KF><<<dim3(plan.hkv, plan.B), kThreads, 0, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "query rotation launch");
  decode_kernel<KF, VF, PACK><<<dim3(plan.n_splits + 1, plan.hkv, plan.B), kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "decode kernel launch");
}

template <int KF, int VF>
tq_status run_decode(DecodeArgs& a, const DecodePlan& plan, int sink_smem_floats, cudaStream_t st) {
  size_t smem = decode_smem_bytes<KF, VF>();
  smem = std::max<size_t>(smem, static_cast<size_t>(sink_smem_floats) * sizeof(float));
  a.pack = plan.group <= 4;
  return a.pack ? run_decode_v<KF, VF, true>(a, plan, smem, st) : run_decode_v<KF, VF, false>(a, plan, smem, st);
}

constexpr int fid(int mse, int mixed, int prod) { return mse | (mixed << 3) | (prod << 4); }

}  // namespace

DecodePlan plan_decode(const tq_params* p, int B, int hq, int hkv, int max_len) {
  DecodePlan pl{};
  pl.B = B;
  pl.hq = hq;
  pl.hkv = hkv;
  pl.group = hq / hkv;
  pl.max_len = max_len;
  int sms = 148;
  {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int64_t units = static_cast<int64_t>(B) * hkv;
  const int64_t target = static_cast<int64_t>(sms) * 2 * 8;  // about eight waves of resident CTAs
  int64_t per = (static_cast<int64_t>(std::max(max_len, 1)) * units + target - 1) / target;
  const int quantum = kTok * kWarps;  // 128 tokens: one tile per warp
  per = std::max<int64_t>(per, 4 * quantum);
  per = (per + quantum - 1) / quantum * quantum;
  pl.split_tokens = static_cast<int>(per);
  pl.n_splits = std::max(1, static_cast<int>((std::max(max_len, 1) + per - 1) / per));
  pl.part_floats = 2 + (p->fv.prod ? 2 * kDim : kDim);
  const size_t tickets = (static_cast<size_t>(units) * sizeof(int32_t) + 255) & ~size_t(255);
  const size_t qfrag = static_cast<size_t>(units) * kQfragWords * sizeof(uint32_t);
  pl.ws_partials_bytes = static_cast<size_t>(units) * (pl.n_splits + 1) * kMaxG * pl.part_floats * sizeof(float);
  pl.ws_total_bytes = tickets + ((qfrag + 255) & ~size_t(255)) + pl.ws_partials_bytes;
  return pl;
}

tq_status launch_decode(const tq_params* p, const void* q, int q_bf16, const tq_cache* c, const DecodePlan& plan,
                        void* out, int out_bf16, void* ws, float sparse_thr, cudaStream_t st) {
  DecodeArgs a{};
  a.q = q;
  a.q_bf16 = q_bf16;
  a.k_codes = c->k_codes;
  a.k_norms = c->k_norms;
  a.k_qjl = c->k_qjl;
  a.k_res = c->k_res_norms;
  a.v_codes = c->v_codes;
  a.v_norms = c->v_norms;
  a.v_qjl = c->v_qjl;
  a.v_res = c->v_res_norms;
  a.k_sink = c->k_sink;
  a.v_sink = c->v_sink;
  a.lens = c->lens;
  a.status = c->status;
  a.hkv = plan.hkv;
  a.group = plan.group;
  a.hq = plan.hq;
  a.capacity = c->capacity;
  a.n_sink = c->n_sink;
  a.max_len = plan.max_len;
  a.n_splits = plan.n_splits;
  a.split_tokens = plan.split_tokens;
  a.part_floats = plan.part_floats;
  const size_t units = static_cast<size_t>(plan.B) * plan.hkv;
  char* w = static_cast<char*>(ws);
  a.tickets = reinterpret_cast<int32_t*>(w);
  w += (units * sizeof(int32_t) + 255) & ~size_t(255);
  a.qfrag = reinterpret_cast<uint32_t*>(w);
  w += (units * kQfragWords * sizeof(uint32_t) + 255) & ~size_t(255);
  a.parts = reinterpret_cast<float*>(w);
  a.out = out;
  a.out_bf16 = out_bf16;
  a.pit = p->pit32;
  a.st = p->st32;
  a.pi = p->pi32;
  a.s = p->s32;
  a.cbs = p->cbs32;
  a.sig = p->sig32;
  a.sparse_thr = sparse_thr;
  const int sink_floats = kMaxG * kDim + kMaxG * c->n_sink + 2 * kMaxG + 64;

  const int kf = p->fk.id(), vf = p->fv.id();
#define TQ_CASE(K, V) \
  if (kf == (K) && vf == (V)) return run_decode<(K), (V)>(a, plan, sink_floats, st);
  // symmetric formats
  TQ_CASE(fid(1, 0, 0), fid(1, 0, 0))
  TQ_CASE(fid(2, 0, 0), fid(2, 0, 0))
  TQ_CASE(fid(3, 0, 0), fid(3, 0, 0))
  TQ_CASE(fid(4, 0, 0), fid(4, 0, 0))
  TQ_CASE(fid(3, 1, 0), fid(3, 1, 0))
  TQ_CASE(fid(0, 0, 1), fid(0, 0, 1))
  TQ_CASE(fid(1, 0, 1), fid(1, 0, 1))
  TQ_CASE(fid(2, 0, 1), fid(2, 0, 1))
  TQ_CASE(fid(3, 0, 1), fid(3, 0, 1))
  // asymmetric K/V widths
  TQ_CASE(fid(4, 0, 0), fid(3, 0, 0))
  TQ_CASE(fid(4, 0, 0), fid(2, 0, 0))
  TQ_CASE(fid(3, 0, 0), fid(2, 0, 0))
#undef TQ_CASE
  return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: this K/V format pair has no decode kernel");
}

}  // namespace tq
