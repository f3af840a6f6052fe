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
//   2. decode_kernel: persistent, one CTA per SM; a producer warp streams
//      the packed cache into shared memory with bulk copies, fifteen consumer
//      warps walk 16-token tiles of it:
//        scores S^T[16 tok x 8 heads] = C_k[16 x 128] Q~^T  (mma.sync m16n8k16)
//        online softmax (base 2), sparse-V mask, P' = p * ||v||
//        O^T[128 x 8 heads] += C_v^T[128 x 16 tok] P'^T    (mma.sync m16n8k16)
//      The dequantized codebook values for both MMAs come straight from
//      per-lane-replicated shared-memory tables indexed by packed code bytes
//      (two or four codes per lookup, no bank conflicts), so no fp16 tile is
//      ever written back to memory.  Warps merge in shared memory and the CTA
//      writes one (m, l, acc) partial per piece of a (sequence, kv-head).
//   3. merge_kernel: one CTA per (sequence, query head) attends the bf16 sink,
//      combines the pieces and applies Pi^T / S^T once.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_internal.h"
#include "tq_sm100.cuh"

namespace tq {
namespace {

using namespace sm100;

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
// of rows r < 64 hold half2(c3[r & 7], c3[r >> 3]) -- and, when region A spans
// all 256 rows anyway (t3_wide), every row r holds the entry of r & 63, so a
// 3-bit pair in the low six bits of any byte is looked up with one byte
// permute.  Region B (row stride 256 B, 8 B per lane): four 2-bit centroids of
// byte r.  With 2- and 3-bit widths only (t2a), bytes [0, 128) of region A row
// r hold half2(c2[r & 3], c2[(r >> 2) & 3]) instead, and there is no region B.  Entry (r, lane) sits at r*256 + lane*4 (or *8): every lane hits its
// own bank.
template <int KF, int VF>
struct Lut {
  static constexpr bool t4 = Fmt<KF>::uses(4) || Fmt<VF>::uses(4);
  static constexpr bool t3 = Fmt<KF>::uses(3) || Fmt<VF>::uses(3);
  static constexpr bool t2 = Fmt<KF>::uses(2) || Fmt<VF>::uses(2);
  static constexpr int region_a = (t4 || (t3 && t2)) ? 65536 : (t3 ? 16384 : 0);
  static constexpr bool t3_wide = t3 && region_a == 65536;
  // 2-bit and 3-bit widths without 4-bit ones: the 2-bit pair table takes the
  // free bytes [0, 128) of region A instead of a region B of its own
  static constexpr bool t2a = t2 && t3 && !t4;
  static constexpr int region_b_off = region_a;  // 0 or 65536: a 64 KB boundary
  static constexpr int bytes = region_a + (t2 && !t2a ? 65536 : 0);
};

// The tables live at shared-window address kLutAddr (64 KB aligned), so a
// lookup address is (code byte << 8) | lane offset | table base, formed by a
// single byte permute or logic op with the base folded into the lane offset.
constexpr uint32_t kLutAddr = 0x10000;

__device__ __forceinline__ uint32_t h2bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = 0)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
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

// Shared-memory loads on 32-bit shared-window addresses (`base` is the
// shared address of a table or stage, `off` a byte offset).
__device__ __forceinline__ uint32_t lds32(uint32_t base, uint32_t off) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(base + off));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t base, uint32_t off) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(base + off));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t base, uint32_t off) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(base + off));
  return v;
}
__device__ __forceinline__ float ldsf(uint32_t base, uint32_t off) { return __uint_as_float(lds32(base, off)); }
// Lookup-table reads: the tables are written once before the main loop and
// only read after it, so these loads are pure functions of their address and
// the compiler may schedule them freely (the stage reads above stay ordered
// by the pipeline's barriers).
__device__ __forceinline__ uint32_t lut32(uint32_t base, uint32_t off) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(base + off));
  return v;
}
__device__ __forceinline__ uint2 lut64(uint32_t base, uint32_t off) {
  uint2 v;
  asm("ld.shared.v2.b32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(base + off));
  return v;
}

// byte k of w placed at bits 8..15; bits 0..7 and 16..31 from lb (the lane
// offset and the table base; lb's bits 8..15 are zero)
__device__ __forceinline__ uint32_t byte_addr(uint32_t w, uint32_t lb, int k) {
  return __byte_perm(w, lb, 0x7604 | (k << 4));
}

// half2 of +-c from bits p and p+16 of w (bit set -> +c); c_bits = half2(c, c)
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int p, uint32_t c_bits) {
  const uint32_t x = w << (15 - p);
  return (~x & 0x80008000u) | c_bits;
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
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

  // row: shared address of the token's code row
  __device__ __forceinline__ void load(uint32_t row, int t) {
    const int o = BYTE0 + t * BYTES;
    if constexpr (BYTES == 16) {
      const uint4 v = lds128(row, o);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if constexpr (BYTES == 12) {
      w[0] = lds32(row, o); w[1] = lds32(row, o + 4); w[2] = lds32(row, o + 8);
    } else if constexpr (BYTES == 8) {
      const uint2 v = lds64(row, o);
      w[0] = v.x; w[1] = v.y;
    } else if constexpr (BYTES == 6) {
      const int al = o & ~3;
      const uint32_t lo = lds32(row, al), hi = lds32(row, al + 4);
      const int sh = (o & 3) * 8;
      w[0] = __funnelshift_r(lo, hi, sh);
      w[1] = hi >> sh;
    } else {
      static_assert(BYTES == 4, "unsupported K chunk");
      w[0] = lds32(row, o);
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

  // k-step S: (lo, hi) = A-fragment registers for k = 2t..2t+1 and 2t+8..2t+9.
  // T3W (3-bit): the pair table spans 256 rows, so the pair at bit 12S (6,
  // 30: after a 6-bit shift; 12, 36 / 18, 42: after 12 / 18) is the low six
  // bits of byte 0 or 3 of w[0] or of a funnel shift of (w[0], w[1]).
  // T2A (2-bit): the pair table in region A; the pair in the high nibble of a
  // byte is looked up after a 4-bit shift of the word.
  template <int S, bool T3W = false, bool T2A = false>
  __device__ __forceinline__ void decode(uint32_t smem, uint32_t lane4, uint32_t lane8,
                                         uint32_t c_bits, uint32_t& lo, uint32_t& hi) const {
    constexpr int s = S;
    if constexpr (B == 3 && T3W && ND == 64) {
      const uint32_t lb = lane4 + 128;
      const uint32_t w1 = w[WORDS > 1 ? 1 : 0];
      constexpr int kb = S >= 2 ? 3 : 0;  // byte of the low field
      const uint32_t src_lo = (S & 1) ? __funnelshift_r(w[0], w1, 12) : w[0];
      const uint32_t src_hi = (S & 1) ? __funnelshift_r(w[0], w1, 18) : __funnelshift_r(w[0], w1, 6);
      lo = lut32(smem, byte_addr(src_lo, lb, kb));
      hi = lut32(smem, byte_addr(src_hi, lb, kb));
    } else if constexpr (B == 4) {
      const uint32_t ww = w[s >> 1];
      lo = lut32(smem, byte_addr(ww, lane4, 2 * (s & 1)));
      hi = lut32(smem, byte_addr(ww, lane4, 2 * (s & 1) + 1));
    } else if constexpr (B == 3) {
      lo = lut32(smem, pair3<2 * S>(lane4 + 128));
      hi = lut32(smem, pair3<2 * S + 1>(lane4 + 128));
    } else if constexpr (B == 2 && T2A) {
      const uint32_t ww = w[s >> 2];
      lo = lut32(smem, byte_addr(ww, lane4, s & 3));
      hi = lut32(smem, byte_addr(ww >> 4, lane4, s & 3));
    } else if constexpr (B == 2) {
      const uint2 v = lut64(smem, byte_addr(w[s >> 2], lane8, s & 3));
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

  __device__ __forceinline__ void load(uint32_t row, int g) {
    constexpr int bits = ND * B / 8;
    if constexpr (bits == 64) {
      const uint2 v = lds64(row, BYTE0 + 8 * g);
      x = static_cast<uint64_t>(v.x) | (static_cast<uint64_t>(v.y) << 32);
    } else if constexpr (bits == 32) {
      x = lds32(row, BYTE0 + 4 * g);
    } else if constexpr (bits == 16) {
      const int o = BYTE0 + 2 * g;
      x = (lds32(row, o & ~3) >> ((o & 2) * 8)) & 0xFFFFu;
    } else if constexpr (bits == 48) {
      const int o = BYTE0 + 6 * g, al = o & ~3;
      const uint64_t v = static_cast<uint64_t>(lds32(row, al)) | (static_cast<uint64_t>(lds32(row, al + 4)) << 32);
      x = (v >> ((o & 3) * 8)) & 0xFFFFFFFFFFFFull;
    } else {
      static_assert(bits == 24, "unsupported V chunk");
      const int o = BYTE0 + 3 * g, al = o & ~3, sh = (o & 3) * 8;
      uint64_t v = lds32(row, al);
      if (sh > 8) v |= static_cast<uint64_t>(lds32(row, al + 4)) << 32;  // field crosses into the next word
      x = (v >> sh) & 0xFFFFFFull;
    }
  }

  // rows g (coordinate 2mt) and g+8 (2mt+1) for every m-tile, tokens (A, B)
  template <bool T2A = false>
  __device__ __forceinline__ static void decode(const VChunk& a, const VChunk& b, uint32_t smem,
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
          rg[4 * wd + k] = lut32(smem, byte_addr(ev, lane4, k));
          rg8[4 * wd + k] = lut32(smem, byte_addr(od, lane4, k));
        }
      }
    } else if constexpr (B == 3) {
      // 24-bit halves of 8 codes: interleave the two tokens' 3-bit fields
      // into 6-bit (A | B << 3) fields, evens and odds apart
      constexpr uint32_t E = 0x1C71C7u;  // 3-bit fields at bits 0, 6, 12, 18
      const uint32_t lb = lane4 + 128;
      static_for<MT / 4>([&](auto hh) {
        constexpr int h = decltype(hh)::value;
        const uint32_t xa = static_cast<uint32_t>(a.x >> (24 * h)), xb = static_cast<uint32_t>(b.x >> (24 * h));
        const uint32_t ev = (xa & E) | ((xb << 3) & ~E);
        const uint32_t od = ((xa >> 3) & E) | (xb & ~E);
        static_for<4>([&](auto kk) {
          constexpr int k = decltype(kk)::value;
          rg[4 * h + k] = lut32(smem, addr6<6 * k>(ev, lb));
          rg8[4 * h + k] = lut32(smem, addr6<6 * k>(od, lb));
        });
      });
    } else if constexpr (B == 2) {
      const uint32_t xa = static_cast<uint32_t>(a.x), xb = static_cast<uint32_t>(b.x);
      const uint32_t ev = (xa & 0x33333333u) | ((xb & 0x33333333u) << 2);
      const uint32_t od = ((xa >> 2) & 0x33333333u) | (xb & 0xCCCCCCCCu);
#pragma unroll
      for (int j = 0; j < MT / 2; ++j) {
        if constexpr (T2A) {
          rg[2 * j] = lut32(smem, byte_addr(ev, lane4, j));
          rg[2 * j + 1] = lut32(smem, byte_addr(ev >> 4, lane4, j));
          rg8[2 * j] = lut32(smem, byte_addr(od, lane4, j));
          rg8[2 * j + 1] = lut32(smem, byte_addr(od >> 4, lane4, j));
        } else {
          const uint2 e = lut64(smem, byte_addr(ev, lane8, j));
          const uint2 o = lut64(smem, byte_addr(od, lane8, j));
          rg[2 * j] = e.x;
          rg[2 * j + 1] = e.y;
          rg8[2 * j] = o.x;
          rg8[2 * j + 1] = o.y;
        }
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
  int B, hkv, group, hq, capacity, n_sink, max_len, part_floats;
  int ctas;   // CTAs of the decode grid (pieces a unit can be cut into)
  int chunk;  // quantized tokens per scheduled chunk
  int merge_chunk;  // pieces the merge kernel stages in shared memory at a time
  float* parts;
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
  uint32_t dyn_bytes;  // dynamic shared memory granted to the decode kernel
  float qscale;      // factor on the rotated query: log2(e)/sqrt(d) for attention, 1 for search
  // inner-product search only
  int64_t n_db;            // database rows (k_* planes)
  int topk;                // k <= kSearchMaxK
  uint64_t* cand;          // per (query, CTA) candidate lists [group][ctas][32]
  float* out_scores;       // [group][topk]
  int64_t* out_rows;       // [group][topk]
  const uint32_t* bound_in;  // per-query starting bound (ordered score) or null
  uint32_t* bound_out;       // the merge writes the k-th best score here instead of results
};

__device__ __forceinline__ float load_q(const void* q, int bf16, int64_t i) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]) : reinterpret_cast<const float*>(q)[i];
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

// Programmatic dependent launch.  The three kernels of one decode call run
// back to back on one stream; the second and third are launched with
// programmatic stream serialization, so they may start while the previous one
// still runs.  pdl_launch lets the next kernel be scheduled; pdl_wait blocks
// the calling thread until the previous kernel has finished and its writes
// are visible (a no-op in a kernel launched without the attribute).
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// ---------------------------------------------------------------------------
// 1. query rotation: one CTA per (sequence, kv-head).  Threads 0..127 form
//    Pi q for all heads (one output coordinate each), threads 128..255 form
//    S q (prod keys); then the fp16 B-fragments are written.
// ---------------------------------------------------------------------------
constexpr int kQrotThreads = 512;
constexpr int kQrotSplit = kQrotThreads / kDim;  // slices of the k range per output coordinate

template <int KF>
__global__ void __launch_bounds__(kQrotThreads) qrot_kernel(DecodeArgs a) {
  using KR = KRow<KF>;
  using FK = Fmt<KF>;
  extern __shared__ float4 s_mat4[];              // Pi^T [k][j], then S^T [k][j] (prod keys)
  __shared__ __align__(16) float qsT[kDim][kMaxG];  // query, [k][head]
  __shared__ float qt[kMaxG][kDim];
  __shared__ float qsk[kMaxG][kSketch];
  __shared__ float s_p[kQrotSplit][kMaxG][kDim];  // partial sums over k slices
  const int kvh = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int G = a.group;
  pdl_launch();  // the decode kernel's prologue and cache stream may start
  {
    // stage the matrices with asynchronous 16-byte copies, all in flight
    constexpr int N4 = kDim * kDim / 4 / kQrotThreads;
    const float4* pit4 = reinterpret_cast<const float4*>(a.pit);
#pragma unroll
    for (int i = 0; i < N4; ++i)
      cp_async16(smem_u32(s_mat4 + i * kQrotThreads + tid), pit4 + i * kQrotThreads + tid);
    if constexpr (FK::prod) {
      const float4* st4 = reinterpret_cast<const float4*>(a.st);
#pragma unroll
      for (int i = 0; i < N4; ++i)
        cp_async16(smem_u32(s_mat4 + kDim * kDim / 4 + i * kQrotThreads + tid), st4 + i * kQrotThreads + tid);
    }
  }
  for (int i = tid; i < kMaxG * kDim; i += kQrotThreads) {
    const int h = i % kMaxG, d = i / kMaxG;
    qsT[d][h] = h < G ? load_q(a.q, a.q_bf16, (static_cast<int64_t>(b) * a.hq + kvh * G + h) * kDim + d) : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  const float scale = a.qscale;
  // thread (j, ks) sums k in [ks * 32, ks * 32 + 32) for output coordinate j
  // of every head; the slices are added in shared memory
  const int j = tid & (kDim - 1), ks = tid >> 7;
  const float4* q4 = reinterpret_cast<const float4*>(&qsT[0][0]);
  for (int mtx = 0; mtx < (FK::prod ? 2 : 1); ++mtx) {
    const float* mat = reinterpret_cast<const float*>(s_mat4) + mtx * kDim * kDim;
    float acc[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) acc[h] = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < kDim / kQrotSplit; ++kk) {
      const int k = ks * (kDim / kQrotSplit) + kk;
      const float m = mat[k * kDim + j];
      const float4 x0 = q4[2 * k], x1 = q4[2 * k + 1];
      acc[0] = fmaf(m, x0.x, acc[0]);
      acc[1] = fmaf(m, x0.y, acc[1]);
      acc[2] = fmaf(m, x0.z, acc[2]);
      acc[3] = fmaf(m, x0.w, acc[3]);
      acc[4] = fmaf(m, x1.x, acc[4]);
      acc[5] = fmaf(m, x1.y, acc[5]);
      acc[6] = fmaf(m, x1.z, acc[6]);
      acc[7] = fmaf(m, x1.w, acc[7]);
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) s_p[ks][h][j] = acc[h];
    __syncthreads();
    for (int i = tid; i < kMaxG * kDim; i += kQrotThreads) {
      const int h = i / kDim, jj = i % kDim;
      float v = 0.f;
#pragma unroll
      for (int s = 0; s < kQrotSplit; ++s) v += s_p[s][h][jj];
      if (mtx == 1) {
        qsk[h][jj] = v * scale;
      } else {
        const int wj = FK::width(jj);
        qt[h][jj] = wj > 0 ? v * (scale / a.sig[wj]) : 0.f;
      }
    }
    __syncthreads();
  }
  // B fragments: lane (g, t) supplies column g; k-steps 0..7 from the MSE
  // segments, 8..15 from the QJL segment.  Unpacked: column g = head g, halves
  // hi (x = 0) and lo (x = 1).  Packed (group <= 4): column g < 4 = hi of head
  // g, column g >= 4 = lo of head g - 4, in x = 0.
  uint32_t* dst = const_cast<uint32_t*>(a.qfrag) + (static_cast<int64_t>(b) * a.hkv + kvh) * kQfragWords;
  for (int i = tid; i < 16 * 32; i += kQrotThreads) {
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

// Shared addresses of the planes of one staged chunk.
struct UnitPlanes {
  uint32_t kcodes, vcodes, knorm, vnorm, kq, vq, kres, vres;
};

// One pipeline stage in shared memory: the planes of CH consecutive tokens,
// each copied by one bulk copy.
constexpr int kConsumers = 15;                // consumer warps of the persistent kernel
constexpr int kThreadsP = (kConsumers + 1) * 32;  // + one producer warp
template <int KF, int VF, int kChunk>
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

// Shared memory of the persistent kernel: pipeline stages, the lookup tables at
// kLutAddr, and a scratch area (warp combine in 64-coordinate slices, split
// merge, sink scores).  Stages go below kLutAddr while they fit, the rest
// above the tables.
constexpr int kSliceDims = 64;
// Cross-warp combine area of write_piece: per warp and head the running max,
// the sum and one slice of the accumulator.
constexpr int kScratchBytes = (kConsumers * kMaxG * kSliceDims + 2 * kConsumers * kMaxG) * 4;
constexpr int kSmemBudget = 227 * 1024 - 1024;  // dynamic bytes requested per block
constexpr int kDynBaseMax = 4096;                // assumed upper bound of the dynamic base address
constexpr int kSmemEnd = 227 * 1024;             // assumed end of the usable shared window

__host__ __device__ constexpr int plan_end(int stage, int n_stages, int lut, int scratch) {
  int cur = kDynBaseMax, in_gap = 0;
  while (in_gap < n_stages && cur + stage <= static_cast<int>(kLutAddr)) {
    cur += stage;
    ++in_gap;
  }
  const bool scratch_low = cur + scratch <= static_cast<int>(kLutAddr);
  return static_cast<int>(kLutAddr) + lut + (n_stages - in_gap) * stage + (scratch_low ? 0 : scratch);
}

// Chunk shape of a format pair: tokens per consumer warp (32 or 16) and the
// number of stages, the deepest that fits.
template <int KF, int VF>
struct DecodeCfg {
  static constexpr int lut = Lut<KF, VF>::bytes;
  static constexpr int scr = kScratchBytes;
  static constexpr int s32 = StageLayout<KF, VF, 32 * kConsumers>::bytes;
  static constexpr int s16 = StageLayout<KF, VF, 16 * kConsumers>::bytes;
  static constexpr bool fit32 = plan_end(s32, 2, lut, scr) <= kSmemEnd;
  static constexpr int WT = fit32 ? 32 : 16;
  static constexpr int CH = WT * kConsumers;
  static constexpr int stage = fit32 ? s32 : s16;
  static constexpr int S = plan_end(stage, 4, lut, scr) <= kSmemEnd   ? 4
                           : plan_end(stage, 3, lut, scr) <= kSmemEnd ? 3
                                                                       : 2;
};

template <int KF, int VF, bool PACK>
struct WarpState {
  static constexpr int VMT = 8 + (Fmt<VF>::prod ? 8 : 0);  // m-tiles of the V accumulator
  float oacc[VMT][4];
  float m0, m1, l0, l1;
};

template <bool PACK>
using QFrag = uint32_t[8][2][PACK ? 1 : 2];

// Token order inside a 16-token subtile.  MMA row / column k of a subtile
// holds physical token pi[k] (K and V use the same order, so the scores,
// softmax weights and V columns line up).  The order only changes which
// shared-memory banks the code loads hit: lane (g, t) reads K rows pi[g],
// pi[g + 8] and V rows pi[2t], pi[2t + 1], pi[2t + 8], pi[2t + 9], and rows of
// 24..64 bytes make some orders collide less.  pi[k] is nibble k of the word;
// the words come from a search over a model of these loads (bank_perm.py next
// to this file), identity where no order helps.
__host__ __device__ constexpr uint64_t token_order(int kf, int vf) {
  return kf == 2 && vf == 2     ? 0xFE095427B86D1AC3ull
         : kf == 4 && vf == 4   ? 0xB2CD41F863905AE7ull
         : kf == 11 && vf == 11 ? 0x2AE619D534F8BC70ull
         : kf == 10 && vf == 10 ? 0xA428EC6031F97DB5ull
         : kf == 18 && vf == 18 ? 0xB6C51FA82907D43Eull
         : kf == 4 && vf == 2   ? 0xB856274109A3DEFCull
         : kf == 3 && vf == 2   ? 0xC1B7502E948F3D6Aull
                                : 0xFEDCBA9876543210ull;
}

// This lane's physical rows within a subtile: K rows (score rows g, g + 8)
// and V rows (MMA columns 2t, 2t + 1, 2t + 8, 2t + 9).
struct TokRows {
  int kA, kB, v0, v1, v8, v9;
};
template <int KF, int VF>
__device__ __forceinline__ TokRows tok_rows(int g, int t) {
  constexpr uint64_t pi = token_order(KF, VF);
  auto at = [](int k) { return static_cast<int>((pi >> (4 * k)) & 15u); };
  return TokRows{at(g), at(g + 8), at(2 * t), at(2 * t + 1), at(2 * t + 8), at(2 * t + 9)};
}

// Scores of one 16-token subtile whose rows start at `srow` of the staged
// planes: s2 (base 2) for tokens g (s2[0], s2[1]) and g+8 (s2[2], s2[3]),
// columns 2t, 2t+1; masked tokens get -inf.  Two MMA accumulator chains.
// HI: the query's fp16 high halves only (column g = head g, no low halves):
// one MMA per k-step for up to 8 heads, scores within about 2^-12 of
// ||q|| ||x|| (the search's precision; attention keeps both halves).
template <int KF, bool PACK, bool T3W, bool T2A, bool HI = false>
__device__ __forceinline__ void subtile_scores(const UnitPlanes& u, int srow, const TokRows& tr, bool okA, bool okB,
                                               int g, int t,
                                               const QFrag<PACK || HI>& bq, const QFrag<PACK || HI>& bqs,
                                               uint32_t lut_a, uint32_t lut_b,
                                               uint32_t lane4, uint32_t lane8, uint32_t c1k, float (&s2)[4]) {
  static_assert(!(PACK && HI), "packed halves or high halves only");
  using FK = Fmt<KF>;
  using KR = KRow<KF>;
  constexpr int NX = (PACK || HI) ? 1 : 2;
  const uint32_t one2 = 0x3C003C00u;  // half2(1, 1)
  const int rA = srow + tr.kA, rB = srow + tr.kB;
  const uint32_t ka = u.kcodes + rA * FK::code_bytes;
  const uint32_t kb = u.kcodes + rB * FK::code_bytes;
  float ca[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float cq[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  if constexpr (FK::nseg > 0) {
    typename KR::S0 xa, xb;
    xa.load(ka, t);
    xb.load(kb, t);
    const uint32_t lk = FK::b0 == 2 ? lut_b : lut_a;
    static_for<KR::S0::KSTEPS>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      xa.template decode<s, T3W, T2A>(lk, lane4, lane8, c1k, la, ha);
      xb.template decode<s, T3W, T2A>(lk, lane4, lane8, c1k, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x) mma16816(ca[(NX * s + x) & 1], la, lb, ha, hb, bq[s][0][x], bq[s][1][x]);
    });
  }
  if constexpr (FK::nseg > 1) {
    typename KR::S1 xa, xb;
    xa.load(ka, t);
    xb.load(kb, t);
    const uint32_t lk = FK::b1 == 2 ? lut_b : lut_a;
    static_for<KR::S1::KSTEPS>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      xa.template decode<s, T3W, T2A>(lk, lane4, lane8, c1k, la, ha);
      xb.template decode<s, T3W, T2A>(lk, lane4, lane8, c1k, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x)
        mma16816(ca[(NX * s + x + 1) & 1], la, lb, ha, hb, bq[KR::S0::KSTEPS + s][0][x], bq[KR::S0::KSTEPS + s][1][x]);
    });
  }
  float gA = 0.f, gB = 0.f;
  if constexpr (FK::prod) {
    typename KR::Q xa, xb;
    xa.load(u.kq + rA * (kSketch / 8), t);
    xb.load(u.kq + rB * (kSketch / 8), t);
    static_for<8>([&](auto ss) {
      constexpr int s = decltype(ss)::value;
      uint32_t la, ha, lb, hb;
      xa.template decode<s>(lut_a, lane4, lane8, one2, la, ha);
      xb.template decode<s>(lut_a, lane4, lane8, one2, lb, hb);
#pragma unroll
      for (int x = 0; x < NX; ++x) mma16816(cq[(NX * s + x) & 1], la, lb, ha, hb, bqs[s][0][x], bqs[s][1][x]);
    });
    gA = kQjlScale * ldsf(u.kres, rA * 4);
    gB = kQjlScale * ldsf(u.kres, rB * 4);
  }
  float sc[4], sq[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sc[j] = ca[0][j] + ca[1][j];
    sq[j] = cq[0][j] + cq[1][j];
  }
  if constexpr (PACK) {
    // columns c and c+4 hold the hi and lo halves of one head: add them
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sc[i] += __shfl_xor_sync(0xffffffffu, sc[i], 2);
      if constexpr (FK::prod) sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], 2);
    }
  }
  const float nA = ldsf(u.knorm, rA * 4), nB = ldsf(u.knorm, rB * 4);
  if constexpr (FK::prod) {
    s2[0] = nA * fmaf(gA, sq[0], sc[0]);
    s2[1] = nA * fmaf(gA, sq[1], sc[1]);
    s2[2] = nB * fmaf(gB, sq[2], sc[2]);
    s2[3] = nB * fmaf(gB, sq[3], sc[3]);
  } else {
    s2[0] = nA * sc[0];
    s2[1] = nA * sc[1];
    s2[2] = nB * sc[2];
    s2[3] = nB * sc[3];
  }
  if (!okA) s2[0] = s2[1] = -INFINITY;
  if (!okB) s2[2] = s2[3] = -INFINITY;
}

// O^T += C_v^T P'^T for one 16-token subtile (rows from `srow`); p holds the
// softmax weights of tokens g (p[0], p[1]) and g+8 (p[2], p[3]).
template <int VF, int VMT, bool T2A>
__device__ __forceinline__ void subtile_pv(const UnitPlanes& u, int srow, const TokRows& tr, bool okA, bool okB,
                                           int g, int t,
                                           const float (&p)[4], uint32_t lut_a,
                                           uint32_t lut_b, uint32_t lane4, uint32_t lane8, uint32_t c1v,
                                           float (&oacc)[VMT][4]) {
  using FV = Fmt<VF>;
  using VR = VRow<VF>;
  const uint32_t one2 = 0x3C003C00u;
  const float wA = okA ? ldsf(u.vnorm, (srow + tr.kA) * 4) : 0.f, wB = okB ? ldsf(u.vnorm, (srow + tr.kB) * 4) : 0.f;
  const uint32_t pb0 = movmatrix_t(h2bits(p[0] * wA, p[1] * wA));
  const uint32_t pb1 = movmatrix_t(h2bits(p[2] * wB, p[3] * wB));
  // rows of MMA columns 2t, 2t+1, 2t+8, 2t+9
  const uint32_t r0p = u.vcodes + (srow + tr.v0) * FV::code_bytes;
  const uint32_t r1p = u.vcodes + (srow + tr.v1) * FV::code_bytes;
  const uint32_t r8p = u.vcodes + (srow + tr.v8) * FV::code_bytes;
  const uint32_t r9p = u.vcodes + (srow + tr.v9) * FV::code_bytes;
  if constexpr (FV::nseg > 0) {
    constexpr int MT = VR::S0::MT;
    typename VR::S0 xa, xb, xc, xd;
    xa.load(r0p, g);
    xb.load(r1p, g);
    xc.load(r8p, g);
    xd.load(r9p, g);
    uint32_t r0[MT], r08[MT], r1[MT], r18[MT];
    const uint32_t lut = FV::b0 == 2 ? lut_b : lut_a;
    VR::S0::template decode<T2A>(xa, xb, lut, lane4, lane8, c1v, r0, r08);
    VR::S0::template decode<T2A>(xc, xd, lut, lane4, lane8, c1v, r1, r18);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) mma16816(oacc[mt], r0[mt], r08[mt], r1[mt], r18[mt], pb0, pb1);
  }
  if constexpr (FV::nseg > 1) {
    constexpr int MT = VR::S1::MT;
    typename VR::S1 xa, xb, xc, xd;
    xa.load(r0p, g);
    xb.load(r1p, g);
    xc.load(r8p, g);
    xd.load(r9p, g);
    uint32_t r0[MT], r08[MT], r1[MT], r18[MT];
    const uint32_t lut = FV::b1 == 2 ? lut_b : lut_a;
    VR::S1::template decode<T2A>(xa, xb, lut, lane4, lane8, c1v, r0, r08);
    VR::S1::template decode<T2A>(xc, xd, lut, lane4, lane8, c1v, r1, r18);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) mma16816(oacc[VR::S0::MT + mt], r0[mt], r08[mt], r1[mt], r18[mt], pb0, pb1);
  }
  if constexpr (FV::prod) {
    const float uA = okA ? wA * ldsf(u.vres, (srow + tr.kA) * 4) : 0.f,
                uB = okB ? wB * ldsf(u.vres, (srow + tr.kB) * 4) : 0.f;
    const uint32_t qb0 = movmatrix_t(h2bits(p[0] * uA, p[1] * uA));
    const uint32_t qb1 = movmatrix_t(h2bits(p[2] * uB, p[3] * uB));
    typename VR::Q xa, xb, xc, xd;
    xa.load(u.vq + (srow + tr.v0) * (kSketch / 8), g);
    xb.load(u.vq + (srow + tr.v1) * (kSketch / 8), g);
    xc.load(u.vq + (srow + tr.v8) * (kSketch / 8), g);
    xd.load(u.vq + (srow + tr.v9) * (kSketch / 8), g);
    uint32_t r0[8], r08[8], r1[8], r18[8];
    VR::Q::decode(xa, xb, lut_a, lane4, lane8, one2, r0, r08);
    VR::Q::decode(xc, xd, lut_a, lane4, lane8, one2, r1, r18);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) mma16816(oacc[8 + mt], r0[mt], r08[mt], r1[mt], r18[mt], qb0, qb1);
  }
}

// One warp tile of 32 tokens (two 16-token subtiles) starting at stage row
// `srow`, unit-relative row `row0`; tokens at or past `nq` are masked (their
// scores are -inf and their value weights 0, so a subtile past the end adds
// nothing; computing it anyway keeps the two subtiles free of branches, which
// lets their lookup and MMA chains interleave).  SPARSE: skip the PV MMAs of
// a subtile whose weights are all below the sparse-V threshold.
template <int KF, int VF, bool PACK, int WT, bool SPARSE>
__device__ __forceinline__ void compute_tile(const UnitPlanes& u, int srow, int row0, int nq, const TokRows& tr,
                                             WarpState<KF, VF, PACK>& W, const QFrag<PACK>& bq,
                                             const QFrag<PACK>& bqs, int g, int t, uint32_t lut_a,
                                             uint32_t lut_b, uint32_t lane4, uint32_t lane8,
                                             uint32_t c1k, uint32_t c1v, float thr) {
  constexpr int VMT = WarpState<KF, VF, PACK>::VMT;
  constexpr bool second = WT == 2 * kTok;
  const bool ok0A = row0 + tr.kA < nq, ok0B = row0 + tr.kB < nq;
  const bool ok1A = row0 + kTok + tr.kA < nq, ok1B = row0 + kTok + tr.kB < nq;
  float s0[4], s1[4];
  subtile_scores<KF, PACK, Lut<KF, VF>::t3_wide, Lut<KF, VF>::t2a>(u, srow, tr, ok0A, ok0B, g, t, bq, bqs, lut_a, lut_b, lane4, lane8, c1k, s0);
  if constexpr (second)
    subtile_scores<KF, PACK, Lut<KF, VF>::t3_wide, Lut<KF, VF>::t2a>(u, srow + kTok, tr, ok1A, ok1B, g, t, bq, bqs, lut_a, lut_b, lane4, lane8, c1k, s1);
  else
    s1[0] = s1[1] = s1[2] = s1[3] = -INFINITY;
  // online softmax over the 32 tokens (base 2), columns 2t and 2t+1.  The
  // running maximum moves only when some lane sees a larger score (rare
  // after the first tiles), and each lane keeps its own partial sum (the
  // eight lanes of a column are added when the piece is written), so most
  // tiles take no cross-lane step.
  float p0[4], p1[4];
  {
    float mx0 = fmaxf(fmaxf(s0[0], s0[2]), fmaxf(s1[0], s1[2]));
    float mx1 = fmaxf(fmaxf(s0[1], s0[3]), fmaxf(s1[1], s1[3]));
    if (__any_sync(0xffffffffu, (mx0 > W.m0) | (mx1 > W.m1))) {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(W.m0, mx0), mn1 = fmaxf(W.m1, mx1);
      const float al0 = fast_exp2(W.m0 - mn0), al1 = fast_exp2(W.m1 - mn1);
      W.l0 *= al0;
      W.l1 *= al1;
#pragma unroll
      for (int i = 0; i < VMT; ++i) {
        W.oacc[i][0] *= al0;
        W.oacc[i][1] *= al1;
        W.oacc[i][2] *= al0;
        W.oacc[i][3] *= al1;
      }
      W.m0 = mn0;
      W.m1 = mn1;
    }
    p0[0] = fast_exp2(s0[0] - W.m0);
    p0[1] = fast_exp2(s0[1] - W.m1);
    p0[2] = fast_exp2(s0[2] - W.m0);
    p0[3] = fast_exp2(s0[3] - W.m1);
    p1[0] = fast_exp2(s1[0] - W.m0);
    p1[1] = fast_exp2(s1[1] - W.m1);
    p1[2] = fast_exp2(s1[2] - W.m0);
    p1[3] = fast_exp2(s1[3] - W.m1);
    W.l0 += (p0[0] + p0[2]) + (p1[0] + p1[2]);
    W.l1 += (p0[1] + p0[3]) + (p1[1] + p1[3]);
  }
  if constexpr (!SPARSE) {
    subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow, tr, ok0A, ok0B, g, t, p0, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
    if constexpr (second)
      subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow + kTok, tr, ok1A, ok1B, g, t, p1, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
  } else {
    // sparse V: exp(s - m) / l over the tokens seen so far bounds the final
    // weight, and this lane's partial sum is at most l, so p < thr * l_lane
    // only skips tokens whose final weight is below thr
    const float c0 = thr * W.l0, c1 = thr * W.l1;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      p0[i] = p0[i] >= c0 ? p0[i] : 0.f;
      p0[i + 1] = p0[i + 1] >= c1 ? p0[i + 1] : 0.f;
      p1[i] = p1[i] >= c0 ? p1[i] : 0.f;
      p1[i + 1] = p1[i + 1] >= c1 ? p1[i + 1] : 0.f;
    }
    if (__any_sync(0xffffffffu, (p0[0] + p0[1] + p0[2] + p0[3]) > 0.f))
      subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow, tr, ok0A, ok0B, g, t, p0, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
    if (second && __any_sync(0xffffffffu, (p1[0] + p1[1] + p1[2] + p1[3]) > 0.f))
      subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow + kTok, tr, ok1A, ok1B, g, t, p1, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
  }
}

// ---------------------------------------------------------------------------
// 2. persistent decode kernel
//
// One CTA per SM: consumer warps 0..14 decode, warp 15 streams the packed
// cache with bulk copies (full / empty mbarriers, bounded waits).
//
// Schedule.  Unit u = b * hkv + h (sequence b, kv-head h).  Its quantized
// tokens form ceil(nq / kChunk) chunks; the chunks of all units, in unit
// order, make one list of C chunks cut into gridDim.x equal contiguous ranges,
// one per CTA, so every CTA streams the same number of bytes.  A unit may span
// several CTAs (its pieces).  Piece (u, cta) writes partial slot u + cta:
// both indices only grow along the list, so slots are distinct and there are
// at most U + P - 1 of them.  The merge kernel finds a unit's pieces from the
// same schedule.  No CTA waits for another.
// ---------------------------------------------------------------------------
struct UnitInfo {
  int len, ns, nq, chunks;
};

__device__ __forceinline__ UnitInfo unit_info(const DecodeArgs& a, int u, int kChunk) {
  const int b = u / a.hkv;
  const int len = min(max(a.lens[b], 0), a.max_len);
  UnitInfo r;
  r.len = len;
  r.ns = min(a.n_sink, len);
  r.nq = len - r.ns;
  r.chunks = (r.nq + kChunk - 1) / kChunk;
  return r;
}

__device__ __forceinline__ int64_t range_start(int i, int64_t C, int P) { return static_cast<int64_t>(i) * C / P; }

// Chunks of each kv-head unit of sequence b (all units of a sequence are alike).
__device__ __forceinline__ int seq_chunks(const DecodeArgs& a, int b, int kChunk) {
  const int len = min(max(a.lens[b], 0), a.max_len);
  return (len - min(a.n_sink, len) + kChunk - 1) / kChunk;
}

// CTA whose range holds chunk c: the largest i with i*C/P <= c.
__device__ __forceinline__ int cta_of_chunk(int64_t c, int64_t C, int P) {
  return static_cast<int>(((c + 1) * P - 1) / C);
}

// Ranges are empty when C < P; such CTAs hold no piece of any unit.
__device__ __forceinline__ bool cta_has_chunks(int i, int64_t C, int P) {
  return range_start(i + 1, C, P) > range_start(i, C, P);
}

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumers * 32) : "memory");
}


// Partial slot: per head of the unit's group, [max, sum, 2 unused, accumulator]
// (kPartAcc floats before the accumulator keep every row 16-byte aligned).
constexpr int kPartAcc = 4;
__device__ __forceinline__ float* part_slot(const DecodeArgs& a, int64_t slot) {
  return a.parts + slot * a.group * a.part_floats;
}

__device__ __forceinline__ void store_out(const DecodeArgs& a, int64_t i, float v) {
  if (a.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(a.out)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(a.out)[i] = v;
}

// Cross-warp combine of one piece into partial slot `slot`, in 64-coordinate
// slices of the accumulator (consumer threads).  LANE_SUMS: each lane holds
// its own partial softmax sums (dense path), added over the column first.
template <int KF, int VF, bool PACK, bool LANE_SUMS>
__device__ void write_piece(const DecodeArgs& a, const WarpState<KF, VF, PACK>& W, int64_t slot, float* sm,
                            int warp, int g, int t) {
  using FV = Fmt<VF>;
  using VR = VRow<VF>;
  constexpr int NT = kConsumers * 32;
  constexpr int VMT = WarpState<KF, VF, PACK>::VMT;
  constexpr int WD = FV::prod ? 2 * kDim : kDim;
  const int tid = threadIdx.x;
  float* wm = sm;                          // [warp][head]
  float* wl = wm + kConsumers * kMaxG;     // [warp][head]
  float* wacc = wl + kConsumers * kMaxG;   // [warp][head][kSliceDims]
  float* dst = part_slot(a, slot);
  const int PF = a.part_floats;
  float l0 = W.l0, l1 = W.l1;
  if constexpr (LANE_SUMS) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }
  if (g == 0) {
    wm[warp * kMaxG + 2 * t] = W.m0;
    wm[warp * kMaxG + 2 * t + 1] = W.m1;
    wl[warp * kMaxG + 2 * t] = l0;
    wl[warp * kMaxG + 2 * t + 1] = l1;
  }
#pragma unroll 1
  for (int pass = 0; pass < WD / kSliceDims; ++pass) {
    const int lo = pass * kSliceDims;
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
      float* w0 = wacc + (warp * kMaxG + 2 * t) * kSliceDims - lo;
      float* w1 = wacc + (warp * kMaxG + 2 * t + 1) * kSliceDims - lo;
      if (d0 >= lo && d0 < lo + kSliceDims) {
        w0[d0] = W.oacc[mt][0];
        w1[d0] = W.oacc[mt][1];
      }
      if (d1 >= lo && d1 < lo + kSliceDims) {
        w0[d1] = W.oacc[mt][2];
        w1[d1] = W.oacc[mt][3];
      }
    }
    consumers_sync();
    for (int i = tid; i < a.group * kSliceDims; i += NT) {
      const int h = i / kSliceDims, j = i % kSliceDims;
      float M = -INFINITY;
      for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, wm[w * kMaxG + h]);
      float s = 0.f, l = 0.f;
      for (int w = 0; w < kConsumers; ++w) {
        const float mw = wm[w * kMaxG + h];
        if (mw > -INFINITY) {
          const float f = exp2f(mw - M);
          s += wacc[(w * kMaxG + h) * kSliceDims + j] * f;
          l += wl[w * kMaxG + h] * f;
        }
      }
      dst[h * PF + kPartAcc + lo + j] = s;
      if (pass == 0 && j == 0) {
        dst[h * PF + 0] = M;
        dst[h * PF + 1] = l;
      }
    }
    consumers_sync();
  }
}

// ---------------------------------------------------------------------------
// 3. merge: one CTA per unit (sequence, kv-head), all heads of its group.
//    The unit's quantized tokens were streamed as pieces by consecutive CTAs
//    of the decode grid; its bf16 sink tokens are attended here.  Partial
//    results are combined by their maxima (the usual online-softmax merge),
//    Pi^T (and S^T for prod values) is applied once, and the result is
//    divided by the softmax sum.  The matrix rows and the sink run before
//    pdl_wait, overlapping the tail of the decode kernel.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 512;
constexpr int kMaxPieces = 1024;  // bound on the decode grid size
constexpr int kMaxSink = 4096;    // sink weights live in shared memory

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Merge shared memory beyond the static arrays: sink weights [n_sink][8],
// piece maxima / weights and sums [ctas][8] each, and a staging buffer of
// merge_chunk pieces (G x part_floats floats each).
constexpr size_t kMergeStageBytes = 128 * 1024;
inline int merge_chunk_pieces(int group, int part_floats) {
  const size_t per = static_cast<size_t>(group) * part_floats * sizeof(float);
  return static_cast<int>(std::max<size_t>(1, kMergeStageBytes / per));
}
inline size_t merge_dyn_bytes(int n_sink, int ctas, int group, int part_floats) {
  return (static_cast<size_t>(n_sink) + 2 * static_cast<size_t>(ctas)) * kMaxG * sizeof(float) +
         static_cast<size_t>(merge_chunk_pieces(group, part_floats)) * group * part_floats * sizeof(float);
}

template <int VF>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(DecodeArgs a) {
  using FV = Fmt<VF>;
  constexpr int NT = kMergeThreads;
  constexpr int WD = FV::prod ? 2 * kDim : kDim;  // accumulator: rotated | sketch
  constexpr int NS = NT / WD;                     // piece slices of the accumulation
  constexpr int RS = WD / 4;                      // matrix rows per un-rotation slice
  extern __shared__ float4 s_dyn4[];
  __shared__ float s_red[4 * kMaxG * kDim];       // slice partials
  __shared__ __align__(16) float s_acc[WD][kMaxG];  // merged accumulator, [j][head]
  __shared__ float s_osk[kMaxG][kDim];            // sink values, original domain
  __shared__ float s_q[kMaxG][4][33];  // query quarters, padded: the four quarters sit in different banks
  __shared__ float s_ms[kMaxG], s_ls[kMaxG], s_M[kMaxG], s_L[kMaxG];
  __shared__ long long s_C, s_cu0;
  float* s_sc = reinterpret_cast<float*>(s_dyn4);  // [n_sink][8]
  float* s_f = s_sc + a.n_sink * kMaxG;             // [pieces][8]: maxima, then weights
  float* s_l = s_f + a.ctas * kMaxG;                // [pieces][8]: sums
  float* s_part = s_l + a.ctas * kMaxG;             // staged pieces [merge_chunk][G][part_floats]
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.group, P = a.ctas, CH = a.chunk, PF = a.part_floats;
  const int b = u / a.hkv, kvh = u % a.hkv;
  const int64_t orow = (static_cast<int64_t>(b) * a.hq + kvh * G) * kDim;  // head 0 of the group
  const UnitInfo ui = unit_info(a, u, CH);
  if (ui.len == 0) {
    for (int i = tid; i < G * kDim; i += NT) store_out(a, orow + i, 0.f);
    return;
  }
  // this thread's matrix rows for the un-rotation: column o, rows
  // [sl*RS, (sl+1)*RS) of [Pi; sqrt(pi/2)/m S]
  const int o = tid & (kDim - 1), sl4 = tid >> 7;
  float pm[RS];
  if (ui.chunks > 0) {
    const int j0 = sl4 * RS;
    const bool sk = FV::prod && j0 >= kDim;
    const float* mat = sk ? a.s + (j0 - kDim) * kDim : a.pi + j0 * kDim;
#pragma unroll
    for (int jj = 0; jj < RS; ++jj) pm[jj] = __ldg(mat + jj * kDim + o) * (sk ? kQjlScale : 1.f);
  }
  // where the unit's chunks sit in the decode schedule (warp 0)
  if (warp == 0 && ui.chunks > 0) {
    long long tot = 0, before = 0;
    for (int v = lane; v < a.B; v += 32) {
      const int ch = seq_chunks(a, v, CH);
      tot += ch;
      if (v < b) before += ch;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, off);
      before += __shfl_xor_sync(0xffffffffu, before, off);
    }
    if (lane == 0) {
      s_C = tot * a.hkv;
      s_cu0 = before * a.hkv + static_cast<long long>(kvh) * ui.chunks;
    }
  }
  // sink: scores with the original query, softmax weights, weighted values
  if (ui.ns > 0) {
    for (int i = tid; i < kMaxG * kDim; i += NT)
      s_q[i / kDim][(i % kDim) >> 5][i & 31] = i < G * kDim ? load_q(a.q, a.q_bf16, orow + i) : 0.f;
    __syncthreads();
    // sink rows are staged through shared memory (the piece staging buffer,
    // not yet in use) in chunks of up to SC tokens with 16-byte asynchronous
    // copies, so each chunk costs one memory round trip
    const char* ks = reinterpret_cast<const char*>(a.k_sink) + static_cast<int64_t>(u) * a.n_sink * kDim * 2;
    const char* vs = reinterpret_cast<const char*>(a.v_sink) + static_cast<int64_t>(u) * a.n_sink * kDim * 2;
    const __nv_bfloat16* srow = reinterpret_cast<const __nv_bfloat16*>(s_part);
    const int SC = a.merge_chunk * G * PF * 4 / (kDim * 2);  // rows that fit the staging buffer
    const float scale = kLog2e * rsqrtf(static_cast<float>(kDim));
    auto stage_rows = [&](const char* src, int c0, int cnt) {
      const float4* s4 = reinterpret_cast<const float4*>(src + static_cast<int64_t>(c0) * kDim * 2);
      for (int e = tid; e < cnt * kDim * 2 / 16; e += NT) cp_async16(smem_u32(s_part) + 16 * e, s4 + e);
      cp_async_wait_all();
      __syncthreads();
    };
    for (int c0 = 0; c0 < ui.ns; c0 += SC) {
      const int cnt = min(SC, ui.ns - c0);
      stage_rows(ks, c0, cnt);
      // thread (token, quarter): dot products over 32 coordinates for every
      // head, then added across the four quarters (adjacent lanes)
      for (int tb = 0; tb < cnt; tb += NT / 4) {
        const int tt = tb + (tid >> 2), qtr = tid & 3;
        float d[kMaxG];
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) d[h] = 0.f;
        if (tt < cnt) {
          const uint4* kr = reinterpret_cast<const uint4*>(srow + tt * kDim + 32 * qtr);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 kw = kr[c];
            const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float k0 = __uint_as_float(w4[e] << 16), k1 = __uint_as_float(w4[e] & 0xFFFF0000u);
              const int j = 8 * c + 2 * e;
#pragma unroll
              for (int h = 0; h < kMaxG; ++h) d[h] = fmaf(k1, s_q[h][qtr][j + 1], fmaf(k0, s_q[h][qtr][j], d[h]));
            }
          }
        }
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
          d[h] += __shfl_xor_sync(0xffffffffu, d[h], 1);
          d[h] += __shfl_xor_sync(0xffffffffu, d[h], 2);
        }
        if (tt < cnt && qtr == 0)
#pragma unroll
          for (int h = 0; h < kMaxG; ++h)
            if (h < G) s_sc[(c0 + tt) * kMaxG + h] = d[h] * scale;
      }
      __syncthreads();  // the staging buffer is refilled
    }
    if (warp < G) {  // warp h: max, weights and sum of head h
      const int h = warp;
      float mx = -INFINITY;
      for (int tt = lane; tt < ui.ns; tt += 32) mx = fmaxf(mx, s_sc[tt * kMaxG + h]);
      mx = warp_max(mx);
      float sum = 0.f;
      for (int tt = lane; tt < ui.ns; tt += 32) {
        const float pw = exp2f(s_sc[tt * kMaxG + h] - mx);
        s_sc[tt * kMaxG + h] = pw;
        sum += pw;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        s_ms[h] = mx;
        s_ls[h] = sum;
      }
    }
    __syncthreads();
    {
      float acc[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) acc[h] = 0.f;
      for (int c0 = 0; c0 < ui.ns; c0 += SC) {
        const int cnt = min(SC, ui.ns - c0);
        stage_rows(vs, c0, cnt);
        for (int tt = sl4; tt < cnt; tt += 4) {
          const float v = __bfloat162float(srow[tt * kDim + o]);
          const float4 p0 = s_dyn4[(c0 + tt) * 2], p1 = s_dyn4[(c0 + tt) * 2 + 1];
          acc[0] = fmaf(p0.x, v, acc[0]);
          acc[1] = fmaf(p0.y, v, acc[1]);
          acc[2] = fmaf(p0.z, v, acc[2]);
          acc[3] = fmaf(p0.w, v, acc[3]);
          acc[4] = fmaf(p1.x, v, acc[4]);
          acc[5] = fmaf(p1.y, v, acc[5]);
          acc[6] = fmaf(p1.z, v, acc[6]);
          acc[7] = fmaf(p1.w, v, acc[7]);
        }
        __syncthreads();  // the staging buffer is refilled
      }
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) s_red[(sl4 * kMaxG + h) * kDim + o] = acc[h];
    }
    __syncthreads();
    for (int i = tid; i < G * kDim; i += NT) {
      const int h = i / kDim, j = i % kDim;
      s_osk[h][j] = s_red[(0 * kMaxG + h) * kDim + j] + s_red[(1 * kMaxG + h) * kDim + j] +
                    s_red[(2 * kMaxG + h) * kDim + j] + s_red[(3 * kMaxG + h) * kDim + j];
    }
  } else if (tid < kMaxG) {
    s_ms[tid] = -INFINITY;
    s_ls[tid] = 0.f;
  }
  __syncthreads();
  // the pieces: written by the decode kernel
  pdl_wait();
  const bool has_pieces = ui.chunks > 0;
  int first = 0, n_p = 0;
  long long C = 0;
  if (has_pieces) {
    C = s_C;
    const long long cu0 = s_cu0;
    first = cta_of_chunk(cu0, C, P);
    n_p = cta_of_chunk(cu0 + ui.chunks - 1, C, P) - first + 1;
  }
  // the maxima and sums of all pieces, gathered at once
  for (int e = tid; e < n_p * G; e += NT) {
    const int i = e / G, h = e % G;
    float m = -INFINITY, l = 0.f;
    if (cta_has_chunks(first + i, C, P)) {
      const float* pp = part_slot(a, u + first + i) + h * PF;
      m = __ldcg(pp);
      l = __ldcg(pp + 1);
    }
    s_f[i * kMaxG + h] = m;
    s_l[i * kMaxG + h] = l;
  }
  __syncthreads();
  if (warp < G) {  // warp h: merged maximum, the pieces' weights and the sum for head h
    const int h = warp;
    float M = s_ms[h];
    for (int i = lane; i < n_p; i += 32) M = fmaxf(M, s_f[i * kMaxG + h]);
    M = warp_max(M);
    float L = 0.f;
    for (int i = lane; i < n_p; i += 32) {
      const float m = s_f[i * kMaxG + h];
      const float f = m > -INFINITY ? exp2f(m - M) : 0.f;
      L = fmaf(s_l[i * kMaxG + h], f, L);
      s_f[i * kMaxG + h] = f;
    }
    L = warp_sum(L);
    if (lane == 0) {
      const float fs = s_ms[h] > -INFINITY ? exp2f(s_ms[h] - M) : 0.f;
      s_M[h] = fs;  // sink weight relative to the merged maximum
      s_L[h] = fmaf(s_ls[h], fs, L);
    }
  }
  __syncthreads();
  if (has_pieces) {
    {
      // the accumulators: consecutive slots, staged chunk by chunk with
      // 16-byte asynchronous copies
      const int j = tid % WD, sl = tid / WD;
      float acc[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) acc[h] = 0.f;
      const int slot_floats = G * PF;
      for (int c0 = 0; c0 < n_p; c0 += a.merge_chunk) {
        const int cnt = min(a.merge_chunk, n_p - c0);
        const float4* src = reinterpret_cast<const float4*>(part_slot(a, u + first + c0));
        const int n16 = cnt * slot_floats / 4;
        for (int e = tid; e < n16; e += NT) cp_async16(smem_u32(s_part) + 16 * e, src + e);
        cp_async_wait_all();
        __syncthreads();
        for (int i = sl; i < cnt; i += NS) {
          const float* pp = s_part + i * slot_floats + kPartAcc + j;
#pragma unroll
          for (int h = 0; h < kMaxG; ++h) {
            // weight 0: a piece of a CTA with an empty range, whose slot was
            // not written in this call
            const float f = h < G ? s_f[(c0 + i) * kMaxG + h] : 0.f;
            if (f != 0.f) acc[h] = fmaf(pp[h * PF], f, acc[h]);
          }
        }
        __syncthreads();  // the staging buffer is refilled
      }
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) s_red[(sl * kMaxG + h) * WD + j] = acc[h];
    }
    __syncthreads();
    for (int i = tid; i < kMaxG * WD; i += NT) {
      const int j = i / kMaxG, h = i % kMaxG;
      float v = 0.f;
#pragma unroll
      for (int sl = 0; sl < NS; ++sl) v += s_red[(sl * kMaxG + h) * WD + j];
      if (j < kDim) v = FV::width(j) > 0 ? v / a.sig[FV::width(j)] : 0.f;
      s_acc[j][h] = h < G ? v : 0.f;
    }
    __syncthreads();
    // un-rotation: out_h[o] = sum_j Pi[j][o] A_h[j] + sqrt(pi/2)/m sum_j S[j][o] B_h[j]
    float r[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) r[h] = 0.f;
    const float4* acc4 = reinterpret_cast<const float4*>(&s_acc[sl4 * RS][0]);
#pragma unroll
    for (int jj = 0; jj < RS; ++jj) {
      const float4 x0 = acc4[2 * jj], x1 = acc4[2 * jj + 1];
      r[0] = fmaf(pm[jj], x0.x, r[0]);
      r[1] = fmaf(pm[jj], x0.y, r[1]);
      r[2] = fmaf(pm[jj], x0.z, r[2]);
      r[3] = fmaf(pm[jj], x0.w, r[3]);
      r[4] = fmaf(pm[jj], x1.x, r[4]);
      r[5] = fmaf(pm[jj], x1.y, r[5]);
      r[6] = fmaf(pm[jj], x1.z, r[6]);
      r[7] = fmaf(pm[jj], x1.w, r[7]);
    }
    __syncthreads();  // s_red is reused
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) s_red[(sl4 * kMaxG + h) * kDim + o] = r[h];
    __syncthreads();
  }
  for (int i = tid; i < G * kDim; i += NT) {
    const int h = i / kDim, j = i % kDim;
    float v = 0.f;
    if (has_pieces)
      v = s_red[(0 * kMaxG + h) * kDim + j] + s_red[(1 * kMaxG + h) * kDim + j] + s_red[(2 * kMaxG + h) * kDim + j] +
          s_red[(3 * kMaxG + h) * kDim + j];
    if (ui.ns > 0) v = fmaf(s_M[h], s_osk[h][j], v);
    const float L = s_L[h];
    store_out(a, orow + i, L > 0.f ? v / L : 0.f);
  }
}

// The lookup tables of a format pair (see Lut), written by the consumer
// threads (thread index tid < kConsumers * 32) from the sigma-scaled
// centroids cb staged in shared memory.
template <typename L>
__device__ __forceinline__ void build_luts(unsigned char* lut_mem, const float* cb, int tid) {
  constexpr int NTC = kConsumers * 32;
  if constexpr (L::t4) {
    for (int i = tid; i < 256 * 32; i += NTC) {
      const int r = i >> 5, ln = i & 31;
      *reinterpret_cast<uint32_t*>(lut_mem + r * 256 + ln * 4) = h2bits(cb[4 * kBookSlots + (r & 15)], cb[4 * kBookSlots + (r >> 4)]);
    }
  }
  if constexpr (L::t3) {
    constexpr int rows = L::t3_wide ? 256 : 64;
    for (int i = tid; i < rows * 32; i += NTC) {
      const int r = i >> 5, ln = i & 31, e = r & 63;
      *reinterpret_cast<uint32_t*>(lut_mem + r * 256 + 128 + ln * 4) = h2bits(cb[3 * kBookSlots + (e & 7)], cb[3 * kBookSlots + (e >> 3)]);
    }
  }
  if constexpr (L::t2a) {
    for (int i = tid; i < 256 * 32; i += NTC) {
      const int r = i >> 5, ln = i & 31;
      *reinterpret_cast<uint32_t*>(lut_mem + r * 256 + ln * 4) =
          h2bits(cb[2 * kBookSlots + (r & 3)], cb[2 * kBookSlots + ((r >> 2) & 3)]);
    }
  } else if constexpr (L::t2) {
    for (int i = tid; i < 256 * 32; i += NTC) {
      const int r = i >> 5, ln = i & 31;
      uint2 v;
      v.x = h2bits(cb[2 * kBookSlots + (r & 3)], cb[2 * kBookSlots + ((r >> 2) & 3)]);
      v.y = h2bits(cb[2 * kBookSlots + ((r >> 4) & 3)], cb[2 * kBookSlots + (r >> 6)]);
      *reinterpret_cast<uint2*>(lut_mem + L::region_b_off + r * 256 + ln * 8) = v;
    }
  }
}

template <int KF, int VF, bool PACK, bool SPARSE>
__global__ void __launch_bounds__(kThreadsP, 1) decode_kernel(DecodeArgs a) {
  using FK = Fmt<KF>;
  using FV = Fmt<VF>;
  using L = Lut<KF, VF>;
  using CF = DecodeCfg<KF, VF>;
  constexpr int CH = CF::CH, WT = CF::WT, S = CF::S;
  using SL = StageLayout<KF, VF, CH>;
  constexpr int NX = PACK ? 1 : 2;
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_launch();  // the merge kernel may be scheduled as CTAs retire
  // Shared-memory layout (shared-window addresses): stages below kLutAddr
  // while they fit, the tables at kLutAddr, then the other stages and the
  // scratch area.  Checked against the allocation before anything runs.
  const uint32_t dyn0 = smem_u32(smem);
  uint32_t low0 = (dyn0 + 127u) & ~127u, n_low = 0;
  while (n_low < S && low0 + (n_low + 1) * SL::bytes <= kLutAddr) ++n_low;
  const uint32_t high0 = kLutAddr + L::bytes;
  uint32_t end = high0 + (S - n_low) * SL::bytes, scratch_addr;
  const uint32_t scr_bytes = kScratchBytes;
  if (low0 + n_low * SL::bytes + scr_bytes <= kLutAddr) {
    scratch_addr = low0 + n_low * SL::bytes;
  } else {
    scratch_addr = end;
    end += scr_bytes;
  }
  if (dyn0 > kLutAddr || end > dyn0 + a.dyn_bytes) {
    if (threadIdx.x == 0) atomicOr(a.status, 8);
    return;
  }
  auto stage_addr = [&](int s) -> uint32_t {
    return s < static_cast<int>(n_low) ? low0 + s * SL::bytes : high0 + (s - n_low) * SL::bytes;
  };
  float* scratch = reinterpret_cast<float*>(smem + (scratch_addr - dyn0));
  unsigned char* lut_mem = smem + (kLutAddr - dyn0);
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ long long s_c0, s_c1;
  __shared__ int s_u0, s_lc0;
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int P = gridDim.x, cta = blockIdx.x;
  const int U = a.B * a.hkv;

  // ---- codebooks to shared memory, schedule (warp 0) and barriers (thread 32);
  // the producer starts streaming right after, while the consumers build
  // the lookup tables
  __shared__ float s_cb[(kMaxBits + 1) * kBookSlots];
  if (tid < (kMaxBits + 1) * kBookSlots) s_cb[tid] = a.cbs[tid];
  if (warp == 0) {
    // schedule (one warp): total chunks C, this CTA's range [c0, c1) and the
    // unit / local chunk where it starts
    long long C = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      int ch = b0 + lane < a.B ? seq_chunks(a, b0 + lane, CH) : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ch += __shfl_xor_sync(0xffffffffu, ch, off);
      C += ch;
    }
    C *= a.hkv;
    const long long c0 = range_start(cta, C, P), c1 = range_start(cta + 1, C, P);
    int u0 = U, lc0 = 0;
    long long base = 0;
    for (int b0 = 0; b0 < a.B && c0 < c1; b0 += 32) {
      const int b = b0 + lane;
      const long long ch = b < a.B ? seq_chunks(a, b, CH) : 0;
      long long incl = ch;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const long long lo = base + (incl - ch) * a.hkv, hi = base + incl * a.hkv;
      const unsigned hit = __ballot_sync(0xffffffffu, b < a.B && ch > 0 && c0 >= lo && c0 < hi);
      if (hit) {
        const int src = __ffs(hit) - 1;
        if (lane == src) {
          const long long off = c0 - lo;
          const int h = static_cast<int>(off / ch);
          u0 = b * a.hkv + h;
          lc0 = static_cast<int>(off - h * ch);
        }
        u0 = __shfl_sync(0xffffffffu, u0, src);
        lc0 = __shfl_sync(0xffffffffu, lc0, src);
        break;
      }
      base += __shfl_sync(0xffffffffu, incl, 31) * a.hkv;
    }
    if (cta == 0)
      for (int b = lane; b < a.B; b += 32)
        if (a.lens[b] > a.max_len) atomicOr(a.status, 2);
    if (lane == 0) {
      s_c0 = c0;
      s_c1 = c1;
      s_u0 = u0;
      s_lc0 = lc0;
      s_abort = 0;
    }
  }
  if (tid == 32) {
#pragma unroll
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kConsumers);
    }
    mbar_fence_init();
  }
  __syncthreads();
  const long long c0 = s_c0, c1 = s_c1;

  if (warp == kConsumers) {
    // ---- producer: one lane streams the CTA's chunks through the stages
    if (lane == 0 && c0 < c1) {
      int u = s_u0, lc = s_lc0;
      UnitInfo ui = unit_info(a, u, CH);
      const int nk = static_cast<int>(c1 - c0);
      int s = 0;
      uint32_t round = 0;  // parity of k / S
      for (int k = 0; k < nk; ++k) {
        while (lc >= ui.chunks) {
          ++u;
          lc = 0;
          ui = unit_info(a, u, CH);
        }
        if (k >= S && !mbar_wait(&empty_bar[s], round ^ 1u)) s_abort = 1;
        if (s_abort) break;
        const int64_t ubase = static_cast<int64_t>(u) * a.capacity;
        const int r0 = lc * CH;
        const int rows = min(CH, (ui.nq + kTok - 1) / kTok * kTok - r0);  // <= capacity - r0
        const uint32_t st = stage_addr(s);
        uint64_t* bar = &full_bar[s];
        mbar_expect_tx(bar, SL::tx_bytes(rows));
        const int64_t row = ubase + r0;
        if constexpr (FK::code_bytes > 0) bulk_g2s_addr(st + SL::kc, a.k_codes + row * FK::code_bytes, rows * FK::code_bytes, bar);
        if constexpr (FV::code_bytes > 0) bulk_g2s_addr(st + SL::vc, a.v_codes + row * FV::code_bytes, rows * FV::code_bytes, bar);
        bulk_g2s_addr(st + SL::kn, a.k_norms + row, rows * 4, bar);
        bulk_g2s_addr(st + SL::vn, a.v_norms + row, rows * 4, bar);
        if constexpr (FK::prod) {
          bulk_g2s_addr(st + SL::kq, a.k_qjl + row * (kSketch / 8), rows * (kSketch / 8), bar);
          bulk_g2s_addr(st + SL::kr, a.k_res + row, rows * 4, bar);
        }
        if constexpr (FV::prod) {
          bulk_g2s_addr(st + SL::vq, a.v_qjl + row * (kSketch / 8), rows * (kSketch / 8), bar);
          bulk_g2s_addr(st + SL::vr, a.v_res + row, rows * 4, bar);
        }
        ++lc;
        if (++s == S) {
          s = 0;
          round ^= 1u;
        }
      }
    }
    return;
  }

  // ---- lookup tables (consumer threads)
  build_luts<L>(lut_mem, s_cb, tid);
  consumers_sync();  // tables complete

  // ---- consumers
  // table bases are folded into the lane offsets (see kLutAddr)
  const uint32_t lut_a = 0, lut_b = 0;
  const uint32_t lane4 = kLutAddr | (lane * 4), lane8 = (kLutAddr + L::region_b_off) | (lane * 8);
  const uint32_t c1k = FK::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const uint32_t c1v = FV::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const float thr = a.sparse_thr;
  const TokRows trows = tok_rows<KF, VF>(g, t);

  pdl_wait();  // the rotated query fragments

  WarpState<KF, VF, PACK> wst;
  QFrag<PACK> bq, bqs;
  int u = -1;
  UnitInfo ui{};
  int walk_u = s_u0, walk_lc = s_lc0;
  UnitInfo wui = c0 < c1 ? unit_info(a, walk_u, CH) : UnitInfo{};
  const int nk = static_cast<int>(c1 - c0);
  int s = 0;
  uint32_t round = 0;  // parity of k / S
  for (int k = 0; k < nk; ++k) {
    while (walk_lc >= wui.chunks) {
      ++walk_u;
      walk_lc = 0;
      wui = unit_info(a, walk_u, CH);
    }
    if (walk_u != u) {
      if (u >= 0) write_piece<KF, VF, PACK, true>(a, wst, u + cta, scratch, warp, g, t);
      u = walk_u;
      ui = wui;
      const uint32_t* qf = a.qfrag + static_cast<int64_t>(u) * kQfragWords;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int x = 0; x < NX; ++x) {
            bq[ks][r][x] = qf[((ks * 2 + r) * 2 + x) * 32 + lane];
            if constexpr (FK::prod) bqs[ks][r][x] = qf[(((8 + ks) * 2 + r) * 2 + x) * 32 + lane];
          }
#pragma unroll
      for (int i = 0; i < WarpState<KF, VF, PACK>::VMT; ++i) wst.oacc[i][0] = wst.oacc[i][1] = wst.oacc[i][2] = wst.oacc[i][3] = 0.f;
      wst.m0 = wst.m1 = -INFINITY;
      wst.l0 = wst.l1 = 0.f;
    }
    if (!s_abort && !mbar_wait(&full_bar[s], round)) s_abort = 1;
    const int row0 = walk_lc * CH + warp * WT;
    if (!s_abort && row0 < ui.nq) {
      const uint32_t st = stage_addr(s);
      UnitPlanes sp;
      sp.kcodes = st + SL::kc;
      sp.vcodes = st + SL::vc;
      sp.knorm = st + SL::kn;
      sp.vnorm = st + SL::vn;
      sp.kq = st + SL::kq;
      sp.kres = st + SL::kr;
      sp.vq = st + SL::vq;
      sp.vres = st + SL::vr;
      compute_tile<KF, VF, PACK, WT, SPARSE>(sp, warp * WT, row0, ui.nq, trows, wst, bq, bqs, g, t, lut_a, lut_b, lane4, lane8,
                                 c1k, c1v, thr);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    ++walk_lc;
    if (++s == S) {
      s = 0;
      round ^= 1u;
    }
  }
  if (u >= 0) write_piece<KF, VF, PACK, true>(a, wst, u + cta, scratch, warp, g, t);
  if (s_abort && tid == 0) atomicOr(a.status, 4);
}

// ---------------------------------------------------------------------------
// 4. Inner-product search over a quantized database (the method page's second
//    application: similarity search in place of product quantization).  Every
//    database row is scored with the estimator the decode kernel uses,
//    <q, x^> = ||x|| (<Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, z>) (query
//    scale 1 instead of log2(e)/sqrt(d)), and the k best rows per query are
//    kept: larger score first, equal scores in row order.
//
//    search_kernel: persistent, the decode kernel's producer / consumer
//    pipeline over contiguous ranges of database chunks (K planes only).
//    Each consumer warp keeps, per query, its best candidates as a sorted
//    column across its lanes (lane j = j-th best); a subtile's scores are
//    first tested against a per-query bound shared by the CTA's warps (the
//    best k-th score of any warp's list), and only rows that reach it are
//    inserted.  At the end the 15 warps' lists of each query are merged into
//    the CTA's list.
//    search_merge_kernel: one CTA per query merges the CTAs' lists.
// ---------------------------------------------------------------------------
constexpr int kSearchMaxK = 32;      // one list entry per lane
constexpr int kSearchMaxCtas = 256;  // bound on the search grid (merge stages all lists)

// Candidate key: the score in an order-preserving unsigned form above the
// complemented row, so a larger key is a better candidate (ties on the score
// go to the lower row).  0 stands for "no candidate".
__device__ __forceinline__ uint64_t cand_key(float v, uint32_t row) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t o = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(o) << 32) | static_cast<uint64_t>(~row);
}
__device__ __forceinline__ float key_score(uint64_t key) {
  if (key == 0) return -INFINITY;
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}
__device__ __forceinline__ int64_t key_row(uint64_t key) {
  return key == 0 ? -1 : static_cast<int64_t>(~static_cast<uint32_t>(key));
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
    v = o > v ? o : v;
  }
  return v;
}

// Insert the candidates c0..c3 (0: none) of the lanes into one query's list
// (lane j holds entry j).  Lanes below k hold the list; a candidate that does
// not beat entry k-1 is dropped.  Kept compact (one loop, no unrolling): it
// runs only for the rare rows that reach the bound.
__device__ __noinline__ uint64_t topk_offer(uint64_t ent, uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                            int lane, int k) {
  unsigned m0 = __ballot_sync(0xffffffffu, c0 != 0), m1 = __ballot_sync(0xffffffffu, c1 != 0);
  unsigned m2 = __ballot_sync(0xffffffffu, c2 != 0), m3 = __ballot_sync(0xffffffffu, c3 != 0);
#pragma unroll 1
  while (m0 | m1 | m2 | m3) {
    // the lowest pending lane of the first non-empty candidate set
    const int w = m0 ? 0 : m1 ? 1 : m2 ? 2 : 3;
    const unsigned m = w == 0 ? m0 : w == 1 ? m1 : w == 2 ? m2 : m3;
    const uint64_t c = w == 0 ? c0 : w == 1 ? c1 : w == 2 ? c2 : c3;
    const int src = __ffs(m) - 1;
    const unsigned rest = m & (m - 1);
    m0 = w == 0 ? rest : m0;
    m1 = w == 1 ? rest : m1;
    m2 = w == 2 ? rest : m2;
    m3 = w == 3 ? rest : m3;
    const uint64_t cc = __shfl_sync(0xffffffffu, c, src);
    const int pos = __popc(__ballot_sync(0xffffffffu, ent > cc));
    const uint64_t up = __shfl_up_sync(0xffffffffu, ent, 1);
    if (pos < k) {
      if (lane == pos)
        ent = cc;
      else if (lane > pos)
        ent = up;
    }
  }
  return ent;
}

// Order-preserving unsigned form of a score and back (ord_score(-inf) =
// 0x007FFFFF: the "no bound yet" threshold).
__device__ __forceinline__ uint32_t ord_score(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float unord_score(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}
constexpr uint32_t kNoBound = 0x007FFFFFu;  // ord_score(-inf)

// Offer the NS 16-token subtiles of one warp tile: for subtile i, lane
// (g, t) holds the scores of rows row[i][0] (s[i][0], s[i][1]) and row[i][1]
// (s[i][2], s[i][3]) for queries 2t and 2t + 1 (ok[i][*]: the row exists).
// The warp's lists live in shared memory, lists[h * 32 + j] = entry j of
// query h.  s_thr[h] (shared by the CTA's warps) is the best k-th score any
// warp's list of query h holds: a row scoring below it has k better rows
// listed already, so it cannot be in the result.  One reduction finds the
// queries with rows at or above their bound; only those are offered.
template <int NS>
__device__ __forceinline__ void offer_tile(uint64_t* lists, uint32_t* s_thr, const float (&s)[NS][4],
                                           const bool (&ok)[NS][2], const uint32_t (&row)[NS][2], int t, int lane,
                                           int Q, int k) {
  static_assert(NS == 1 || NS == 2, "one or two subtiles per warp tile");
  const int h0 = 2 * t, h1 = 2 * t + 1;
  const float b0 = h0 < Q ? unord_score(s_thr[h0 & (kMaxG - 1)]) : INFINITY;
  const float b1 = h1 < Q ? unord_score(s_thr[h1 & (kMaxG - 1)]) : INFINITY;
  bool p0 = false, p1 = false;
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    p0 |= (ok[i][0] && s[i][0] >= b0) || (ok[i][1] && s[i][2] >= b0);
    p1 |= (ok[i][0] && s[i][1] >= b1) || (ok[i][1] && s[i][3] >= b1);
  }
  unsigned heads = __reduce_or_sync(0xffffffffu, (p0 ? 1u << h0 : 0u) | (p1 ? 1u << h1 : 0u));
#pragma unroll 1
  while (heads) {
    const int h = __ffs(heads) - 1;
    heads &= heads - 1;
    const bool own = t == (h >> 1), odd = h & 1;
    const float th = odd ? b1 : b0;
    uint64_t c[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < NS; ++i) {
      const float va = odd ? s[i][1] : s[i][0], vb = odd ? s[i][3] : s[i][2];
      c[2 * i] = (own && ok[i][0] && va >= th) ? cand_key(va, row[i][0]) : 0;
      c[2 * i + 1] = (own && ok[i][1] && vb >= th) ? cand_key(vb, row[i][1]) : 0;
    }
    const uint64_t ent = topk_offer(lists[h * 32 + lane], c[0], c[1], c[2], c[3], lane, k);
    lists[h * 32 + lane] = ent;
    const uint64_t kth = __shfl_sync(0xffffffffu, ent, k - 1);
    if (lane == 0 && kth != 0) atomicMax(&s_thr[h], static_cast<uint32_t>(kth >> 32));
  }
}

template <int KF, bool PACK>
__global__ void __launch_bounds__(kThreadsP, 1) search_kernel(DecodeArgs a) {
  using FK = Fmt<KF>;
  using L = Lut<KF, 0>;
  using CF = DecodeCfg<KF, 0>;
  constexpr int CH = CF::CH, WT = CF::WT, S = CF::S;
  using SL = StageLayout<KF, 0, CH>;
  // up to 4 queries: high and low halves packed in one MMA; more: high halves only
  constexpr bool HI = !PACK;
  constexpr int kRowBytes = FK::code_bytes + 4 + (FK::prod ? kSketch / 8 + 4 : 0);
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_launch();  // the merge kernel may be scheduled as CTAs retire
  // shared-memory layout as in decode_kernel
  const uint32_t dyn0 = smem_u32(smem);
  uint32_t low0 = (dyn0 + 127u) & ~127u, n_low = 0;
  while (n_low < S && low0 + (n_low + 1) * SL::bytes <= kLutAddr) ++n_low;
  const uint32_t high0 = kLutAddr + L::bytes;
  uint32_t end = high0 + (S - n_low) * SL::bytes, scratch_addr;
  if (low0 + n_low * SL::bytes + kScratchBytes <= kLutAddr) {
    scratch_addr = low0 + n_low * SL::bytes;
  } else {
    scratch_addr = end;
    end += kScratchBytes;
  }
  if (dyn0 > kLutAddr || end > dyn0 + a.dyn_bytes) {
    if (threadIdx.x == 0) atomicOr(a.status, 8);
    return;
  }
  auto stage_addr = [&](int s) -> uint32_t {
    return s < static_cast<int>(n_low) ? low0 + s * SL::bytes : high0 + (s - n_low) * SL::bytes;
  };
  uint64_t* scratch = reinterpret_cast<uint64_t*>(smem + (scratch_addr - dyn0));
  unsigned char* lut_mem = smem + (kLutAddr - dyn0);
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ volatile int s_abort;
  __shared__ float s_cb[(kMaxBits + 1) * kBookSlots];
  __shared__ uint32_t s_thr[kMaxG];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int P = gridDim.x, cta = blockIdx.x;
  const int Q = a.group, k = a.topk;
  const int64_t n = a.n_db;
  const int64_t C = (n + CH - 1) / CH;
  const int64_t c0 = range_start(cta, C, P), c1 = range_start(cta + 1, C, P);
  if (tid < (kMaxBits + 1) * kBookSlots) s_cb[tid] = a.cbs[tid];
  if (tid >= 96 && tid < 96 + kMaxG) s_thr[tid - 96] = kNoBound;
  if (tid == 32) {
#pragma unroll
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kConsumers);
    }
    s_abort = 0;
    mbar_fence_init();
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---- producer: rows in groups of four by bulk copy (every plane slice a
    // multiple of 16 bytes), the last n % 4 rows by plain copies
    if (lane == 0 && c0 < c1) {
      const int nk = static_cast<int>(c1 - c0);
      int s = 0;
      uint32_t round = 0;
      for (int kk = 0; kk < nk; ++kk) {
        if (kk >= S && !mbar_wait(&empty_bar[s], round ^ 1u)) s_abort = 1;
        if (s_abort) break;
        const int64_t r0 = (c0 + kk) * CH;
        const int rows = static_cast<int>(n - r0 < CH ? n - r0 : CH);
        const int rows4 = rows & ~3;
        const uint32_t st = stage_addr(s);
        unsigned char* stp = smem + (st - dyn0);
        for (int r = rows4; r < rows; ++r) {
          const int64_t row = r0 + r;
          for (int w = 0; w < FK::code_bytes / 4; ++w)
            reinterpret_cast<uint32_t*>(stp + SL::kc + r * FK::code_bytes)[w] =
                reinterpret_cast<const uint32_t*>(a.k_codes + row * FK::code_bytes)[w];
          reinterpret_cast<float*>(stp + SL::kn)[r] = a.k_norms[row];
          if constexpr (FK::prod) {
            for (int w = 0; w < kSketch / 32; ++w)
              reinterpret_cast<uint32_t*>(stp + SL::kq + r * (kSketch / 8))[w] =
                  reinterpret_cast<const uint32_t*>(a.k_qjl + row * (kSketch / 8))[w];
            reinterpret_cast<float*>(stp + SL::kr)[r] = a.k_res[row];
          }
        }
        uint64_t* bar = &full_bar[s];
        if (rows4 > 0) {
          mbar_expect_tx(bar, static_cast<uint32_t>(rows4) * kRowBytes);
          if constexpr (FK::code_bytes > 0)
            bulk_g2s_addr(st + SL::kc, a.k_codes + r0 * FK::code_bytes, rows4 * FK::code_bytes, bar);
          bulk_g2s_addr(st + SL::kn, a.k_norms + r0, rows4 * 4, bar);
          if constexpr (FK::prod) {
            bulk_g2s_addr(st + SL::kq, a.k_qjl + r0 * (kSketch / 8), rows4 * (kSketch / 8), bar);
            bulk_g2s_addr(st + SL::kr, a.k_res + r0, rows4 * 4, bar);
          }
        } else {
          mbar_arrive(bar);
        }
        if (++s == S) {
          s = 0;
          round ^= 1u;
        }
      }
      // bulk copies still in flight land before the CTA may exit
      for (int kk = nk - S; kk < nk; ++kk)
        if (kk >= 0) mbar_wait(&full_bar[kk % S], (kk / S) & 1);
    }
    return;
  }

  // ---- lookup tables (consumer threads)
  build_luts<L>(lut_mem, s_cb, tid);
  consumers_sync();  // tables complete
  const uint32_t lut_a = 0, lut_b = 0;
  const uint32_t lane4 = kLutAddr | (lane * 4), lane8 = (kLutAddr + L::region_b_off) | (lane * 8);
  const uint32_t c1k = FK::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const TokRows tr = tok_rows<KF, 0>(g, t);

  pdl_wait();  // the rotated query fragments (and the starting bounds)
  if (a.bound_in && tid < Q) atomicMax(&s_thr[tid], a.bound_in[tid]);
  QFrag<true> bq, bqs;  // slot 0: packed halves, or (unpacked layout) the high halves
  {
    const uint32_t* qf = a.qfrag;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        bq[ks][r][0] = qf[((ks * 2 + r) * 2 + 0) * 32 + lane];
        if constexpr (FK::prod) bqs[ks][r][0] = qf[(((8 + ks) * 2 + r) * 2 + 0) * 32 + lane];
      }
  }
  // this warp's lists of the queries: [h][32] in the scratch area
  uint64_t* lists = scratch + warp * kMaxG * 32;
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) lists[h * 32 + lane] = 0;

  const int nk = static_cast<int>(c1 - c0);
  int s = 0;
  uint32_t round = 0;
  for (int kk = 0; kk < nk; ++kk) {
    if (!s_abort && !mbar_wait(&full_bar[s], round)) s_abort = 1;
    const int64_t row0 = (c0 + kk) * CH + warp * WT;
    const bool abort_w = __shfl_sync(0xffffffffu, static_cast<int>(s_abort), 0) != 0;  // one view per warp
    if (!abort_w && row0 < n) {
      const uint32_t st = stage_addr(s);
      UnitPlanes sp;
      sp.kcodes = st + SL::kc;
      sp.knorm = st + SL::kn;
      sp.kq = st + SL::kq;
      sp.kres = st + SL::kr;
      sp.vcodes = sp.vnorm = sp.vq = sp.vres = 0;
      // both subtiles' scores first (their lookup and MMA chains
      // interleave), then one offer
      constexpr int NS = WT / kTok;
      float sc[NS][4];
      bool ok[NS][2];
      uint32_t rows[NS][2];
#pragma unroll
      for (int sub = 0; sub < NS; ++sub) {
        const int64_t rb = row0 + sub * kTok;
        ok[sub][0] = rb + tr.kA < n;
        ok[sub][1] = rb + tr.kB < n;
        rows[sub][0] = static_cast<uint32_t>(rb + tr.kA);
        rows[sub][1] = static_cast<uint32_t>(rb + tr.kB);
        subtile_scores<KF, PACK, L::t3_wide, L::t2a, HI>(sp, warp * WT + sub * kTok, tr, ok[sub][0], ok[sub][1], g,
                                                          t, bq, bqs, lut_a, lut_b, lane4, lane8, c1k, sc[sub]);
      }
      offer_tile<NS>(lists, s_thr, sc, ok, rows, t, lane, Q, k);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    if (++s == S) {
      s = 0;
      round ^= 1u;
    }
  }

  // ---- the CTA's list per query: merge the consumer warps' lists
  consumers_sync();
  if (warp < Q) {
    const int h = warp;
    int pos = 0;
    uint64_t head = lane < kConsumers ? scratch[(lane * kMaxG + h) * 32] : 0;
    uint64_t* dst = a.cand + (static_cast<int64_t>(h) * P + cta) * 32;
    for (int r = 0; r < 32; ++r) {
      const uint64_t best = warp_max_u64(head);
      if (lane == 0) dst[r] = best;
      if (best != 0 && head == best) {  // keys are unique apart from 0
        ++pos;
        head = pos < 32 ? scratch[(lane * kMaxG + h) * 32 + pos] : 0;
      }
    }
  }
  if (s_abort && tid == 0) atomicOr(a.status, 4);
}

// One CTA per query: the top k of the CTAs' sorted lists.
constexpr int kSearchMergeThreads = 256;
__global__ void __launch_bounds__(kSearchMergeThreads) search_merge_kernel(DecodeArgs a) {
  extern __shared__ uint64_t s_keys[];  // [ctas][32]
  const int h = blockIdx.x, P = a.ctas, k = a.topk, tid = threadIdx.x, lane = tid & 31;
  pdl_wait();  // the CTAs' lists
  const uint64_t* src = a.cand + static_cast<int64_t>(h) * P * 32;
  for (int i = tid; i < P * 32; i += kSearchMergeThreads) s_keys[i] = src[i];
  __syncthreads();
  if (tid >= 32) return;
  // lane owns lists lane, lane + 32, ... (at most kSearchMaxCtas / 32)
  constexpr int J = kSearchMaxCtas / 32;
  int pos[J];
  uint64_t head[J];
  uint64_t mine = 0;
#pragma unroll
  for (int j = 0; j < J; ++j) {
    const int l = lane + 32 * j;
    pos[j] = 0;
    head[j] = l < P ? s_keys[l * 32] : 0;
    mine = head[j] > mine ? head[j] : mine;
  }
  float* os = a.out_scores + static_cast<int64_t>(h) * k;
  int64_t* orow = a.out_rows + static_cast<int64_t>(h) * k;
  for (int r = 0; r < k; ++r) {
    const uint64_t best = warp_max_u64(mine);
    if (lane == 0) {
      if (a.bound_out) {
        // k rows score at least the k-th best: a bound for the full pass
        if (r == k - 1) a.bound_out[h] = best != 0 ? static_cast<uint32_t>(best >> 32) : kNoBound;
      } else {
        os[r] = key_score(best);
        orow[r] = key_row(best);
      }
    }
    if (best != 0 && mine == best) {
      uint64_t m = 0;
#pragma unroll
      for (int j = 0; j < J; ++j) {
        if (head[j] == best) {
          ++pos[j];
          head[j] = pos[j] < 32 ? s_keys[(lane + 32 * j) * 32 + pos[j]] : 0;
        }
        m = head[j] > m ? head[j] : m;
      }
      mine = m;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int num_sms_cached() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

template <int KF, int VF>
size_t decode_smem_bytes() {
  using CF = DecodeCfg<KF, VF>;
  return static_cast<size_t>(plan_end(CF::stage, CF::S, CF::lut, kScratchBytes) - kDynBaseMax);
}
template <int KF, int VF>
constexpr bool decode_smem_bytes_fits() {
  using CF = DecodeCfg<KF, VF>;
  return plan_end(CF::stage, CF::S, CF::lut, kScratchBytes) <= kSmemEnd;
}

// Launch with programmatic stream serialization: the kernel may start before
// the previous kernel on the stream has finished (it calls pdl_wait before
// reading that kernel's output).
template <typename Kernel>
cudaError_t launch_overlapped(Kernel kernel, dim3 grid, int threads, size_t smem, cudaStream_t st,
                              const DecodeArgs& a) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

template <int KF, int VF, bool PACK, bool SPARSE>
tq_status run_decode_v(DecodeArgs& a, const DecodePlan& plan, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_dyn_smem<decode_kernel<KF, VF, PACK, SPARSE>>(static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel attribute");
  // the query rotation waits for all earlier work on the stream (the appends
  // that filled the cache); the two kernels after it overlap their prologues
  // with its tail
  const size_t qrot_smem = static_cast<size_t>(Fmt<KF>::prod ? 2 : 1) * kDim * kDim * sizeof(float);
  e = ensure_dyn_smem<qrot_kernel<KF>>(static_cast<int>(qrot_smem));
  if (e != cudaSuccess) return cuda_fail(e, "query rotation attribute");
  qrot_kernel<KF><<<dim3(plan.hkv, plan.B), kQrotThreads, qrot_smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "query rotation launch");
  e = launch_overlapped(decode_kernel<KF, VF, PACK, SPARSE>, dim3(plan.ctas), kThreadsP, smem, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  const size_t merge_smem = merge_dyn_bytes(a.n_sink, plan.ctas, plan.group, plan.part_floats);
  if (merge_smem > 48 * 1024) {
    e = ensure_dyn_smem<merge_kernel<VF>>(static_cast<int>(merge_smem));
    if (e != cudaSuccess) return cuda_fail(e, "merge kernel attribute");
  }
  e = launch_overlapped(merge_kernel<VF>, dim3(plan.B * plan.hkv), kMergeThreads, merge_smem, st, a);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "merge kernel launch");
}

template <int KF, int VF>
tq_status run_decode(DecodeArgs& a, const DecodePlan& plan, cudaStream_t st) {
  if (decode_smem_bytes<KF, VF>() + kDynBaseMax > static_cast<size_t>(kSmemEnd))
    return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: no shared-memory plan for this format");
  const size_t smem = kSmemBudget;  // the whole window: one CTA per SM
  a.dyn_bytes = static_cast<uint32_t>(smem);
  a.pack = plan.group <= 4;
  a.chunk = DecodeCfg<KF, VF>::CH;
  if (a.sparse_thr > 0.f)
    return a.pack ? run_decode_v<KF, VF, true, true>(a, plan, smem, st) : run_decode_v<KF, VF, false, true>(a, plan, smem, st);
  return a.pack ? run_decode_v<KF, VF, true, false>(a, plan, smem, st) : run_decode_v<KF, VF, false, false>(a, plan, smem, st);
}

constexpr int fid(int mse, int mixed, int prod) { return mse | (mixed << 3) | (prod << 4); }

template <int KF, bool PACK>
tq_status run_search(DecodeArgs& a, int groups_ctas, cudaStream_t st) {
  static_assert(decode_smem_bytes_fits<KF, 0>(), "no shared-memory plan for this search format");
  // A large database is searched twice: first its leading rows, one chunk
  // per CTA, whose k-th best score per query becomes the starting bound of
  // the full pass (k rows reach it, so rows below it are never results);
  // the full pass then inserts few rows into its lists.
  const int64_t n_pre = static_cast<int64_t>(groups_ctas) * DecodeCfg<KF, 0>::CH;
  const bool prefix = a.bound_out != nullptr && a.n_db >= 8 * n_pre;
  uint32_t* bound = a.bound_out;
  a.bound_out = nullptr;
  cudaError_t e = ensure_dyn_smem<search_kernel<KF, PACK>>(kSmemBudget);
  if (e != cudaSuccess) return cuda_fail(e, "search kernel attribute");
  const size_t qrot_smem = static_cast<size_t>(Fmt<KF>::prod ? 2 : 1) * kDim * kDim * sizeof(float);
  e = ensure_dyn_smem<qrot_kernel<KF>>(static_cast<int>(qrot_smem));
  if (e != cudaSuccess) return cuda_fail(e, "query rotation attribute");
  qrot_kernel<KF><<<dim3(1, 1), kQrotThreads, qrot_smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "query rotation launch");
  const size_t merge_smem = static_cast<size_t>(groups_ctas) * 32 * sizeof(uint64_t);
  if (merge_smem > 48 * 1024) {
    e = ensure_dyn_smem<search_merge_kernel>(static_cast<int>(merge_smem));
    if (e != cudaSuccess) return cuda_fail(e, "search merge attribute");
  }
  a.bound_in = nullptr;
  if (prefix) {
    DecodeArgs pre = a;
    pre.n_db = n_pre;
    pre.bound_out = bound;
    e = launch_overlapped(search_kernel<KF, PACK>, dim3(groups_ctas), kThreadsP, kSmemBudget, st, pre);
    if (e != cudaSuccess) return cuda_fail(e, "search kernel launch");
    e = launch_overlapped(search_merge_kernel, dim3(a.group), kSearchMergeThreads, merge_smem, st, pre);
    if (e != cudaSuccess) return cuda_fail(e, "search merge launch");
    a.bound_in = bound;
  }
  e = launch_overlapped(search_kernel<KF, PACK>, dim3(groups_ctas), kThreadsP, kSmemBudget, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "search kernel launch");
  e = launch_overlapped(search_merge_kernel, dim3(a.group), kSearchMergeThreads, merge_smem, st, a);
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "search merge launch");
}

}  // namespace

DecodePlan plan_decode(const tq_params* p, int B, int hq, int hkv, int max_len) {
  DecodePlan pl{};
  pl.B = B;
  pl.hq = hq;
  pl.hkv = hkv;
  pl.group = hq / hkv;
  pl.max_len = max_len;
  pl.ctas = num_sms_cached() < kMaxPieces ? num_sms_cached() : kMaxPieces;
  pl.part_floats = kPartAcc + (p->fv.prod ? 2 * kDim : kDim);
  const size_t units = static_cast<size_t>(B) * hkv;
  const size_t qfrag = (units * kQfragWords * sizeof(uint32_t) + 255) & ~size_t(255);
  // piece (u, cta) uses slot u + cta: fewer than units + ctas slots
  const size_t slots = units + pl.ctas;
  pl.ws_total_bytes = qfrag + slots * pl.group * pl.part_floats * sizeof(float);
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
  a.B = plan.B;
  a.hkv = plan.hkv;
  a.group = plan.group;
  a.hq = plan.hq;
  a.capacity = c->capacity;
  a.n_sink = c->n_sink;
  a.max_len = plan.max_len;
  a.part_floats = plan.part_floats;
  a.ctas = plan.ctas;
  a.merge_chunk = merge_chunk_pieces(plan.group, plan.part_floats);
  if (c->n_sink > kMaxSink) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: n_sink above 4096");
  const size_t units = static_cast<size_t>(plan.B) * plan.hkv;
  char* w = static_cast<char*>(ws);
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
  a.qscale = kLog2e / std::sqrt(static_cast<float>(kDim));

  const int kf = p->fk.id(), vf = p->fv.id();
#define TQ_CASE(K, V) \
  if (kf == (K) && vf == (V)) return run_decode<(K), (V)>(a, plan, st);
  // symmetric formats
  TQ_CASE(fid(1, 0, 0), fid(1, 0, 0))
  TQ_CASE(fid(2, 0, 0), fid(2, 0, 0))
  TQ_CASE(fid(3, 0, 0), fid(3, 0, 0))
  TQ_CASE(fid(4, 0, 0), fid(4, 0, 0))
  TQ_CASE(fid(3, 1, 0), fid(3, 1, 0))
  TQ_CASE(fid(2, 1, 0), fid(2, 1, 0))
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

int search_ctas() { return std::min(num_sms_cached(), kSearchMaxCtas); }

size_t search_workspace_bytes() {
  return static_cast<size_t>(kQfragWords) * sizeof(uint32_t) +
         static_cast<size_t>(kMaxG) * search_ctas() * 32 * sizeof(uint64_t) + 256;
}

int search_max_k() { return kSearchMaxK; }

tq_status launch_search(const tq_params* p, const FormatSpec& f, const tq_packed* db, int64_t n, const void* q,
                        int q_bf16, int n_queries, int k, float* scores, int64_t* rows, void* ws,
                        cudaStream_t st) {
  const int P = search_ctas();
  char* w = static_cast<char*>(ws);
  for (int g0 = 0; g0 < n_queries; g0 += kMaxG) {
    // one pass over the database per group of up to kMaxG queries
    DecodeArgs a{};
    a.group = std::min(kMaxG, n_queries - g0);
    a.q = static_cast<const char*>(q) + static_cast<size_t>(g0) * kDim * (q_bf16 ? 2 : 4);
    a.q_bf16 = q_bf16;
    a.k_codes = db->codes;
    a.k_norms = db->norms;
    a.k_qjl = db->qjl;
    a.k_res = db->res_norms;
    a.status = p->status32;
    a.B = 1;
    a.hkv = 1;
    a.hq = a.group;
    a.ctas = P;
    a.qfrag = reinterpret_cast<uint32_t*>(w);
    a.cand = reinterpret_cast<uint64_t*>(w + kQfragWords * sizeof(uint32_t));
    a.bound_out = reinterpret_cast<uint32_t*>(w + kQfragWords * sizeof(uint32_t) +
                                              static_cast<size_t>(kMaxG) * P * 32 * sizeof(uint64_t));
    a.pit = p->pit32;
    a.st = p->st32;
    a.pi = p->pi32;
    a.s = p->s32;
    a.cbs = p->cbs32;
    a.sig = p->sig32;
    a.pack = a.group <= 4;
    a.dyn_bytes = kSmemBudget;
    a.qscale = 1.f;
    a.n_db = n;
    a.topk = k;
    a.out_scores = scores + static_cast<size_t>(g0) * k;
    a.out_rows = rows + static_cast<size_t>(g0) * k;
    tq_status r = TQ_ERR_UNSUPPORTED;
    const int kf = f.id();
#define TQ_CASE(K)                                                                           \
  if (kf == (K)) r = a.pack ? run_search<(K), true>(a, P, st) : run_search<(K), false>(a, P, st); \
  else
    TQ_CASE(fid(1, 0, 0))
    TQ_CASE(fid(2, 0, 0))
    TQ_CASE(fid(3, 0, 0))
    TQ_CASE(fid(4, 0, 0))
    TQ_CASE(fid(2, 1, 0))
    TQ_CASE(fid(3, 1, 0))
    TQ_CASE(fid(0, 0, 1))
    TQ_CASE(fid(1, 0, 1))
    TQ_CASE(fid(2, 0, 1))
    TQ_CASE(fid(3, 0, 1))
    return fail(TQ_ERR_UNSUPPORTED, "tq_search: no search kernel for this format");
#undef TQ_CASE
    if (r != TQ_OK) return r;
  }
  return TQ_OK;
}

}  // namespace tq
