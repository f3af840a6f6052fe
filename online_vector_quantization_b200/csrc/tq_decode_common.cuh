// Building blocks shared by the decode-attention kernels (tq_attn.cu) and the
// inner-product search kernels (tq_search.cu): the packed-row formats, the
// shared-memory lookup tables of codebook values, the decoding of code
// chunks into fp16 MMA fragments, the query rotation kernel, the pipeline
// stage layout and the scoring of one 16-token subtile.
//
// Method: page "TurboQuant-MLX: quantizzare pesi e KV cache per LLM
// open-weight su Mac", section "Il metodo TurboQuant, in breve": a key is
// ||k|| Pi^T c[idx] (+ the QJL correction sqrt(pi/2)/m ||r|| S^T z), so
//   <q, k> = ||k|| ( <Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, z> ).
// Everything here lives in an unnamed namespace: each including file gets
// its own copy.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_internal.h"
#include "tq_layout.cuh"
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
// Formats (id = mse_bits | mixed << 4 | prod << 5).  Segments of the MSE row:
// one uniform segment of 128 coordinates, or (mixed) 64 coordinates at
// mse+1 bits followed by 64 at mse bits.
// ---------------------------------------------------------------------------
template <int F>
struct Fmt {
  static constexpr int mse = F & 15;
  static constexpr bool mixed = (F >> 4) & 1;
  static constexpr bool prod = (F >> 5) & 1;
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
// r hold half2(c2[r & 3], c2[(r >> 2) & 3]) instead, and there is no region B.
// With 8-bit keys (t8), bytes [0, 128) of row r hold half2(c8[r], c8[r]): one
// code byte, one lookup.  Entry (r, lane) sits at r*256 + lane*4 (or *8):
// every lane hits its own bank.
template <int KF, int VF>
struct Lut {
  static constexpr bool t8 = Fmt<KF>::uses(8);
  static constexpr bool t4 = Fmt<KF>::uses(4) || Fmt<VF>::uses(4);
  static constexpr bool t3 = Fmt<KF>::uses(3) || Fmt<VF>::uses(3);
  static constexpr bool t2 = Fmt<KF>::uses(2) || Fmt<VF>::uses(2);
  static_assert(!Fmt<VF>::uses(8), "8-bit codes are decoded on the key side only");
  static_assert(!(t8 && (t4 || t2)), "8-bit keys pair with 3-bit (or 1-bit) values");
  static constexpr int region_a = (t8 || t4 || (t3 && t2)) ? 65536 : (t3 ? 16384 : 0);
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
    if constexpr (BYTES == 32) {
      const uint4 v0 = lds128(row, o), v1 = lds128(row, o + 16);
      w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
      w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    } else if constexpr (BYTES == 16) {
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

  // the lane's piece at byte OFF of its lane block in a tiled code plane
  template <int OFF, typename Blk>
  __device__ __forceinline__ void from_block(const Blk& blk) {
    blk.template words<OFF, WORDS>(w);
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
    } else if constexpr (B == 8) {
      // one lookup per code byte; the low halves of two entries form a pair
      const uint32_t ww = w[s];
      const uint32_t e0 = lut32(smem, byte_addr(ww, lane4, 0)), e1 = lut32(smem, byte_addr(ww, lane4, 1));
      const uint32_t e2 = lut32(smem, byte_addr(ww, lane4, 2)), e3 = lut32(smem, byte_addr(ww, lane4, 3));
      lo = __byte_perm(e0, e1, 0x5410);
      hi = __byte_perm(e2, e3, 0x5410);
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

  // the token's piece (ND * B / 64 bytes) at byte OFF of the lane block
  template <int OFF, typename Blk>
  __device__ __forceinline__ void from_block(const Blk& blk) {
    constexpr int bits = ND * B / 8;
    uint32_t v[2];
    blk.template words<OFF, 2>(v);
    const uint64_t y = static_cast<uint64_t>(v[0]) | (static_cast<uint64_t>(v[1]) << 32);
    x = bits == 64 ? y : (y & ((1ull << bits) - 1ull));
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

// One lane's block of a tiled code plane (see tq_layout.cuh): loaded with one
// 16-, 8- and 4-byte shared load per column, conflict-free across the warp.
template <int F>
__host__ __device__ constexpr CodeTile code_tile() {
  return make_code_tile(Fmt<F>::mse, Fmt<F>::mixed, Fmt<F>::code_bytes);
}

template <int F>
struct LaneBlock {
  static constexpr CodeTile CT = code_tile<F>();
  static constexpr int WORDS = CT.lane_bytes() / 4 > 0 ? CT.lane_bytes() / 4 : 1;
  uint32_t w[WORDS];

  // tile: shared address of the 16-token tile
  __device__ __forceinline__ void load(uint32_t tile, int lane) {
    static_for<CT.c16()>([&](auto jj) {
      constexpr int j = decltype(jj)::value;
      const uint4 v = lds128(tile, j * 512 + lane * 16);
      w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
    });
    if constexpr (CT.c8() > 0) {
      const uint2 v = lds64(tile, 512 * CT.c16() + lane * 8);
      w[4 * CT.c16()] = v.x;
      w[4 * CT.c16() + 1] = v.y;
    }
    if constexpr (CT.c4() > 0) w[4 * CT.c16() + 2 * CT.c8()] = lds32(tile, 512 * CT.c16() + 256 * CT.c8() + lane * 4);
  }

  // NW little-endian words starting at byte OFF of the block (bytes past the
  // block's end are unspecified)
  template <int OFF, int NW>
  __device__ __forceinline__ void words(uint32_t (&out)[NW]) const {
    constexpr int w0 = OFF / 4, sh = (OFF % 4) * 8;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const uint32_t lo = w[min(w0 + i, WORDS - 1)], hi = w[min(w0 + i + 1, WORDS - 1)];
      out[i] = sh == 0 ? lo : __funnelshift_r(lo, hi, sh);
    }
  }
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
  int unit_slack;  // empty schedule slots at the start of each unit
  int merge_chunk;  // pieces the merge kernel stages in shared memory at a time
  int merge_heads;  // query heads per merge CTA (the group, or 1: one CTA per (unit, head))
  float* parts;
  const uint32_t* qfrag;

  void* out;
  int out_bf16;
  const float* pit;  // Pi^T
  const float* st;   // S^T
  const float* pi;   // Pi
  const float* s;    // S
  const float* cbs;  // sigma-scaled centroids [5][16] (the values the MMAs see)
  const float* cbs8;  // sigma-scaled 8-bit centroids [256] (8-bit formats)
  const uint8_t* lut_img;  // the decode kernel's lookup tables, prebuilt (params)
  const float* sig;  // sigma per width [5]
  float sparse_thr;
  unsigned long long* sv_stats;  // sparse-V tallies [4] (device) or null
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

// B fragments of a rotated query: lane (g, t) supplies column g; k-steps 0..7
// from the MSE segments, 8..15 from the QJL segment.  Unpacked: column g =
// head g, halves hi (x = 0) and lo (x = 1).  Packed (group <= 4): column g < 4
// = hi of head g, column g >= 4 = lo of head g - 4, in x = 0.  Word
// ((ks * 2 + r) * 2 + x) * 32 + lane of a unit's kQfragWords.
//
// The coordinates behind the words of k-step ks for lane quarter t (dims[0..3]
// = halves lo.x, lo.y, hi.x, hi.y); false where the format leaves the k-step
// unused.  All four lie in one 32-coordinate block (block 0 for an unused
// k-step).
template <int KF>
__host__ __device__ __forceinline__ bool qfrag_dims(int ks, int t, int (&dims)[4]) {
  using KR = KRow<KF>;
  using FK = Fmt<KF>;
  for (int e = 0; e < 4; ++e) dims[e] = 0;
  if (ks < 8) {
    if constexpr (FK::nseg == 0) {
      return false;
    } else {
      if (FK::nseg == 1 || ks < KR::S0::KSTEPS) {
        for (int e = 0; e < 4; ++e) dims[e] = KR::S0::dim(0, t, ks, e);
      } else {
        for (int e = 0; e < 4; ++e) dims[e] = KR::S1::dim(64, t, ks - KR::S0::KSTEPS, e);
      }
      return true;
    }
  }
  if constexpr (!FK::prod) {
    return false;
  } else {
    for (int e = 0; e < 4; ++e) dims[e] = KR::Q::dim(0, t, ks - 8, e);
    return true;
  }
}

// ---------------------------------------------------------------------------
// 1. query rotation: Pi q (MSE keys) and S q (prod keys) as fp16 fragments.
//    One CTA per (32-coordinate slice of one matrix, kv-head, sequence):
//    blockIdx.x = 4 * m + slice, m = 0 for Pi (formats with MSE codes), the
//    last m for S (prod keys).  Thread (jj, ks) sums k in [16 ks, 16 ks + 16)
//    for output coordinate 32 slice + jj of every head, the 8 partial sums
//    meet in shared memory, and the slice writes the fragment words whose
//    coordinates it holds (qfrag_dims keeps each word inside one slice).
// ---------------------------------------------------------------------------
constexpr int kQrotThreads = 256;
constexpr int kQrotSlice = 32;                          // output coordinates per CTA
constexpr int kQrotKSplit = kQrotThreads / kQrotSlice;  // slices of the k range
constexpr int kQrotK = kDim / kQrotKSplit;              // k per thread

template <int KF>
constexpr int qrot_matrices() {
  return (Fmt<KF>::nseg > 0 ? 1 : 0) + (Fmt<KF>::prod ? 1 : 0);
}

template <int KF>
__global__ void __launch_bounds__(kQrotThreads) qrot_kernel(DecodeArgs a) {
  using FK = Fmt<KF>;
  __shared__ __align__(16) float qsT[kDim][kMaxG];  // query, [k][head]
  __shared__ float s_p[kQrotKSplit][kMaxG][kQrotSlice];
  __shared__ float s_v[kMaxG][kQrotSlice];          // the slice's scaled outputs
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int m = (FK::nseg > 0 ? 0 : 1) + static_cast<int>(blockIdx.x) / 4, sl = blockIdx.x % 4;
  const int G = a.group;
  const int jj = tid % kQrotSlice, kq = tid / kQrotSlice, j = sl * kQrotSlice + jj;
  // this thread's matrix entries (Pi^T or S^T, [k][j]: coalesced over j)
  const float* mat = m ? a.st : a.pit;
  float mv[kQrotK];
#pragma unroll
  for (int i = 0; i < kQrotK; ++i) mv[i] = __ldg(mat + (kq * kQrotK + i) * kDim + j);
  // Launched behind the previous kernel on the stream (an append, say), the
  // matrix loads above overlap its tail; the query, and the cache lengths the
  // decode kernel reads, are only read once that kernel has finished.
  pdl_wait();
  pdl_launch();  // the decode kernel's prologue and cache stream may start
  for (int i = tid; i < kMaxG * kDim; i += kQrotThreads) {
    const int h = i % kMaxG, d = i / kMaxG;
    qsT[d][h] = h < G ? load_q(a.q, a.q_bf16, (static_cast<int64_t>(b) * a.hq + kvh * G + h) * kDim + d) : 0.f;
  }
  __syncthreads();
  float acc[kMaxG];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) acc[h] = 0.f;
  const float4* q4 = reinterpret_cast<const float4*>(&qsT[0][0]);
#pragma unroll
  for (int i = 0; i < kQrotK; ++i) {
    const int k = kq * kQrotK + i;
    const float4 x0 = q4[2 * k], x1 = q4[2 * k + 1];
    acc[0] = fmaf(mv[i], x0.x, acc[0]);
    acc[1] = fmaf(mv[i], x0.y, acc[1]);
    acc[2] = fmaf(mv[i], x0.z, acc[2]);
    acc[3] = fmaf(mv[i], x0.w, acc[3]);
    acc[4] = fmaf(mv[i], x1.x, acc[4]);
    acc[5] = fmaf(mv[i], x1.y, acc[5]);
    acc[6] = fmaf(mv[i], x1.z, acc[6]);
    acc[7] = fmaf(mv[i], x1.w, acc[7]);
  }
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) s_p[kq][h][jj] = acc[h];
  __syncthreads();
  {
    const int h = tid / kQrotSlice;  // kQrotThreads = kMaxG * kQrotSlice
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < kQrotKSplit; ++i) v += s_p[i][h][jj];
    if (m == 0) {
      const int wj = FK::width(j);
      v = wj > 0 ? v * (a.qscale / a.sig[wj]) : 0.f;
    } else {
      v *= a.qscale;
    }
    s_v[h][jj] = v;
  }
  __syncthreads();
  // the words of this matrix's k-steps whose coordinates lie in the slice
  uint32_t* dst = const_cast<uint32_t*>(a.qfrag) + (static_cast<int64_t>(b) * a.hkv + kvh) * kQfragWords;
  {
    const int ks = 8 * m + tid / 32, lane = tid % 32, g = lane >> 2, t = lane & 3;
    int dims[4];
    if (qfrag_dims<KF>(ks, t, dims) && dims[0] / kQrotSlice == sl) {
      const int head = a.pack ? (g & 3) : g;
      const float* src = &s_v[head][0];
      const int o = sl * kQrotSlice;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const float x0 = src[dims[2 * r] - o], x1 = src[dims[2 * r + 1] - o];
        const __half2 hv = __floats2half2_rn(x0, x1);
        const float2 hf = __half22float2(hv);
        const uint32_t hi = *reinterpret_cast<const uint32_t*>(&hv);
        const uint32_t lo = h2bits(x0 - hf.x, x1 - hf.y);
        if (a.pack) {
          dst[((ks * 2 + r) * 2 + 0) * 32 + lane] = g < 4 ? hi : lo;
          dst[((ks * 2 + r) * 2 + 1) * 32 + lane] = 0;
        } else {
          dst[((ks * 2 + r) * 2 + 0) * 32 + lane] = hi;
          dst[((ks * 2 + r) * 2 + 1) * 32 + lane] = lo;
        }
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

// This lane's rows within a 16-token subtile: K rows (score rows g, g + 8)
// and V rows (MMA columns 2t, 2t + 1, 2t + 8, 2t + 9).  In a tiled code plane
// the tile layout already gives every lane its own banks, so tokens sit in
// MMA row / column order.
struct TokRows {
  int kA, kB, v0, v1, v8, v9;
};
__device__ __forceinline__ TokRows tok_rows(int g, int t) {
  return TokRows{g, g + 8, 2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
}

// Scores of one 16-token subtile whose rows start at `srow` of the staged
// planes: s2 (base 2) for tokens g (s2[0], s2[1]) and g+8 (s2[2], s2[3]),
// columns 2t, 2t+1; masked tokens get -inf.  Two MMA accumulator chains.
// HI: the query's fp16 high halves only (column g = head g, no low halves):
// one MMA per k-step for up to 8 heads, scores within about 2^-12 of
// ||q|| ||x|| (the search's precision; attention keeps both halves).
// TILED: the K code plane is a tiled cache plane (tq_layout.cuh: token g and
// g + 8 of the subtile are this lane's rows A and B); otherwise rows are
// packed rows in token order tr (the search's database).
template <int KF, bool PACK, bool T3W, bool T2A, bool HI = false, bool TILED = false>
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
  [[maybe_unused]] LaneBlock<KF> blk;
  if constexpr (TILED && FK::nseg > 0) blk.load(u.kcodes + (srow >> 4) * code_tile<KF>().tile_bytes(), 4 * g + t);
  if constexpr (FK::nseg > 0) {
    typename KR::S0 xa, xb;
    if constexpr (TILED) {
      xa.template from_block<code_tile<KF>().koff(0, 0)>(blk);
      xb.template from_block<code_tile<KF>().koff(1, 0)>(blk);
    } else {
      xa.load(ka, t);
      xb.load(kb, t);
    }
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
    if constexpr (TILED) {
      xa.template from_block<code_tile<KF>().koff(0, 1)>(blk);
      xb.template from_block<code_tile<KF>().koff(1, 1)>(blk);
    } else {
      xa.load(ka, t);
      xb.load(kb, t);
    }
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

__device__ __forceinline__ int64_t range_start(int i, int64_t C, int P) { return static_cast<int64_t>(i) * C / P; }

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kConsumers * 32) : "memory");
}

// The lookup tables of a format pair (see Lut), written by the consumer
// threads (thread index tid < kConsumers * 32) from the sigma-scaled
// centroids cb (widths 1..4) and cb8 (the 8-bit codebook, 8-bit keys only).
template <typename L>
__device__ __forceinline__ void build_luts(unsigned char* lut_mem, const float* cb, int tid,
                                           const float* cb8 = nullptr) {
  constexpr int NTC = kConsumers * 32;
  if constexpr (L::t8) {
    for (int i = tid; i < 256 * 32; i += NTC) {
      const int r = i >> 5, ln = i & 31;
      *reinterpret_cast<uint32_t*>(lut_mem + r * 256 + ln * 4) = h2bits(cb8[r], cb8[r]);
    }
  }
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

// The query rotation of B sequences x hkv kv-heads; overlapped: launched with
// programmatic stream serialization (see qrot_kernel).
template <int KF>
cudaError_t launch_qrot(const DecodeArgs& a, int B, int hkv, cudaStream_t st, bool overlapped = false) {
  const cudaError_t e = ensure_max_carveout<qrot_kernel<KF>>();
  if (e != cudaSuccess) return e;
  const dim3 grid(4 * qrot_matrices<KF>(), hkv, B);
  if (overlapped) return launch_overlapped(qrot_kernel<KF>, grid, kQrotThreads, 0, st, a);
  qrot_kernel<KF><<<grid, kQrotThreads, 0, st>>>(a);
  return cudaGetLastError();
}

constexpr int fid(int mse, int mixed, int prod) { return mse | (mixed << 4) | (prod << 5); }

}  // namespace
}  // namespace tq
