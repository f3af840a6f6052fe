// Rotate + quantize + pack kernels (plain rows and streaming cache append) and
// the fp64 dequantizer.
//
// Method: page "TurboQuant-MLX: quantizzare pesi e KV cache per LLM
// open-weight su Mac", section "Il metodo TurboQuant, in breve" -- rotate by
// Pi, quantize each rotated coordinate of the unit vector to its Lloyd-Max
// centroid, keep the norm; the prod variant adds sign(S r) of the residual.
// Streaming append in 64-token chunks: "Greetings from TurboQuant-MLX"
// (turboquant_plus issue 59), item 2.
//
// Kernel shape: persistent CTAs of 256 threads; Pi^T (and the residual sketch
// matrix (S Pi^T)^T in prod mode) stay in shared memory for the CTA's life;
// each 64-vector tile is staged transposed in shared memory and multiplied
// with 4x8 register blocking in fp32 (the decision needs fp32-level rotation
// accuracy: a coordinate within ~1e-6 of a bound is the only place the code
// may differ from an fp64 reference).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "tq_internal.h"
#include "tq_layout.cuh"
#include "tq_sm100.cuh"

namespace tq {
namespace {

constexpr int kTile = 64;       // vectors per tile
constexpr int kThreads = 256;

struct QuantArgs {
  const void* x;
  int x_bf16;
  int64_t n;
  int mse_bits, mixed, prod, code_bytes;
  const float* pi;   // Pi [d][d] (y = Pi u)
  const float* pit;  // Pi^T [d][d]
  const float* mt;   // (S Pi^T)^T [d][m]
  const float* cb;   // [5][16]
  const float* bd;   // [5][16]
  // 8-bit codebook (mse_bits == 8): code-search cells, fp64 Pi^T
  const float2* cell8;
  int cell8_n;
  float cell8_inv_w;
  const double* pit64;
  // plain destination (row = vector index)
  uint8_t* codes;
  float* norms;
  uint8_t* qjl;
  float* res;
  // append destination (code planes tiled, tq_layout.cuh; kside: the keys' arrangement)
  int append;
  int kside;
  const int32_t* seq_ids;
  int32_t* lens;
  int n_tok, hkv, capacity, n_sink, cache_seqs;
  uint16_t* sink;  // bf16 [n_seq][hkv][n_sink][d]
  int32_t* status;  // device word; bit 4 = a pipeline wait timed out
  const uint8_t* tc_img;  // tensor-core B operand images (tq_params::tc_img)
  // A second plane (the tensor-core kernels, appends whose K and V formats
  // are equal): one launch quantizes the keys (plane 0, the fields above) and
  // the values (plane 1, these, in the values' arrangement); tiles
  // [0, tiles of n) are plane 0's, the next as many plane 1's.
  int planes;
  const void* x2;
  uint8_t* codes2;
  float* norms2;
  uint8_t* qjl2;
  float* res2;
  uint16_t* sink2;
  // Folded length update of an append: every CTA of the append's kernels
  // (arrive_total of them) counts itself in bits 16..31 of the cache's status
  // word once it has read lens for the last time; the last one adds n_tok to
  // the length of each of the n_seq_in appended sequences (or flags bit 1)
  // and returns the count to zero.  0 = no update in this launch.
  int arrive_total;
  int n_seq_in;
  // Launched with programmatic stream serialization (the tensor-core kernel
  // of an append): the CTAs may start while the previous kernel on the stream
  // still runs, and set up shared memory, barriers and tensor memory before
  // they wait for it; every global access comes after the wait.
  int overlapped;
  // Append input in head-major tiles (the MSE tensor-core kernel): tile =
  // 128 consecutive tokens (over the n_seq_in x n_tok chunk, token-major) of
  // one kv-head, so a warp's 32 rows go to consecutive rows of one cache unit
  // and its tiled stores land in a few tiles instead of eight units.
  int head_major;
};


// Lets the next kernel on the stream, when it is launched with programmatic
// stream serialization (the decode call's query rotation), start its own
// independent prologue; it waits for this grid before reading its outputs.
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Waits until the previous kernel on the stream has finished and its writes
// are visible (returns at once when this grid was launched without
// programmatic stream serialization).
__device__ __forceinline__ void wait_prerequisites() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

// The input and destinations of plane pl.
struct PlaneDst {
  const void* x;
  uint8_t* codes;
  float* norms;
  uint8_t* qjl;
  float* res;
  uint16_t* sink;
  int kside;
};
__device__ __forceinline__ PlaneDst plane_dst(const QuantArgs& a, int pl) {
  return pl ? PlaneDst{a.x2, a.codes2, a.norms2, a.qjl2, a.res2, a.sink2, 0}
            : PlaneDst{a.x, a.codes, a.norms, a.qjl, a.res, a.sink, a.kside};
}

// The end of an append kernel's CTA (every thread calls it, after the CTA's
// last read of lens): see QuantArgs::arrive_total.  A sequence whose append
// does not fit (or whose index or stored length is out of range) keeps its
// length, and bit 1 is set in the status word.
__device__ void append_arrive(const QuantArgs& a, int count = 1) {
  if (!a.append || a.arrive_total <= 0) return;
  __shared__ int s_last;
  // No fence: every read of lens in this CTA has been consumed (its rows
  // computed) before the barrier, nothing in this kernel reads the rows it
  // writes, and later kernels on the stream see all of it at its end.
  __syncthreads();
  if (threadIdx.x == 0) {
    const int old = atomicAdd(a.status, count << 16);
    s_last = ((old >> 16) & 0xFFFF) + count == a.arrive_total;
  }
  __syncthreads();
  if (!s_last) return;
  const int limit = a.n_sink + a.capacity;
  for (int i = threadIdx.x; i < a.n_seq_in; i += blockDim.x) {
    const int seq = a.seq_ids[i];
    const int len = (seq >= 0 && seq < a.cache_seqs) ? __ldcg(a.lens + seq) : -1;
    if (len < 0 || len + a.n_tok > limit)
      atomicOr(a.status, 1);
    else
      a.lens[seq] = len + a.n_tok;
  }
  __syncthreads();
  if (threadIdx.x == 0) atomicAnd(a.status, 0xFFFF);
}

struct SmemQuant {
  float pit[kDim][kDim];     // pit[k][j] = Pi[j][k]
  float xs[kDim][kTile];     // x transposed: xs[k][v]
  float nu[kTile];
  float inv_nu[kTile];
  uint8_t codes[kTile][kDim];
  int64_t row[kTile];        // destination row, -1 = none (tail or sink token)
};

struct SmemProd {
  float mt[kDim][kSketch];   // mt[j][i] = M[i][j], M = S Pi^T
  float rs[kDim][kTile];     // rotated-domain residual, transposed
};

// Destination row of vector v for an append: (seq, head, pos - n_sink);
// also copies sink tokens.  Returns -1 when there is nothing to quantize.
__device__ int64_t append_row(const QuantArgs& a, int64_t v, int* seq_out, int* head_out, int* pos_out) {
  const int head = static_cast<int>(v % a.hkv);
  const int64_t st = v / a.hkv;
  const int tok = static_cast<int>(st % a.n_tok);
  const int s_local = static_cast<int>(st / a.n_tok);
  const int seq = a.seq_ids[s_local];
  *seq_out = seq;
  *head_out = head;
  *pos_out = 0;
  if (seq < 0 || seq >= a.cache_seqs) return -1;          // rejected by the length update
  const int len = __ldcg(a.lens + seq);  // written by the previous append's last CTA
  *pos_out = len + tok;
  if (len < 0 || len + a.n_tok > a.n_sink + a.capacity) return -1;
  const int pos = len + tok;
  if (pos < a.n_sink) return -2;                           // sink token
  return (static_cast<int64_t>(seq) * a.hkv + head) * a.capacity + (pos - a.n_sink);
}

// n bytes of a packed row (32-bit words, nw of them) from row byte src to dst,
// in the widest stores the destination's alignment allows.
__device__ __forceinline__ void store_row_bytes(uint8_t* dst, const uint32_t* words, int nw, int src, int n) {
  while (n > 0) {
    const int w = src >> 2, sh = 8 * (src & 3);
    const uint32_t lo = words[w], hi = w + 1 < nw ? words[w + 1] : 0u;
    const uint32_t v = sh ? __funnelshift_r(lo, hi, sh) : lo;
    const uintptr_t ad = reinterpret_cast<uintptr_t>(dst);
    if (n >= 4 && (ad & 3) == 0) {
      *reinterpret_cast<uint32_t*>(dst) = v;
      dst += 4; src += 4; n -= 4;
    } else if (n >= 2 && (ad & 1) == 0) {
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(v);
      dst += 2; src += 2; n -= 2;
    } else {
      *dst = static_cast<uint8_t>(v);
      dst += 1; src += 1; n -= 1;
    }
  }
}

// Store the code words of a packed row as token (row & 15) of its 16-token
// tile in a tiled cache code plane (tq_layout.cuh).  row = unit * capacity +
// quantized position (capacity a multiple of 64, so tiles never straddle
// units).  Each piece is a contiguous run of the packed row and of its lane
// block; a run is split where the lane block changes column.
__device__ __forceinline__ void store_tiled_codes(uint8_t* plane, const CodeTile& ct, bool kside, int64_t row,
                                                  const uint32_t* words) {
  uint8_t* tile = plane + (row >> 4) * ct.tile_bytes();
  const int tok = static_cast<int>(row & 15), nw = ct.cb / 4;
  for (int s = 0; s < ct.nseg; ++s) {
    const int parts = kside ? 4 : 8;
    const int pb = kside ? ct.kpiece(s) : ct.vpiece(s);
    const int off = kside ? ct.koff(tok >> 3, s) : ct.voff((tok & 1) + 2 * (tok >> 3), s);
    for (int q = 0; q < parts; ++q) {
      const int L = kside ? 4 * (tok & 7) + q : 4 * q + ((tok & 7) >> 1);
      int src = ct.seg_byte(s) + q * pb, p = off, n = pb;
      while (n > 0) {
        // bytes of this column left from lane-block byte p
        const int c16 = 16 * ct.c16(), c8 = c16 + 8 * ct.c8();
        const int room = p < c16 ? 16 - (p & 15) : p < c8 ? 8 - ((p - c16) & 7) : 4 - ((p - c8) & 3);
        const int m = n < room ? n : room;
        store_row_bytes(tile + ct.tile_off(L, p), words, nw, src, m);
        src += m; p += m; n -= m;
      }
    }
  }
}

// The same store with the format known at compile time (the tensor-core
// kernels): every piece's row bytes, lane-block offset, column and alignment
// are constants, the row's words stay in registers, and each run is written
// with the widest stores its alignment allows (tiles are 16-byte aligned).
template <int MSE, int MIXED, int CB>
struct TiledStore {
  static constexpr CodeTile CT = make_code_tile(MSE, MIXED, CB);

  template <int SRC>
  static __device__ __forceinline__ uint32_t get4(const uint32_t* w) {
    constexpr int i = SRC / 4, sh = 8 * (SRC % 4);
    if constexpr (sh == 0)
      return w[i];
    else if constexpr (i + 1 < CB / 4)
      return __funnelshift_r(w[i], w[i + 1], sh);
    else
      return w[i] >> sh;
  }

  // N bytes from row byte SRC to byte LOFF of lane L's block
  template <int SRC, int N, int LOFF>
  static __device__ __forceinline__ void piece(uint8_t* tile, int L, const uint32_t* w) {
    if constexpr (N > 0) {
      constexpr int e16 = 16 * CT.c16(), e8 = e16 + 8 * CT.c8();
      constexpr int width = LOFF < e16 ? 16 : LOFF < e8 ? 8 : 4;
      constexpr int cstart = LOFF < e16 ? (LOFF / 16) * 16 : LOFF < e8 ? e16 : e8;
      constexpr int cbase = LOFF < e16 ? (LOFF / 16) * 512 : LOFF < e8 ? 512 * CT.c16() : 512 * CT.c16() + 256 * CT.c8();
      constexpr int inoff = LOFF - cstart, room = width - inoff, m0 = N < room ? N : room;
      constexpr int M = (width >= 8 && inoff % 8 == 0 && m0 >= 8) ? 8
                        : (inoff % 4 == 0 && m0 >= 4)               ? 4
                        : (inoff % 2 == 0 && m0 >= 2)               ? 2
                                                                    : 1;
      uint8_t* dst = tile + cbase + L * width + inoff;
      if constexpr (M == 8)
        *reinterpret_cast<uint2*>(dst) = make_uint2(get4<SRC>(w), get4<SRC + 4>(w));
      else if constexpr (M == 4)
        *reinterpret_cast<uint32_t*>(dst) = get4<SRC>(w);
      else if constexpr (M == 2)
        *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(get4<SRC>(w));
      else
        *dst = static_cast<uint8_t>(get4<SRC>(w));
      piece<SRC + M, N - M, LOFF + M>(tile, L, w);
    }
  }

  // keys: the pieces of token role ROLE (0: token g, 1: token g + 8), quarters Q.. of segment S..
  template <int ROLE, int S = 0, int Q = 0>
  static __device__ __forceinline__ void kpieces(uint8_t* tile, int g, const uint32_t* w) {
    if constexpr (S < CT.nseg) {
      if constexpr (Q < 4) {
        piece<CT.seg_byte(S) + Q * CT.kpiece(S), CT.kpiece(S), CT.koff(ROLE, S)>(tile, 4 * g + Q, w);
        kpieces<ROLE, S, Q + 1>(tile, g, w);
      } else {
        kpieces<ROLE, S + 1, 0>(tile, g, w);
      }
    }
  }
  // values: the pieces of member M (token 2t, 2t+1, 2t+8, 2t+9), eighths G.. of segment S..
  template <int M, int S = 0, int G = 0>
  static __device__ __forceinline__ void vpieces(uint8_t* tile, int t, const uint32_t* w) {
    if constexpr (S < CT.nseg) {
      if constexpr (G < 8) {
        piece<CT.seg_byte(S) + G * CT.vpiece(S), CT.vpiece(S), CT.voff(M, S)>(tile, 4 * G + t, w);
        vpieces<M, S, G + 1>(tile, t, w);
      } else {
        vpieces<M, S + 1, 0>(tile, t, w);
      }
    }
  }

  static __device__ __forceinline__ void row(uint8_t* plane, bool kside, int64_t r, const uint32_t* w) {
    uint8_t* tile = plane + (r >> 4) * CT.tile_bytes();
    const int tok = static_cast<int>(r & 15);
    if (kside) {
      if (tok < 8)
        kpieces<0>(tile, tok, w);
      else
        kpieces<1>(tile, tok - 8, w);
    } else {
      const int t = (tok & 7) >> 1;
      switch ((tok & 1) + 2 * (tok >> 3)) {
        case 0: vpieces<0>(tile, t, w); break;
        case 1: vpieces<1>(tile, t, w); break;
        case 2: vpieces<2>(tile, t, w); break;
        default: vpieces<3>(tile, t, w); break;
      }
    }
  }
};

template <int BF16>
__device__ void load_tile(const QuantArgs& a, SmemQuant& s, int64_t v0) {
  // 16-byte chunks; lanes walk vectors so the transposed shared stores of a
  // warp hit 32 consecutive banks.
  constexpr int kElems = BF16 ? 8 : 4;
  constexpr int kChunks = kDim / kElems;
  const int tid = threadIdx.x;
  for (int it = tid; it < kTile * kChunks; it += kThreads) {
    const int v = (it & 31) + 32 * ((it >> 5) & 1);
    const int chunk = it >> 6;
    const int64_t gv = v0 + v;
    float vals[kElems];
    if (gv < a.n) {
      const char* src = static_cast<const char*>(a.x) + (gv * kDim + chunk * kElems) * (BF16 ? 2 : 4);
      uint4 raw = *reinterpret_cast<const uint4*>(src);
      if (BF16) {
        const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
        for (int e = 0; e < kElems; ++e) vals[e] = __bfloat162float(h[e]);
      } else {
        const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
        for (int e = 0; e < kElems; ++e) vals[e] = f[e];
      }
    } else {
#pragma unroll
      for (int e = 0; e < kElems; ++e) vals[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < kElems; ++e) s.xs[chunk * kElems + e][v] = vals[e];
  }
}

__device__ __forceinline__ int quantize_coord(float u, const float* bd, int bits) {
  // number of bounds strictly below u (bounds ascending, unused slots +inf)
  int idx = 0;
  for (int step = (1 << bits) >> 1; step > 0; step >>= 1)
    if (bd[idx + step - 1] < u) idx += step;
  return idx;
}

// Bits [32w, 32w+32) of a packed row whose codes sit in smem (one byte each).
__device__ __forceinline__ uint32_t pack_word(const uint8_t* codes, int w, int mse_bits, int mixed) {
  uint32_t out = 0;
  const int lo = 32 * w, hi = lo + 32;
  // segment 0: coordinates [0, n0) at width b0 from bit 0; segment 1 after it
  const int b0 = mixed ? mse_bits + 1 : mse_bits;
  const int n0 = mixed ? kDim / 2 : kDim;
  const int seg1_bit = n0 * b0;
  for (int seg = 0; seg < (mixed ? 2 : 1); ++seg) {
    const int b = seg ? mse_bits : b0;
    const int base_bit = seg ? seg1_bit : 0;
    const int j0 = seg ? n0 : 0, j1 = seg ? kDim : n0;
    int first = j0 + max(0, (lo - base_bit) / b - 1);
    for (int j = first; j < j1; ++j) {
      const int bit = base_bit + (j - j0) * b;
      if (bit >= hi) break;
      if (bit + b <= lo) continue;
      const uint32_t c = codes[j];
      const int sh = bit - lo;
      out |= sh >= 0 ? (c << sh) : (c >> (-sh));
    }
  }
  return out;
}

template <int BF16>
__global__ void __launch_bounds__(kThreads, 1) quantize_kernel(QuantArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemQuant& s = *reinterpret_cast<SmemQuant*>(smem_raw);
  launch_dependents();
  SmemProd* sp = a.prod ? reinterpret_cast<SmemProd*>(smem_raw + sizeof(SmemQuant)) : nullptr;
  __shared__ float cb_s[kMaxBits + 1][kBookSlots];
  __shared__ float bd_s[kMaxBits + 1][kBookSlots];
  const int tid = threadIdx.x;

  for (int i = tid; i < kDim * kDim / 4; i += kThreads)
    reinterpret_cast<float4*>(&s.pit[0][0])[i] = reinterpret_cast<const float4*>(a.pit)[i];
  if (a.prod)
    for (int i = tid; i < kDim * kSketch / 4; i += kThreads)
      reinterpret_cast<float4*>(&sp->mt[0][0])[i] = reinterpret_cast<const float4*>(a.mt)[i];
  for (int i = tid; i < (kMaxBits + 1) * kBookSlots; i += kThreads) {
    cb_s[i / kBookSlots][i % kBookSlots] = a.cb[i];
    bd_s[i / kBookSlots][i % kBookSlots] = a.bd[i];
  }

  const int tv = tid >> 4;  // vectors 4tv .. 4tv+3
  const int tj = tid & 15;  // dims 8tj .. 8tj+7
  const int64_t n_tiles = (a.n + kTile - 1) / kTile;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t v0 = tile * kTile;
    __syncthreads();  // previous tile fully consumed
    load_tile<BF16>(a, s, v0);
    if (tid < kTile) {
      const int64_t gv = v0 + tid;
      int64_t row = -1;
      if (gv < a.n) {
        if (a.append) {
          int seq, head, pos;
          row = append_row(a, gv, &seq, &head, &pos);
          if (row == -2) {
            // sink token: keep the bf16 value (input converted) and skip
            uint16_t* dst = a.sink + ((static_cast<int64_t>(seq) * a.hkv + head) * a.n_sink + pos) * kDim;
            const char* src = static_cast<const char*>(a.x) + gv * kDim * (BF16 ? 2 : 4);
            for (int k = 0; k < kDim; ++k) {
              float f = BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(src)[k])
                             : reinterpret_cast<const float*>(src)[k];
              __nv_bfloat16 h = __float2bfloat16_rn(f);
              dst[k] = *reinterpret_cast<uint16_t*>(&h);
            }
            row = -1;
          }
        } else {
          row = gv;
        }
      }
      s.row[tid] = row;
    }
    __syncthreads();
    if (tid < kTile) {
      float ss = 0.f;
      for (int k = 0; k < kDim; ++k) ss = fmaf(s.xs[k][tid], s.xs[k][tid], ss);
      const float nu = sqrtf(ss);
      s.nu[tid] = nu;
      s.inv_nu[tid] = nu > 0.f ? 1.f / nu : 0.f;
    }

    // y = Pi x for 4 vectors x 8 dims per thread
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < kDim; ++k) {
      const float4 xv = *reinterpret_cast<const float4*>(&s.xs[k][4 * tv]);
      const float4 p0 = *reinterpret_cast<const float4*>(&s.pit[k][8 * tj]);
      const float4 p1 = *reinterpret_cast<const float4*>(&s.pit[k][8 * tj + 4]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
      const float pa[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(xa[i], pa[j], acc[i][j]);
    }
    __syncthreads();  // nu ready; xs no longer needed

    float g2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int v = 4 * tv + i;
      const float inv = s.inv_nu[v];
      const bool zero = !(s.nu[v] > 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int dim = 8 * tj + j;
        const int b = (a.mixed && dim < kDim / 2) ? a.mse_bits + 1 : a.mse_bits;
        const float u = acc[i][j] * inv;
        int idx = 0;
        float c = 0.f;
        if (b > 0 && !zero) {
          idx = quantize_coord(u, bd_s[b], b);
          c = cb_s[b][idx];
        }
        s.codes[v][dim] = static_cast<uint8_t>(idx);
        if (a.prod) {
          const float r = zero ? 0.f : u - c;
          sp->rs[dim][v] = r;
          g2[i] = fmaf(r, r, g2[i]);
        }
      }
    }
    __syncthreads();

    // pack codes and write norms
    const int words = a.code_bytes / 4;
    if (a.append) {
      // a cache's tiled code plane: one thread per row
      if (words > 0 && tid < kTile && s.row[tid] >= 0) {
        uint32_t rw[kMaxBits * 4];
        for (int w = 0; w < words; ++w) rw[w] = pack_word(s.codes[tid], w, a.mse_bits, a.mixed);
        store_tiled_codes(a.codes, make_code_tile(a.mse_bits, a.mixed, a.code_bytes), a.kside, s.row[tid], rw);
      }
    } else {
      for (int it = tid; it < kTile * words; it += kThreads) {
        const int v = it / words, w = it % words;
        const int64_t row = s.row[v];
        if (row < 0) continue;
        reinterpret_cast<uint32_t*>(a.codes + row * a.code_bytes)[w] =
            pack_word(s.codes[v], w, a.mse_bits, a.mixed);
      }
    }
    if (tid < kTile && s.row[tid] >= 0) a.norms[s.row[tid]] = s.nu[tid];

    if (a.prod) {
      // gamma = ||r||: reduce over the 16 threads sharing tv (lanes of one half-warp)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) g2[i] += __shfl_xor_sync(0xffffffffu, g2[i], off);
      // sketch t = M r for 4 vectors x 8 sketch rows
      float t[4][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) t[i][j] = 0.f;
#pragma unroll 4
      for (int k = 0; k < kDim; ++k) {
        const float4 rv = *reinterpret_cast<const float4*>(&sp->rs[k][4 * tv]);
        const float4 m0 = *reinterpret_cast<const float4*>(&sp->mt[k][8 * tj]);
        const float4 m1 = *reinterpret_cast<const float4*>(&sp->mt[k][8 * tj + 4]);
        const float ra[4] = {rv.x, rv.y, rv.z, rv.w};
        const float ma[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) t[i][j] = fmaf(ra[i], ma[j], t[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int v = 4 * tv + i;
        const int64_t row = s.row[v];
        if (row < 0) continue;
        const bool zero = !(s.nu[v] > 0.f);
        uint32_t byte = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) byte |= (t[i][j] >= 0.f ? 1u : 0u) << j;
        a.qjl[row * (kSketch / 8) + tj] = zero ? 0 : static_cast<uint8_t>(byte);
        if (tj == 0) a.res[row] = zero ? 0.f : sqrtf(g2[i]);
      }
    }
  }
  append_arrive(a);
}

// ---------------------------------------------------------------------------
// Tensor-core rotate + quantize + pack (bf16 input, MSE and mixed formats).
//
// y = Pi x for a tile of 128 vectors is one 128 x 128 x 128 product on the
// fifth-generation tensor cores: A = the bf16 tile (exact input), B = Pi split
// as Pi_hi + Pi_lo in bf16 (16 mantissa bits together; the rounding error of
// a rotated unit-vector coordinate stays near 1e-6, under the 1e-5 band in
// which a code may legitimately differ), both products accumulated in fp32 in
// tensor memory.  Warp roles in a persistent CTA (one per SM):
//   warp 8      TMA producer: tiles of x, 128 rows x 256 B, into a 4-deep ring
//               (two 64-column boxes, 128-byte swizzle);
//   warp 9      allocates 256 TMEM columns and issues the MMAs (one thread);
//   warps 0..7  two epilogue groups taking alternate tiles, each with its own
//               128-column accumulator: thread = one vector (TMEM lane); norm
//               from the staged bf16 row, 32-column TMEM loads, codes by a
//               branch-free search over the symmetric decision bounds, packing
//               in registers, 16- or 8-byte stores of the packed row.
// ---------------------------------------------------------------------------
constexpr int kTcRows = 128;                      // vectors per tile (MMA M)
constexpr int kTcStages = 4;                      // x tiles in flight
constexpr int kTcBox = kTcRows * 128;             // one 64-column box: 16 KB
constexpr int kTcTile = 2 * kTcBox;               // one 128 x 128 bf16 tile: 32 KB
constexpr int kTcThreads = 10 * 32;
constexpr int kTcSmem = 2 * kTcTile + kTcStages * kTcTile + 1024;  // Pi hi/lo, x ring, alignment slack
constexpr int kTcCols = 256;                      // TMEM columns: two 128-column accumulators
constexpr int kTcSmemWide = 3 * kTcTile + 3 * kTcTile + 1024;  // 8-bit: Pi a/b/c, three x stages

// Code of u for a width-W codebook whose decision bounds are symmetric about
// 0: pb[i] = the i-th positive bound (pb[0] = 0 is the middle one).  Equals the
// count of bounds strictly below u except on exact ties with a bound.
template <int W>
__device__ __forceinline__ uint32_t sym_code(float u, const float (&pb)[8]) {
  constexpr uint32_t H = 1u << (W - 1);
  const float a = fabsf(u);
  uint32_t j;
  if constexpr (W == 1) {
    j = 0;
  } else if constexpr (W == 2) {
    j = a > pb[1] ? 1u : 0u;
  } else if constexpr (W == 3) {
    const bool c1 = a > pb[2];
    const bool c0 = a > (c1 ? pb[3] : pb[1]);
    j = (c1 ? 2u : 0u) + (c0 ? 1u : 0u);
  } else {
    const bool c2 = a > pb[4];
    const bool c1 = a > (c2 ? pb[6] : pb[2]);
    const float t0 = c2 ? (c1 ? pb[7] : pb[5]) : (c1 ? pb[3] : pb[1]);
    const bool c0 = a > t0;
    j = (c2 ? 4u : 0u) + (c1 ? 2u : 0u) + (c0 ? 1u : 0u);
  }
  return u > 0.f ? H + j : H - 1u - j;
}

// 8-bit code of u from the cell table of the positive half (cells hold the
// count of positive bounds at or below their start and the one bound inside
// them): the count of bounds strictly below u, except on exact ties.
__device__ __forceinline__ uint32_t code8(float u, const float2* cells, int n_cells, float inv_w) {
  const float a = fabsf(u);
  const int c = min(static_cast<int>(a * inv_w), n_cells - 1);
  const float2 cell = cells[c];
  const uint32_t j = static_cast<uint32_t>(cell.x) + (a > cell.y ? 1u : 0u);
  return u > 0.f ? 128u + j : 127u - j;
}

// 32 codes of width W from one 32-column TMEM chunk, packed LSB-first into W words.
template <int W>
__device__ __forceinline__ void pack_chunk(const uint32_t (&y)[32], float inv_nu, const float (&pb)[8],
                                           uint32_t* out) {
#pragma unroll
  for (int w = 0; w < W; ++w) out[w] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t c = sym_code<W>(__uint_as_float(y[j]) * inv_nu, pb);
    const int bit = j * W, wi = bit >> 5, sh = bit & 31;
    out[wi] |= c << sh;
    if (sh + W > 32) out[wi + 1] |= c >> (32 - sh);
  }
}

template <int B, int MIXED>
struct TcFormat {
  static constexpr int b0 = MIXED ? B + 1 : B;     // width of columns 0..63
  static constexpr int b1 = B;                     // width of columns 64..127
  static constexpr int words = 2 * b0 + 2 * b1;    // packed row, 32-bit words
  static constexpr int bytes = 4 * words;
};

// Tiles of one plane, and the row of tile-local row r (-1: past the end).
__host__ __device__ __forceinline__ int64_t plane_tile_count(const QuantArgs& a) {
  if (a.head_major) {
    const int64_t nt = a.n / a.hkv;
    return ((nt + kTcRows - 1) / kTcRows) * a.hkv;
  }
  return (a.n + kTcRows - 1) / kTcRows;
}
template <bool HM>
__device__ __forceinline__ int64_t tile_row(const QuantArgs& a, int64_t lt, int r) {
  if constexpr (HM) {
    const int64_t ts = (lt / a.hkv) * kTcRows + r;  // token index over the chunk
    return ts < a.n / a.hkv ? ts * a.hkv + lt % a.hkv : -1;
  } else {
    const int64_t v = lt * kTcRows + r;
    return v < a.n ? v : -1;
  }
}

// HM: a.head_major (compiled apart so that the row-major path keeps its code).
template <int B, int MIXED, bool HM>
__global__ void __launch_bounds__(kTcThreads, 1) quantize_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                    const __grid_constant__ CUtensorMap xmap2,
                                                                    QuantArgs a) {
  using namespace sm100;
  using TF = TcFormat<B, MIXED>;
  launch_dependents();
  // 8-bit codes: Pi in three bf16 terms (the 255 bounds sit ~1.5e-3 apart,
  // so the rotation must be good to ~1e-8) and one fewer x stage to make room
  constexpr bool kWide = B == kWideBits;
  constexpr int NPI = kWide ? 3 : 2, NST = kWide ? 3 : kTcStages;
  extern __shared__ __align__(16) unsigned char smem_tc[];
  __shared__ __align__(8) uint64_t x_full[NST], x_empty[NST], t_full[2], t_empty[2], b_full;
  __shared__ float2 s_cell8[kWide ? kCell8Max : 1];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_pb[2][8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t raw = smem_u32(smem_tc);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t pih = base, pil = base + kTcTile, xs0 = base + NPI * kTcTile;

  // Pi (row j = output coordinate, K = input coordinate) as bf16 hi and lo
  // halves arrives by bulk copy from the prepared images
  if constexpr (kWide) {
    for (int i = tid; i < a.cell8_n; i += kTcThreads) s_cell8[i] = a.cell8[i];
  } else if (tid < 16) {
    const int seg = tid >> 3, i = tid & 7;
    const int w = seg ? TF::b1 : TF::b0;
    const int half = 1 << (w - 1);
    s_pb[seg][i] = i < half ? a.bd[w * kBookSlots + half - 1 + i] : 0.f;
  }
  if (warp == 9) {
    tmem_alloc(&s_tmem, kTcCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1 + 4);  // the MMA commit and the four epilogue warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&t_full[b], 1);
      mbar_init(&t_empty[b], 4);
    }
    mbar_init(&b_full, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // everything above touched only shared memory, tensor memory and the
  // parameter tables; the input, the cache and its lengths come after
  wait_prerequisites();
  const uint32_t tmem = s_tmem;
  const int64_t plane_tiles = HM ? ((a.n / a.hkv + kTcRows - 1) / kTcRows) * a.hkv : (a.n + kTcRows - 1) / kTcRows;
  const int64_t n_tiles = plane_tiles * a.planes;

  if (warp == 8) {
    // ---- producer: the B operand once, then the x tiles
    if (lane == 0) {
      prefetch_tensormap(&xmap);
      if (a.planes > 1) prefetch_tensormap(&xmap2);
      mbar_expect_tx(&b_full, NPI * kTcTile);
      if constexpr (kWide) {
#pragma unroll
        for (int t = 0; t < 3; ++t)
          bulk_g2s_addr(pih + t * kTcTile, a.tc_img + (kTcImgPiA + t) * kTcImgBytes, kTcTile, &b_full);
      } else {
        bulk_g2s_addr(pih, a.tc_img + kTcImgPiHi * kTcImgBytes, kTcTile, &b_full);
        bulk_g2s_addr(pil, a.tc_img + kTcImgPiLo * kTcImgBytes, kTcTile, &b_full);
      }
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
        const int s = i % NST;
        if (i >= NST && !mbar_wait(&x_empty[s], ((i / NST) - 1) & 1)) s_abort = 1;
        if (s_abort) break;
        mbar_expect_tx(&x_full[s], kTcTile);
        const int pl = tile >= plane_tiles;
        const CUtensorMap* map = pl ? &xmap2 : &xmap;
        const int64_t lt = tile - pl * plane_tiles;
        if constexpr (HM) {
          const int head = static_cast<int>(lt % a.hkv), t0 = static_cast<int>((lt / a.hkv) * kTcRows);
          tma_load_3d(xs0 + s * kTcTile, map, 0, head, t0, &x_full[s]);
          tma_load_3d(xs0 + s * kTcTile + kTcBox, map, 64, head, t0, &x_full[s]);
        } else {
          const int row0 = static_cast<int>(lt * kTcRows);
          tma_load_2d(xs0 + s * kTcTile, map, 0, row0, &x_full[s]);
          tma_load_2d(xs0 + s * kTcTile + kTcBox, map, 64, row0, &x_full[s]);
        }
      }
      // loads still in flight land before the CTA may exit
      for (int k = i - NST; k < i; ++k)
        if (k >= 0) mbar_wait(&x_full[k % NST], (k / NST) & 1);
      mbar_wait(&b_full, 0);
    }
  } else if (warp == 9) {
    // ---- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTcRows, kDim);
      if (!mbar_wait(&b_full, 0)) s_abort = 1;
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
        const int s = i % NST, buf = i & 1;
        if (!mbar_wait(&x_full[s], (i / NST) & 1)) s_abort = 1;
        if (i >= 2 && !s_abort && !mbar_wait(&t_empty[buf], ((i >> 1) - 1) & 1)) s_abort = 1;
        if (s_abort) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kDim;
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t off = (k >> 2) * kTcBox + (k & 3) * 32;
          const uint64_t ad = sw128_kmajor_desc(xs0 + s * kTcTile + off);
          umma_bf16(d, ad, sw128_kmajor_desc(pih + off), idesc, k > 0);
          umma_bf16(d, ad, sw128_kmajor_desc(pil + off), idesc, true);
          if constexpr (kWide) umma_bf16(d, ad, sw128_kmajor_desc(pih + 2 * kTcTile + off), idesc, true);
        }
        umma_commit(&x_empty[s]);
        umma_commit(&t_full[buf]);
      }
    }
  } else {
    // ---- epilogue: group g takes tiles i = g (mod 2); thread = TMEM lane = row
    const int g = warp >> 2, q = warp & 3, r = 32 * q + lane;
    float pb0[8], pb1[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      pb0[k] = s_pb[0][k];
      pb1[k] = s_pb[1][k];
    }
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
      if ((i & 1) != g) continue;
      if (s_abort) break;
      const int s = i % NST, buf = i & 1;
      // norm of the row from the staged bf16 tile
      if (!mbar_wait(&x_full[s], (i / NST) & 1)) {
        s_abort = 1;
        break;
      }
      float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int bx = 0; bx < 2; ++bx)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = xs0 + s * kTcTile + bx * kTcBox + r * 128 + ((c ^ (r & 7)) << 4);
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(addr));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
            ss2 = __ffma2_rn(f, f, ss2);
          }
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_empty[s]);
      const float nu = sqrtf(ss2.x + ss2.y);
      const float inv = nu > 0.f ? 1.f / nu : 0.f;
      if (!mbar_wait(&t_full[buf], (i >> 1) & 1)) {
        s_abort = 1;
        break;
      }
      tc_fence_after();
      uint32_t words[TF::words];
      const uint32_t tbase = tmem + buf * kDim + (static_cast<uint32_t>(32 * q) << 16);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t y[32];
        tmem_ld32(tbase + 32 * c, y);
        tmem_wait_ld();
        if constexpr (kWide) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            uint32_t wd = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              wd |= code8(__uint_as_float(y[4 * jj + e]) * inv, s_cell8, a.cell8_n, a.cell8_inv_w) << (8 * e);
            words[8 * c + jj] = wd;
          }
        } else if (c < 2) {
          pack_chunk<TF::b0>(y, inv, pb0, words + c * TF::b0);
        } else {
          pack_chunk<TF::b1>(y, inv, pb1, words + 2 * TF::b0 + (c - 2) * TF::b1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[buf]);
      // outputs
      const int pl = tile >= plane_tiles;
      const PlaneDst pd = plane_dst(a, pl);
      const int64_t v = tile_row<HM>(a, tile - pl * plane_tiles, r);
      if (v >= 0) {
        int64_t row = v;
        if (a.append) {
          int seq, head, pos;
          row = append_row(a, v, &seq, &head, &pos);
          if (row == -2) {
            uint16_t* dst = pd.sink + ((static_cast<int64_t>(seq) * a.hkv + head) * a.n_sink + pos) * kDim;
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(pd.x) + v * kDim);
#pragma unroll
            for (int k = 0; k < kDim / 8; ++k) reinterpret_cast<uint4*>(dst)[k] = src[k];
          }
        }
        if (row >= 0) {
          if (!(nu > 0.f)) {
#pragma unroll
            for (int w = 0; w < TF::words; ++w) words[w] = 0u;
          }
          if (a.append) {
            TiledStore<B, MIXED, TF::bytes>::row(pd.codes, pd.kside, row, words);
          } else {
            uint8_t* dst = pd.codes + row * TF::bytes;
            if constexpr (TF::bytes % 16 == 0) {
#pragma unroll
              for (int w = 0; w < TF::words; w += 4)
                *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
            } else {
#pragma unroll
              for (int w = 0; w < TF::words; w += 2)
                *reinterpret_cast<uint2*>(dst + 4 * w) = make_uint2(words[w], words[w + 1]);
            }
          }
          pd.norms[row] = nu;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcCols);
  }
  if (tid == 0 && s_abort && a.status) atomicOr(a.status, 4);
  append_arrive(a);
}

// ---------------------------------------------------------------------------
// Tensor-core quantize for prod formats (bf16 input): total bits = MB + 1,
// an MB-bit MSE stage and the 1-bit QJL sketch of the residual.
//
// A sketch sign may differ from the exact one only where |(S r)_i| < 1e-5,
// and a rotation error in the unit vector reaches (S r)_i amplified by the
// norm of a row of S (about sqrt(m)), so both products run at about 24
// significant bits:
//   D1 = X (Pi_a + Pi_b + Pi_c)^T      rotation; x is exact in bf16, Pi is
//                                       split into three bf16 terms
//   D2 = 2^10 rho (M_hi + M_lo)^T      sketch, M = S Pi^T; rho = y / nu - c[idx]
//                                       the rotated-domain residual, split
//                                       into two fp16 terms (rho_lo M_lo dropped)
// S r = S Pi^T rho because r = Pi^T rho, and only the sign of D2 is kept, so
// the power-of-two scale on rho never needs undoing.  The epilogue writes the
// rho halves into the TMEM columns of D1 it has just read, and the sketch
// MMAs take their A operand from there.  Shared memory: Pi (96 KB), M (64 KB)
// and one x tile per epilogue group (64 KB).
// ---------------------------------------------------------------------------
constexpr int kTpSmem = 3 * kTcTile + 2 * kTcTile + 2 * kTcTile + 1024;  // Pi a/b/c, M hi/lo, x x2, slack
constexpr int kTpCols = 512;                                                // per group: D1 (128) | D2 (128)
constexpr float kRhoScale = 1024.f;

// Code and centroid of u for a width-W codebook symmetric about 0: pb = the
// positive bounds (pb[0] = 0), pc = the positive centroids, ascending.
template <int W>
__device__ __forceinline__ uint32_t sym_code_c(float u, const float (&pb)[8], const float (&pc)[8], float& c) {
  constexpr uint32_t H = 1u << (W - 1);
  const float a = fabsf(u);
  uint32_t j;
  float m;
  if constexpr (W == 1) {
    j = 0;
    m = pc[0];
  } else if constexpr (W == 2) {
    const bool c0 = a > pb[1];
    j = c0 ? 1u : 0u;
    m = c0 ? pc[1] : pc[0];
  } else {
    static_assert(W == 3, "prod MSE stages use 1..3 bits");
    const bool c1 = a > pb[2];
    const bool c0 = a > (c1 ? pb[3] : pb[1]);
    j = (c1 ? 2u : 0u) + (c0 ? 1u : 0u);
    m = c1 ? (c0 ? pc[3] : pc[2]) : (c0 ? pc[1] : pc[0]);
  }
  const bool pos = u > 0.f;
  c = pos ? m : -m;
  return pos ? H + j : H - 1u - j;
}

__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int MB>
__global__ void __launch_bounds__(kTcThreads, 1) quantize_tc_prod_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                         const __grid_constant__ CUtensorMap xmap2,
                                                                         QuantArgs a) {
  using namespace sm100;
  constexpr int CW = MB > 0 ? 4 * MB : 1;  // packed MSE words per row (unused for MB = 0)
  launch_dependents();
  extern __shared__ __align__(16) unsigned char smem_tp[];
  __shared__ __align__(8) uint64_t x_full[2], x_empty[2], t1_full[2], rho_full[2], t2_full[2], t_empty[2], b_full;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ float s_pb[8], s_pc[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t raw = smem_u32(smem_tp);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t pia = base, mh = base + 3 * kTcTile, xs0 = base + 5 * kTcTile;

  // B operands by bulk copy from the prepared images: Pi (row j, K = input
  // coordinate) in three bf16 terms, M = S Pi^T (row i = sketch index, K =
  // rotated coordinate) in two fp16 terms
  if constexpr (MB > 0) {
    if (tid < 8) {
      constexpr int half = 1 << (MB - 1);
      s_pb[tid] = tid < half ? a.bd[MB * kBookSlots + half - 1 + tid] : 0.f;
      s_pc[tid] = tid < half ? a.cb[MB * kBookSlots + half + tid] : 0.f;
    }
  }
  if (warp == 9) {
    tmem_alloc(&s_tmem, kTpCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&x_full[b], 1);
      mbar_init(&x_empty[b], 1 + 4);  // the rotation MMAs' commit and the four warps reading the norm
      mbar_init(&t1_full[b], 1);
      mbar_init(&rho_full[b], 4);
      mbar_init(&t2_full[b], 1);
      mbar_init(&t_empty[b], 4);
    }
    mbar_init(&b_full, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int64_t plane_tiles = (a.n + kTcRows - 1) / kTcRows;
  const int64_t n_tiles = plane_tiles * a.planes;

  if (warp == 8) {
    // ---- producer: the B operands once, then tile i into the x stage of its
    // epilogue group (i & 1)
    if (lane == 0) {
      prefetch_tensormap(&xmap);
      if (a.planes > 1) prefetch_tensormap(&xmap2);
      mbar_expect_tx(&b_full, 5 * kTcTile);
      for (int k = 0; k < 3; ++k)
        bulk_g2s_addr(pia + k * kTcTile, a.tc_img + (kTcImgPiA + k) * kTcImgBytes, kTcTile, &b_full);
      for (int k = 0; k < 2; ++k)
        bulk_g2s_addr(mh + k * kTcTile, a.tc_img + (kTcImgMHi + k) * kTcImgBytes, kTcTile, &b_full);
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
        const int s = i & 1;
        if (i >= 2 && !mbar_wait(&x_empty[s], ((i >> 1) - 1) & 1)) s_abort = 1;
        if (s_abort) break;
        mbar_expect_tx(&x_full[s], kTcTile);
        const int pl = tile >= plane_tiles;
        const CUtensorMap* map = pl ? &xmap2 : &xmap;
        const int row0 = static_cast<int>((tile - pl * plane_tiles) * kTcRows);
        tma_load_2d(xs0 + s * kTcTile, map, 0, row0, &x_full[s]);
        tma_load_2d(xs0 + s * kTcTile + kTcBox, map, 64, row0, &x_full[s]);
      }
      for (int k = i - 2; k < i; ++k)  // loads still in flight land before the CTA may exit
        if (k >= 0) mbar_wait(&x_full[k & 1], (k >> 1) & 1);
      mbar_wait(&b_full, 0);
    }
  } else if (warp == 9) {
    // ---- MMA issue: rotation of tile i, then the sketch of tile i - 1
    if (lane == 0) {
      constexpr uint32_t id_rot = idesc_bf16_f32(kTcRows, kDim);
      constexpr uint32_t id_sk = idesc_f16_f32(kTcRows, kSketch);
      if (!mbar_wait(&b_full, 0)) s_abort = 1;
      auto sketch = [&](int j) {  // D2 of local tile j, A = the residual halves in D1's columns
        const int b = j & 1;
        if (!mbar_wait(&rho_full[b], (j >> 1) & 1)) {
          s_abort = 1;
          return;
        }
        tc_fence_after();
        const uint32_t acc = tmem + b * 256;
        const uint32_t d = acc + 128;
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t off = (k >> 2) * kTcBox + (k & 3) * 32;
          const uint32_t ahi = acc + 32 * (k >> 1) + 8 * (k & 1), alo = ahi + 16;
          const uint64_t bh = sw128_kmajor_desc(mh + off);
          umma_f16_ts(d, ahi, bh, id_sk, k > 0);
          umma_f16_ts(d, ahi, sw128_kmajor_desc(mh + kTcTile + off), id_sk, true);
          umma_f16_ts(d, alo, bh, id_sk, true);
        }
        umma_commit(&t2_full[b]);
      };
      int i = 0;
      for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
        const int b = i & 1;
        if (!mbar_wait(&x_full[b], (i >> 1) & 1)) s_abort = 1;
        if (i >= 2 && !s_abort && !mbar_wait(&t_empty[b], ((i >> 1) - 1) & 1)) s_abort = 1;
        if (s_abort) break;
        tc_fence_after();
        const uint32_t d = tmem + b * 256;
#pragma unroll
        for (int k = 0; k < kDim / 16; ++k) {
          const uint32_t off = (k >> 2) * kTcBox + (k & 3) * 32;
          const uint64_t ad = sw128_kmajor_desc(xs0 + b * kTcTile + off);
          umma_bf16(d, ad, sw128_kmajor_desc(pia + off), id_rot, k > 0);
          umma_bf16(d, ad, sw128_kmajor_desc(pia + kTcTile + off), id_rot, true);
          umma_bf16(d, ad, sw128_kmajor_desc(pia + 2 * kTcTile + off), id_rot, true);
        }
        umma_commit(&x_empty[b]);
        umma_commit(&t1_full[b]);
        if (i >= 1) sketch(i - 1);
        if (s_abort) break;
      }
      if (i >= 1 && !s_abort) sketch(i - 1);
    }
  } else {
    // ---- epilogue: group g takes tiles i = g (mod 2); thread = TMEM lane = row
    const int g = warp >> 2, q = warp & 3, r = 32 * q + lane;
    float pb[8], pc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      pb[k] = s_pb[k];
      pc[k] = s_pc[k];
    }
    const uint32_t lanes = static_cast<uint32_t>(32 * q) << 16;
    int i = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
      if ((i & 1) != g) continue;
      if (s_abort) break;
      const int ph = (i >> 1) & 1;
      const uint32_t xs = xs0 + g * kTcTile;
      if (!mbar_wait(&x_full[g], ph)) {
        s_abort = 1;
        break;
      }
      float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int bx = 0; bx < 2; ++bx)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = xs + bx * kTcBox + r * 128 + ((c ^ (r & 7)) << 4);
          uint4 v;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(addr));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = make_float2(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
            ss2 = __ffma2_rn(f, f, ss2);
          }
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(&x_empty[g]);
      const float nu = sqrtf(ss2.x + ss2.y);
      const float inv = nu > 0.f ? 1.f / nu : 0.f;
      if (!mbar_wait(&t1_full[g], ph)) {
        s_abort = 1;
        break;
      }
      tc_fence_after();
      uint32_t words[CW];
      float g2 = 0.f;
      const uint32_t acc = tmem + g * 256 + lanes;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t y[32];
        tmem_ld32(acc + 32 * c, y);
        tmem_wait_ld();
        if constexpr (MB > 0) {
#pragma unroll
          for (int w = 0; w < MB; ++w) words[c * MB + w] = 0u;
        }
        // residual of columns 32c..32c+31, scaled, as fp16 hi / lo pairs:
        // hi in columns 32c..32c+15, lo in 32c+16..32c+31 (over the D1
        // values just read)
        uint32_t o[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float rr[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int j = 2 * e + h;
            const float u = __uint_as_float(y[j]) * inv;
            if constexpr (MB > 0) {
              float cv;
              const uint32_t code = sym_code_c<MB>(u, pb, pc, cv);
              const int bit = j * MB, wi = bit >> 5, sh = bit & 31;
              words[c * MB + wi] |= code << sh;
              if (sh + MB > 32) words[c * MB + wi + 1] |= code >> (32 - sh);
              rr[h] = u - cv;
            } else {
              rr[h] = u;
            }
            g2 = fmaf(rr[h], rr[h], g2);
          }
          const float s0 = rr[0] * kRhoScale, s1 = rr[1] * kRhoScale;
          const uint32_t hi = f16x2_bits(s0, s1);
          const __half2 hh = *reinterpret_cast<const __half2*>(&hi);
          o[e] = hi;
          o[16 + e] = f16x2_bits(s0 - __low2float(hh), s1 - __high2float(hh));
        }
        tmem_st32(acc + 32 * c, o);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&rho_full[g]);
      if (!mbar_wait(&t2_full[g], ph)) {
        s_abort = 1;
        break;
      }
      tc_fence_after();
      uint32_t z[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t y[32];
        tmem_ld32(acc + 128 + 32 * c, y);
        tmem_wait_ld();
        uint32_t bits = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) bits |= (__uint_as_float(y[j]) >= 0.f ? 1u : 0u) << j;
        z[c] = bits;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&t_empty[g]);
      // outputs
      const int pl = tile >= plane_tiles;
      const PlaneDst pd = plane_dst(a, pl);
      const int64_t v = (tile - pl * plane_tiles) * kTcRows + r;
      if (v < a.n) {
        int64_t row = v;
        if (a.append) {
          int seq, head, pos;
          row = append_row(a, v, &seq, &head, &pos);
          if (row == -2) {
            uint16_t* dst = pd.sink + ((static_cast<int64_t>(seq) * a.hkv + head) * a.n_sink + pos) * kDim;
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(pd.x) + v * kDim);
#pragma unroll
            for (int k = 0; k < kDim / 8; ++k) reinterpret_cast<uint4*>(dst)[k] = src[k];
          }
        }
        if (row >= 0) {
          const bool zero = !(nu > 0.f);
          if constexpr (MB > 0) {
            if (zero) {
#pragma unroll
              for (int w = 0; w < CW; ++w) words[w] = 0u;
            }
            if (a.append) {
              TiledStore<MB, 0, 16 * MB>::row(pd.codes, pd.kside, row, words);
            } else {
              uint8_t* dst = pd.codes + row * (16 * MB);
#pragma unroll
              for (int w = 0; w < CW; w += 4)
                *reinterpret_cast<uint4*>(dst + 4 * w) = make_uint4(words[w], words[w + 1], words[w + 2], words[w + 3]);
            }
          }
          pd.norms[row] = nu;
          *reinterpret_cast<uint4*>(pd.qjl + row * (kSketch / 8)) =
              zero ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(z[0], z[1], z[2], z[3]);
          pd.res[row] = zero ? 0.f : sqrtf(g2);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTpCols);
  }
  if (tid == 0 && s_abort && a.status) atomicOr(a.status, 4);
  append_arrive(a);
}

// 8-bit codes for rows the tensor-core kernel does not take (fp32 input):
// one block per vector, thread j = rotated coordinate j.  The rotation runs
// in fp64 from Pi^T in fp64: the 255 bounds of the 8-bit codebook sit
// ~1.5e-3 apart near 0, where an fp32 rotation error of ~1e-7 would move more
// codes across a bound than the parity contract allows.
__global__ void __launch_bounds__(kDim) quantize8_kernel(QuantArgs a) {
  __shared__ double xs[kDim];
  __shared__ double red[kDim / 32];
  launch_dependents();
  __shared__ __align__(16) uint32_t words[kDim / 4];
  __shared__ float2 s_cell8[kCell8Max];
  __shared__ long long s_row;
  __shared__ int s_seq, s_head, s_pos;
  const int j = threadIdx.x, lane = j & 31, warp = j >> 5;
  for (int i = j; i < a.cell8_n; i += kDim) s_cell8[i] = a.cell8[i];
  for (int64_t v = blockIdx.x; v < a.n; v += gridDim.x) {
    const double xj = a.x_bf16 ? static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(a.x)[v * kDim + j]))
                               : static_cast<double>(static_cast<const float*>(a.x)[v * kDim + j]);
    if (j == 0) {
      int seq = 0, head = 0, pos = 0;
      s_row = a.append ? append_row(a, v, &seq, &head, &pos) : v;
      s_seq = seq;
      s_head = head;
      s_pos = pos;
    }
    xs[j] = xj;
    double sq = xj * xj;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) red[warp] = sq;
    __syncthreads();
    const int64_t row = s_row;
    if (row == -2) {  // a sink token: kept in bf16
      a.sink[((static_cast<int64_t>(s_seq) * a.hkv + s_head) * a.n_sink + s_pos) * kDim + j] =
          __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<float>(xj)));
    } else if (row >= 0) {
      const double nu = sqrt(red[0] + red[1] + red[2] + red[3]);
      double y = 0.0;
#pragma unroll 8
      for (int k = 0; k < kDim; ++k) y = fma(a.pit64[k * kDim + j], xs[k], y);
      const uint32_t code =
          nu > 0.0 ? code8(static_cast<float>(y / nu), s_cell8, a.cell8_n, a.cell8_inv_w) : 0u;
      // four codes per word, lane-wise
      const uint32_t part = code << (8 * (j & 3));
      const uint32_t w4 = part | __shfl_xor_sync(0xffffffffu, part, 1);
      const uint32_t w = w4 | __shfl_xor_sync(0xffffffffu, w4, 2);
      if ((j & 3) == 0) words[j >> 2] = w;
      __syncthreads();
      if (a.append) {
        if (j == 0) store_tiled_codes(a.codes, make_code_tile(kWideBits, 0, 16 * kWideBits), a.kside, row, words);
      } else if (j < kDim / 4) {
        reinterpret_cast<uint32_t*>(a.codes + row * (16 * kWideBits))[j] = words[j];
      }
      if (j == 0) a.norms[row] = static_cast<float>(nu);
    }
    __syncthreads();
  }
  append_arrive(a);
}

// Arrivals on behalf of `count` CTAs of an append kernel that could not be
// launched, so that the length update still happens once and the count
// returns to zero.
__global__ void append_arrive_kernel(QuantArgs a, int count) { append_arrive(a, count); }

// Row import / export between packed rows (tq_quantize's format) and the
// quantized rows of one cache unit: codes converted to / from the tiled code
// plane, norms, QJL rows and residual norms copied.  One thread per row.
__global__ void cache_rows_kernel(int to_cache, CodeTile ct, int kside, uint8_t* codes, float* norms, uint8_t* qjl,
                                  float* res, int64_t unit_row0, uint8_t* r_codes, float* r_norms, uint8_t* r_qjl,
                                  float* r_res, int64_t n) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t row = unit_row0 + i;
  if (ct.nseg > 0) {
    uint8_t* tile = codes + (row >> 4) * ct.tile_bytes();
    uint8_t* prow = r_codes + i * ct.cb;
    if (to_cache) {
      uint32_t w[kMaxBits * 4];
      for (int k = 0; k < ct.cb / 4; ++k) w[k] = reinterpret_cast<const uint32_t*>(prow)[k];
      store_tiled_codes(codes, ct, kside, row, w);
    } else {
      for_each_tile_byte(ct, kside, static_cast<int>(row & 15), [&](int src, int dst) { prow[src] = tile[dst]; });
    }
  }
  if (to_cache) {
    norms[row] = r_norms[i];
    if (qjl) {
      for (int k = 0; k < kSketch / 8; ++k) qjl[row * (kSketch / 8) + k] = r_qjl[i * (kSketch / 8) + k];
      res[row] = r_res[i];
    }
  } else {
    r_norms[i] = norms[row];
    if (qjl) {
      for (int k = 0; k < kSketch / 8; ++k) r_qjl[i * (kSketch / 8) + k] = qjl[row * (kSketch / 8) + k];
      r_res[i] = res[row];
    }
  }
}

// x_hat = nu (Pi^T c + sqrt(pi/2)/m gamma S^T z), fp64 accumulation.
constexpr int kDeqVecs = 8;
__global__ void __launch_bounds__(kDim) dequantize_kernel(
    const uint8_t* codes, const float* norms, const uint8_t* qjl, const float* res, int64_t n,
    int mse_bits, int mixed, int prod, int code_bytes, const double* pi64, const double* s64,
    const double* cb64, const double* cb8_64, float* out) {
  __shared__ double chat[kDeqVecs][kDim];
  __shared__ double zs[kDeqVecs][kSketch];
  const int i = threadIdx.x;
  const int64_t v0 = static_cast<int64_t>(blockIdx.x) * kDeqVecs;
  for (int v = 0; v < kDeqVecs; ++v) {
    const int64_t gv = v0 + v;
    double c = 0.0, z = 0.0;
    if (gv < n) {
      const int b = (mixed && i < kDim / 2) ? mse_bits + 1 : mse_bits;
      if (b > 0) {
        const int bit = (mixed && i >= kDim / 2) ? (kDim / 2) * (mse_bits + 1) + (i - kDim / 2) * b : i * b;
        const uint8_t* row = codes + gv * code_bytes;
        uint32_t w = row[bit >> 3];
        if ((bit & 7) + b > 8) w |= static_cast<uint32_t>(row[(bit >> 3) + 1]) << 8;
        const int idx = (w >> (bit & 7)) & ((1u << b) - 1);
        c = b == kWideBits ? cb8_64[idx] : cb64[b * kBookSlots + idx];
      }
      if (prod) z = ((qjl[gv * (kSketch / 8) + (i >> 3)] >> (i & 7)) & 1) ? 1.0 : -1.0;
    }
    chat[v][i] = c;
    zs[v][i] = z;
  }
  __syncthreads();
  double acc[kDeqVecs], accz[kDeqVecs];
  for (int v = 0; v < kDeqVecs; ++v) acc[v] = accz[v] = 0.0;
  for (int j = 0; j < kDim; ++j) {
    const double pji = pi64[j * kDim + i];
    for (int v = 0; v < kDeqVecs; ++v) acc[v] = fma(pji, chat[v][j], acc[v]);
  }
  if (prod)
    for (int l = 0; l < kSketch; ++l) {
      const double sli = s64[l * kDim + i];
      for (int v = 0; v < kDeqVecs; ++v) accz[v] = fma(sli, zs[v][l], accz[v]);
    }
  const double kappa = 1.2533141373155002512078826424055 / kSketch;  // sqrt(pi/2)/m
  for (int v = 0; v < kDeqVecs; ++v) {
    const int64_t gv = v0 + v;
    if (gv >= n) break;
    double xh = acc[v];
    if (prod) xh += kappa * static_cast<double>(res[gv]) * accz[v];
    out[gv * kDim + i] = static_cast<float>(static_cast<double>(norms[gv]) * xh);
  }
}

int g_num_sms = 0;

int num_sms() {
  if (!g_num_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

size_t quant_smem(int prod) { return sizeof(SmemQuant) + (prod ? sizeof(SmemProd) : 0); }

// cuTensorMapEncodeTiled from the driver, looked up once (no link-time
// dependency on libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

template <int MB>
tq_status launch_tc_prod(const QuantArgs& a, const CUtensorMap* maps, int grid, cudaStream_t st) {
  cudaError_t e =
      ensure_dyn_smem<quantize_tc_prod_kernel<MB>>(kTpSmem);
  if (e == cudaSuccess) {
    quantize_tc_prod_kernel<MB><<<grid, kTcThreads, kTpSmem, st>>>(maps[0], maps[1], a);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tensor-core prod quantize kernel launch");
}

template <int B, int MIXED, bool HM>
tq_status launch_tc_hm(const QuantArgs& a, const CUtensorMap* maps, int grid, cudaStream_t st) {
  constexpr int smem = B == kWideBits ? kTcSmemWide : kTcSmem;
  cudaError_t e = ensure_dyn_smem<quantize_tc_kernel<B, MIXED, HM>>(smem);
  if (e == cudaSuccess && a.overlapped) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, quantize_tc_kernel<B, MIXED, HM>, maps[0], maps[1], a);
  } else if (e == cudaSuccess) {
    quantize_tc_kernel<B, MIXED, HM><<<grid, kTcThreads, smem, st>>>(maps[0], maps[1], a);
    e = cudaGetLastError();
  }
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tensor-core quantize kernel launch");
}
template <int B, int MIXED>
tq_status launch_tc(const QuantArgs& a, const CUtensorMap* maps, int grid, cudaStream_t st) {
  return a.head_major ? launch_tc_hm<B, MIXED, true>(a, maps, grid, st) : launch_tc_hm<B, MIXED, false>(a, maps, grid, st);
}

bool tc_format(const QuantArgs& a) {
  return a.prod ? (!a.mixed && a.mse_bits >= 0 && a.mse_bits <= 3)
                : (a.mse_bits >= 1 && (a.mixed ? (a.mse_bits == 2 || a.mse_bits == 3)
                                               : (a.mse_bits <= 4 || a.mse_bits == kWideBits)));
}

// bf16 rows: tensor-core rotation (MSE 1..4 and 8 bits, mixed 2.5 and 3.5, prod 1..4).
bool tc_eligible(const QuantArgs& a) {
  return a.x_bf16 && tc_format(a) && a.n <= (int64_t(1) << 31) &&
         (reinterpret_cast<uintptr_t>(a.x) & 15) == 0 &&
         (a.planes < 2 || (reinterpret_cast<uintptr_t>(a.x2) & 15) == 0) && encode_tiled() != nullptr;
}

// The grid run_quantize launches for a (the CTAs an append's length update
// counts).
int64_t quantize_grid(const QuantArgs& a) {
  if (a.n <= 0) return 0;
  if (tc_eligible(a)) return std::min<int64_t>(plane_tile_count(a) * a.planes, num_sms());
  if (a.mse_bits == kWideBits) return std::min<int64_t>(a.n, 64LL * num_sms());
  return std::min<int64_t>((a.n + kTile - 1) / kTile, num_sms());
}

bool encode_rows(CUtensorMap* map, const void* x, int64_t n) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDim) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kTcRows)};
  const cuuint32_t estr[2] = {1, 1};
  return encode_tiled()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same rows as [tokens][heads][d]: a box of 128 tokens of one head.
bool encode_heads(CUtensorMap* map, const void* x, int64_t n, int hkv) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kDim), static_cast<cuuint64_t>(hkv),
                              static_cast<cuuint64_t>(n / hkv)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kDim) * 2, static_cast<cuuint64_t>(kDim) * 2 * hkv};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kTcRows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_tiled()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(x), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

tq_status run_quantize_tc(const QuantArgs& a, cudaStream_t st) {
  CUtensorMap maps[2];
  auto encode = [&](CUtensorMap* m, const void* x) {
    return a.head_major ? encode_heads(m, x, a.n, a.hkv) : encode_rows(m, x, a.n);
  };
  if (!encode(&maps[0], a.x)) return fail(TQ_ERR_CUDA, "tq_quantize: cuTensorMapEncodeTiled failed");
  if (a.planes > 1) {
    if (!encode(&maps[1], a.x2)) return fail(TQ_ERR_CUDA, "tq_append: cuTensorMapEncodeTiled failed");
  } else {
    maps[1] = maps[0];
  }
  const int grid = static_cast<int>(quantize_grid(a));
  if (a.prod) {
    switch (a.mse_bits) {
      case 0: return launch_tc_prod<0>(a, maps, grid, st);
      case 1: return launch_tc_prod<1>(a, maps, grid, st);
      case 2: return launch_tc_prod<2>(a, maps, grid, st);
      case 3: return launch_tc_prod<3>(a, maps, grid, st);
      default: return fail(TQ_ERR_UNSUPPORTED, "tq_quantize: no tensor-core kernel for this format");
    }
  }
  switch (a.mse_bits * 2 + a.mixed) {
    case 2: return launch_tc<1, 0>(a, maps, grid, st);
    case 4: return launch_tc<2, 0>(a, maps, grid, st);
    case 5: return launch_tc<2, 1>(a, maps, grid, st);
    case 6: return launch_tc<3, 0>(a, maps, grid, st);
    case 7: return launch_tc<3, 1>(a, maps, grid, st);
    case 8: return launch_tc<4, 0>(a, maps, grid, st);
    case 16: return launch_tc<kWideBits, 0>(a, maps, grid, st);
    default: return fail(TQ_ERR_UNSUPPORTED, "tq_quantize: no tensor-core kernel for this format");
  }
}

// Launches the quantize kernel for a (a.planes == 2 only where tc_eligible).
tq_status run_quantize(QuantArgs& a, cudaStream_t st) {
  if (a.n <= 0) return TQ_OK;
  if (tc_eligible(a)) return run_quantize_tc(a, st);
  if (a.planes != 1) return fail(TQ_ERR_UNSUPPORTED, "two-plane quantize needs the tensor-core kernels");
  const int64_t grid = quantize_grid(a);
  if (a.mse_bits == kWideBits) {
    quantize8_kernel<<<static_cast<unsigned>(grid), kDim, 0, st>>>(a);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TQ_OK : cuda_fail(e, "8-bit quantize kernel launch");
  }
  const size_t smem = quant_smem(a.prod);
  cudaError_t e;
  if (a.x_bf16) {
    e = ensure_dyn_smem<quantize_kernel<1>>(static_cast<int>(smem));
    if (e == cudaSuccess) quantize_kernel<1><<<grid, kThreads, smem, st>>>(a);
  } else {
    e = ensure_dyn_smem<quantize_kernel<0>>(static_cast<int>(smem));
    if (e == cudaSuccess) quantize_kernel<0><<<grid, kThreads, smem, st>>>(a);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "quantize kernel launch");
}

void fill_format(QuantArgs& a, const tq_params* p, const FormatSpec& f) {
  a.mse_bits = f.mse_bits;
  a.mixed = f.mixed;
  a.prod = f.prod;
  a.code_bytes = f.code_bytes;
  a.pi = p->pi32;
  a.pit = p->pit32;
  a.mt = p->mt32;
  a.status = p->status32;
  a.tc_img = p->tc_img;
  a.cb = p->cb32;
  a.bd = p->bd32;
  a.cell8 = p->cell8;
  a.cell8_n = p->cell8_n;
  a.cell8_inv_w = p->cell8_inv_w;
  a.pit64 = p->pit64;
}

}  // namespace

tq_status launch_quantize(const tq_params* p, const FormatSpec& f, const void* x, int x_bf16, int64_t n,
                          const tq_packed* out, cudaStream_t st) {
  QuantArgs a{};
  fill_format(a, p, f);
  a.planes = 1;
  a.x = x;
  a.x_bf16 = x_bf16;
  a.n = n;
  a.codes = out->codes;
  a.norms = out->norms;
  a.qjl = out->qjl;
  a.res = out->res_norms;
  return run_quantize(a, st);
}

namespace {

// The values' quantize kernel of an append runs on a side stream of the
// library, concurrently with the keys' kernel on the caller's stream: for a
// streaming chunk each grid holds a fraction of the SMs, so the two overlap
// instead of queueing.  The side stream forks from and joins the caller's
// stream through events (both recorded and waited inside one critical
// section, so concurrent callers cannot cross their dependencies); the
// pattern is valid under stream capture.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kSideDevices = 64;
std::mutex g_side_mu;
SideStream g_side[kSideDevices];

tq_status side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "tq_append: cudaGetDevice");
  if (dev < 0 || dev >= kSideDevices) return fail(TQ_ERR_UNSUPPORTED, "tq_append: device index too large");
  SideStream& s = g_side[dev];
  if (!s.stream) {
    e = cudaStreamCreateWithFlags(&s.stream, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      s = SideStream{};
      return cuda_fail(e, "tq_append: side stream");
    }
  }
  *out = &s;
  return TQ_OK;
}

}  // namespace

tq_status launch_append(const tq_params* p, const tq_cache* c, const int32_t* seq_ids, const void* k,
                        const void* v, int x_bf16, int n_tok, int n_seq, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(n_seq) * n_tok * c->n_kv_heads;
  QuantArgs q[2];
  for (int which = 0; which < 2; ++which) {
    const FormatSpec& f = which ? p->fv : p->fk;
    QuantArgs& a = q[which];
    a = QuantArgs{};
    fill_format(a, p, f);
    a.planes = 1;
    a.x = which ? v : k;
    a.x_bf16 = x_bf16;
    a.n = n;
    a.codes = which ? c->v_codes : c->k_codes;
    a.norms = which ? c->v_norms : c->k_norms;
    a.qjl = which ? c->v_qjl : c->k_qjl;
    a.res = which ? c->v_res_norms : c->k_res_norms;
    a.append = 1;
    a.kside = which == 0;
    a.seq_ids = seq_ids;
    a.lens = c->lens;
    a.n_tok = n_tok;
    a.hkv = c->n_kv_heads;
    a.capacity = c->capacity;
    a.n_sink = c->n_sink;
    a.cache_seqs = c->n_seq;
    a.sink = which ? c->v_sink : c->k_sink;
    a.status = c->status;
    a.n_seq_in = n_seq;
    a.head_major = !f.prod && tc_eligible(a);
  }
  // equal K and V formats on the tensor-core kernels: one launch for both
  QuantArgs both = q[0];
  both.planes = 2;
  both.x2 = v;
  both.codes2 = c->v_codes;
  both.norms2 = c->v_norms;
  both.qjl2 = c->v_qjl;
  both.res2 = c->v_res_norms;
  both.sink2 = c->v_sink;
  if (p->fk.id() == p->fv.id() && tc_eligible(both)) {
    both.arrive_total = static_cast<int>(quantize_grid(both));
    both.overlapped = 1;
    return run_quantize(both, st);
  }
  // otherwise K on the caller's stream and V on a side stream, concurrently;
  // the last CTA of either kernel updates the lengths
  const int64_t g0 = quantize_grid(q[0]), total = g0 + quantize_grid(q[1]);
  if (total > 0xFFFF) return fail(TQ_ERR_UNSUPPORTED, "tq_append: too many CTAs for the length update");
  q[0].arrive_total = q[1].arrive_total = static_cast<int>(total);
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* side = nullptr;
  tq_status sst = side_stream(&side);
  if (sst != TQ_OK) return sst;
  cudaError_t fe = cudaEventRecord(side->fork, st);
  if (fe == cudaSuccess) fe = cudaStreamWaitEvent(side->stream, side->fork, 0);
  if (fe != cudaSuccess) return cuda_fail(fe, "tq_append: fork");
  tq_status s = run_quantize(q[0], st);
  if (s == TQ_OK) {
    s = run_quantize(q[1], side->stream);
    // K's CTAs are counting already: arrive for the values' kernel
    if (s != TQ_OK) append_arrive_kernel<<<1, 128, 0, st>>>(q[0], static_cast<int>(total - g0));
  }
  // the side stream is joined to the caller's stream even on failure
  fe = cudaEventRecord(side->join, side->stream);
  if (fe == cudaSuccess) fe = cudaStreamWaitEvent(st, side->join, 0);
  if (s != TQ_OK) return s;
  return fe == cudaSuccess ? TQ_OK : cuda_fail(fe, "tq_append: join");
}

tq_status launch_cache_rows(const tq_params* p, const tq_cache* c, int which, int seq, int kv_head, int row0,
                            int64_t n, const tq_packed* rows, int to_cache, cudaStream_t st) {
  if (n == 0) return TQ_OK;
  const FormatSpec& f = which == TQ_K ? p->fk : p->fv;
  const CodeTile ct = make_code_tile(f.mse_bits, f.mixed, f.code_bytes);
  const int64_t unit_row0 = (static_cast<int64_t>(seq) * c->n_kv_heads + kv_head) * c->capacity + row0;
  const bool k = which == TQ_K;
  const int64_t blocks = (n + 127) / 128;
  cache_rows_kernel<<<static_cast<unsigned>(blocks), 128, 0, st>>>(
      to_cache, ct, k, k ? c->k_codes : c->v_codes, k ? c->k_norms : c->v_norms, f.prod ? (k ? c->k_qjl : c->v_qjl) : nullptr,
      f.prod ? (k ? c->k_res_norms : c->v_res_norms) : nullptr, unit_row0, rows->codes, rows->norms,
      f.prod ? rows->qjl : nullptr, f.prod ? rows->res_norms : nullptr, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, to_cache ? "tq_cache_write_rows" : "tq_cache_read_rows");
}

tq_status launch_dequantize(const tq_params* p, const FormatSpec& f, const tq_packed* in, int64_t n,
                            float* out, cudaStream_t st) {
  const int64_t blocks = (n + kDeqVecs - 1) / kDeqVecs;
  if (blocks > 0x7fffffff) return fail(TQ_ERR_UNSUPPORTED, "tq_dequantize: n too large");
  dequantize_kernel<<<static_cast<unsigned>(blocks), kDim, 0, st>>>(
      in->codes, in->norms, in->qjl, in->res_norms, n, f.mse_bits, f.mixed, f.prod, f.code_bytes, p->pi64,
      p->s64, p->cb64, p->cb8_64, out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "dequantize kernel launch");
}

}  // namespace tq
