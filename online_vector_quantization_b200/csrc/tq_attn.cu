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
//   1. decode_kernel: persistent, one CTA per SM; a producer warp streams
//      the packed cache into shared memory with bulk copies, fifteen consumer
//      warps rotate the query at each (sequence, kv-head) unit they start
//      (q -> Pi q and S q, scaled by log2(e)/sqrt(d), as fp16 MMA
//      B-fragments) and walk 16-token tiles of the stream:
//        scores S^T[16 tok x 8 heads] = C_k[16 x 128] Q~^T  (mma.sync m16n8k16)
//        online softmax (base 2), sparse-V mask, P' = p * ||v||
//        O^T[128 x 8 heads] += C_v^T[128 x 16 tok] P'^T    (mma.sync m16n8k16)
//      The dequantized codebook values for both MMAs come straight from
//      per-lane-replicated shared-memory tables indexed by packed code bytes
//      (two or four codes per lookup, no bank conflicts), so no fp16 tile is
//      ever written back to memory.  Warps merge in shared memory and the CTA
//      writes one (m, l, acc) partial per piece of a (sequence, kv-head).
//   2. merge_kernel: one CTA per (sequence, kv-head), or per (sequence,
//      query head) for small batches, attends the bf16 sink, combines the
//      pieces and applies Pi^T / S^T once.  (The formats, tables and subtile
//      scoring live in tq_decode_common.cuh, shared with the inner-product
//      search.)

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "tq_internal.h"
#include "tq_sm100.cuh"
#include "tq_decode_common.cuh"

namespace tq {
namespace {

using namespace sm100;

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
  // tiled V codes (tq_layout.cuh): this lane's block holds tokens 2t, 2t+1,
  // 2t+8, 2t+9 (MMA columns) of the subtile, its eighth g of each segment
  constexpr CodeTile CT = code_tile<VF>();
  [[maybe_unused]] LaneBlock<VF> blk;
  if constexpr (FV::nseg > 0) blk.load(u.vcodes + (srow >> 4) * CT.tile_bytes(), 4 * g + t);
  if constexpr (FV::nseg > 0) {
    constexpr int MT = VR::S0::MT;
    typename VR::S0 xa, xb, xc, xd;
    xa.template from_block<CT.voff(0, 0)>(blk);
    xb.template from_block<CT.voff(1, 0)>(blk);
    xc.template from_block<CT.voff(2, 0)>(blk);
    xd.template from_block<CT.voff(3, 0)>(blk);
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
    xa.template from_block<CT.voff(0, 1)>(blk);
    xb.template from_block<CT.voff(1, 1)>(blk);
    xc.template from_block<CT.voff(2, 1)>(blk);
    xd.template from_block<CT.voff(3, 1)>(blk);
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

// Sparse-V tallies of one lane (summed over the grid when the caller asks for
// them): (token, query head) weights examined and dropped, 32-token warp
// tiles examined and tiles whose value work was skipped.
struct SparseTally {
  unsigned examined = 0, dropped = 0, tiles = 0, tiles_skipped = 0;
};

// One warp tile of 32 tokens (two 16-token subtiles) starting at stage row
// `srow`, unit-relative row `row0`; tokens at or past `nq` are masked (their
// scores are -inf and their value weights 0, so a subtile past the end adds
// nothing; computing it anyway keeps the two subtiles free of branches, which
// lets their lookup and MMA chains interleave).  SPARSE: 0 dense; 1 sparse V
// (weights below the bound are dropped, and the PV work of a tile whose
// weights are all dropped is skipped); 2 the same with tallies.
template <int KF, int VF, bool PACK, int WT, int SPARSE>
__device__ __forceinline__ void compute_tile(const UnitPlanes& u, int srow, int row0, int nq, const TokRows& tr,
                                             WarpState<KF, VF, PACK>& W, const QFrag<PACK>& bq,
                                             const QFrag<PACK>& bqs, int g, int t, uint32_t lut_a,
                                             uint32_t lut_b, uint32_t lane4, uint32_t lane8,
                                             uint32_t c1k, uint32_t c1v, float thr, int group, SparseTally& tally) {
  constexpr int VMT = WarpState<KF, VF, PACK>::VMT;
  constexpr bool second = WT == 2 * kTok;
  const bool ok0A = row0 + tr.kA < nq, ok0B = row0 + tr.kB < nq;
  const bool ok1A = row0 + kTok + tr.kA < nq, ok1B = row0 + kTok + tr.kB < nq;
  float s0[4], s1[4];
  subtile_scores<KF, PACK, Lut<KF, VF>::t3_wide, Lut<KF, VF>::t2a, false, true>(u, srow, tr, ok0A, ok0B, g, t, bq, bqs, lut_a, lut_b, lane4, lane8, c1k, s0);
  if constexpr (second)
    subtile_scores<KF, PACK, Lut<KF, VF>::t3_wide, Lut<KF, VF>::t2a, false, true>(u, srow + kTok, tr, ok1A, ok1B, g, t, bq, bqs, lut_a, lut_b, lane4, lane8, c1k, s1);
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
  if constexpr (SPARSE == 0) {
    subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow, tr, ok0A, ok0B, g, t, p0, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
    if constexpr (second)
      subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow + kTok, tr, ok1A, ok1B, g, t, p1, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
  } else {
    // Sparse V ("Greetings from TurboQuant-MLX", item 3): the value of a token
    // whose weight is below thr is left out (the denominator keeps it).  The
    // final weight is exp(s - M) / L with M, L the max and sum over all the
    // unit's tokens; exp(s - m) / l_c with m this warp's running max and l_c
    // the sum over the tokens this warp's column has seen (the eight lanes'
    // partial sums) is never below it, and l_c >= 1 (the token at the running
    // max counts exp(0)).  So a weight below thr * max(l_c, 1) is below thr in
    // the end: no token the exact rule keeps is dropped.
    float lc0 = W.l0, lc1 = W.l1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      lc0 += __shfl_xor_sync(0xffffffffu, lc0, off);
      lc1 += __shfl_xor_sync(0xffffffffu, lc1, off);
    }
    const float c0 = thr * fmaxf(lc0, 1.f), c1 = thr * fmaxf(lc1, 1.f);
    const bool col0 = 2 * t < group, col1 = 2 * t + 1 < group;  // real heads (packed: the hi columns)
    const bool okr[4] = {ok0A, ok0B, ok1A, ok1B};
    float* pp[4] = {&p0[0], &p0[2], &p1[0], &p1[2]};
    bool keep = false;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float* pr = pp[r];
      const bool d0 = pr[0] < c0, d1 = pr[1] < c1;
      if constexpr (SPARSE == 2) {
        if (okr[r]) {
          tally.examined += col0 + col1;
          tally.dropped += (col0 && d0) + (col1 && d1);
        }
      }
      pr[0] = d0 ? 0.f : pr[0];
      pr[1] = d1 ? 0.f : pr[1];
      // columns past the group (empty heads) never keep a tile alive
      keep |= (col0 && pr[0] > 0.f) | (col1 && pr[1] > 0.f);
    }
    if constexpr (SPARSE == 2) ++tally.tiles;
    // the value work is skipped only when every weight of the warp tile was
    // dropped; otherwise both subtiles run without branches, as on the dense
    // path (a per-subtile branch costs more than it saves at GQA widths)
    if (__any_sync(0xffffffffu, keep)) {
      subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow, tr, ok0A, ok0B, g, t, p0, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
      if constexpr (second)
        subtile_pv<VF, VMT, Lut<KF, VF>::t2a>(u, srow + kTok, tr, ok1A, ok1B, g, t, p1, lut_a, lut_b, lane4, lane8, c1v, W.oacc);
    } else if constexpr (SPARSE == 2) {
      ++tally.tiles_skipped;
    }
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
// A unit with quantized tokens occupies slack + chunks slots of the list:
// `slack` (a.unit_slack) empty slots model the fixed cost a CTA pays when it
// starts a unit (combining the previous piece, rotating the query, merging),
// so CTAs whose ranges cross more units get fewer chunks.  Empty slots are
// skipped by the producer and the consumers alike.
struct UnitInfo {
  int len, ns, nq, chunks, slack, slots;
};

// lens: the cache's lengths (global), or the decode kernel's copy of them in
// shared memory.  Read as volatile: a kernel launched with programmatic
// stream serialization may run beside the one that wrote them, so they are
// fetched from L2, never from a stale L1 line.
__device__ __forceinline__ UnitInfo unit_info(const DecodeArgs& a, const volatile int* lens, int u, int kChunk) {
  const int b = u / a.hkv;
  const int len = min(max(lens[b], 0), a.max_len);
  UnitInfo r;
  r.len = len;
  r.ns = min(a.n_sink, len);
  r.nq = len - r.ns;
  r.chunks = (r.nq + kChunk - 1) / kChunk;
  r.slack = r.chunks > 0 ? a.unit_slack : 0;
  r.slots = r.chunks + r.slack;
  return r;
}


// Slots of each kv-head unit of sequence b (all units of a sequence are alike).
__device__ __forceinline__ int seq_slots(const DecodeArgs& a, const volatile int* lens, int b, int kChunk) {
  const int len = min(max(lens[b], 0), a.max_len);
  const int ch = (len - min(a.n_sink, len) + kChunk - 1) / kChunk;
  return ch > 0 ? ch + a.unit_slack : 0;
}

// CTA whose range holds chunk c: the largest i with i*C/P <= c.
__device__ __forceinline__ int cta_of_chunk(int64_t c, int64_t C, int P) {
  return static_cast<int>(((c + 1) * P - 1) / C);
}

// Ranges are empty when C < P; such CTAs hold no piece of any unit.
__device__ __forceinline__ bool cta_has_chunks(int i, int64_t C, int P) {
  return range_start(i + 1, C, P) > range_start(i, C, P);
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

// Cross-warp combine of one piece into partial slot `slot` (consumer
// threads).  Every warp rescales its accumulator to the CTA's maximum before
// storing it, so the combine is a plain sum over warps, done in 64-coordinate
// slices of the accumulator.  LANE_SUMS: each lane holds its own partial
// softmax sums (dense path), added over the column first.
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
  consumers_sync();
  // this lane's two columns: the CTA's maximum and this warp's factor
  float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
  for (int w = 0; w < kConsumers; ++w) {
    M0 = fmaxf(M0, wm[w * kMaxG + 2 * t]);
    M1 = fmaxf(M1, wm[w * kMaxG + 2 * t + 1]);
  }
  const float f0 = W.m0 > -INFINITY ? exp2f(W.m0 - M0) : 0.f;
  const float f1 = W.m1 > -INFINITY ? exp2f(W.m1 - M1) : 0.f;
  if (tid < a.group) {  // the piece's maximum and sum of head tid
    const int h = tid;
    float M = -INFINITY, l = 0.f;
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, wm[w * kMaxG + h]);
    for (int w = 0; w < kConsumers; ++w) {
      const float mw = wm[w * kMaxG + h];
      if (mw > -INFINITY) l = fmaf(wl[w * kMaxG + h], exp2f(mw - M), l);
    }
    dst[h * PF + 0] = M;
    dst[h * PF + 1] = l;
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
        w0[d0] = W.oacc[mt][0] * f0;
        w1[d0] = W.oacc[mt][1] * f1;
      }
      if (d1 >= lo && d1 < lo + kSliceDims) {
        w0[d1] = W.oacc[mt][2] * f0;
        w1[d1] = W.oacc[mt][3] * f1;
      }
    }
    consumers_sync();
    for (int i = tid; i < a.group * kSliceDims; i += NT) {
      const int h = i / kSliceDims, j = i % kSliceDims;
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) acc += wacc[(w * kMaxG + h) * kSliceDims + j];
      dst[h * PF + kPartAcc + lo + j] = acc;
    }
    consumers_sync();
  }
}

// ---------------------------------------------------------------------------
// 3. merge: one CTA per unit (sequence, kv-head) and group of merge_heads
//    query heads (all heads of the unit's group, or one head each when the
//    units are too few to fill the GPU otherwise).
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
// merge_chunk pieces (the CTA's heads x part_floats floats each).  Small
// enough for two merge CTAs per SM.
constexpr size_t kMergeStageBytes = 32 * 1024;
inline int merge_chunk_pieces(int group, int part_floats) {
  const size_t per = static_cast<size_t>(group) * part_floats * sizeof(float);
  return static_cast<int>(std::max<size_t>(1, kMergeStageBytes / per));
}
inline size_t merge_dyn_bytes(int n_sink, int ctas, int group, int part_floats, int mh) {
  return (static_cast<size_t>(n_sink) + 2 * static_cast<size_t>(ctas)) * mh * sizeof(float) +
         static_cast<size_t>(merge_chunk_pieces(group, part_floats)) * group * part_floats * sizeof(float);
}

// MH: heads per CTA the kernel is compiled for (1, 4 or 8; a.merge_heads <= MH).
template <int VF, int MH>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(DecodeArgs a) {
  static_assert(MH == 1 || MH == 4 || MH == 8, "heads per merge CTA");
  pdl_launch();  // the next append's kernel may set itself up meanwhile (it waits for this grid)
  using FV = Fmt<VF>;
  constexpr int NT = kMergeThreads;
  constexpr int WD = FV::prod ? 2 * kDim : kDim;  // accumulator: rotated | sketch
  constexpr int NS = NT / WD;                     // piece slices of the accumulation
  constexpr int RS = WD / 4;                      // matrix rows per un-rotation slice
  extern __shared__ float4 s_dyn4[];
  __shared__ float s_red[4 * MH * kDim];       // slice partials
  __shared__ __align__(16) float s_acc[WD][MH];  // merged accumulator, [j][head]
  __shared__ float s_osk[MH][kDim];            // sink values, original domain
  __shared__ float s_q[MH][4][33];  // query quarters, padded: the four quarters sit in different banks
  __shared__ float s_ms[MH], s_ls[MH], s_M[MH], s_L[MH];
  __shared__ long long s_C, s_cu0;
  float* s_sc = reinterpret_cast<float*>(s_dyn4);  // [n_sink][MH]
  float* s_f = s_sc + a.n_sink * MH;             // [pieces][MH]: maxima, then weights
  float* s_l = s_f + a.ctas * MH;                // [pieces][MH]: sums
  float* s_part = s_l + a.ctas * MH;             // staged pieces [merge_chunk][G][part_floats]
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.merge_heads, h0 = blockIdx.y * G;  // this CTA's heads: h0 .. h0 + G - 1 of the group
  const int P = a.ctas, CH = a.chunk, PF = a.part_floats;
  const int b = u / a.hkv, kvh = u % a.hkv;
  // head h0 of the unit's group
  const int64_t orow = (static_cast<int64_t>(b) * a.hq + kvh * a.group + h0) * kDim;
  const UnitInfo ui = unit_info(a, a.lens, u, CH);
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
      const int ch = seq_slots(a, a.lens, v, CH);
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
      s_cu0 = before * a.hkv + static_cast<long long>(kvh) * ui.slots + ui.slack;
    }
  }
  // sink: scores with the original query, softmax weights, weighted values
  if (ui.ns > 0) {
    for (int i = tid; i < MH * kDim; i += NT)
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
        float d[MH];
#pragma unroll
        for (int h = 0; h < MH; ++h) d[h] = 0.f;
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
              for (int h = 0; h < MH; ++h) d[h] = fmaf(k1, s_q[h][qtr][j + 1], fmaf(k0, s_q[h][qtr][j], d[h]));
            }
          }
        }
#pragma unroll
        for (int h = 0; h < MH; ++h) {
          d[h] += __shfl_xor_sync(0xffffffffu, d[h], 1);
          d[h] += __shfl_xor_sync(0xffffffffu, d[h], 2);
        }
        if (tt < cnt && qtr == 0)
#pragma unroll
          for (int h = 0; h < MH; ++h)
            if (h < G) s_sc[(c0 + tt) * MH + h] = d[h] * scale;
      }
      __syncthreads();  // the staging buffer is refilled
    }
    if (warp < G) {  // warp h: max, weights and sum of head h
      const int h = warp;
      float mx = -INFINITY;
      for (int tt = lane; tt < ui.ns; tt += 32) mx = fmaxf(mx, s_sc[tt * MH + h]);
      mx = warp_max(mx);
      float sum = 0.f;
      for (int tt = lane; tt < ui.ns; tt += 32) {
        const float pw = exp2f(s_sc[tt * MH + h] - mx);
        s_sc[tt * MH + h] = pw;
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
      float acc[MH];
#pragma unroll
      for (int h = 0; h < MH; ++h) acc[h] = 0.f;
      for (int c0 = 0; c0 < ui.ns; c0 += SC) {
        const int cnt = min(SC, ui.ns - c0);
        stage_rows(vs, c0, cnt);
        for (int tt = sl4; tt < cnt; tt += 4) {
          const float v = __bfloat162float(srow[tt * kDim + o]);
          if constexpr (MH == 1) {
            acc[0] = fmaf(s_sc[c0 + tt], v, acc[0]);
          } else {
#pragma unroll
            for (int q4 = 0; q4 < MH / 4; ++q4) {
              const float4 pw = s_dyn4[(c0 + tt) * (MH / 4) + q4];
              acc[4 * q4] = fmaf(pw.x, v, acc[4 * q4]);
              acc[4 * q4 + 1] = fmaf(pw.y, v, acc[4 * q4 + 1]);
              acc[4 * q4 + 2] = fmaf(pw.z, v, acc[4 * q4 + 2]);
              acc[4 * q4 + 3] = fmaf(pw.w, v, acc[4 * q4 + 3]);
            }
          }
        }
        __syncthreads();  // the staging buffer is refilled
      }
#pragma unroll
      for (int h = 0; h < MH; ++h) s_red[(sl4 * MH + h) * kDim + o] = acc[h];
    }
    __syncthreads();
    for (int i = tid; i < G * kDim; i += NT) {
      const int h = i / kDim, j = i % kDim;
      s_osk[h][j] = s_red[(0 * MH + h) * kDim + j] + s_red[(1 * MH + h) * kDim + j] +
                    s_red[(2 * MH + h) * kDim + j] + s_red[(3 * MH + h) * kDim + j];
    }
  } else if (tid < MH) {
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
  // this CTA's heads of each piece: G x PF consecutive floats at head h0,
  // staged with 16-byte asynchronous copies, merge_chunk pieces at a time
  const int slot_floats = G * PF, per4 = slot_floats / 4;
  auto stage = [&](int c0, int cnt) {
    for (int e = tid; e < cnt * per4; e += NT) {
      const int i = e / per4, q4 = e - i * per4;
      const float4* src = reinterpret_cast<const float4*>(part_slot(a, u + first + c0 + i) + h0 * PF);
      cp_async16(smem_u32(s_part) + 16 * e, src + q4);
    }
    cp_async_wait_all();
    __syncthreads();
  };
  // usually every piece fits one staging pass: the maxima and sums are then
  // read from the staged copies, one memory round trip after the wait
  const bool one_pass = has_pieces && n_p <= a.merge_chunk;
  if (one_pass) stage(0, n_p);
  for (int e = tid; e < n_p * G; e += NT) {
    const int i = e / G, h = e % G;
    float m = -INFINITY, l = 0.f;
    if (cta_has_chunks(first + i, C, P)) {
      if (one_pass) {
        const float* pp = s_part + i * slot_floats + h * PF;
        m = pp[0];
        l = pp[1];
      } else {
        const float* pp = part_slot(a, u + first + i) + (h0 + h) * PF;
        m = __ldcg(pp);
        l = __ldcg(pp + 1);
      }
    }
    s_f[i * MH + h] = m;
    s_l[i * MH + h] = l;
  }
  __syncthreads();
  if (warp < G) {  // warp h: merged maximum, the pieces' weights and the sum for head h
    const int h = warp;
    float M = s_ms[h];
    for (int i = lane; i < n_p; i += 32) M = fmaxf(M, s_f[i * MH + h]);
    M = warp_max(M);
    float L = 0.f;
    for (int i = lane; i < n_p; i += 32) {
      const float m = s_f[i * MH + h];
      const float f = m > -INFINITY ? exp2f(m - M) : 0.f;
      L = fmaf(s_l[i * MH + h], f, L);
      s_f[i * MH + h] = f;
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
      // the accumulators (already staged in the one-pass case)
      const int j = tid % WD, sl = tid / WD;
      float acc[MH];
#pragma unroll
      for (int h = 0; h < MH; ++h) acc[h] = 0.f;
      for (int c0 = 0; c0 < n_p; c0 += a.merge_chunk) {
        const int cnt = min(a.merge_chunk, n_p - c0);
        if (!one_pass) stage(c0, cnt);
        for (int i = sl; i < cnt; i += NS) {
          const float* pp = s_part + i * slot_floats + kPartAcc + j;
#pragma unroll
          for (int h = 0; h < MH; ++h) {
            // weight 0: a piece of a CTA with an empty range, whose slot was
            // not written in this call
            const float f = h < G ? s_f[(c0 + i) * MH + h] : 0.f;
            if (f != 0.f) acc[h] = fmaf(pp[h * PF], f, acc[h]);
          }
        }
        if (!one_pass) __syncthreads();  // the staging buffer is refilled
      }
#pragma unroll
      for (int h = 0; h < MH; ++h) s_red[(sl * MH + h) * WD + j] = acc[h];
    }
    __syncthreads();
    for (int i = tid; i < MH * WD; i += NT) {
      const int j = i / MH, h = i % MH;
      float v = 0.f;
#pragma unroll
      for (int sl = 0; sl < NS; ++sl) v += s_red[(sl * MH + h) * WD + j];
      if (j < kDim) v = FV::width(j) > 0 ? v / a.sig[FV::width(j)] : 0.f;
      s_acc[j][h] = h < G ? v : 0.f;
    }
    __syncthreads();
    // un-rotation: out_h[o] = sum_j Pi[j][o] A_h[j] + sqrt(pi/2)/m sum_j S[j][o] B_h[j]
    float r[MH];
#pragma unroll
    for (int h = 0; h < MH; ++h) r[h] = 0.f;
#pragma unroll
    for (int jj = 0; jj < RS; ++jj) {
      if constexpr (MH == 1) {
        r[0] = fmaf(pm[jj], s_acc[sl4 * RS + jj][0], r[0]);
      } else {
        const float4* acc4 = reinterpret_cast<const float4*>(&s_acc[sl4 * RS + jj][0]);
#pragma unroll
        for (int q4 = 0; q4 < MH / 4; ++q4) {
          const float4 x = acc4[q4];
          r[4 * q4] = fmaf(pm[jj], x.x, r[4 * q4]);
          r[4 * q4 + 1] = fmaf(pm[jj], x.y, r[4 * q4 + 1]);
          r[4 * q4 + 2] = fmaf(pm[jj], x.z, r[4 * q4 + 2]);
          r[4 * q4 + 3] = fmaf(pm[jj], x.w, r[4 * q4 + 3]);
        }
      }
    }
    __syncthreads();  // s_red is reused
#pragma unroll
    for (int h = 0; h < MH; ++h) s_red[(sl4 * MH + h) * kDim + o] = r[h];
    __syncthreads();
  }
  for (int i = tid; i < G * kDim; i += NT) {
    const int h = i / kDim, j = i % kDim;
    float v = 0.f;
    if (has_pieces)
      v = s_red[(0 * MH + h) * kDim + j] + s_red[(1 * MH + h) * kDim + j] + s_red[(2 * MH + h) * kDim + j] +
          s_red[(3 * MH + h) * kDim + j];
    if (ui.ns > 0) v = fmaf(s_M[h], s_osk[h][j], v);
    const float L = s_L[h];
    store_out(a, orow + i, L > 0.f ? v / L : 0.f);
  }
}


template <int KF, int VF, bool PACK, int SPARSE>
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
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ long long s_c0, s_c1;
  __shared__ int s_u0, s_lc0;
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int P = gridDim.x, cta = blockIdx.x;
  const int U = a.B * a.hkv;
  // the lengths, read once: every later unit lookup is a shared-memory load
  constexpr int kLenCache = 128;
  __shared__ int s_len[kLenCache];
  if (a.B <= kLenCache)
    for (int b = tid; b < a.B; b += kThreadsP) s_len[b] = __ldcg(a.lens + b);
  const volatile int* lens = a.B <= kLenCache ? s_len : a.lens;

  // ---- barriers (thread 32); the producer starts the copy of the lookup
  // tables (built once per parameter set) while warp 0 computes the schedule
  __shared__ __align__(8) uint64_t lut_bar;
  if (tid == 32) {
#pragma unroll
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kConsumers);
    }
    mbar_init(&lut_bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if constexpr (L::bytes > 0) {
    if (tid == kConsumers * 32) {
      mbar_expect_tx(&lut_bar, L::bytes);
      constexpr int kPart = 32768;
#pragma unroll
      for (int off = 0; off < L::bytes; off += kPart)
        bulk_g2s_addr(kLutAddr + off, a.lut_img + off, min(kPart, L::bytes - off), &lut_bar);
    }
  }
  if (warp == 0) {
    // schedule (one warp): total chunks C, this CTA's range [c0, c1) and the
    // unit / local chunk where it starts
    long long C = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      int ch = b0 + lane < a.B ? seq_slots(a, lens, b0 + lane, CH) : 0;
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
      const long long ch = b < a.B ? seq_slots(a, lens, b, CH) : 0;
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
        if (lens[b] > a.max_len) atomicOr(a.status, 2);
    if (lane == 0) {
      s_c0 = c0;
      s_c1 = c1;
      s_u0 = u0;
      s_lc0 = lc0;
      s_abort = 0;
    }
  }
  __syncthreads();
  const long long c0 = s_c0, c1 = s_c1;

  if (warp == kConsumers) {
    // ---- producer: one lane streams the CTA's chunks through the stages
    if (lane == 0 && c0 < c1) {
      int u = s_u0, lc = s_lc0;
      UnitInfo ui = unit_info(a, lens, u, CH);
      const int nk = static_cast<int>(c1 - c0);
      int s = 0, n_streamed = 0;
      uint32_t round = 0;  // parity of (chunks streamed) / S
      for (int k = 0; k < nk; ++k) {
        while (lc >= ui.slots) {
          ++u;
          lc = 0;
          ui = unit_info(a, lens, u, CH);
        }
        if (lc < ui.slack) {  // an empty slot
          ++lc;
          continue;
        }
        if (n_streamed >= S && !mbar_wait(&empty_bar[s], round ^ 1u)) s_abort = 1;
        if (s_abort) break;
        ++n_streamed;
        const int64_t ubase = static_cast<int64_t>(u) * a.capacity;
        const int r0 = (lc - ui.slack) * CH;
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

  bool luts_ready = L::bytes == 0;  // waited for before the first tile
  bool frags_ready = false;         // the rotated query, waited for at the first unit

  // ---- consumers
  // table bases are folded into the lane offsets (see kLutAddr)
  const uint32_t lut_a = 0, lut_b = 0;
  const uint32_t lane4 = kLutAddr | (lane * 4), lane8 = (kLutAddr + L::region_b_off) | (lane * 8);
  const uint32_t c1k = FK::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const uint32_t c1v = FV::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const float thr = a.sparse_thr;
  const TokRows trows = tok_rows(g, t);

  WarpState<KF, VF, PACK> wst;
  QFrag<PACK> bq, bqs;
  int u = -1;
  UnitInfo ui{};
  int walk_u = s_u0, walk_lc = s_lc0;
  UnitInfo wui = c0 < c1 ? unit_info(a, lens, walk_u, CH) : UnitInfo{};
  const int nk = static_cast<int>(c1 - c0);
  int s = 0;
  uint32_t round = 0;  // parity of k / S
  SparseTally tally;
  for (int k = 0; k < nk; ++k) {
    while (walk_lc >= wui.slots) {
      ++walk_u;
      walk_lc = 0;
      wui = unit_info(a, lens, walk_u, CH);
    }
    if (walk_lc < wui.slack) {  // an empty slot
      ++walk_lc;
      continue;
    }
    if (walk_u != u) {
      if (u >= 0) write_piece<KF, VF, PACK, true>(a, wst, u + cta, scratch, warp, g, t);
      u = walk_u;
      ui = wui;
      if (!frags_ready) {
        pdl_wait();  // the query rotation kernel's fragments
        frags_ready = true;
      }
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
    if (!luts_ready) {
      if (!mbar_wait(&lut_bar, 0)) s_abort = 1;
      luts_ready = true;
    }
    if (!s_abort && !mbar_wait(&full_bar[s], round)) s_abort = 1;
    const int row0 = (walk_lc - ui.slack) * CH + warp * WT;
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
                                             c1k, c1v, thr, a.group, tally);
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
  if (!luts_ready) mbar_wait(&lut_bar, 0);  // no copy may target a finished CTA
  if (s_abort && tid == 0) atomicOr(a.status, 4);
  if constexpr (SPARSE == 2) {
    {
      unsigned long long v[4] = {tally.examined, tally.dropped, lane == 0 ? tally.tiles : 0u,
                                 lane == 0 ? tally.tiles_skipped : 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], off);
      }
      if (lane == 0)
#pragma unroll
        for (int i = 0; i < 4; ++i) atomicAdd(a.sv_stats + i, v[i]);
    }
  }
}


// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------



template <int KF, int VF, bool PACK, int SPARSE>
tq_status run_decode_v(DecodeArgs& a, const DecodePlan& plan, size_t smem, cudaStream_t st) {
  cudaError_t e = ensure_dyn_smem<decode_kernel<KF, VF, PACK, SPARSE>>(static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel attribute");
  // the query rotation loads its matrix entries while the previous kernel on
  // the stream (the append that filled the cache, say) finishes, and reads
  // the query only after it; the decode kernel after it starts its prologue
  // (tables, schedule, first bulk copies) while the rotation runs, and the
  // merge kernel overlaps its prologue with the decode kernel's tail
  e = launch_qrot<KF>(a, plan.B, plan.hkv, st, true);
  if (e != cudaSuccess) return cuda_fail(e, "query rotation launch");
  e = launch_overlapped(decode_kernel<KF, VF, PACK, SPARSE>, dim3(plan.ctas), kThreadsP, smem, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  // static and dynamic shared memory together pass 48 KB: opt in every time
  auto merge = [&](auto mh) -> tq_status {
    constexpr int MH = decltype(mh)::value;
    const size_t merge_smem = merge_dyn_bytes(a.n_sink, plan.ctas, a.merge_heads, plan.part_floats, MH);
    cudaError_t me = ensure_dyn_smem<merge_kernel<VF, MH>>(static_cast<int>(merge_smem));
    if (me == cudaSuccess) me = ensure_max_carveout<merge_kernel<VF, MH>>();
    if (me != cudaSuccess) return cuda_fail(me, "merge kernel attribute");
    me = launch_overlapped(merge_kernel<VF, MH>, dim3(plan.B * plan.hkv, plan.group / a.merge_heads), kMergeThreads,
                           merge_smem, st, a);
    return me == cudaSuccess ? TQ_OK : cuda_fail(me, "merge kernel launch");
  };
  if (a.merge_heads == 1) return merge(IntC<1>{});
  return a.merge_heads <= 4 ? merge(IntC<4>{}) : merge(IntC<8>{});
}

template <int KF, int VF>
tq_status run_decode(DecodeArgs& a, const DecodePlan& plan, cudaStream_t st) {
  if (decode_smem_bytes<KF, VF>() + kDynBaseMax > static_cast<size_t>(kSmemEnd))
    return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: no shared-memory plan for this format");
  const size_t smem = kSmemBudget;  // the whole window: one CTA per SM
  a.dyn_bytes = static_cast<uint32_t>(smem);
  a.pack = plan.group <= 4;
  a.chunk = DecodeCfg<KF, VF>::CH;
  // a unit start costs about two 480-token chunks of streaming
  a.unit_slack = std::max(1, 960 / DecodeCfg<KF, VF>::CH);
  if (a.sparse_thr > 0.f && a.sv_stats)
    return a.pack ? run_decode_v<KF, VF, true, 2>(a, plan, smem, st) : run_decode_v<KF, VF, false, 2>(a, plan, smem, st);
  if (a.sparse_thr > 0.f)
    return a.pack ? run_decode_v<KF, VF, true, 1>(a, plan, smem, st) : run_decode_v<KF, VF, false, 1>(a, plan, smem, st);
  return a.pack ? run_decode_v<KF, VF, true, 0>(a, plan, smem, st) : run_decode_v<KF, VF, false, 0>(a, plan, smem, st);
}



}  // namespace

namespace {
// The lookup tables of a format pair, built once into global memory: the
// decode kernel's shared-memory table region, byte for byte.
template <int KF, int VF>
__global__ void __launch_bounds__(kConsumers * 32) lut_image_kernel(unsigned char* img, const float* cbs,
                                                                       const float* cbs8) {
  build_luts<Lut<KF, VF>>(img, cbs, threadIdx.x, cbs8);
}

template <int KF, int VF>
size_t lut_bytes_of() {
  return Lut<KF, VF>::bytes;
}

template <int K, int V>
struct PairTag {
  static constexpr int kf = K, vf = V;
};

// Calls fn(PairTag<KF, VF>{}) for a format pair with a decode kernel;
// returns false otherwise.
template <typename Fn>
bool dispatch_pair(int kf, int vf, Fn&& fn) {
#define TQ_PAIR(K, V)                \
  if (kf == (K) && vf == (V)) {      \
    fn(PairTag<(K), (V)>{});         \
    return true;                     \
  }
  TQ_PAIR(fid(1, 0, 0), fid(1, 0, 0))
  TQ_PAIR(fid(2, 0, 0), fid(2, 0, 0))
  TQ_PAIR(fid(3, 0, 0), fid(3, 0, 0))
  TQ_PAIR(fid(4, 0, 0), fid(4, 0, 0))
  TQ_PAIR(fid(3, 1, 0), fid(3, 1, 0))
  TQ_PAIR(fid(2, 1, 0), fid(2, 1, 0))
  TQ_PAIR(fid(0, 0, 1), fid(0, 0, 1))
  TQ_PAIR(fid(1, 0, 1), fid(1, 0, 1))
  TQ_PAIR(fid(2, 0, 1), fid(2, 0, 1))
  TQ_PAIR(fid(3, 0, 1), fid(3, 0, 1))
  TQ_PAIR(fid(4, 0, 0), fid(3, 0, 0))
  TQ_PAIR(fid(4, 0, 0), fid(2, 0, 0))
  TQ_PAIR(fid(3, 0, 0), fid(2, 0, 0))
  TQ_PAIR(fid(8, 0, 0), fid(3, 0, 0))
#undef TQ_PAIR
  return false;
}
}  // namespace

size_t decode_lut_bytes(const FormatSpec& fk, const FormatSpec& fv) {
  size_t bytes = 0;
  dispatch_pair(fk.id(), fv.id(), [&](auto tag) {
    using T = decltype(tag);
    bytes = lut_bytes_of<T::kf, T::vf>();
  });
  return bytes;
}

tq_status build_decode_luts(tq_params* p) {
  cudaError_t e = cudaSuccess;
  dispatch_pair(p->fk.id(), p->fv.id(), [&](auto tag) {
    using T = decltype(tag);
    if (Lut<T::kf, T::vf>::bytes == 0) return;
    lut_image_kernel<T::kf, T::vf><<<1, kConsumers * 32>>>(p->lut_img, p->cbs32, p->cbs8_32);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaStreamSynchronize(nullptr);
  });
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_params_create: decode lookup tables");
}

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
  // piece (u, cta) uses slot u + cta: fewer than units + ctas slots
  const size_t slots = units + pl.ctas;
  pl.ws_qfrag_bytes = (units * kQfragWords * sizeof(uint32_t) + 255) & ~size_t(255);
  pl.ws_parts_bytes = (slots * pl.group * pl.part_floats * sizeof(float) + 255) & ~size_t(255);
  pl.ws_total_bytes = pl.ws_qfrag_bytes + pl.ws_parts_bytes;
  return pl;
}

tq_status launch_decode(const tq_params* p, const void* q, int q_bf16, const tq_cache* c, const DecodePlan& plan,
                        void* out, int out_bf16, void* ws, float sparse_thr, unsigned long long* sv_stats,
                        cudaStream_t st) {
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
  // few units (small batches, long contexts): one merge CTA per (unit, head)
  // so the merge work spreads over the GPU; otherwise one per unit
  {
    const long long units = static_cast<long long>(plan.B) * plan.hkv;
    a.merge_heads = units * plan.group <= 2LL * num_sms_cached() ? 1 : plan.group;
  }
  a.merge_chunk = merge_chunk_pieces(a.merge_heads, plan.part_floats);
  if (c->n_sink > kMaxSink) return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: n_sink above 4096");
  a.qfrag = static_cast<uint32_t*>(ws);
  a.parts = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.ws_qfrag_bytes);
  a.out = out;
  a.out_bf16 = out_bf16;
  a.pit = p->pit32;
  a.st = p->st32;
  a.pi = p->pi32;
  a.s = p->s32;
  a.cbs = p->cbs32;
  a.cbs8 = p->cbs8_32;
  a.lut_img = p->lut_img;
  a.sig = p->sig32;
  a.sparse_thr = sparse_thr;
  a.sv_stats = sv_stats;
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
  TQ_CASE(fid(8, 0, 0), fid(3, 0, 0))
#undef TQ_CASE
  return fail(TQ_ERR_UNSUPPORTED, "tq_decode_attn: this K/V format pair has no decode kernel");
}


}  // namespace tq
