// Top-k inner-product search over a quantized database: the second
// application of the quantizer on the page "TurboQuant-MLX: quantizzare pesi
// e KV cache per LLM open-weight su Mac", section "Il metodo TurboQuant, in
// breve" (similarity search in place of product quantization).  Every
// database row is scored with the estimator the decode kernels use,
//   <q, x^> = ||x|| (<Pi q, c[idx]> + sqrt(pi/2)/m ||r|| <S q, z>)
// (query scale 1 instead of log2(e)/sqrt(d)), and the k best rows per query
// are kept: larger score first, equal scores in row order.
//
// Kernels of one search (per group of up to 8 queries)
//   1. qrot_kernel (shared with decode): Pi q and S q as fp16 MMA fragments.
//   2. search_kernel over the leading rows (one chunk per CTA) and
//      search_merge_kernel in bound mode: each query's k-th best score there
//      becomes the starting bound of the full pass (large databases only).
//   3. search_kernel: persistent, the decode kernel's producer / consumer
//      pipeline over contiguous ranges of database chunks (K planes only).
//      Each consumer warp keeps, per query, its best candidates as a sorted
//      column across its lanes (lane j = j-th best) in shared memory; a warp
//      tile's scores are first tested against a per-query bound shared by
//      the CTA's warps (the best k-th score of any list), and only rows that
//      reach it are inserted.  At the end the 15 warps' lists of each query
//      are merged into the CTA's list.
//   4. search_merge_kernel: one CTA per query merges the CTAs' lists.
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

constexpr int kSearchMaxK = 32;      // one list entry per lane
constexpr int kSearchMaxCtas = 256;  // bound on the search grid (merge stages all lists)
// the consumer warps' candidate lists ([warp][query][32] keys) live in the
// scratch area of the decode kernel's shared-memory plan
static_assert(kConsumers * kMaxG * 32 * sizeof(uint64_t) <= kScratchBytes, "search lists exceed the scratch area");
static_assert(kMaxG <= kConsumers, "one merging warp per query");

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

// Candidate key: the score in an order-preserving unsigned form above the
// complemented row, so a larger key is a better candidate (ties on the score
// go to the lower row).  0 stands for "no candidate".
__device__ __forceinline__ uint64_t cand_key(float v, uint32_t row) {
  return (static_cast<uint64_t>(ord_score(v)) << 32) | static_cast<uint64_t>(~row);
}
__device__ __forceinline__ float key_score(uint64_t key) {
  return key == 0 ? -INFINITY : unord_score(static_cast<uint32_t>(key >> 32));
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


// Merge up to 32 candidates at once into a list (lane j holds entry j, both
// sorted by a bitonic network): the candidates c0..c3 of the eight lanes
// (g, t) that own a query are gathered one per lane (tile row L from lane
// (L & 7, t), component (L >> 4) * 2 + ((L >> 3) & 1)), sorted descending,
// and the list keeps the 32 largest of both (elementwise maximum against the
// reversed candidates, then a bitonic clean-up).  Cheaper than one insertion
// per candidate when many rows reach the bound (the first tiles).
__device__ __noinline__ uint64_t topk_merge32(uint64_t ent, uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                              int t_own, int lane) {
  const int src = ((lane & 7) << 2) | t_own, comp = ((lane >> 4) << 1) | ((lane >> 3) & 1);
  const uint64_t v0 = __shfl_sync(0xffffffffu, c0, src), v1 = __shfl_sync(0xffffffffu, c1, src);
  const uint64_t v2 = __shfl_sync(0xffffffffu, c2, src), v3 = __shfl_sync(0xffffffffu, c3, src);
  uint64_t key = comp == 0 ? v0 : comp == 1 ? v1 : comp == 2 ? v2 : v3;
#pragma unroll
  for (int k2 = 2; k2 <= 32; k2 <<= 1)
#pragma unroll
    for (int j = k2 >> 1; j > 0; j >>= 1) {
      const uint64_t o = __shfl_xor_sync(0xffffffffu, key, j);
      const bool keep_max = ((lane & j) == 0) == ((lane & k2) == 0);
      key = keep_max ? (o > key ? o : key) : (o < key ? o : key);
    }
  const uint64_t rev = __shfl_sync(0xffffffffu, key, 31 - lane);
  uint64_t m = ent > rev ? ent : rev;
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    const uint64_t o = __shfl_xor_sync(0xffffffffu, m, j);
    m = (lane & j) == 0 ? (o > m ? o : m) : (o < m ? o : m);
  }
  return m;
}

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
    const int n_c = __popc(__ballot_sync(0xffffffffu, c[0] != 0)) + __popc(__ballot_sync(0xffffffffu, c[1] != 0)) +
                    __popc(__ballot_sync(0xffffffffu, c[2] != 0)) + __popc(__ballot_sync(0xffffffffu, c[3] != 0));
    const uint64_t ent = n_c > 6 ? topk_merge32(lists[h * 32 + lane], c[0], c[1], c[2], c[3], h >> 1, lane)
                                 : topk_offer(lists[h * 32 + lane], c[0], c[1], c[2], c[3], lane, k);
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
  build_luts<L>(lut_mem, s_cb, tid, a.cbs8);
  consumers_sync();  // tables complete
  const uint32_t lut_a = 0, lut_b = 0;
  const uint32_t lane4 = kLutAddr | (lane * 4), lane8 = (kLutAddr + L::region_b_off) | (lane * 8);
  const uint32_t c1k = FK::mse == 1 ? h2bits(a.cbs[1 * kBookSlots + 1], a.cbs[1 * kBookSlots + 1]) : 0u;
  const TokRows tr = tok_rows(g, t);

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
    // the CTA's k best (the grid's k best are among the CTAs' k best)
    for (int r = 0; r < k; ++r) {
      const uint64_t best = warp_max_u64(head);
      if (lane == 0) dst[r] = best;
      if (best != 0 && head == best) {  // keys are unique apart from 0
        ++pos;
        head = pos < 32 ? scratch[(lane * kMaxG + h) * 32 + pos] : 0;
      }
    }
    if (lane >= k) dst[lane] = 0;
  }
  if (s_abort && tid == 0) atomicOr(a.status, 4);
}

// One CTA per query: the top k of the CTAs' sorted lists.
constexpr int kSearchMergeThreads = 256;
__global__ void __launch_bounds__(kSearchMergeThreads) search_merge_kernel(DecodeArgs a) {
  extern __shared__ uint64_t s_keys[];  // [ctas][32]
  const int h = blockIdx.x, P = a.ctas, k = a.topk, tid = threadIdx.x, lane = tid & 31;
  pdl_wait();  // the CTAs' lists
  // all 16-byte pieces of the lists in flight at once
  const uint64_t* src = a.cand + static_cast<int64_t>(h) * P * 32;
  for (int i = tid; i < P * 16; i += kSearchMergeThreads) cp_async16(smem_u32(s_keys + 2 * i), src + 2 * i);
  cp_async_wait_all();
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
  e = launch_qrot<KF>(a, 1, 1, st);
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
    a.cbs8 = p->cbs8_32;
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
    TQ_CASE(fid(8, 0, 0))
    return fail(TQ_ERR_UNSUPPORTED, "tq_search: no search kernel for this format");
#undef TQ_CASE
    if (r != TQ_OK) return r;
  }
  return TQ_OK;
}

}  // namespace tq
