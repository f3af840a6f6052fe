// The tiled layout of the cache's code planes, shared by the kernels that
// write the cache (streaming append, row import) and those that read it
// (decode attention, row export).
//
// A (sequence, kv-head) unit's quantized tokens form tiles of 16 tokens; tile
// i holds tokens 16i .. 16i + 15 in 16 * code_bytes bytes, tiles back to back.
// Inside a tile, the bytes are arranged for the decoding warp (32 lanes, lane
// L = 4g + t) so that each lane reads its share with at most three
// conflict-free shared-memory loads:
//   keys   (which = K): lane (g, t) owns tokens g and g + 8 and, of each code
//          segment, its quarter t: [A.seg0 | B.seg0 | A.seg1 | B.seg1] with
//          A = token g, B = token g + 8;
//   values (which = V): lane (g, t) owns tokens 2t, 2t+1, 2t+8, 2t+9 and, of
//          each segment, its eighth g: [a.seg0 | b.seg0 | c.seg0 | d.seg0 |
//          a.seg1 | ... | d.seg1] with a, b, c, d those tokens in order.
// Segments are those of the packed row (one of 128 coordinates, or two of 64
// in mixed rows); a piece is the contiguous run of bytes of the packed row
// that holds the lane's coordinates, copied as is.  Every piece is a whole
// number of bytes, so a byte of the tile belongs to exactly one token.
// A lane block is code_bytes / 2 bytes, stored as columns: the first 16 bytes
// of every lane (lane L's at 16 L), then the next 16 while 16 remain, then 8,
// then 4.
#pragma once

#include <stdint.h>

namespace tq {

struct CodeTile {
  int cb;    // packed row bytes (code_bytes)
  int b0;    // bits of segment 0
  int nd0;   // coordinates of segment 0 (128, or 64 in mixed rows)
  int b1;    // bits of segment 1 (mixed rows only)
  int nseg;  // segments: 0 (no codes), 1 or 2

  __host__ __device__ constexpr int lane_bytes() const { return cb / 2; }
  __host__ __device__ constexpr int tile_bytes() const { return 16 * cb; }
  __host__ __device__ constexpr int c16() const { return lane_bytes() / 16; }
  __host__ __device__ constexpr int c8() const { return (lane_bytes() % 16) / 8; }
  __host__ __device__ constexpr int c4() const { return (lane_bytes() % 8) / 4; }
  // tile byte of byte p of lane L's block
  __host__ __device__ constexpr int tile_off(int L, int p) const {
    return p < 16 * c16()             ? (p / 16) * 512 + L * 16 + p % 16
           : p < 16 * c16() + 8 * c8() ? 512 * c16() + L * 8 + (p - 16 * c16())
                                       : 512 * c16() + 256 * c8() + L * 4 + (p - 16 * c16() - 8 * c8());
  }
  __host__ __device__ constexpr int seg_bits(int s) const { return s == 0 ? b0 : b1; }
  __host__ __device__ constexpr int seg_dims(int s) const { return s == 0 ? nd0 : 64; }
  // first byte of segment s in the packed row
  __host__ __device__ constexpr int seg_byte(int s) const { return s == 0 ? 0 : nd0 * b0 / 8; }
  // keys: bytes of a quarter of segment s, and its place in the lane block
  __host__ __device__ constexpr int kpiece(int s) const { return seg_dims(s) * seg_bits(s) / 32; }
  __host__ __device__ constexpr int koff(int role, int s) const {
    return (s == 0 ? 0 : 2 * kpiece(0)) + role * kpiece(s);
  }
  // values: bytes of an eighth of segment s, and its place in the lane block
  __host__ __device__ constexpr int vpiece(int s) const { return seg_dims(s) * seg_bits(s) / 64; }
  __host__ __device__ constexpr int voff(int member, int s) const {
    return (s == 0 ? 0 : 4 * vpiece(0)) + member * vpiece(s);
  }
};

// The tile description of a format: mse_bits and mixed as in the packed row
// (prod formats: the MSE stage's bits), code_bytes the row's code bytes.
__host__ __device__ constexpr CodeTile make_code_tile(int mse_bits, int mixed, int code_bytes) {
  return CodeTile{code_bytes, mixed ? mse_bits + 1 : mse_bits, mixed ? 64 : 128, mse_bits,
                  mixed ? 2 : (mse_bits > 0 ? 1 : 0)};
}

// Byte k of a packed row held as little-endian 32-bit words.
__host__ __device__ __forceinline__ uint32_t row_byte(const uint32_t* words, int k) {
  return (words[k >> 2] >> (8 * (k & 3))) & 0xFFu;
}

// Calls fn(row_byte_index, tile_byte_offset) for every code byte of token tok
// (0..15) of a tile, for the keys' (kside) or the values' arrangement.
template <typename Fn>
__host__ __device__ __forceinline__ void for_each_tile_byte(const CodeTile& ct, bool kside, int tok, Fn&& fn) {
  for (int s = 0; s < ct.nseg; ++s) {
    if (kside) {
      const int g = tok & 7, role = tok >> 3, pb = ct.kpiece(s);
      for (int t = 0; t < 4; ++t) {
        const int L = 4 * g + t, src = ct.seg_byte(s) + t * pb, dst = ct.koff(role, s);
        for (int i = 0; i < pb; ++i) fn(src + i, ct.tile_off(L, dst + i));
      }
    } else {
      const int t = (tok & 7) >> 1, member = (tok & 1) + 2 * (tok >> 3), pb = ct.vpiece(s);
      for (int g = 0; g < 8; ++g) {
        const int L = 4 * g + t, src = ct.seg_byte(s) + g * pb, dst = ct.voff(member, s);
        for (int i = 0; i < pb; ++i) fn(src + i, ct.tile_off(L, dst + i));
      }
    }
  }
}

}  // namespace tq
