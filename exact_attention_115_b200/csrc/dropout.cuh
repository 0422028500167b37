// Dropout keep masks drawn inside the attention kernels.
//
// The weights P of one head index bh = b·H + h form an [Nq, Nk] matrix cut
// into 4×4 blocks.  Block (query block rb, key block cb) is one call of the
// Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) with counter
// (cb, rb, bh, offset) and key (seed low, seed high): output word i belongs
// to query row 4·rb + i, byte j (least significant first) of that word to key
// 4·cb + j.  A weight is kept iff its byte is below the threshold
// T = round((1 − p)·256) (1 ≤ T ≤ 255), and kept weights are scaled by
// 256 / T.  The study notes on FlashAttention V1/V2 (51CTO), section
// "算法的改进", mention the dropout steps of the V1 algorithm; the generator
// and this layout are this library's choice.
//
// Four neighbouring lanes of a warp own four consecutive rows (forward: query
// rows) or keys (backward) of a tile, so they share every block of a 16-wide
// column group: each lane draws one block and a 4×4 exchange across the lanes
// hands every lane its own 16 bytes.
#pragma once
#include <cstdint>

#include "launch.h"  // DropoutParams

namespace fa {

// Philox4x32-10: ten rounds of two 32×32→64 products and a key-mixed swap.
// The round keys (the seed advanced by the Weyl constants, rk[r]) come
// precomputed from the host, so a round is two wide products and two
// three-way XORs.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const uint32_t (&rk)[10][2]) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = uint64_t(0xD2511F53u) * c.x;
    const uint64_t p1 = uint64_t(0xCD9E8D57u) * c.z;
    c = make_uint4(uint32_t(p1 >> 32) ^ c.y ^ rk[r][0], uint32_t(p1),
                   uint32_t(p0 >> 32) ^ c.w ^ rk[r][1], uint32_t(p0));
  }
  return c;
}

// 4×4 transpose of words across the four lanes of an aligned lane group:
// on entry lane m of the group holds a[0..3]; on exit it holds, in a[n], what
// lane n held in a[m].  Two butterfly stages (lane bit 1, then lane bit 0).
__device__ __forceinline__ void lane4_transpose(uint32_t a[4], int m) {
  {
    const bool h = (m >> 1) & 1;
    const uint32_t x0 = h ? a[0] : a[2], x1 = h ? a[1] : a[3];
    const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, 2);
    const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, 2);
    if (h) { a[0] = y0; a[1] = y1; } else { a[2] = y0; a[3] = y1; }
  }
  {
    const bool l = m & 1;
    const uint32_t x0 = l ? a[0] : a[1], x1 = l ? a[2] : a[3];
    const uint32_t y0 = __shfl_xor_sync(0xffffffffu, x0, 1);
    const uint32_t y1 = __shfl_xor_sync(0xffffffffu, x1, 1);
    if (l) { a[0] = y0; a[2] = y1; } else { a[1] = y0; a[3] = y1; }
  }
}

// 4×4 transpose of the bytes of w[0..3]: byte i of the result's word j is
// byte j of w[i].
__device__ __forceinline__ void byte4_transpose(uint32_t w[4]) {
  const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140), t1 = __byte_perm(w[0], w[1], 0x7362);
  const uint32_t t2 = __byte_perm(w[2], w[3], 0x5140), t3 = __byte_perm(w[2], w[3], 0x7362);
  w[0] = __byte_perm(t0, t2, 0x5410);
  w[1] = __byte_perm(t0, t2, 0x7632);
  w[2] = __byte_perm(t1, t3, 0x5410);
  w[3] = __byte_perm(t1, t3, 0x7632);
}

// Keep bytes (0xFF keep, 0x00 drop) of 16 consecutive key columns of this
// lane's query row (forward).  `row` is the lane's query row (the four lanes
// of the group hold rows 4·(row/4) + 0..3 in lane order) and `col0` the
// group's first column (a multiple of 16).  out[n] covers columns
// col0 + 4n .. col0 + 4n + 3, byte j ↔ column col0 + 4n + j.
__device__ __forceinline__ void keep16_row(const DropoutParams& d, int bh, int row, int col0,
                                           uint32_t out[4]) {
  const int m = row & 3;
  const uint4 w = philox4x32_10(make_uint4(uint32_t(col0 / 4 + m), uint32_t(row >> 2), uint32_t(bh),
                                           d.offset),
                                d.rk);
  out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;  // block m, word i ↔ row 4·rb + i
  lane4_transpose(out, m);  // out[n] = word m (this row) of block n
#pragma unroll
  for (int n = 0; n < 4; ++n) out[n] = __vcmpltu4(out[n], d.t4);
}

// Keep bytes of 16 consecutive query rows for this lane's key (backward).
// `key` is the lane's key (the group's lanes hold keys 4·(key/4) + 0..3 in
// lane order) and `row0` the group's first query row (a multiple of 16).
// out[n] covers rows row0 + 4n .. row0 + 4n + 3, byte i ↔ row row0 + 4n + i.
__device__ __forceinline__ void keep16_col(const DropoutParams& d, int bh, int key, int row0,
                                           uint32_t out[4]) {
  const int m = key & 3;
  const uint4 w = philox4x32_10(make_uint4(uint32_t(key >> 2), uint32_t(row0 / 4 + m), uint32_t(bh),
                                           d.offset),
                                d.rk);
  out[0] = w.x; out[1] = w.y; out[2] = w.z; out[3] = w.w;  // block m: word i ↔ row, byte j ↔ key
  byte4_transpose(out);      // out[j]: byte i ↔ row 4·rb + i, for key 4·cb + j
  lane4_transpose(out, m);   // out[n] = block n's word for this key
#pragma unroll
  for (int n = 0; n < 4; ++n) out[n] = __vcmpltu4(out[n], d.t4);
}

// Expand the keep bytes b and b+1 of `k` into a mask for a packed pair of
// 16-bit values (low half ↔ byte b).
__device__ __forceinline__ uint32_t keep_pair_mask(uint32_t k, int b) {
  return __byte_perm(k, 0, b == 0 ? 0x1100 : 0x3322);
}

// The keep byte b of `k` as a 32-bit all-ones / zero mask.
__device__ __forceinline__ uint32_t keep_word_mask(uint32_t k, int b) {
  return __byte_perm(k, 0, 0x1111u * uint32_t(b));
}

}  // namespace fa
