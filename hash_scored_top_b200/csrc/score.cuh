// Soft collision scoring, SOCKET step 3 (SOCKET technical summary, section
// 中核メカニズム：ソフト LSH, step 3): score_n = |v_n| * sum_l T_l(id_l(n)).
//
// Work unit: one warp scores one block of 32 consecutive keys. The bucket
// IDs are stored key-block interleaved (per 32-key block, table l's 32 IDs
// are 32 contiguous bytes), so lane t loads the 32 IDs of table t of the block
// with two 16-byte loads -- a warp reads the block's L*32 bytes fully
// coalesced. Lane t then looks up T_t(id) for each of the 32 keys; all lanes
// read a different table column at every step, so the 32 lookups of a warp
// instruction fall in 32 different banks (conflict-free by construction).
//
// Shared-memory table layout: row b (bucket) at byte b*256, column l at l*4,
// 256 rows x 64 columns of f32 (64 KB), placed at a 64 KB-aligned shared
// address. The address of entry (id, column) is then the column's address
// with byte 1 replaced by the ID -- a single byte-permute per lookup.
// Rows >= 2^P and columns >= L hold zero, so any stored byte is a valid row.
//
// The 32 per-table values of a key live in 32 different lanes; a butterfly
// reduce-scatter (5 exchange rounds) leaves lane t with key t's sum. The sum
// is a fixed binary tree of depth 5 (6 with two table chunks), which bounds
// the f32 relative error of a score by 8 * 2^-24 (entry rounding, tree,
// product with the norm) -- below the 1e-6 near-tie window of the selection.
#pragma once

#include "common.cuh"

namespace hst {

constexpr int TABLE_BYTES = 65536;     // 256 buckets x 64 columns x 4 bytes
constexpr int TABLE_COLS = 64;

// Ids of one 32-key block for this lane: chunk c covers table 32c + lane.
template <int NCHUNK>
struct IdBlock {
  uint4 w[NCHUNK][2];
  uint16_t norm;
};

template <int NCHUNK, bool NORM = true>
__device__ __forceinline__ void load_id_block(IdBlock<NCHUNK>& blk, const uint8_t* __restrict__ ids_blk,
                                              const __half* __restrict__ norms_blk, int L, int lane) {
#pragma unroll
  for (int c = 0; c < NCHUNK; ++c) {
    const int l = 32 * c + lane;
    if (l < L) {
      const uint8_t* p = ids_blk + (size_t)l * 32;
      blk.w[c][0] = ldg_stream(p);
      blk.w[c][1] = ldg_stream(p + 16);
    } else {
      blk.w[c][0] = make_uint4(0, 0, 0, 0);
      blk.w[c][1] = make_uint4(0, 0, 0, 0);
    }
  }
  if (NORM) blk.norm = ldg_u16(norms_blk + lane);
}

__device__ __forceinline__ uint32_t word_of(const uint4 (&w)[2], int n) {
  const uint4& q = w[n >> 4];
  const int e = (n >> 2) & 3;
  return e == 0 ? q.x : e == 1 ? q.y : e == 2 ? q.z : q.w;
}

// Sum over lanes of v[n] lands in lane n (v[0] on return).
__device__ __forceinline__ float butterfly_reduce_scatter(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(FULL, send, s);
    }
  }
  return v[0];
}

// Score (f32, >= 0) of key (block start + lane). col_addr[c] is the shared
// address of table column 32c + lane in bucket row 0.
template <int NCHUNK, bool NORM = true>
__device__ __forceinline__ float score_id_block(const IdBlock<NCHUNK>& blk, const uint32_t (&col_addr)[NCHUNK],
                                                int lane) {
  float v[32];
#pragma unroll
  for (int c = 0; c < NCHUNK; ++c) {
#pragma unroll
    for (int n = 0; n < 32; ++n) {
      const uint32_t w = word_of(blk.w[c], n);
      const uint32_t addr = __byte_perm(col_addr[c], w, 0x3240u | ((uint32_t)(n & 3) << 4));
      const float t = lds_f32(addr);
      v[n] = (c == 0) ? t : v[n] + t;
    }
  }
  const float mass = butterfly_reduce_scatter(v, lane);
  if (!NORM) return mass;    // hard-hash scores: exact small integers
  const float s = __half2float(__ushort_as_half(blk.norm)) * mass;
  return fmaxf(s, 0.0f);     // scores are >= 0; NaN (0 * inf) maps to 0
}

}  // namespace hst
