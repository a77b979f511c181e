// Soft collision scoring, SOCKET step 3 (SOCKET technical summary, section
// 中核メカニズム：ソフト LSH, step 3): score_n = |v_n| * sum_l T_l(id_l(n)).
//
// Work unit: one lane scores one key; a warp scores 32 consecutive keys.
// Lane t loads its key's LP ID bytes (the rotated key-major layout of
// common.cuh) with 16-byte loads; a warp reads 32 * LP contiguous bytes.
// At step j the byte the lane reads belongs to table 32c + (j + t) mod S_c
// (t = key index mod 32), so the 32 lanes look up 32 different tables.
//
// Shared-memory tables: one per ID chunk, 64 KB each at a 64 KB-aligned
// shared address; row b (bucket) at byte b*256, column x at 4x, and column x
// holds table 32c + (x mod S_c) -- every table appears 64 / S_c times. Lane t
// at step j reads column t + j (< 64), whose bank is (t + j) mod 32: the 32
// lookups of a warp hit 32 banks. The address is the lane's column-0 address
// with byte 1 replaced by the ID (one byte-permute) plus the compile-time
// offset 4j in the load instruction. Rows >= 2^P and tables >= L hold zero.
//
// The LP values of a key go to 8 (16 for LP = 64) partial sums of at most 6
// (4 for LP = 64) terms that are added in a fixed tree, so an f32 score of
// non-negative terms carries at most 10 roundings of 2^-24 (entry, sums, norm
// product) -- below the 1e-6 relative near-tie window of the selection.
#pragma once

#include "common.cuh"

namespace hst {

constexpr int TABLE_BYTES = 65536;     // 256 buckets x 64 columns x 4 bytes
constexpr int TABLE_COLS = 64;

template <int LP>
struct KeyIds {
  uint4 w[LP / 16];
  uint16_t norm;
};

// One key's IDs (and norm). Key rows of 32 and 64 bytes are read with 32-byte
// loads, so each request of a warp covers whole 32-byte sectors; 16- and
// 48-byte rows with 16-byte loads. ids_key is aligned to its row size's
// largest power-of-two divisor (up to 32 bytes).
template <int LP, bool NORM>
__device__ __forceinline__ void load_key_ids(KeyIds<LP>& k, const uint8_t* __restrict__ ids_key,
                                             const __half* __restrict__ norm_key) {
  if constexpr (LP % 32 == 0) {
#pragma unroll
    for (int i = 0; i < LP / 32; ++i) ldg_stream32(ids_key + 32 * i, k.w[2 * i], k.w[2 * i + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < LP / 16; ++i) k.w[i] = ldg_stream(ids_key + 16 * i);
  }
  if (NORM) k.norm = ldg_u16(norm_key);
}

template <int J>
__device__ __forceinline__ float lds_imm(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(4 * J));
  return v;
}

// Number of partial sums (more would spill registers at 48-byte rows).
template <int LP>
struct ScoreAcc {
  static constexpr int N = LP > 48 ? 16 : 8;
};

template <int LP, int J>
struct ScoreStep {
  // Looks up byte J of the key (unrolled over J by recursion).
  static __device__ __forceinline__ void run(const KeyIds<LP>& k, uint32_t col0, uint32_t col1,
                                             float (&acc)[ScoreAcc<LP>::N]) {
    constexpr int NA = ScoreAcc<LP>::N;
    constexpr int C = J >= 32 ? 1 : 0;
    constexpr int JL = J - 32 * C;
    const uint4& q = k.w[J / 16];
    constexpr int E = (J / 4) % 4;
    const uint32_t w = E == 0 ? q.x : E == 1 ? q.y : E == 2 ? q.z : q.w;
    const uint32_t a = __byte_perm(C ? col1 : col0, w, 0x3240u | ((uint32_t)(J & 3) << 4));
    const float v = lds_imm<JL>(a);
    if (J < NA) acc[J % NA] = v;
    else acc[J % NA] += v;
    ScoreStep<LP, J + 1>::run(k, col0, col1, acc);
  }
};
template <int LP>
struct ScoreStep<LP, LP> {
  static __device__ __forceinline__ void run(const KeyIds<LP>&, uint32_t, uint32_t, float (&)[ScoreAcc<LP>::N]) {}
};

// Score (f32, >= 0) of this lane's key. colX = shared address of column
// `lane` (row 0) of the table of chunk X.
template <int LP, bool NORM>
__device__ __forceinline__ float score_key(const KeyIds<LP>& k, uint32_t col0, uint32_t col1) {
  constexpr int NA = ScoreAcc<LP>::N;
  float acc[NA];
  ScoreStep<LP, 0>::run(k, col0, col1, acc);
#pragma unroll
  for (int w = NA / 2; w >= 1; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) acc[i] = acc[2 * i] + acc[2 * i + 1];
  const float mass = acc[0];
  if (!NORM) return mass;    // hard-hash scores: exact small integers
  const float s = __half2float(__ushort_as_half(k.norm)) * mass;
  return fmaxf(s, 0.0f);     // scores are >= 0; NaN (0 * inf) maps to 0
}

// Column x of chunk c's table holds table 32c + (x mod S_c).
__host__ __device__ inline int column_table(int L, int c, int x) { return 32 * c + x % id_chunk_size(L, c); }

}  // namespace hst
