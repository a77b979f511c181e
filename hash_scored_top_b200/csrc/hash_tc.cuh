// Tensor-core hashing of bf16 keys with P = 8 hyperplanes per table (SOCKET
// technical summary, section 中核メカニズム：ソフト LSH, step 1; the hard-hash
// codes of the HATA digest, section 3, are the same computation with 16
// tables of 8). For a tile of 128 keys the projections K_tile . R^T are one
// tcgen05 MMA chain over the head dimension (M = 128 keys, N = the
// hyperplanes, bf16 operands in shared memory, f32 accumulators in tensor
// memory). With P = 8, columns 8l .. 8l + 7 of a key's row are table l's
// hyperplanes, so the key's ID bytes are the sign bits of its row taken 8 at a
// time. The value norm is a float64 sum of squares rounded once to the nearest
// f16.
//
// The kernel hashes key ranges of more than a few keys (prefill); the
// decode-time append of a few keys per pair stays on the SIMT append kernel,
// whose latency hides behind the selection kernel that follows it. The two
// sum the f32 projection in different orders, so a key's sign bit can differ
// between them only where its projection is within f32 rounding of zero.
//
// Thread roles (256 threads): warps 0-3 decode the accumulators -- warp w
// owns tensor-memory lanes 32w .. 32w + 31, i.e. rows 32w .. 32w + 31 of the
// tile, one key per thread. Warps 4-7 take the value norms (row m in thread
// 128 + m); thread 128 also issues the tile loads and the MMAs. Bulk tiles
// arrive by TMA tensor copies into rings of key and value stages (128-byte
// swizzle). When two accumulator buffers fit in tensor memory (8L <= 256),
// the MMAs of tile i + 1 run while tile i is decoded.
#pragma once

#include <cuda.h>

#include "hash_kernels.cuh"

namespace hst {

constexpr int TC_M = 128;               // keys per tile = MMA M = tensor-memory lanes used
constexpr int TC_THREADS = 256;
constexpr int TC_MAX_KSTAGES = 4;
constexpr int TC_VSTAGES = 2;
constexpr int TC_SMEM_MAX = 232448;     // dynamic shared memory of one CTA at most
constexpr int TC_SMEM_SM = 233472;      // shared memory of one SM
constexpr uint32_t TC_ATOM = TC_M * 128;  // one 128-row x 128-byte swizzle column of a tile

// Shared-memory plan (host and device compute the same one). Operands are
// K-major with the 128-byte swizzle: a matrix of r rows x d bf16 is d / 64
// column atoms of r rows x 128 bytes (atom a at a * r * 128), row n at n * 128
// inside the atom, its 16-byte chunk c at ((c ^ n) & 7) * 16.
//  R      [npad rows][d]; rows >= 8L are zero
//  K ring kstages x [128 rows][d]
//  V ring vstages x [128 rows][d] (0 stages without norms)
//  ctl    mbarriers fullK[4], fullV[2], mma[2], R (8 B each); tensor-memory
//         base address (4 B); failure flag (4 B)
// ahead = 1: two accumulator buffers, the MMAs of tile i + 1 are issued while
// tile i is decoded (needs 2 * ncols <= 512 and 3 key stages).
struct TcPlan {
  int npad, ncols, kstages, vstages, ahead;
  uint32_t r_off, k_off, v_off, tile_bytes, ctl_off, smem;
};

__host__ __device__ inline TcPlan tc_plan(int d, int L, bool values) {
  TcPlan p;
  p.npad = (8 * L + 31) / 32 * 32;
  p.ncols = 32;
  while (p.ncols < p.npad) p.ncols *= 2;
  p.tile_bytes = (uint32_t)TC_M * d * 2;
  p.r_off = 0;
  p.k_off = (uint32_t)p.npad * d * 2;
  p.vstages = values ? TC_VSTAGES : 0;
  const uint32_t room = (uint32_t)TC_SMEM_MAX - p.k_off - 128 - (uint32_t)p.vstages * p.tile_bytes;
  p.kstages = (int)(room / p.tile_bytes);
  if (p.kstages > TC_MAX_KSTAGES) p.kstages = TC_MAX_KSTAGES;
  p.ahead = 2 * p.ncols <= 512 && p.kstages >= 3 ? 1 : 0;
  p.v_off = p.k_off + (uint32_t)p.kstages * p.tile_bytes;
  p.ctl_off = p.v_off + (uint32_t)p.vstages * p.tile_bytes;
  p.smem = p.ctl_off + 128;
  return p;
}

// ---------------------------------------------------------------- tcgen05 wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] . B[smem]^T, bf16 inputs, f32 accumulators.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives once on the mbarrier when every MMA this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}

// 32 (or 64) consecutive f32 columns of this thread's tensor-memory lane; the
// wait takes the registers as operands so that no use is scheduled before it.
#define HST_TMEM_LD32(addr, v)                                                                                   \
  asm volatile(                                                                                                  \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"            \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                 \
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),           \
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),     \
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),   \
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])    \
      : "r"(addr))
#define HST_TMEM_WAIT(v)                                                                                         \
  asm volatile("tcgen05.wait::ld.sync.aligned;"                                                                  \
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),  \
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),         \
                 "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),       \
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),       \
                 "+r"(v[29]), "+r"(v[30]), "+r"(v[31])                                                            \
               :                                                                                                 \
               : "memory")

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  HST_TMEM_LD32(taddr, v);
  HST_TMEM_WAIT(v);
}
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v)[32], uint32_t (&x)[32]) {
  HST_TMEM_LD32(taddr, v);
  HST_TMEM_LD32(taddr + 32u, x);
  HST_TMEM_WAIT(v);
  HST_TMEM_WAIT(x);
}

// Sign word of 32 accumulator columns: bit j = [column j > 0], four
// independent byte chains.
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&v)[32]) {
  uint32_t by[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t b = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) b |= (__uint_as_float(v[8 * q + k]) > 0.f ? 1u : 0u) << k;
    by[q] = b;
  }
  return by[0] | (by[1] << 8) | (by[2] << 16) | (by[3] << 24);
}

// Shared-memory operand descriptor, K-major, 128-byte swizzle: 8-row x
// 128-byte atoms (rows 128 bytes apart, atom start 1024-byte aligned), `sbo`
// bytes between 8-row groups; the k offset inside the atom is added to the
// start address; descriptor version 1, layout type 2.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (2ull << 61);
}
// 2-D TMA tensor copy (no multicast) of the box at (x, y) into shared memory,
// completing its bytes on the mbarrier.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}
// Instruction descriptor: f32 accumulators, bf16 A and B, both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TC_M >> 4) << 24);
}

// Rotates the 4*NW bytes of w so that byte j becomes input byte (j + r) mod 4NW.
template <int NW>
__device__ __forceinline__ void rotate_bytes(uint32_t (&w)[NW], int r) {
  const int rw = r >> 2;
#pragma unroll
  for (int s = 1; s < NW; s <<= 1) {
    uint32_t u[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) u[i] = (rw & s) ? w[(i + s) % NW] : w[i];
#pragma unroll
    for (int i = 0; i < NW; ++i) w[i] = u[i];
  }
  const uint32_t sh = 8u * (uint32_t)(r & 3);
  uint32_t u[NW];
#pragma unroll
  for (int i = 0; i < NW; ++i) u[i] = __funnelshift_r(w[i], w[(i + 1) % NW], sh);
#pragma unroll
  for (int i = 0; i < NW; ++i) w[i] = u[i];
}

// Float64 norm of row m of a value tile in the swizzled operand layout at
// vbase: chunk c's 8 squares are summed in order into p_c, then p is folded
// in halves (p_c += p_{c+h} for h = D/16, ..., 1), and the square root of p_0
// is returned.
template <int D>
__device__ __forceinline__ double value_norm_tile(uint32_t vbase, int m) {
  constexpr int CPR = D / 8;
  double p[CPR];
#pragma unroll
  for (int c = 0; c < CPR; ++c) {
    uint32_t w[4];
    const uint32_t a = vbase + (uint32_t)(c >> 3) * TC_ATOM + (uint32_t)m * 128u + (uint32_t)(((c ^ m) & 7) * 16);
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a));
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double lo = (double)bf16lo_to_f32(w[e]), hi = (double)bf16hi_to_f32(w[e]);
      s = fma(lo, lo, s);
      s = fma(hi, hi, s);
    }
    p[c] = s;
  }
#pragma unroll
  for (int h = CPR / 2; h > 0; h >>= 1)
#pragma unroll
    for (int c = 0; c < h; ++c) p[c] = p[c] + p[c + h];
  return sqrt(p[0]);
}

// Which keys the tiles hold: tile u covers keys key0 .. key0 + 127 of pair
// u / tiles_per_pair, key0 = (tile_key0 + u % tiles_per_pair) * 128.
struct TcRows {
  int tiles_per_pair;  // tiles covering [n_begin, n_begin + n_count) in one pair
  int tile_key0;       // first tile index (keys tile_key0 * 128 ..)
  int n_tiles;
};
struct TcTile {
  int pair, key0;
};
__device__ __forceinline__ TcTile tc_tile(const TcRows& tr, int u) {
  TcTile t;
  t.pair = u / tr.tiles_per_pair;
  t.key0 = (tr.tile_key0 + (u - t.pair * tr.tiles_per_pair)) * TC_M;
  return t;
}
// (pair, key) of row m; returns whether the key is one to write (inside
// [n_begin, n_begin + n_count)).
__device__ __forceinline__ bool tc_row(const HashParams& p, const TcTile& t, int m, int* pair, int* key) {
  *pair = t.pair;
  *key = t.key0 + m;
  return *key >= p.n_begin && *key < p.n_begin + p.n_count;
}

// Launch: TC_THREADS threads, tc_plan(...).smem bytes of dynamic shared
// memory, persistent over the tiles (CTA b takes tiles b, b + gridDim.x, ...).
// mapK / mapV: 2-D bf16 tensor maps of K and V as [pairs * Ncap rows][D],
// box 64 x 128, 128-byte swizzle (rows past the last pair read as zero).
// mapR: the hyperplanes [8L rows][D], box 64 x 32, 128-byte swizzle (rows
// past 8L read as zero).
// Limit (SM clocks) of the main loop's waits; the drain on the way out always
// waits up to kWaitLimit. Lowered only by the test hook sk_test_set_wait_limit.
__device__ long long g_tc_wait_limit = kWaitLimit;

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 1)
    hash_keys_tcgen05_kernel(const HashParams p, const TcRows tr, const __grid_constant__ CUtensorMap mapK,
                             const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapR) {
  // a selection kernel launched after this one as its programmatic dependent
  // may start now: it waits (griddepcontrol.wait) before reading any bucket
  // ID or norm, and reads nothing else this kernel writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(1024) unsigned char dyn[];
  constexpr int KS = D / 16;                 // MMA k steps
  constexpr int NATOM = D / 64;              // 128-byte column atoms per row
  const bool values = p.V != nullptr;
  const TcPlan pl = tc_plan(D, p.L, values);
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool decoder = tid < TC_M;
  const int m = tid & (TC_M - 1);            // this thread's row of every tile
  const int LPB = ids_bytes_per_key(p.L);
  const int SK = pl.kstages, SV = pl.vstages, A = pl.ahead;
  const int rn = pl.npad;                    // rows of R in shared memory
  const uint32_t s0 = smem_u32(dyn);
  constexpr uint32_t kTslot = 72, kFail = 76;   // control-block offsets after the 9 mbarriers
  const uint32_t fullK = s0 + pl.ctl_off, fullV = fullK + 32, mmab = fullK + 48, rbar = fullK + 64;
  const uint32_t tslot = fullK + kTslot;
  volatile int* fail = reinterpret_cast<volatile int*>(dyn + pl.ctl_off + kFail);
  const long long lim = g_tc_wait_limit;
  // thread 128's record of the ring positions it issued and saw complete, for
  // the drain on the way out (the loop stops early after a wait gave up)
  int k_issued = 0, k_seen = 0, v_issued = 0, v_seen = 0, m_issued = 0;
  bool r_seen = false;
  auto kstage = [&](int j) { return s0 + pl.k_off + (uint32_t)(j % SK) * pl.tile_bytes; };
  auto vstage = [&](int j) { return s0 + pl.v_off + (uint32_t)(j % (SV > 0 ? SV : 1)) * pl.tile_bytes; };

  if (warp == 0) {
    tmem_alloc(tslot, (uint32_t)pl.ncols * (A ? 2u : 1u));
    tmem_relinquish();
  }
  if (tid == TC_M) {
    for (int j = 0; j < 9; ++j) mbar_init(fullK + 8u * j, 1);
    *fail = 0;
    fence_mbar_init();
    // the hyperplanes, 32 rows x 64 columns per box, into the R operand layout
    mbar_arrive_expect_tx(rbar, (uint32_t)rn * D * 2u);
    for (int b = 0; b < rn / 32; ++b)
#pragma unroll
      for (int a = 0; a < NATOM; ++a)
        tma_load_2d(s0 + pl.r_off + (uint32_t)a * (uint32_t)rn * 128u + (uint32_t)b * 4096u, &mapR, 64 * a,
                    32 * b, rbar);
  }

  // thread 128: TMA copies of ring position j's keys (or values)
  auto tma_rows = [&](const CUtensorMap* map, int j, uint32_t dst, uint32_t bar) -> bool {
    const int u = (int)blockIdx.x + j * (int)gridDim.x;
    if (u >= tr.n_tiles) return false;
    const TcTile t = tc_tile(tr, u);
    const int row = t.pair * p.Ncap + t.key0;
    mbar_arrive_expect_tx(bar, pl.tile_bytes);
#pragma unroll
    for (int a = 0; a < NATOM; ++a) tma_load_2d(dst + (uint32_t)a * TC_ATOM, map, 64 * a, row, bar);
    return true;
  };
  auto tma_keys = [&](int j) {
    if (tma_rows(&mapK, j, kstage(j), fullK + 8u * (uint32_t)(j % SK))) k_issued = j + 1;
  };
  auto tma_values = [&](int j) {
    if (tma_rows(&mapV, j, vstage(j), fullV + 8u * (uint32_t)(j % SV))) v_issued = j + 1;
  };
  // accumulator buffer of ring position j, and the parity of its mbarrier phase
  auto buf_of = [&](int j) { return A ? (uint32_t)(j & 1) : 0u; };
  auto par_of = [&](int j) { return A ? (uint32_t)((j >> 1) & 1) : (uint32_t)(j & 1); };
  // thread 128: the MMAs of ring position j into accumulator buffer buf_of(j)
  bool r_ready = false;
  auto issue_mma = [&](int j, uint32_t tbase) {
    if (!r_ready) {
      if (!mbar_wait_bounded(rbar, 0u, lim)) {
        *fail = 1;
        return;                              // no MMA on operands that have not arrived
      }
      r_ready = r_seen = true;
    }
    tc_fence_after_sync();
    const uint32_t buf = buf_of(j);
    const uint32_t ks = kstage(j);
    for (int n0 = 0; n0 < rn; n0 += 256) {
      const int nn = min(256, rn - n0);
      const uint32_t idesc = umma_idesc_bf16(nn);
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        const uint32_t koff = (uint32_t)(s >> 2) * TC_ATOM + (uint32_t)(s & 3) * 32u;
        const uint32_t roff =
            (uint32_t)(s >> 2) * (uint32_t)rn * 128u + (uint32_t)n0 * 128u + (uint32_t)(s & 3) * 32u;
        tc_mma_bf16(tbase + buf * (uint32_t)pl.ncols + (uint32_t)n0, umma_desc_sw128(ks + koff, 1024u),
                    umma_desc_sw128(s0 + pl.r_off + roff, 1024u), idesc, s > 0 ? 1u : 0u);
      }
    }
    tc_commit(mmab + 8u * buf);
    m_issued = j + 1;
  };
  // the keys of ring position j have landed (else the loop stops; no MMA is
  // issued on them)
  auto wait_keys = [&](int j) -> bool {
    if (!mbar_wait_bounded(fullK + 8u * (uint32_t)(j % SK), (uint32_t)((j / SK) & 1), lim)) {
      *fail = 1;
      return false;
    }
    k_seen = j + 1;
    return true;
  };

  const int G = (int)gridDim.x;
  const int my_tiles = tr.n_tiles > (int)blockIdx.x ? (tr.n_tiles - 1 - (int)blockIdx.x) / G + 1 : 0;
  if (tid == TC_M) {
    for (int j = 0; j < SK - 1; ++j) tma_keys(j);
    for (int j = 0; j < SV - 1; ++j) tma_values(j);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(dyn + pl.ctl_off + kTslot);
  if (A && tid == TC_M && my_tiles > 0) {
    if (wait_keys(0)) issue_mma(0, tbase);
  }

  for (int i = 0; i < my_tiles; ++i) {
    const int u = (int)blockIdx.x + i * G;
    tc_fence_before_sync();                  // the decoded buffer's tensor-memory reads are done
    __syncthreads();                         // ... and tile i - 1's stages are consumed
    if (*fail) break;
    const TcTile t = tc_tile(tr, u);
    int pair, key;
    const bool mine = tc_row(p, t, m, &pair, &key);
    const size_t kidx = (size_t)pair * p.Ncap + key;

    if (!decoder) {
      if (tid == TC_M) {
        tma_keys(i + SK - 1);                // into the stages of tile i - 1
        if (SV > 0) tma_values(i + SV - 1);
        const int j = i + A;
        if (j < my_tiles && wait_keys(j)) issue_mma(j, tbase);
      }
      bool okv = true;
      if (SV > 0) {
        okv = mbar_wait_bounded(fullV + 8u * (uint32_t)(i % SV), (uint32_t)((i / SV) & 1), lim);
        if (!okv) *fail = 1;
        else if (tid == TC_M) v_seen = i + 1;
      }
      if (values && okv) {
        const double nrm = value_norm_tile<D>(vstage(i), m);
        if (mine) p.norms[kidx] = __double2half(nrm);
      }
    } else {
      // the row's signs: bit j of word b is column 32b + j, i.e. hyperplane
      // j % 8 of table 4b + j / 8; columns >= 8L are zero and give zero bits
      const uint32_t buf = buf_of(i);
      if (!mbar_wait_bounded(mmab + 8u * buf, par_of(i), lim)) {
        *fail = 1;                           // the accumulators are not ready: leave the row unwritten
        continue;
      }
      tc_fence_after_sync();
      const uint32_t ta = tbase + ((uint32_t)(32 * warp) << 16) + buf * (uint32_t)pl.ncols;
      uint32_t w[16];
#pragma unroll
      for (int b = 0; b < 16; ++b) w[b] = 0u;
#pragma unroll
      for (int b = 0; b < 16; b += 2) {
        if (32 * (b + 1) < rn) {
          uint32_t v[32], x[32];
          tmem_ld64(ta + (uint32_t)(32 * b), v, x);
          w[b] = sign_word(v);
          w[b + 1] = sign_word(x);
        } else if (32 * b < rn) {
          uint32_t v[32];
          tmem_ld32(ta + (uint32_t)(32 * b), v);
          w[b] = sign_word(v);
        }
      }
      if (mine) {
        // rotated layout: byte j of chunk c (tables 32c ..) of key n holds table 32c + (j + n) mod S_c
        uint4* out = reinterpret_cast<uint4*>(p.ids + kidx * LPB);
        if (LPB == 16) {
          uint32_t c0[4] = {w[0], w[1], w[2], w[3]};
          rotate_bytes<4>(c0, key & 15);
          out[0] = make_uint4(c0[0], c0[1], c0[2], c0[3]);
        } else {
          uint32_t c0[8] = {w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]};
          rotate_bytes<8>(c0, key & 31);
          out[0] = make_uint4(c0[0], c0[1], c0[2], c0[3]);
          out[1] = make_uint4(c0[4], c0[5], c0[6], c0[7]);
          if (LPB == 48) {
            uint32_t c1[4] = {w[8], w[9], w[10], w[11]};
            rotate_bytes<4>(c1, key & 15);
            out[2] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
          } else if (LPB == 64) {
            uint32_t c1[8] = {w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]};
            rotate_bytes<8>(c1, key & 31);
            out[2] = make_uint4(c1[0], c1[1], c1[2], c1[3]);
            out[3] = make_uint4(c1[4], c1[5], c1[6], c1[7]);
          }
        }
      }
    }
  }
  // Drain: everything thread 128 issued and did not see complete (after a
  // wait gave up, the loop stopped with copies and MMAs still in flight) is
  // waited for, up to the full limit each, before the tensor memory is freed
  // and the CTA's shared memory is released.
  if (tid == TC_M) {
    if (!r_seen) mbar_wait_bounded(rbar, 0u);
    for (int j = k_seen; j < k_issued; ++j) mbar_wait_bounded(fullK + 8u * (uint32_t)(j % SK), (uint32_t)((j / SK) & 1));
    for (int j = v_seen; j < v_issued; ++j) mbar_wait_bounded(fullV + 8u * (uint32_t)(j % SV), (uint32_t)((j / SV) & 1));
    for (int j = max(0, m_issued - (A ? 2 : 1)); j < m_issued; ++j) mbar_wait_bounded(mmab + 8u * buf_of(j), par_of(j));
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, (uint32_t)pl.ncols * (A ? 2u : 1u));
  }
}

}  // namespace hst
