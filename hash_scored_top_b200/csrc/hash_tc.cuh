// Tensor-core hashing of bf16 keys with P = 8 hyperplanes per table (SOCKET
// technical summary, section 中核メカニズム：ソフト LSH, step 1; the hard-hash
// codes of the HATA digest, section 3, are the same computation with 16
// tables of 8). The projections of 16 keys on the 8 hyperplanes of one table
// are one chain of mma.sync m16n8k16 over the head dimension (bf16 products
// are exact, the sums are f32), so with P = 8 the sign pattern of a tile row
// is that key's bucket ID. The value norm is a float64 sum of squares rounded
// once to the nearest f16.
//
// The bulk kernel (prefill, 64-key units) and the append kernel (decode time,
// one CTA per key) issue the same MMA chain per table -- operand fragments
// filled from the same bf16 values, k steps in the same order, accumulator
// from zero -- and the MMA computes each output element from its own row and
// column only, so a key gets the same ID bytes either way.
#pragma once

#include "attend.cuh"
#include "hash_kernels.cuh"

namespace hst {

constexpr int HTC_TPW = 4;          // tables per warp (B fragments held in registers)
constexpr int HTC_KEYS = 64;        // keys per unit of the bulk kernel
constexpr int HTC_STAGES = 3;       // units in flight per CTA (cp.async ring)
constexpr int HTC_APPEND_THREADS = 256;

__host__ __device__ inline int htc_threads(int L) { return 32 * ((L + HTC_TPW - 1) / HTC_TPW); }

// Shared memory of the bulk kernel: per stage the unit's key rows [64][D + 8]
// bf16 (the 16-byte pad makes the ldmatrix rows conflict-free) and, when
// norms are wanted, its value rows [64][D]; then two ID-byte buffers
// [64][LPB] (the unit being computed and the one being written out).
__host__ __device__ inline size_t htc_stage_bytes(int D, bool values) {
  return (size_t)HTC_KEYS * (D + 8) * 2 + (values ? (size_t)HTC_KEYS * D * 2 : 0);
}
__host__ __device__ inline size_t htc_smem_bytes(int D, int L, bool values) {
  return HTC_STAGES * htc_stage_bytes(D, values) + 2 * (size_t)HTC_KEYS * ids_bytes_per_key(L);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Float64 norm of a value row held as D/8 chunks of 8 bf16, chunk j in lane
// j of a group of D/8 lanes: each lane sums its 8 squares in order, then the
// group adds by an xor tree. Every lane of the group returns the norm.
template <int D>
__device__ __forceinline__ double value_norm_chunks(uint4 chunk) {
  constexpr int CPR = D / 8;
  const uint32_t w[4] = {chunk.x, chunk.y, chunk.z, chunk.w};
  double ss = 0.0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const double lo = (double)bf16lo_to_f32(w[e]), hi = (double)bf16hi_to_f32(w[e]);
    ss = fma(lo, lo, ss);
    ss = fma(hi, hi, ss);
  }
#pragma unroll
  for (int o = CPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
  return sqrt(ss);
}

// Sign byte of one table from an m16n8 accumulator: lane (r, q) holds
// hyperplanes 2q, 2q + 1 of rows r (acc 0, 1) and r + 8 (acc 2, 3). Returns
// the byte of row r in .x and of row r + 8 in .y, on every lane.
__device__ __forceinline__ uint2 htc_sign_bytes(const float (&acc)[4]) {
  const int q = threadIdx.x & 3;
  uint32_t v0 = (acc[0] > 0.f ? 1u : 0u) << (2 * q) | (acc[1] > 0.f ? 1u : 0u) << (2 * q + 1);
  uint32_t v1 = (acc[2] > 0.f ? 1u : 0u) << (2 * q) | (acc[3] > 0.f ? 1u : 0u) << (2 * q + 1);
  v0 |= __shfl_xor_sync(FULL, v0, 1);
  v1 |= __shfl_xor_sync(FULL, v1, 1);
  v0 |= __shfl_xor_sync(FULL, v0, 2);
  v1 |= __shfl_xor_sync(FULL, v1, 2);
  return make_uint2(v0, v1);
}

// B fragments of table t for k step k: hyperplane row 8t + g, columns
// 16k + 2q (+1) and 16k + 8 + 2q (+1), as bf16 pairs.
__device__ __forceinline__ uint2 htc_b_frag(const __nv_bfloat16* __restrict__ R, int D, int t, int k) {
  const int lane = threadIdx.x & 31;
  const uint32_t* row = reinterpret_cast<const uint32_t*>(R + (size_t)(8 * t + (lane >> 2)) * D);
  return make_uint2(__ldg(row + 8 * k + (lane & 3)), __ldg(row + 8 * k + 4 + (lane & 3)));
}

// Bulk: keys [n_begin, n_begin + n_count) of every pair, in units of 64 keys
// aligned to multiples of 64 (a unit's keys outside the range are computed
// and not written; rows at or past Ncap are zero-filled). Persistent: CTA b
// takes units b, b + gridDim.x, ..., with HTC_STAGES units of keys (and
// values) in flight through cp.async. Warp w holds the B fragments of tables
// 4w .. 4w + 3 in registers for the whole kernel and runs them over the 4 row
// tiles of every unit; all warps then take the unit's value norms.
// Launch with htc_threads(L) threads and htc_smem_bytes(D, L, V != nullptr).
template <int D>
__global__ void __launch_bounds__(512, 1) hash_keys_tc_kernel(const HashParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  constexpr int KS = D / 16;                 // k steps
  constexpr int RW = D + 8;                  // padded key row, bf16 elements
  constexpr int CPR = D / 8;                 // 16-byte chunks per row
  const bool values = p.V != nullptr;
  const int LPB = ids_bytes_per_key(p.L);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane & 3, g = lane >> 2;
  const int nthreads = blockDim.x, nwarps = nthreads >> 5;
  const uint32_t stage_bytes = (uint32_t)htc_stage_bytes(D, values);
  const uint32_t smem0 = smem_u32(dyn);
  uint8_t* idsb0 = dyn + HTC_STAGES * stage_bytes;

  const int n_end = p.n_begin + p.n_count;
  const int u_begin = p.n_begin / HTC_KEYS, u_end = (n_end + HTC_KEYS - 1) / HTC_KEYS;
  const int units_per_pair = u_end - u_begin;
  const int total = p.pairs * units_per_pair;
  // first key of unit u (of its pair), or -1 past the end; the pair in *pair
  auto unit_key0 = [&](int u, int* pair) {
    if (u >= total) return -1;
    *pair = u / units_per_pair;
    return (u_begin + (u - *pair * units_per_pair)) * HTC_KEYS;
  };

  // cp.async copies of the unit at (pair, k0) into stage st
  auto issue = [&](int pair, int k0, int st) {
    if (k0 < 0) return;
    const size_t base = ((size_t)pair * p.Ncap + k0) * D;
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.K) + base;
    const uint32_t ks = smem0 + st * stage_bytes;
    for (int e = tid; e < HTC_KEYS * CPR; e += nthreads) {
      const int row = e / CPR, c = e % CPR;
      const bool ok = k0 + row < p.Ncap;
      cp_async16(ks + (uint32_t)(row * RW + 8 * c) * 2, ok ? kb + (size_t)row * D + 8 * c : kb, ok);
    }
    if (values) {
      const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(p.V) + base;
      const uint32_t vs = ks + HTC_KEYS * RW * 2;
      for (int e = tid; e < HTC_KEYS * CPR; e += nthreads) {
        const bool ok = k0 + e / CPR < p.Ncap;
        cp_async16(vs + (uint32_t)e * 16, ok ? vb + (size_t)e * 8 : vb, ok);
      }
    }
  };

  // ID bytes of the unit at (pair, k0) from buffer ib to global; clears ib
  auto write_out = [&](int pair, int k0, uint8_t* ib) {
    uint32_t* out = reinterpret_cast<uint32_t*>(p.ids + ((size_t)pair * p.Ncap + k0) * LPB);
    uint32_t* src = reinterpret_cast<uint32_t*>(ib);
    const bool whole = k0 >= p.n_begin && k0 + HTC_KEYS <= n_end;
    for (int e = tid; e < HTC_KEYS * LPB / 4; e += nthreads) {
      if (whole) {
        out[e] = src[e];
      } else {
        const int key = k0 + (4 * e) / LPB;
        if (key >= p.n_begin && key < n_end) out[e] = src[e];
      }
      src[e] = 0u;
    }
  };

  // the ring holds units i .. i + HTC_STAGES - 2 ahead of the loop (HTC_STAGES == 3)
  int pair_cur = 0, pair_n1 = 0, pair_n2 = 0, pair_prev = 0;
  int k0_cur = unit_key0(blockIdx.x, &pair_cur);
  int k0_n1 = unit_key0(blockIdx.x + gridDim.x, &pair_n1);
  int k0_prev = -1;
  issue(pair_cur, k0_cur, 0);
  cp_async_commit();
  issue(pair_n1, k0_n1, 1);
  cp_async_commit();
  for (int e = tid; e < 2 * HTC_KEYS * LPB / 4; e += nthreads) reinterpret_cast<uint32_t*>(idsb0)[e] = 0u;

  uint32_t bf[HTC_TPW][KS][2];
#pragma unroll
  for (int j = 0; j < HTC_TPW; ++j) {
    const int t = min(warp * HTC_TPW + j, p.L - 1);
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const uint2 b = htc_b_frag(p.R, D, t, k);
      bf[j][k][0] = b.x;
      bf[j][k][1] = b.y;
    }
  }
  const int ntab = min(HTC_TPW, p.L - warp * HTC_TPW);     // tables of this warp (>= 1)
  const uint32_t a_lane = (uint32_t)(((lane & 15) * RW + (lane >> 4) * 8) * 2);
  // this lane stores table 4w + q: its byte of key n sits at
  // off + ((t - off - n) mod S); S divides 64, so the key's offset in the unit decides
  const int t_mine = warp * HTC_TPW + q;
  const int pos_off = t_mine >= 32 ? 32 : 0;
  const int pos_mask = id_chunk_size(p.L, pos_off >> 5) - 1;
  const int pos_base = t_mine - pos_off - g;

  int i = 0;
  for (; k0_cur >= 0; ++i) {
    cp_async_wait<HTC_STAGES - 2>();
    __syncthreads();               // unit i landed for every thread; unit i - 1 fully consumed
    const int k0_n2 = unit_key0(blockIdx.x + (i + 2) * gridDim.x, &pair_n2);
    issue(pair_n2, k0_n2, (i + 2) % HTC_STAGES);
    cp_async_commit();
    if (k0_prev >= 0) write_out(pair_prev, k0_prev, idsb0 + ((i - 1) & 1) * HTC_KEYS * LPB);

    const uint32_t ks = smem0 + (i % HTC_STAGES) * stage_bytes;
    uint8_t* ib = idsb0 + (i & 1) * HTC_KEYS * LPB;
#pragma unroll 1
    for (int mt = 0; mt < HTC_KEYS / 16; ++mt) {
      float acc[HTC_TPW][4];
#pragma unroll
      for (int j = 0; j < HTC_TPW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      const uint32_t a_addr = ks + (uint32_t)(mt * 16 * RW * 2) + a_lane;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(a_addr + 32u * k, a0, a1, a2, a3);
#pragma unroll
        for (int j = 0; j < HTC_TPW; ++j)
          if (j < ntab) mma_bf16_16816(acc[j], a0, a1, a2, a3, bf[j][k][0], bf[j][k][1]);
      }
      // byte j of v0 / v1: the ID of table 4w + j for rows g / g + 8, after the
      // or-reduction over the 4 lanes of the row (each holds 2 hyperplanes)
      uint32_t v0 = 0u, v1 = 0u;
#pragma unroll
      for (int j = 0; j < HTC_TPW; ++j) {
        const uint32_t b = 1u << (8 * j + 2 * q);
        v0 |= (acc[j][0] > 0.f ? b : 0u) | (acc[j][1] > 0.f ? 2u * b : 0u);
        v1 |= (acc[j][2] > 0.f ? b : 0u) | (acc[j][3] > 0.f ? 2u * b : 0u);
      }
      v0 |= __shfl_xor_sync(FULL, v0, 1);
      v1 |= __shfl_xor_sync(FULL, v1, 1);
      v0 |= __shfl_xor_sync(FULL, v0, 2);
      v1 |= __shfl_xor_sync(FULL, v1, 2);
      if (q < ntab) {
        const int r0 = mt * 16 + g;
        ib[r0 * LPB + pos_off + ((pos_base - 16 * mt) & pos_mask)] = (uint8_t)(v0 >> (8 * q));
        ib[(r0 + 8) * LPB + pos_off + ((pos_base - 16 * mt - 8) & pos_mask)] = (uint8_t)(v1 >> (8 * q));
      }
    }
    if (values) {                  // value norms: a group of D/8 lanes per key
      const uint4* vs = reinterpret_cast<const uint4*>(dyn + (i % HTC_STAGES) * stage_bytes + HTC_KEYS * RW * 2);
      constexpr int KPW = 32 / CPR;
      for (int r = warp * KPW; r < HTC_KEYS; r += nwarps * KPW) {
        const int row = r + lane / CPR;
        const double nrm = value_norm_chunks<D>(vs[row * CPR + lane % CPR]);
        const int key = k0_cur + row;
        if (lane % CPR == 0 && key >= p.n_begin && key < n_end)
          p.norms[(size_t)pair_cur * p.Ncap + key] = __double2half(nrm);
      }
    }
    pair_prev = pair_cur;
    k0_prev = k0_cur;
    pair_cur = pair_n1;
    k0_cur = k0_n1;
    pair_n1 = pair_n2;
    k0_n1 = k0_n2;
  }
  cp_async_wait<0>();
  __syncthreads();
  if (k0_prev >= 0) write_out(pair_prev, k0_prev, idsb0 + ((i - 1) & 1) * HTC_KEYS * LPB);
}

// Append: one CTA of 256 threads per (pair, key) for a few keys per pair (a
// decode step appends one). The key is row 0 of the A operand (rows 1..15
// zero); warp w runs tables w, w + 8, ... with fragments loaded straight from
// global memory, and the last warp takes the value norm with the bulk
// kernel's lane grouping. A selection kernel launched after this one as its
// programmatic dependent may start at once: it waits (griddepcontrol.wait)
// before reading any bucket ID or norm and reads nothing else written here.
template <int D>
__global__ void __launch_bounds__(HTC_APPEND_THREADS) hash_keys_tc_append_kernel(const HashParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ __align__(16) uint8_t idsb[64];
  constexpr int KS = D / 16;
  constexpr int CPR = D / 8;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane & 3, g = lane >> 2;
  const int pair = blockIdx.x;
  const int key = p.n_begin + blockIdx.y;
  const int LPB = ids_bytes_per_key(p.L);
  const size_t row_off = ((size_t)pair * p.Ncap + key) * D;
  if (tid < 16) reinterpret_cast<uint32_t*>(idsb)[tid] = 0u;
  const uint32_t* krow = reinterpret_cast<const uint32_t*>(reinterpret_cast<const __nv_bfloat16*>(p.K) + row_off);
  uint32_t a0[KS], a2[KS];
#pragma unroll
  for (int k = 0; k < KS; ++k) {
    a0[k] = g == 0 ? __ldg(krow + 8 * k + q) : 0u;        // row 0, columns 16k + 2q, +1
    a2[k] = g == 0 ? __ldg(krow + 8 * k + 4 + q) : 0u;    // row 0, columns 16k + 8 + 2q, +1
  }
  __syncthreads();
  for (int t = warp; t < p.L; t += HTC_APPEND_THREADS / 32) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const uint2 b = htc_b_frag(p.R, D, t, k);
      mma_bf16_16816(acc, a0[k], 0u, a2[k], 0u, b.x, b.y);
    }
    const uint2 by = htc_sign_bytes(acc);
    if (lane == 0) idsb[id_byte_pos(p.L, t, key)] = (uint8_t)by.x;
  }
  if (p.V && warp == HTC_APPEND_THREADS / 32 - 1) {
    const uint4* vrow = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.V) + row_off);
    const double nrm = value_norm_chunks<D>(lane < CPR ? __ldg(vrow + lane) : make_uint4(0u, 0u, 0u, 0u));
    if (lane == 0) p.norms[(size_t)pair * p.Ncap + key] = __double2half(nrm);
  }
  __syncthreads();
  if (tid < LPB) p.ids[((size_t)pair * p.Ncap + key) * LPB + tid] = idsb[tid];
}

}  // namespace hst
