// Prefill hashing, SOCKET step 1 (SOCKET technical summary, section
// 中核メカニズム：ソフト LSH, step 1: keys are hashed into L tables by random
// projections, one bucket ID per table, and the value norm is cached), and the
// 128-bit sign codes of the hard-hash variant (HATA digest, section 3), which
// are the same computation with 16 "tables" of 8 hyperplanes.
//
// This file holds the SIMT kernel (f32 projections, any key dtype). The
// tensor-core kernel for bf16 keys is in hash_tc.cuh.
//
// Bit j of the ID of table l is [k . r_{l*P+j} > 0]; IDs are written in the
// rotated key-major layout of common.cuh (ids_bytes_per_key bytes per key).
// The value norm is accumulated in float64 and rounded once to the nearest
// f16 (ties to even).
#pragma once

#include "common.cuh"
#include "table.cuh"

namespace hst {

struct HashParams {
  const void* K;
  const void* V;           // nullptr: no norms (hard-hash codes)
  const __nv_bfloat16* R;  // [L*P][d]
  uint8_t* ids;
  __half* norms;
  int Hkv, Ncap, n_begin, n_count, d, L, P;
  int pairs;
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

constexpr int HASH_THREADS = 256;

// Shared memory: R as bf16 [d][LP] (dim-major) + one key tile f32 [32][d] +
// sign masks [LP] u32.
template <typename KVT>
__global__ void __launch_bounds__(HASH_THREADS) hash_keys_simt_kernel(const HashParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int LP = p.L * p.P;
  const int d = p.d;
  __nv_bfloat16* Rs = reinterpret_cast<__nv_bfloat16*>(dyn);                  // [d][LP]
  float* Ks = reinterpret_cast<float*>(dyn + (((size_t)d * LP * 2 + 15) & ~(size_t)15));  // [32][d]
  uint32_t* bits = reinterpret_cast<uint32_t*>(Ks + 32 * d);                  // [LP]
  for (int e = threadIdx.x; e < LP * d; e += blockDim.x) {
    const int m = e / d, c = e % d;
    Rs[c * LP + m] = p.R[e];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int first_blk = p.n_begin / 32;
  const int last_blk = (p.n_begin + p.n_count - 1) / 32;
  const int nblk = last_blk - first_blk + 1;
  const long total = (long)p.pairs * nblk;
  for (long unit = blockIdx.x; unit < total; unit += gridDim.x) {
    const int pair = (int)(unit / nblk);
    const int blk = first_blk + (int)(unit % nblk);
    const size_t pair_keys = (size_t)pair * p.Ncap;
    const KVT* Kb = reinterpret_cast<const KVT*>(p.K) + (pair_keys + (size_t)blk * 32) * d;
    for (int e = threadIdx.x; e < 32 * d; e += blockDim.x) Ks[e] = to_f32(Kb[e]);
    __syncthreads();
    // sign masks: thread handles projection m, all 32 keys of the block
    for (int m = threadIdx.x; m < LP; m += blockDim.x) {
      uint32_t mask = 0;
      for (int n = 0; n < 32; ++n) {
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(Ks[n * d + c], __bfloat162float(Rs[c * LP + m]), acc);
        mask |= (acc > 0.f ? 1u : 0u) << n;
      }
      bits[m] = mask;
    }
    __syncthreads();
    // IDs in the rotated key-major layout: byte b of key n holds table
    // id_byte_table(L, b, n); keys in range only
    const int LPB = ids_bytes_per_key(p.L);
    uint8_t* ids_blk = p.ids + (pair_keys + (size_t)blk * 32) * LPB;
    for (int e = threadIdx.x; e < LPB * 32; e += blockDim.x) {
      const int n = e / LPB, bpos = e % LPB;
      const int key = blk * 32 + n;
      if (key >= p.n_begin && key < p.n_begin + p.n_count) {
        const int l = id_byte_table(p.L, bpos, key);
        uint32_t id = 0;
        if (l < p.L)
          for (int j = 0; j < p.P; ++j) id |= ((bits[l * p.P + j] >> n) & 1u) << j;
        ids_blk[e] = (uint8_t)id;
      }
    }
    // value norms (f64 accumulate, one rounding to f16)
    if (p.V) {
      const KVT* Vb = reinterpret_cast<const KVT*>(p.V) + (pair_keys + (size_t)blk * 32) * d;
      for (int n = warp; n < 32; n += nw) {
        const int key = blk * 32 + n;
        double ss = 0.0;
        for (int c = lane; c < d; c += 32) {
          const double v = (double)to_f32(Vb[(size_t)n * d + c]);
          ss = fma(v, v, ss);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
        if (lane == 0 && key >= p.n_begin && key < p.n_begin + p.n_count)
          p.norms[pair_keys + key] = __double2half(sqrt(ss));
      }
    }
    __syncthreads();
  }
}

// Append path: one CTA of L*P threads per (pair, key) for a few keys (a decode
// step appends one token). Thread m forms projection m with the same f32 FMA
// sequence as hash_keys_simt_kernel (c = 0..d-1), so both paths give
// identical IDs; the norm is the same float64 reduction.
template <typename KVT>
__global__ void __launch_bounds__(512) hash_keys_append_kernel(const HashParams p) {
  __shared__ float ks[128];
  __shared__ uint32_t bits[16];       // 512 projection signs
  // launched as the programmatic dependent of the kernel that copies this
  // step's query and key/value rows in, wait for it first (a no-op for an
  // ordinary launch): the selection started below reads the query at once
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // a selection kernel launched after this one as its programmatic dependent
  // may start now: it waits (griddepcontrol.wait) before reading any bucket
  // ID or norm, and reads nothing else this kernel writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int pair = blockIdx.x;
  const int key = p.n_begin + blockIdx.y;
  const int d = p.d, LP = p.L * p.P;
  const size_t pair_keys = (size_t)pair * p.Ncap;
  const KVT* krow = reinterpret_cast<const KVT*>(p.K) + (pair_keys + key) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) ks[c] = to_f32(krow[c]);
  if (threadIdx.x < 16) bits[threadIdx.x] = 0u;
  __syncthreads();
  const int m = threadIdx.x;
  bool bit = false;
  if (m < LP) {
    const uint4* r = reinterpret_cast<const uint4*>(p.R + (size_t)m * d);
    float acc = 0.f;
    for (int c8 = 0; c8 < d / 8; ++c8) {
      const uint4 w = __ldg(r + c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc = fmaf(ks[8 * c8 + 2 * e], bf16lo_to_f32(ws[e]), acc);
        acc = fmaf(ks[8 * c8 + 2 * e + 1], bf16hi_to_f32(ws[e]), acc);
      }
    }
    bit = acc > 0.f;
  }
  const uint32_t mask = __ballot_sync(FULL, bit);
  if ((threadIdx.x & 31) == 0 && threadIdx.x < LP) bits[threadIdx.x >> 5] = mask;
  __syncthreads();
  const int LPB = ids_bytes_per_key(p.L);
  if (threadIdx.x < LPB) {
    const int bpos = threadIdx.x;
    const int l = id_byte_table(p.L, bpos, key);
    uint32_t id = 0;
    if (l < p.L) {
      for (int j = 0; j < p.P; ++j) {
        const int mm = l * p.P + j;
        id |= ((bits[mm >> 5] >> (mm & 31)) & 1u) << j;
      }
    }
    p.ids[(pair_keys + key) * LPB + bpos] = (uint8_t)id;
  }
  if (p.V && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const KVT* vrow = reinterpret_cast<const KVT*>(p.V) + (pair_keys + key) * d;
    double ss = 0.0;
    for (int c = lane; c < d; c += 32) {
      const double v = (double)to_f32(vrow[c]);
      ss = fma(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    if (lane == 0) p.norms[pair_keys + key] = __double2half(sqrt(ss));
  }
}

// ---------------------------------------------------------------- hard-hash tables
// Table of the hard-hash decode: for code byte m and byte value x,
//   U_m(x) = sum_h (8 - popcount(x ^ qcode_h[m])),
// so that sum_m U_m(code_n[m]) = sum_h (128 - Hamming(qcode_h, code_n)).
// The query codes use float64 projections (sign of q_h . r_c). Computes the
// bytes m in [m0, m0 + nm); scratch holds hamming_scratch_bytes.
__host__ __device__ inline size_t hamming_scratch_bytes(int G, int d, int nm) {
  return (size_t)G * (d + 8) * 8 + (size_t)G * 16 * 4 + (size_t)nm * 8 * d * 2;
}

template <int D, typename QT, typename Store, typename Hook = NoHook>
__device__ void build_hamming_table(const QT* __restrict__ Qg, int G, const __nv_bfloat16* __restrict__ R128,
                                    int m0, int nm, void* scratch, Store store, Hook before_store = Hook()) {
  const int tid = threadIdx.x;
  double* qd = reinterpret_cast<double*>(scratch);                 // G padded rows (not normalised: the sign is enough)
  uint32_t* qbyte = reinterpret_cast<uint32_t*>(qd + G * qpad_row<D>());  // [G][16]
  __nv_bfloat16* rs = reinterpret_cast<__nv_bfloat16*>(qbyte + G * 16);   // [8 nm][D]
  for (int i = tid; i < G * D; i += blockDim.x) qd[qpad_index<D>(i / D, i % D)] = (double)to_f32(Qg[i]);
  for (int i = tid; i < G * 16; i += blockDim.x) qbyte[i] = 0u;
  stage_rows<D>(R128, 8 * m0, 8 * nm, rs);
  __syncthreads();
  project_rows_mma<D>(qd, G, rs, 8 * nm, [&](int item, double z) {
    const int h = item / (8 * nm), mi = item % (8 * nm);
    if (z > 0.0) atomicOr(&qbyte[h * 16 + m0 + mi / 8], 1u << (mi % 8));
  });
  __syncthreads();
  before_store();
  for (int item = tid; item < 256 * nm; item += blockDim.x) {
    const int x = item % 256;
    const int m = m0 + item / 256;
    int u = 0;
    for (int h = 0; h < G; ++h) u += 8 - __popc((uint32_t)x ^ qbyte[h * 16 + m]);
    store(x, m, (float)u);
  }
  __syncthreads();
}

}  // namespace hst
