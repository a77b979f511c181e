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
// key-block interleaved layout (per 32-key block, table l's 32 IDs are 32
// contiguous bytes). The value norm is accumulated in float64 and rounded
// once to the nearest f16 (ties to even).
#pragma once

#include "common.cuh"

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
    // IDs: item (l, n) -> byte at blk*32*L + l*32 + n, keys in range only
    uint8_t* ids_blk = p.ids + (pair_keys + (size_t)blk * 32) * p.L;
    for (int e = threadIdx.x; e < p.L * 32; e += blockDim.x) {
      const int l = e / 32, n = e % 32;
      const int key = blk * 32 + n;
      if (key >= p.n_begin && key < p.n_begin + p.n_count) {
        uint32_t id = 0;
        for (int j = 0; j < p.P; ++j) id |= ((bits[l * p.P + j] >> n) & 1u) << j;
        ids_blk[l * 32 + n] = (uint8_t)id;
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

// ---------------------------------------------------------------- hard-hash tables
// Table of the hard-hash decode: for code byte m and byte value x,
//   U_m(x) = sum_h (8 - popcount(x ^ qcode_h[m])),
// so that sum_m U_m(code_n[m]) = sum_h (128 - Hamming(qcode_h, code_n)).
// The query codes use float64 projections (sign of q_h . r_c).
template <typename QT, typename Store>
__device__ void build_hamming_table(const QT* __restrict__ Qg, int G, int d, const __nv_bfloat16* __restrict__ R128,
                                    int m_first, int m_step, uint32_t* qbyte /* smem [G][16] */, Store store) {
  const int tid = threadIdx.x;
  const int nm = (16 - m_first + m_step - 1) / m_step;      // code bytes handled here
  for (int i = tid; i < G * 16; i += blockDim.x) qbyte[i] = 0u;
  __syncthreads();
  for (int item = tid; item < G * nm * 8; item += blockDim.x) {
    const int j = item % 8;
    const int m = m_first + ((item / 8) % nm) * m_step;
    const int h = item / (8 * nm);
    const QT* q = Qg + (size_t)h * d;
    const __nv_bfloat16* r = R128 + (size_t)(8 * m + j) * d;
    double z = 0.0;
    for (int e = 0; e < d; ++e) z = fma((double)to_f32(q[e]), (double)__bfloat162float(r[e]), z);
    if (z > 0.0) atomicOr(&qbyte[h * 16 + m], 1u << j);
  }
  __syncthreads();
  for (int item = tid; item < 256 * nm; item += blockDim.x) {
    const int x = item % 256;
    const int m = m_first + (item / 256) * m_step;
    int u = 0;
    for (int h = 0; h < G; ++h) u += 8 - __popc((uint32_t)x ^ qbyte[h * 16 + m]);
    store(x, m, (float)u);
  }
  __syncthreads();
}

}  // namespace hst
