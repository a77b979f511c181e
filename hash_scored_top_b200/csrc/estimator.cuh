// The soft-count attention estimator of SOCKET (SOCKET technical summary,
// section 主要な貢献 item 4 and section 理論的基盤): over the selected keys
// S of a (batch, KV-head) pair, every query head h of the group gets
//   o_h = sum_{i in S} c_{h,i} v_i / sum_{i in S} c_{h,i},
//   c_{h,i} = sum_l p_{h,l}(id_l(i)),
// the soft collision count of key i under the head's own soft bucket
// assignment (the same float64 factors as the bucket tables, table.cuh).
// Only the selected keys' values and cached bucket IDs are read, not their
// keys.
//
// grid = (pairs, splits), EST_THREADS threads; CTA (pair, s) takes keys
// idx[s * keys_per_split ..]. Pass A, over chunks of lchunk tables: the
// heads' per-bit factors of the chunk, then every key's counts (lanes over
// tables, a fixed xor-tree sum over the lanes) added to a float64 count per
// (key, head) in shared memory. Pass B: warps over keys, lanes over value
// columns, f32 accumulation of c v and of c. The warps' partials are added in
// warp order; the splits' partials go to the workspace and the last CTA of the
// pair (counted with an atomic) adds them in split order and divides.
#pragma once

#include "hash_kernels.cuh"
#include "score.cuh"
#include "table.cuh"

namespace hst {

constexpr int EST_THREADS = 512;
constexpr int EST_WARPS = EST_THREADS / 32;
constexpr int EST_MAX_KEYS = 512;      // keys per CTA at most (their counts stay in shared memory)

struct EstParams {
  const void* Q;
  const void* V;
  const __nv_bfloat16* R;
  const uint8_t* ids;
  const int* idx;                // [pairs][k]
  float* part;                   // [pairs][splits][G][D + 1]: (sum c, sum c v) per head
  unsigned int* counters;        // [pairs], zero on entry, left zero
  float* O;                      // [B][Hq][D]
  int Hq, Hkv, Ncap, L, P, k, keys_per_split, splits, lchunk;
  float tau;
};

// Shared bytes: the factor scratch of one chunk (reused for the warps'
// partials), then the counts, then a flag word.
__host__ __device__ inline size_t est_region_a_bytes(int G, int d, int lchunk, int P) {
  const size_t f = table_scratch_dbl_bytes(G, d, lchunk, P);
  const size_t w = (size_t)EST_WARPS * G * (d + 1) * 4;
  return ((f > w ? f : w) + 15) & ~(size_t)15;
}
__host__ __device__ inline size_t est_smem_bytes(int G, int d, int lchunk, int P) {
  return est_region_a_bytes(G, d, lchunk, P) + (size_t)EST_MAX_KEYS * G * 8 + 16;
}

template <typename KVT>
__device__ __forceinline__ void load_row4(const KVT* row, int lane, float (&v)[4]);
template <>
__device__ __forceinline__ void load_row4<__nv_bfloat16>(const __nv_bfloat16* row, int lane, float (&v)[4]) {
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(row) + lane);
  v[0] = bf16lo_to_f32(w.x);
  v[1] = bf16hi_to_f32(w.x);
  v[2] = bf16lo_to_f32(w.y);
  v[3] = bf16hi_to_f32(w.y);
}
template <>
__device__ __forceinline__ void load_row4<float>(const float* row, int lane, float (&v)[4]) {
  const float4 w = __ldg(reinterpret_cast<const float4*>(row) + lane);
  v[0] = w.x;
  v[1] = w.y;
  v[2] = w.z;
  v[3] = w.w;
}

template <int D, typename KVT>
__global__ void __launch_bounds__(EST_THREADS, 1) soft_count_attend_kernel(const EstParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int VPL = D / 32;                        // value columns per lane (2 or 4)
  const int pair = blockIdx.x, split = blockIdx.y;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = split * p.keys_per_split;
  const int cnt = max(0, min(p.k - i0, p.keys_per_split));
  const size_t pair_keys = (size_t)pair * p.Ncap;
  const KVT* Qg = reinterpret_cast<const KVT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  const int* list = p.idx + (size_t)pair * p.k + i0;
  const int LPB = ids_bytes_per_key(p.L);
  const size_t dbl = est_region_a_bytes(G, D, p.lchunk, p.P);
  double* cnts = reinterpret_cast<double*>(smem + dbl);      // [cnt][G]
  unsigned int* last_flag = reinterpret_cast<unsigned int*>(smem + dbl + (size_t)EST_MAX_KEYS * G * 8);
  for (int e = tid; e < cnt * G; e += EST_THREADS) cnts[e] = 0.0;

  // ---- pass A: counts, table chunk by table chunk
  for (int l0 = 0; l0 < p.L; l0 += p.lchunk) {
    const int nl = min(p.lchunk, p.L - l0);
    const BucketFactors bf = bucket_factors<D, KVT>(Qg, G, p.R, p.P, p.tau, l0, nl, smem, nullptr, nullptr, true);
    for (int j = warp; j < cnt; j += EST_WARPS) {
      const int key = min(max(__ldg(list + j), 0), p.Ncap - 1);
      const uint8_t* idrow = p.ids + (pair_keys + key) * LPB;
      // lane t: table l0 + t (and l0 + t + 32)
      int idv[2] = {0, 0};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int li = lane + 32 * r;
        if (li < nl) idv[r] = idrow[id_byte_pos(p.L, l0 + li, key)];
      }
      for (int h = 0; h < G; ++h) {
        double c = 0.0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int li = lane + 32 * r;
          if (li < nl) {
            const int hl = h * nl + li;
            c += bf.lo[hl * bf.slo + (idv[r] & (bf.nlo - 1))] * bf.hi[hl * bf.shi + (idv[r] >> bf.plo)];
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(FULL, c, o);
        if (lane == 0) cnts[j * G + h] += c;
      }
    }
    __syncthreads();         // the factor scratch is reused by the next chunk
  }

  // ---- pass B: sum c v and sum c per head, warps over keys, lanes over columns
  float acc[8][VPL];
  float csum[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    csum[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[h][e] = 0.f;
  }
  for (int j = warp; j < cnt; j += EST_WARPS) {
    const int key = min(max(__ldg(list + j), 0), p.Ncap - 1);
    const KVT* vrow = reinterpret_cast<const KVT*>(p.V) + (pair_keys + key) * D;
    float v[4];
    if constexpr (VPL == 4) {
      load_row4<KVT>(vrow, lane, v);
    } else {
      const float a0 = to_f32(vrow[2 * lane]), a1 = to_f32(vrow[2 * lane + 1]);
      v[0] = a0;
      v[1] = a1;
      v[2] = v[3] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < G) {
        const float c = (float)cnts[j * G + h];
        csum[h] += c;
#pragma unroll
        for (int e = 0; e < VPL; ++e) acc[h][e] = fmaf(c, v[e], acc[h][e]);
      }
    }
  }
  __syncthreads();
  // warp partials into the (dead) factor scratch: [warp][G][D + 1]
  float* wp = reinterpret_cast<float*>(smem);
  const int stride = G * (D + 1);
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < G) {
      if (lane == 0) wp[warp * stride + h * (D + 1)] = csum[h];
#pragma unroll
      for (int e = 0; e < VPL; ++e) wp[warp * stride + h * (D + 1) + 1 + VPL * lane + e] = acc[h][e];
    }
  }
  __syncthreads();
  float* mine = p.part + ((size_t)pair * p.splits + split) * stride;
  for (int e = tid; e < stride; e += EST_THREADS) {
    float t = 0.f;
    for (int w = 0; w < EST_WARPS; ++w) t += wp[w * stride + e];
    mine[e] = t;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) *last_flag = (atomicAdd(&p.counters[pair], 1u) == (unsigned)p.splits - 1u) ? 1u : 0u;
  __syncthreads();
  if (*last_flag == 0u) return;
  // ---- last CTA of the pair: splits in order, then the division
  __threadfence();
  const float* part = p.part + (size_t)pair * p.splits * stride;
  for (int e = tid; e < G * D; e += EST_THREADS) {
    const int h = e / D, dv = e % D;
    float cs = 0.f, o = 0.f;
    for (int s = 0; s < p.splits; ++s) {
      cs += __ldcg(part + (size_t)s * stride + h * (D + 1));
      o += __ldcg(part + (size_t)s * stride + h * (D + 1) + 1 + dv);
    }
    p.O[((size_t)b * p.Hq + kvh * G + h) * D + dv] = o / cs;
  }
  if (tid == 0) p.counters[pair] = 0u;
}

}  // namespace hst
