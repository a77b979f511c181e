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
// Two kernels. est_factor_kernel, grid (pairs, table chunks): the per-bit
// factors of every head's soft assignment (the float64 lo / hi products of
// table.cuh, rounded to f32), written once per pair to a factor image in the
// workspace, F[pair][h][l][32] (lo at [0, 16), hi at [16, 32)).
// soft_count_attend_kernel, grid (pairs, splits), launched as the factor
// kernel's programmatic dependent: CTA (pair, s) takes keys
// idx[s * keys_per_split ..], and first issues asynchronous copies of all
// their value rows into shared memory (every copy of the CTA in flight at
// once), then, once the factor kernel is done, of the pair's factor image;
// each key's ID row is read into registers when its count is formed. Pass A, one thread per key: c_{h,i} summed over the tables in f32
// (all lanes of a warp read the same factor row, so the lookups do not
// conflict; f32: the counts feed an f32 weighted sum anyway, each is within
// (L + 2) 2^-24 of the exact one, and the f32 factor image is half the
// shared memory of a float64 one). Pass B: warps over keys,
// lanes over value
// columns, f32 accumulation of c v and of c. The warps' partials are added in
// warp order; the splits' partials go to the workspace and the last CTA of
// the pair (counted with an atomic) adds them in split order and divides.
#pragma once

#include "hash_kernels.cuh"
#include "hash_tc.cuh"
#include "score.cuh"
#include "table.cuh"

namespace hst {

constexpr int EST_THREADS = 256;
constexpr int EST_WARPS = EST_THREADS / 32;
constexpr int EST_F = 32;              // floats per (head, table) in the factor image
constexpr int EST_TABLES_PER_CTA = 4;  // tables per CTA of the factor kernel

struct EstFactorParams {
  const void* Q;
  const __nv_bfloat16* R;
  float* F;                      // [pairs][G][L][EST_F]
  int Hq, Hkv, L, P;
  float tau;
};

struct EstParams {
  const void* V;
  const uint8_t* ids;
  const int* idx;                // [pairs][k]
  const float* F;                // factor image
  float* part;                   // [pairs][splits][G][D + 1]: (sum c, sum c v) per head
  unsigned int* counters;        // [pairs], zero on entry, left zero
  float* O;                      // [B][Hq][D]
  unsigned long long* phase_ts;  // optional: [pairs * splits][24] clock stamps (profiling)
  int Hq, Hkv, Ncap, L, P, k, keys_per_split, splits;
};

// Profiling stamps of the attend kernel (see sk_profile_phases): the SM clock
// at each phase; the global timer at the start (slot 22) and the end (23).
__device__ __forceinline__ void est_stamp(unsigned long long* ts, int phase) {
  if (ts != nullptr && threadIdx.x == 0) {
    const size_t cta = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    ts[cta * 24 + phase] = (unsigned long long)clock64();
    if (phase == 0 || phase == 7) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      ts[cta * 24 + 22 + (phase == 7)] = t;
    }
  }
}

// Shared bytes of the factor kernel (bucket_factors with staged rows).
__host__ __device__ inline size_t est_factor_smem_bytes(int G, int d, int P) {
  return table_scratch_bytes(G, d, EST_TABLES_PER_CTA, P);
}

__host__ __device__ inline size_t est_align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Shared-memory plan of the attend kernel for `kps` keys per CTA: the factor
// image (reused for the warps' partials), the counts, the key indices, the
// staged ID rows and value rows, a flag word. Offsets in bytes.
struct EstSmem {
  size_t counts, keys, vrows, flag, total;
};
__host__ __device__ inline EstSmem est_smem_plan(int G, int d, int L, int kps, int kv_bytes) {
  EstSmem s;
  const size_t f = (size_t)G * L * EST_F * 4;
  const size_t w = (size_t)EST_WARPS * G * (d + 1) * 4;
  s.counts = est_align16(f > w ? f : w);
  s.keys = s.counts + est_align16((size_t)kps * G * 4);
  s.vrows = s.keys + est_align16((size_t)kps * 4);
  s.flag = s.vrows + (size_t)kps * d * kv_bytes;
  s.total = s.flag + 16;
  return s;
}
// Bytes of shared memory per key in the plan above (for the host's choice of kps).
__host__ __device__ inline size_t est_bytes_per_key(int G, int d, int L, int kv_bytes) {
  (void)L;
  return (size_t)G * 4 + 4 + (size_t)d * kv_bytes;
}

// The ID bytes of one key in table order: its rotated row (see common.cuh)
// loaded into registers and rotated back per chunk, so that byte l holds the
// ID of table l (a compile-time position in the unrolled loops below).
template <int LP>
struct KeyRowIds {
  uint32_t w[LP / 4];
};
template <int LP>
__device__ __forceinline__ void load_key_row_ids(KeyRowIds<LP>& r, const uint8_t* __restrict__ row, int key) {
#pragma unroll
  for (int i = 0; i < LP / 16; ++i) {
    const uint4 x = ldg_stream(row + 16 * i);
    r.w[4 * i] = x.x;
    r.w[4 * i + 1] = x.y;
    r.w[4 * i + 2] = x.z;
    r.w[4 * i + 3] = x.w;
  }
  // chunk 0: S = 16 (LP = 16) or 32; byte j holds table (j + key) mod S
  constexpr int S0 = LP == 16 ? 16 : 32;
  {
    uint32_t c[S0 / 4];
#pragma unroll
    for (int i = 0; i < S0 / 4; ++i) c[i] = r.w[i];
    rotate_bytes<S0 / 4>(c, (S0 - key % S0) % S0);
#pragma unroll
    for (int i = 0; i < S0 / 4; ++i) r.w[i] = c[i];
  }
  if constexpr (LP > 32) {
    constexpr int S1 = LP - 32;
    uint32_t c[S1 / 4];
#pragma unroll
    for (int i = 0; i < S1 / 4; ++i) c[i] = r.w[8 + i];
    rotate_bytes<S1 / 4>(c, (S1 - key % S1) % S1);
#pragma unroll
    for (int i = 0; i < S1 / 4; ++i) r.w[8 + i] = c[i];
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int D, typename QT>
__global__ void __launch_bounds__(256) est_factor_kernel(const EstFactorParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  // the attend kernel, launched as this kernel's programmatic dependent, may
  // start its copies now: it reads the factor image only after
  // griddepcontrol.wait, i.e. after this grid has completed
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int pair = blockIdx.x;
  const int l0 = blockIdx.y * EST_TABLES_PER_CTA;
  const int nl = min(EST_TABLES_PER_CTA, p.L - l0);
  if (nl <= 0) return;                         // uniform over the CTA
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const QT* Qg = reinterpret_cast<const QT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  const BucketFactors bf = bucket_factors<D, QT>(Qg, G, p.R, p.P, p.tau, l0, nl, smem);
  const int nhi = bf.shi - 1;
  float* F = p.F + (size_t)pair * G * p.L * EST_F;
  for (int e = threadIdx.x; e < G * nl * EST_F; e += blockDim.x) {
    const int hl = e / EST_F, j = e % EST_F;   // hl = h * nl + li
    const int h = hl / nl, li = hl % nl;
    double v = 0.0;
    if (j < 16) {
      if (j < bf.nlo) v = bf.lo[hl * bf.slo + j];
    } else if (j - 16 < nhi) {
      v = bf.hi[hl * bf.shi + (j - 16)];
    }
    F[((size_t)h * p.L + l0 + li) * EST_F + j] = (float)v;
  }
}

template <typename KVT>
__device__ __forceinline__ void row4_from_smem(const unsigned char* row, int lane, float (&v)[4]);
template <>
__device__ __forceinline__ void row4_from_smem<__nv_bfloat16>(const unsigned char* row, int lane, float (&v)[4]) {
  const uint2 w = reinterpret_cast<const uint2*>(row)[lane];
  v[0] = bf16lo_to_f32(w.x);
  v[1] = bf16hi_to_f32(w.x);
  v[2] = bf16lo_to_f32(w.y);
  v[3] = bf16hi_to_f32(w.y);
}
template <>
__device__ __forceinline__ void row4_from_smem<float>(const unsigned char* row, int lane, float (&v)[4]) {
  const float4 w = reinterpret_cast<const float4*>(row)[lane];
  v[0] = w.x;
  v[1] = w.y;
  v[2] = w.z;
  v[3] = w.w;
}
template <typename KVT>
__device__ __forceinline__ void row2_from_smem(const unsigned char* row, int lane, float (&v)[4]) {
  const KVT* r = reinterpret_cast<const KVT*>(row);
  v[0] = to_f32(r[2 * lane]);
  v[1] = to_f32(r[2 * lane + 1]);
  v[2] = v[3] = 0.f;
}

template <int D, typename KVT, int LP>
__global__ void __launch_bounds__(EST_THREADS, 2) soft_count_attend_kernel(const EstParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int VPL = D / 32;                        // value columns per lane (2 or 4)
  constexpr int ROW = D * (int)sizeof(KVT);          // bytes of a value row
  const int pair = blockIdx.x, split = blockIdx.y;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int L = p.L;
  const int i0 = split * p.keys_per_split;
  const int cnt = max(0, min(p.k - i0, p.keys_per_split));
  const size_t pair_keys = (size_t)pair * p.Ncap;
  const EstSmem sp = est_smem_plan(G, D, L, p.keys_per_split, (int)sizeof(KVT));
  float* fs = reinterpret_cast<float*>(smem);                    // [G][L][EST_F]
  float* cnts = reinterpret_cast<float*>(smem + sp.counts);      // [cnt][G]
  int* keys_s = reinterpret_cast<int*>(smem + sp.keys);          // [cnt]
  unsigned char* vrows = smem + sp.vrows;                        // [cnt][ROW]
  unsigned int* last_flag = reinterpret_cast<unsigned int*>(smem + sp.flag);

  est_stamp(p.phase_ts, 0);
  // ---- staging: the key list, then every ID row and value row of the CTA
  const int* list = p.idx + (size_t)pair * p.k + i0;
  for (int j = tid; j < cnt; j += EST_THREADS) keys_s[j] = min(max(__ldg(list + j), 0), p.Ncap - 1);
  __syncthreads();
  est_stamp(p.phase_ts, 1);
  {
    const int v_chunks = ROW / 16;
    const uint32_t v_base = smem_u32(vrows);
    const unsigned char* V = reinterpret_cast<const unsigned char*>(p.V);
    for (int e = tid; e < cnt * v_chunks; e += EST_THREADS) {
      const int j = e / v_chunks, c = e % v_chunks;
      cp_async16(v_base + (uint32_t)(j * ROW + 16 * c), V + (pair_keys + keys_s[j]) * ROW + 16 * c);
    }
    cp_async_commit();
    est_stamp(p.phase_ts, 2);
    // the factor image is written by the factor kernel: copy it only once
    // that grid has completed (a no-op wait for an ordinary launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    est_stamp(p.phase_ts, 3);
    const float* F = p.F + (size_t)pair * G * L * EST_F;
    const uint32_t f_base = smem_u32(fs);
    for (int e = tid; e < G * L * EST_F / 4; e += EST_THREADS) cp_async16(f_base + 16u * e, F + 4 * e);
    cp_async_commit();
    cp_async_wait_all();
  }
  __syncthreads();
  est_stamp(p.phase_ts, 4);

  // ---- pass A: counts, one thread per key. The key's ID row is read into
  // registers and rotated back to table order (load_key_row_ids), so table l
  // is byte l. Eight tables at a time: their IDs and factor pairs are loaded
  // together, their probabilities (lo * hi) added as a fixed tree, then to the
  // running count. The factors are float64 results rounded to f32, and the
  // count is an f32 sum: its relative error stays below (L + 2) 2^-24.
  const int plo = p.P / 2;
  const int mlo = (1 << plo) - 1;
  for (int j = tid; j < cnt; j += EST_THREADS) {
    const int key = keys_s[j];
    KeyRowIds<LP> r;
    load_key_row_ids<LP>(r, p.ids + (pair_keys + key) * LP, key);
    float c[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) c[h] = 0.f;
#pragma unroll
    for (int l0 = 0; l0 < LP; l0 += 8) {
      if (l0 < L) {
        // every load is unconditional inside the group: a table past the
        // last reads table L - 1 and is masked out
        int idv[8];
        bool live[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int l = l0 + u;
          idv[u] = (int)((r.w[l >> 2] >> (8 * (l & 3))) & 255u);
          live[u] = l < L;
        }
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (h < G) {
            const float* f = fs + (size_t)h * L * EST_F;
            float q[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int lc = min(l0 + u, L - 1);
              const float a = f[lc * EST_F + (idv[u] & mlo)];
              const float bq = f[lc * EST_F + 16 + (idv[u] >> plo)];
              q[u] = live[u] ? a * bq : 0.f;
            }
            c[h] += ((q[0] + q[1]) + (q[2] + q[3])) + ((q[4] + q[5]) + (q[6] + q[7]));
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 8; ++h)
      if (h < G) cnts[j * G + h] = c[h];
  }
  __syncthreads();
  est_stamp(p.phase_ts, 5);

  // ---- pass B: sum c v and sum c per head, warps over keys (each warp's
  // keys in increasing order), lanes over value columns; four keys' rows
  // and counts loaded at a time
  float acc[8][VPL];
  float csum[8];
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    csum[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[h][e] = 0.f;
  }
  for (int j0 = warp; j0 < cnt; j0 += 4 * EST_WARPS) {
    float v[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = min(j0 + u * EST_WARPS, cnt - 1);
      if constexpr (VPL == 4) {
        row4_from_smem<KVT>(vrows + (size_t)j * ROW, lane, v[u]);
      } else {
        row2_from_smem<KVT>(vrows + (size_t)j * ROW, lane, v[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = j0 + u * EST_WARPS;
      if (j < cnt) {                                 // uniform over the warp
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (h < G) {
            const float cf = cnts[j * G + h];
            csum[h] += cf;
#pragma unroll
            for (int e = 0; e < VPL; ++e) acc[h][e] = fmaf(cf, v[u][e], acc[h][e]);
          }
        }
      }
    }
  }
  __syncthreads();
  // warp partials into the (dead) factor image: [warp][G][D + 1]
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
  est_stamp(p.phase_ts, 6);
  if (tid == 0) *last_flag = (atomicAdd(&p.counters[pair], 1u) == (unsigned)p.splits - 1u) ? 1u : 0u;
  __syncthreads();
  if (*last_flag == 0u) {
    est_stamp(p.phase_ts, 7);
    return;
  }
  // ---- last CTA of the pair: splits in order, then the division
  __threadfence();
  const float* part = p.part + (size_t)pair * p.splits * stride;
  for (int e = tid; e < G * D; e += EST_THREADS) {
    const int h = e / D, dv = e % D;
    float cs = 0.f, o = 0.f;
    // eight splits' values loaded at a time, then added in split order
    for (int s0 = 0; s0 < p.splits; s0 += 8) {
      float a[8], bv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int sp_ = min(s0 + u, p.splits - 1);
        a[u] = __ldcg(part + (size_t)sp_ * stride + h * (D + 1));
        bv[u] = __ldcg(part + (size_t)sp_ * stride + h * (D + 1) + 1 + dv);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (s0 + u < p.splits) {
          cs += a[u];
          o += bv[u];
        }
      }
    }
    p.O[((size_t)b * p.Hq + kvh * G + h) * D + dv] = o / cs;
  }
  if (tid == 0) p.counters[pair] = 0u;
  est_stamp(p.phase_ts, 7);
}

}  // namespace hst
