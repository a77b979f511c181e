// Adaptive k over the soft collision scores, after the Tactic digest ("Tactic:
// Adaptive Sparse Attention with Clustering and Distribution Fitting for
// Long-Context LLMs", section 3 中核となる技術的要素: tokens are chosen until
// their cumulative score reaches a target), applied to SOCKET's step 4. For
// one unit (a KV head's group, or one query head) with scores s_i >= 0:
//   k = min{ k : sum of the k largest s_i >= mass * sum_i s_i },
// clamped to [k_min, min(k_max, N)], and the unit's list is the exact top-k
// with that k (ties to the lower index), ascending.
//
// One cluster of C CTAs per unit, as the plain top-k kernel. The sum S is a
// float64 sum in a fixed order (thread, warp, CTA rank), so it is the same in
// every CTA and every run. The masses are then 64-bit fixed-point integers,
// floor(s * 2^(62 - e)) with S < 2^e, and the smallest k is found by a radix
// search on the sort keys (the f32 bit patterns) whose histograms count mass
// as well as keys; integer sums do not depend on the order of the atomics, so
// the decision is deterministic. Truncation moves a unit's mass by at most
// one part in 2^62 / (keys), far below the scores' own f32 rounding. Then the
// plain count-based radix select takes the top k.
#pragma once

#include "select.cuh"
#include "socket_kernels.cuh"

namespace hst {

struct AdaptParams {
  const float* scores;   // [units][Ncap]
  int* idx;              // [units][k_max]: the first kcount entries ascending, the rest -1
  int* kcount;           // [units]
  int Ncap, N, k_min, k_max, C, keys_per_cta;
  float mass;
};

struct AdaptShared {
  double part[SEL_MAX_C];            // every CTA's float64 score sum
  unsigned long long scan_tmp[32];   // block-scan scratch
  unsigned long long mass_above;     // broadcast of the level's result
  uint32_t bin, cnt_above, found, pad;
};

constexpr uint32_t kAdaptFixedBytes = (uint32_t)(((sizeof(SelShared) + 15) & ~15) +
                                                 4 * (hist_words(0) + hist_words(1) + hist_words(2)) +
                                                 8 * (1 << 11) + ((sizeof(AdaptShared) + 15) & ~15));

// Block-wide exclusive scan of one unsigned 64-bit value per thread.
__device__ __forceinline__ unsigned long long block_exclusive_scan_u64(unsigned long long v, AdaptShared* as) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) as->scan_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long t = lane < nw ? as->scan_tmp[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(FULL, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) as->scan_tmp[lane] = t;
  }
  __syncthreads();
  const unsigned long long before = warp > 0 ? as->scan_tmp[warp - 1] : 0ull;
  __syncthreads();
  return before + x - v;
}

// One level of the mass search over nbins bins (descending bin order across
// the threads, BPT bins each): the cluster-wide mass and count of every bin,
// then the bin where the running mass from the top first reaches `need`.
template <int BPT>
__device__ void resolve_mass_level(const unsigned long long* mh, const uint32_t* hc, int nbins, unsigned long long need,
                                   int C, SelShared* sh, AdaptShared* as) {
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int base = nbins - (tid + 1) * BPT;
  const bool mine = base >= 0;
  if (tid == 0) {
    as->found = 0u;
    as->bin = 0u;
    as->cnt_above = 0u;
    as->mass_above = 0ull;
  }
  unsigned long long m[BPT];
  uint32_t c[BPT];
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    m[j] = 0ull;
    c[j] = 0u;
  }
  if (mine) {
    for (int r = 0; r < C; ++r) {
      const unsigned long long* pm = cluster.map_shared_rank(mh, r) + base;
      const uint32_t* pc = cluster.map_shared_rank(hc, r) + base;
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        m[j] += pm[j];
        c[j] += pc[j];
      }
    }
  }
  unsigned long long lm = 0ull;
  uint32_t lc = 0u;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    lm += m[j];
    lc += c[j];
  }
  const unsigned long long mb = block_exclusive_scan_u64(lm, as);
  const uint32_t cb = block_exclusive_scan(lc, sh);
  if (mine && mb < need && need <= mb + lm) {
    unsigned long long run = mb;
    uint32_t crun = cb;
#pragma unroll
    for (int j = BPT - 1; j >= 0; --j) {
      if (run < need && need <= run + m[j]) {
        as->bin = (uint32_t)(base + j);
        as->mass_above = run;
        as->cnt_above = crun;
        as->found = 1u;
      }
      run += m[j];
      crun += c[j];
    }
  }
  __syncthreads();
}

__device__ __forceinline__ unsigned long long fixed_mass(uint32_t key, int sc) {
  return __double2ull_rz(ldexp((double)__uint_as_float(key), sc));
}

__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_adaptive_topk_kernel(const AdaptParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  const int C = p.C;
  const int rank = (int)cluster_ctarank();
  const int unit = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* a = dyn;
  SelShared* sh = reinterpret_cast<SelShared*>(a);
  a += (sizeof(SelShared) + 15) & ~15;
  uint32_t* h0 = reinterpret_cast<uint32_t*>(a);
  uint32_t* h1 = h0 + hist_words(0);
  uint32_t* h2 = h1 + hist_words(1);
  a += 4 * (hist_words(0) + hist_words(1) + hist_words(2));
  unsigned long long* mh = reinterpret_cast<unsigned long long*>(a);   // [2048] mass per bin
  a += 8 * (1 << 11);
  AdaptShared* as = reinterpret_cast<AdaptShared*>(a);
  a += (sizeof(AdaptShared) + 15) & ~15;
  uint32_t* keys = reinterpret_cast<uint32_t*>(a);
  uint32_t* hist[3] = {h0, h1, h2};
  // split cluster barrier: this arrive, and the wait just before the first
  // store into another CTA (every CTA of the cluster has started by then)
  cluster_arrive_relaxed();

  for (int i = tid; i < hist_words(0) + hist_words(1) + hist_words(2); i += blockDim.x) h0[i] = 0u;
  for (int i = tid; i < (1 << 11); i += blockDim.x) mh[i] = 0ull;
  const int k0 = rank * p.keys_per_cta;
  const int n_local = max(0, min(p.N - k0, p.keys_per_cta));
  const float* src = p.scores + (size_t)unit * p.Ncap + k0;
  double ssum = 0.0;
  for (int i = tid; i < n_local; i += blockDim.x) {
    const uint32_t key = key_of(fmaxf(src[i], 0.0f));
    keys[i] = key;
    ssum += (double)__uint_as_float(key);
  }
  // the CTA's sum in a fixed order (lanes, then warps), sent to every CTA
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(FULL, ssum, o);
  double* wsum = reinterpret_cast<double*>(as->scan_tmp);
  if (lane == 0) wsum[warp] = ssum;
  __syncthreads();
  cluster_wait();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += wsum[w];
    for (int r = 0; r < C; ++r) *cluster.map_shared_rank(&as->part[rank], r) = t;
  }
  __syncthreads();
  cluster_sync();
  double S = 0.0;
  for (int r = 0; r < C; ++r) S += as->part[r];

  // ---- the adaptive k
  const int n_all = p.N;
  int k_mass = 0;
  unsigned long long target = 0ull;
  int sc = 0;
  if (S > 0.0) {
    sc = 62 - (ilogb(S) + 1);                      // S < 2^(62 - sc)
    target = (unsigned long long)ceil(ldexp((double)p.mass * S, sc));
  }
  if (target > 0ull) {
    unsigned long long need = target;
    uint32_t prefix = 0, cnt_total = 0;
    int pshift = 32;
    bool reached = true;
#pragma unroll 1
    for (int lvl = 0; lvl < SEL_LEVELS; ++lvl) {
      const int bits = sel_bits(lvl), shift = sel_shift(lvl);
      const uint32_t mask = (1u << bits) - 1u;
      for (int i = tid; i < n_local; i += blockDim.x) {
        const uint32_t k = keys[i];
        if (pshift >= 32 || (k >> pshift) == prefix) {
          const uint32_t bn = (k >> shift) & mask;
          atomicAdd(&mh[bn], fixed_mass(k, sc));
          atomicAdd(&hist[lvl][bn], 1u);
        }
      }
      __syncthreads();
      cluster_sync();
      if (bits == 11) resolve_mass_level<2>(mh, hist[lvl], 1 << 11, need, C, sh, as);
      else resolve_mass_level<1>(mh, hist[lvl], 1 << 9, need, C, sh, as);
      const bool found = as->found != 0u;
      const uint32_t bn = as->bin, ca = as->cnt_above;
      const unsigned long long ma = as->mass_above;
      cluster_sync();                              // every CTA has read every CTA's bins
      for (int i = tid; i < (1 << 11); i += blockDim.x) mh[i] = 0ull;
      for (int i = tid; i < hist_words(lvl); i += blockDim.x) hist[lvl][i] = 0u;
      __syncthreads();
      if (!found) {                                // the whole unit's mass stays below the target
        reached = false;
        break;
      }
      need -= ma;
      cnt_total += ca;
      prefix = (prefix << bits) | bn;
      pshift = shift;
    }
    if (reached) {
      const unsigned long long ft = fixed_mass(prefix, sc);   // every key of the final bin equals prefix
      k_mass = (int)cnt_total + (int)((need + ft - 1ull) / ft);
    } else {
      k_mass = n_all;
    }
  }
  const int k = max(p.k_min, min(k_mass, min(p.k_max, n_all)));

  // ---- the exact top-k with that k (the bins are zero again)
  histogram_pass([&](int i) { return keys[i]; }, n_local, sel_shift(0), sel_bits(0), 32, 0u, h0);
  __syncthreads();
  cluster_sync();
  auto key_at = [&](int i) -> uint32_t { return keys[i]; };
  const SelThreshold th = cluster_threshold<FUSED_THREADS>(key_at, n_local, hist, (uint32_t)k, C, sh);
  int* out = p.idx + (size_t)unit * p.k_max;
  ordered_compact(key_at, n_local, th, C, rank, sh, [&](uint32_t pos, int i) {
    if (pos < (uint32_t)k) out[pos] = k0 + i;
  });
  if (rank == 0) {
    for (int j = k + tid; j < p.k_max; j += blockDim.x) out[j] = -1;
    if (tid == 0) p.kcount[unit] = k;
  }
  cluster_sync();
}

}  // namespace hst
