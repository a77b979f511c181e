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
//
// Shared-memory traffic: a bin's mass is two 32-bit words (low word, high
// word plus the carry out of the low word), so every histogram update is a
// native 32-bit atomic; the level-0 key counts are taken while the scores
// are loaded and serve both the mass search and the top-k; each level of the
// mass search has bins of its own, so one cluster barrier per level suffices.
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

constexpr int kAdaptHistWords = hist_words(0) + hist_words(1) + hist_words(2);
// counts (one word per bin) and masses (two words per bin) of the three levels
constexpr uint32_t kAdaptFixedBytes = (uint32_t)(((sizeof(SelShared) + 15) & ~15) + 4 * kAdaptHistWords +
                                                 8 * kAdaptHistWords + ((sizeof(AdaptShared) + 15) & ~15));

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
// mlo, mhi: the level's low and high mass words; hc: its key counts.
template <int BPT>
__device__ void resolve_mass_level(const uint32_t* mlo, const uint32_t* mhi, const uint32_t* hc, int nbins,
                                   unsigned long long need, int C, SelShared* sh, AdaptShared* as) {
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
      const uint32_t* pl = cluster.map_shared_rank(mlo, r) + base;
      const uint32_t* ph = cluster.map_shared_rank(mhi, r) + base;
      const uint32_t* pc = cluster.map_shared_rank(hc, r) + base;
      if constexpr (BPT % 4 == 0) {
        // 16-byte reads: a read of another CTA's shared memory costs about
        // the same whatever its width
#pragma unroll
        for (int j = 0; j < BPT; j += 4) {
          const uint4 l = *reinterpret_cast<const uint4*>(pl + j);
          const uint4 h = *reinterpret_cast<const uint4*>(ph + j);
          const uint4 n = *reinterpret_cast<const uint4*>(pc + j);
          m[j] += ((unsigned long long)h.x << 32) | l.x;
          m[j + 1] += ((unsigned long long)h.y << 32) | l.y;
          m[j + 2] += ((unsigned long long)h.z << 32) | l.z;
          m[j + 3] += ((unsigned long long)h.w << 32) | l.w;
          c[j] += n.x;
          c[j + 1] += n.y;
          c[j + 2] += n.z;
          c[j + 3] += n.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          m[j] += ((unsigned long long)ph[j] << 32) | pl[j];
          c[j] += pc[j];
        }
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

// floor(x * 2^sc) for the bit pattern `key` of a finite float x >= 0, from
// its IEEE-754 binary32 fields: x = (2^23 + f) * 2^(e - 150) for a biased
// exponent e >= 1, and f * 2^-149 for e = 0. Callers have x <= S < 2^(62 - sc),
// so a left shift stays below 2^62; a right shift truncates, as floor does.
__device__ __forceinline__ unsigned long long fixed_mass(uint32_t key, int sc) {
  const uint32_t e = key >> 23, f = key & 0x7fffffu;
  const unsigned long long m = e != 0u ? (unsigned long long)(f | 0x800000u) : (unsigned long long)f;
  const int sh = (e != 0u ? (int)e - 150 : -149) + sc;
  if (sh >= 0) return m << sh;
  return sh > -32 ? (m >> -sh) : 0ull;
}

// f(key) for this CTA's keys i < n, read four at a time (keys: 16-byte
// aligned, readable up to n rounded up to 4).
template <typename F>
__device__ __forceinline__ void for_each_key4(const uint32_t* keys, int n, F f) {
  const int n4 = (n + 3) >> 2;
  for (int g = threadIdx.x; g < n4; g += blockDim.x) {
    const uint4 q = reinterpret_cast<const uint4*>(keys)[g];
    const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (4 * g + j < n) f(kv[j]);
  }
}

// Keys a CTA holds in shared memory: room for a multiple of 128 keys (the
// compaction reads whole 128-key chunks).
__host__ __device__ constexpr int adapt_key_slots(int keys_per_cta) { return (keys_per_cta + 127) & ~127; }

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
  // masses, level by level: low words of the level's bins, then high words
  uint32_t* mass_words = h0 + kAdaptHistWords;
  a += 12 * kAdaptHistWords;
  AdaptShared* as = reinterpret_cast<AdaptShared*>(a);
  a += (sizeof(AdaptShared) + 15) & ~15;
  uint32_t* keys = reinterpret_cast<uint32_t*>(a);
  uint32_t* hist[3] = {h0, h1, h2};
  // split cluster barrier: this arrive, and the wait just before the first
  // store into another CTA (every CTA of the cluster has started by then)
  cluster_arrive_relaxed();

  for (int i = tid; i < 3 * kAdaptHistWords; i += blockDim.x) h0[i] = 0u;
  __syncthreads();
  const int k0 = rank * p.keys_per_cta;
  const int n_local = max(0, min(p.N - k0, p.keys_per_cta));
  const float* src = p.scores + (size_t)unit * p.Ncap + k0;
  constexpr uint32_t mask0 = (1u << sel_bits(0)) - 1u;
  // the keys, this CTA's float64 sum and its level-0 key counts
  double ssum = 0.0;
  int n_vec = 0;
  if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
    n_vec = n_local & ~3;
    for (int g = tid; g < n_vec / 4; g += blockDim.x) {
      const float4 v = reinterpret_cast<const float4*>(src)[g];
      const uint4 kk = make_uint4(key_of(fmaxf(v.x, 0.0f)), key_of(fmaxf(v.y, 0.0f)), key_of(fmaxf(v.z, 0.0f)),
                                  key_of(fmaxf(v.w, 0.0f)));
      reinterpret_cast<uint4*>(keys)[g] = kk;
      ssum += (double)__uint_as_float(kk.x);
      ssum += (double)__uint_as_float(kk.y);
      ssum += (double)__uint_as_float(kk.z);
      ssum += (double)__uint_as_float(kk.w);
      atomicAdd(&h0[(kk.x >> sel_shift(0)) & mask0], 1u);
      atomicAdd(&h0[(kk.y >> sel_shift(0)) & mask0], 1u);
      atomicAdd(&h0[(kk.z >> sel_shift(0)) & mask0], 1u);
      atomicAdd(&h0[(kk.w >> sel_shift(0)) & mask0], 1u);
    }
  }
  for (int i = n_vec + tid; i < n_local; i += blockDim.x) {
    const uint32_t key = key_of(fmaxf(src[i], 0.0f));
    keys[i] = key;
    ssum += (double)__uint_as_float(key);
    atomicAdd(&h0[(key >> sel_shift(0)) & mask0], 1u);
  }
  for (int i = n_local + tid; i < ((n_local + 127) & ~127); i += blockDim.x) keys[i] = 0u;   // the last chunk's tail
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
  cluster_sync();   // every CTA's sum and level-0 counts are complete
  double S = 0.0;
  for (int r = 0; r < C; ++r) S += as->part[r];

  // ---- the adaptive k
  const int n_all = p.N;
  int k_mass = 0;
  bool reached = false;          // the search ended on one key value v, with n_above keys above it
  uint32_t v = 0u, n_above = 0u;
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
    reached = true;
    uint32_t* mlo = mass_words;
#pragma unroll 1
    for (int lvl = 0; lvl < SEL_LEVELS; ++lvl) {
      const int bits = sel_bits(lvl), shift = sel_shift(lvl);
      const uint32_t mask = (1u << bits) - 1u;
      uint32_t* mhi = mlo + (1 << bits);
      uint32_t* hc = hist[lvl];
      for_each_key4(keys, n_local, [&](uint32_t k) {
        if (pshift >= 32 || (k >> pshift) == prefix) {
          const uint32_t bn = (k >> shift) & mask;
          const unsigned long long fm = fixed_mass(k, sc);
          const uint32_t lo = (uint32_t)fm;
          const uint32_t old = atomicAdd(&mlo[bn], lo);
          const uint32_t hi = (uint32_t)(fm >> 32) + (old + lo < old ? 1u : 0u);   // carry out of the low word
          if (hi != 0u) atomicAdd(&mhi[bn], hi);
          if (lvl > 0) atomicAdd(&hc[bn], 1u);      // level 0 was counted with the load
        }
      });
      __syncthreads();
      cluster_sync();
      resolve_mass_level<4>(mlo, mhi, hc, 1 << bits, need, C, sh, as);
      const bool found = as->found != 0u;
      const uint32_t bn = as->bin, ca = as->cnt_above;
      const unsigned long long ma = as->mass_above;
      // the next level writes bins of its own, so other CTAs may still read these
      if (!found) {                                // the whole unit's mass stays below the target
        reached = false;
        break;
      }
      need -= ma;
      cnt_total += ca;
      prefix = (prefix << bits) | bn;
      pshift = shift;
      mlo = mhi + (1 << bits);
    }
    if (reached) {
      const unsigned long long ft = fixed_mass(prefix, sc);   // every key of the final bin equals prefix
      k_mass = (int)cnt_total + (int)((need + ft - 1ull) / ft);
      v = prefix;
      n_above = cnt_total;
    } else {
      k_mass = n_all;
    }
  }
  const int k = max(p.k_min, min(k_mass, min(p.k_max, n_all)));

  // ---- the exact top-k with that k: from the mass search's last bin when k
  // was not clamped, else by the count search (level-0 counts from the load,
  // published by the barrier after the sums; the other levels zeroed). Then
  // the thread-contiguous compaction, staged in the mass bins (its barrier
  // comes before the first staged write, and after every CTA's last read of
  // them)
  auto pass = [&](int shift, int bits, int pshift, uint32_t prefix, uint32_t* h) {
    const uint32_t mask = (1u << bits) - 1u;
    for_each_key4(keys, n_local, [&](uint32_t key) {
      if (pshift >= 32 || (key >> pshift) == prefix) atomicAdd(&h[(key >> shift) & mask], 1u);
    });
  };
  SelThreshold th;
  if (reached && k == k_mass) {
    // the k-th largest key is v itself: keys above v, and the first
    // k - n_above keys equal to v (1 <= k - n_above <= keys equal to v)
    th.t = v;
    th.take_eq = (uint32_t)k - n_above;
  } else {
    if (target > 0ull) {
      cluster_sync();                              // every CTA has read every CTA's level-1 and level-2 bins
      for (int i = tid; i < hist_words(1) + hist_words(2); i += blockDim.x) h1[i] = 0u;
      __syncthreads();
    }
    th = cluster_threshold_by<FUSED_THREADS / 2>(pass, hist, (uint32_t)k, C, sh);
  }
  int* out = p.idx + (size_t)unit * p.k_max;
  const uint32_t keys_s = (uint32_t)__cvta_generic_to_shared(keys);
  auto key_addr = [&](int i) -> uint32_t { return keys_s + 4u * (uint32_t)i; };
  auto g0_of = [&](int c) { return c * p.keys_per_cta; };
  contiguous_compact(key_addr, n_local, th, C, rank, g0_of, sh, [&](uint32_t pos, int i) {
    if (pos < (uint32_t)k) out[pos] = k0 + i;
  }, out, (uint32_t)k, mass_words, 2 * kAdaptHistWords);
  if (rank == 0) {
    for (int j = k + tid; j < p.k_max; j += blockDim.x) out[j] = -1;
    if (tid == 0) p.kcount[unit] = k;
  }
  cluster_sync();
}

}  // namespace hst
