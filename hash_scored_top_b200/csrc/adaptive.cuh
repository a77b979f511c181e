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
// top k: when k was not clamped, the search's last bin is the k-th largest
// key itself; otherwise the plain count-based radix select finds it.
//
// Shared-memory traffic: a bin's mass is two 32-bit words (low word, high
// word plus the carry out of the low word), so every histogram update is a
// native 32-bit atomic; the level-0 key counts are taken while the scores
// are loaded and serve both the mass search and the top-k; each level of the
// mass search has bins of its own, so one cluster barrier per level suffices;
// a level is resolved over groups of 32 bins first, so a CTA reads the other
// CTAs' group sums and one group's bins, not every bin.
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
  unsigned long long scan_tmp[32];   // per-warp float64 score sums
  unsigned long long mass_above;     // broadcast of the level's result
  uint32_t bin, cnt_above, found, pad;
};

constexpr int kAdaptHistWords = hist_words(0) + hist_words(1) + hist_words(2);
// per level, three words (mass low and high, count) per group of 32 bins
constexpr int kAdaptGroupWords = 3 * (kAdaptHistWords / 32);
// counts (one word per bin), masses (two words per bin) and group sums of the three levels
constexpr uint32_t kAdaptFixedBytes = (uint32_t)(((sizeof(SelShared) + 15) & ~15) + 4 * kAdaptHistWords +
                                                 8 * kAdaptHistWords + 4 * kAdaptGroupWords +
                                                 ((sizeof(AdaptShared) + 15) & ~15));
static_assert((4 * kAdaptGroupWords) % 16 == 0, "the keys after the group sums stay 16-byte aligned");

// This CTA's mass and count of every group of 32 bins of one level (all
// warps; the level's atomics are complete): glo, ghi, gc [ngroups].
__device__ __forceinline__ void group_sums(const uint32_t* mlo, const uint32_t* mhi, const uint32_t* hc, int ngroups,
                                           uint32_t* glo, uint32_t* ghi, uint32_t* gc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int g = warp; g < ngroups; g += nw) {
    const int b = g * 32 + lane;
    unsigned long long m = ((unsigned long long)mhi[b] << 32) | mlo[b];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(FULL, m, o);
    const uint32_t c = __reduce_add_sync(FULL, hc[b]);
    if (lane == 0) {
      glo[g] = (uint32_t)m;
      ghi[g] = (uint32_t)(m >> 32);
      gc[g] = c;
    }
  }
}

// Exclusive scan over the lanes of a warp (lane 0 first) of a mass and a count.
__device__ __forceinline__ void warp_exclusive_scan2(unsigned long long m, uint32_t c, unsigned long long& m_before,
                                                     uint32_t& c_before) {
  const int lane = threadIdx.x & 31;
  unsigned long long im = m;
  uint32_t ic = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long ym = __shfl_up_sync(FULL, im, o);
    const uint32_t yc = __shfl_up_sync(FULL, ic, o);
    if (lane >= o) {
      im += ym;
      ic += yc;
    }
  }
  m_before = im - m;
  c_before = ic - c;
}

// One level of the mass search (warp 0 only): the cluster-wide mass and count
// of every group of 32 bins (descending), the group where the running mass
// from the top first reaches `need`, then that group's 32 bins. Reads of
// other CTAs' shared memory: three words per group and per bin of that group,
// from every CTA. Writes found, bin, mass_above (mass in bins above it) and
// cnt_above to `as`. ngroups <= 64.
__device__ void resolve_mass_grouped(const uint32_t* mlo, const uint32_t* mhi, const uint32_t* hc,
                                     const uint32_t* glo, const uint32_t* ghi, const uint32_t* gc, int ngroups,
                                     unsigned long long need, int C, AdaptShared* as) {
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31;
  // lane l: groups ngroups - 1 - 2l and ngroups - 2 - 2l
  const int ga = ngroups - 1 - 2 * lane, gb = ga - 1;
  unsigned long long ma = 0ull, mb = 0ull;
  uint32_t ca = 0u, cb = 0u;
  for (int r = 0; r < C; ++r) {
    const uint32_t* pl = cluster.map_shared_rank(glo, r);
    const uint32_t* ph = cluster.map_shared_rank(ghi, r);
    const uint32_t* pc = cluster.map_shared_rank(gc, r);
    if (ga >= 0) {
      ma += ((unsigned long long)ph[ga] << 32) | pl[ga];
      ca += pc[ga];
    }
    if (gb >= 0) {
      mb += ((unsigned long long)ph[gb] << 32) | pl[gb];
      cb += pc[gb];
    }
  }
  unsigned long long m_before;
  uint32_t c_before;
  warp_exclusive_scan2(ma + mb, ca + cb, m_before, c_before);
  int grp = -1;
  unsigned long long g_mass = 0ull;
  uint32_t g_cnt = 0u;
  if (m_before < need && need <= m_before + ma) {
    grp = ga;
    g_mass = m_before;
    g_cnt = c_before;
  } else if (m_before + ma < need && need <= m_before + ma + mb) {
    grp = gb;
    g_mass = m_before + ma;
    g_cnt = c_before + ca;
  }
  const unsigned hit = __ballot_sync(FULL, grp >= 0);
  if (hit == 0u) {                      // the whole unit's mass stays below the target
    if (lane == 0) as->found = 0u;
    return;
  }
  const int src = __ffs(hit) - 1;
  grp = __shfl_sync(FULL, grp, src);
  g_mass = __shfl_sync(FULL, g_mass, src);
  g_cnt = __shfl_sync(FULL, g_cnt, src);
  // the group's bins, lane l: bin 32 grp + 31 - l
  const int bin = grp * 32 + 31 - lane;
  unsigned long long m = 0ull;
  uint32_t c = 0u;
  for (int r = 0; r < C; ++r) {
    m += ((unsigned long long)cluster.map_shared_rank(mhi, r)[bin] << 32) | cluster.map_shared_rank(mlo, r)[bin];
    c += cluster.map_shared_rank(hc, r)[bin];
  }
  warp_exclusive_scan2(m, c, m_before, c_before);
  const unsigned long long before = g_mass + m_before;
  const unsigned hit2 = __ballot_sync(FULL, before < need && need <= before + m);
  if (hit2 == 0u) {                     // cannot happen: the group's mass covers the rest of need
    if (lane == 0) as->found = 0u;
    return;
  }
  if (lane == __ffs(hit2) - 1) {
    as->found = 1u;
    as->bin = (uint32_t)bin;
    as->mass_above = before;
    as->cnt_above = g_cnt + c_before;
  }
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
  // group sums, level by level: low words, high words, counts
  uint32_t* group_words = mass_words + 2 * kAdaptHistWords;
  a += 12 * kAdaptHistWords + 4 * kAdaptGroupWords;
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
    uint32_t* gw = group_words;
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
      const int ng = (1 << bits) / 32;
      group_sums(mlo, mhi, hc, ng, gw, gw + ng, gw + 2 * ng);
      __syncthreads();
      cluster_sync();
      if (warp == 0) resolve_mass_grouped(mlo, mhi, hc, gw, gw + ng, gw + 2 * ng, ng, need, C, as);
      __syncthreads();
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
      gw += 3 * ng;
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
