// Exact deterministic top-k across a thread-block cluster, SOCKET step 4
// (SOCKET technical summary, section 中核メカニズム：ソフト LSH, step 4:
// the top-k keys are chosen deterministically).
//
// The keys of one (batch, KV-head) pair are split over the C CTAs of a
// cluster; CTA c holds the 32-bit sort keys of an ascending index range in
// shared memory. Sort keys are the bit patterns of non-negative f32 scores,
// which order like the scores as unsigned integers.
//
// Selection is a most-significant-digit radix select over three digit levels
// (bits 30..20, 19..9, 8..0): every CTA histograms the digit of its keys that
// match the prefix found so far, each CTA sums the cluster's histograms
// through distributed shared memory, and a descending scan finds the bin that
// holds the k-th largest key. A level ends the search early when the whole
// bin is taken. After the last level the threshold t is exact and the tie
// rule applies: among keys equal to t, the lowest indices are taken.
//
// Output order: every CTA counts its selected keys, publishes (greater,
// equal) counts to the whole cluster, and writes its keys in ascending index
// order at the offset of the CTAs before it, so the result is ascending.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace hst {

namespace cg = cooperative_groups;

constexpr int SEL_MAX_C = 16;
constexpr int SEL_LEVELS = 3;
__host__ __device__ constexpr int sel_bits(int level) { return level == 2 ? 9 : 11; }
__host__ __device__ constexpr int sel_shift(int level) { return level == 0 ? 20 : level == 1 ? 9 : 0; }

// Broadcast results and scratch of the selection, in shared memory.
struct SelShared {
  uint32_t bin;                  // bin of the k-th largest key at the current level
  uint32_t above;                // cluster-wide count in bins above it
  uint32_t total_in_bin;         // cluster-wide count in the bin
  uint32_t pad;
  uint32_t warp_tmp[32];         // block-scan scratch
  uint32_t cnt_w[32][2];         // compaction: per-warp (greater, equal) counts
  uint32_t off_w[32][2];         // compaction: per-warp (selected, equal) offsets
  uint32_t counts[SEL_MAX_C][2]; // (greater, equal) published by every CTA of the cluster
};

// Block-wide exclusive scan of one value per thread (thread order).
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, SelShared* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(FULL, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh->warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < nw ? sh->warp_tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(FULL, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) sh->warp_tmp[lane] = t;   // inclusive warp totals
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? sh->warp_tmp[warp - 1] : 0u;
  __syncthreads();
  return before + x - v;
}

// Cluster-wide resolution of one histogram level of nbins bins; thread t
// handles bins [nbins - (t + 1) * BPT, nbins - t * BPT) (none once that is
// negative). `hist` is this CTA's histogram (same shared offset in every CTA).
// need >= 1 keys are still to be taken among the keys that match the prefix.
// Writes sh->bin, sh->above, sh->total_in_bin.
template <int BPT>
__device__ void resolve_level(const uint32_t* hist, int nbins, uint32_t need, int C, SelShared* sh) {
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int base = nbins - (tid + 1) * BPT;            // this thread: bins [base, base + BPT)
  const bool mine = base >= 0;
  if (tid == 0) {            // defaults, overwritten by the thread that holds the k-th key
    sh->bin = 0;
    sh->above = 0;
    sh->total_in_bin = 0;
  }
  uint32_t tot[BPT];
#pragma unroll
  for (int j = 0; j < BPT; ++j) tot[j] = 0;
  if (mine) {
    for (int c = 0; c < C; ++c) {
      const uint32_t* h = cluster.map_shared_rank(hist, c) + base;
      if constexpr (BPT % 4 == 0) {
#pragma unroll
        for (int j = 0; j < BPT; j += 4) {
          const uint4 v = *reinterpret_cast<const uint4*>(h + j);
          tot[j] += v.x; tot[j + 1] += v.y; tot[j + 2] += v.z; tot[j + 3] += v.w;
        }
      } else if constexpr (BPT % 2 == 0) {
#pragma unroll
        for (int j = 0; j < BPT; j += 2) {
          const uint2 v = *reinterpret_cast<const uint2*>(h + j);
          tot[j] += v.x; tot[j + 1] += v.y;
        }
      } else {
#pragma unroll
        for (int j = 0; j < BPT; ++j) tot[j] += h[j];
      }
    }
  }
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) local += tot[j];
  const uint32_t before = block_exclusive_scan(local, sh);   // keys in bins above this thread's
  if (mine && before < need && need <= before + local) {
    uint32_t run = before;
#pragma unroll
    for (int j = BPT - 1; j >= 0; --j) {                      // descending bins
      if (run < need && need <= run + tot[j]) {
        sh->bin = (uint32_t)(base + j);
        sh->above = run;
        sh->total_in_bin = tot[j];
      }
      run += tot[j];
    }
  }
  __syncthreads();
}

// Counts keys matching the prefix in bin (key >> shift) & mask of `hist`.
// pshift >= 32 means "no prefix" (all keys).
template <typename KeyAt>
__device__ __forceinline__ void histogram_pass(KeyAt key_at, int n, int shift, int bits, int pshift,
                                               uint32_t prefix, uint32_t* hist) {
  const uint32_t mask = (1u << bits) - 1u;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t k = key_at(i);
    const bool match = pshift >= 32 ? true : ((k >> pshift) == prefix);
    if (match) atomicAdd(&hist[(k >> shift) & mask], 1u);
  }
}

__device__ __forceinline__ void sel_stamp(unsigned long long* ts, int phase) {
  if (ts != nullptr && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    ts[blockIdx.x * 24 + phase] = t;
  }
}

// Threshold of the pair, identical in every CTA of the cluster.
struct SelThreshold {
  uint32_t t;        // keys > t are selected
  uint32_t take_eq;  // keys == t: the first take_eq of them in index order (UINT_MAX: all)
};

// The three-level search (NT threads per CTA). hist[0] holds this CTA's
// level-0 histogram and the cluster has synchronised since it was filled;
// hist[1], hist[2] are zeroed.
template <int NT, typename KeyAt>
__device__ SelThreshold cluster_threshold(KeyAt key_at, int n_local, uint32_t* const* hist, uint32_t k, int C,
                                          SelShared* sh, unsigned long long* ts = nullptr) {
  uint32_t need = k;
  uint32_t prefix = 0;
  int pshift = 32;
  SelThreshold th;
#pragma unroll
  for (int lvl = 0; lvl < SEL_LEVELS; ++lvl) {
    if (lvl > 0) {
      histogram_pass(key_at, n_local, sel_shift(lvl), sel_bits(lvl), pshift, prefix, hist[lvl]);
      __syncthreads();
      sel_stamp(ts, 14 + 2 * lvl);
      cluster_sync();
      sel_stamp(ts, 15 + 2 * lvl);
    }
    constexpr int B01 = (1 << 11) / NT > 0 ? (1 << 11) / NT : 1;
    constexpr int B2 = (1 << 9) / NT > 0 ? (1 << 9) / NT : 1;
    if (lvl < 2) resolve_level<B01>(hist[lvl], 1 << 11, need, C, sh);
    else resolve_level<B2>(hist[lvl], 1 << 9, need, C, sh);
    need -= sh->above;
    prefix = (prefix << sel_bits(lvl)) | sh->bin;
    pshift = sel_shift(lvl);
    const bool whole = need == sh->total_in_bin;
    if (whole || lvl == SEL_LEVELS - 1) {
      th.t = prefix << sel_shift(lvl);          // smallest key of the bin (exact key at the last level)
      th.take_eq = whole ? 0xffffffffu : need;  // whole bin: every key >= t
      break;
    }
  }
  return th;
}

// Ordered compaction of this CTA's selected keys (ascending index i in [0, n)):
// pass 1 counts, the counts are exchanged across the cluster, pass 2 calls
// emit(pos, i) with the key's position in the pair's ascending output.
// rank: this CTA's rank; keys of CTA c precede those of CTA c + 1.
template <typename KeyAt, typename Emit>
__device__ void ordered_compact(KeyAt key_at, int n, const SelThreshold& th, int C, int rank, SelShared* sh,
                                Emit emit, unsigned long long* ts = nullptr) {
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const bool all_eq = th.take_eq == 0xffffffffu;
  const int nchunks = (n + 31) / 32;
  const int per_warp = (nchunks + nw - 1) / nw;
  const int c0 = warp * per_warp;
  const int c1 = min(nchunks, c0 + per_warp);
  // pass 1: per-warp counts of (key > t) and (key == t); "> t" means ">= t" when all ties are taken
  uint32_t n_gt = 0, n_eq = 0;
  for (int ch = c0; ch < c1; ++ch) {
    const int i = ch * 32 + lane;
    const bool valid = i < n;
    const uint32_t k = valid ? key_at(i) : 0u;
    const bool gt = valid && (all_eq ? k >= th.t : k > th.t);
    const bool eq = valid && !all_eq && k == th.t;
    n_gt += __popc(__ballot_sync(FULL, gt));
    n_eq += __popc(__ballot_sync(FULL, eq));
  }
  if (lane == 0) {
    sh->cnt_w[warp][0] = n_gt;
    sh->cnt_w[warp][1] = n_eq;
  }
  __syncthreads();
  // CTA totals, published to every CTA of the cluster
  if (threadIdx.x < C) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < nw; ++w) {
      g += sh->cnt_w[w][0];
      e += sh->cnt_w[w][1];
    }
    uint32_t* dst = cluster.map_shared_rank(&sh->counts[rank][0], (unsigned)threadIdx.x);
    dst[0] = g;
    dst[1] = e;
  }
  sel_stamp(ts, 19);
  cluster_sync();
  sel_stamp(ts, 20);
  // this CTA's tie quota and output offset, from the published counts
  if (threadIdx.x == 0) {
    uint32_t eq_before = 0, sel_before = 0, my_take = 0, my_off = 0;
    for (int c = 0; c < C; ++c) {
      const uint32_t e = sh->counts[c][1];
      const uint32_t left = th.take_eq > eq_before ? th.take_eq - eq_before : 0u;
      const uint32_t take = all_eq ? 0u : (left < e ? left : e);
      if (c == rank) {
        my_take = take;
        my_off = sel_before;
      }
      sel_before += sh->counts[c][0] + take;
      eq_before += e;
    }
    // per-warp offsets inside this CTA
    uint32_t sel = my_off, eqr = 0;
    for (int w = 0; w < nw; ++w) {
      sh->off_w[w][0] = sel;
      sh->off_w[w][1] = eqr;
      const uint32_t left = my_take > eqr ? my_take - eqr : 0u;
      const uint32_t e = sh->cnt_w[w][1];
      sel += sh->cnt_w[w][0] + (left < e ? left : e);
      eqr += e;
    }
    sh->pad = my_take;
  }
  __syncthreads();
  sel_stamp(ts, 21);
  const uint32_t my_take = sh->pad;
  // pass 2: emit in index order
  uint32_t sel_run = sh->off_w[warp][0];
  uint32_t eq_run = sh->off_w[warp][1];
  const uint32_t ltmask = lanemask_lt();
  for (int ch = c0; ch < c1; ++ch) {
    const int i = ch * 32 + lane;
    const bool valid = i < n;
    const uint32_t k = valid ? key_at(i) : 0u;
    const bool gt = valid && (all_eq ? k >= th.t : k > th.t);
    const bool eq = valid && !all_eq && k == th.t;
    const uint32_t meq = __ballot_sync(FULL, eq);
    const bool take = gt || (eq && (eq_run + __popc(meq & ltmask)) < my_take);
    const uint32_t msel = __ballot_sync(FULL, take);
    if (take) emit(sel_run + __popc(msel & ltmask), i);
    sel_run += __popc(msel);
    eq_run += __popc(meq);
  }
  __syncthreads();
}

}  // namespace hst
