// Exact deterministic top-k across a thread-block cluster, SOCKET step 4
// (SOCKET technical summary, section 中核メカニズム：ソフト LSH, step 4:
// the top-k keys are chosen deterministically).
//
// The keys of one (batch, KV-head) pair are split over the C CTAs of a
// cluster; CTA c holds the 32-bit sort keys of its slice in shared memory.
// Sort keys are the bit patterns of non-negative f32 scores (monotone as
// unsigned integers) or small non-negative integers (hard-hash scores).
// Selection is a most-significant-digit radix select over up to three digit
// levels: every CTA histograms the digit of its keys that match the prefix
// found so far, the histograms are summed across the cluster through
// distributed shared memory, and the bin holding the k-th largest key is
// found by a descending scan. A level stops early when the whole bin is
// taken. The final level resolves exact ties: among keys equal to the
// threshold, the ones with the lowest key index are taken (CTAs hold
// ascending index ranges, so CTA order then lane order is index order).
// The chosen indices are written in ascending order.
#pragma once

#include "common.cuh"

namespace hst {

constexpr int SEL_MAX_C = 16;

// One digit level: key bits [shift, shift + bits).
struct DigitLevel {
  int shift;
  int bits;
};

// Broadcast results of the selection, in shared memory.
struct SelShared {
  uint32_t bin;                 // bin of the k-th largest key at the current level
  uint32_t above;               // cluster-wide count in bins above it
  uint32_t total_in_bin;        // cluster-wide count in the bin
  uint32_t warp_tmp[32];        // block-scan scratch
  uint32_t red[32][SEL_MAX_C];  // per-warp, per-CTA partial sums
  uint32_t above_c[SEL_MAX_C];  // per-CTA count above the bin (this level)
  uint32_t eq_c[SEL_MAX_C];     // per-CTA count in the bin (this level)
  uint32_t cnt_w[32][2];        // compaction: per-warp (greater, equal) counts
  uint32_t off_w[32][2];        // compaction: per-warp (selected, equal) offsets
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

// Cluster-wide resolution of one histogram level. hist_addr is the shared
// address of this CTA's histogram (nbins u32; the same offset in every CTA).
// need >= 1 keys are still to be taken among keys matching the prefix.
// Writes sh->bin / above / total_in_bin and, for every CTA c < C,
// sh->above_c[c] and sh->eq_c[c].
__device__ void resolve_level(uint32_t hist_addr, int nbins, uint32_t need, int C, SelShared* sh) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
  const int bpt = (nbins + nthr - 1) / nthr;          // bins per thread (descending order)
  if (tid == 0) {            // defaults, overwritten by the thread that holds the k-th key
    sh->bin = 0;
    sh->above = 0;
    sh->total_in_bin = 0;
  }
  uint32_t local = 0;
  for (int j = 0; j < bpt; ++j) {
    const int bin = nbins - 1 - (tid * bpt + j);
    if (bin >= 0) {
      for (int c = 0; c < C; ++c) local += ld_cluster_u32(mapa(hist_addr + 4u * bin, c));
    }
  }
  const uint32_t before = block_exclusive_scan(local, sh);
  if (before < need && need <= before + local) {
    uint32_t run = before;
    for (int j = 0; j < bpt; ++j) {
      const int bin = nbins - 1 - (tid * bpt + j);
      if (bin < 0) break;
      uint32_t tot = 0;
      for (int c = 0; c < C; ++c) tot += ld_cluster_u32(mapa(hist_addr + 4u * bin, c));
      if (run + tot >= need) {
        sh->bin = (uint32_t)bin;
        sh->above = run;
        sh->total_in_bin = tot;
        break;
      }
      run += tot;
    }
  }
  __syncthreads();
  const int bin_sel = min((int)sh->bin, nbins - 1);
  // per-CTA counts above the bin
  for (int c = 0; c < C; ++c) {
    uint32_t part = 0;
    for (int j = 0; j < bpt; ++j) {
      const int bin = nbins - 1 - (tid * bpt + j);
      if (bin > bin_sel) part += ld_cluster_u32(mapa(hist_addr + 4u * bin, c));
    }
    part = warp_sum(part);
    if (lane == 0) sh->red[warp][c] = part;
  }
  __syncthreads();
  if (tid < C) {
    uint32_t s = 0;
    for (int w = 0; w < nw; ++w) s += sh->red[w][tid];
    sh->above_c[tid] = s;
    sh->eq_c[tid] = ld_cluster_u32(mapa(hist_addr + 4u * bin_sel, tid));
  }
  __syncthreads();
}

// Histogram pass over this CTA's keys: keys whose bits above `lv.shift + lv.bits`
// ... i.e. (key >> pshift) == prefix are counted in bin (key >> lv.shift) & mask.
// pshift == 32 means "no prefix" (all keys).
template <typename KeyAt>
__device__ __forceinline__ void histogram_pass(KeyAt key_at, int n, DigitLevel lv, int pshift, uint32_t prefix,
                                               uint32_t* hist) {
  const uint32_t mask = (1u << lv.bits) - 1u;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t k = key_at(i);
    const bool match = pshift >= 32 ? true : ((k >> pshift) == prefix);
    if (match) atomicAdd(&hist[(k >> lv.shift) & mask], 1u);
  }
}

// Result of the cluster selection for this CTA.
struct SelPlan {
  uint32_t t;          // threshold key: select keys > t, and ties == t by rank
  uint32_t take_eq;    // ties == t this CTA takes (UINT_MAX: all)
  uint32_t out_off;    // position of this CTA's first selected key in the output
  uint32_t n_sel;      // keys this CTA selects
};

// Full selection over up to 3 levels. `hist[l]` are this CTA's zeroed
// histograms (u32, 1 << levels[l].bits bins); level 0 is filled by the caller
// before the cluster barrier that precedes this call (sync_before_first).
// k: keys to select for the pair (1 <= k <= total keys). rank: this CTA.
template <typename KeyAt>
__device__ SelPlan cluster_select(KeyAt key_at, int n_local, const DigitLevel* levels, int nlevels,
                                  uint32_t* const* hist, uint32_t k, int C, int rank, SelShared* sh) {
  uint32_t need = k;
  uint32_t prefix = 0;        // digits found so far (at the current level's granularity)
  int pshift = 32;
  uint32_t acc_above[SEL_MAX_C];
#pragma unroll
  for (int c = 0; c < SEL_MAX_C; ++c) acc_above[c] = 0;
  SelPlan plan;
  for (int lvl = 0; lvl < nlevels; ++lvl) {
    const DigitLevel lv = levels[lvl];
    if (lvl > 0) {
      histogram_pass(key_at, n_local, lv, pshift, prefix, hist[lvl]);
      __syncthreads();
      cluster_sync();
    }
    resolve_level(smem_u32(hist[lvl]), 1 << lv.bits, need, C, sh);
    const uint32_t bin = sh->bin;
    for (int c = 0; c < C; ++c) acc_above[c] += sh->above_c[c];
    need -= sh->above;
    prefix = (prefix << lv.bits) | bin;
    pshift = lv.shift;
    const bool whole = (need == sh->total_in_bin);
    if (whole || lvl == nlevels - 1) {
      // threshold = smallest key in the bin (whole) or the exact key (last level, shift 0)
      plan.t = prefix << lv.shift;
      uint32_t eq_before = 0, sel_before = 0;
      for (int c = 0; c < C; ++c) {
        uint32_t take;
        if (whole) {
          take = sh->eq_c[c];
        } else {
          const uint32_t left = need > eq_before ? need - eq_before : 0u;
          take = left < sh->eq_c[c] ? left : sh->eq_c[c];
        }
        const uint32_t sel_c = acc_above[c] + take;
        if (c == rank) {
          plan.out_off = sel_before;
          plan.n_sel = sel_c;
          plan.take_eq = whole ? 0xffffffffu : take;
        }
        sel_before += sel_c;
        eq_before += sh->eq_c[c];
      }
      break;
    }
  }
  return plan;
}

// Ordered compaction of this CTA's selected keys. Keys i in [0, n) with
// key > t, or key >= t when take_eq == UINT_MAX, or key == t among the first
// take_eq such keys in index order, are emitted in ascending i at output
// positions plan.out_off, plan.out_off + 1, ... via emit(pos, i).
template <typename KeyAt, typename Emit>
__device__ void ordered_compact(KeyAt key_at, int n, const SelPlan& plan, SelShared* sh, Emit emit) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const bool all_eq = plan.take_eq == 0xffffffffu;
  const int nchunks = (n + 31) / 32;
  const int per_warp = (nchunks + nw - 1) / nw;
  const int c0 = warp * per_warp;
  const int c1 = min(nchunks, c0 + per_warp);
  // pass 1: per-warp counts of (key > t) and (key == t)
  uint32_t n_gt = 0, n_eq = 0;
  for (int ch = c0; ch < c1; ++ch) {
    const int i = ch * 32 + lane;
    uint32_t k = 0;
    bool valid = i < n;
    if (valid) k = key_at(i);
    const bool gt = valid && (all_eq ? k >= plan.t : k > plan.t);
    const bool eq = valid && !all_eq && k == plan.t;
    n_gt += __popc(__ballot_sync(FULL, gt));
    n_eq += __popc(__ballot_sync(FULL, eq));
  }
  if (lane == 0) {
    sh->cnt_w[warp][0] = n_gt;
    sh->cnt_w[warp][1] = n_eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t sel = 0, eq = 0;
    for (int w = 0; w < nw; ++w) {
      sh->off_w[w][0] = sel;
      sh->off_w[w][1] = eq;
      const uint32_t left = all_eq ? 0u : (plan.take_eq > eq ? plan.take_eq - eq : 0u);
      const uint32_t e = sh->cnt_w[w][1];
      sel += sh->cnt_w[w][0] + (left < e ? left : e);
      eq += e;
    }
  }
  __syncthreads();
  // pass 2: emit in order
  uint32_t sel_run = sh->off_w[warp][0];
  uint32_t eq_run = sh->off_w[warp][1];
  const uint32_t ltmask = lanemask_lt();
  for (int ch = c0; ch < c1; ++ch) {
    const int i = ch * 32 + lane;
    uint32_t k = 0;
    const bool valid = i < n;
    if (valid) k = key_at(i);
    const bool gt = valid && (all_eq ? k >= plan.t : k > plan.t);
    const bool eq = valid && !all_eq && k == plan.t;
    const uint32_t meq = __ballot_sync(FULL, eq);
    const bool take = gt || (eq && (eq_run + __popc(meq & ltmask)) < plan.take_eq);
    const uint32_t msel = __ballot_sync(FULL, take);
    if (take) emit(plan.out_off + sel_run + __popc(msel & ltmask), i);
    sel_run += __popc(msel);
    eq_run += __popc(meq);
  }
  __syncthreads();
}

}  // namespace hst
