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
  uint32_t coarse[SEL_MAX_C][64]; // binned path: coarse histogram sums of every CTA of the cluster
  uint32_t over[SEL_MAX_C];      // binned path: keys above the bins' range, per CTA
  uint32_t selc[SEL_MAX_C];      // binned path: selected boundary candidates of every CTA
  uint32_t over_local;           // binned path: this CTA's keys above the range
  uint32_t ncand;                // binned path: boundary candidates of this CTA
  uint32_t pad2[2];
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
    ts[blockIdx.x * 24 + phase] = (unsigned long long)clock64();
  }
}

// Threshold of the pair, identical in every CTA of the cluster.
struct SelThreshold {
  uint32_t t;        // keys > t are selected
  uint32_t take_eq;  // keys == t: the first take_eq of them in index order (UINT_MAX: all)
};

// The three-level search (bins resolved as if by NT threads per CTA: 2048 / NT
// bins per thread). hist[0] holds this CTA's level-0 histogram and the
// cluster has synchronised since it was filled; hist[1], hist[2] are zeroed.
// pass(shift, bits, pshift, prefix, hist) counts this CTA's keys that match
// the prefix into the level's histogram, as histogram_pass does.
template <int NT, typename Pass>
__device__ SelThreshold cluster_threshold_by(Pass pass, uint32_t* const* hist, uint32_t k, int C, SelShared* sh,
                                             unsigned long long* ts = nullptr) {
  uint32_t need = k;
  uint32_t prefix = 0;
  int pshift = 32;
  SelThreshold th;
#pragma unroll
  for (int lvl = 0; lvl < SEL_LEVELS; ++lvl) {
    if (lvl > 0) {
      pass(sel_shift(lvl), sel_bits(lvl), pshift, prefix, hist[lvl]);
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

// cluster_threshold_by with the plain histogram pass over key_at(i), i < n_local.
template <int NT, typename KeyAt>
__device__ SelThreshold cluster_threshold(KeyAt key_at, int n_local, uint32_t* const* hist, uint32_t k, int C,
                                          SelShared* sh, unsigned long long* ts = nullptr) {
  auto pass = [&](int shift, int bits, int pshift, uint32_t prefix, uint32_t* h) {
    histogram_pass(key_at, n_local, shift, bits, pshift, prefix, h);
  };
  return cluster_threshold_by<NT>(pass, hist, k, C, sh, ts);
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


// ---------------------------------------------------------------- binned path
// The usual selection: while the scores are computed, every CTA counts its
// keys into a histogram of fixed bins (f32 keys: one bin per 2^16 bit
// patterns, i.e. 1/128 of an octave, over scores in [2^-16, 2^16); integer
// keys: one bin per value). At the barrier after scoring every CTA has pushed
// 64 coarse sums of its histogram and its count of keys above the range into
// every CTA of the cluster. One warp then finds the coarse bin, and within it
// (reading 64 fine bins of each CTA) the bin b* that holds the k-th largest
// key. Keys above b* are all taken; the keys of b* (few) are gathered from
// every CTA and ordered exactly (key descending, index ascending); the emit
// pass writes the selection in index order. If the k-th key is outside the
// range or b* holds more than BIN_CAND_CAP keys, the exact radix select above
// runs instead (the decision is the same in every CTA).
constexpr int BIN_COUNT = 4096;
constexpr int BIN_COARSE = 64;                 // coarse bins, of 64 fine bins each
constexpr int BIN_CAND_CAP = 256;
constexpr uint32_t BIN_F32_BASE = 111u << 7;   // (key >> 16) of the f32 2^-16

// Bin of a sort key: < 0 below the range, >= BIN_COUNT above it.
template <bool INT_KEYS>
__device__ __forceinline__ int key_bin(uint32_t key) {
  if (INT_KEYS) return (int)min(key, (uint32_t)BIN_COUNT);
  return (int)(key >> 16) - (int)BIN_F32_BASE;
}

// Smallest and largest key of bin b.
template <bool INT_KEYS>
__device__ __forceinline__ uint32_t bin_lo(int b) {
  return INT_KEYS ? (uint32_t)b : ((uint32_t)b + BIN_F32_BASE) << 16;
}
template <bool INT_KEYS>
__device__ __forceinline__ uint32_t bin_hi(int b) {
  return INT_KEYS ? (uint32_t)b : (((uint32_t)b + BIN_F32_BASE + 1u) << 16) - 1u;
}

// Counts one key into this CTA's histogram (BIN_COUNT words) or its
// above-range counter.
template <bool INT_KEYS>
__device__ __forceinline__ void bin_count(uint32_t key, uint32_t* hist, SelShared* sh) {
  const int b = key_bin<INT_KEYS>(key);
  if (b >= BIN_COUNT) atomicAdd(&sh->over_local, 1u);
  else if (b >= 0) atomicAdd(&hist[b], 1u);
}

// Words of scratch binned_select needs: own and gathered candidates, flags,
// per-thread counts.
__host__ __device__ constexpr int bin_scratch_words() { return 2 * BIN_CAND_CAP * 2 + BIN_CAND_CAP + 1024; }

// Stores this CTA's coarse sums and above-range count into every CTA of the
// cluster. Call with all 1024 threads after the histogram is complete and
// before the cluster barrier that follows scoring.
__device__ __forceinline__ void publish_coarse(const uint32_t* hist, int C, int rank, SelShared* sh) {
  const int t = threadIdx.x;
  uint32_t v = 0;
  if (t < BIN_COUNT / 4) {
    const uint4 q = reinterpret_cast<const uint4*>(hist)[t];
    v = q.x + q.y + q.z + q.w;
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(FULL, v, o);
  if ((t & 15) == 0 && t < BIN_COUNT / 4) {
    const uint32_t a = smem_u32(&sh->coarse[rank][t >> 4]);
    for (int c = 0; c < C; ++c) st_cluster_u32(mapa(a, (uint32_t)c), v);
  }
  if (t == 0) {
    const uint32_t a = smem_u32(&sh->over[rank]);
    for (int c = 0; c < C; ++c) st_cluster_u32(mapa(a, (uint32_t)c), sh->over_local);
  }
}

// One warp: over 64 bins in descending order (bin = hi - 2 * lane - j, j < 2,
// counts cnt(bin)), finds the bin holding the need-th key after `before`
// keys. Returns true and sets (bin, before keys above it, its count) if found.
__device__ __forceinline__ bool warp_pick_desc(uint32_t c_hi, uint32_t c_lo, uint32_t before, uint32_t need, int hi,
                                               int& bin, uint32_t& above, uint32_t& cnt) {
  const int lane = threadIdx.x & 31;
  const uint32_t pair = c_hi + c_lo;
  uint32_t incl = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(FULL, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t ex = before + incl - pair;
  const bool in_hi = ex < need && need <= ex + c_hi;
  const bool in_lo = !in_hi && ex + c_hi < need && need <= ex + pair;
  const uint32_t m = __ballot_sync(FULL, in_hi || in_lo);
  if (m == 0u) return false;
  const int src = __ffs(m) - 1;
  const int b = in_hi ? hi - 2 * lane : hi - 2 * lane - 1;
  const uint32_t a = in_hi ? ex : ex + c_hi;
  const uint32_t c = in_hi ? c_hi : c_lo;
  bin = __shfl_sync(FULL, b, src);
  above = __shfl_sync(FULL, a, src);
  cnt = __shfl_sync(FULL, c, src);
  return true;
}

template <typename KeyAddr>
__device__ __forceinline__ uint4 lds_key4(KeyAddr key_addr, int i) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(key_addr(i)));
  return v;
}

// Returns false (having changed nothing) when the exact radix path must run
// instead. key_at(i) / key_addr(i): local key i < n and its shared address
// (keys are read four at a time from 128-key chunks, which lie in one
// contiguous 16-byte aligned run; keys past n up to the chunk end must be 0,
// which is below every bin of f32 keys). hist: this CTA's histogram, at the same offset in every CTA.
// g0_of(c): first global index of CTA c. emit(pos, i) as in ordered_compact.
// scratch: bin_scratch_words() words, the same offset in every CTA. The
// cluster has synchronised since publish_coarse.
// Ordered compaction with a tie quota, thread-contiguous: keys > th.t (>= t
// when th.take_eq is all) are taken, and of the keys == t the first
// th.take_eq in index order across the cluster. Each thread owns `gpt`
// consecutive groups of 4 keys (keys past n up to the 128-key chunk must not
// compare above t); one block scan of packed (greater, equal) counts gives the
// positions. Writes the pair's list through `stage` (stage_cap words) when
// this CTA's part fits, else with emit(pos, i). out: the pair's index list.
template <typename KeyAddr, typename G0Of, typename Emit>
__device__ void contiguous_compact(KeyAddr key_addr, int n, const SelThreshold& th, int C, int rank, G0Of g0_of,
                                   SelShared* sh, Emit emit, int* out, uint32_t k, uint32_t* stage,
                                   uint32_t stage_cap, unsigned long long* ts = nullptr) {
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const bool all_eq = th.take_eq == 0xffffffffu;
  const int ngroups = ((n + 127) & ~127) / 4;
  const int gpt = ((ngroups + (int)blockDim.x - 1) / (int)blockDim.x) | 1;
  const int g_begin = min(ngroups, tid * gpt), g_end = min(ngroups, g_begin + gpt);
  uint32_t n_gt = 0, n_eq = 0;
  for (int g = g_begin; g < g_end; ++g) {
    const uint4 q = lds_key4(key_addr, 4 * g);
    const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const bool valid = 4 * g + j < n;
      n_gt += (valid && (all_eq ? kv[j] >= th.t : kv[j] > th.t)) ? 1u : 0u;
      n_eq += (valid && !all_eq && kv[j] == th.t) ? 1u : 0u;
    }
  }
  // packed scan: greater counts in the low 16 bits, equal counts in the high
  const uint32_t mine = n_gt | (n_eq << 16);
  const uint32_t excl = block_exclusive_scan(mine, sh);
  if (tid == (int)blockDim.x - 1) {
    const uint32_t tot = excl + mine;
    sh->cnt_w[0][0] = tot & 0xffffu;
    sh->cnt_w[0][1] = tot >> 16;
  }
  __syncthreads();
  if (tid < C) {
    uint32_t* dst = cluster.map_shared_rank(&sh->counts[rank][0], (unsigned)tid);
    dst[0] = sh->cnt_w[0][0];
    dst[1] = sh->cnt_w[0][1];
  }
  sel_stamp(ts, 19);
  cluster_sync();
  sel_stamp(ts, 20);
  // this CTA's tie quota and first output position
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
  const uint32_t cta_cnt = sh->counts[rank][0] + my_take;
  const bool staged = cta_cnt <= stage_cap;
  const uint32_t ex_gt = excl & 0xffffu, ex_eq = excl >> 16;
  uint32_t pos = ex_gt + (ex_eq < my_take ? ex_eq : my_take);   // position inside this CTA's part
  uint32_t eq_seen = ex_eq;
  const int g0 = g0_of(rank);
  if (n_gt + n_eq > 0) {
    for (int g = g_begin; g < g_end; ++g) {
      const uint4 q = lds_key4(key_addr, 4 * g);
      const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = 4 * g + j;
        if (i >= n) continue;
        bool take = all_eq ? kv[j] >= th.t : kv[j] > th.t;
        if (!all_eq && kv[j] == th.t) take = eq_seen++ < my_take;
        if (take) {
          if (staged) stage[pos] = (uint32_t)(g0 + i);
          else emit(my_off + pos, i);
          ++pos;
        }
      }
    }
  }
  __syncthreads();
  if (staged) {
    for (uint32_t e = tid; e < cta_cnt; e += blockDim.x)
      if (my_off + e < k) out[my_off + e] = (int)stage[e];
  }
  sel_stamp(ts, 21);
}

// The selection is written to out[0..k) (the pair's index list, global
// index = g0_of(rank) + local index): through `stage` (stage_cap words of
// shared memory) and coalesced stores when this CTA's part fits, else with
// emit(pos, i) directly.
template <bool INT_KEYS, typename KeyAt, typename KeyAddr, typename G0Of, typename Emit>
__device__ bool binned_select(KeyAt key_at, KeyAddr key_addr, int n, uint32_t k, int C, int rank, G0Of g0_of,
                              const uint32_t* hist, SelShared* sh, uint32_t* scratch, Emit emit, int* out,
                              uint32_t* stage, uint32_t stage_cap, unsigned long long* ts = nullptr) {
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  uint2* own = reinterpret_cast<uint2*>(scratch);            // [BIN_CAND_CAP] (key, local index)
  uint2* all = own + BIN_CAND_CAP;                            // [BIN_CAND_CAP] (key, global index)
  uint32_t* flag = reinterpret_cast<uint32_t*>(all + BIN_CAND_CAP);
  // resolve (warp 0): coarse bins, then the fine bins of the chosen coarse bin
  if (warp == 0) {
    uint32_t over = 0, ch = 0, cl = 0;
    for (int c = 0; c < C; ++c) {
      over += sh->over[c];
      ch += sh->coarse[c][63 - 2 * lane];
      cl += sh->coarse[c][62 - 2 * lane];
    }
    int cb = -1, bstar = -1;
    uint32_t before = 0, ccnt = 0, above = 0, in_bin = 0;
    bool ok = over < k && warp_pick_desc(ch, cl, over, k, 63, cb, before, ccnt);
    if (ok) {
      const int f_hi = cb * 64 + 63 - 2 * lane;
      uint32_t fh = 0, fl = 0;
      for (int c = 0; c < C; ++c) {
        const uint32_t* h = cluster.map_shared_rank(hist, c);
        fh += h[f_hi];
        fl += h[f_hi - 1];
      }
      ok = warp_pick_desc(fh, fl, before, k, cb * 64 + 63, bstar, above, in_bin);
    }
    if (lane == 0) {
      sh->bin = ok ? (uint32_t)bstar : 0xffffffffu;
      sh->above = above;
      sh->total_in_bin = in_bin;
      sh->ncand = 0u;
    }
  }
  if (tid < SEL_MAX_C) sh->selc[tid] = 0u;
  __syncthreads();
  sel_stamp(ts, 19);
  if (sh->bin == 0xffffffffu) return false;                           // the k-th key is outside the range
  const int bstar = (int)sh->bin;
  const uint32_t above = sh->above, in_bin = sh->total_in_bin;
  if (!INT_KEYS && in_bin > (uint32_t)BIN_CAND_CAP) return false;     // too many keys at the boundary
  const uint32_t need = k - above;                                    // 1 <= need <= in_bin
  if (INT_KEYS) {
    // every key of bin b* has the value b*: take the first `need` of them in index order
    SelThreshold th;
    th.t = bin_lo<true>(bstar);
    th.take_eq = need == in_bin ? 0xffffffffu : need;   // whole bin: every key >= t
    contiguous_compact(key_addr, n, th, C, rank, g0_of, sh, emit, out, k, stage, stage_cap, ts);
    return true;
  }
  const uint32_t lo = bin_lo<false>(bstar), hi = bin_hi<false>(bstar);
  // Each thread owns `gpt` consecutive groups of 4 keys (gpt odd: the 16-byte
  // reads of a warp hit distinct banks); the tail up to the 128-key chunk
  // is 0. Pass 1 counts the keys above b* per thread and gathers this CTA's
  // candidates.
  uint32_t* cnt_t = flag + BIN_CAND_CAP;                     // [blockDim.x] per-thread counts
  const int ngroups = ((n + 127) & ~127) / 4;
  const int gpt = ((ngroups + (int)blockDim.x - 1) / (int)blockDim.x) | 1;
  const int g_begin = min(ngroups, tid * gpt), g_end = min(ngroups, g_begin + gpt);
  uint32_t n_above = 0;
  for (int gi = 0; gi < gpt; ++gi) {           // same trip count in every lane: the warp vote below
    const int g = g_begin + gi;
    const bool in = g < g_end;
    const uint4 q = in ? lds_key4(key_addr, 4 * g) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
    bool any = false;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      n_above += kv[j] > hi ? 1u : 0u;
      any |= kv[j] - lo <= hi - lo;            // lo <= key <= hi
    }
    if (__any_sync(FULL, any)) {               // rare: a boundary candidate
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (kv[j] - lo <= hi - lo) {
          const uint32_t slot = atomicAdd(&sh->ncand, 1u);
          if (slot < (uint32_t)BIN_CAND_CAP) own[slot] = make_uint2(kv[j], (uint32_t)(4 * g + j));
        }
      }
    }
  }
  cnt_t[tid] = n_above;
  n_above = __reduce_add_sync(FULL, n_above);
  if (lane == 0) sh->cnt_w[warp][0] = n_above;
  __syncthreads();
  if (tid < C) {
    uint32_t a = 0;
    for (int w = 0; w < nw; ++w) a += sh->cnt_w[w][0];
    uint32_t* dst = cluster.map_shared_rank(&sh->counts[rank][0], (unsigned)tid);
    dst[0] = a;
    dst[1] = sh->ncand;
  }
  sel_stamp(ts, 16);
  cluster_sync();
  sel_stamp(ts, 17);
  // gather every CTA's candidates (in_bin of them in total)
  const int m = (int)in_bin;
  for (int e = tid; e < m; e += blockDim.x) {
    int c = 0, off = 0;
    while (c < C - 1 && e >= off + (int)sh->counts[c][1]) off += (int)sh->counts[c++][1];
    const uint2 v = *cluster.map_shared_rank(own + (e - off), (unsigned)c);
    all[e] = make_uint2(v.x, (uint32_t)g0_of(c) + v.y);
    flag[e] = 0u;
  }
  __syncthreads();
  sel_stamp(ts, 20);
  // exact order among the candidates (key descending, then index ascending):
  // thread t counts, for candidate t % m, the candidates ahead of it among
  // j = t / m, t / m + stride, ... (all threads share the m * m comparisons)
  uint32_t* ahead_cnt = flag;                        // [m], zeroed by the gather
  {
    const int per = max(1, (int)blockDim.x / max(m, 1));   // threads per candidate
    const int e = tid % max(m, 1), part = tid / max(m, 1);
    if (m > 0 && part < per) {
      const uint2 me = all[e];
      uint32_t a = 0;
      for (int j = part; j < m; j += per) {
        const uint2 o = all[j];
        a += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1u : 0u;
      }
      if (a) atomicAdd(&ahead_cnt[e], a);
    }
  }
  __syncthreads();
  sel_stamp(ts, 21);
  // taken candidates of this CTA become all ones (> hi), the others 0 (< lo);
  // selc[c]: candidates taken in CTA c
  {
    int off = 0;
    for (int c = 0; c < rank; ++c) off += (int)sh->counts[c][1];
    const int mine = (int)sh->counts[rank][1];
    const uint32_t g0 = (uint32_t)g0_of(rank);
    for (int e = tid; e < m; e += blockDim.x) {
      const bool take = ahead_cnt[e] < need;
      if (take) {
        int c = 0, o = 0;
        while (c < C - 1 && e >= o + (int)sh->counts[c][1]) o += (int)sh->counts[c++][1];
        atomicAdd(&sh->selc[c], 1u);
      }
      if (e >= off && e < off + mine) {
        const uint32_t i = all[e].y - g0;
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(key_addr((int)i)), "r"(take ? 0xffffffffu : 0u) : "memory");
        if (take) atomicAdd(&cnt_t[((int)i / 4) / gpt], 1u);
      }
    }
  }
  __syncthreads();
  if (tid == 0) {                                   // read after the scan's barriers
    uint32_t run = 0;
    for (int c = 0; c < rank; ++c) run += sh->counts[c][0] + sh->selc[c];
    sh->bin = run;                                   // this CTA's first output position
  }
  sel_stamp(ts, 4);
  // output positions: exclusive scan of the per-thread counts
  const uint32_t mine_cnt = cnt_t[tid];
  const uint32_t excl = block_exclusive_scan(mine_cnt, sh);
  if (tid == (int)blockDim.x - 1) sh->total_in_bin = excl + mine_cnt;   // this CTA's count
  __syncthreads();
  sel_stamp(ts, 18);
  // pass 2: each thread writes its keys > hi in index order
  const uint32_t cta_base = sh->bin, cta_cnt = sh->total_in_bin;
  const bool staged = cta_cnt <= stage_cap;
  const int g0 = g0_of(rank);
  uint32_t pos = excl;
  if (mine_cnt > 0) {
    for (int g = g_begin; g < g_end; ++g) {
      const uint4 q = lds_key4(key_addr, 4 * g);
      const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (kv[j] > hi) {
          if (staged) stage[pos] = (uint32_t)(g0 + 4 * g + j);
          else emit(cta_base + pos, 4 * g + j);
          ++pos;
        }
      }
    }
  }
  __syncthreads();
  if (staged) {
    for (uint32_t e = tid; e < cta_cnt; e += blockDim.x)
      if (cta_base + e < k) out[cta_base + e] = (int)stage[e];
  }
  return true;
}

}  // namespace hst
