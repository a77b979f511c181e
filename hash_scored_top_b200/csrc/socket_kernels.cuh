// SOCKET decode kernels: the fused one-launch decode step and the unfused
// chain (bucket table -> scores -> top-k -> sparse attention -> merge),
// plus dense decode attention. See table.cuh, score.cuh, select.cuh and
// attend.cuh for the steps.
#pragma once

#include <cooperative_groups.h>

#include "attend.cuh"
#include "common.cuh"
#include "hash_kernels.cuh"
#include "score.cuh"
#include "select.cuh"
#include "table.cuh"

namespace hst {

namespace cg = cooperative_groups;

// ---------------------------------------------------------------- shared constants
constexpr int SMEM_BASE_EXPECTED = 1024;         // dynamic shared window start on sm_100
constexpr int SMEM_DYN_MAX = 232448;             // 227 KB opt-in per block
__host__ __device__ constexpr int hist_words(int level) { return 1 << sel_bits(level); }
constexpr int FUSED_THREADS = 1024;              // 32 warps: enough loads in flight to stream HBM
constexpr int FUSED_WARPS = FUSED_THREADS / 32;
// 32-key blocks in flight per warp while scoring (a third one measured no
// faster at 32-byte rows and spills at longer ones: registers are capped at 64)
template <int LP>
__host__ __device__ constexpr int score_pf() { return 2; }
constexpr uint32_t SCORE_L2_PREFETCH = 96u * 1024u;   // bytes of each CTA's key slice prefetched into L2
constexpr uint32_t NEXT_L2_PREFETCH = 512u * 1024u;   // bytes of ID rows prefetched for the next wave's CTA
constexpr int ATTEND_THREADS = 256;              // the attention kernel
constexpr int ATTEND_WARPS = ATTEND_THREADS / 32;
constexpr int ATTEND_BUFS = 2;                    // bf16: K/V slots per computing warp
constexpr int ATTEND_MMA_WARPS = 6;               // bf16: computing warps
constexpr int ATTEND_SLOTS = ATTEND_MMA_WARPS * ATTEND_BUFS > ATTEND_WARPS ? ATTEND_MMA_WARPS * ATTEND_BUFS
                                                                           : ATTEND_WARPS;
constexpr int ATTEND_MAX_SPLITS = 128;           // one head's partials fit in the warp slots

__device__ __forceinline__ uint32_t key_of(float s) { return __float_as_uint(s); }

static_assert(bin_scratch_words() * 4 <= TABLE_BYTES, "the selection scratch lives in the first table");
static_assert(hist_words(0) + hist_words(1) >= BIN_COUNT, "the selection bins live in the first two radix histograms");
static_assert(FUSED_THREADS * 4 == BIN_COUNT, "publish_coarse reads four bins per thread");
static_assert(ATTEND_MMA_WARPS <= ATTEND_WARPS && ATTEND_SLOTS <= 32, "one mbarrier and phase word per slot");

__host__ __device__ constexpr int table_chunks(int LP) { return LP > 32 ? 2 : 1; }

struct FusedParams {
  const void* Q;
  const void* K;
  const void* V;
  const __nv_bfloat16* R;
  const uint8_t* ids;
  const __half* norms;
  float* O;
  int* idx_out;                   // [pairs][k] ascending (always written)
  unsigned int* counters;         // [pairs] zeroed here for the attention kernel's merge (may be null)
  unsigned long long* phase_ts;   // optional: [grid][PHASES] clock stamps (profiling)
  int Hq, Hkv, Ncap, N, L, P, k, C, blocks_per_cta, chunk;
  float tau, scale;
  // units per cache pair: 1 (one index set per KV head), or G when every
  // query head is its own unit (Hkv then counts query heads); the cached
  // IDs, norms, keys and values of unit u are those of pair u / pair_div
  int pair_div = 1;
  // optional: the units' table images [units][nch][256][64], built by a
  // table kernel beforehand (bucket_table_kernel / hamming_table_kernel);
  // every CTA copies its unit's image instead of building tables
  const float* tables = nullptr;
  // CTAs of one wave when the grid runs in several (0: one wave): once it has
  // scored its slice, CTA b asks for CTA b + next_stride's slice in L2, so the
  // next wave's reads overlap this wave's selection
  int next_stride = 0;
};

constexpr int PHASES = 24;

// Profiling stamps (see sk_profile_phases): the SM clock at each phase, and
// the global timer at the start (slot 22) and the exit (slot 23).
__device__ __forceinline__ void stamp(unsigned long long* ts, int phase) {
  if (ts != nullptr && threadIdx.x == 0) {
    ts[blockIdx.x * PHASES + phase] = (unsigned long long)clock64();
    if (phase == 0 || phase == 7) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      ts[blockIdx.x * PHASES + 22 + (phase == 7)] = t;
    }
  }
}

// Where the sort keys of a CTA live: the first nA in segment A, the rest in B.
struct FusedKeys {
  uint32_t keysA, nA, keysB;
  __device__ __forceinline__ uint32_t addr(uint32_t i) const { return i < nA ? keysA + 4u * i : keysB + 4u * (i - nA); }
};

// Shared-memory plan of the selection kernel (addresses are shared-window
// addresses). The nch tables (64 KB each) start at the first 64 KB-aligned
// address; segment A lies before them, segment B after. The selection state
// and histograms open segment A; sort keys fill the rest of A, then B.
struct FusedSmem {
  uint32_t base, tbl0, tbl1, segA_end, segB, segB_end;
  uint32_t sel, hist0, hist1, hist2;
  uint32_t keysA, nA, keysB;
  __device__ void plan(uint32_t dyn_base, uint32_t dyn_size, int nch) {
    base = dyn_base;
    tbl0 = (dyn_base + 65535u) & ~65535u;
    tbl1 = tbl0 + TABLE_BYTES;
    segA_end = tbl0;
    segB = tbl0 + (uint32_t)nch * TABLE_BYTES;
    segB_end = dyn_base + dyn_size;
    uint32_t a = dyn_base;
    sel = a;   a += (sizeof(SelShared) + 15u) & ~15u;
    hist0 = a; a += 4u * hist_words(0);
    hist1 = a; a += 4u * hist_words(1);
    hist2 = a; a += 4u * hist_words(2);
    keysA = a;
    nA = (segA_end > a) ? ((segA_end - a) / 4u) & ~127u : 0u;   // whole 128-key chunks
    keysB = segB;
  }
  __device__ uint32_t key_capacity() const { return nA + (segB_end > segB ? (segB_end - segB) / 4u : 0u); }
  __device__ __forceinline__ FusedKeys keys() const { return FusedKeys{keysA, nA, keysB}; }
};

template <typename T>
__device__ __forceinline__ T* sptr(unsigned char* dyn, uint32_t base, uint32_t addr) {
  return reinterpret_cast<T*>(dyn + (addr - base));
}

// Zeroes every copy of the padding cells of the chunk tables: rows >= 2^P
// and columns whose table is >= L. The other cells are written by the table
// build of the cluster.
template <int LP>
__device__ __forceinline__ void zero_table_padding_all(float* t0, float* t1, int L, int P) {
  const int nb = 1 << P;
#pragma unroll
  for (int c = 0; c < table_chunks(LP); ++c) {
    float* t = c ? t1 : t0;
    const int S = id_chunk_size(L, c);
    if (nb == 256 && 32 * c + S <= L) continue;       // no padding in this chunk
    for (int e = threadIdx.x; e < 256 * TABLE_COLS; e += blockDim.x) {
      const int b = e / TABLE_COLS, x = e % TABLE_COLS;
      if (b >= nb || 32 * c + x % S >= L) t[e] = 0.f;
    }
  }
}

// Scores keys of blocks blk0 + warp + i * NW (i < nb) into sort keys in
// shared memory and counts them into the CTA's selection histogram. buf holds
// the first score_pf<LP>() blocks, already requested.
template <int LP, bool NORM>
__device__ __forceinline__ void score_blocks(KeyIds<LP> (&buf)[score_pf<LP>()], const uint8_t* __restrict__ ids_pair,
                                             const __half* __restrict__ norms_pair, int N, int blk0, int nb,
                                             uint32_t col0, uint32_t col1, const FusedKeys keys, uint32_t* hist,
                                             SelShared* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int it = 0; it < nb; it += score_pf<LP>()) {
#pragma unroll
    for (int u = 0; u < score_pf<LP>(); ++u) {
      const int i = it + u;
      if (i < nb) {
        const KeyIds<LP> cur = buf[u];
        if (i + score_pf<LP>() < nb) {
          const int key = (blk0 + warp + (i + score_pf<LP>()) * nw) * 32 + lane;
          load_key_ids<LP, NORM>(buf[u], ids_pair + (size_t)key * LP, norms_pair + key);
        }
        const float s = score_key<LP, NORM>(cur, col0, col1);
        const int gkey = (blk0 + warp + i * nw) * 32 + lane;
        if (gkey < N) {
          // soft scores sort by their f32 bits; hard-hash scores are small integers
          const uint32_t key = NORM ? key_of(s) : (uint32_t)s;
          const uint32_t li = (uint32_t)(gkey - blk0 * 32);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(keys.addr(li)), "r"(key) : "memory");
          bin_count<!NORM>(key, hist, sh);
        }
      }
    }
  }
}

template <int LP, bool NORM>
__device__ __forceinline__ void prefetch_blocks(KeyIds<LP> (&buf)[score_pf<LP>()], const uint8_t* __restrict__ ids_pair,
                                                const __half* __restrict__ norms_pair, int blk0, int nb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int u = 0; u < score_pf<LP>(); ++u) {
    if (u < nb) {
      const int key = (blk0 + warp + u * nw) * 32 + lane;
      load_key_ids<LP, NORM>(buf[u], ids_pair + (size_t)key * LP, norms_pair + key);
    }
  }
}

// Shared-memory plan of the attention stage: query stage, one mbarrier and
// phase word per slot, K/V slots (computing warp w owns slots w * nbuf ..;
// its partial goes into its first slot once its keys are done), the CTA's
// merged result.
struct AttendSmem {
  uint32_t qs;             // query rows (bf16 path)
  uint32_t mbar0;          // 8 bytes per slot
  uint32_t phases;         // 4 bytes per slot
  uint32_t slot0;          // slot s: slot0 + s * slot_stride
  uint32_t slot_stride;
  int ncw;                 // computing warps (one partial each)
  int nbuf;                // slots per computing warp
  uint32_t result;         // merged (M[G], L[G], O[G][D])
};

// Exact attention of cnt keys (keys(i), i < cnt) into merged per-CTA results
// (cM, cL, cO) using warps 0..ncw-1; all threads call it. For bf16 the caller
// has staged Q at as.qs, initialised the slot mbarriers and zeroed phases.
template <int D, typename KVT, typename KeyFn>
__device__ __forceinline__ void attend_and_merge(unsigned char* dyn, uint32_t base, const AttendSmem& as,
                                                 const KVT* Qg, const KVT* Kp, const KVT* Vp, int G, float scale,
                                                 KeyFn keys, int cnt, int nrows, float*& cM, float*& cL, float*& cO) {
  const int ncw = as.ncw;
  const PartialView pv = partial_view(sptr<float>(dyn, base, as.slot0), (int)(as.nbuf * as.slot_stride / 4u), G, D);
  cM = sptr<float>(dyn, base, as.result);
  cL = cM + G;
  cO = cL + G;
  if constexpr (sizeof(KVT) == 2) {
    attend_tiles_bf16<D, ATTEND_BUFS>(reinterpret_cast<const __nv_bfloat16*>(Kp),
                                      reinterpret_cast<const __nv_bfloat16*>(Vp), keys, cnt, nrows, G, scale, as.qs,
                                      as.slot0, as.slot_stride, as.mbar0, sptr<uint32_t>(dyn, base, as.phases), ncw,
                                      pv);
  } else {
    attend_keys_f32<D>(reinterpret_cast<const float*>(Qg), reinterpret_cast<const float*>(Kp),
                       reinterpret_cast<const float*>(Vp), keys, cnt, nrows, G, scale, ncw, pv);
  }
  __syncthreads();
  merge_partials(pv, ncw, cM, cL, cO);
}

// Sets up the attention stage: stages Q (bf16), initialises one mbarrier per
// slot and zeroes the phase words. Ends with __syncthreads().
template <int D, typename KVT>
__device__ __forceinline__ void attend_setup(unsigned char* dyn, uint32_t base, const AttendSmem& as, const KVT* Qg,
                                             int G) {
  if constexpr (sizeof(KVT) == 2) {
    stage_q<D>(reinterpret_cast<const __nv_bfloat16*>(Qg), G, sptr<unsigned char>(dyn, base, as.qs));
    if ((int)threadIdx.x < as.ncw * as.nbuf) {
      mbar_init(as.mbar0 + 8u * threadIdx.x, 1);
      sptr<uint32_t>(dyn, base, as.phases)[threadIdx.x] = 0u;
    }
    if (threadIdx.x == 0) fence_mbar_init();
  }
  __syncthreads();
}

// ---------------------------------------------------------------- selection kernel
// One cluster of C CTAs per (batch, KV-head) pair; grid = pairs * C. CTA r
// scores the keys of blocks [r * blocks_per_cta, ...); the cluster then finds
// the exact top-k and writes the pair's ascending index list to p.idx_out.
// HATA = false: SOCKET soft-LSH scores from the ids/norms cache.
// HATA = true: hard-hash scores from 128-bit codes (16 byte-tables, no norm);
// R holds the 128 code hyperplanes and ids the codes.
template <int D, int LP, typename QT, bool HATA>
__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_select_kernel(const FusedParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int NCH = table_chunks(LP);
  const int C = p.C;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x / C;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint32_t dyn_size;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  FusedSmem fs;
  fs.plan(smem_u32(dyn), dyn_size, NCH);
  // The host sizes slices from the same plan; a mismatch (a host bug) is
  // flagged and every CTA of the grid leaves here (the test is uniform).
  if (fs.segB > fs.segB_end || (((uint32_t)p.blocks_per_cta * 32u + 127u) & ~127u) > fs.key_capacity()) {
    if (tid == 0) atomicOr(&g_error_word, ERR_LAYOUT);
    return;
  }
  stamp(p.phase_ts, 0);
  SelShared* sh = sptr<SelShared>(dyn, fs.base, fs.sel);
  uint32_t* hist[3] = {sptr<uint32_t>(dyn, fs.base, fs.hist0), sptr<uint32_t>(dyn, fs.base, fs.hist1),
                       sptr<uint32_t>(dyn, fs.base, fs.hist2)};
  float* tab0 = sptr<float>(dyn, fs.base, fs.tbl0);
  float* tab1 = sptr<float>(dyn, fs.base, fs.tbl1);
  uint32_t* tab0u = sptr<uint32_t>(dyn, fs.base, fs.tbl0);   // selection scratch once scoring is done

  const int nblk_pair = (p.N + 31) / 32;
  const int blk0 = min(nblk_pair, rank * p.blocks_per_cta);
  const int blk1 = min(nblk_pair, blk0 + p.blocks_per_cta);
  const int n_local = max(0, min(p.N, blk1 * 32) - blk0 * 32);
  const int nb = max(0, (blk1 - blk0 - warp + FUSED_WARPS - 1) / FUSED_WARPS);
  const size_t pair_keys = (size_t)(pair / p.pair_div) * p.Ncap;
  const uint8_t* ids_pair = p.ids + pair_keys * LP;
  const __half* norms_pair = p.norms + pair_keys;

  // ---- setup. The cluster barrier is split: this arrive, and the wait just
  // before the first store into another CTA (the tables), so the barrier's
  // latency hides behind the table build.
  cluster_arrive_relaxed();
  if (warp == 1 && blk1 > blk0) {
    // the first SCORE_L2_PREFETCH bytes of this CTA's slice stream into L2
    // while the tables are built (more only delays the table's own loads)
    constexpr uint32_t kChunk = 32768u;
    const uint32_t slice = (uint32_t)(blk1 - blk0) * 32u;               // keys
    const uint32_t want = min(slice, SCORE_L2_PREFETCH / (LP + 2u)) & ~31u;
    const char* ids0 = reinterpret_cast<const char*>(ids_pair + (size_t)blk0 * 32 * LP);
    const uint32_t ids_bytes = want * LP;
    for (uint32_t off = (uint32_t)lane * kChunk; off < ids_bytes; off += 32u * kChunk)
      prefetch_l2_bulk(ids0 + off, min(kChunk, ids_bytes - off));
    if (!HATA && lane == 31 && want > 0) prefetch_l2_bulk(norms_pair + (size_t)blk0 * 32, want * 2u);
  }
  if (tid == 0) sh->over_local = 0u;
  for (int i = tid; i < BIN_COUNT; i += blockDim.x) hist[0][i] = 0u;     // hist0 + hist1: the selection bins
  if (p.tables == nullptr) zero_table_padding_all<LP>(tab0, tab1, p.L, p.P);   // a copied image has its zeros
  if (rank == 0 && tid == 0 && p.counters) p.counters[pair] = 0u;     // for the attention kernel's merge
  stamp(p.phase_ts, 8);

  // ---- SOCKET step 2: this CTA builds a range of tables (4-table aligned) and
  // stores every entry into all its column copies in every CTA of the cluster.
  const QT* Qg = reinterpret_cast<const QT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  const int per = ((p.L + C - 1) / C + 3) & ~3;
  if (p.tables != nullptr) {
    // precomputed: this CTA copies its unit's image (L2-resident) into its
    // own tables; no table entry crosses CTAs
    const uint4* src = reinterpret_cast<const uint4*>(p.tables + (size_t)pair * NCH * 256 * TABLE_COLS);
    uint4* dst = reinterpret_cast<uint4*>(tab0);           // tab1 follows tab0 directly
    for (int e = tid; e < NCH * 256 * TABLE_COLS / 4; e += blockDim.x) dst[e] = __ldg(src + e);
    cluster_wait();                                          // pairs with the arrive at entry
  } else {
    const int l0 = min(p.L, rank * per);
    const int nl = min(p.L, l0 + per) - l0;
    const uint32_t t0a = fs.tbl0, t1a = fs.tbl1;
    const int L = p.L;
    auto store = [=](int bb, int l, float v) {
      const int c = l >= 32 ? 1 : 0;
      const int S = id_chunk_size(L, c);
      const uint32_t row = (c ? t1a : t0a) + (uint32_t)bb * (TABLE_COLS * 4u);
      for (int x = l - 32 * c; x < TABLE_COLS; x += S)
        for (int r = 0; r < C; ++r) st_cluster_f32(mapa(row + 4u * x, (uint32_t)r), v);
    };
    // groups of 4 tables (4-aligned, inside one chunk): one 16-byte store per copy
    auto store4 = [=](int bb, int l, const float* v, int cnt) {
      if (cnt < 4) {
        for (int q = 0; q < cnt; ++q) store(bb, l + q, v[q]);
        return;
      }
      const int c = l >= 32 ? 1 : 0;
      const int S = id_chunk_size(L, c);
      const uint32_t row = (c ? t1a : t0a) + (uint32_t)bb * (TABLE_COLS * 4u);
      for (int x = l - 32 * c; x < TABLE_COLS; x += S)
        for (int r = 0; r < C; ++r) st_cluster_v4f32(mapa(row + 4u * x, (uint32_t)r), v);
    };
    auto before_store = [] { cluster_wait(); };    // every CTA of the cluster has started
    void* scratch = sptr<void>(dyn, fs.base, fs.keysA);
    if constexpr (HATA) {
      // the 16 byte-tables of the hard-hash variant (popcounts of the query
      // codes): every CTA builds all of them in its own memory (about 13 us;
      // decodes of several waves copy them from a table kernel's image instead)
      auto local_store = [=](int bb, int l, float v) {
        float* row = tab0 + bb * TABLE_COLS;
        for (int x = l; x < TABLE_COLS; x += 16) row[x] = v;
      };
      // scratch in segment B (the keys are not written yet): the 128 staged
      // hyperplane rows do not fit segment A
      build_hamming_table<D>(Qg, G, p.R, 0, p.L, sptr<void>(dyn, fs.base, fs.segB), local_store, before_store);
    } else if (nl <= 0) {
      cluster_wait();
    } else {
      // doubles in segment A, staged hyperplane rows in segment B (neither
      // holds keys yet)
      build_bucket_table<D, QT, decltype(store4), decltype(before_store), 4>(Qg, G, p.R, p.P, p.tau, l0, nl, scratch,
                                                                            store4, p.phase_ts, before_store,
                                                                            sptr<void>(dyn, fs.base, fs.segB));
    }
  }
  stamp(p.phase_ts, 9);
  if (p.tables != nullptr) {
    __syncthreads();                       // this CTA's copy is complete
  } else if constexpr (!HATA) {
    cluster_sync();                        // every table entry has landed in every CTA
  }
  // Launched as the programmatic dependent of the key-append kernel, the
  // kernel got here while that kernel may still run: the bucket IDs and norms
  // are read only after it completed (a no-op for an ordinary launch).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  KeyIds<LP> buf[score_pf<LP>()];
  prefetch_blocks<LP, !HATA>(buf, ids_pair, norms_pair, blk0, nb);
  stamp(p.phase_ts, 1);

  // ---- SOCKET step 3: scores of this CTA's slice, kept on chip
  const FusedKeys keys = fs.keys();
  score_blocks<LP, !HATA>(buf, ids_pair, norms_pair, p.N, blk0, nb, fs.tbl0 + 4u * lane, fs.tbl1 + 4u * lane, keys,
                          hist[0], sh);
  stamp(p.phase_ts, 11);
  if (p.next_stride > 0 && warp == 1) {
    // the slice of the CTA one wave later (same rank arithmetic as above)
    const int nx = (int)blockIdx.x + p.next_stride;
    if (nx < (int)gridDim.x) {
      const int nb0 = min(nblk_pair, (nx % C) * p.blocks_per_cta);
      const int nb1 = min(nblk_pair, nb0 + p.blocks_per_cta);
      if (nb1 > nb0) {
        constexpr uint32_t kChunk = 32768u;
        const size_t npk = (size_t)((nx / C) / p.pair_div) * p.Ncap + (size_t)nb0 * 32;
        const uint32_t keys_n = min((uint32_t)(nb1 - nb0) * 32u, NEXT_L2_PREFETCH / LP) & ~31u;   // 16-byte sizes
        const char* src = reinterpret_cast<const char*>(p.ids + npk * LP);
        const uint32_t bytes = keys_n * LP;
        for (uint32_t off = (uint32_t)lane * kChunk; off < bytes; off += 32u * kChunk)
          prefetch_l2_bulk(src + off, min(kChunk, bytes - off));
        if (!HATA && lane == 31) prefetch_l2_bulk(p.norms + npk, keys_n * 2u);
      }
    }
  }
  // keys past the slice, up to its last 128-key chunk, read as 0
  if (warp == 0) {
    const int tail_end = (n_local + 127) & ~127;
    for (int i = n_local + lane; i < tail_end; i += 32)
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(keys.addr((uint32_t)i)), "r"(0u) : "memory");
  }
  __syncthreads();
  publish_coarse(hist[0], C, rank, sh);
  cluster_sync();     // every CTA's scores and histogram sums are final; the tables are no longer read
  stamp(p.phase_ts, 2);

  // ---- SOCKET step 4a: exact top-k across the cluster, ascending indices to idx_out
  auto key_at = [=](int i) -> uint32_t { return lds_u32(keys.addr((uint32_t)i)); };
  auto key_addr = [=](int i) -> uint32_t { return keys.addr((uint32_t)i); };
  const int bpc = p.blocks_per_cta;
  auto g0_of = [=](int c) -> int { return min(nblk_pair, c * bpc) * 32; };
  int* idx_out = p.idx_out + (size_t)pair * p.k;
  const int kk = p.k, g0 = blk0 * 32;
  auto emit = [=](uint32_t pos, int i) {
    if (pos < (uint32_t)kk) idx_out[pos] = g0 + i;
  };
  const bool done = binned_select<HATA>(key_at, key_addr, n_local, (uint32_t)p.k, C, rank, g0_of, hist[0], sh, tab0u,
                                       emit, idx_out, tab0u + bin_scratch_words(),
                                       (uint32_t)(TABLE_BYTES / 4 - bin_scratch_words()), p.phase_ts);
  if (!done) {
    // exact radix select over the whole key range; every CTA has finished
    // reading the other CTAs' bins before any reuses its own
    cluster_sync();
    for (int i = tid; i < hist_words(0); i += blockDim.x) hist[0][i] = 0u;
    for (int i = tid; i < hist_words(1); i += blockDim.x) hist[1][i] = 0u;
    for (int i = tid; i < hist_words(2); i += blockDim.x) hist[2][i] = 0u;
    __syncthreads();
    histogram_pass(key_at, n_local, sel_shift(0), sel_bits(0), 32, 0u, hist[0]);
    __syncthreads();
    cluster_sync();
    const SelThreshold th = cluster_threshold<FUSED_THREADS>(key_at, n_local, hist, (uint32_t)p.k, C, sh,
                                                             p.phase_ts);
    stamp(p.phase_ts, 3);
    ordered_compact(key_at, n_local, th, C, rank, sh, emit, p.phase_ts);
  }
  stamp(p.phase_ts, 12);
  // the attention kernel may start once every CTA has written its indices
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  cluster_sync();   // peers may still read this CTA's shared memory until here
  stamp(p.phase_ts, 7);
}

// ---------------------------------------------------------------- unfused chain
struct TableParams {
  const void* Q;
  const __nv_bfloat16* R;
  float* T;            // [pairs][nch][256][64], the shared-memory table image
  int Hq, Hkv, L, P;
  float tau;
};

// grid = (pairs, ny): CTA y computes a contiguous range of tables and writes
// every copy of its entries; CTA y = 0 also writes the zero padding.
template <int D, int LP, typename QT>
__global__ void __launch_bounds__(256) bucket_table_kernel(const TableParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  constexpr int NCH = table_chunks(LP);
  const int pair = blockIdx.x;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const QT* Qg = reinterpret_cast<const QT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  float* T = p.T + (size_t)pair * NCH * 256 * TABLE_COLS;
  if (blockIdx.y == 0) {
    const int nbk = 1 << p.P;
    for (int e = threadIdx.x; e < NCH * 256 * TABLE_COLS; e += blockDim.x) {
      const int c = e / (256 * TABLE_COLS), bb = (e / TABLE_COLS) % 256, x = e % TABLE_COLS;
      if (bb >= nbk || column_table(p.L, c, x) >= p.L) T[e] = 0.f;
    }
  }
  const int per = (p.L + gridDim.y - 1) / gridDim.y;
  const int l0 = min(p.L, (int)blockIdx.y * per);
  const int nl = min(p.L, l0 + per) - l0;
  if (nl <= 0) return;
  build_bucket_table<D>(Qg, G, p.R, p.P, p.tau, l0, nl, reinterpret_cast<double*>(dyn),
                        [&](int bb, int l, float v) {
                          const int c = l >= 32 ? 1 : 0;
                          const int S = id_chunk_size(p.L, c);
                          float* row = T + ((size_t)c * 256 + bb) * TABLE_COLS;
                          for (int x = l - 32 * c; x < TABLE_COLS; x += S) row[x] = v;
                        });
}

// The hard-hash variant's 16 byte-tables of a pair into its table image (one
// 64-column chunk, table m in columns m, m + 16, m + 32, m + 48). grid = pairs.
template <int D, typename QT>
__global__ void __launch_bounds__(256) hamming_table_kernel(const TableParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int pair = blockIdx.x;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const QT* Qg = reinterpret_cast<const QT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  float* T = p.T + (size_t)pair * 256 * TABLE_COLS;
  build_hamming_table<D>(Qg, G, p.R, 0, 16, dyn, [&](int x, int m, float v) {
    float* row = T + (size_t)x * TABLE_COLS;
    for (int c = m; c < TABLE_COLS; c += 16) row[c] = v;
  });
}

struct ScoreParams {
  const float* T;
  const uint8_t* ids;
  const __half* norms;
  float* scores;           // [units][Ncap]
  int Ncap, N, blocks_per_cta;
  int pair_div = 1;        // units per cache pair, as in FusedParams
};

// grid = (pairs, chunks); the pair's table image is copied to 64 KB-aligned
// shared memory, then each lane scores one key of a 32-key block, with the
// warp's next blocks already requested. NORM = false: hard-hash
// scores (ids holds the 128-bit codes, the image the 16 byte-tables, no norm).
template <int LP, bool NORM = true>
__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_score_kernel(const ScoreParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  constexpr int NCH = table_chunks(LP);
  const int pair = blockIdx.x;
  const uint32_t base = smem_u32(dyn);
  const uint32_t tbl = (base + 65535u) & ~65535u;
  uint32_t dyn_size;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  if (tbl + NCH * TABLE_BYTES > base + dyn_size) {     // uniform over the grid
    if (threadIdx.x == 0) atomicOr(&g_error_word, ERR_LAYOUT);
    return;
  }
  float* t = sptr<float>(dyn, base, tbl);
  const float4* src = reinterpret_cast<const float4*>(p.T + (size_t)pair * NCH * 256 * TABLE_COLS);
  for (int e = threadIdx.x; e < NCH * 256 * TABLE_COLS / 4; e += blockDim.x)
    reinterpret_cast<float4*>(t)[e] = __ldg(src + e);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const size_t pair_keys = (size_t)(pair / p.pair_div) * p.Ncap;
  const int nblk = (p.N + 31) / 32;
  const int blk0 = min(nblk, (int)blockIdx.y * p.blocks_per_cta);
  const int blk1 = min(nblk, blk0 + p.blocks_per_cta);
  // this warp's blocks blk0 + warp + i * nw (i < nb), the next PF of them in
  // flight while one is scored
  constexpr int PF = score_pf<LP>();
  const int nb = max(0, (blk1 - blk0 - warp + nw - 1) / nw);
  const uint8_t* ids_pair = p.ids + pair_keys * LP;
  const __half* norms_pair = NORM ? p.norms + pair_keys : nullptr;
  float* out = p.scores + (size_t)pair * p.Ncap;
  KeyIds<LP> buf[PF];
#pragma unroll
  for (int u = 0; u < PF; ++u) {
    if (u < nb) {
      const int key = (blk0 + warp + u * nw) * 32 + lane;
      load_key_ids<LP, NORM>(buf[u], ids_pair + (size_t)key * LP, norms_pair + key);
    }
  }
  for (int it = 0; it < nb; it += PF) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int i = it + u;
      if (i < nb) {
        const KeyIds<LP> cur = buf[u];
        if (i + PF < nb) {
          const int key = (blk0 + warp + (i + PF) * nw) * 32 + lane;
          load_key_ids<LP, NORM>(buf[u], ids_pair + (size_t)key * LP, norms_pair + key);
        }
        const float sc = score_key<LP, NORM>(cur, tbl + 4u * lane, tbl + TABLE_BYTES + 4u * lane);
        const int key = (blk0 + warp + i * nw) * 32 + lane;
        if (key < p.N) out[key] = sc;
      }
    }
  }
}

struct TopkParams {
  const float* scores;
  int* idx;
  int Ncap, N, k, C, keys_per_cta;
};

// One cluster of C CTAs per pair; CTA r holds keys [r * keys_per_cta, ...).
__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_topk_kernel(const TopkParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int C = p.C;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x / C;
  SelShared* sh = reinterpret_cast<SelShared*>(dyn);
  uint32_t* h0 = reinterpret_cast<uint32_t*>(dyn + ((sizeof(SelShared) + 15) & ~15));
  uint32_t* h1 = h0 + hist_words(0);
  uint32_t* h2 = h1 + hist_words(1);
  uint32_t* keys = h2 + hist_words(2);
  for (int i = threadIdx.x; i < hist_words(0); i += blockDim.x) h0[i] = 0u;
  for (int i = threadIdx.x; i < hist_words(1); i += blockDim.x) h1[i] = 0u;
  for (int i = threadIdx.x; i < hist_words(2); i += blockDim.x) h2[i] = 0u;
  __syncthreads();
  const int k0 = rank * p.keys_per_cta;
  const int n_local = max(0, min(p.N - k0, p.keys_per_cta));
  const float* src = p.scores + (size_t)pair * p.Ncap + k0;
  for (int i = threadIdx.x; i < n_local; i += blockDim.x) {
    const uint32_t key = key_of(fmaxf(src[i], 0.0f));
    keys[i] = key;
    atomicAdd(&h0[key >> 20], 1u);
  }
  __syncthreads();
  cluster_sync();
  uint32_t* hist[3] = {h0, h1, h2};
  auto key_at = [&](int i) -> uint32_t { return keys[i]; };
  const SelThreshold th = cluster_threshold<FUSED_THREADS>(key_at, n_local, hist, (uint32_t)p.k, C, sh);
  int* out = p.idx + (size_t)pair * p.k;
  ordered_compact(key_at, n_local, th, C, rank, sh, [&](uint32_t pos, int i) {
    if (pos < (uint32_t)p.k) out[pos] = k0 + i;
  });
  cluster_sync();
}

struct AttendParams {
  const void* Q;
  const void* K;
  const void* V;
  const int* idx;          // [pairs][n] key list (sparse) or nullptr (dense: keys 0..n-1)
  float* part;             // [pairs][splits][G][D + 2]: (m, l, o[D]) per head
  unsigned int* counters;  // [pairs], zero on entry; left zero on exit
  float* O;                // [B][Hq][D]
  unsigned long long* phase_ts;  // optional: [pairs * splits][PHASES] clock stamps (profiling)
  int Hq, Hkv, Ncap, n, keys_per_split, splits;
  float scale;
  int pair_div = 1;        // units per cache pair, as in FusedParams
  const int* counts = nullptr;   // optional [units]: keys of each unit's list (<= n)
  // paged K/V (with idx): K and V are pools [num_pages][page_size][D] and key
  // n of cache pair c is row n % page_size of page page_table[c][n / page_size]
  const int* page_table = nullptr;   // [cache pairs][max_pages]
  int max_pages = 0, page_size = 0, num_pages = 0;
};

__device__ __forceinline__ void attend_stamp(unsigned long long* ts, int phase) {
  if (ts != nullptr && threadIdx.x == 0) {
    const size_t cta = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    ts[cta * PHASES + phase] = (unsigned long long)clock64();
    if (phase == 0 || phase == 7) {
      unsigned long long t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      ts[cta * PHASES + 22 + (phase == 7)] = t;
    }
  }
}

// Shared bytes of socket_attend_kernel: query stage, mbarriers and phases,
// warp slots, partials, the CTA's index list, a flag word.
template <int D>
__host__ __device__ inline size_t attend_smem_bytes(int G, int keys_per_split) {
  return q_stage_bytes<D>() + 8 * 32 + 4 * 32 + (size_t)ATTEND_SLOTS * kv_slot_bytes<D>() +
         ((partial_floats(G, D) * 4 + 15) & ~(size_t)15) + (((size_t)keys_per_split * 4 + 15) & ~(size_t)15) + 16;
}

// Exact attention over a key list, split over keys: grid = (pairs, splits).
// Each CTA attends over its range and forms one partial (m, l, o) per head.
// CLUSTER = true: the splits of a pair form one thread-block cluster; after a
// cluster barrier CTA r merges heads r, r + splits, ... reading every CTA's
// partial from its shared memory (split order). CLUSTER = false: the partial
// goes to the workspace and the last CTA of a pair to finish (counted with an
// atomic) merges the pair's partials in split order. Either way the result
// does not depend on the order the CTAs ran. Launched after the selection
// kernel with programmatic dependent launch: everything before
// griddepcontrol.wait overlaps that kernel's tail.
template <int D, typename KVT, bool CLUSTER>
__global__ void __launch_bounds__(ATTEND_THREADS) socket_attend_kernel(const AttendParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  attend_stamp(p.phase_ts, 0);
  const int pair = blockIdx.x, split = blockIdx.y;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  int i0 = split * p.keys_per_split;
  const size_t pair_keys = (size_t)(pair / p.pair_div) * p.Ncap;
  const KVT* Qg = reinterpret_cast<const KVT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  const uint32_t base = smem_u32(dyn);
  AttendSmem as;
  {
    uint32_t a = base;
    as.qs = a;       a += q_stage_bytes<D>();
    as.mbar0 = a;    a += 8u * 32u;
    as.phases = a;   a += 4u * 32u;
    as.slot0 = a;
    as.slot_stride = kv_slot_bytes<D>();
    a += ATTEND_SLOTS * kv_slot_bytes<D>();
    as.ncw = sizeof(KVT) == 2 ? ATTEND_MMA_WARPS : ATTEND_WARPS;
    as.nbuf = sizeof(KVT) == 2 ? ATTEND_BUFS : 1;
    as.result = a;
    a += (uint32_t)((partial_floats(G, D) * 4 + 15) & ~(size_t)15);
  }
  const size_t smem_total = attend_smem_bytes<D>(G, p.idx ? p.keys_per_split : 0);
  uint32_t* last_flag = reinterpret_cast<uint32_t*>(dyn + (smem_total - 16));
  int* list_s = reinterpret_cast<int*>(dyn + (as.result - base) + ((partial_floats(G, D) * 4 + 15) & ~(size_t)15));
  attend_setup<D, KVT>(dyn, base, as, Qg, G);
  attend_stamp(p.phase_ts, 1);
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the key list is complete from here on
  attend_stamp(p.phase_ts, 2);
  // this unit's list length: n, or its count (clamped to [0, n]) when the
  // lists have per-unit lengths
  const int n_unit = p.counts ? min(max(__ldcg(p.counts + pair), 0), p.n) : p.n;
  int cnt = max(0, min(n_unit - i0, p.keys_per_split));
  if (p.counts) {
    // per-unit lengths (planned for the longest): the unit's own keys split
    // evenly over its splits, so that every split has work
    i0 = (int)((long long)split * n_unit / p.splits);
    cnt = (int)((long long)(split + 1) * n_unit / p.splits) - i0;
  }
  const bool paged = p.page_table != nullptr;
  const size_t key0 = paged ? 0 : pair_keys;            // a paged pool is addressed by physical row
  const KVT* Kp = reinterpret_cast<const KVT*>(p.K) + key0 * D;
  const KVT* Vp = reinterpret_cast<const KVT*>(p.V) + key0 * D;
  float *cM, *cL, *cO;
  if (p.idx) {
    const int* list = p.idx + (size_t)pair * p.n + i0;      // one coalesced load of this CTA's indices
    int nrows = p.Ncap;
    if (paged) {
      // logical key -> physical pool row; an entry outside the pool is
      // flagged and read as page 0 (every access stays inside the pool)
      const int* pt = p.page_table + (size_t)(pair / p.pair_div) * p.max_pages;
      const int last = p.max_pages * p.page_size - 1;
      for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
        const int n = min(max(__ldcg(list + i), 0), last);
        int pg = __ldg(pt + n / p.page_size);
        if (pg < 0 || pg >= p.num_pages) {
          atomicOr(&g_error_word, ERR_RANGE);
          pg = 0;
        }
        list_s[i] = pg * p.page_size + n % p.page_size;
      }
      nrows = p.num_pages * p.page_size;
    } else {
      for (int i = threadIdx.x; i < cnt; i += blockDim.x) list_s[i] = __ldcg(list + i);
    }
    __syncthreads();
    attend_stamp(p.phase_ts, 3);
    attend_and_merge<D, KVT>(dyn, base, as, Qg, Kp, Vp, G, p.scale, [=](int i) { return list_s[i]; }, cnt, nrows,
                             cM, cL, cO);
  } else {
    attend_and_merge<D, KVT>(dyn, base, as, Qg, Kp, Vp, G, p.scale, [=](int i) { return i0 + i; }, cnt, p.Ncap, cM,
                             cL, cO);
  }
  attend_stamp(p.phase_ts, 4);
  if constexpr (CLUSTER) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster_sync();            // every split's partial is final
    attend_stamp(p.phase_ts, 5);
    for (int h = split; h < G; h += p.splits) {
      for (int dv = threadIdx.x; dv < D; dv += blockDim.x) {
        float mm = -INFINITY;
        for (int sp = 0; sp < p.splits; ++sp) mm = fmaxf(mm, *cluster.map_shared_rank(cM + h, sp));
        float lsum = 0.f, o = 0.f;
        for (int sp = 0; sp < p.splits; ++sp) {
          const float m = *cluster.map_shared_rank(cM + h, sp);
          if (m != -INFINITY) {
            const float w = exp2f(m - mm);
            lsum += w * *cluster.map_shared_rank(cL + h, sp);
            o += w * *cluster.map_shared_rank(cO + h * D + dv, sp);
          }
        }
        p.O[((size_t)b * p.Hq + kvh * G + h) * D + dv] = o / lsum;
      }
    }
    attend_stamp(p.phase_ts, 6);
    cluster_sync();            // the other CTAs read this CTA's partial until here
    attend_stamp(p.phase_ts, 7);
    return;
  }
  float* mine = p.part + ((size_t)pair * p.splits + split) * G * (D + 2);
  for (int e = threadIdx.x; e < G * (D + 2); e += blockDim.x) {
    const int h = e / (D + 2), j = e % (D + 2);
    mine[e] = j == 0 ? cM[h] : j == 1 ? cL[h] : cO[h * D + j - 2];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) *last_flag = (atomicAdd(&p.counters[pair], 1u) == (unsigned)p.splits - 1u) ? 1u : 0u;
  __syncthreads();
  attend_stamp(p.phase_ts, 5);
  if (*last_flag == 0u) {
    attend_stamp(p.phase_ts, 7);
    return;
  }
  // ---- last CTA of the pair: merge the splits in order, one head at a time:
  // the head's partials are copied into shared memory (the warp slots are
  // free; splits <= ATTEND_MAX_SPLITS keeps them in bounds) with independent
  // loads, then combined there.
  __threadfence();
  const float* part = p.part + (size_t)pair * p.splits * G * (D + 2);
  const size_t stride = (size_t)G * (D + 2);
  float* ps = reinterpret_cast<float*>(dyn + (as.slot0 - base));
  for (int h = 0; h < G; ++h) {
    for (int e = threadIdx.x; e < p.splits * (D + 2); e += blockDim.x)
      ps[e] = __ldcg(part + (size_t)(e / (D + 2)) * stride + (size_t)h * (D + 2) + e % (D + 2));
    __syncthreads();
    for (int dv = threadIdx.x; dv < D; dv += blockDim.x) {
      float mm = -INFINITY;
      for (int sp = 0; sp < p.splits; ++sp) mm = fmaxf(mm, ps[sp * (D + 2)]);
      float lsum = 0.f, o = 0.f;
      for (int sp = 0; sp < p.splits; ++sp) {
        const float m = ps[sp * (D + 2)];
        if (m != -INFINITY) {
          const float w = exp2f(m - mm);
          lsum += w * ps[sp * (D + 2) + 1];
          o += w * ps[sp * (D + 2) + 2 + dv];
        }
      }
      p.O[((size_t)b * p.Hq + kvh * G + h) * D + dv] = o / lsum;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) p.counters[pair] = 0u;
  attend_stamp(p.phase_ts, 6);
  attend_stamp(p.phase_ts, 7);
}

// ---------------------------------------------------------------- paged gather
// Copies the selected keys' K and V rows from a paged pool into contiguous
// rows Ks, Vs [units][n][ROW bytes], with plain 16-byte loads: the pool may be
// pinned host memory (read over the host link) as well as device memory. Half
// a warp copies one K row and the other half the matching V row; each warp
// keeps GATHER_UNROLL row pairs in flight. grid = (units, chunks of
// GATHER_KEYS keys).
struct GatherParams {
  const void* K;
  const void* V;
  const int* page_table;   // [cache pairs][max_pages]
  const int* idx;          // [units][n]
  void* Ks;
  void* Vs;
  int n, max_pages, page_size, num_pages, pair_div;
};

constexpr int GATHER_THREADS = 256;
constexpr int GATHER_KEYS = 64;
constexpr int GATHER_UNROLL = 4;

template <int ROW>
__global__ void __launch_bounds__(GATHER_THREADS) paged_gather_kernel(const GatherParams p) {
  constexpr int CH = ROW / 16;                       // 16-byte chunks per row: 8, 16 or 32
  constexpr int CPL = (CH + 15) / 16;                // chunks per lane of the half warp
  const int unit = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, c = lane & 15;
  const int* pt = p.page_table + (size_t)(unit / p.pair_div) * p.max_pages;
  const int last = p.max_pages * p.page_size - 1;
  const unsigned char* src_base = reinterpret_cast<const unsigned char*>(half ? p.V : p.K);
  unsigned char* dst_base = reinterpret_cast<unsigned char*>(half ? p.Vs : p.Ks) + (size_t)unit * p.n * ROW;
  const int j_end = min(p.n, (int)(blockIdx.y + 1) * GATHER_KEYS);
  for (int j0 = blockIdx.y * GATHER_KEYS + warp; j0 < j_end; j0 += (GATHER_THREADS / 32) * GATHER_UNROLL) {
    uint4 v[GATHER_UNROLL][CPL];
    size_t row[GATHER_UNROLL];
#pragma unroll
    for (int u = 0; u < GATHER_UNROLL; ++u) {
      const int j = j0 + u * (GATHER_THREADS / 32);
      row[u] = 0;
      if (j < j_end) {
        const int n = min(max(__ldg(p.idx + (size_t)unit * p.n + j), 0), last);
        int pg = __ldg(pt + n / p.page_size);
        if (pg < 0 || pg >= p.num_pages) {
          atomicOr(&g_error_word, ERR_RANGE);
          pg = 0;
        }
        row[u] = (size_t)pg * p.page_size + n % p.page_size;
      }
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const int ch = c + 16 * q;
        v[u][q] = (j < j_end && ch < CH) ? *reinterpret_cast<const uint4*>(src_base + row[u] * ROW + 16 * ch)
                                         : make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < GATHER_UNROLL; ++u) {
      const int j = j0 + u * (GATHER_THREADS / 32);
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        const int ch = c + 16 * q;
        if (j < j_end && ch < CH) *reinterpret_cast<uint4*>(dst_base + (size_t)j * ROW + 16 * ch) = v[u][q];
      }
    }
  }
}

}  // namespace hst
