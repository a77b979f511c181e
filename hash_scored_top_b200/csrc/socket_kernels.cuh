// SOCKET decode kernels: the fused one-launch decode step and the unfused
// chain (bucket table -> scores -> top-k -> sparse attention -> merge),
// plus dense decode attention. See table.cuh, score.cuh, select.cuh and
// attend.cuh for the steps.
#pragma once

#include "attend.cuh"
#include "common.cuh"
#include "hash_kernels.cuh"
#include "score.cuh"
#include "select.cuh"
#include "table.cuh"

namespace hst {

// ---------------------------------------------------------------- shared constants
constexpr int SMEM_BASE_EXPECTED = 1024;         // dynamic shared window start on sm_100
constexpr int SMEM_DYN_MAX = 232448;             // 227 KB opt-in per block
constexpr int HIST1_BITS = 11, HIST2_BITS = 11, HIST3_BITS = 9;
constexpr int FUSED_THREADS = 256;
constexpr int FUSED_WARPS = FUSED_THREADS / 32;
constexpr int SCORE_PF = 4;                      // 32-key blocks in flight per warp

__device__ __forceinline__ uint32_t key_of(float s) { return __float_as_uint(s); }

// Digit levels for f32 score keys (bit 31 is always 0 for s >= 0).
__device__ __forceinline__ void f32_levels(DigitLevel (&lv)[3]) {
  lv[0] = {20, HIST1_BITS};
  lv[1] = {9, HIST2_BITS};
  lv[2] = {0, HIST3_BITS};
}

struct FusedParams {
  const void* Q;
  const void* K;
  const void* V;
  const __nv_bfloat16* R;
  const uint8_t* ids;
  const __half* norms;
  float* O;
  int* idx_out;
  int Hq, Hkv, Ncap, N, L, P, k, C, blocks_per_cta, chunk;
  float tau, scale;
};

// Shared-memory plan of the fused kernel (all addresses are shared-window
// addresses). The 64 KB table sits at a 64 KB-aligned address; sort keys
// fill segment A (after the fixed items) and then segment B (after the table).
struct FusedSmem {
  uint32_t base, tbl, segA, segA_end, segB, segB_end;
  uint32_t sel, hist1, hist2, hist3;
  uint32_t keysA, nA;        // first nA keys in segment A
  uint32_t keysB;            // the rest in segment B
  __device__ void plan(uint32_t dyn_base, uint32_t dyn_size) {
    base = dyn_base;
    tbl = (dyn_base + 65535u) & ~65535u;
    segA = dyn_base;
    segA_end = tbl;
    segB = tbl + TABLE_BYTES;
    segB_end = dyn_base + dyn_size;
    uint32_t a = segA;
    sel = a;   a += (sizeof(SelShared) + 15u) & ~15u;
    hist1 = a; a += 4u << HIST1_BITS;
    hist2 = a; a += 4u << HIST2_BITS;
    hist3 = a; a += 4u << HIST3_BITS;
    keysA = a;
    nA = (segA_end > a) ? (segA_end - a) / 4u : 0u;
    keysB = segB;
  }
  __device__ uint32_t key_capacity() const { return nA + (segB_end - segB) / 4u; }
  __device__ __forceinline__ uint32_t key_addr(uint32_t i) const {
    return i < nA ? keysA + 4u * i : keysB + 4u * (i - nA);
  }
};

template <typename T>
__device__ __forceinline__ T* sptr(unsigned char* dyn, uint32_t base, uint32_t addr) {
  return reinterpret_cast<T*>(dyn + (addr - base));
}

// Zero rows >= 2^P and columns >= L of a table at shared address tbl.
__device__ __forceinline__ void zero_table_padding(unsigned char* dyn, uint32_t base, uint32_t tbl, int L, int P) {
  float* t = sptr<float>(dyn, base, tbl);
  const int nb = 1 << P;
  for (int e = threadIdx.x; e < 256 * TABLE_COLS; e += blockDim.x) {
    const int b = e / TABLE_COLS, l = e % TABLE_COLS;
    if (b >= nb || l >= L) t[e] = 0.f;
  }
}

// Scores this CTA's blocks [blk0, blk1) into sort keys (fs.key_addr) and the
// level-1 histogram. Warp w takes blocks blk0 + w, blk0 + w + NW, ...
template <int NCHUNK, bool NORM>
__device__ __forceinline__ void score_slice(const uint8_t* __restrict__ ids_pair,
                                            const __half* __restrict__ norms_pair, int L, int N, int blk0,
                                            int blk1, const FusedSmem& fs, uint32_t* hist1) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t col_addr[NCHUNK];
#pragma unroll
  for (int c = 0; c < NCHUNK; ++c) col_addr[c] = fs.tbl + 4u * (32 * c + lane);
  const int nb = (blk1 - blk0 - warp + nw - 1) / nw;
  IdBlock<NCHUNK> buf[SCORE_PF];
#pragma unroll
  for (int u = 0; u < SCORE_PF; ++u) {
    if (u < nb) {
      const int blk = blk0 + warp + u * nw;
      load_id_block<NCHUNK, NORM>(buf[u], ids_pair + (size_t)blk * 32 * L, norms_pair + (size_t)blk * 32, L, lane);
    }
  }
  for (int it = 0; it < nb; it += SCORE_PF) {
#pragma unroll
    for (int u = 0; u < SCORE_PF; ++u) {
      const int i = it + u;
      if (i < nb) {
        const IdBlock<NCHUNK> cur = buf[u];
        if (i + SCORE_PF < nb) {
          const int blk = blk0 + warp + (i + SCORE_PF) * nw;
          load_id_block<NCHUNK, NORM>(buf[u], ids_pair + (size_t)blk * 32 * L, norms_pair + (size_t)blk * 32, L,
                                      lane);
        }
        const float s = score_id_block<NCHUNK, NORM>(cur, col_addr, lane);
        const int blk = blk0 + warp + i * nw;
        const int gkey = blk * 32 + lane;
        if (gkey < N) {
          const uint32_t key = key_of(s);
          const uint32_t li = (uint32_t)(gkey - blk0 * 32);
          asm volatile("st.shared.u32 [%0], %1;" :: "r"(fs.key_addr(li)), "r"(key) : "memory");
          atomicAdd(&hist1[key >> 20], 1u);
        }
      }
    }
  }
}

// ---------------------------------------------------------------- fused decode
// One cluster of C CTAs per (batch, KV-head) pair; grid = pairs * C.
// HATA = false: SOCKET soft-LSH scores (ids/norms cache, tables l = rank mod C).
// HATA = true: hard-hash scores from 128-bit codes (16 byte tables, no norm),
// with R holding the 128 code hyperplanes and ids the codes.
template <int D, int NCHUNK, typename KVT, bool HATA>
__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_decode_fused_kernel(const FusedParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int C = p.C;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x / C;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  uint32_t dyn_size;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  FusedSmem fs;
  fs.plan(smem_u32(dyn), dyn_size);
  SelShared* sh = sptr<SelShared>(dyn, fs.base, fs.sel);
  uint32_t* hist[3] = {sptr<uint32_t>(dyn, fs.base, fs.hist1), sptr<uint32_t>(dyn, fs.base, fs.hist2),
                       sptr<uint32_t>(dyn, fs.base, fs.hist3)};

  const int nblk_pair = (p.N + 31) / 32;
  const int blk0 = min(nblk_pair, rank * p.blocks_per_cta);
  const int blk1 = min(nblk_pair, blk0 + p.blocks_per_cta);
  const int n_local = max(0, min(p.N, blk1 * 32) - blk0 * 32);
  // The host sizes slices from the same plan; a mismatch (a host bug) is flagged
  // and the kernel then selects and gathers nothing. The test is the same in every
  // CTA of the cluster.
  const bool fits = fs.tbl + TABLE_BYTES <= fs.base + dyn_size &&
                    (uint32_t)p.blocks_per_cta * 32u <= fs.key_capacity();
  if (!fits) {              // uniform across the cluster: every CTA leaves here
    if (tid == 0) atomicOr(&g_error_word, ERR_LAYOUT);
    return;
  }

  // ---- setup: zero histograms and table padding; let peers know we started
  for (int i = tid; i < (1 << HIST1_BITS); i += blockDim.x) hist[0][i] = 0u;
  for (int i = tid; i < (1 << HIST2_BITS); i += blockDim.x) hist[1][i] = 0u;
  for (int i = tid; i < (1 << HIST3_BITS); i += blockDim.x) hist[2][i] = 0u;
  zero_table_padding(dyn, fs.base, fs.tbl, p.L, p.P);
  cluster_sync();

  // ---- SOCKET step 2: this CTA's share of the bucket tables, written to every CTA
  const KVT* Qg = reinterpret_cast<const KVT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  {
    const uint32_t tbl = fs.tbl;
    auto store = [&](int bb, int l, float v) {
      const uint32_t a = tbl + (uint32_t)bb * 256u + 4u * (uint32_t)l;
      for (int r = 0; r < C; ++r) st_cluster_f32(mapa(a, r), v);
    };
    if constexpr (HATA) {
      build_hamming_table(Qg, G, D, p.R, rank, C, sptr<uint32_t>(dyn, fs.base, fs.segB), store);
    } else {
      build_bucket_table(Qg, G, D, p.R, p.L, p.P, p.tau, rank, C, sptr<double>(dyn, fs.base, fs.segB), store);
    }
  }
  cluster_sync();

  // ---- SOCKET step 3: scores of this CTA's slice (kept on chip) + level-1 histogram
  const size_t pair_keys = (size_t)pair * p.Ncap;
  {
    const uint8_t* ids_pair = p.ids + pair_keys * p.L;
    const __half* norms_pair = p.norms + pair_keys;
    score_slice<NCHUNK, !HATA>(ids_pair, norms_pair, p.L, p.N, blk0, blk1, fs, hist[0]);
  }
  __syncthreads();
  cluster_sync();

  // ---- SOCKET step 4a: exact top-k across the cluster
  DigitLevel lv[3];
  f32_levels(lv);
  auto key_at = [&](int i) -> uint32_t { return lds_u32(fs.key_addr((uint32_t)i)); };
  const int nl = n_local;
  const SelPlan plan = cluster_select(key_at, nl, lv, 3, hist, (uint32_t)p.k, C, rank, sh);
  // emit: the position's owner CTA gathers it; idx_out gets the ascending list
  const int chunk = p.chunk;
  const uint32_t list = fs.tbl;                       // table is dead: index list
  int* idx_out = p.idx_out ? p.idx_out + (size_t)pair * p.k : nullptr;
  ordered_compact(key_at, nl, plan, sh, [&](uint32_t pos, int i) {
    if (pos >= (uint32_t)p.k) return;       // cannot happen for a consistent plan
    const int g = blk0 * 32 + i;
    const uint32_t owner = pos / (uint32_t)chunk;
    const uint32_t slot = pos - owner * (uint32_t)chunk;
    st_cluster_u32(mapa(list + 4u * slot, owner), (uint32_t)g);
    if (idx_out) idx_out[pos] = g;
  });
  cluster_sync();

  // ---- SOCKET step 4b: exact attention over this CTA's share of the selection
  const int my_begin = rank * chunk;
  const int cnt = max(0, min(p.k - my_begin, chunk));
  const int* my_list = sptr<int>(dyn, fs.base, list);
  // partial slots and the CTA result live in segment B (sort keys are dead)
  PartialView pv;
  pv.G = G;
  pv.D = D;
  float* pbase = sptr<float>(dyn, fs.base, fs.segB);
  pv.pm = pbase;
  pv.pl = pv.pm + FUSED_WARPS * G;
  pv.po = pv.pl + FUSED_WARPS * G;
  float* cM = pv.po + (size_t)FUSED_WARPS * G * D;
  float* cL = cM + G;
  float* cO = cL + G;
  const KVT* Kp = reinterpret_cast<const KVT*>(p.K) + pair_keys * D;
  const KVT* Vp = reinterpret_cast<const KVT*>(p.V) + pair_keys * D;
  const float scale_log2 = p.scale * LOG2E;
  const int nrows = p.N;
  if constexpr (sizeof(KVT) == 2) {
    const bool packed = G <= 4;
    uint32_t qb[D / 32][4];
    load_q_frag<D>(qb, reinterpret_cast<const __nv_bfloat16*>(Qg), G, lane);
    MmaAttendState<D> st;
    st.init();
    const int ntiles = (cnt + 15) / 16;
    KVTile<D> cur, nxt;
    int t = warp;
    if (t < ntiles) {
      load_kv_tile<D>(cur, reinterpret_cast<const __nv_bfloat16*>(Kp), reinterpret_cast<const __nv_bfloat16*>(Vp),
                      [&](int i) { return my_list[t * 16 + i]; }, min(16, cnt - t * 16), nrows, lane);
    }
    for (; t < ntiles; t += FUSED_WARPS) {
      const int tn = t + FUSED_WARPS;
      if (tn < ntiles) {
        load_kv_tile<D>(nxt, reinterpret_cast<const __nv_bfloat16*>(Kp), reinterpret_cast<const __nv_bfloat16*>(Vp),
                        [&](int i) { return my_list[tn * 16 + i]; }, min(16, cnt - tn * 16), nrows, lane);
      }
      mma_attend_tile<D>(st, cur, qb, scale_log2, packed, lane);
      cur = nxt;
    }
    store_mma_partial<D>(st, pv, warp, packed, lane);
  } else {
    float q[8][D / 32];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
      for (int i = 0; i < D / 32; ++i)
        q[h][i] = h < G ? reinterpret_cast<const float*>(Qg)[h * D + lane + 32 * i] * scale_log2 : 0.f;
    SimtAttendState<D> st;
    st.init();
    for (int j = warp; j < cnt; j += FUSED_WARPS) {
      const int row = min(max(my_list[j], 0), nrows - 1);
      simt_attend_key<D>(st, reinterpret_cast<const float*>(Kp) + (size_t)row * D,
                         reinterpret_cast<const float*>(Vp) + (size_t)row * D, q, G, lane);
    }
    store_simt_partial<D>(st, pv, warp, lane);
  }
  __syncthreads();
  merge_partials(pv, FUSED_WARPS, cM, cL, cO);
  cluster_sync();

  // ---- cross-CTA merge: CTA `rank` finalises heads h with h % C == rank
  const uint32_t aM = smem_u32(cM), aL = smem_u32(cL), aO = smem_u32(cO);
  for (int h = rank; h < G; h += C) {
    float mm = -INFINITY;
    for (int r = 0; r < C; ++r) mm = fmaxf(mm, ld_cluster_f32(mapa(aM + 4u * h, r)));
    float lsum = 0.f;
    for (int r = 0; r < C; ++r) {
      const float mr = ld_cluster_f32(mapa(aM + 4u * h, r));
      if (mr != -INFINITY) lsum += exp2f(mr - mm) * ld_cluster_f32(mapa(aL + 4u * h, r));
    }
    for (int e = tid; e < D; e += blockDim.x) {
      float o = 0.f;
      for (int r = 0; r < C; ++r) {
        const float mr = ld_cluster_f32(mapa(aM + 4u * h, r));
        if (mr != -INFINITY) o += exp2f(mr - mm) * ld_cluster_f32(mapa(aO + 4u * (h * D + e), r));
      }
      p.O[((size_t)b * p.Hq + kvh * G + h) * D + e] = o / lsum;
    }
  }
  cluster_sync();   // peers may still read this CTA's shared memory until here
}

// ---------------------------------------------------------------- unfused chain
struct TableParams {
  const void* Q;
  const __nv_bfloat16* R;
  float* T;            // [pairs][256][64]
  int Hq, Hkv, d, L, P;
  float tau;
};

template <typename QT>
__global__ void __launch_bounds__(256) bucket_table_kernel(const TableParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int pair = blockIdx.x;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const QT* Qg = reinterpret_cast<const QT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * p.d;
  float* T = p.T + (size_t)pair * 256 * TABLE_COLS;
  // padding (rows >= 2^P, columns >= L) is zero; CTA y = 0 writes it
  if (blockIdx.y == 0) {
    const int nb = 1 << p.P;
    for (int e = threadIdx.x; e < 256 * TABLE_COLS; e += blockDim.x) {
      const int bb = e / TABLE_COLS, l = e % TABLE_COLS;
      if (bb >= nb || l >= p.L) T[e] = 0.f;
    }
  }
  build_bucket_table(Qg, G, p.d, p.R, p.L, p.P, p.tau, (int)blockIdx.y, (int)gridDim.y,
                     reinterpret_cast<double*>(dyn),
                     [&](int bb, int l, float v) { T[bb * TABLE_COLS + l] = v; });
}

struct ScoreParams {
  const float* T;
  const uint8_t* ids;
  const __half* norms;
  float* scores;
  int Ncap, N, L, blocks_per_cta;
};

// grid = (pairs, chunks); the 64 KB table of the pair is copied to a 64 KB-aligned
// shared address, then each warp scores 32-key blocks.
template <int NCHUNK>
__global__ void __launch_bounds__(256, 1) socket_score_kernel(const ScoreParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int pair = blockIdx.x;
  const uint32_t base = smem_u32(dyn);
  const uint32_t tbl = (base + 65535u) & ~65535u;
  uint32_t dyn_size;
  asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_size));
  if (tbl + TABLE_BYTES > base + dyn_size) {     // uniform over the grid
    if (threadIdx.x == 0) atomicOr(&g_error_word, ERR_LAYOUT);
    return;
  }
  float* t = sptr<float>(dyn, base, tbl);
  const float4* src = reinterpret_cast<const float4*>(p.T + (size_t)pair * 256 * TABLE_COLS);
  for (int e = threadIdx.x; e < 256 * TABLE_COLS / 4; e += blockDim.x)
    reinterpret_cast<float4*>(t)[e] = __ldg(src + e);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t col_addr[NCHUNK];
#pragma unroll
  for (int c = 0; c < NCHUNK; ++c) col_addr[c] = tbl + 4u * (32 * c + lane);
  const size_t pair_keys = (size_t)pair * p.Ncap;
  const int nblk = (p.N + 31) / 32;
  const int blk0 = blockIdx.y * p.blocks_per_cta;
  const int blk1 = min(nblk, blk0 + p.blocks_per_cta);
  for (int blk = blk0 + warp; blk < blk1; blk += nw) {
    IdBlock<NCHUNK> ib;
    load_id_block(ib, p.ids + (pair_keys + (size_t)blk * 32) * p.L, p.norms + pair_keys + (size_t)blk * 32, p.L,
                  lane);
    const float s = score_id_block(ib, col_addr, lane);
    const int key = blk * 32 + lane;
    if (key < p.N) p.scores[pair_keys + key] = s;
  }
}

struct TopkParams {
  const float* scores;
  int* idx;
  int Ncap, N, k, C, keys_per_cta;
};

// One cluster of C CTAs per pair; CTA r holds keys [r*keys_per_cta, ...).
__global__ void __launch_bounds__(FUSED_THREADS, 1) socket_topk_kernel(const TopkParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int C = p.C;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x / C;
  SelShared* sh = reinterpret_cast<SelShared*>(dyn);
  uint32_t* h1 = reinterpret_cast<uint32_t*>(dyn + ((sizeof(SelShared) + 15) & ~15));
  uint32_t* h2 = h1 + (1 << HIST1_BITS);
  uint32_t* h3 = h2 + (1 << HIST2_BITS);
  uint32_t* keys = h3 + (1 << HIST3_BITS);
  for (int i = threadIdx.x; i < (1 << HIST1_BITS); i += blockDim.x) h1[i] = 0u;
  for (int i = threadIdx.x; i < (1 << HIST2_BITS); i += blockDim.x) h2[i] = 0u;
  for (int i = threadIdx.x; i < (1 << HIST3_BITS); i += blockDim.x) h3[i] = 0u;
  __syncthreads();
  const int k0 = rank * p.keys_per_cta;
  const int n_local = max(0, min(p.N - k0, p.keys_per_cta));
  const float* src = p.scores + (size_t)pair * p.Ncap + k0;
  for (int i = threadIdx.x; i < n_local; i += blockDim.x) {
    const uint32_t key = key_of(fmaxf(src[i], 0.0f));
    keys[i] = key;
    atomicAdd(&h1[key >> 20], 1u);
  }
  __syncthreads();
  cluster_sync();
  DigitLevel lv[3];
  f32_levels(lv);
  uint32_t* hist[3] = {h1, h2, h3};
  auto key_at = [&](int i) -> uint32_t { return keys[i]; };
  const SelPlan plan = cluster_select(key_at, n_local, lv, 3, hist, (uint32_t)p.k, C, rank, sh);
  int* out = p.idx + (size_t)pair * p.k;
  ordered_compact(key_at, n_local, plan, sh, [&](uint32_t pos, int i) {
    if (pos < (uint32_t)p.k) out[pos] = k0 + i;
  });
  cluster_sync();
}

struct AttendParams {
  const void* Q;
  const void* K;
  const void* V;
  const int* idx;        // [pairs][k] (sparse) or nullptr (dense: keys 0..n-1)
  float* part;           // [pairs][splits][G][D + 2]: (m, l, o[D]) per head
  int Hq, Hkv, Ncap, n, keys_per_split, splits;
  float scale;
};

// grid = (pairs, splits). Each CTA attends over its range of the key list and
// writes one partial (m, l, unnormalised o) per head.
template <int D, typename KVT>
__global__ void __launch_bounds__(FUSED_THREADS) attend_split_kernel(const AttendParams p) {
  extern __shared__ __align__(1024) unsigned char dyn[];
  const int pair = blockIdx.x, split = blockIdx.y;
  const int G = p.Hq / p.Hkv;
  const int b = pair / p.Hkv, kvh = pair % p.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int i0 = split * p.keys_per_split;
  const int cnt = max(0, min(p.n - i0, p.keys_per_split));
  const int* list = p.idx ? p.idx + (size_t)pair * p.n + i0 : nullptr;
  const size_t pair_keys = (size_t)pair * p.Ncap;
  const KVT* Qg = reinterpret_cast<const KVT*>(p.Q) + (size_t)(b * p.Hq + kvh * G) * D;
  const KVT* Kp = reinterpret_cast<const KVT*>(p.K) + pair_keys * D;
  const KVT* Vp = reinterpret_cast<const KVT*>(p.V) + pair_keys * D;
  PartialView pv;
  pv.G = G;
  pv.D = D;
  pv.pm = reinterpret_cast<float*>(dyn);
  pv.pl = pv.pm + FUSED_WARPS * G;
  pv.po = pv.pl + FUSED_WARPS * G;
  float* cM = pv.po + (size_t)FUSED_WARPS * G * D;
  float* cL = cM + G;
  float* cO = cL + G;
  const float scale_log2 = p.scale * LOG2E;
  const int nrows = p.Ncap;
  auto row_of = [&](int j) { return list ? list[j] : i0 + j; };
  if constexpr (sizeof(KVT) == 2) {
    const bool packed = G <= 4;
    uint32_t qb[D / 32][4];
    load_q_frag<D>(qb, reinterpret_cast<const __nv_bfloat16*>(Qg), G, lane);
    MmaAttendState<D> st;
    st.init();
    const int ntiles = (cnt + 15) / 16;
    KVTile<D> cur, nxt;
    int t = warp;
    if (t < ntiles) {
      load_kv_tile<D>(cur, reinterpret_cast<const __nv_bfloat16*>(Kp), reinterpret_cast<const __nv_bfloat16*>(Vp),
                      [&](int i) { return row_of(t * 16 + i); }, min(16, cnt - t * 16), nrows, lane);
    }
    for (; t < ntiles; t += FUSED_WARPS) {
      const int tn = t + FUSED_WARPS;
      if (tn < ntiles) {
        load_kv_tile<D>(nxt, reinterpret_cast<const __nv_bfloat16*>(Kp), reinterpret_cast<const __nv_bfloat16*>(Vp),
                        [&](int i) { return row_of(tn * 16 + i); }, min(16, cnt - tn * 16), nrows, lane);
      }
      mma_attend_tile<D>(st, cur, qb, scale_log2, packed, lane);
      cur = nxt;
    }
    store_mma_partial<D>(st, pv, warp, packed, lane);
  } else {
    float q[8][D / 32];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
      for (int i = 0; i < D / 32; ++i)
        q[h][i] = h < G ? reinterpret_cast<const float*>(Qg)[h * D + lane + 32 * i] * scale_log2 : 0.f;
    SimtAttendState<D> st;
    st.init();
    for (int j = warp; j < cnt; j += FUSED_WARPS) {
      const int row = min(max(row_of(j), 0), nrows - 1);
      simt_attend_key<D>(st, reinterpret_cast<const float*>(Kp) + (size_t)row * D,
                         reinterpret_cast<const float*>(Vp) + (size_t)row * D, q, G, lane);
    }
    store_simt_partial<D>(st, pv, warp, lane);
  }
  __syncthreads();
  merge_partials(pv, FUSED_WARPS, cM, cL, cO);
  float* out = p.part + ((size_t)pair * p.splits + split) * G * (D + 2);
  for (int e = threadIdx.x; e < G * (D + 2); e += blockDim.x) {
    const int h = e / (D + 2), j = e % (D + 2);
    out[e] = j == 0 ? cM[h] : j == 1 ? cL[h] : cO[h * D + j - 2];
  }
}

// grid = pairs * G; block = D threads. Merges the splits of one head in order.
__global__ void merge_splits_kernel(const float* __restrict__ part, float* __restrict__ O, int Hq, int Hkv, int D,
                                    int splits) {
  const int G = Hq / Hkv;
  const int pair = blockIdx.x / G, h = blockIdx.x % G;
  const int b = pair / Hkv, kvh = pair % Hkv;
  const float* base = part + (size_t)pair * splits * G * (D + 2) + (size_t)h * (D + 2);
  const size_t stride = (size_t)G * (D + 2);
  float mm = -INFINITY;
  for (int s = 0; s < splits; ++s) mm = fmaxf(mm, base[s * stride]);
  float lsum = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float m = base[s * stride];
    if (m != -INFINITY) lsum += exp2f(m - mm) * base[s * stride + 1];
  }
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float o = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float m = base[s * stride];
      if (m != -INFINITY) o += exp2f(m - mm) * base[s * stride + 2 + e];
    }
    O[((size_t)b * Hq + kvh * G + h) * D + e] = o / lsum;
  }
}

}  // namespace hst
