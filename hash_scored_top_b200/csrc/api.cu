// C ABI of libhash_scored_top.so: argument validation, launch planning and
// launches. Every entry point validates on the host before launching
// anything, allocates nothing, and runs asynchronously on the caller's stream.
#include <algorithm>
#include <climits>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cudaTypedefs.h>

#include "../../include/hash_scored_top.h"
#include "socket_kernels.cuh"
#include "estimator.cuh"
#include "adaptive.cuh"
#include "hash_tc.cuh"
#include "step_io.cuh"

using namespace hst;

namespace {

thread_local std::string g_last_error = "no error";
unsigned long long* g_phase_ts = nullptr;     // profiling hook, see sk_profile_phases

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return SK_OK;
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Raises a kernel's dynamic shared-memory limit (and allows 16-CTA clusters)
// once per kernel; later calls with the same or a smaller size skip the
// driver call. Kernels are told apart by address.
struct KernelAttr {
  const void* fn;
  size_t smem;
  bool big_cluster;
};

template <typename Kern>
cudaError_t set_kernel_smem(Kern kern, size_t smem, bool big_cluster = false) {
  static std::mutex mu;
  static std::vector<KernelAttr> done;
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(mu);
  KernelAttr* rec = nullptr;
  for (auto& r : done)
    if (r.fn == fn) rec = &r;
  if (rec == nullptr) {
    done.push_back(KernelAttr{fn, 0, false});
    rec = &done.back();
  }
  cudaError_t e = cudaSuccess;
  if (smem > rec->smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) rec->smem = smem;
  }
  if (e == cudaSuccess && big_cluster && !rec->big_cluster) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e == cudaSuccess) rec->big_cluster = true;
  }
  return e;
}

constexpr int kMaxL = 64;
constexpr int kNumSMs = 148;

// Shapes common to the decode-side calls.
int check_heads(int B, int Hq, int Hkv, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1) return fail(SK_ERR_INVALID_ARG, "B, Hq, Hkv must be >= 1");
  if (Hq % Hkv) return fail(SK_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (d != 64 && d != 128) return fail(SK_ERR_UNSUPPORTED, "head dim d=%d: only 64 and 128 are supported", d);
  return SK_OK;
}

int check_cache(int Ncap, int N) {
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  if (N < 1 || N > Ncap) return fail(SK_ERR_INVALID_ARG, "N=%d must be in [1, Ncap=%d]", N, Ncap);
  return SK_OK;
}

int check_tables(int L, int P, float tau) {
  if (P < 1 || P > 8) return fail(SK_ERR_UNSUPPORTED, "P=%d: 1 <= P <= 8 (bucket IDs are bytes)", P);
  if (L < 1 || L > kMaxL) return fail(SK_ERR_UNSUPPORTED, "L=%d: 1 <= L <= %d", L, kMaxL);
  if (!(tau > 0.f)) return fail(SK_ERR_INVALID_ARG, "tau must be > 0");
  return SK_OK;
}

int check_dtype(sk_dtype t) {
  if (t != SK_F32 && t != SK_BF16) return fail(SK_ERR_INVALID_ARG, "unknown dtype %d", (int)t);
  return SK_OK;
}

#define SK_TRY(expr)            \
  do {                          \
    const int _rc = (expr);     \
    if (_rc != SK_OK) return _rc; \
  } while (0)

#define SK_NONNULL(ptr)                                                          \
  do {                                                                           \
    if ((ptr) == nullptr) return fail(SK_ERR_INVALID_ARG, "%s is NULL", #ptr);   \
  } while (0)

// Alignment the kernels' vector loads and bulk copies rely on.
#define SK_ALIGNED(ptr, bytes)                                                                   \
  do {                                                                                           \
    if (reinterpret_cast<uintptr_t>(ptr) % (bytes))                                              \
      return fail(SK_ERR_INVALID_ARG, "%s must be %d-byte aligned", #ptr, (int)(bytes));         \
  } while (0)

// ---------------------------------------------------------------- plans
// Splits over keys of the attention kernel: one wave of ~2 CTAs per SM
// (sparse) or several waves (dense), at least 16 keys each.
int attend_splits(int n, int pairs, bool dense) {
  const int target = (dense ? 4 : 2) * kNumSMs;
  int splits = dense ? (target + pairs - 1) / pairs : target / pairs;
  int max_splits = (n + 15) / 16;
  if (max_splits > ATTEND_MAX_SPLITS) max_splits = ATTEND_MAX_SPLITS;
  if (splits > max_splits) splits = max_splits;
  return splits < 1 ? 1 : splits;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of the attention kernel: partials, then one counter per pair.
size_t attend_ws_bytes(int pairs, int splits, int G, int d) {
  return align256((size_t)pairs * splits * G * (d + 2) * sizeof(float)) + align256((size_t)pairs * 4);
}

int table_chunks_of(int L) { return ids_bytes_per_key(L) > 32 ? 2 : 1; }

// Fused-kernel plan: cluster size C and slice sizes, or C = 0 if the shape
// cannot run fused.
struct FusedPlan {
  int C = 0, blocks_per_cta = 0, chunk = 0;
};

// Capacities of the fused kernel's shared-memory plan, with the dynamic
// window starting at byte SMEM_BASE_EXPECTED (the kernel re-checks).
constexpr uint32_t kTableAddr = 65536;
constexpr uint32_t kFixedBytes = ((sizeof(SelShared) + 15u) & ~15u) + 4u * (hist_words(0) + hist_words(1) +
                                                                             hist_words(2));
constexpr uint32_t kSegAFree = kTableAddr - SMEM_BASE_EXPECTED - kFixedBytes;
uint32_t seg_b_bytes(int nch) { return SMEM_BASE_EXPECTED + SMEM_DYN_MAX - kTableAddr - nch * TABLE_BYTES; }
uint32_t fused_key_capacity(int nch) { return ((kSegAFree / 4u) & ~127u) + seg_b_bytes(nch) / 4u; }

FusedPlan plan_select(int pairs, int N, int k, int G, int d, int L, int P, bool hata, int max_c) {
  FusedPlan fp;
  const int nch = table_chunks_of(L);
  const int nblk = (N + 31) / 32;
  // one CTA per SM for every pair at once, in clusters of at most 8 CTAs
  // (16-CTA clusters need a free GPC each and do not all fit at once); larger
  // clusters only when a pair's keys do not fit
  int c = 1;
  while (c * 2 <= std::min(max_c, 8) && pairs * c * 2 <= kNumSMs) c *= 2;
  for (; c <= max_c; c *= 2) {
    const int bpc = (nblk + c - 1) / c;
    const int per = ((L + c - 1) / c + 3) & ~3;
    const int nl = per < L ? per : L;
    // the hard-hash variant builds all its 16 tables in every CTA, with its
    // scratch in segment B; the soft tables' scratch is in segment A
    const bool fits = hata ? hamming_scratch_bytes(G, d, L) <= seg_b_bytes(nch)
                           : table_scratch_dbl_bytes(G, d, nl, P) <= kSegAFree &&
                                 table_scratch_rows_bytes(d, nl, P) <= seg_b_bytes(nch);
    if ((((uint32_t)bpc * 32u + 127u) & ~127u) <= fused_key_capacity(nch) && fits) {
      fp.C = c;
      fp.blocks_per_cta = bpc;
      fp.chunk = (k + c - 1) / c;
      return fp;
    }
  }
  (void)k;
  return fp;
}

int max_cluster_size() {
  static int cached = 0;
  if (cached) return cached;
  // 16-CTA clusters need the non-portable opt-in and a free GPC; probe once.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(16, 1, 1);
  cfg.blockDim = dim3(FUSED_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_DYN_MAX;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 16;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = socket_select_kernel<128, 32, __nv_bfloat16, false>;
  int n = 0;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_DYN_MAX) == cudaSuccess &&
      cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) {
    cached = 16;
  } else {
    cached = 8;
  }
  cudaGetLastError();
  return cached;
}

// pdl: launch as the programmatic dependent of the previous kernel in the
// stream (the kernel waits before reading what that kernel writes).
template <typename Kern, typename Params>
int launch_cluster(Kern kern, int grid, int C, size_t smem, cudaStream_t s, const Params& p, bool pdl = false) {
  if (set_kernel_smem(kern, smem, C > 8) != cudaSuccess) return check_launch("cudaFuncSetAttribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(FUSED_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "fused launch: %s", cudaGetErrorString(e));
  return check_launch("fused kernel");
}

template <int D, typename QT, bool HATA>
int launch_select_t(const FusedParams& p0, int pairs, bool pdl, cudaStream_t s) {
  const int grid = pairs * p0.C;
  FusedParams p = p0;
  auto go = [&](auto kern) {
    if (grid > kNumSMs) {
      // CTAs per wave: clusters that fit at once (occupancy API, cached per
      // kernel and cluster size) times the cluster size
      static std::mutex mu;
      static std::vector<std::pair<std::pair<const void*, int>, int>> cache;
      const void* fn = reinterpret_cast<const void*>(kern);
      int n = -1;
      {
        std::lock_guard<std::mutex> lock(mu);
        for (const auto& e : cache)
          if (e.first.first == fn && e.first.second == p.C) n = e.second;
      }
      if (n < 0) {
        n = 0;
        if (set_kernel_smem(kern, SMEM_DYN_MAX, p.C > 8) == cudaSuccess) {
          cudaLaunchConfig_t cfg = {};
          cfg.gridDim = dim3(grid, 1, 1);
          cfg.blockDim = dim3(FUSED_THREADS, 1, 1);
          cfg.dynamicSmemBytes = SMEM_DYN_MAX;
          cudaLaunchAttribute attr[1];
          attr[0].id = cudaLaunchAttributeClusterDimension;
          attr[0].val.clusterDim.x = (unsigned)p.C;
          attr[0].val.clusterDim.y = 1;
          attr[0].val.clusterDim.z = 1;
          cfg.attrs = attr;
          cfg.numAttrs = 1;
          if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();
        std::lock_guard<std::mutex> lock(mu);
        cache.push_back({{fn, p.C}, n});
      }
      p.next_stride = n * p.C < grid ? n * p.C : 0;
    }
    return launch_cluster(kern, grid, p.C, SMEM_DYN_MAX, s, p, pdl);
  };
  switch (ids_bytes_per_key(p.L)) {
    case 16: return go(socket_select_kernel<D, 16, QT, HATA>);
    case 32: return go(socket_select_kernel<D, 32, QT, HATA>);
    case 48: return go(socket_select_kernel<D, 48, QT, HATA>);
    default: return go(socket_select_kernel<D, 64, QT, HATA>);
  }
}

int launch_select(const FusedParams& p, int pairs, int d, sk_dtype q, bool hata, bool pdl, cudaStream_t s) {
  if (hata) {
    if (d == 128) return q == SK_BF16 ? launch_select_t<128, __nv_bfloat16, true>(p, pairs, pdl, s)
                                      : launch_select_t<128, float, true>(p, pairs, pdl, s);
    return q == SK_BF16 ? launch_select_t<64, __nv_bfloat16, true>(p, pairs, pdl, s)
                        : launch_select_t<64, float, true>(p, pairs, pdl, s);
  }
  if (d == 128) return q == SK_BF16 ? launch_select_t<128, __nv_bfloat16, false>(p, pairs, pdl, s)
                                    : launch_select_t<128, float, false>(p, pairs, pdl, s);
  return q == SK_BF16 ? launch_select_t<64, __nv_bfloat16, false>(p, pairs, pdl, s)
                      : launch_select_t<64, float, false>(p, pairs, pdl, s);
}

// ---------------------------------------------------------------- unfused pieces
template <int D, int LP, typename QT>
int launch_tables_t(const TableParams& tp, int pairs, int G, cudaStream_t s) {
  const int ny = tp.L < 16 ? tp.L : 16;
  const size_t smem = table_scratch_bytes(G, D, (tp.L + ny - 1) / ny, tp.P);
  if (smem > (size_t)SMEM_DYN_MAX) return fail(SK_ERR_UNSUPPORTED, "bucket table scratch too large (G=%d)", G);
  auto kern = bucket_table_kernel<D, LP, QT>;
  set_kernel_smem(kern, smem);
  kern<<<dim3(pairs, ny), 256, smem, s>>>(tp);
  return check_launch("bucket_table_kernel");
}

template <int D, typename QT>
int launch_tables_d(const TableParams& tp, int pairs, int G, cudaStream_t s) {
  switch (ids_bytes_per_key(tp.L)) {
    case 16: return launch_tables_t<D, 16, QT>(tp, pairs, G, s);
    case 32: return launch_tables_t<D, 32, QT>(tp, pairs, G, s);
    case 48: return launch_tables_t<D, 48, QT>(tp, pairs, G, s);
    default: return launch_tables_t<D, 64, QT>(tp, pairs, G, s);
  }
}

int launch_tables(const void* Q, sk_dtype q, const void* R, int B, int Hq, int Hkv, int d, int L, int P, float tau,
                  float* T, cudaStream_t s) {
  TableParams tp;
  tp.Q = Q;
  tp.R = reinterpret_cast<const __nv_bfloat16*>(R);
  tp.T = T;
  tp.Hq = Hq;
  tp.Hkv = Hkv;
  tp.L = L;
  tp.P = P;
  tp.tau = tau;
  const int G = Hq / Hkv, pairs = B * Hkv;
  if (d == 128) return q == SK_BF16 ? launch_tables_d<128, __nv_bfloat16>(tp, pairs, G, s)
                                    : launch_tables_d<128, float>(tp, pairs, G, s);
  return q == SK_BF16 ? launch_tables_d<64, __nv_bfloat16>(tp, pairs, G, s)
                      : launch_tables_d<64, float>(tp, pairs, G, s);
}

// Chunks of the unfused score kernel: one wave of CTAs (one per SM) over all
// pairs when the pairs fit, else one CTA per pair.
dim3 score_grid(int pairs, int nblk, int* blocks_per_cta) {
  const int chunks = std::max(1, std::min(kNumSMs / std::max(1, pairs), nblk));
  *blocks_per_cta = (nblk + chunks - 1) / chunks;
  return dim3(pairs, (nblk + *blocks_per_cta - 1) / *blocks_per_cta);
}

template <int LP, bool NORM = true>
int launch_score_t(const ScoreParams& sp, dim3 grid, cudaStream_t s) {
  const int smem = (int)(kTableAddr + table_chunks(LP) * TABLE_BYTES - SMEM_BASE_EXPECTED);
  set_kernel_smem(socket_score_kernel<LP, NORM>, smem);
  socket_score_kernel<LP, NORM><<<grid, FUSED_THREADS, smem, s>>>(sp);
  return check_launch("socket_score_kernel");
}

// The hard-hash variant's tables (16 byte-tables from R128) into T.
int launch_hamming_tables(const void* Q, sk_dtype q, const void* R128, int B, int Hq, int Hkv, int d, float* T,
                          cudaStream_t s) {
  TableParams tp;
  tp.Q = Q;
  tp.R = reinterpret_cast<const __nv_bfloat16*>(R128);
  tp.T = T;
  tp.Hq = Hq;
  tp.Hkv = Hkv;
  tp.L = 16;
  tp.P = 8;
  tp.tau = 1.f;
  const int G = Hq / Hkv, pairs = B * Hkv;
  const size_t smem = hamming_scratch_bytes(G, d, 16);
  if (d == 128) {
    auto kern = q == SK_BF16 ? hamming_table_kernel<128, __nv_bfloat16> : hamming_table_kernel<128, float>;
    set_kernel_smem(kern, smem);
    kern<<<pairs, 256, smem, s>>>(tp);
  } else {
    auto kern = q == SK_BF16 ? hamming_table_kernel<64, __nv_bfloat16> : hamming_table_kernel<64, float>;
    set_kernel_smem(kern, smem);
    kern<<<pairs, 256, smem, s>>>(tp);
  }
  return check_launch("hamming_table_kernel");
}

// Hard-hash scores from the codes (16 bytes per key, no norms).
int launch_hamming_score(const float* T, const void* codes, int pairs, int Ncap, int N, float* scores, cudaStream_t s) {
  ScoreParams sp;
  sp.T = T;
  sp.ids = reinterpret_cast<const uint8_t*>(codes);
  sp.norms = nullptr;
  sp.scores = scores;
  sp.Ncap = Ncap;
  sp.N = N;
  const dim3 grid = score_grid(pairs, (N + 31) / 32, &sp.blocks_per_cta);
  return launch_score_t<16, false>(sp, grid, s);
}

int launch_score(const float* T, const void* ids, const void* norms, int pairs, int Ncap, int N, int L, float* scores,
                 cudaStream_t s, int pair_div = 1) {
  ScoreParams sp;
  sp.pair_div = pair_div;
  sp.T = T;
  sp.ids = reinterpret_cast<const uint8_t*>(ids);
  sp.norms = reinterpret_cast<const __half*>(norms);
  sp.scores = scores;
  sp.Ncap = Ncap;
  sp.N = N;
  const dim3 grid = score_grid(pairs, (N + 31) / 32, &sp.blocks_per_cta);
  switch (ids_bytes_per_key(L)) {
    case 16: return launch_score_t<16>(sp, grid, s);
    case 32: return launch_score_t<32>(sp, grid, s);
    case 48: return launch_score_t<48>(sp, grid, s);
    default: return launch_score_t<64>(sp, grid, s);
  }
}

size_t table_image_bytes(int pairs, int L) { return (size_t)pairs * table_chunks_of(L) * TABLE_BYTES; }

constexpr int kTopkFixed = (int)kFixedBytes;

int topk_cluster_size(int N, int max_c) {
  const int cap = (SMEM_DYN_MAX - kTopkFixed) / 4;
  for (int c = 1; c <= max_c; c *= 2)
    if ((N + c - 1) / c <= cap) return c;
  return 0;
}

int launch_topk(const float* scores, int pairs, int Ncap, int N, int k, int* idx, cudaStream_t s) {
  const int C = topk_cluster_size(N, max_cluster_size());
  if (C == 0) return fail(SK_ERR_UNSUPPORTED, "top-k: N=%d too large", N);
  TopkParams tp;
  tp.scores = scores;
  tp.idx = idx;
  tp.Ncap = Ncap;
  tp.N = N;
  tp.k = k;
  tp.C = C;
  tp.keys_per_cta = (N + C - 1) / C;
  const size_t smem = kTopkFixed + (size_t)tp.keys_per_cta * 4;
  auto kern = socket_topk_kernel;
  if (set_kernel_smem(kern, smem, C > 8) != cudaSuccess) return check_launch("cudaFuncSetAttribute(topk smem)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs * C, 1, 1);
  cfg.blockDim = dim3(FUSED_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tp);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "top-k launch: %s", cudaGetErrorString(e));
  return check_launch("socket_topk_kernel");
}

// Adaptive top-k: one cluster per unit, the unit's scores split over its CTAs.
int launch_adaptive_topk(const float* scores, int units, int Ncap, int N, float mass, int k_min, int k_max, int* idx,
                         int* kcount, cudaStream_t s) {
  const int cap = (int)((SMEM_DYN_MAX - kAdaptFixedBytes) / 4);
  // keys per CTA: a multiple of 4, so every CTA's scores start on 16 bytes
  auto per_cta = [&](int c) { return ((N + c - 1) / c + 3) & ~3; };
  int C = 0;
  for (int c = 1; c <= max_cluster_size(); c *= 2)
    if (adapt_key_slots(per_cta(c)) <= cap) {
      C = c;
      break;
    }
  if (C == 0) return fail(SK_ERR_UNSUPPORTED, "adaptive top-k: N=%d too large", N);
  AdaptParams ap;
  ap.scores = scores;
  ap.idx = idx;
  ap.kcount = kcount;
  ap.Ncap = Ncap;
  ap.N = N;
  ap.k_min = k_min;
  ap.k_max = k_max;
  ap.C = C;
  ap.keys_per_cta = per_cta(C);
  ap.mass = mass;
  const size_t smem = kAdaptFixedBytes + (size_t)adapt_key_slots(ap.keys_per_cta) * 4;
  auto kern = socket_adaptive_topk_kernel;
  if (set_kernel_smem(kern, smem, C > 8) != cudaSuccess) return check_launch("cudaFuncSetAttribute(adaptive smem)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(units * C, 1, 1);
  cfg.blockDim = dim3(FUSED_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ap);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "adaptive top-k launch: %s", cudaGetErrorString(e));
  return check_launch("socket_adaptive_topk_kernel");
}

// Clusters of S CTAs (1, S, 1) that fit on the GPU at once with this launch
// shape, from the occupancy API (cached per kernel, S and shared size).
template <typename Kern>
int attend_active_clusters(Kern kern, int pairs, int S, size_t smem) {
  struct Rec {
    const void* fn;
    int S;
    size_t smem;
    int n;
  };
  static std::mutex mu;
  static std::vector<Rec> cache;
  const void* fn = reinterpret_cast<const void*>(kern);
  std::lock_guard<std::mutex> lock(mu);
  for (const Rec& r : cache)
    if (r.fn == fn && r.S == S && r.smem == smem) return r.n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs, S, 1);
  cfg.blockDim = dim3(ATTEND_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = (unsigned)S;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();
  cache.push_back(Rec{fn, S, smem, n});
  return n;
}

template <int D, typename KVT>
int launch_attend_t(AttendParams ap, int pairs, int G, bool pdl, bool cluster, cudaStream_t s) {
  auto kern = cluster ? socket_attend_kernel<D, KVT, true> : socket_attend_kernel<D, KVT, false>;
  if (cluster) {
    // the largest cluster (at most the planned split count) whose clusters,
    // one per pair, all fit on the GPU at once
    const int s0 = ap.splits;
    int S = s0;
    for (;;) {
      const size_t sm = attend_smem_bytes<D>(G, (ap.n + S - 1) / S);
      if (set_kernel_smem(kern, sm, S > 8) != cudaSuccess) return check_launch("cudaFuncSetAttribute(attend smem)");
      if (S == 1 || attend_active_clusters(kern, pairs, S, sm) >= pairs) break;
      S = S > 8 ? 8 : S / 2;
    }
    ap.splits = S;
    ap.keys_per_split = (ap.n + S - 1) / S;
  }
  const size_t smem = attend_smem_bytes<D>(G, ap.idx ? ap.keys_per_split : 0);
  if (set_kernel_smem(kern, smem, cluster && ap.splits > 8) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(attend smem)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs, ap.splits, 1);
  cfg.blockDim = dim3(ATTEND_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster) {                       // the splits of a pair form one cluster
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = (unsigned)ap.splits;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ap);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "attention launch: %s", cudaGetErrorString(e));
  return check_launch("socket_attend_kernel");
}

// Attention over idx (sparse, n = k) or all keys (dense, idx = NULL, n = N).
// Sparse attention with allow_cluster merges its splits inside a cluster
// (at most max_cluster_size() splits); otherwise the splits merge through
// workspace ws (partials + counters). zero_counters: clear the counters first
// (standalone calls); otherwise the selection kernel did.
// pair_div / counts: see AttendParams (units per cache pair; per-unit list
// lengths).
int launch_attend(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx, int B, int Hq, int Hkv,
                  int Ncap, int n, int d, float scale, float* O, void* ws, size_t ws_bytes, bool pdl,
                  bool zero_counters, cudaStream_t s, bool allow_cluster = true, int pair_div = 1,
                  const int* counts = nullptr, const int* page_table = nullptr, int max_pages = 0,
                  int page_size = 0, int num_pages = 0) {
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  AttendParams ap;
  ap.pair_div = pair_div;
  ap.counts = counts;
  ap.page_table = page_table;
  ap.max_pages = max_pages;
  ap.page_size = page_size;
  ap.num_pages = num_pages;
  ap.Q = Q;
  ap.K = K;
  ap.V = V;
  ap.idx = idx;
  ap.O = O;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.Ncap = Ncap;
  ap.n = n;
  ap.splits = attend_splits(n, pairs, idx == nullptr);
  const bool cluster = allow_cluster && idx != nullptr;
  if (cluster) ap.splits = std::min(ap.splits, max_cluster_size());
  ap.keys_per_split = (n + ap.splits - 1) / ap.splits;
  ap.scale = scale;
  ap.phase_ts = g_phase_ts ? g_phase_ts + (size_t)16 * pairs * PHASES : nullptr;   // after the selection's CTAs
  const size_t need = attend_ws_bytes(pairs, ap.splits, G, d);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  ap.part = reinterpret_cast<float*>(ws);
  ap.counters = reinterpret_cast<unsigned int*>(reinterpret_cast<char*>(ws) +
                                                align256((size_t)pairs * ap.splits * G * (d + 2) * sizeof(float)));
  if (zero_counters && !cluster) {
    const cudaError_t e = cudaMemsetAsync(ap.counters, 0, (size_t)pairs * 4, s);
    if (e != cudaSuccess) return fail(SK_ERR_CUDA, "counter reset: %s", cudaGetErrorString(e));
  }
  if (d == 128) return kv == SK_BF16 ? launch_attend_t<128, __nv_bfloat16>(ap, pairs, G, pdl, cluster, s)
                                     : launch_attend_t<128, float>(ap, pairs, G, pdl, cluster, s);
  return kv == SK_BF16 ? launch_attend_t<64, __nv_bfloat16>(ap, pairs, G, pdl, cluster, s)
                       : launch_attend_t<64, float>(ap, pairs, G, pdl, cluster, s);
}

// ---------------------------------------------------------------- paged K/V
// Where a pool lives: device memory (read by the attention kernel's bulk
// copies through the page table) or host memory that the device can read
// (gathered with plain loads first). Anything else is rejected.
enum PoolKind { POOL_DEVICE = 0, POOL_HOST = 1, POOL_BAD = 2 };

PoolKind pool_kind(const void* ptr) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return POOL_BAD;
  }
  if (a.type == cudaMemoryTypeDevice) return POOL_DEVICE;
  if (a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeManaged) return a.devicePointer ? POOL_HOST : POOL_BAD;
  return POOL_BAD;
}

// Workspace of the paged attention: for a host pool, the gathered K and V rows
// and the attention workspace over them (dense, one split set per pair); for a
// device pool, the sparse attention workspace. Sized for the larger.
size_t paged_attend_ws_bytes(int pairs, int G, int d, int k, int kv_bytes) {
  const size_t host = 2 * align256((size_t)pairs * k * d * kv_bytes) + attend_ws_bytes(pairs, attend_splits(k, pairs, true), G, d);
  return std::max(host, attend_ws_bytes(pairs, attend_splits(k, pairs, false), G, d));
}

int launch_gather(const GatherParams& gp, int units, int row_bytes, cudaStream_t s) {
  const dim3 grid(units, (gp.n + GATHER_KEYS - 1) / GATHER_KEYS);
  switch (row_bytes) {
    case 128: paged_gather_kernel<128><<<grid, GATHER_THREADS, 0, s>>>(gp); break;
    case 256: paged_gather_kernel<256><<<grid, GATHER_THREADS, 0, s>>>(gp); break;
    case 512: paged_gather_kernel<512><<<grid, GATHER_THREADS, 0, s>>>(gp); break;
    default: return fail(SK_ERR_UNSUPPORTED, "row of %d bytes", row_bytes);
  }
  return check_launch("paged_gather_kernel");
}

// Attention over idx [units][k] with K/V in a paged pool (see AttendParams).
int paged_attend_impl(const void* Q, const void* K_pool, const void* V_pool, sk_dtype kv, const int* page_table,
                      int max_pages, int page_size, int num_pages, const int* idx, int B, int Hq, int Hkv, int d, int k,
                      float scale, float* O, void* ws, size_t ws_bytes, cudaStream_t s, int pair_div = 1) {
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const int esz = kv == SK_BF16 ? 2 : 4;
  const PoolKind kk = pool_kind(K_pool), kvk = pool_kind(V_pool);
  if (kk == POOL_BAD || kvk == POOL_BAD || kk != kvk)
    return fail(SK_ERR_INVALID_ARG, "K_pool and V_pool must both be device memory or both device-readable host memory");
  const size_t need = paged_attend_ws_bytes(pairs, G, d, k, esz);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  if (kk == POOL_DEVICE)
    return launch_attend(Q, K_pool, V_pool, kv, idx, B, Hq, Hkv, 32, k, d, scale, O, ws, ws_bytes, false, true, s,
                         true, pair_div, nullptr, page_table, max_pages, page_size, num_pages);
  // host pool: gather the rows into the workspace, then dense attention over them
  char* w = reinterpret_cast<char*>(ws);
  void* Ks = w;
  void* Vs = w + align256((size_t)pairs * k * d * esz);
  char* aw = w + 2 * align256((size_t)pairs * k * d * esz);
  GatherParams gp;
  cudaPointerAttributes ak, av;
  cudaPointerGetAttributes(&ak, K_pool);
  cudaPointerGetAttributes(&av, V_pool);
  gp.K = ak.devicePointer;
  gp.V = av.devicePointer;
  gp.page_table = page_table;
  gp.idx = idx;
  gp.Ks = Ks;
  gp.Vs = Vs;
  gp.n = k;
  gp.max_pages = max_pages;
  gp.page_size = page_size;
  gp.num_pages = num_pages;
  gp.pair_div = pair_div;
  SK_TRY(launch_gather(gp, pairs, d * esz, s));
  return launch_attend(Q, Ks, Vs, kv, nullptr, B, Hq, Hkv, k, k, d, scale, O, aw, ws_bytes - (size_t)(aw - w), false,
                       true, s);
}

// Workspace of a decode step: the index list (when idx_out is NULL), the
// attention workspace, then room for the units' table images (used when the
// selection takes more than one wave of clusters; see decode_impl).
size_t decode_ws_bytes(int B, int Hq, int Hkv, int k, int d, int L) {
  const int pairs = B * Hkv, G = Hq / Hkv;
  return align256((size_t)pairs * k * 4) + attend_ws_bytes(pairs, attend_splits(k, pairs, false), G, d) +
         align256(table_image_bytes(pairs, L));
}

// Workspace of the unfused decode chain: tables, scores, then a decode workspace.
size_t chain_ws_bytes(int B, int Hq, int Hkv, int Ncap, int d, int L, int k) {
  const int pairs = B * Hkv;
  return align256(table_image_bytes(pairs, L)) + align256((size_t)pairs * Ncap * 4) + decode_ws_bytes(B, Hq, Hkv, k, d, L);
}

// Workspace of the selection alone: none when it runs as one cluster kernel,
// else the unfused chain's tables and scores.
size_t select_ws_bytes(const FusedPlan& fp, int pairs, int Ncap, int L) {
  if (fp.C > 0) return 0;
  return align256(table_image_bytes(pairs, L)) + align256((size_t)pairs * Ncap * 4);
}

// 2-D tensor map of a [rows][d] bf16 matrix for TMA tiles of 64 columns x
// box_rows rows with the 128-byte swizzle (the layout the tcgen05 hash
// kernel's operands use). The driver's encoder is looked up once through the
// runtime.
int encode_rows_map(CUtensorMap* map, const void* base, long rows, int d, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (encode == nullptr) return fail(SK_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SK_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SK_OK;
}

constexpr int kAppendMaxKeys = 16;

int hash_launch(const void* K, const void* V, sk_dtype kv, const void* R, int B, int Hkv, int Ncap, int n_begin,
                int n_count, int d, int L, int P, void* ids, void* norms, cudaStream_t s, bool pdl = false) {
  HashParams hp;
  hp.K = K;
  hp.V = V;
  hp.R = reinterpret_cast<const __nv_bfloat16*>(R);
  hp.ids = reinterpret_cast<uint8_t*>(ids);
  hp.norms = reinterpret_cast<__half*>(norms);
  hp.Hkv = Hkv;
  hp.Ncap = Ncap;
  hp.n_begin = n_begin;
  hp.n_count = n_count;
  hp.d = d;
  hp.L = L;
  hp.P = P;
  hp.pairs = B * Hkv;
  const int LP = L * P;
  if (kv == SK_BF16 && P == 8 && n_count > kAppendMaxKeys) {   // tcgen05 projections, tiles of 128 keys
    const TcPlan pl = tc_plan(d, L, V != nullptr);
    TcRows tr;
    tr.tile_key0 = n_begin / TC_M;
    tr.tiles_per_pair = (n_begin + n_count - 1) / TC_M - tr.tile_key0 + 1;
    tr.n_tiles = hp.pairs * tr.tiles_per_pair;
    CUtensorMap mapK, mapV, mapR;
    std::memset(&mapV, 0, sizeof(mapV));
    SK_TRY(encode_rows_map(&mapR, R, (long)8 * L, d, 32));
    SK_TRY(encode_rows_map(&mapK, K, (long)hp.pairs * Ncap, d, TC_M));
    if (V != nullptr) SK_TRY(encode_rows_map(&mapV, V, (long)hp.pairs * Ncap, d, TC_M));
    // at most 512 / (the columns one CTA allocates) CTAs may share an SM's
    // tensor memory: ask for enough shared memory that no more fit
    const int share = 512 / (pl.ncols * (pl.ahead ? 2 : 1));
    size_t smem = pl.smem;
    const size_t floor_bytes = (size_t)(TC_SMEM_SM / (share + 1)) - 1024 + 16;
    if (smem < floor_bytes) smem = floor_bytes;
    int per_sm = 1;
    if (d == 64) {
      set_kernel_smem(hash_keys_tcgen05_kernel<64>, smem);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hash_keys_tcgen05_kernel<64>, TC_THREADS, smem);
    } else {
      set_kernel_smem(hash_keys_tcgen05_kernel<128>, smem);
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, hash_keys_tcgen05_kernel<128>, TC_THREADS, smem);
    }
    const long slots = (long)(per_sm > 0 ? per_sm : 1) * kNumSMs;
    const int grid = (int)(tr.n_tiles < slots ? tr.n_tiles : slots);
    if (d == 64) hash_keys_tcgen05_kernel<64><<<grid, TC_THREADS, smem, s>>>(hp, tr, mapK, mapV, mapR);
    else hash_keys_tcgen05_kernel<128><<<grid, TC_THREADS, smem, s>>>(hp, tr, mapK, mapV, mapR);
    return check_launch("hash_keys_tcgen05_kernel");
  }
  if (n_count <= kAppendMaxKeys) {      // decode-time append: a few keys per pair
    const dim3 grid(hp.pairs, n_count);
    const int threads = (LP + 31) / 32 * 32;
    // pdl: the programmatic dependent of the kernel that wrote the step's inputs
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const cudaError_t e = kv == SK_BF16 ? cudaLaunchKernelEx(&cfg, hash_keys_append_kernel<__nv_bfloat16>, hp)
                                        : cudaLaunchKernelEx(&cfg, hash_keys_append_kernel<float>, hp);
    if (e != cudaSuccess) return fail(SK_ERR_CUDA, "append launch: %s", cudaGetErrorString(e));
    return check_launch("hash_keys_append_kernel");
  }
  const size_t smem = (((size_t)d * LP * 2 + 15) & ~(size_t)15) + (size_t)32 * d * 4 + (size_t)LP * 4;
  const long units = (long)hp.pairs * ((n_begin + n_count - 1) / 32 - n_begin / 32 + 1);
  const int grid = (int)(units < 8L * kNumSMs ? units : 8L * kNumSMs);
  if (kv == SK_BF16) {
    set_kernel_smem(hash_keys_simt_kernel<__nv_bfloat16>, smem);
    hash_keys_simt_kernel<__nv_bfloat16><<<grid, HASH_THREADS, smem, s>>>(hp);
  } else {
    set_kernel_smem(hash_keys_simt_kernel<float>, smem);
    hash_keys_simt_kernel<float><<<grid, HASH_THREADS, smem, s>>>(hp);
  }
  return check_launch("hash_keys_simt_kernel");
}

// Soft-count estimator plan: keys per CTA of the attend kernel. Two CTAs per
// SM when a CTA's factor image and at least 32 keys fit half the shared
// memory, else one; then as many keys per CTA as make the grid about one wave
// (at least 64), within the shared memory.
struct EstPlan {
  int keys_per_split = 0, splits = 0;
  size_t smem = 0;
};

EstPlan plan_estimator(int pairs, int k, int G, int d, int L, int kv_bytes) {
  EstPlan ep;
  const size_t fixed = est_smem_plan(G, d, L, 0, kv_bytes).total + 64;   // plus alignment slack
  const size_t per_key = est_bytes_per_key(G, d, L, kv_bytes);
  const size_t half = (size_t)SMEM_DYN_MAX / 2 - 1024;
  const bool two = fixed + 32 * per_key <= half;
  const size_t budget = two ? half : (size_t)SMEM_DYN_MAX;
  if (fixed + per_key > budget) return ep;                           // nothing fits
  const int fit = (int)((budget - fixed) / per_key);
  const int ctas = (two ? 2 : 1) * kNumSMs;
  const int want_splits = std::max(1, ctas / pairs);                  // at most one wave
  // at least 64 keys per CTA (fewer splits to merge), as far as they fit
  int kps = std::min(fit, std::max(64, (k + want_splits - 1) / want_splits));
  kps = std::max(1, kps);
  ep.keys_per_split = kps;
  ep.splits = (k + kps - 1) / kps;
  ep.smem = est_smem_plan(G, d, L, kps, kv_bytes).total;
  return ep;
}

// Workspace of the estimator: the factor image, the split partials, the counters.
size_t est_factor_bytes(int pairs, int G, int L) { return align256((size_t)pairs * G * L * EST_F * 4); }
size_t est_part_bytes(int pairs, int splits, int G, int d) { return align256((size_t)pairs * splits * G * (d + 1) * 4); }
size_t est_ws_bytes(int pairs, int splits, int G, int d, int L) {
  return est_factor_bytes(pairs, G, L) + est_part_bytes(pairs, splits, G, d) + align256((size_t)pairs * 4);
}

template <int D, typename KVT, int LP>
int launch_estimator_t(const EstFactorParams& fp, const EstParams& ep, int pairs, size_t smem, cudaStream_t s) {
  const int G = fp.Hq / fp.Hkv;
  auto fk = est_factor_kernel<D, KVT>;
  const size_t fsm = est_factor_smem_bytes(G, D, fp.P);
  if (set_kernel_smem(fk, fsm) != cudaSuccess) return check_launch("cudaFuncSetAttribute(estimator factors smem)");
  fk<<<dim3(pairs, (fp.L + EST_TABLES_PER_CTA - 1) / EST_TABLES_PER_CTA), 256, fsm, s>>>(fp);
  SK_TRY(check_launch("est_factor_kernel"));
  auto kern = soft_count_attend_kernel<D, KVT, LP>;
  if (set_kernel_smem(kern, smem) != cudaSuccess) return check_launch("cudaFuncSetAttribute(estimator smem)");
  // programmatic dependent of the factor kernel: the copies of the keys' ID
  // and value rows overlap it; the factor image is read after its completion
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs, ep.splits, 1);
  cfg.blockDim = dim3(EST_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ep);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "estimator launch: %s", cudaGetErrorString(e));
  return check_launch("soft_count_attend_kernel");
}

template <int LP>
int launch_estimator_d(const EstFactorParams& fp, const EstParams& ep, int pairs, size_t smem, int d, sk_dtype kv,
                       cudaStream_t s) {
  if (d == 128) return kv == SK_BF16 ? launch_estimator_t<128, __nv_bfloat16, LP>(fp, ep, pairs, smem, s)
                                     : launch_estimator_t<128, float, LP>(fp, ep, pairs, smem, s);
  return kv == SK_BF16 ? launch_estimator_t<64, __nv_bfloat16, LP>(fp, ep, pairs, smem, s)
                       : launch_estimator_t<64, float, LP>(fp, ep, pairs, smem, s);
}

}  // namespace

// ================================================================ C ABI
extern "C" {

const char* sk_last_error(void) { return g_last_error.c_str(); }

const char* sk_version(void) { return "hash_scored_top_b200 0.1 (sm_100a)"; }

int socket_hash_keys(const void* K, const void* V, sk_dtype kv, const void* R, int B, int Hkv, int Ncap, int n_begin,
                     int n_count, int d, int L, int P, void* ids, void* norms, void* stream) {
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hkv, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  SK_TRY(check_tables(L, P, 1.f));
  if (L * P > 512) return fail(SK_ERR_UNSUPPORTED, "L*P=%d > 512", L * P);
  if (n_begin < 0 || n_count < 0 || (long)n_begin + n_count > Ncap)
    return fail(SK_ERR_INVALID_ARG, "key range [%d, %d+%d) outside [0, Ncap=%d)", n_begin, n_begin, n_count, Ncap);
  if (n_count == 0) return SK_OK;
  return hash_launch(K, V, kv, R, B, Hkv, Ncap, n_begin, n_count, d, L, P, ids, norms, as_stream(stream));
}

int socket_score(const void* Q, sk_dtype q, const void* R, const void* ids, const void* norms, int B, int Hq, int Hkv,
                 int Ncap, int N, int d, int L, int P, float tau, float* scores, void* ws, size_t ws_bytes,
                 void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(scores);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(q));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  const size_t need = table_image_bytes(B * Hkv, L);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  cudaStream_t s = as_stream(stream);
  float* T = reinterpret_cast<float*>(ws);
  SK_TRY(launch_tables(Q, q, R, B, Hq, Hkv, d, L, P, tau, T, s));
  return launch_score(T, ids, norms, B * Hkv, Ncap, N, L, scores, s);
}

int socket_topk(const float* scores, int B, int Hkv, int Ncap, int N, int k, int* idx, void* ws, size_t ws_bytes,
                void* stream) {
  (void)ws;
  (void)ws_bytes;
  SK_NONNULL(scores);
  SK_NONNULL(idx);
  if (B < 1 || Hkv < 1) return fail(SK_ERR_INVALID_ARG, "B, Hkv must be >= 1");
  SK_TRY(check_cache(Ncap, N));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  return launch_topk(scores, B * Hkv, Ncap, N, k, idx, as_stream(stream));
}

int socket_sparse_attend(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx, int B, int Hq,
                         int Hkv, int Ncap, int d, int k, float scale, float* O, void* ws, size_t ws_bytes,
                         void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(idx);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  if (k < 1) return fail(SK_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, ws, ws_bytes, false, true,
                       as_stream(stream));
}

}  // extern "C"

namespace {

// Fixed scratch of socket_sparse_attend_noalloc: the attention partials and
// the per-pair merge counters. It lives in the library's own device image, so
// every GPU that loads the library holds these bytes until the process exits,
// and every call of the entry point on that GPU shares them.
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device. In host code the
// array's name stands for a host-side shadow symbol, not device memory, so the
// address must come from the runtime; it is looked up once per device (with
// that device current) and cached.
int noalloc_scratch_address(void** out) {
  constexpr int kMaxDevices = 64;
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(SK_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(SK_ERR_CUDA, "static scratch address on device %d: %s", dev, cudaGetErrorString(e));
    addr[dev] = p;
  }
  *out = addr[dev];
  return SK_OK;
}

}  // namespace

extern "C" {

size_t sk_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int socket_sparse_attend_noalloc(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx, int B,
                                 int Hq, int Hkv, int Ncap, int d, int k, float scale, float* O, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(idx);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  if (k < 1) return fail(SK_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  // same split count as socket_sparse_attend, hence the same partial layout
  const size_t need = attend_ws_bytes(pairs, attend_splits(k, pairs, false), G, d);
  if (need > kNoAllocScratchBytes)
    return fail(SK_ERR_WORKSPACE,
                "socket_sparse_attend_noalloc: B=%d Hkv=%d G=%d d=%d needs %zu bytes of scratch, above the fixed "
                "%zu-byte static scratch; call socket_sparse_attend with a caller workspace instead",
                B, Hkv, G, d, need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  SK_TRY(noalloc_scratch_address(&scratch));
  // the merge counters keep the previous call's contents and must start at
  // zero; the partials are written before they are read
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, scratch, kNoAllocScratchBytes,
                       /*pdl=*/false, /*zero_counters=*/true, as_stream(stream), /*allow_cluster=*/false);
}

namespace {

// The decode step: selection kernel (tables, scores, exact top-k -> index list)
// then the attention kernel (programmatic dependent launch), or the unfused
// chain when the selection cannot keep a pair's keys on chip.
// per_head: every query head is its own unit (its own table, index set and
// attention); the kernels then see Hq "KV heads" of group size 1, each unit
// reading the cache of KV head h / G.
int decode_impl(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, const void* ids,
                const void* norms, int B, int Hq, int Hkv_cache, int Ncap, int N, int d, int L, int P, float tau,
                int k, float scale, float* O, int* idx_out, void* ws, size_t ws_bytes, bool hata, bool attend,
                cudaStream_t s, bool after_append = false, bool per_head = false) {
  const int pair_div = per_head ? Hq / Hkv_cache : 1;
  const int Hkv = per_head ? Hq : Hkv_cache;
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const FusedPlan fp = plan_select(pairs, N, k, G, d, L, P, hata, max_cluster_size());

  const size_t need = !attend ? select_ws_bytes(fp, pairs, Ncap, L)
                      : fp.C > 0 ? decode_ws_bytes(B, Hq, Hkv, k, d, L) : chain_ws_bytes(B, Hq, Hkv, Ncap, d, L, k);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  char* w = reinterpret_cast<char*>(ws);
  if (fp.C == 0) {        // unfused chain through the workspace
    float* T = reinterpret_cast<float*>(w);
    w += align256(table_image_bytes(pairs, L));
    float* scores = reinterpret_cast<float*>(w);
    w += align256((size_t)pairs * Ncap * 4);
    int* idx = idx_out ? idx_out : reinterpret_cast<int*>(w);
    w += align256((size_t)pairs * k * 4);
    if (hata) {            // hard-hash chain: byte-tables, integer scores from the codes
      SK_TRY(launch_hamming_tables(Q, kv, R, B, Hq, Hkv, d, T, s));
      SK_TRY(launch_hamming_score(T, ids, pairs, Ncap, N, scores, s));
    } else {
      SK_TRY(launch_tables(Q, kv, R, B, Hq, Hkv, d, L, P, tau, T, s));
      SK_TRY(launch_score(T, ids, norms, pairs, Ncap, N, L, scores, s, pair_div));
    }
    SK_TRY(launch_topk(scores, pairs, Ncap, N, k, idx, s));
    if (!attend) return SK_OK;
    return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, w,
                         attend_ws_bytes(pairs, attend_splits(k, pairs, false), G, d), false, true, s, true, pair_div);
  }
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(w);
  const int splits = attend_splits(k, pairs, false);
  unsigned int* counters = nullptr;
  if (attend) {
    w += align256((size_t)pairs * k * 4);
    counters = reinterpret_cast<unsigned int*>(w + align256((size_t)pairs * splits * G * (d + 2) * sizeof(float)));
  }
  FusedParams p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.R = reinterpret_cast<const __nv_bfloat16*>(R);
  p.ids = reinterpret_cast<const uint8_t*>(ids);
  p.norms = reinterpret_cast<const __half*>(norms);
  p.O = O;
  p.idx_out = idx;
  p.counters = counters;
  p.phase_ts = g_phase_ts;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Ncap = Ncap;
  p.N = N;
  p.L = L;
  p.P = P;
  p.k = k;
  p.C = fp.C;
  p.blocks_per_cta = fp.blocks_per_cta;
  p.chunk = fp.chunk;
  p.tau = tau;
  p.scale = scale;
  p.pair_div = pair_div;
  // A selection of more than one wave of clusters gets its units' tables
  // from a table kernel run once beforehand: every later wave would otherwise
  // rebuild them (the hard-hash byte-tables take ~13 us per CTA). The
  // selection then starts after that kernel (an ordinary launch).
  const bool precompute = attend && (long)pairs * fp.C > kNumSMs;
  if (precompute) {
    float* T = reinterpret_cast<float*>(w + attend_ws_bytes(pairs, splits, G, d));
    if (hata) SK_TRY(launch_hamming_tables(Q, kv, R, B, Hq, Hkv, d, T, s));
    else SK_TRY(launch_tables(Q, kv, R, B, Hq, Hkv, d, L, P, tau, T, s));
    p.tables = T;
  }
  SK_TRY(launch_select(p, pairs, d, kv, hata, after_append && !precompute, s));
  if (!attend) return SK_OK;
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, w, attend_ws_bytes(pairs, splits, G, d),
                       true, false, s, true, pair_div);
}

// Workspace of the adaptive decode chain (units = B Hkv or B Hq): tables,
// scores, then the attention workspace planned for k_max keys per unit.
size_t adaptive_ws_bytes(int B, int Hq, int Hu, int Ncap, int d, int L, int k_max) {
  const int units = B * Hu, G = Hq / Hu;
  return align256(table_image_bytes(units, L)) + align256((size_t)units * Ncap * 4) +
         attend_ws_bytes(units, attend_splits(k_max, units, false), G, d);
}

// The adaptive decode: bucket tables -> scores -> adaptive top-k -> attention
// over each unit's kcount keys.
int adaptive_impl(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, const void* ids,
                  const void* norms, int B, int Hq, int Hkv_cache, int Ncap, int N, int d, int L, int P, float tau,
                  bool per_head, float mass, int k_min, int k_max, float scale, float* O, int* idx, int* kcount,
                  void* ws, size_t ws_bytes, cudaStream_t s) {
  const int pair_div = per_head ? Hq / Hkv_cache : 1;
  const int Hu = per_head ? Hq : Hkv_cache;
  const int units = B * Hu, G = Hq / Hu;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const size_t need = adaptive_ws_bytes(B, Hq, Hu, Ncap, d, L, k_max);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  char* w = reinterpret_cast<char*>(ws);
  float* T = reinterpret_cast<float*>(w);
  w += align256(table_image_bytes(units, L));
  float* scores = reinterpret_cast<float*>(w);
  w += align256((size_t)units * Ncap * 4);
  SK_TRY(launch_tables(Q, kv, R, B, Hq, Hu, d, L, P, tau, T, s));
  SK_TRY(launch_score(T, ids, norms, units, Ncap, N, L, scores, s, pair_div));
  SK_TRY(launch_adaptive_topk(scores, units, Ncap, N, mass, k_min, k_max, idx, kcount, s));
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hu, Ncap, k_max, d, scale, O, w,
                       attend_ws_bytes(units, attend_splits(k_max, units, false), G, d), false, true, s, true,
                       pair_div, kcount);
}

}  // namespace

int socket_decode(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, const void* ids,
                  const void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau, int k,
                  float scale, float* O, int* idx_out, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  return decode_impl(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, scale, O, idx_out, ws, ws_bytes,
                     false, true, as_stream(stream));
}

}  // extern "C" (reopened below)

namespace {
// The device's address of page-locked host memory that it can read and write
// directly (16-byte aligned), or null (pageable memory, or anything else):
// the step then uses DMA copies, which accept any host memory.
void* mapped_host(const void* ptr) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  if ((reinterpret_cast<uintptr_t>(a.devicePointer) & 15) != 0) return nullptr;
  return a.devicePointer;
}

// The argument checks of socket_decode_append (no launch).
int socket_decode_append_check(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R,
                               const void* ids, const void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d,
                               int L, int P, float tau, int k, const float* O, const void* ws, size_t ws_bytes) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (L * P > 512) return fail(SK_ERR_UNSUPPORTED, "L*P=%d > 512", L * P);
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  // the workspace check comes before the first launch: a failure launches nothing
  {
    const int pairs = B * Hkv, G = Hq / Hkv;
    if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
    const FusedPlan fp = plan_select(pairs, N, k, G, d, L, P, false, max_cluster_size());
    const size_t need = fp.C > 0 ? decode_ws_bytes(B, Hq, Hkv, k, d, L) : chain_ws_bytes(B, Hq, Hkv, Ncap, d, L, k);
    if (ws == nullptr || ws_bytes < need)
      return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  }
  return SK_OK;
}
}  // namespace

extern "C" {

}  // extern "C" (reopened below)

namespace {
// The step of socket_decode_append after its checks; pdl: the hashing kernel
// is the programmatic dependent of a kernel that wrote the step's inputs.
int append_and_decode(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, void* ids, void* norms,
                      int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau, int k, float scale,
                      float* O, int* idx_out, void* ws, size_t ws_bytes, cudaStream_t s, bool pdl) {
  SK_TRY(hash_launch(K, V, kv, R, B, Hkv, Ncap, N - 1, 1, d, L, P, ids, norms, s, pdl));
  return decode_impl(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, scale, O, idx_out, ws, ws_bytes,
                     false, true, s, true);
}
}  // namespace

extern "C" {

int socket_decode_append(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, void* ids,
                         void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau, int k,
                         float scale, float* O, int* idx_out, void* ws, size_t ws_bytes, void* stream) {
  SK_TRY(socket_decode_append_check(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, O, ws,
                                    ws_bytes));
  const cudaStream_t s = as_stream(stream);
  return append_and_decode(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, scale, O, idx_out, ws,
                           ws_bytes, s, false);
}

int socket_decode_step_host(const void* Q_host, const void* K_new_host, const void* V_new_host, void* Q, void* K,
                            void* V, sk_dtype kv, const void* R, void* ids, void* norms, int B, int Hq, int Hkv,
                            int Ncap, int N, int d, int L, int P, float tau, int k, float scale, float* O,
                            float* O_host, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q_host);
  SK_NONNULL(K_new_host);
  SK_NONNULL(V_new_host);
  SK_NONNULL(O_host);
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(O);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  // everything the step checks, before the first copy: a failure moves and launches nothing
  SK_TRY(socket_decode_append_check(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, O, ws, ws_bytes));
  const cudaStream_t s = as_stream(stream);
  const size_t es = kv == SK_BF16 ? 2 : 4;
  const size_t row = (size_t)d * es;                 // a multiple of 16 bytes (d % 32 == 0)
  char* krow = reinterpret_cast<char*>(K) + (size_t)(N - 1) * row;
  char* vrow = reinterpret_cast<char*>(V) + (size_t)(N - 1) * row;
  const void* qd = mapped_host(Q_host);
  const void* kd = mapped_host(K_new_host);
  const void* vd = mapped_host(V_new_host);
  void* od = mapped_host(O_host);
  cudaError_t e = cudaSuccess;
  if (qd && kd && vd) {
    // one kernel reads the three inputs from host memory: the query, and the
    // new token's rows into row N - 1 of every pair (Ncap rows apart)
    StepCopyParams cp = {};
    cp.jobs = 3;
    cp.src[0] = static_cast<const char*>(qd);
    cp.dst[0] = static_cast<char*>(Q);
    cp.rows[0] = B * Hq;
    cp.src[1] = static_cast<const char*>(kd);
    cp.dst[1] = krow;
    cp.rows[1] = B * Hkv;
    cp.src[2] = static_cast<const char*>(vd);
    cp.dst[2] = vrow;
    cp.rows[2] = B * Hkv;
    for (int j = 0; j < 3; ++j) {
      cp.row16[j] = (int)(row / 16);
      cp.src_pitch[j] = row;
      cp.dst_pitch[j] = j == 0 ? row : (size_t)Ncap * row;
    }
    const long long words = (long long)(B * Hq) * (long long)(row / 16);
    const int blocks = (int)std::min<long long>(kNumSMs, (words + STEP_COPY_THREADS - 1) / STEP_COPY_THREADS);
    step_copy_kernel<<<blocks, STEP_COPY_THREADS, 0, s>>>(cp);
    SK_TRY(check_launch("step_copy_kernel"));
  } else {
    e = cudaMemcpyAsync(Q, Q_host, (size_t)B * Hq * row, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(krow, (size_t)Ncap * row, K_new_host, row, row, (size_t)B * Hkv, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(vrow, (size_t)Ncap * row, V_new_host, row, row, (size_t)B * Hkv, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return fail(SK_ERR_CUDA, "step input copy: %s", cudaGetErrorString(e));
  }
  // with the copy kernel, the hashing kernel is its programmatic dependent
  SK_TRY(append_and_decode(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, scale, O, nullptr, ws,
                           ws_bytes, s, qd && kd && vd));
  const size_t obytes = (size_t)B * Hq * d * sizeof(float);
  if (od) {
    StepCopyParams cp = {};
    cp.jobs = 1;
    cp.src[0] = reinterpret_cast<const char*>(O);
    cp.dst[0] = static_cast<char*>(od);
    cp.rows[0] = 1;
    cp.row16[0] = (int)(obytes / 16);
    cp.src_pitch[0] = obytes;
    cp.dst_pitch[0] = obytes;
    // the programmatic dependent of the attention kernel: launched ahead, it
    // reads O once that kernel has completed
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<size_t>(kNumSMs, (obytes / 16 + STEP_COPY_THREADS - 1) / STEP_COPY_THREADS));
    cfg.blockDim = dim3(STEP_COPY_THREADS);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, step_copy_kernel, cp);
    if (e != cudaSuccess) return fail(SK_ERR_CUDA, "step output copy launch: %s", cudaGetErrorString(e));
    SK_TRY(check_launch("step_copy_kernel"));
  } else {
    e = cudaMemcpyAsync(O_host, O, obytes, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return fail(SK_ERR_CUDA, "step output copy: %s", cudaGetErrorString(e));
  }
  return SK_OK;
}

int socket_select(const void* Q, sk_dtype q, const void* R, const void* ids, const void* norms, int B, int Hq, int Hkv,
                  int Ncap, int N, int d, int L, int P, float tau, int k, int* idx, void* ws, size_t ws_bytes,
                  void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(idx);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(q));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  return decode_impl(Q, nullptr, nullptr, q, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, 0.f, nullptr, idx,
                     ws, ws_bytes, false, false, as_stream(stream));
}

int socket_decode_heads(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, const void* ids,
                        const void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau,
                        int k, float scale, float* O, int* idx_out, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  return decode_impl(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, scale, O, idx_out, ws, ws_bytes,
                     false, true, as_stream(stream), false, /*per_head=*/true);
}

int socket_decode_adaptive(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R, const void* ids,
                           const void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau,
                           int per_head, float mass, int k_min, int k_max, float scale, float* O, int* idx,
                           int* kcount, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(O);
  SK_NONNULL(idx);
  SK_NONNULL(kcount);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (per_head != 0 && per_head != 1) return fail(SK_ERR_INVALID_ARG, "per_head=%d must be 0 or 1", per_head);
  if (!(mass > 0.f && mass <= 1.f)) return fail(SK_ERR_INVALID_ARG, "mass must be in (0, 1]");
  if (k_min < 1 || k_min > k_max || k_max > N)
    return fail(SK_ERR_INVALID_ARG, "need 1 <= k_min (%d) <= k_max (%d) <= N (%d)", k_min, k_max, N);
  return adaptive_impl(Q, K, V, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, per_head == 1, mass, k_min,
                       k_max, scale, O, idx, kcount, ws, ws_bytes, as_stream(stream));
}

// Shared checks of the paged entry points.
static int check_pages(const int* page_table, int max_pages, int page_size, int num_pages) {
  SK_NONNULL(page_table);
  if (max_pages < 1 || page_size < 1 || num_pages < 1)
    return fail(SK_ERR_INVALID_ARG, "max_pages=%d, page_size=%d, num_pages=%d must be >= 1", max_pages, page_size,
                num_pages);
  if ((long long)max_pages * page_size > INT_MAX || (long long)num_pages * page_size > INT_MAX)
    return fail(SK_ERR_UNSUPPORTED, "more than 2^31 - 1 rows per pair or per pool");
  return SK_OK;
}

int socket_sparse_attend_paged(const void* Q, const void* K_pool, const void* V_pool, sk_dtype kv, const int* page_table,
                               int max_pages, int page_size, int num_pages, const int* idx, int B, int Hq, int Hkv,
                               int d, int k, float scale, float* O, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K_pool);
  SK_NONNULL(V_pool);
  SK_NONNULL(idx);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K_pool, 16);
  SK_ALIGNED(V_pool, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_pages(page_table, max_pages, page_size, num_pages));
  if (k < 1) return fail(SK_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  return paged_attend_impl(Q, K_pool, V_pool, kv, page_table, max_pages, page_size, num_pages, idx, B, Hq, Hkv, d, k,
                           scale, O, ws, ws_bytes, as_stream(stream));
}

int socket_decode_paged(const void* Q, const void* K_pool, const void* V_pool, sk_dtype kv, const int* page_table,
                        int max_pages, int page_size, int num_pages, const void* R, const void* ids, const void* norms,
                        int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau, int k, float scale,
                        float* O, int* idx_out, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K_pool);
  SK_NONNULL(V_pool);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(norms);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K_pool, 16);
  SK_ALIGNED(V_pool, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_ALIGNED(norms, 2);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  SK_TRY(check_pages(page_table, max_pages, page_size, num_pages));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  if ((long long)max_pages * page_size < N)
    return fail(SK_ERR_INVALID_ARG, "max_pages * page_size = %lld < N = %d", (long long)max_pages * page_size, N);
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const FusedPlan fp = plan_select(pairs, N, k, G, d, L, P, false, max_cluster_size());
  const size_t list_bytes = align256((size_t)pairs * k * 4);
  const size_t sel = align256(select_ws_bytes(fp, pairs, Ncap, L));
  const size_t need = list_bytes + sel + paged_attend_ws_bytes(pairs, G, d, k, kv == SK_BF16 ? 2 : 4);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  char* w = reinterpret_cast<char*>(ws);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(w);
  const cudaStream_t s = as_stream(stream);
  // selection from the (contiguous) hashed-key cache, then the paged attention
  SK_TRY(decode_impl(Q, nullptr, nullptr, kv, R, ids, norms, B, Hq, Hkv, Ncap, N, d, L, P, tau, k, 0.f, nullptr, idx,
                     w + list_bytes, sel, false, false, s));
  return paged_attend_impl(Q, K_pool, V_pool, kv, page_table, max_pages, page_size, num_pages, idx, B, Hq, Hkv, d, k,
                           scale, O, w + list_bytes + sel, ws_bytes - list_bytes - sel, s);
}

int hata_hash_keys(const void* K, sk_dtype kv, const void* R128, int B, int Hkv, int Ncap, int n_begin, int n_count,
                   int d, void* codes, void* stream) {
  SK_NONNULL(K);
  SK_NONNULL(R128);
  SK_NONNULL(codes);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(R128, 16);
  SK_ALIGNED(codes, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hkv, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  if (n_begin < 0 || n_count < 0 || (long)n_begin + n_count > Ncap)
    return fail(SK_ERR_INVALID_ARG, "key range [%d, %d+%d) outside [0, Ncap=%d)", n_begin, n_begin, n_count, Ncap);
  if (n_count == 0) return SK_OK;
  // 128 code bits = 16 "tables" of 8 hyperplanes
  return hash_launch(K, nullptr, kv, R128, B, Hkv, Ncap, n_begin, n_count, d, 16, 8, codes, nullptr,
                     as_stream(stream));
}

int hata_decode(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R128, const void* codes, int B,
                int Hq, int Hkv, int Ncap, int N, int d, int k, float scale, float* O, int* idx_out, void* ws,
                size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R128);
  SK_NONNULL(codes);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R128, 16);
  SK_ALIGNED(codes, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  if (Hq / Hkv > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", Hq / Hkv);
  // 128 code bits = 16 byte-tables of 8 hyperplanes; no norms
  return decode_impl(Q, K, V, kv, R128, codes, codes, B, Hq, Hkv, Ncap, N, d, 16, 8, 1.f, k, scale, O, idx_out, ws,
                     ws_bytes, true, true, as_stream(stream));
}

int dense_decode(const void* Q, const void* K, const void* V, sk_dtype kv, int B, int Hq, int Hkv, int Ncap, int N,
                 int d, float scale, float* O, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(K, 16);
  SK_ALIGNED(V, 16);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  return launch_attend(Q, K, V, kv, nullptr, B, Hq, Hkv, Ncap, N, d, scale, O, ws, ws_bytes, false, true,
                       as_stream(stream));
}


int socket_soft_count_attend(const void* Q, const void* V, sk_dtype kv, const void* R, const void* ids, const int* idx,
                             int B, int Hq, int Hkv, int Ncap, int d, int L, int P, float tau, int k, float* O,
                             void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(V);
  SK_NONNULL(R);
  SK_NONNULL(ids);
  SK_NONNULL(idx);
  SK_NONNULL(O);
  SK_ALIGNED(Q, 16);
  SK_ALIGNED(V, 16);
  SK_ALIGNED(R, 16);
  SK_ALIGNED(ids, 32);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  SK_TRY(check_tables(L, P, tau));
  if (k < 1) return fail(SK_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const EstPlan plan = plan_estimator(pairs, k, G, d, L, kv == SK_BF16 ? 2 : 4);
  if (plan.splits == 0) return fail(SK_ERR_UNSUPPORTED, "estimator scratch does not fit (G=%d, L=%d)", G, L);
  const size_t need = est_ws_bytes(pairs, plan.splits, G, d, L);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  char* w = reinterpret_cast<char*>(ws);
  EstFactorParams fp;
  fp.Q = Q;
  fp.R = reinterpret_cast<const __nv_bfloat16*>(R);
  fp.F = reinterpret_cast<float*>(w);
  fp.Hq = Hq;
  fp.Hkv = Hkv;
  fp.L = L;
  fp.P = P;
  fp.tau = tau;
  EstParams ep;
  ep.V = V;
  ep.ids = reinterpret_cast<const uint8_t*>(ids);
  ep.idx = idx;
  ep.F = fp.F;
  ep.part = reinterpret_cast<float*>(w + est_factor_bytes(pairs, G, L));
  ep.counters = reinterpret_cast<unsigned int*>(w + est_factor_bytes(pairs, G, L) +
                                                est_part_bytes(pairs, plan.splits, G, d));
  ep.O = O;
  ep.Hq = Hq;
  ep.Hkv = Hkv;
  ep.Ncap = Ncap;
  ep.L = L;
  ep.P = P;
  ep.k = k;
  ep.keys_per_split = plan.keys_per_split;
  ep.splits = plan.splits;
  ep.phase_ts = g_phase_ts;
  cudaStream_t s = as_stream(stream);
  const cudaError_t e = cudaMemsetAsync(ep.counters, 0, (size_t)pairs * 4, s);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "counter reset: %s", cudaGetErrorString(e));
  switch (ids_bytes_per_key(L)) {
    case 16: return launch_estimator_d<16>(fp, ep, pairs, plan.smem, d, kv, s);
    case 32: return launch_estimator_d<32>(fp, ep, pairs, plan.smem, d, kv, s);
    case 48: return launch_estimator_d<48>(fp, ep, pairs, plan.smem, d, kv, s);
    default: return launch_estimator_d<64>(fp, ep, pairs, plan.smem, d, kv, s);
  }
}

size_t sk_workspace_bytes(int op, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, int k) {
  const size_t bad = (size_t)-1;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv) return bad;
  const int pairs = B * Hkv, G = Hq / Hkv;
  switch (op) {
    case SK_OP_HASH_KEYS:
    case SK_OP_HATA_HASH:
    case SK_OP_TOPK:
      return 0;
    case SK_OP_SCORE:
      if (L < 1 || L > kMaxL) return bad;
      return table_image_bytes(pairs, L);
    case SK_OP_SPARSE_ATTEND:
      if (k < 1) return bad;
      return attend_ws_bytes(pairs, attend_splits(k, pairs, false), G, d);
    case SK_OP_DENSE_DECODE:
      if (N < 1) return bad;
      return attend_ws_bytes(pairs, attend_splits(N, pairs, true), G, d);
    case SK_OP_SOFT_COUNT: {
      if (k < 1 || G > 8 || L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      // the split count (hence the partials) depends on the value dtype:
      // the larger of the two
      const int sp = std::max(plan_estimator(pairs, k, G, d, L, 2).splits, plan_estimator(pairs, k, G, d, L, 4).splits);
      return est_ws_bytes(pairs, sp, G, d, L);
    }
    case SK_OP_SELECT: {
      if (k < 1 || N < 1 || G > 8 || L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      return select_ws_bytes(plan_select(pairs, N, k, G, d, L, P, false, 8), pairs, Ncap, L);
    }
    case SK_OP_DECODE:
    case SK_OP_HATA_DECODE: {
      if (k < 1 || N < 1 || G > 8) return bad;
      if (op == SK_OP_HATA_DECODE) {
        L = 16;
        P = 8;
      }
      if (L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      // the unfused chain runs when the selection cannot hold a pair's keys on
      // chip; 8-CTA clusters are always available, 16-CTA ones may not be
      const FusedPlan fp = plan_select(pairs, N, k, G, d, L, P, op == SK_OP_HATA_DECODE, 8);
      if (fp.C > 0) return decode_ws_bytes(B, Hq, Hkv, k, d, L);
      return chain_ws_bytes(B, Hq, Hkv, Ncap, d, L, k);
    }
    case SK_OP_DECODE_HEADS: {
      // one unit per query head: Hq "KV heads" of group size 1
      if (k < 1 || N < 1 || L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      const FusedPlan fp = plan_select(B * Hq, N, k, 1, d, L, P, false, 8);
      if (fp.C > 0) return decode_ws_bytes(B, Hq, Hq, k, d, L);
      return chain_ws_bytes(B, Hq, Hq, Ncap, d, L, k);
    }
    case SK_OP_SPARSE_ATTEND_PAGED:
      if (k < 1 || G > 8) return bad;
      return paged_attend_ws_bytes(pairs, G, d, k, 4);          // f32 rows: the larger staging
    case SK_OP_DECODE_PAGED: {
      if (k < 1 || N < 1 || G > 8 || L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      const FusedPlan fp = plan_select(pairs, N, k, G, d, L, P, false, 8);
      return align256((size_t)pairs * k * 4) + align256(select_ws_bytes(fp, pairs, Ncap, L)) +
             paged_attend_ws_bytes(pairs, G, d, k, 4);
    }
    case SK_OP_DECODE_ADAPTIVE:
    case SK_OP_DECODE_ADAPTIVE_HEADS: {
      // k is k_max
      const int Hu = op == SK_OP_DECODE_ADAPTIVE_HEADS ? Hq : Hkv;
      if (k < 1 || N < 1 || Hq / Hu > 8 || L < 1 || L > kMaxL || P < 1 || P > 8) return bad;
      return adaptive_ws_bytes(B, Hq, Hu, Ncap, d, L, k);
    }
    default:
      return bad;
  }
}

int sk_test_set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : kWaitLimit;
  const cudaError_t e = cudaMemcpyToSymbol(g_tc_wait_limit, &v, sizeof(v));
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "wait limit: %s", cudaGetErrorString(e));
  return SK_OK;
}

int sk_profile_phases(unsigned long long* device_buffer) {
  g_phase_ts = device_buffer;
  return SK_OK;
}

int sk_check_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word));
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "error word: %s", cudaGetErrorString(e));
  if (word) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    if (word & ERR_TIMEOUT) return fail(SK_ERR_TIMEOUT, "a device-side bounded wait gave up");
    if (word & ERR_RANGE)
      return fail(SK_ERR_INVALID_ARG, "a page-table entry was outside [0, num_pages); its rows were read from page 0");
    return fail(SK_ERR_UNSUPPORTED, "a kernel's shared-memory plan did not fit; it wrote nothing");
  }
  return SK_OK;
}

}  // extern "C"
