// C ABI of libhash_scored_top.so: argument validation, launch planning and
// launches. Every entry point validates on the host before launching
// anything, allocates nothing, and runs asynchronously on the caller's stream.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/hash_scored_top.h"
#include "socket_kernels.cuh"

using namespace hst;

namespace {

thread_local std::string g_last_error = "no error";

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

// ---------------------------------------------------------------- plans
constexpr int kAttendKeysPerSplit = 256;

int attend_splits(int n, int pairs, bool dense) {
  if (!dense) return (n + kAttendKeysPerSplit - 1) / kAttendKeysPerSplit;
  // dense: aim at ~4 CTAs per SM, at least 512 keys per split
  int splits = (4 * kNumSMs + pairs - 1) / pairs;
  const int max_splits = (n + 511) / 512;
  if (splits > max_splits) splits = max_splits;
  return splits < 1 ? 1 : splits;
}

size_t attend_part_bytes(int pairs, int splits, int G, int d) {
  return (size_t)pairs * splits * G * (d + 2) * sizeof(float);
}

size_t attend_smem_bytes(int G, int d) {
  return (size_t)(2 * FUSED_WARPS * G + FUSED_WARPS * G * d + 2 * G + G * d) * sizeof(float);
}

// Fused-kernel plan: cluster size C and slice sizes, or C = 0 if the shape
// cannot run fused.
struct FusedPlan {
  int C = 0, blocks_per_cta = 0, chunk = 0;
};

// Capacities of the fused kernel's shared-memory plan, with the dynamic
// window starting at byte SMEM_BASE_EXPECTED (the kernel re-checks).
constexpr uint32_t kTableAddr = 65536;
constexpr uint32_t kSegBBytes = SMEM_BASE_EXPECTED + SMEM_DYN_MAX - kTableAddr - TABLE_BYTES;
uint32_t fused_key_capacity() {
  const uint32_t fixed = ((sizeof(SelShared) + 15u) & ~15u) + (4u << HIST1_BITS) + (4u << HIST2_BITS) +
                         (4u << HIST3_BITS);
  const uint32_t segA = kTableAddr - SMEM_BASE_EXPECTED;
  return (segA - fixed) / 4u + kSegBBytes / 4u;
}

FusedPlan plan_fused(int pairs, int N, int k, int G, int d, int L, int P, bool hata, int max_c) {
  FusedPlan fp;
  if (G > 8) return fp;
  const int nblk = (N + 31) / 32;
  int c = 1;
  while (c * 2 <= max_c && pairs * c * 2 <= kNumSMs) c *= 2;
  for (; c <= max_c; c *= 2) {
    const int bpc = (nblk + c - 1) / c;
    const int chunk = (k + c - 1) / c;
    const int nl = (L + c - 1) / c;
    const size_t scratch = hata ? (size_t)G * 16 * 4 : (size_t)table_scratch_doubles(G, d, nl, P) * 8;
    const size_t attend = attend_smem_bytes(G, d);
    if ((uint32_t)bpc * 32u <= fused_key_capacity() && chunk * 4 <= TABLE_BYTES && scratch <= kSegBBytes &&
        attend <= kSegBBytes) {
      fp.C = c;
      fp.blocks_per_cta = bpc;
      fp.chunk = chunk;
      return fp;
    }
  }
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
  auto kern = socket_decode_fused_kernel<128, 1, __nv_bfloat16, false>;
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

template <typename Kern>
int launch_cluster(Kern kern, int grid, int C, size_t smem, cudaStream_t s, const FusedParams& p) {
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(smem)");
  if (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(cluster)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return fail(SK_ERR_CUDA, "fused launch: %s", cudaGetErrorString(e));
  return check_launch("fused kernel");
}

template <int D, typename KVT, bool HATA>
int launch_fused_t(const FusedParams& p, int pairs, cudaStream_t s) {
  if (p.L <= 32) return launch_cluster(socket_decode_fused_kernel<D, 1, KVT, HATA>, pairs * p.C, p.C, SMEM_DYN_MAX, s, p);
  return launch_cluster(socket_decode_fused_kernel<D, 2, KVT, HATA>, pairs * p.C, p.C, SMEM_DYN_MAX, s, p);
}

int launch_fused(const FusedParams& p, int pairs, int d, sk_dtype kv, bool hata, cudaStream_t s) {
  if (hata) {
    if (d == 128) return kv == SK_BF16 ? launch_fused_t<128, __nv_bfloat16, true>(p, pairs, s)
                                       : launch_fused_t<128, float, true>(p, pairs, s);
    return kv == SK_BF16 ? launch_fused_t<64, __nv_bfloat16, true>(p, pairs, s)
                         : launch_fused_t<64, float, true>(p, pairs, s);
  }
  if (d == 128) return kv == SK_BF16 ? launch_fused_t<128, __nv_bfloat16, false>(p, pairs, s)
                                     : launch_fused_t<128, float, false>(p, pairs, s);
  return kv == SK_BF16 ? launch_fused_t<64, __nv_bfloat16, false>(p, pairs, s)
                       : launch_fused_t<64, float, false>(p, pairs, s);
}

// ---------------------------------------------------------------- unfused pieces
int launch_tables(const void* Q, sk_dtype q, const void* R, int B, int Hq, int Hkv, int d, int L, int P, float tau,
                  float* T, cudaStream_t s) {
  TableParams tp;
  tp.Q = Q;
  tp.R = reinterpret_cast<const __nv_bfloat16*>(R);
  tp.T = T;
  tp.Hq = Hq;
  tp.Hkv = Hkv;
  tp.d = d;
  tp.L = L;
  tp.P = P;
  tp.tau = tau;
  const int G = Hq / Hkv;
  const int ny = L < 16 ? L : 16;
  const size_t smem = (size_t)table_scratch_doubles(G, d, (L + ny - 1) / ny, P) * 8;
  if (smem > (size_t)SMEM_DYN_MAX) return fail(SK_ERR_UNSUPPORTED, "bucket table scratch too large (G=%d)", G);
  dim3 grid(B * Hkv, ny);
  if (q == SK_BF16) {
    cudaFuncSetAttribute(bucket_table_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    bucket_table_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(tp);
  } else {
    cudaFuncSetAttribute(bucket_table_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    bucket_table_kernel<float><<<grid, 256, smem, s>>>(tp);
  }
  return check_launch("bucket_table_kernel");
}

constexpr int kScoreBlocksPerCta = 256;

int launch_score(const float* T, const void* ids, const void* norms, int pairs, int Ncap, int N, int L, float* scores,
                 cudaStream_t s) {
  ScoreParams sp;
  sp.T = T;
  sp.ids = reinterpret_cast<const uint8_t*>(ids);
  sp.norms = reinterpret_cast<const __half*>(norms);
  sp.scores = scores;
  sp.Ncap = Ncap;
  sp.N = N;
  sp.L = L;
  sp.blocks_per_cta = kScoreBlocksPerCta;
  const int nblk = (N + 31) / 32;
  dim3 grid(pairs, (nblk + kScoreBlocksPerCta - 1) / kScoreBlocksPerCta);
  const int smem = (int)(kTableAddr + TABLE_BYTES - SMEM_BASE_EXPECTED);
  if (L <= 32) {
    cudaFuncSetAttribute(socket_score_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    socket_score_kernel<1><<<grid, 256, smem, s>>>(sp);
  } else {
    cudaFuncSetAttribute(socket_score_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    socket_score_kernel<2><<<grid, 256, smem, s>>>(sp);
  }
  return check_launch("socket_score_kernel");
}

constexpr int kTopkFixed = (int)(((sizeof(SelShared) + 15) & ~15) + (4 << HIST1_BITS) + (4 << HIST2_BITS) +
                                 (4 << HIST3_BITS));

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
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return check_launch("cudaFuncSetAttribute(topk smem)");
  if (C > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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

template <int D, typename KVT>
int launch_attend_t(const AttendParams& ap, int pairs, int G, cudaStream_t s) {
  const size_t smem = attend_smem_bytes(G, D);
  cudaFuncSetAttribute(attend_split_kernel<D, KVT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  attend_split_kernel<D, KVT><<<dim3(pairs, ap.splits), FUSED_THREADS, smem, s>>>(ap);
  return check_launch("attend_split_kernel");
}

// Attention over idx (sparse, n = k) or all keys (dense, idx = NULL, n = N).
int launch_attend(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx, int B, int Hq, int Hkv,
                  int Ncap, int n, int d, float scale, float* O, void* ws, size_t ws_bytes, cudaStream_t s) {
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  AttendParams ap;
  ap.Q = Q;
  ap.K = K;
  ap.V = V;
  ap.idx = idx;
  ap.Hq = Hq;
  ap.Hkv = Hkv;
  ap.Ncap = Ncap;
  ap.n = n;
  ap.splits = attend_splits(n, pairs, idx == nullptr);
  ap.keys_per_split = (n + ap.splits - 1) / ap.splits;
  ap.scale = scale;
  const size_t need = attend_part_bytes(pairs, ap.splits, G, d);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  ap.part = reinterpret_cast<float*>(ws);
  int rc;
  if (d == 128) rc = kv == SK_BF16 ? launch_attend_t<128, __nv_bfloat16>(ap, pairs, G, s)
                                   : launch_attend_t<128, float>(ap, pairs, G, s);
  else rc = kv == SK_BF16 ? launch_attend_t<64, __nv_bfloat16>(ap, pairs, G, s)
                          : launch_attend_t<64, float>(ap, pairs, G, s);
  if (rc != SK_OK) return rc;
  merge_splits_kernel<<<pairs * G, d, 0, s>>>(ap.part, O, Hq, Hkv, d, ap.splits);
  return check_launch("merge_splits_kernel");
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of the unfused decode chain: tables, scores, indices, attention partials.
size_t chain_ws_bytes(int B, int Hq, int Hkv, int Ncap, int d, int k) {
  const int pairs = B * Hkv, G = Hq / Hkv;
  return align256((size_t)pairs * TABLE_BYTES) + align256((size_t)pairs * Ncap * 4) +
         align256((size_t)pairs * k * 4) + align256(attend_part_bytes(pairs, attend_splits(k, pairs, false), G, d));
}

int hash_launch(const void* K, const void* V, sk_dtype kv, const void* R, int B, int Hkv, int Ncap, int n_begin,
                int n_count, int d, int L, int P, void* ids, void* norms, cudaStream_t s) {
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
  const size_t smem = (((size_t)d * LP * 2 + 15) & ~(size_t)15) + (size_t)32 * d * 4 + (size_t)LP * 4;
  const long units = (long)hp.pairs * ((n_begin + n_count - 1) / 32 - n_begin / 32 + 1);
  const int grid = (int)(units < 8L * kNumSMs ? units : 8L * kNumSMs);
  if (kv == SK_BF16) {
    cudaFuncSetAttribute(hash_keys_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    hash_keys_simt_kernel<__nv_bfloat16><<<grid, HASH_THREADS, smem, s>>>(hp);
  } else {
    cudaFuncSetAttribute(hash_keys_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    hash_keys_simt_kernel<float><<<grid, HASH_THREADS, smem, s>>>(hp);
  }
  return check_launch("hash_keys_simt_kernel");
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
  SK_TRY(check_dtype(q));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  const size_t need = (size_t)B * Hkv * TABLE_BYTES;
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
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  if (Ncap < 32 || Ncap % 32) return fail(SK_ERR_INVALID_ARG, "Ncap=%d must be a positive multiple of 32", Ncap);
  if (k < 1) return fail(SK_ERR_INVALID_ARG, "k=%d must be >= 1", k);
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, ws, ws_bytes, as_stream(stream));
}

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
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  SK_TRY(check_tables(L, P, tau));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  cudaStream_t s = as_stream(stream);
  const FusedPlan fp = plan_fused(pairs, N, k, G, d, L, P, false, max_cluster_size());
  if (fp.C > 0) {
    FusedParams p;
    p.Q = Q;
    p.K = K;
    p.V = V;
    p.R = reinterpret_cast<const __nv_bfloat16*>(R);
    p.ids = reinterpret_cast<const uint8_t*>(ids);
    p.norms = reinterpret_cast<const __half*>(norms);
    p.O = O;
    p.idx_out = idx_out;
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
    return launch_fused(p, pairs, d, kv, false, s);
  }
  // unfused chain through the workspace
  const size_t need = chain_ws_bytes(B, Hq, Hkv, Ncap, d, k);
  if (ws == nullptr || ws_bytes < need)
    return fail(SK_ERR_WORKSPACE, "workspace: need %zu bytes, got %zu", need, ws == nullptr ? (size_t)0 : ws_bytes);
  char* w = reinterpret_cast<char*>(ws);
  float* T = reinterpret_cast<float*>(w);
  w += align256((size_t)pairs * TABLE_BYTES);
  float* scores = reinterpret_cast<float*>(w);
  w += align256((size_t)pairs * Ncap * 4);
  int* idx = idx_out ? idx_out : reinterpret_cast<int*>(w);
  w += align256((size_t)pairs * k * 4);
  const size_t part_bytes = align256(attend_part_bytes(pairs, attend_splits(k, pairs, false), G, d));
  SK_TRY(launch_tables(Q, kv, R, B, Hq, Hkv, d, L, P, tau, T, s));
  SK_TRY(launch_score(T, ids, norms, pairs, Ncap, N, L, scores, s));
  SK_TRY(launch_topk(scores, pairs, Ncap, N, k, idx, s));
  return launch_attend(Q, K, V, kv, idx, B, Hq, Hkv, Ncap, k, d, scale, O, w, part_bytes, s);
}

int hata_hash_keys(const void* K, sk_dtype kv, const void* R128, int B, int Hkv, int Ncap, int n_begin, int n_count,
                   int d, void* codes, void* stream) {
  SK_NONNULL(K);
  SK_NONNULL(R128);
  SK_NONNULL(codes);
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
  (void)ws;
  (void)ws_bytes;
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(R128);
  SK_NONNULL(codes);
  SK_NONNULL(O);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  if (k < 1 || k > N) return fail(SK_ERR_INVALID_ARG, "k=%d must be in [1, N=%d]", k, N);
  const int pairs = B * Hkv, G = Hq / Hkv;
  if (G > 8) return fail(SK_ERR_UNSUPPORTED, "group size G=%d > 8", G);
  const FusedPlan fp = plan_fused(pairs, N, k, G, d, 16, 8, true, max_cluster_size());
  if (fp.C == 0) return fail(SK_ERR_UNSUPPORTED, "hard-hash decode: N=%d / k=%d too large for one cluster", N, k);
  FusedParams p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.R = reinterpret_cast<const __nv_bfloat16*>(R128);
  p.ids = reinterpret_cast<const uint8_t*>(codes);
  p.norms = nullptr;
  p.O = O;
  p.idx_out = idx_out;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Ncap = Ncap;
  p.N = N;
  p.L = 16;
  p.P = 8;
  p.k = k;
  p.C = fp.C;
  p.blocks_per_cta = fp.blocks_per_cta;
  p.chunk = fp.chunk;
  p.tau = 1.f;
  p.scale = scale;
  return launch_fused(p, pairs, d, kv, true, as_stream(stream));
}

int dense_decode(const void* Q, const void* K, const void* V, sk_dtype kv, int B, int Hq, int Hkv, int Ncap, int N,
                 int d, float scale, float* O, void* ws, size_t ws_bytes, void* stream) {
  SK_NONNULL(Q);
  SK_NONNULL(K);
  SK_NONNULL(V);
  SK_NONNULL(O);
  SK_TRY(check_dtype(kv));
  SK_TRY(check_heads(B, Hq, Hkv, d));
  SK_TRY(check_cache(Ncap, N));
  return launch_attend(Q, K, V, kv, nullptr, B, Hq, Hkv, Ncap, N, d, scale, O, ws, ws_bytes, as_stream(stream));
}

size_t sk_workspace_bytes(int op, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, int k) {
  const size_t bad = (size_t)-1;
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv) return bad;
  const int pairs = B * Hkv, G = Hq / Hkv;
  switch (op) {
    case SK_OP_HASH_KEYS:
    case SK_OP_HATA_HASH:
    case SK_OP_TOPK:
    case SK_OP_HATA_DECODE:
      return 0;
    case SK_OP_SCORE:
      return (size_t)pairs * TABLE_BYTES;
    case SK_OP_SPARSE_ATTEND:
      if (k < 1) return bad;
      return attend_part_bytes(pairs, attend_splits(k, pairs, false), G, d);
    case SK_OP_DENSE_DECODE:
      if (N < 1) return bad;
      return attend_part_bytes(pairs, attend_splits(N, pairs, true), G, d);
    case SK_OP_DECODE: {
      if (k < 1 || N < 1 || G > 8) return bad;
      const FusedPlan fp = plan_fused(pairs, N, k, G, d, L, P, false, 8);
      if (fp.C > 0) return 0;
      return chain_ws_bytes(B, Hq, Hkv, Ncap, d, k);
    }
    default:
      return bad;
  }
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
    return fail(SK_ERR_UNSUPPORTED, "a kernel's shared-memory plan did not fit; it wrote nothing");
  }
  return SK_OK;
}

}  // extern "C"
