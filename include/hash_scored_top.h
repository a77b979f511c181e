/*
 * hash_scored_top.h -- C ABI of libhash_scored_top.so: hash-scored top-k sparse
 * decode attention on NVIDIA B200 (sm_100a).
 *
 * The method is SOCKET (technical summary "SOCKET - SOft Collision Kernel
 * EsTimator for sparse attention", gist.science/ja/paper/2602.06283, section
 * 中核メカニズム：ソフト LSH, steps 1-4), plus a hard-hash (Hamming) variant
 * after the HATA digest ("HATA: Hash-Aware Top-k Attention",
 * aibr.jp/archives/117328, section 3). Each entry point below names the step
 * it implements.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor arguments are DEVICE pointers to contiguous memory owned by
 *   the caller. Alignment: ids 32 bytes; codes, Q, K, V, R, R128 16 bytes;
 *   norms 2 bytes (cudaMalloc and torch allocations satisfy all of these);
 *   a misaligned pointer is rejected with SK_ERR_INVALID_ARG. The library allocates nothing and frees nothing; scratch
 *   memory is passed in as `ws` / `ws_bytes` (query the size with
 *   sk_workspace_bytes). `stream` is a cudaStream_t (NULL = legacy default).
 * - Calls are asynchronous on `stream`. Arguments are validated on the host
 *   before anything is launched; on failure nothing is launched, a non-zero
 *   sk_status is returned and sk_last_error() describes it. A failed launch
 *   returns SK_ERR_CUDA with the CUDA error text in sk_last_error().
 * - Results are deterministic: repeated calls on the same inputs give
 *   bit-identical outputs (no floating-point atomics touch result values).
 * - Shapes: B batch, Hq query heads, Hkv KV heads (Hq % Hkv == 0, group size
 *   G = Hq / Hkv, query head h reads KV head h / G), d head dim (64 or 128),
 *   Ncap cache capacity in keys (multiple of 32), N <= Ncap keys in use,
 *   L hash tables of P hyperplanes each (2^P buckets per table), k keys kept.
 *   A "pair" is one (batch, KV head); pair p = b * Hkv + kvh.
 *
 * Memory layouts
 * --------------
 *   Q      [B][Hq][d]          dtype `kv` (f32 or bf16)
 *   K, V   [B][Hkv][Ncap][d]   dtype `kv`
 *   O      [B][Hq][d]          f32
 *   R      [L*P][d]            bf16; row l*P + j is hyperplane j of table l
 *   R128   [128][d]            bf16; hyperplanes of the 128-bit hard-hash codes
 *   norms  [B][Hkv][Ncap]      f16; cached |v| of each key
 *   ids    [B][Hkv][Ncap][LP] uint8, LP = 16 (L <= 16), 32 (L <= 32),
 *          48 (L <= 48) or 64 (L <= 64) bytes per key, in chunks of S_0, S_1
 *          tables: [16], [32], [32, 16] or [32, 32]. Inside chunk c (tables
 *          32c, 32c+1, ...), byte 32c + j of key n holds the bucket ID of table
 *          32c + (j + n) mod S_c, and 0 where that table is >= L ("rotated
 *          key-major": 32 consecutive keys read 32 different tables at every
 *          byte position). P <= 8, so an ID is one byte.
 *   codes  [B][Hkv][Ncap][16] uint8 in the same layout with 16 "tables": byte
 *          j of key n holds byte (j + n) mod 16 of its 128-bit code; code bit c
 *          is bit c % 8 of code byte c / 8.
 *   scores [B][Hkv][Ncap]      f32 (only the first N per pair are written)
 *   idx    [B][Hkv][k]         int32, ascending key indices
 */
#ifndef HASH_SCORED_TOP_H
#define HASH_SCORED_TOP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SK_F32 = 0, SK_BF16 = 1 } sk_dtype;

typedef enum {
  SK_OK = 0,
  SK_ERR_INVALID_ARG = 1,  /* bad shape, null pointer, out-of-range parameter */
  SK_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not 64/128)  */
  SK_ERR_CUDA = 3,         /* a CUDA call or launch failed                    */
  SK_ERR_TIMEOUT = 4,      /* a device-side bounded wait gave up              */
  SK_ERR_WORKSPACE = 5     /* ws is NULL or smaller than required             */
} sk_status;

/* Operation codes for sk_workspace_bytes. */
typedef enum {
  SK_OP_HASH_KEYS = 0,
  SK_OP_SCORE = 1,
  SK_OP_TOPK = 2,
  SK_OP_SPARSE_ATTEND = 3,
  SK_OP_DECODE = 4,
  SK_OP_HATA_HASH = 5,
  SK_OP_HATA_DECODE = 6,
  SK_OP_DENSE_DECODE = 7,
  SK_OP_SELECT = 8,
  SK_OP_SOFT_COUNT = 9,
  SK_OP_DECODE_HEADS = 10,
  SK_OP_DECODE_ADAPTIVE = 11,        /* k is k_max */
  SK_OP_DECODE_ADAPTIVE_HEADS = 12,  /* k is k_max */
  SK_OP_SPARSE_ATTEND_PAGED = 13,
  SK_OP_DECODE_PAGED = 14
} sk_op;

/*
 * Prefill hashing, SOCKET step 1: for keys n in [n_begin, n_begin + n_count)
 * of every pair, writes the L bucket IDs (bit j of table l's ID is
 * [k_n . r_{l*P+j} > 0], least significant bit first) and the value norm
 * |v_n| rounded to the nearest f16 (ties to even).
 * K, V: [B][Hkv][Ncap][d] (dtype kv); R: [L*P][d] bf16.
 * ids, norms: outputs in the layouts above. Keys outside the range are not
 * touched, so appending one decoded token is n_begin = N, n_count = 1.
 * The projections accumulate in f32; the norm in f64. Ranges of more than
 * 16 keys with bf16 keys and P == 8 run on the tensor cores, shorter ranges
 * (decode-time appends) on a low-latency kernel; the two add the f32
 * projection up in different orders, so a key's bit can depend on which one
 * hashed it only where its projection is within f32 rounding of zero.
 * Requires 1 <= P <= 8, 1 <= L <= 64, L*P <= 512, 0 <= n_begin,
 * n_begin + n_count <= Ncap (n_count == 0 is a no-op).
 */
int socket_hash_keys(const void* K, const void* V, sk_dtype kv, const void* R, int B, int Hkv,
                     int Ncap, int n_begin, int n_count, int d, int L, int P, void* ids,
                     void* norms, void* stream);

/*
 * Soft collision scores, SOCKET steps 2-3: for every pair, the soft bucket
 * assignment p_{h,l}(b) = softmax_b(sum_j s_bj * (q_hat_h . r_{l*P+j}) / tau)
 * (s_bj = +1 if bit j of b is set, else -1; q_hat = q / |q|), summed over the
 * G query heads of the pair, and then score_n = norm_n * sum_l T_l(id_l(n))
 * for n < N. Q: [B][Hq][d] in dtype q. scores: [B][Hkv][Ncap] f32 output.
 * The bucket tables go through ws: sk_workspace_bytes(SK_OP_SCORE, ...) bytes.
 * Requires 1 <= P <= 8, 1 <= L <= 64, tau > 0.
 */
int socket_score(const void* Q, sk_dtype q, const void* R, const void* ids, const void* norms,
                 int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau,
                 float* scores, void* ws, size_t ws_bytes, void* stream);

/*
 * Deterministic top-k, SOCKET step 4: per pair, the k largest of the first N
 * scores (non-negative f32), ties going to the lower key index; writes the
 * chosen indices in ascending order to idx [B][Hkv][k]. Requires 1 <= k <= N.
 * ws: sk_workspace_bytes(SK_OP_TOPK, ...) bytes (may be 0 -> ws may be NULL).
 */
int socket_topk(const float* scores, int B, int Hkv, int Ncap, int N, int k, int* idx, void* ws,
                size_t ws_bytes, void* stream);

/*
 * Exact attention over the selected subset, SOCKET step 4: for every query
 * head h of pair p, O_h = softmax_i(q_h . k_i * scale) v_i over i in idx[p]
 * (renormalised over the subset), with f32 accumulation. Entries of idx must
 * lie in [0, Ncap). ws: sk_workspace_bytes(SK_OP_SPARSE_ATTEND, ...) bytes.
 * Requires 1 <= G <= 8 for bf16 K/V.
 */
int socket_sparse_attend(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx,
                         int B, int Hq, int Hkv, int Ncap, int d, int k, float scale, float* O,
                         void* ws, size_t ws_bytes, void* stream);

/*
 * socket_sparse_attend without a workspace argument, for callers that cannot
 * allocate device memory: a host whose memory manager has already reserved
 * the free HBM (a serving engine that pre-sizes its KV cache, for instance),
 * or code on a latency-critical path where cudaMalloc / cudaFree, which can
 * synchronise the device, are not allowed. The paper has no counterpart: it
 * is a packaging of the same attention, not a step of the method.
 *
 * Same arguments, layout and result as socket_sparse_attend minus ws and
 * ws_bytes. Instead of a caller buffer it uses one fixed static device array
 * of sk_noalloc_scratch_bytes() bytes (4 MiB) inside the library, which every
 * GPU that loads the library holds until the process exits. It allocates
 * nothing. Shapes whose partials exceed that size (roughly B*Hkv above ~1000
 * pairs at G = 8, d = 128) return SK_ERR_WORKSPACE with a message naming the
 * needed and the available bytes, launching nothing.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. Each call clears the merge counters it needs on `stream` before
 * the kernel runs. Every call on a device shares the one array: calls whose
 * kernels overlap on the GPU (different streams, or threads that do not
 * order their streams) race on it and give wrong results. Order them on one
 * stream, or use socket_sparse_attend with a buffer per stream.
 */
int socket_sparse_attend_noalloc(const void* Q, const void* K, const void* V, sk_dtype kv, const int* idx,
                                 int B, int Hq, int Hkv, int Ncap, int d, int k, float scale, float* O,
                                 void* stream);

/* Size in bytes of the static scratch socket_sparse_attend_noalloc uses. */
size_t sk_noalloc_scratch_bytes(void);

/*
 * The decode step, SOCKET steps 2-4: bucket tables, scores, exact top-k and
 * attention over the selection. Two kernels on `stream`: a selection kernel
 * (one thread-block cluster per pair; the pair's scores stay in the
 * cluster's shared memory, never in HBM) writes the index list, and an
 * attention kernel, launched as its programmatic dependent, gathers the
 * selected K/V rows and merges its key splits in a fixed order. The result
 * equals socket_score -> socket_topk -> socket_sparse_attend. idx_out
 * (nullable) receives the selected indices [B][Hkv][k] ascending. When the
 * selection takes more than one wave of clusters, a table kernel first builds
 * every pair's bucket tables once (into ws) and the selection kernel copies
 * them (same tables, same results). Shapes whose keys do not fit one
 * cluster's shared memory run that unfused chain instead (same results). Requires 1 <= P <= 8, 1 <= L <= 64, 1 <= k <= N,
 * tau > 0, G <= 8. ws: sk_workspace_bytes(SK_OP_DECODE, ...) bytes.
 */
int socket_decode(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R,
                  const void* ids, const void* norms, int B, int Hq, int Hkv, int Ncap, int N,
                  int d, int L, int P, float tau, int k, float scale, float* O, int* idx_out,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * One decode step of a decoder loop: appends the current token (key N - 1,
 * already written to K and V by the caller) to the hashed cache exactly like
 * socket_hash_keys(..., n_begin = N - 1, n_count = 1, ...), then runs
 * socket_decode over the N keys (results identical to those two calls). The
 * selection kernel is launched as the programmatic dependent of the hashing
 * kernel: its bucket-table build overlaps the hashing, and it reads bucket
 * IDs and norms only after the hashing completed. ids and norms are updated
 * in place (row N - 1). Requires L * P <= 512 and everything socket_decode
 * requires. ws: sk_workspace_bytes(SK_OP_DECODE, ...) bytes.
 */
int socket_decode_append(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R,
                         void* ids, void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L,
                         int P, float tau, int k, float scale, float* O, int* idx_out, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * One decode step from host buffers (the serving loop's step: the token's
 * query and key/value rows arrive from the host, its output goes back).
 * On `stream`, in order: copies Q_host [B][Hq][d] into Q (device), the new
 * token's rows K_new_host and V_new_host [B][Hkv][d] into row N - 1 of
 * every pair of K and V (one strided copy each), runs socket_decode_append
 * over the N keys (SOCKET page, 中核メカニズム：ソフト LSH, steps 1-4: the
 * appended key's hashing, then the selection and the sparse attention), and
 * copies O [B][Hq][d] float32 into O_host (O holds it too). Host buffers in
 * kv's dtype (Q in it too). Page-locked host memory that the device maps
 * (cudaHostAlloc, pinned tensors), 16-byte aligned, is read and written by a
 * small copy kernel chained to the step's kernels by programmatic launch;
 * any other host memory goes through DMA copies. The buffers must hold the
 * sizes above (the device reads and writes exactly those bytes). All of it
 * is asynchronous on `stream`: O_host holds the result once the stream has
 * synchronised. Every argument is checked before the first copy, so an
 * error moves and launches nothing. Requires what socket_decode_append
 * requires. ws: sk_workspace_bytes(SK_OP_DECODE, ...) bytes.
 */
int socket_decode_step_host(const void* Q_host, const void* K_new_host, const void* V_new_host,
                            void* Q, void* K, void* V, sk_dtype kv, const void* R, void* ids,
                            void* norms, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P,
                            float tau, int k, float scale, float* O, float* O_host, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * Selection only, SOCKET steps 2-4 without the attention: the index list of
 * socket_decode (bucket tables, scores, exact top-k with ties to the lower
 * index), written ascending to idx [B][Hkv][k], for callers that run their
 * own attention over the selected keys. Q: [B][Hq][d] in dtype q. One
 * cluster kernel; shapes it cannot hold on chip run socket_score ->
 * socket_topk through ws. ws: sk_workspace_bytes(SK_OP_SELECT, ...) bytes
 * (0 when the cluster kernel runs; ws may then be NULL).
 * Requires 1 <= P <= 8, 1 <= L <= 64, 1 <= k <= N, tau > 0, G <= 8.
 */
int socket_select(const void* Q, sk_dtype q, const void* R, const void* ids, const void* norms,
                  int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P, float tau, int k,
                  int* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * socket_decode with one index set per QUERY head: head h scores the keys of
 * KV head h / G with its own soft assignment, score_{h,n} = norm_n *
 * sum_l p_{h,l}(id_l(n)) (no sum over the group), takes its own exact top-k
 * (ties to the lower index) and attends over it. With G = 1 this is
 * socket_decode. The same two kernels run with the B * Hq query heads as
 * their units, each reading its KV head's cache, so the group's bucket IDs are
 * read once per query head (from L2 after the first). idx_out (nullable):
 * [B][Hq][k] ascending. Requires what socket_decode requires except G <= 8.
 * ws: sk_workspace_bytes(SK_OP_DECODE_HEADS, ...) bytes.
 */
int socket_decode_heads(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R,
                        const void* ids, const void* norms, int B, int Hq, int Hkv, int Ncap, int N,
                        int d, int L, int P, float tau, int k, float scale, float* O, int* idx_out,
                        void* ws, size_t ws_bytes, void* stream);

/*
 * Decode with an adaptive k (Tactic digest, "Tactic: Adaptive Sparse
 * Attention with Clustering and Distribution Fitting for Long-Context LLMs",
 * aibr.jp/archives/79195, section 3 中核となる技術的要素: tokens are taken
 * until their cumulative score reaches a target), applied to the soft
 * collision scores: for every unit (per_head = 0: a KV head's group, scored
 * by the group-summed table as in socket_decode; per_head = 1: one query
 * head, as in socket_decode_heads),
 *   k = min{ k : sum of the k largest scores >= mass * sum of all N scores },
 * clamped to [k_min, k_max], then the exact top-k (ties to the lower index)
 * and attention over it. idx: [units][k_max] int32, the first kcount[u]
 * entries ascending and the rest -1; kcount: [units] int32; units = B * Hkv
 * or B * Hq. The float64 score sum is formed in a fixed order and the
 * cumulative masses are 64-bit fixed-point integers, so the result is
 * deterministic; it can differ from an exact-arithmetic k only where the
 * target lies within the scores' f32 rounding of a cumulative sum. Four
 * kernels: bucket tables, scores (to ws), the adaptive top-k (one cluster per
 * unit), attention. Requires 0 < mass <= 1, 1 <= k_min <= k_max <= N, and
 * what socket_decode requires (G <= 8 only for per_head = 0).
 * ws: sk_workspace_bytes(SK_OP_DECODE_ADAPTIVE or SK_OP_DECODE_ADAPTIVE_HEADS,
 * ..., k = k_max) bytes.
 */
int socket_decode_adaptive(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R,
                           const void* ids, const void* norms, int B, int Hq, int Hkv, int Ncap, int N,
                           int d, int L, int P, float tau, int per_head, float mass, int k_min,
                           int k_max, float scale, float* O, int* idx, int* kcount, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Sparse attention (as socket_sparse_attend) with K and V in a paged pool
 * (HATA digest, sections 3-4: the offloaded KV cache; HGA page, section 3:
 * hot and routed pages). K_pool, V_pool: [num_pages][page_size][d] (dtype kv);
 * page_table: [B][Hkv][max_pages] int32 device array; key n of pair p is row
 * n % page_size of page page_table[p][n / page_size]. idx: [B][Hkv][k] key
 * indices in [0, max_pages * page_size). The pools may be device memory
 * (the attention kernel reads the selected rows through the page table) or
 * pinned host memory that the device can address (the selected rows are first
 * copied into ws with plain loads over the host link, then attended). Both
 * pools must be of the same kind. A page-table entry outside [0, num_pages) is
 * read as page 0 and reported by sk_check_status (SK_ERR_INVALID_ARG).
 * Requires max_pages, page_size, num_pages >= 1, G <= 8, and fewer than 2^31
 * rows per pool. ws: sk_workspace_bytes(SK_OP_SPARSE_ATTEND_PAGED, ..., k).
 */
int socket_sparse_attend_paged(const void* Q, const void* K_pool, const void* V_pool, sk_dtype kv,
                               const int* page_table, int max_pages, int page_size, int num_pages,
                               const int* idx, int B, int Hq, int Hkv, int d, int k, float scale,
                               float* O, void* ws, size_t ws_bytes, void* stream);

/*
 * The decode step of socket_decode with a paged K/V cache: the selection
 * (steps 2-4) reads the contiguous hashed-key cache (ids, norms as above),
 * then socket_sparse_attend_paged gathers the selected rows from the pools.
 * Same results as socket_decode over the cache the pages describe.
 * Requires max_pages * page_size >= N and what both calls require.
 * ws: sk_workspace_bytes(SK_OP_DECODE_PAGED, ...) bytes.
 */
int socket_decode_paged(const void* Q, const void* K_pool, const void* V_pool, sk_dtype kv,
                        const int* page_table, int max_pages, int page_size, int num_pages,
                        const void* R, const void* ids, const void* norms, int B, int Hq, int Hkv,
                        int Ncap, int N, int d, int L, int P, float tau, int k, float scale, float* O,
                        int* idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Hard-hash codes (HATA digest, section 3, with seeded random hyperplanes
 * standing in for the learned hash): for keys n in [n_begin, n_begin+n_count)
 * of every pair, code bit c = [k_n . r_c > 0] for the 128 rows of R128,
 * written to `codes` in the layout above. The same kernels as
 * socket_hash_keys with 16 tables of 8 hyperplanes and no values.
 */
int hata_hash_keys(const void* K, sk_dtype kv, const void* R128, int B, int Hkv, int Ncap,
                   int n_begin, int n_count, int d, void* codes, void* stream);

/*
 * Hard-hash decode step: query codes from R128, score_n = sum over the G
 * query heads of (128 - popcount(code_q ^ code_n)), exact top-k (ties to the
 * lower index) and exact attention over the selection, as socket_decode.
 * ws: sk_workspace_bytes(SK_OP_HATA_DECODE, ...) bytes.
 */
int hata_decode(const void* Q, const void* K, const void* V, sk_dtype kv, const void* R128,
                const void* codes, int B, int Hq, int Hkv, int Ncap, int N, int d, int k,
                float scale, float* O, int* idx_out, void* ws, size_t ws_bytes, void* stream);

/*
 * Dense decode attention over all N cached keys (the FlashAttention-style
 * baseline the SOCKET page compares against, section 実験結果):
 * O_h = softmax(q_h . K^T * scale) V, split over keys with an exact merge.
 * ws: sk_workspace_bytes(SK_OP_DENSE_DECODE, ...) bytes.
 */
int dense_decode(const void* Q, const void* K, const void* V, sk_dtype kv, int B, int Hq, int Hkv,
                 int Ncap, int N, int d, float scale, float* O, void* ws, size_t ws_bytes,
                 void* stream);

/*
 * The soft-count attention estimator (SOCKET technical summary, section
 * 主要な貢献 item 4, the estimator whose end-to-end error the paper bounds,
 * and section 理論的基盤, the soft score as a kernel estimate): over the
 * selected keys idx[p] of every pair, each query head h of the pair gets
 *   O_h = sum_i c_{h,i} v_i / sum_i c_{h,i},  c_{h,i} = sum_l p_{h,l}(id_l(i)),
 * the soft collision counts of the head's own soft bucket assignment (as in
 * socket_score, with no value-norm weight) in place of the softmax weights.
 * Reads the selected keys' values and cached bucket IDs, not their keys.
 * V: [B][Hkv][Ncap][d] (dtype kv); Q: [B][Hq][d] (dtype kv); R, ids as above;
 * idx: [B][Hkv][k] int32 in [0, Ncap) (any order; the result does not depend
 * on it beyond f32 rounding of the sums); O: [B][Hq][d] f32. The soft
 * assignment's factors are float64 rounded to f32; the counts (relative
 * error below (L + 2) 2^-24) and the weighted sums are f32 sums in a fixed
 * order (deterministic). Two
 * kernels: the heads' soft-assignment factors once per pair (into ws), then
 * the counts and weighted sums, split over the keys.
 * Requires 1 <= P <= 8, 1 <= L <= 64, tau > 0, k >= 1, G <= 8.
 * ws: sk_workspace_bytes(SK_OP_SOFT_COUNT, ..., k) bytes.
 */
int socket_soft_count_attend(const void* Q, const void* V, sk_dtype kv, const void* R, const void* ids, const int* idx,
                             int B, int Hq, int Hkv, int Ncap, int d, int L, int P, float tau, int k, float* O,
                             void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes needed by `op` for these shapes (0 if none). Arguments an
 * op does not use are ignored. Returns (size_t)-1 for invalid shapes. */
size_t sk_workspace_bytes(int op, int B, int Hq, int Hkv, int Ncap, int N, int d, int L, int P,
                          int k);

/* Synchronises `stream`, then reports and clears the library's device error
 * word: SK_ERR_TIMEOUT if a device-side bounded wait of an earlier kernel gave
 * up, SK_ERR_UNSUPPORTED if a kernel found its shared-memory plan did not fit
 * (it then wrote nothing); SK_ERR_CUDA on a pending CUDA error; else SK_OK. */
int sk_check_status(void* stream);

/* Profiling hook: while `device_buffer` is non-NULL, every selection kernel
 * launch (socket_decode, socket_select, hata_decode) writes, per CTA, the SM
 * clock (clock64) at each phase to device_buffer[cta * 24 + phase] (phases
 * such as start, tables built, scores done, histogram, candidates, indices
 * written, exit) and the global timer (ns) at start and exit to slots 22 and
 * 23. The attention kernel of those calls and of socket_sparse_attend
 * stamps its CTAs (pair-major within each split) from entry 16 * B * Hkv * 24
 * on. The buffer must hold 24 entries per CTA: 16 * B * Hkv for the
 * selection plus B * Hkv * splits (at most 128 splits) for the attention.
 * Pass NULL to turn it off. One store per phase per CTA. */
int sk_profile_phases(unsigned long long* device_buffer);

/*
 * Test hook, not for production use: sets the limit, in SM clocks, of the
 * main-loop waits of the tensor-core hashing kernel (socket_hash_keys /
 * hata_hash_keys on bf16 keys with P = 8; cycles <= 0 restores the default of
 * about one second). With a tiny limit its waits give up while its copies and
 * MMAs are still in flight, which exercises the failure path: the kernel
 * stops, waits (with the default limit) for everything it issued, frees its
 * tensor memory and returns; the next sk_check_status reports
 * SK_ERR_TIMEOUT. Affects every later call on the current device until reset.
 */
int sk_test_set_wait_limit(long long cycles);

/* Thread-local description of the last non-OK return (never NULL). */
const char* sk_last_error(void);

/* Library version string. */
const char* sk_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HASH_SCORED_TOP_H */
