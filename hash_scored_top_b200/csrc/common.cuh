// Shared device utilities for the hash-scored top-k decode kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace hst {

constexpr unsigned FULL = 0xffffffffu;

// ---------------------------------------------------------------- error word
// Set by a kernel that has to give up (a bounded wait that ran out, a
// shared-memory plan that does not fit) -- never by a trap. Read and cleared by
// sk_check_status on the host. The library is a single translation unit.
__device__ unsigned int g_error_word = 0u;
constexpr unsigned ERR_TIMEOUT = 1u;   // a bounded wait gave up
constexpr unsigned ERR_LAYOUT = 2u;    // a launch's shared-memory plan did not fit
constexpr unsigned ERR_RANGE = 4u;     // a page-table entry outside the pool (read as page 0)

// ---------------------------------------------------------------- bucket-ID cache layout
// Each key stores its L bucket IDs in LP bytes, split in chunks of S_0, S_1
// tables: L <= 16 -> [16]; L <= 32 -> [32]; L <= 48 -> [32, 16]; L <= 64 ->
// [32, 32]. Inside chunk c (tables 32c ..), byte j of key n holds the ID of
// table 32c + (j + n) mod S_c, zero where that table is >= L. A warp scoring
// 32 consecutive keys then reads, at step j, 32 different tables -- one per
// lane -- which is what makes its shared-memory lookups conflict-free.
__host__ __device__ constexpr int ids_bytes_per_key(int L) {
  return L <= 16 ? 16 : L <= 32 ? 32 : L <= 48 ? 48 : 64;
}
__host__ __device__ constexpr int id_chunk_size(int L, int chunk) {
  return chunk == 0 ? (L <= 16 ? 16 : 32) : (L <= 48 ? 16 : 32);
}
// Byte position of table l's ID inside the bytes of key n.
__host__ __device__ inline int id_byte_pos(int L, int l, int n) {
  const int c = l >= 32 ? 1 : 0;
  const int S = id_chunk_size(L, c);
  return 32 * c + (((l - 32 * c - n) % S) + S) % S;
}
// Table whose ID sits at byte b of key n (>= L: padding).
__host__ __device__ inline int id_byte_table(int L, int b, int n) {
  const int c = b >= 32 ? 1 : 0;
  const int S = id_chunk_size(L, c);
  return 32 * c + ((b - 32 * c) + n) % S;
}

// ---------------------------------------------------------------- loads
// Asks the TMA unit to bring [p, p + bytes) into L2 (no completion to wait
// for). p and bytes must be multiples of 16.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 32 bytes in one request (sm_100 256-bit load); p must be 32-byte aligned.
__device__ __forceinline__ void ldg_stream32(const void* p, uint4& lo, uint4& hi) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
               : "l"(p));
}

__device__ __forceinline__ uint16_t ldg_u16(const void* p) {
  unsigned short r;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

// Full cluster barrier with release/acquire semantics (shared and global
// writes before it are visible to every thread of the cluster after it).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" :: "r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_v4f32(uint32_t addr, const float* v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(v[0]), "f"(v[1]), "f"(v[2]),
               "f"(v[3]) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ---------------------------------------------------------------- mbarriers and bulk copies
__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}

// Makes mbarrier initialisations visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier shared-memory accesses (generic proxy) before
// later bulk copies into the same memory (async proxy).
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking: whether the phase with the given parity has completed.
__device__ __forceinline__ bool mbar_test_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most `limit`
// SM clocks (by default about one second); on giving up sets ERR_TIMEOUT and
// returns false.
constexpr long long kWaitLimit = 2000000000LL;
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t addr, uint32_t parity, long long limit = kWaitLimit) {
  if (limit < kWaitLimit) {
    // a lowered limit (test hook only): the blocking try_wait below may itself
    // wait longer than the limit, so test once without blocking, then poll
    if (mbar_test_wait(addr, parity)) return true;
    const long long t0 = clock64();
    while (clock64() - t0 <= limit)
      if (mbar_test_wait(addr, parity)) return true;
    atomicOr(&g_error_word, ERR_TIMEOUT);
    return false;
  }
  if (mbar_try_wait(addr, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(addr, parity)) {
    if (clock64() - t0 > limit) {
      atomicOr(&g_error_word, ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// 1-D bulk copy (TMA engine) global -> this CTA's shared memory, completing
// `bytes` of transaction count on the mbarrier. Both addresses 16-byte
// aligned, bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t mbar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(mbar)
               : "memory");
}

// ---------------------------------------------------------------- bf16 pairs
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace hst
