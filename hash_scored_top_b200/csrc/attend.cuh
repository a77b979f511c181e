// Exact attention over a list of selected keys, SOCKET step 4 (SOCKET
// technical summary, section 中核メカニズム：ソフト LSH, step 4: exact
// attention on the selected subset), for the G query heads of one KV head.
//
// bf16 K/V, one warp per 16-key tile:
//   * the warp's lanes issue one 1-D bulk copy (TMA engine) per selected K or
//     V row into the warp's shared-memory slot (rows padded to 2D + 16 bytes,
//     which makes the ldmatrix reads below conflict-free) and wait on the
//     slot's mbarrier (bounded wait);
//   * tensor cores (mma.sync m16n8k16, bf16 in, f32 accumulate) with the keys
//     on the M side:  S^T[16 keys x 8 head slots] = K_tile . Q^T and
//     O^T[d x 8 slots] += V_tile^T . P^T; K and Q^T fragments come from
//     ldmatrix, V^T fragments from ldmatrix.trans, and P^T moves from the
//     accumulator layout to the operand layout with movmatrix.trans;
//   * P is split as P_hi + P_lo (both bf16) so the PV product carries ~16
//     mantissa bits of P: for G <= 4 the lo parts ride in head slots 4..7 of
//     the same MMA, for 5 <= G <= 8 a second MMA adds them.
// Softmax: per head a running max m and sum l in the log2 domain (logits are
// pre-multiplied by scale * log2(e)).
//
// f32 K/V: a SIMT path, one head per warp (lanes over the head dim).
#pragma once

#include "common.cuh"

namespace hst {

constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& a0, uint32_t& a1, uint32_t& a2, uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& b0, uint32_t& b1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(b0), "=r"(b1) : "r"(addr));
}

// Padded row stride of K/V/Q rows in shared memory (bytes).
template <int D>
__host__ __device__ constexpr int kv_row_bytes() { return 2 * D + 16; }
// One warp slot: 16 K rows then 16 V rows.
template <int D>
__host__ __device__ constexpr int kv_slot_bytes() { return 32 * kv_row_bytes<D>(); }
// Q^T staging: 8 head rows.
template <int D>
__host__ __device__ constexpr int q_stage_bytes() { return 8 * kv_row_bytes<D>(); }

// Copies the group's bf16 query rows into padded rows at `qs` (rows >= G zero).
// All threads of the block; the caller synchronises afterwards.
template <int D>
__device__ __forceinline__ void stage_q(const __nv_bfloat16* __restrict__ Qg, int G, unsigned char* qs) {
  constexpr int RS = kv_row_bytes<D>();
  for (int e = threadIdx.x; e < 8 * (D / 8); e += blockDim.x) {
    const int h = e / (D / 8), c8 = e % (D / 8);
    const uint4 v = h < G ? *reinterpret_cast<const uint4*>(Qg + (size_t)h * D + 8 * c8) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(qs + h * RS + 16 * c8) = v;
  }
}

// Per-warp running state for the G head slots of this lane (2 per lane).
template <int D>
struct MmaAttendState {
  float acc[D / 16][4];   // O^T fragments: rows dv = 16j + r (+8), columns = head slots 2c, 2c+1
  float m[2];
  float l[2];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < D / 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }
};

// Issues the bulk copies of one tile's K and V rows into a warp slot.
// keys(i) is the cache row of tile key i < nvalid; rows are clamped into
// [0, nrows). The tile's transaction bytes are armed on `mbar` first.
template <int D, typename KeyFn>
__device__ __forceinline__ void issue_tile_copies(uint32_t slot, uint32_t mbar, const __nv_bfloat16* __restrict__ Kp,
                                                  const __nv_bfloat16* __restrict__ Vp, KeyFn keys, int nvalid,
                                                  int nrows, int lane) {
  constexpr int RS = kv_row_bytes<D>();
  fence_proxy_async_shared();
  if (lane == 0) mbar_arrive_expect_tx(mbar, (uint32_t)nvalid * 2u * D * 2u);
  __syncwarp();
  const int i = lane & 15;
  if (i < nvalid) {
    const int row = min(max(keys(i), 0), nrows - 1);
    const __nv_bfloat16* src = (lane < 16 ? Kp : Vp) + (size_t)row * D;
    bulk_copy_g2s(slot + (lane < 16 ? 0u : 16u * RS) + (uint32_t)i * RS, src, 2u * D, mbar);
  }
}

// One 16-key step of attention for a warp, reading the tile from its slot.
template <int D>
__device__ __forceinline__ void mma_attend_slot(MmaAttendState<D>& st, uint32_t slot, uint32_t qs, int nvalid,
                                                float scale_log2, bool packed, int lane) {
  constexpr int RS = kv_row_bytes<D>();
  const int r = lane >> 2, c = lane & 3, mtx = lane >> 3, mrow = lane & 7;
  const uint32_t kslot = slot, vslot = slot + 16u * RS;
  // padding V rows hold stale data: zero them (their P is 0; keep 0 * v finite)
  if (nvalid < 16) {
    const int i = lane & 15;
    if (i >= nvalid && lane < 16) {
#pragma unroll
      for (int c8 = 0; c8 < D / 8; ++c8)
        asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(vslot + (uint32_t)i * RS + 16u * c8), "r"(0u)
                     : "memory");
    }
    __syncwarp();
  }
  // ---- S^T = K . Q^T
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < D / 16; ++q) {
    uint32_t a0, a1, a2, a3, b0, b1;
    ldsm_x4(kslot + (uint32_t)((mtx & 1) * 8 + mrow) * RS + (uint32_t)(16 * q + (mtx >> 1) * 8) * 2u, a0, a1, a2, a3);
    ldsm_x2(qs + (uint32_t)mrow * RS + (uint32_t)(16 * q + (mtx & 1) * 8) * 2u, b0, b1);
    mma_bf16_16816(s, a0, a1, a2, a3, b0, b1);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] *= scale_log2;
  if (packed) {                      // head slots 4..7 mirror heads 0..3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(FULL, s[i], 2);
      if (c >= 2) s[i] = o;
    }
  }
  if (r >= nvalid) { s[0] = -INFINITY; s[1] = -INFINITY; }
  if (r + 8 >= nvalid) { s[2] = -INFINITY; s[3] = -INFINITY; }

  // ---- online softmax per head slot (2 per lane)
  float p[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float mt = fmaxf(s[i], s[2 + i]);
    mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 4));
    mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
    mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
    const float m_new = fmaxf(st.m[i], mt);
    const bool any = m_new != -INFINITY;
    const float alpha = any ? exp2f(st.m[i] - m_new) : 1.f;
    p[i] = any ? exp2f(s[i] - m_new) : 0.f;
    p[2 + i] = any ? exp2f(s[2 + i] - m_new) : 0.f;
    st.l[i] = st.l[i] * alpha + (p[i] + p[2 + i]);
    st.m[i] = m_new;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      st.acc[j][i] *= alpha;
      st.acc[j][2 + i] *= alpha;
    }
  }

  // ---- P^T fragments (hi / lo split)
  uint32_t bh0, bh1, bl0 = 0, bl1 = 0;
  {
    float hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hi[i] = __bfloat162float(__float2bfloat16_rn(p[i]));
      lo[i] = p[i] - hi[i];
    }
    if (packed) {
      const bool use_lo = c >= 2;
      bh0 = movmatrix_trans(use_lo ? pack_bf16x2(lo[0], lo[1]) : pack_bf16x2(hi[0], hi[1]));
      bh1 = movmatrix_trans(use_lo ? pack_bf16x2(lo[2], lo[3]) : pack_bf16x2(hi[2], hi[3]));
    } else {
      bh0 = movmatrix_trans(pack_bf16x2(hi[0], hi[1]));
      bh1 = movmatrix_trans(pack_bf16x2(hi[2], hi[3]));
      bl0 = movmatrix_trans(pack_bf16x2(lo[0], lo[1]));
      bl1 = movmatrix_trans(pack_bf16x2(lo[2], lo[3]));
    }
  }

  // ---- O^T += V^T . P^T
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4_trans(vslot + (uint32_t)((mtx >> 1) * 8 + mrow) * RS + (uint32_t)(16 * j + (mtx & 1) * 8) * 2u, a0, a1, a2,
                  a3);
    mma_bf16_16816(st.acc[j], a0, a1, a2, a3, bh0, bh1);
    if (!packed) mma_bf16_16816(st.acc[j], a0, a1, a2, a3, bl0, bl1);
  }
}

// Per-warp partial results in shared memory, one slot per warp:
//   pm[w][h], pl[w][h] (max in log2 domain, sum), po[w][h][D] (unnormalised).
// Per-warp partial results (m[G], l[G], o[G][D]); warp w's lies at
// base + w * ws floats (inside that warp's own K/V slot, free once the warp
// has finished its keys).
struct PartialView {
  float* base;
  int ws;
  int G;
  int D;
  __device__ __forceinline__ float& m(int w, int h) const { return base[(size_t)w * ws + h]; }
  __device__ __forceinline__ float& l(int w, int h) const { return base[(size_t)w * ws + G + h]; }
  __device__ __forceinline__ float* o(int w, int h) const { return base + (size_t)w * ws + 2 * G + (size_t)h * D; }
};

// Floats of one warp's partial.
__host__ __device__ inline size_t partial_floats(int G, int D) { return (size_t)G * (D + 2); }

__device__ __forceinline__ PartialView partial_view(float* base, int ws, int G, int D) {
  PartialView pv;
  pv.base = base;
  pv.ws = ws;
  pv.G = G;
  pv.D = D;
  return pv;
}

// Writes a warp's MMA state into partial slot w (heads < G only).
template <int D>
__device__ __forceinline__ void store_mma_partial(MmaAttendState<D>& st, const PartialView& pv, int w, bool packed,
                                                  int lane) {
  const int r = lane >> 2, c = lane & 3;
  float l[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v = st.l[i];
    v += __shfl_xor_sync(FULL, v, 4);
    v += __shfl_xor_sync(FULL, v, 8);
    v += __shfl_xor_sync(FULL, v, 16);
    l[i] = v;
  }
  // packed: O(head) = hi column (lane c < 2) + lo column (lane c ^ 2)
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(FULL, st.acc[j][e], 2);
      if (packed) st.acc[j][e] += o;
    }
  }
  const int hbase = packed ? 2 * (c & 1) : 2 * c;
  const bool writer = packed ? (c < 2) : true;
  if (writer) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int h = hbase + i;
      if (h < pv.G) {
        if (r == 0) {
          pv.m(w, h) = st.m[i];
          pv.l(w, h) = l[i];
        }
        float* po = pv.o(w, h);
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          po[16 * j + r] = st.acc[j][i];
          po[16 * j + r + 8] = st.acc[j][2 + i];
        }
      }
    }
  }
}

// Marks partial slot w as empty (no keys) for every head.
__device__ __forceinline__ void store_empty_partial(const PartialView& pv, int w, int lane) {
  for (int h = lane; h < pv.G; h += 32) {
    pv.m(w, h) = -INFINITY;
    pv.l(w, h) = 0.f;
  }
}

// bf16 attention of `cnt` listed keys by warps 0..ncw-1. Warp w takes the
// 16-key tiles w, w + ncw, ... and cycles through its NBUF slots (slot
// w * NBUF + s at slot0 + (w * NBUF + s) * slot_stride, mbarrier
// mbar0 + 8 (w * NBUF + s), phase bit in phases[w * NBUF + s]): the copies of
// the next NBUF - 1 tiles are in flight while a tile is computed. Results go
// to partial slots 0..ncw-1. Other warps do nothing.
template <int D, int NBUF, typename KeyFn>
__device__ void attend_tiles_bf16(const __nv_bfloat16* __restrict__ Kp, const __nv_bfloat16* __restrict__ Vp,
                                  KeyFn keys, int cnt, int nrows, int G, float scale, uint32_t qs, uint32_t slot0,
                                  uint32_t slot_stride, uint32_t mbar0, uint32_t* phases, int ncw,
                                  const PartialView& pv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp >= ncw) return;
  const bool packed = G <= 4;
  const float scale_log2 = scale * LOG2E;
  MmaAttendState<D> st;
  st.init();
  const int ntiles = (cnt + 15) / 16;
  const int nt = ntiles > warp ? (ntiles - warp + ncw - 1) / ncw : 0;   // this warp's tiles
  uint32_t ph = 0;                          // bit s: phase of slot s
#pragma unroll
  for (int s = 0; s < NBUF; ++s) ph |= (phases[warp * NBUF + s] & 1u) << s;
  auto slot_of = [&](int s) { return slot0 + (uint32_t)(warp * NBUF + s) * slot_stride; };
  auto mbar_of = [&](int s) { return mbar0 + 8u * (uint32_t)(warp * NBUF + s); };
  auto issue = [&](int j) {
    const int t = warp + j * ncw;
    const int nvalid = min(16, cnt - 16 * t);
    issue_tile_copies<D>(slot_of(j % NBUF), mbar_of(j % NBUF), Kp, Vp, [&](int i) { return keys(16 * t + i); },
                         nvalid, nrows, lane);
  };
  for (int j = 0; j < NBUF && j < nt; ++j) issue(j);
  bool ok = true;
  int j = 0;
  for (; j < nt && ok; ++j) {
    const int s = j % NBUF;
    ok = mbar_wait_bounded(mbar_of(s), (ph >> s) & 1u);
    ph ^= 1u << s;
    if (ok) {
      const int t = warp + j * ncw;
      mma_attend_slot<D>(st, slot_of(s), qs, min(16, cnt - 16 * t), scale_log2, packed, lane);
    }
    __syncwarp();
    if (ok && j + NBUF < nt) issue(j + NBUF);
  }
  if (!ok) {
    // a copy never completed: wait once more (bounded) for it and for the
    // tiles issued after it, so that none is left in flight
    const int jf = j - 1;
    mbar_wait_bounded(mbar_of(jf % NBUF), ((ph >> (jf % NBUF)) & 1u) ^ 1u);
    for (int jj = jf + 1; jj < jf + NBUF && jj < nt; ++jj) {
      mbar_wait_bounded(mbar_of(jj % NBUF), (ph >> (jj % NBUF)) & 1u);
      ph ^= 1u << (jj % NBUF);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < NBUF; ++s) phases[warp * NBUF + s] = (ph >> s) & 1u;
  }
  store_mma_partial<D>(st, pv, warp, packed, lane);
}

// f32 attention: warp w handles head w % G for the keys j = w / G, w / G + nwg, ...
// (nwg = ncw / G warps per head). Direct loads, lanes over the head dim.
template <int D, typename KeyFn>
__device__ void attend_keys_f32(const float* __restrict__ Qg, const float* __restrict__ Kp,
                                const float* __restrict__ Vp, KeyFn keys, int cnt, int nrows, int G, float scale,
                                int ncw, const PartialView& pv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp >= ncw) return;
  const int nwg = max(1, ncw / G);
  if (warp >= nwg * G) {
    store_empty_partial(pv, warp, lane);
    return;
  }
  const int h = warp % G;
  const float scale_log2 = scale * LOG2E;
  float q[D / 32], acc[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    q[i] = Qg[h * D + lane + 32 * i] * scale_log2;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = warp / G; j < cnt; j += nwg) {
    const int row = min(max(keys(j), 0), nrows - 1);
    const float* kr = Kp + (size_t)row * D;
    const float* vr = Vp + (size_t)row * D;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) s = fmaf(q[i], kr[lane + 32 * i], s);
    s = warp_sum(s);
    const float m_new = fmaxf(m, s);
    const float alpha = exp2f(m - m_new);
    const float pr = exp2f(s - m_new);
    l = l * alpha + pr;
    m = m_new;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) acc[i] = acc[i] * alpha + pr * vr[lane + 32 * i];
  }
  for (int hh = 0; hh < G; ++hh) {
    if (lane == 0) {
      pv.m(warp, hh) = hh == h ? m : -INFINITY;
      pv.l(warp, hh) = hh == h ? l : 0.f;
    }
  }
  float* po = pv.o(warp, h);
#pragma unroll
  for (int i = 0; i < D / 32; ++i) po[lane + 32 * i] = acc[i];
}

// Merges nslots partial slots into (M[h], Lsum[h], O[h][D]) with a fixed
// slot order; all threads of the block participate. Slots with m = -inf
// contribute nothing.
__device__ __forceinline__ void merge_partials(const PartialView& pv, int nslots, float* M, float* Lsum, float* O) {
  const int G = pv.G, D = pv.D;
  for (int h = threadIdx.x; h < G; h += blockDim.x) {
    float mm = -INFINITY;
    for (int w = 0; w < nslots; ++w) mm = fmaxf(mm, pv.m(w, h));
    float ls = 0.f;
    for (int w = 0; w < nslots; ++w) {
      const float pm = pv.m(w, h);
      if (pm != -INFINITY) ls += exp2f(pm - mm) * pv.l(w, h);
    }
    M[h] = mm;
    Lsum[h] = ls;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
    const int h = e / D;
    const float mm = M[h];
    float o = 0.f;
    for (int w = 0; w < nslots; ++w) {
      const float pm = pv.m(w, h);
      if (pm != -INFINITY) o += exp2f(pm - mm) * pv.o(w, h)[e % D];
    }
    O[e] = o;
  }
  __syncthreads();
}

}  // namespace hst
