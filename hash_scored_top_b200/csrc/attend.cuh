// Exact attention over a list of selected keys, SOCKET step 4 (SOCKET
// technical summary, section 中核メカニズム：ソフト LSH, step 4: exact
// attention on the selected subset), for the G query heads of one KV head.
//
// bf16 K/V: one warp processes 16 keys per step on the tensor cores
// (mma.sync m16n8k16, bf16 in, f32 accumulate), with the keys on the M side:
//   S^T[16 keys x 8 head slots] = K_tile[16 x d] . Q^T[d x 8]
//   O^T[d x 8 slots]           += V_tile^T[d x 16] . P^T[16 x 8]
// Each lane loads its operands straight from global memory with 16-byte
// loads: the contraction index of each product (head dim for QK, key for
// PV) is permuted consistently on both operands, so every fragment register
// is a contiguous 4-byte piece of a loaded 16-byte chunk (no shared memory,
// no ldmatrix). P^T is moved from the accumulator layout to the B-operand
// layout with movmatrix.trans. The probabilities are split P = P_hi + P_lo
// (both bf16) so the PV product carries ~16 mantissa bits of P: for G <= 4
// the lo parts ride in the unused head slots 4..7 of the same MMA; for
// 5 <= G <= 8 a second MMA adds them.
//
// f32 K/V: a plain SIMT path (lanes over the head dim), used for small
// fp32 caches.
//
// Softmax: per head, running max m and sum l in the log2 domain (logits are
// pre-multiplied by scale * log2(e)); exp2 of non-positive arguments only.
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

__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}

// Per-warp partial result of attention over a subset: for head slot i of this
// lane, running max m (log2 domain), lane-partial sum l, and the unnormalised
// output fragment acc.
template <int D>
struct MmaAttendState {
  float acc[D / 16][4];
  float m[2];
  float l[2];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < D / 16; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }
};

// Q^T fragments of a lane: qb[q][e] packs Q[head r][32q + 8c + 2e .. +1], zero
// for head slots >= G. Q is bf16 [G][D] (row stride D).
template <int D>
__device__ __forceinline__ void load_q_frag(uint32_t (&qb)[D / 32][4], const __nv_bfloat16* __restrict__ Qg,
                                            int G, int lane) {
  const int r = lane >> 2, c = lane & 3;
#pragma unroll
  for (int q = 0; q < D / 32; ++q) {
    if (r < G) {
      const uint4 v = *reinterpret_cast<const uint4*>(Qg + (size_t)r * D + 32 * q + 8 * c);
      qb[q][0] = v.x; qb[q][1] = v.y; qb[q][2] = v.z; qb[q][3] = v.w;
    } else {
      qb[q][0] = qb[q][1] = qb[q][2] = qb[q][3] = 0u;
    }
  }
}

// Row loads of one 16-key tile for this lane.
template <int D>
struct KVTile {
  uint4 k[2][D / 32];     // key rows r and r+8: chunk q covers dims 32q + 8c .. +8
  uint4 v[4][D / 64];     // value rows 2c, 2c+1, 2c+8, 2c+9: half covers dims 64*half + 8r .. +8
  bool kvalid[2];
  bool vvalid[4];
};

// keys(i) gives the cache row of tile key i (0..15); nvalid of them are real,
// the rest are padding (loaded from row keys(0), then masked). Rows are
// clamped into [0, nrows) so a bad index can never read outside the cache.
template <int D, typename KeyFn>
__device__ __forceinline__ void load_kv_tile(KVTile<D>& t, const __nv_bfloat16* __restrict__ Kp,
                                             const __nv_bfloat16* __restrict__ Vp, KeyFn keys, int nvalid,
                                             int nrows, int lane) {
  const int r = lane >> 2, c = lane & 3;
  auto clamp_row = [&](int x) { return min(max(x, 0), nrows - 1); };
  const int row0 = clamp_row(keys(0));
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int i = r + 8 * s;
    t.kvalid[s] = i < nvalid;
    const int row = t.kvalid[s] ? clamp_row(keys(i)) : row0;
    const __nv_bfloat16* base = Kp + (size_t)row * D + 8 * c;
#pragma unroll
    for (int q = 0; q < D / 32; ++q) t.k[s][q] = ldg_stream(base + 32 * q);
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int i = 2 * c + (s & 1) + 8 * (s >> 1);
    t.vvalid[s] = i < nvalid;
    const int row = t.vvalid[s] ? clamp_row(keys(i)) : row0;
    const __nv_bfloat16* base = Vp + (size_t)row * D + 8 * r;
#pragma unroll
    for (int h = 0; h < D / 64; ++h) t.v[s][h] = ldg_stream(base + 64 * h);
  }
}

// One 16-key step of attention for a warp. `packed` selects the G <= 4 mode.
template <int D>
__device__ __forceinline__ void mma_attend_tile(MmaAttendState<D>& st, KVTile<D>& t,
                                                const uint32_t (&qb)[D / 32][4], float scale_log2,
                                                bool packed, int lane) {
  const int c = lane & 3;
  // ---- S^T = K . Q^T
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < D / 32; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mma_bf16_16816(s, u4get(t.k[0][q], 2 * h), u4get(t.k[1][q], 2 * h), u4get(t.k[0][q], 2 * h + 1),
                     u4get(t.k[1][q], 2 * h + 1), qb[q][2 * h], qb[q][2 * h + 1]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) s[i] *= scale_log2;
  if (packed) {                      // slots 4..7 mirror heads 0..3
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(FULL, s[i], 2);
      if (c >= 2) s[i] = o;
    }
  }
  if (!t.kvalid[0]) { s[0] = -INFINITY; s[1] = -INFINITY; }
  if (!t.kvalid[1]) { s[2] = -INFINITY; s[3] = -INFINITY; }

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

  // ---- O^T += V^T . P^T  (padding value rows are zeroed)
#pragma unroll
  for (int s2 = 0; s2 < 4; ++s2) {
    if (!t.vvalid[s2]) {
#pragma unroll
      for (int h = 0; h < D / 64; ++h) t.v[s2][h] = make_uint4(0, 0, 0, 0);
    }
  }
#pragma unroll
  for (int j = 0; j < D / 16; ++j) {
    const int h = j >> 2, e = j & 3;
    const uint32_t x0 = u4get(t.v[0][h], e), x1 = u4get(t.v[1][h], e);
    const uint32_t x2 = u4get(t.v[2][h], e), x3 = u4get(t.v[3][h], e);
    const uint32_t a0 = __byte_perm(x0, x1, 0x5410), a1 = __byte_perm(x0, x1, 0x7632);
    const uint32_t a2 = __byte_perm(x2, x3, 0x5410), a3 = __byte_perm(x2, x3, 0x7632);
    mma_bf16_16816(st.acc[j], a0, a1, a2, a3, bh0, bh1);
    if (!packed) mma_bf16_16816(st.acc[j], a0, a1, a2, a3, bl0, bl1);
  }
}

// Per-warp partial results in shared memory, one slot per warp:
//   pm[w][h], pl[w][h] (max in log2 domain, sum), po[w][h][D] (unnormalised).
struct PartialView {
  float* pm;
  float* pl;
  float* po;
  int G;
  int D;
};

// Writes a warp's MMA state into partial slot w (heads < G only).
template <int D>
__device__ __forceinline__ void store_mma_partial(MmaAttendState<D>& st, const PartialView& pv, int w,
                                                  bool packed, int lane) {
  const int r = lane >> 2, c = lane & 3;
  // total l over the 8 key lanes
  float l[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v = st.l[i];
    v += __shfl_xor_sync(FULL, v, 4);
    v += __shfl_xor_sync(FULL, v, 8);
    v += __shfl_xor_sync(FULL, v, 16);
    l[i] = v;
  }
  // packed: O(head) = hi column (lane c<2) + lo column (lane c^2)
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
          pv.pm[w * pv.G + h] = st.m[i];
          pv.pl[w * pv.G + h] = l[i];
        }
        float* po = pv.po + ((size_t)w * pv.G + h) * D;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
          const int dv = 64 * (j >> 2) + 8 * r + 2 * (j & 3);
          po[dv] = st.acc[j][i];
          po[dv + 1] = st.acc[j][2 + i];
        }
      }
    }
  }
}

// ---------------------------------------------------------------- f32 SIMT path
template <int D>
struct SimtAttendState {
  float acc[8][D / 32];   // head slot, dims lane + 32*i
  float m[8];
  float l[8];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) acc[h][i] = 0.f;
    }
  }
};

// One key for all G (<= 8) heads; q[h][i] holds Q[h][lane + 32 i] * scale_log2.
template <int D>
__device__ __forceinline__ void simt_attend_key(SimtAttendState<D>& st, const float* __restrict__ krow,
                                                const float* __restrict__ vrow, const float (&q)[8][D / 32], int G,
                                                int lane) {
  float kv[D / 32], vv[D / 32];
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    kv[i] = krow[lane + 32 * i];
    vv[i] = vrow[lane + 32 * i];
  }
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < G) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) s = fmaf(q[h][i], kv[i], s);
      s = warp_sum(s);
      const float m_new = fmaxf(st.m[h], s);
      const float alpha = exp2f(st.m[h] - m_new);
      const float p = exp2f(s - m_new);
      st.l[h] = st.l[h] * alpha + p;
      st.m[h] = m_new;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) st.acc[h][i] = st.acc[h][i] * alpha + p * vv[i];
    }
  }
}

template <int D>
__device__ __forceinline__ void store_simt_partial(const SimtAttendState<D>& st, const PartialView& pv, int w,
                                                   int lane) {
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    if (h < pv.G) {
      if (lane == 0) {
        pv.pm[w * pv.G + h] = st.m[h];
        pv.pl[w * pv.G + h] = st.l[h];
      }
      float* po = pv.po + ((size_t)w * pv.G + h) * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) po[lane + 32 * i] = st.acc[h][i];
    }
  }
}

// Merges nslots partial slots into (M[h], Lsum[h], O[h][D]) with a fixed
// slot order; all threads of the block participate. Slot results with no
// keys have m = -inf and contribute nothing.
__device__ __forceinline__ void merge_partials(const PartialView& pv, int nslots, float* M, float* Lsum,
                                               float* O) {
  const int G = pv.G, D = pv.D;
  for (int h = threadIdx.x; h < G; h += blockDim.x) {
    float mm = -INFINITY;
    for (int w = 0; w < nslots; ++w) mm = fmaxf(mm, pv.pm[w * G + h]);
    float ls = 0.f;
    for (int w = 0; w < nslots; ++w) {
      const float pm = pv.pm[w * G + h];
      if (pm != -INFINITY) ls += exp2f(pm - mm) * pv.pl[w * G + h];
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
      const float pm = pv.pm[w * G + h];
      if (pm != -INFINITY) o += exp2f(pm - mm) * pv.po[((size_t)w * G + h) * D + (e % D)];
    }
    O[e] = o;
  }
  __syncthreads();
}

}  // namespace hst
