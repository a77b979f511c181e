// Soft bucket table, SOCKET step 2 (SOCKET technical summary, section
// 中核メカニズム：ソフト LSH, step 2: the query's projections onto the
// random hyperplanes go through a temperature softmax over all buckets).
//
// For one (batch, KV-head) pair with query heads h = 0..G-1:
//   q_hat_h = q_h / |q_h|,   z_{h,l,j} = q_hat_h . r_{l*P+j},
//   p_{h,l}(b) = softmax_b( sum_j s_bj z_{h,l,j} / tau ),  s_bj = +-1 by bit j of b,
//   T_l(b) = sum_h p_{h,l}(b).
// The softmax over the 2^P sign patterns factorises over the bits:
//   p_{h,l}(b) = prod_j sigmoid(2 s_bj z_{h,l,j} / tau),
// which is evaluated as lo[b & (2^Plo - 1)] * hi[b >> Plo] with lo/hi the
// products over the low Plo and high P - Plo bits. Everything up to the final
// entry is float64 (the projections decide scores that are compared at 1e-6
// relative, so an f32 projection is not accurate enough); the entry is then
// rounded once to float32.
#pragma once

#include "common.cuh"

namespace hst {

// Bytes of shared scratch build_bucket_table needs for nl tables: float64
// words for the unit queries, bit factors and lo/hi products (the "double"
// part), then the staged bf16 hyperplane rows (the "rows" part). The rows may
// go to a separate buffer (rows_scratch); otherwise they follow the doubles.
__host__ __device__ inline size_t table_scratch_dbl_bytes(int G, int d, int nl, int P) {
  const int plo = P / 2, phi = P - plo;
  size_t dbl = (size_t)G * (d + 8) + (size_t)G * nl * P * 2 + (size_t)G * nl * ((1 << plo) + (1 << phi) + 2);
  dbl = (dbl + 1) & ~(size_t)1;                         // keep the bf16 rows 16-byte aligned
  return dbl * 8;
}
__host__ __device__ inline size_t table_scratch_rows_bytes(int d, int nl, int P) { return (size_t)nl * P * d * 2; }
__host__ __device__ inline size_t table_scratch_bytes(int G, int d, int nl, int P) {
  return table_scratch_dbl_bytes(G, d, nl, P) + table_scratch_rows_bytes(d, nl, P);
}

__device__ __forceinline__ double load_q(const float* q, int i) { return (double)q[i]; }
__device__ __forceinline__ double load_q(const __nv_bfloat16* q, int i) {
  return (double)__bfloat162float(q[i]);
}

// Unit query rows are stored with each of the 8 segments of D / 8 values
// followed by one padding word, so the 8 lanes that read the 8 segments hit
// different banks.
template <int D>
__host__ __device__ constexpr int qpad_row() { return D + 8; }
template <int D>
__device__ __forceinline__ int qpad_index(int h, int c) {
  return h * qpad_row<D>() + (c / (D / 8)) * (D / 8 + 1) + c % (D / 8);
}

// Projections z(h, mi) = qhat_h . r_mi on the fp64 tensor cores (mma
// m8n8k4, f64 in and out): warp w computes 8x8 tiles for 8 heads and 8
// hyperplane rows, accumulating over the head dimension in steps of 4 in a
// fixed order, so every element's value depends only on its inputs. qhat: G
// padded rows (qpad_index); rs: [nrows][D] bf16 rows. Calls out(item, z) once
// per item h * nrows + mi (h < G, mi < nrows).
__device__ __forceinline__ void mma_f64_m8n8k4(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d0), "+d"(d1) : "d"(a), "d"(b));
}

template <int D, typename Out>
__device__ __forceinline__ void project_rows_mma(const double* qhat, int G, const __nv_bfloat16* rs, int nrows,
                                                 Out out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int mt = (G + 7) / 8, nt = (nrows + 7) / 8;
  const int r = lane >> 2, c = lane & 3;     // fragment row; column within the k step
  for (int task = warp; task < mt * nt; task += nw) {
    const int hb = (task / nt) * 8, nb = (task % nt) * 8;
    const int h = hb + r, n = nb + r;        // A row (head), B column (hyperplane row)
    const bool hv = h < G, nv = n < nrows;
    double d0 = 0.0, d1 = 0.0;
#pragma unroll 8
    for (int k0 = 0; k0 < D; k0 += 4) {
      const double a = hv ? qhat[qpad_index<D>(h, k0 + c)] : 0.0;
      const double b = nv ? (double)__bfloat162float(rs[n * D + k0 + c]) : 0.0;
      mma_f64_m8n8k4(d0, d1, a, b);
    }
    // accumulator: row r, columns 2c and 2c + 1 of the tile
    const int n0 = nb + 2 * c;
    if (hv && n0 < nrows) out(h * nrows + n0, d0);
    if (hv && n0 + 1 < nrows) out(h * nrows + n0 + 1, d1);
  }
}

// Unit query rows (one warp per head) into qhat (padded rows, qpad_index),
// float64. Each lane loads its D / 32 values once, then normalises them.
template <int D, typename QT>
__device__ __forceinline__ void unit_queries(const QT* __restrict__ Qg, int G, double* qhat) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int h = warp; h < G; h += nwarps) {
    double x[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) x[i] = load_q(Qg + (size_t)h * D, lane + 32 * i);
    double ss = 0.0;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) ss = fma(x[i], x[i], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    const double inv = 1.0 / sqrt(ss);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) qhat[qpad_index<D>(h, lane + 32 * i)] = x[i] * inv;
  }
}

// Copies hyperplane rows [row0, row0 + nrows) (bf16, D wide) to shared rs.
template <int D>
__device__ __forceinline__ void stage_rows(const __nv_bfloat16* __restrict__ R, int row0, int nrows,
                                           __nv_bfloat16* rs) {
  const uint4* src = reinterpret_cast<const uint4*>(R + (size_t)row0 * D);
  uint4* dst = reinterpret_cast<uint4*>(rs);
  for (int e = threadIdx.x; e < nrows * (D / 8); e += blockDim.x) dst[e] = __ldg(src + e);
}

struct NoHook {
  __device__ void operator()() const {}
};

// The per-bit factors of tables [l0, l0 + nl) for every head of the group,
// float64, left in scratch: p_{h,l0+li}(b) = lo[hl * slo + (b & (nlo - 1))] *
// hi[hl * shi + (b >> plo)] with hl = h * nl + li.
struct BucketFactors {
  const double* lo;
  const double* hi;
  int slo, shi, plo, nlo;
};

// Steps 1-3 of the table build (unit queries, projections on the fp64 tensor
// cores, per-bit sigmoids, products over the low and high bits). Same
// arguments as build_bucket_table; all threads of the block call it; it ends
// with __syncthreads().
// rows_global = true: the hyperplane rows are read from R in global memory
// (not staged), so scratch needs only table_scratch_dbl_bytes.
template <int D, typename QT>
__device__ BucketFactors bucket_factors(const QT* __restrict__ Qg, int G, const __nv_bfloat16* __restrict__ R, int P,
                                        float tau, int l0, int nl, void* scratch, unsigned long long* ts = nullptr,
                                        void* rows_scratch = nullptr, bool rows_global = false) {
  auto tstamp = [&](int ph) {
    if (ts != nullptr && threadIdx.x == 0) {
      ts[blockIdx.x * 24 + ph] = (unsigned long long)clock64();
    }
  };
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int plo = P / 2, phi = P - plo;
  const int nlo = 1 << plo, nhi = 1 << phi;
  // lo/hi rows are padded by one word (17 or 9 words) so that the lanes of a
  // warp, which read different rows, hit different banks
  const int slo = nlo + 1, shi = nhi + 1;
  double* qhat = reinterpret_cast<double*>(scratch);   // G padded rows
  double* sig = qhat + G * qpad_row<D>();               // [G][nl][P][2]: P(bit=0), P(bit=1)
  double* lo = sig + G * nl * P * 2;                    // [G][nl][slo]
  double* hi = lo + G * nl * slo;                       // [G][nl][shi]
  const int ndbl = (G * qpad_row<D>() + G * nl * P * 2 + G * nl * (slo + shi) + 1) & ~1;   // 16-byte aligned rows
  const __nv_bfloat16* rs = rows_global ? R + (size_t)l0 * P * D
                           : rows_scratch ? reinterpret_cast<const __nv_bfloat16*>(rows_scratch)   // [nl * P][D]
                                          : reinterpret_cast<const __nv_bfloat16*>(qhat + ndbl);

  // 1. unit query rows; this CTA's hyperplane rows
  unit_queries<D>(Qg, G, qhat);
  if (!rows_global) stage_rows<D>(R, l0 * P, nl * P, const_cast<__nv_bfloat16*>(rs));
  __syncthreads();
  tstamp(5);

  // 2. projections z and the per-bit factors sigmoid(+-2z/tau)
  const double two_over_tau = 2.0 / (double)tau;
  project_rows_mma<D>(qhat, G, rs, nl * P, [&](int item, double z) {
    const double x = two_over_tau * z;                  // logit gap between bit=1 and bit=0
    const double e = exp(-fabs(x));
    const double p_big = 1.0 / (1.0 + e);               // sigmoid(|x|)
    const double p_small = e * p_big;                   // sigmoid(-|x|)
    sig[item * 2 + 1] = x >= 0.0 ? p_big : p_small;     // bit j = 1
    sig[item * 2 + 0] = x >= 0.0 ? p_small : p_big;     // bit j = 0
  });
  __syncthreads();
  tstamp(6);

  // 3. products over the low / high bits
  for (int item = tid; item < G * nl * (nlo + nhi); item += nthr) {
    const int m = item % (nlo + nhi);
    const int hl = item / (nlo + nhi);                  // h * nl + li
    const double* sg = sig + (size_t)hl * P * 2;
    double prod = 1.0;
    if (m < nlo) {
      for (int j = 0; j < plo; ++j) prod *= sg[j * 2 + ((m >> j) & 1)];
      lo[hl * slo + m] = prod;
    } else {
      const int mh = m - nlo;
      for (int j = 0; j < phi; ++j) prod *= sg[(plo + j) * 2 + ((mh >> j) & 1)];
      hi[hl * shi + mh] = prod;
    }
  }
  __syncthreads();
  tstamp(13);
  return BucketFactors{lo, hi, slo, shi, plo, nlo};
}

// Computes T_l(b) for the tables l in [l0, l0 + nl) and every bucket b < 2^P.
// VEC = 1: calls store(b, l, value_f32) once per entry. VEC = 4: calls
// store(b, l, v, cnt) once per bucket and group of 4 tables l .. l + cnt - 1
// (groups start at l0 + 4g; cnt < 4 only for the last group), v[0..cnt).
// Qg points at the G query rows of the pair (row stride D); scratch holds
// table_scratch_bytes, or table_scratch_dbl_bytes when rows_scratch (16-byte
// aligned, table_scratch_rows_bytes) is given. All threads of the block must call this; it calls
// before_store() (all threads, converged) just before the first store and
// ends with __syncthreads().
template <int D, typename QT, typename Store, typename Hook = NoHook, int VEC = 1>
__device__ void build_bucket_table(const QT* __restrict__ Qg, int G, const __nv_bfloat16* __restrict__ R, int P,
                                   float tau, int l0, int nl, void* scratch, Store store,
                                   unsigned long long* ts = nullptr, Hook before_store = Hook(),
                                   void* rows_scratch = nullptr) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const BucketFactors bf = bucket_factors<D, QT>(Qg, G, R, P, tau, l0, nl, scratch, ts, rows_scratch);
  const double* lo = bf.lo;
  const double* hi = bf.hi;
  const int slo = bf.slo, shi = bf.shi, plo = bf.plo, nlo = bf.nlo;

  // 4. table entries, summed over the group's heads
  before_store();
  const int nb = 1 << P;
  if constexpr (VEC == 4) {
    const int ng = (nl + 3) / 4;
    for (int item = tid; item < nb * ng; item += nthr) {
      const int g = item % ng;
      const int b = item / ng;
      const int cnt = min(4, nl - 4 * g);
      float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q < cnt) {
          double t = 0.0;
          for (int h = 0; h < G; ++h) {
            const int hl = h * nl + 4 * g + q;
            t = fma(lo[hl * slo + (b & (nlo - 1))], hi[hl * shi + (b >> plo)], t);
          }
          v[q] = (float)t;
        }
      }
      store(b, l0 + 4 * g, v, cnt);
    }
  } else {
    for (int item = tid; item < nb * nl; item += nthr) {
      const int li = item % nl;
      const int b = item / nl;
      double t = 0.0;
      for (int h = 0; h < G; ++h) {
        const int hl = h * nl + li;
        t = fma(lo[hl * slo + (b & (nlo - 1))], hi[hl * shi + (b >> plo)], t);
      }
      store(b, l0 + li, (float)t);
    }
  }
  __syncthreads();
}

}  // namespace hst
