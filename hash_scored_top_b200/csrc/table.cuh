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

// Number of float64 scratch words build_bucket_table needs.
__host__ __device__ inline int table_scratch_doubles(int G, int d, int n_my_tables, int P) {
  const int plo = P / 2, phi = P - plo;
  return G * d + G * n_my_tables * P * 2 + G * n_my_tables * ((1 << plo) + (1 << phi));
}

__device__ __forceinline__ double load_q(const float* q, int i) { return (double)q[i]; }
__device__ __forceinline__ double load_q(const __nv_bfloat16* q, int i) {
  return (double)__bfloat162float(q[i]);
}

// Computes T_l(b) for the tables l = l_first + t * l_step (t = 0, 1, ...) < L
// and every bucket b < 2^P, calling store(b, l, value_f32) once per entry.
// Qg points at the G query rows of the pair (row stride d). All threads of
// the block must call this; it ends with __syncthreads().
template <typename QT, typename Store>
__device__ void build_bucket_table(const QT* __restrict__ Qg, int G, int d,
                                   const __nv_bfloat16* __restrict__ R, int L, int P, float tau,
                                   int l_first, int l_step, double* scratch, Store store) {
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int nl = (L - l_first + l_step - 1) / l_step;   // tables handled here
  const int plo = P / 2, phi = P - plo;
  const int nlo = 1 << plo, nhi = 1 << phi;
  double* qhat = scratch;                               // [G][d]
  double* sig = qhat + G * d;                           // [G][nl][P][2]: P(bit=0), P(bit=1)
  double* lo = sig + G * nl * P * 2;                    // [G][nl][nlo]
  double* hi = lo + G * nl * nlo;                       // [G][nl][nhi]

  // 1. unit query rows (one warp per head)
  const int warp = tid >> 5, lane = tid & 31, nwarps = nthr >> 5;
  for (int h = warp; h < G; h += nwarps) {
    double ss = 0.0;
    for (int c = lane; c < d; c += 32) {
      const double x = load_q(Qg + (size_t)h * d, c);
      ss = fma(x, x, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    const double nrm = sqrt(ss);
    for (int c = lane; c < d; c += 32) qhat[h * d + c] = load_q(Qg + (size_t)h * d, c) / nrm;
  }
  __syncthreads();

  // 2. projections z and the per-bit factors sigmoid(+-2z/tau)
  const double two_over_tau = 2.0 / (double)tau;
  for (int item = tid; item < G * nl * P; item += nthr) {
    const int j = item % P;
    const int li = (item / P) % nl;
    const int h = item / (P * nl);
    const int l = l_first + li * l_step;
    const uint4* rrow = reinterpret_cast<const uint4*>(R + (size_t)(l * P + j) * d);
    const double* qh = qhat + h * d;
    double z = 0.0;
    for (int c8 = 0; c8 < d / 8; ++c8) {
      const uint4 w = __ldg(rrow + c8);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        z = fma(qh[c8 * 8 + 2 * e], (double)bf16lo_to_f32(ws[e]), z);
        z = fma(qh[c8 * 8 + 2 * e + 1], (double)bf16hi_to_f32(ws[e]), z);
      }
    }
    const double x = two_over_tau * z;                  // logit gap between bit=1 and bit=0
    const double e = exp(-fabs(x));
    const double p_big = 1.0 / (1.0 + e);               // sigmoid(|x|)
    const double p_small = e / (1.0 + e);               // sigmoid(-|x|)
    sig[item * 2 + 1] = x >= 0.0 ? p_big : p_small;     // bit j = 1
    sig[item * 2 + 0] = x >= 0.0 ? p_small : p_big;     // bit j = 0
  }
  __syncthreads();

  // 3. products over the low / high bits
  for (int item = tid; item < G * nl * (nlo + nhi); item += nthr) {
    const int m = item % (nlo + nhi);
    const int hl = item / (nlo + nhi);                  // h * nl + li
    const double* s = sig + (size_t)hl * P * 2;
    double prod = 1.0;
    if (m < nlo) {
      for (int j = 0; j < plo; ++j) prod *= s[j * 2 + ((m >> j) & 1)];
      lo[hl * nlo + m] = prod;
    } else {
      const int mh = m - nlo;
      for (int j = 0; j < phi; ++j) prod *= s[(plo + j) * 2 + ((mh >> j) & 1)];
      hi[hl * nhi + mh] = prod;
    }
  }
  __syncthreads();

  // 4. table entries, summed over the group's heads
  const int nb = 1 << P;
  for (int item = tid; item < nb * nl; item += nthr) {
    const int li = item % nl;
    const int b = item / nl;
    double t = 0.0;
    for (int h = 0; h < G; ++h) {
      const int hl = h * nl + li;
      t = fma(lo[hl * nlo + (b & (nlo - 1))], hi[hl * nhi + (b >> plo)], t);
    }
    store(b, l_first + li * l_step, (float)t);
  }
  __syncthreads();
}

}  // namespace hst
