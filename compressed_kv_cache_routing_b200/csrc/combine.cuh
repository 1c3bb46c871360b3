// Merge of split-K attention partials and expansion through B_v (BasisKV:
// the attention result is a weighted latent; the per-KV-head basis B_v turns
// it into a value, "Value compression associated with the output
// projection").
//
// Partial j of query head h holds (m_j, l_j, acc_j[r]) with m_j a running
// max in log2 units, l_j = sum 2^(s - m_j), acc_j = sum 2^(s - m_j) Z_t.
// With M = max_j m_j:  l = sum_j l_j 2^(m_j - M),
//                      zbar = sum_j acc_j 2^(m_j - M) / l,
//                      out_h = zbar . B_v  (fp32, d wide).
// A head with no token at all (M = -inf) gets out = 0.
#pragma once

#include "common.cuh"

namespace basiskv {

struct CombineArgs {
  const float* part_ml;   // [NP][G][2] of this unit
  const float* part_acc;  // [NP][G][r] of this unit
  const float* b_v;       // [r][d] of this KV head
  float* out;             // [G][d] of this unit (row stride d)
  int np, g, r, d;
};

// smem: np*g + 2*g + g*r floats.  All NT threads must call it.
template <int NT>
__device__ void combine_unit(const CombineArgs& c, float* smem) {
  const int tid = threadIdx.x;
  float* w = smem;                 // [np][g] merge weights
  float* lsum = w + c.np * c.g;    // [g]
  float* zbar = lsum + c.g;        // [g][r]
  float* mmax = zbar + c.g * c.r;  // [g]
  for (int h = tid; h < c.g; h += NT) {
    float M = -INFINITY;
    for (int j = 0; j < c.np; ++j) M = fmaxf(M, __ldcg(c.part_ml + (j * c.g + h) * 2));
    mmax[h] = M;
  }
  __syncthreads();
  for (int i = tid; i < c.np * c.g; i += NT) {
    const int h = i % c.g;
    const float mj = __ldcg(c.part_ml + i * 2);
    w[i] = (mj == -INFINITY) ? 0.f : exp2f(mj - mmax[h]);
  }
  __syncthreads();
  for (int h = tid; h < c.g; h += NT) {
    float l = 0.f;
    for (int j = 0; j < c.np; ++j) l += w[j * c.g + h] * __ldcg(c.part_ml + (j * c.g + h) * 2 + 1);
    lsum[h] = l;
  }
  __syncthreads();
  for (int i = tid; i < c.g * c.r; i += NT) {
    const int h = i / c.r, a = i % c.r;
    float acc = 0.f;
    for (int j = 0; j < c.np; ++j) {
      const float wj = w[j * c.g + h];
      if (wj != 0.f) acc += wj * __ldcg(c.part_acc + (j * c.g + h) * c.r + a);
    }
    const float l = lsum[h];
    zbar[i] = l > 0.f ? acc / l : 0.f;
  }
  __syncthreads();
  for (int i = tid; i < c.g * c.d; i += NT) {
    const int h = i / c.d, col = i % c.d;
    const float* z = zbar + h * c.r;
    float o = 0.f;
    for (int a = 0; a < c.r; ++a) o = fmaf(z[a], __ldg(c.b_v + a * c.d + col), o);
    c.out[h * c.d + col] = o;
  }
}

}  // namespace basiskv

namespace basiskv {

// One-warp merge of a unit's partials and expansion through B_v (same
// arithmetic as combine_unit).  zbar: g*r floats of this warp's shared
// memory.  np <= 64.
template <int G, int RR, int D>
__device__ void warp_combine(const float* part_ml, const float* part_acc, int np, const float* b_v,
                             float* out, float* zbar) {
  const int lane = threadIdx.x & 31;
  // each lane owns partials j = lane and lane + 32
  float w0[G], w1[G], M[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float m0 = lane < np ? __ldcg(part_ml + (lane * G + h) * 2) : -INFINITY;
    const float m1 = lane + 32 < np ? __ldcg(part_ml + ((lane + 32) * G + h) * 2) : -INFINITY;
    M[h] = warp_max(fmaxf(m0, m1));
    w0[h] = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M[h]);
    w1[h] = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M[h]);
    float ls = 0.f;
    if (lane < np) ls += w0[h] * __ldcg(part_ml + (lane * G + h) * 2 + 1);
    if (lane + 32 < np) ls += w1[h] * __ldcg(part_ml + ((lane + 32) * G + h) * 2 + 1);
    l[h] = warp_sum(ls);
  }
  // zbar[h][i] = sum_j w_jh acc_j[h][i] / l_h, lanes over i; the loads do not
  // depend on one another, so the unrolled loop keeps several in flight
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i0 = 0; i0 < RR; i0 += 32) {  // uniform trip count: shuffles stay converged
      const int i = i0 + lane;
      float acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < np; ++j) {
        const float wj = __shfl_sync(0xffffffffu, j < 32 ? w0[h] : w1[h], j & 31);
        const float v = i < RR ? __ldcg(part_acc + ((size_t)j * G + h) * RR + i) : 0.f;
        acc = fmaf(wj, v, acc);
      }
      if (i < RR) zbar[h * RR + i] = l[h] > 0.f ? acc / l[h] : 0.f;
    }
  }
  __syncwarp();
  // out[h][c] = zbar[h] . B_v[:, c], lanes over c
  constexpr int CPL = (D + 31) / 32;
  float o[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[h][c] = 0.f;
#pragma unroll 8
  for (int i = 0; i < RR; ++i) {
    float bv[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) bv[c] = (lane + 32 * c < D) ? __ldg(b_v + (size_t)i * D + lane + 32 * c) : 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float z = zbar[h * RR + i];
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[h][c] = fmaf(z, bv[c], o[h][c]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c)
      if (lane + 32 * c < D) out[(size_t)h * D + lane + 32 * c] = o[h][c];
  __syncwarp();
}

}  // namespace basiskv
