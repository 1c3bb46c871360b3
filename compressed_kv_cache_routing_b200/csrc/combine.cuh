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
  float* out;             // [G][d] of this unit (row stride d); [G][r] when latent
  int np, g, r, d;
  int latent;             // write zbar itself, before B_v
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
  if (c.latent) {
    for (int i = tid; i < c.g * c.r; i += NT) c.out[i] = zbar[i];
    return;
  }
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

// Count one arrival at `ctr` (warp-collective, after this warp's writes);
// true in every lane of the warp that completes `expected` arrivals, which
// also resets the counter.  Everything the other arrivers wrote before
// arriving is visible to that warp afterwards (read it through L2).
__device__ __forceinline__ bool arrive_count(uint32_t* ctr, uint32_t expected) {
  __syncwarp();
  int last = 0;
  if ((threadIdx.x & 31) == 0) {
    __threadfence();
    last = atomicAdd(ctr, 1u) + 1 == expected;
    if (last) {
      *ctr = 0u;
      __threadfence();
    }
  }
  return __shfl_sync(0xffffffffu, last, 0) != 0;
}

// Merged attention state of a set of partials: lane h < G holds head h's
// running max M and sum L (log2 units); every lane holds its float4 slices
// v = lane + 32k of the [G][r] latent sum (head 4v / r).
template <int G, int RR>
struct MergeOut {
  static constexpr int V = G * RR / 4, VPL = (V + 31) / 32;
  float4 acc[VPL];
  float M, L;
};

// Merge `cnt` <= 8 partials ((m, l) pairs at ml [cnt][G][2], latent sums at
// acc [cnt][G][r], written by other warps): M = max m, w = 2^(m - M),
// L = sum w l, acc = sum w acc, in chunk order.  All loads are issued
// together (float4 slices) so the merge costs about one L2 round trip.
template <int G, int RR>
__device__ void merge_partials(const float* ml, const float* acc, int cnt, MergeOut<G, RR>& o) {
  static_assert(RR % 4 == 0 && 32 % G == 0, "shape");
  constexpr int V = MergeOut<G, RR>::V, VPL = MergeOut<G, RR>::VPL;
  const int lane = threadIdx.x & 31;
  constexpr int JB = VPL >= 4 ? 4 : 8;  // chunks whose slices are loaded together (<= 16 float4 in flight)
  // the first group's latent slices are requested before the (m, l) pairs,
  // so both arrive in one L2 round trip
  float4 x[JB][VPL];
  auto load_group = [&](int j0) {
#pragma unroll
    for (int jj = 0; jj < JB; ++jj)
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int j = j0 + jj, v = lane + 32 * k;
        x[jj][k] = (j < cnt && v < V) ? __ldcg(reinterpret_cast<const float4*>(acc + (size_t)j * G * RR) + v)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
  };
  load_group(0);
  // pairs q = lane and lane + 32: chunk q / G, head q % G (= lane % G)
  float mA = -INFINITY, lA = 0.f, mB = -INFINITY, lB = 0.f;
  if (lane < cnt * G) {
    const float2 x = __ldcg(reinterpret_cast<const float2*>(ml) + lane);
    mA = x.x;
    lA = x.y;
  }
  if (lane + 32 < cnt * G) {
    const float2 x = __ldcg(reinterpret_cast<const float2*>(ml) + lane + 32);
    mB = x.x;
    lB = x.y;
  }
  float M = fmaxf(mA, mB);
#pragma unroll
  for (int off = 16; off >= G; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float wA = mA == -INFINITY ? 0.f : exp2f(mA - M), wB = mB == -INFINITY ? 0.f : exp2f(mB - M);
  float L = wA * lA + wB * lB;
#pragma unroll
  for (int off = 16; off >= G; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  o.M = M;
  o.L = L;
#pragma unroll
  for (int k = 0; k < VPL; ++k) o.acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j0 = 0; j0 < 8; j0 += JB) {
    if (j0 >= cnt) break;
    if (j0 > 0) load_group(j0);
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
      const int j = j0 + jj;
      if (j < cnt) {
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
          const int h = (4 * (lane + 32 * k)) / RR;
          const int q = j * G + (h < G ? h : 0);
          const float wa = __shfl_sync(0xffffffffu, wA, q & 31), wb = __shfl_sync(0xffffffffu, wB, q & 31);
          const float w = q < 32 ? wa : wb;
          o.acc[k].x = fmaf(w, x[jj][k].x, o.acc[k].x);
          o.acc[k].y = fmaf(w, x[jj][k].y, o.acc[k].y);
          o.acc[k].z = fmaf(w, x[jj][k].z, o.acc[k].z);
          o.acc[k].w = fmaf(w, x[jj][k].w, o.acc[k].w);
        }
      }
    }
  }
}

// a <- the merge of a and b (both over disjoint partials of one unit): each
// head rescaled to the larger running max.  Every lane holds M, L of head
// lane % G; a slice's head h is read from lane h.
template <int G, int RR>
__device__ __forceinline__ void merge_into(MergeOut<G, RR>& a, const MergeOut<G, RR>& b) {
  constexpr int VPL = MergeOut<G, RR>::VPL;
  const int lane = threadIdx.x & 31;
  const float M = fmaxf(a.M, b.M);
  const float wa = a.M == -INFINITY ? 0.f : exp2f(a.M - M), wb = b.M == -INFINITY ? 0.f : exp2f(b.M - M);
  a.L = fmaf(wb, b.L, wa * a.L);
  a.M = M;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int h = (4 * (lane + 32 * k)) / RR;
    const float sa = __shfl_sync(0xffffffffu, wa, h < G ? h : 0), sb = __shfl_sync(0xffffffffu, wb, h < G ? h : 0);
    a.acc[k].x = fmaf(sb, b.acc[k].x, sa * a.acc[k].x);
    a.acc[k].y = fmaf(sb, b.acc[k].y, sa * a.acc[k].y);
    a.acc[k].z = fmaf(sb, b.acc[k].z, sa * a.acc[k].z);
    a.acc[k].w = fmaf(sb, b.acc[k].w, sa * a.acc[k].w);
  }
}

// Merge np (>= 1) partials, in groups of 8 taken in slot order.
template <int G, int RR>
__device__ void merge_all(const float* ml, const float* acc, int np, MergeOut<G, RR>& o) {
  merge_partials<G, RR>(ml, acc, min(np, 8), o);
  for (int j0 = 8; j0 < np; j0 += 8) {
    MergeOut<G, RR> t;
    merge_partials<G, RR>(ml + (size_t)j0 * G * 2, acc + (size_t)j0 * G * RR, min(np - j0, 8), t);
    merge_into(o, t);
  }
}

// Latent output: zbar = acc / L per head, written as [G][r] (no B_v).
template <int G, int RR>
__device__ void finish_unit_latent(const MergeOut<G, RR>& mo, float* out) {
  constexpr int V = MergeOut<G, RR>::V, VPL = MergeOut<G, RR>::VPL;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int v = lane + 32 * k;
    const int h = (4 * v) / RR;
    const float Lh = __shfl_sync(0xffffffffu, mo.L, h < G ? h : 0);
    if (v < V) {
      const float inv = Lh > 0.f ? 1.f / Lh : 0.f;
      reinterpret_cast<float4*>(out)[v] =
          make_float4(mo.acc[k].x * inv, mo.acc[k].y * inv, mo.acc[k].z * inv, mo.acc[k].w * inv);
    }
  }
}

// zbar = acc / L per head, out_h = zbar_h . B_v (fp32, d wide; lanes own
// d/32 consecutive columns).  zbar: G*r floats of this warp's shared memory.
template <int G, int RR, int D>
__device__ void finish_unit(const MergeOut<G, RR>& mo, const float* b_v, float* out, float* zbar) {
  constexpr int V = MergeOut<G, RR>::V, VPL = MergeOut<G, RR>::VPL, CPL = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int v = lane + 32 * k;
    const int h = (4 * v) / RR;
    const float Lh = __shfl_sync(0xffffffffu, mo.L, h < G ? h : 0);
    if (v < V) {
      const float inv = Lh > 0.f ? 1.f / Lh : 0.f;
      reinterpret_cast<float4*>(zbar)[v] =
          make_float4(mo.acc[k].x * inv, mo.acc[k].y * inv, mo.acc[k].z * inv, mo.acc[k].w * inv);
    }
  }
  __syncwarp();
  float o[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[h][c] = 0.f;
#pragma unroll 16
  for (int i = 0; i < RR; ++i) {
    float bv[CPL];
    if constexpr (CPL == 4) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(b_v + (size_t)i * D) + lane);
      bv[0] = b.x;
      bv[1] = b.y;
      bv[2] = b.z;
      bv[3] = b.w;
    } else {
      const float2 b = __ldg(reinterpret_cast<const float2*>(b_v + (size_t)i * D) + lane);
      bv[0] = b.x;
      bv[1] = b.y;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float z = zbar[h * RR + i];
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[h][c] = fmaf(z, bv[c], o[h][c]);
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if constexpr (CPL == 4)
      reinterpret_cast<float4*>(out + (size_t)h * D)[lane] = make_float4(o[h][0], o[h][1], o[h][2], o[h][3]);
    else
      reinterpret_cast<float2*>(out + (size_t)h * D)[lane] = make_float2(o[h][0], o[h][1]);
  }
  __syncwarp();
}

}  // namespace basiskv
