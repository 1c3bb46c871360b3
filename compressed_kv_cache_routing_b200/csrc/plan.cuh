// Route-prep for the persistent kernels.  One CTA per (sequence, KV head):
//   - folds the routing bases into the query (qz_h = W_zk.q_h, qr_h = B_r.q_h,
//     fp32) and stores it as the bf16 hi/lo B-fragment words each lane of
//     the routing kernel's tensor-core product needs;
//   - for sequences without a page writes out = 0 and a -1 selection; for
//     sequences whose every page is used (k >= n_b, no routing) writes the
//     identity selection;
//   - CTA (0, 0) writes the work plan: exclusive prefix sums over sequences
//     of routed pages (x Hkv) and of attention items (selected pages x
//     stages per page x Hkv), so that every warp of the persistent kernels
//     can find its contiguous share of the flat work list.
#pragma once

#include "common.cuh"

namespace basiskv {

struct PrepArgs {
  const void* q;           // [B][Hkv*G][d]
  const float* w_zk;       // [Hkv][r][d]
  const float* b_r;        // [Hkv][s][d]
  const int32_t* seq_lens; // [B]
  int32_t* route_off;      // [B+1]
  int32_t* attn_off;       // [B+1]
  uint32_t* qfrag;         // [B*Hkv][fr][32]
  int32_t* sel_out;        // [B][Hkv][topk] or null
  float* out;              // [B][Hkv*G][d] or null
  float* scores;           // [B][Hkv][ld_pt]: -inf past n_b when fill_scores
  int batch, num_kv_heads, gqa_group, head_dim, page_size, rank_r, rank_s;
  int topk, force, attn_sub, ld_pt, fr, fill_scores;
};

constexpr int kPrepThreads = 128;

// Geometry of the routing B fragments for (G, r, s): per n8 tile j, the
// words are [Z k16 blocks x 2][Z k8][R k16 blocks x 2][R k8].
struct FragGeom {
  int nt, z32, z16, z8, s32, s16, s8, zb, sb, per_tile;
  __host__ __device__ FragGeom(int G, int r, int s) {
    nt = (2 * G + 7) / 8;
    z32 = r / 32; z16 = (r % 32) / 16; z8 = (r % 16) / 8;
    s32 = s / 32; s16 = (s % 32) / 16; s8 = (s % 16) / 8;
    zb = 2 * z32 + z16;
    sb = 2 * s32 + s16;
    per_tile = 2 * zb + z8 + 2 * sb + s8;
  }
  __host__ __device__ int words() const { return nt * per_tile; }
};

// Element (inside a row segment) holding logical pair `half` of k16 block
// `blk` for thread t; 32-wide spans first, then one 16-wide block.
__host__ __device__ __forceinline__ int k16_elem(int w32, int blk, int t, int half) {
  if (blk < 2 * w32) return 32 * (blk >> 1) + 8 * t + 4 * (blk & 1) + 2 * half;
  return 32 * w32 + 4 * t + 2 * half;
}

__device__ __forceinline__ float hi_or_lo(float x, bool lo) {
  float h, l;
  split_bf16(x, h, l);
  return lo ? l : h;
}

template <typename T>
__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const PrepArgs a) {
  pdl_launch_dependents();
  extern __shared__ __align__(16) float psm[];
  __shared__ int scan_tmp[kPrepThreads / 32];
  const int tid = threadIdx.x;
  const int G = a.gqa_group, d = a.head_dim, r = a.rank_r, s = a.rank_s, P = a.page_size;
  const int Hkv = a.num_kv_heads;

  if (blockIdx.x == 0 && blockIdx.y == 0) {
    int carry_r = 0, carry_a = 0;
    for (int b0 = 0; b0 < a.batch; b0 += kPrepThreads) {
      const int b = b0 + tid;
      int vr = 0, va = 0;
      if (b < a.batch) {
        const int n = (a.seq_lens[b] + P - 1) / P;
        const bool routed = n > 0 && (a.force || a.topk < n);
        vr = routed ? n * Hkv : 0;
        va = min(a.topk, n) * a.attn_sub * Hkv;
      }
      int tr, ta;
      const int er = block_exclusive_scan<kPrepThreads>(vr, scan_tmp, &tr);
      const int ea = block_exclusive_scan<kPrepThreads>(va, scan_tmp, &ta);
      if (b < a.batch) {
        a.route_off[b] = carry_r + er;
        a.attn_off[b] = carry_a + ea;
      }
      carry_r += tr;
      carry_a += ta;
    }
    if (tid == 0) {
      a.route_off[a.batch] = carry_r;
      a.attn_off[a.batch] = carry_a;
    }
  }

  const int b = blockIdx.y, kvh = blockIdx.x, u = b * Hkv + kvh;
  const int n = (a.seq_lens[b] + P - 1) / P;
  const bool routed = n > 0 && (a.force || a.topk < n);
  if (a.fill_scores)
    for (int j = n + tid; j < a.ld_pt; j += kPrepThreads) a.scores[(size_t)u * a.ld_pt + j] = -INFINITY;
  if (n == 0) {
    if (a.out)
      for (int i = tid; i < G * d; i += kPrepThreads) a.out[(size_t)u * G * d + i] = 0.f;
    if (a.sel_out)
      for (int i = tid; i < a.topk; i += kPrepThreads) a.sel_out[(size_t)u * a.topk + i] = -1;
    return;
  }
  if (!routed) {
    if (a.sel_out)
      for (int i = tid; i < a.topk; i += kPrepThreads) a.sel_out[(size_t)u * a.topk + i] = i < n ? i : -1;
    return;
  }

  // qz / qr in fp32: a thread per basis row computing all G heads; the row is
  // read as float4 (independent loads, L1-resident), q from shared memory
  float* qs = psm;              // [G][d]
  float* qz = qs + G * d;       // [G][r]
  float* qr = qz + G * r;       // [G][s]
  const T* q = static_cast<const T*>(a.q) + (size_t)u * G * d;
  for (int i = tid; i < G * d; i += kPrepThreads) qs[i] = to_f32(q[i]);
  __syncthreads();
  const float* W = a.w_zk + (size_t)kvh * r * d;
  const float* Br = a.b_r + (size_t)kvh * s * d;
  for (int row = tid; row < r + s; row += kPrepThreads) {
    const float* wrow = row < r ? W + (size_t)row * d : Br + (size_t)(row - r) * d;
    float part[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) part[h] = 0.f;
    if ((d & 3) == 0) {
#pragma unroll 4
      for (int c = 0; c < d; c += 4) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(wrow + c));
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          if (h < G) {
            const float* qh = qs + h * d + c;
            part[h] = fmaf(w.x, qh[0], fmaf(w.y, qh[1], fmaf(w.z, qh[2], fmaf(w.w, qh[3], part[h]))));
          }
        }
      }
    } else {
      for (int c = 0; c < d; ++c) {
        const float w = __ldg(wrow + c);
#pragma unroll
        for (int h = 0; h < 8; ++h)
          if (h < G) part[h] = fmaf(w, qs[h * d + c], part[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h < G) {
        if (row < r) qz[h * r + row] = part[h];
        else qr[h * s + (row - r)] = part[h];
      }
    }
  }
  __syncthreads();

  const FragGeom fg(G, r, s);
  uint32_t* dst = a.qfrag + (size_t)u * a.fr * 32;
  for (int idx = tid; idx < fg.words() * 32; idx += kPrepThreads) {
    const int lane = idx & 31, w = idx >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int j = w / fg.per_tile;
    int k = w % fg.per_tile;
    const int h = 4 * j + (g >> 1);
    const bool lo = g & 1;
    const float* src;
    int e;
    if (k < 2 * fg.zb) {
      src = qz + h * r;
      e = k16_elem(fg.z32, k >> 1, t, k & 1);
    } else if ((k -= 2 * fg.zb) < fg.z8) {
      src = qz + h * r;
      e = 32 * fg.z32 + 16 * fg.z16 + 2 * t;
    } else if ((k -= fg.z8) < 2 * fg.sb) {
      src = qr + h * s;
      e = k16_elem(fg.s32, k >> 1, t, k & 1);
    } else {
      src = qr + h * s;
      e = 32 * fg.s32 + 16 * fg.s16 + 2 * t;
    }
    uint32_t word = 0u;
    if (h < G) word = pack_bf16(hi_or_lo(src[e], lo), hi_or_lo(src[e + 1], lo));
    dst[w * 32 + lane] = word;
  }
}

}  // namespace basiskv
