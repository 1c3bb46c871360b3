// Work plan for the persistent kernels of a large batch, whose plan does not
// fit in the kernel parameters.  One CTA per (sequence, KV head):
//   - for sequences without a page writes out = 0 and a -1 selection; for
//     sequences whose every page is used (k >= n_b, no routing) writes the
//     identity selection; with fill_scores, -inf past the last page;
//   - CTA (0, 0) writes the work plan: exclusive prefix sums over sequences
//     of routed pages (x Hkv) and of attention items (selected pages x
//     stages per page x Hkv), so that every warp of the persistent kernels
//     can find its contiguous share of the flat work list.
#pragma once

#include "common.cuh"

namespace basiskv {

struct PrepArgs {
  const int32_t* seq_lens; // [B]
  int32_t* route_off;      // [B+1]
  int32_t* attn_off;       // [B+1]
  int32_t* sel_out;        // [B][Hkv][topk] or null
  float* out;              // [B][Hkv*G][d] or null
  float* scores;           // [B][Hkv][ld_pt]: -inf past n_b when fill_scores
  int batch, num_kv_heads, gqa_group, head_dim, page_size;
  int topk, force, attn_sub, ld_pt, fill_scores;
  int out_width;           // d, or r for the latent output
};

constexpr int kPrepThreads = 128;

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(const PrepArgs a) {
  pdl_launch_dependents();
  __shared__ int scan_tmp[kPrepThreads / 32];
  const int tid = threadIdx.x;
  const int G = a.gqa_group, P = a.page_size;
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
      for (int i = tid; i < G * a.out_width; i += kPrepThreads) a.out[(size_t)u * G * a.out_width + i] = 0.f;
    if (a.sel_out)
      for (int i = tid; i < a.topk; i += kPrepThreads) a.sel_out[(size_t)u * a.topk + i] = -1;
    return;
  }
  if (!routed && a.sel_out)
    for (int i = tid; i < a.topk; i += kPrepThreads) a.sel_out[(size_t)u * a.topk + i] = i < n ? i : -1;
}

}  // namespace basiskv
