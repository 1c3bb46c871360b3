// Page routing for BasisKV decode attention ("the compressed Value cache is
// further reused to help identify which Key pages should be accessed: it
// predicts part of the Key information needed for routing, while a
// Key-specific residual stores what cannot be recovered from Value").
//
// Routing key  Khat_t = Z_t.W_zk + R_t.B_r  is never formed: the kernels fold
// the bases into the query (route-prep),
//     qz_h = W_zk.q_h  (r floats),   qr_h = B_r.q_h  (s floats),
// so that  q_h.Khat_t = Z_t.qz_h + R_t.qr_h  costs r + s multiply-adds per
// token and head and reads only the r + s stored values of each token.
// Page score S_j = max over the G heads and page j's valid tokens.
//
// Two kernels: route_mma_kernel (bf16 pools, tensor cores, persistent over a
// flat page list; the fold is spread over all warps as (unit, row slice)
// tasks written to global memory and tagged, and a warp entering a unit
// reads it back, folding locally only if the slices are late; the
// selection runs in the next grid) and route_generic_kernel (any dtype,
// grid (chunks of pages, Hkv, batch), fold once per CTA, the last CTA of
// each (sequence, KV head) runs the top-k).
#pragma once

#include "common.cuh"
#include "plan.cuh"
#include "topk.cuh"

namespace basiskv {

struct RouteArgs {
  const void* q;            // [B][Hkv*G][d]
  const void* z_pool;       // [slots][Hkv][P][r]
  const void* r_pool;       // [slots][Hkv][P][s]
  const float* w_zk;        // [Hkv][r][d]
  const float* b_r;         // [Hkv][s][d]
  const int32_t* page_table;  // [B][ld_pt]
  const int32_t* seq_lens;  // [B]
  float* scores;            // [B][Hkv][ld_pt]
  int32_t* sel;             // [B][Hkv][ld_sel]
  int32_t* sel_out;         // [B][Hkv][topk] or null
  uint32_t* counters;       // [B][Hkv]
  uint32_t* status;
  int ld_pt, ld_sel, num_slots, num_kv_heads, head_dim, page_size;
  int rank_r, rank_s, gqa_group;
  int topk, pages_per_cta, stages;
  int force;                // route units whose every page would be selected
  int fill_tail;            // chunk 0 writes -inf to scores[n_b .. ld_pt)
  // persistent tensor-core kernel only
  int batch;
  const int32_t* route_off; // [B+1] prefix of routed pages x Hkv (from the prep grid)
  float* qf;                // [B*Hkv][G][r+s] folded queries (fp32)
  uint32_t* fold_flag;      // [B*Hkv][32] per fold slice: the tag of the call that wrote it
  uint32_t tag;             // this call's tag (never 0)
  int plan_n;               // >= 0: plan_off holds route_off (batch <= kPlanMax)
  int32_t plan_off[kPlanMax + 1];
};

constexpr int kRouteThreads = 128;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kMaxStages = 8;

// Pages staged together by route_mma_kernel: about 6 KB per stage, so small
// pages (P = 32 with narrow ranks) share one barrier wait and one issue.
constexpr int route_pages_per_stage(int page_size, int rank_r, int rank_s) {
  const int page_bytes = page_size * (rank_r + rank_s) * 2;
  const int rps = page_bytes > 0 ? 6144 / page_bytes : 1;
  return rps < 1 ? 1 : (rps > 4 ? 4 : rps);
}

struct RouteUnit {
  int b, kvh, u, L, n, first, last;  // pages [first, last) of this CTA
  bool active;
};

__device__ __forceinline__ RouteUnit route_unit(const RouteArgs& a) {
  RouteUnit ru;
  ru.b = blockIdx.z;
  ru.kvh = blockIdx.y;
  ru.u = ru.b * a.num_kv_heads + ru.kvh;
  ru.L = a.seq_lens[ru.b];
  ru.n = (ru.L + a.page_size - 1) / a.page_size;
  if (ru.n > a.ld_pt || ru.L < 0) {
    // a length the page-table row cannot hold (only callers that pass
    // device lengths unchecked can get here): clamp to the row
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.status, kStatusBadLength);
    ru.L = ru.L < 0 ? 0 : a.ld_pt * a.page_size;
    ru.n = ru.L / a.page_size;
  }
  ru.first = blockIdx.x * a.pages_per_cta;
  ru.last = min(ru.n, ru.first + a.pages_per_cta);
  ru.active = ru.first < ru.n && (a.force || a.topk < ru.n);
  return ru;
}

// Route-prep: qz = W_zk.q_h and qr = B_r.q_h for the G heads of the group,
// fp32, into shared memory ([G][r] then [G][s]).  qs: [G][d] fp32 scratch.
template <typename T>
__device__ void route_prep(const RouteArgs& a, const RouteUnit& ru, float* qs, float* qz, float* qr) {
  const int G = a.gqa_group, d = a.head_dim, r = a.rank_r, s = a.rank_s;
  const T* q = static_cast<const T*>(a.q) + ((size_t)ru.b * a.num_kv_heads + ru.kvh) * G * d;
  for (int i = threadIdx.x; i < G * d; i += blockDim.x) qs[i] = to_f32(q[i]);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* W = a.w_zk + (size_t)ru.kvh * r * d;
  const float* Br = a.b_r + (size_t)ru.kvh * s * d;
  for (int row = warp; row < r + s; row += nw) {
    const float* wrow = row < r ? W + (size_t)row * d : Br + (size_t)(row - r) * d;
    for (int h = 0; h < G; ++h) {
      float acc = 0.f;
      for (int c = lane; c < d; c += 32) acc = fmaf(__ldg(wrow + c), qs[h * d + c], acc);
      acc = warp_sum(acc);
      if (lane == 0) {
        if (row < r) qz[h * r + row] = acc;
        else qr[h * s + (row - r)] = acc;
      }
    }
  }
  __syncthreads();
}

// After the scores of this CTA's pages are written: the last CTA of the unit
// selects the pages.
template <int NT>
__device__ void route_finish(const RouteArgs& a, const RouteUnit& ru, TopkSmem& tk, int* flag) {
  const int chunks = (ru.n + a.pages_per_cta - 1) / a.pages_per_cta;
  if (!arrive_last(a.counters + ru.u, (uint32_t)chunks, flag)) return;
  const float* sc = a.scores + (size_t)ru.u * a.ld_pt;
  int32_t* so = a.sel_out ? a.sel_out + (size_t)ru.u * a.topk : nullptr;
  block_topk<NT>(sc, ru.n, a.topk, a.sel + (size_t)ru.u * a.ld_sel, so, a.topk, tk);
}

// ---------------------------------------------------------------------------
// Tensor-core routing for bf16 pools.
//
// Per page, the product  [P tokens x (r+s)] . [(r+s) x 2G]  runs as
// mma.m16n8k16 / m16n8k8 (bf16 in, fp32 accumulate): A = the page's Z (and
// R) rows straight from shared memory, B = the folded query split into
// bf16 hi + lo halves (column 2h = hi(qz_h), 2h+1 = lo(qz_h)), so the fp32
// routing query keeps ~16 significant bits and the stored bf16 data are
// exact.  The k index inside each 16-wide block is permuted so that every
// thread's A fragment is one contiguous 8- or 16-byte shared load:
//   32-wide span, thread t reads elements [8t, 8t+8): block 0 gets
//   {8t..8t+3}, block 1 gets {8t+4..8t+7}; a 16-wide block gives thread t
//   elements [4t, 4t+4); an 8-wide block (m16n8k8) elements [2t, 2t+2).
// The B fragments use the same permutation, so every dot product is a sum
// over the same index set.
//
// Persistent: every warp streams one contiguous share of the flat list of
// routed pages (sequence-major, then KV head, then page) through its own
// ring of `stages` shared buffers filled by bulk copies (cp.async.bulk, L2
// evict-first) completing on mbarriers, and writes one score per page.  The
// selection runs in the next grid (topk_kernel).
template <int G, int RR, int RS>
struct RouteMma {
  static constexpr int NT = (2 * G + 7) / 8;  // n8 tiles of (hi, lo) columns
  static constexpr int Z32 = RR / 32, Z16 = (RR % 32) / 16, Z8 = (RR % 16) / 8;
  static constexpr int S32 = RS / 32, S16 = (RS % 32) / 16, S8 = (RS % 16) / 8;
  static constexpr int ZB = 2 * Z32 + Z16;  // k16 blocks over Z
  static constexpr int SB = 2 * S32 + S16;  // k16 blocks over R
  static_assert(RR % 8 == 0 && RS % 8 == 0, "ranks must be multiples of 8");
};

// physical element (within a row segment) of logical pair `half` (0: k
// 2t..2t+1, 1: k 2t+8..2t+9) of k16 block `blk` for thread t
template <int W32, int W16>
__device__ __forceinline__ int k16_phys(int blk, int t, int half) {
  if (blk < 2 * W32) return 32 * (blk >> 1) + 8 * t + 4 * (blk & 1) + 2 * half;
  return 32 * W32 + 4 * t + 2 * half;
}

// Routing score of one staged page: the max over the G heads and the page's
// `valid` tokens of Z_t.qz_h + R_t.qr_h, from the page's Z rows `zs` and R
// rows `rs` in shared memory and this lane's folded-query fragments `fr`
// (mma tiles: tokens as M, (head, hi|lo) as N).  Returned in every lane.
template <int G, int RR, int RS, int P, int FR>
__device__ __forceinline__ float route_page_score(const __nv_bfloat16* zs, const __nv_bfloat16* rs, int valid,
                                                  const uint32_t (&fr)[FR]) {
  using Shape = RouteMma<G, RR, RS>;
  constexpr int NT = Shape::NT;
  constexpr int FRT = 2 * Shape::ZB + Shape::Z8 + 2 * Shape::SB + Shape::S8;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float best = -INFINITY;
#pragma unroll
  for (int mt = 0; mt < P / 16; ++mt) {
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    const __nv_bfloat16* z0 = zs + (mt * 16 + g) * RR;
    const __nv_bfloat16* z1 = z0 + 8 * RR;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const uint32_t* f = fr + j * FRT;
#pragma unroll
      for (int sp = 0; sp < Shape::Z32; ++sp) {
        const uint4 v0 = lds128(z0 + 32 * sp + 8 * t), v1 = lds128(z1 + 32 * sp + 8 * t);
        mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, f[4 * sp + 0], f[4 * sp + 1]);
        mma_k16(acc[j], v0.z, v1.z, v0.w, v1.w, f[4 * sp + 2], f[4 * sp + 3]);
      }
      if (Shape::Z16) {
        const uint2 v0 = lds64(z0 + 32 * Shape::Z32 + 4 * t), v1 = lds64(z1 + 32 * Shape::Z32 + 4 * t);
        mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, f[2 * Shape::ZB - 2], f[2 * Shape::ZB - 1]);
      }
      if (Shape::Z8) {
        const int o = 32 * Shape::Z32 + 16 * Shape::Z16 + 2 * t;
        mma_k8(acc[j], lds32(z0 + o), lds32(z1 + o), f[2 * Shape::ZB]);
      }
      if (RS > 0) {
        const uint32_t* fs = f + 2 * Shape::ZB + Shape::Z8;
        const __nv_bfloat16* r0 = rs + (mt * 16 + g) * RS;
        const __nv_bfloat16* r1 = r0 + 8 * RS;
#pragma unroll
        for (int sp = 0; sp < Shape::S32; ++sp) {
          const uint4 v0 = lds128(r0 + 32 * sp + 8 * t), v1 = lds128(r1 + 32 * sp + 8 * t);
          mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, fs[4 * sp + 0], fs[4 * sp + 1]);
          mma_k16(acc[j], v0.z, v1.z, v0.w, v1.w, fs[4 * sp + 2], fs[4 * sp + 3]);
        }
        if (Shape::S16) {
          const uint2 v0 = lds64(r0 + 32 * Shape::S32 + 4 * t), v1 = lds64(r1 + 32 * Shape::S32 + 4 * t);
          mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, fs[2 * Shape::SB - 2], fs[2 * Shape::SB - 1]);
        }
        if (Shape::S8) {
          const int o = 32 * Shape::S32 + 16 * Shape::S16 + 2 * t;
          mma_k8(acc[j], lds32(r0 + o), lds32(r1 + o), fs[2 * Shape::SB]);
        }
      }
    }
    // D fragment: rows g, g+8 = tokens; columns 2t, 2t+1 = (hi, lo) of head 4j + t.
    // Rows past the sequence end are dropped by selection, never by arithmetic.
    const int tok0 = mt * 16 + g, tok1 = tok0 + 8;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (4 * j + t < G) {
        if (tok0 < valid) best = fmaxf(best, acc[j][0] + acc[j][1]);
        if (tok1 < valid) best = fmaxf(best, acc[j][2] + acc[j][3]);
      }
    }
  }
  return warp_max(best);
}

// Position in the flat list of routed pages (sequence-major, then KV head,
// then page), advanced one page at a time.
struct RouteCursor {
  int b, kvh, j, n, L;
  const int32_t* off;  // prefix of routed pages x Hkv over sequences
  __device__ __forceinline__ void load(const RouteArgs& a) {
    L = a.seq_lens[b];
    n = (L + a.page_size - 1) / a.page_size;
  }
  __device__ __forceinline__ bool routed(const RouteArgs& a) const {
    return n > 0 && (a.force || a.topk < n);
  }
  // first page at or after flat index f (route_off[b] <= f < route_off[b+1])
  __device__ void seek(const RouteArgs& a, const int32_t* offsets, int f) {
    off = offsets;
    int lo = 0, hi = a.batch;  // first b with off[b] > f, minus one
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= f) lo = mid + 1;
      else hi = mid;
    }
    b = lo - 1;
    load(a);
    const int rel = f - off[b];
    kvh = rel / n;
    j = rel % n;
  }
  __device__ __forceinline__ void advance(const RouteArgs& a) {
    if (++j < n) return;
    j = 0;
    if (++kvh < a.num_kv_heads) return;
    kvh = 0;
    for (++b; b < a.batch; ++b) {
      load(a);
      if (routed(a)) return;
    }
  }
  __device__ __forceinline__ int unit(const RouteArgs& a) const { return b * a.num_kv_heads + kvh; }
};

// Route-prep inside the routing warp: fold W_zk and B_r of KV head kvh into
// the G queries of sequence b (qz_h = W_zk.q_h, qr_h = B_r.q_h, fp32) and
// return this lane's B-fragment words of the split (hi, lo) folded query.
// Lanes own d/32 consecutive channels; for each block of 32/G basis rows a
// lane forms its 32 partial (row, head) dot products and a butterfly
// reduce-scatter (31 shuffles) leaves the sum of (row, head) = (lane/G,
// lane%G) in lane; the sums meet in the warp's shared scratch `qsm`
// ([G][r] then [G][s]) to be regrouped into fragment order.
template <int G, int RR, int RS, int FR, int CPL>
__device__ void warp_fold_query(const RouteArgs& a, int b, int kvh, float* qsm, uint32_t (&fr)[FR]) {
  static_assert(32 % G == 0, "G must divide 32");
  static_assert(CPL == 2 || CPL == 4, "head_dim 64 or 128");
  constexpr int RPB = 32 / G;
  constexpr int ROWS = RR + RS;
  constexpr int d = 32 * CPL;
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)b * a.num_kv_heads + kvh) * G * d +
                           lane * CPL;
  float qv[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int j = 0; j < CPL; ++j) qv[h][j] = __bfloat162float(q[h * d + j]);
  const float* W = a.w_zk + (size_t)kvh * RR * d + lane * CPL;
  const float* Br = a.b_r + (size_t)kvh * RS * d + lane * CPL;
#pragma unroll 1
  for (int row0 = 0; row0 < ROWS; row0 += RPB) {
    float v[32];
#pragma unroll
    for (int rl = 0; rl < RPB; ++rl) {
      const int row = row0 + rl;
      const float* src = row < RR ? W + (size_t)row * d : Br + (size_t)(row - RR) * d;
      float w[CPL];
      if constexpr (CPL == 4) {
        const float4 x = row < ROWS ? __ldg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
        w[0] = x.x;
        w[1] = x.y;
        w[2] = x.z;
        w[3] = x.w;
      } else {
        const float2 x = row < ROWS ? __ldg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
        w[0] = x.x;
        w[1] = x.y;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < CPL; ++j) acc = fmaf(w[j], qv[h][j], acc);
        v[rl * G + h] = acc;
      }
    }
#pragma unroll
    for (int step = 16, cnt = 32; step >= 1; step >>= 1, cnt >>= 1) {
      const bool upper = (lane & step) != 0;
#pragma unroll
      for (int k = 0; k < cnt / 2; ++k) {
        const float send = upper ? v[k] : v[k + cnt / 2];
        const float keep = upper ? v[k + cnt / 2] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, step);
      }
    }
    const int row = row0 + lane / G, h = lane % G;
    if (row < RR) qsm[h * RR + row] = v[0];
    else if (row < ROWS) qsm[G * RR + h * RS + (row - RR)] = v[0];
  }
  __syncwarp();
  // regroup into this lane's fragment words (same order as the kernel reads)
  using Shape = RouteMma<G, RR, RS>;
  const int g = lane >> 2, t = lane & 3;
  int w = 0;
#pragma unroll
  for (int j = 0; j < Shape::NT; ++j) {
    const int hh = 4 * j + (g >> 1);
    const bool lo = g & 1;
    const float* qz = qsm + hh * RR;
    const float* qr = qsm + G * RR + hh * RS;
    auto word = [&](const float* src, int e) {
      if (hh >= G) return 0u;
      float h0, l0, h1, l1;
      split_bf16(src[e], h0, l0);
      split_bf16(src[e + 1], h1, l1);
      return lo ? pack_bf16(l0, l1) : pack_bf16(h0, h1);
    };
#pragma unroll
    for (int blk = 0; blk < Shape::ZB; ++blk) {
      fr[w++] = word(qz, k16_phys<Shape::Z32, Shape::Z16>(blk, t, 0));
      fr[w++] = word(qz, k16_phys<Shape::Z32, Shape::Z16>(blk, t, 1));
    }
    if (Shape::Z8) fr[w++] = word(qz, 32 * Shape::Z32 + 16 * Shape::Z16 + 2 * t);
#pragma unroll
    for (int blk = 0; blk < Shape::SB; ++blk) {
      fr[w++] = word(qr, k16_phys<Shape::S32, Shape::S16>(blk, t, 0));
      fr[w++] = word(qr, k16_phys<Shape::S32, Shape::S16>(blk, t, 1));
    }
    if (Shape::S8) fr[w++] = word(qr, 32 * Shape::S32 + 16 * Shape::S16 + 2 * t);
  }
  __syncwarp();
}

// Route-prep, spread over the routing warps: one fold slice each.
// Rows [slice*32/G, +32/G) of [W_zk; B_r] of unit u's KV head times the G
// queries: lanes own d/32 consecutive channels, each forms its 32 partial
// (row, head) products and a butterfly reduce-scatter (31 shuffles) leaves
// the full sum of (row, head) = (lane/G, lane%G) in the lane.
template <int G, int RR, int RS, int CPL>
__device__ void fold_slice(const void* q_all, const float* w_zk, const float* b_r, float* qf, int num_kv_heads,
                           int u, int slice) {
  constexpr int RPB = 32 / G, ROWS = RR + RS, d = 32 * CPL;
  const int lane = threadIdx.x & 31;
  const int kvh = u % num_kv_heads;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(q_all) + (size_t)u * G * d + lane * CPL;
  float qv[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int j = 0; j < CPL; ++j) qv[h][j] = __bfloat162float(q[h * d + j]);
  const int row0 = slice * RPB;
  float v[32];
#pragma unroll
  for (int rl = 0; rl < RPB; ++rl) {
    const int row = row0 + rl;
    const float* src = row < RR ? w_zk + ((size_t)kvh * RR + row) * d
                                : b_r + ((size_t)kvh * RS + (row - RR)) * d;
    src += lane * CPL;
    float w[CPL];
    if constexpr (CPL == 4) {
      const float4 x = row < ROWS ? __ldg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
      w[0] = x.x;
      w[1] = x.y;
      w[2] = x.z;
      w[3] = x.w;
    } else {
      const float2 x = row < ROWS ? __ldg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
      w[0] = x.x;
      w[1] = x.y;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < CPL; ++j) acc = fmaf(w[j], qv[h][j], acc);
      v[rl * G + h] = acc;
    }
  }
#pragma unroll
  for (int step = 16, cnt = 32; step >= 1; step >>= 1, cnt >>= 1) {
    const bool upper = (lane & step) != 0;
#pragma unroll
    for (int k = 0; k < cnt / 2; ++k) {
      const float send = upper ? v[k] : v[k + cnt / 2];
      const float keep = upper ? v[k + cnt / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, step);
    }
  }
  const int row = row0 + lane / G, h = lane % G;
  if (row < ROWS) qf[((size_t)u * G + h) * ROWS + row] = v[0];
}

template <int G, int RR, int RS, int CPL>
__device__ __forceinline__ void fold_slice(const RouteArgs& a, int u, int slice) {
  fold_slice<G, RR, RS, CPL>(a.q, a.w_zk, a.b_r, a.qf, a.num_kv_heads, u, slice);
}

// This lane's routing B-fragment words for unit u, from the folded query
// (split into bf16 hi + lo columns; same order as route_mma_kernel), read
// from global memory (written by other warps of this grid: read through L2).
template <int G, int RR, int RS, int FR>
__device__ void load_route_frags(const float* qfu, uint32_t (&fr)[FR]) {
  using Shape = RouteMma<G, RR, RS>;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  int w = 0;
#pragma unroll
  for (int j = 0; j < Shape::NT; ++j) {
    const int hh = 4 * j + (g >> 1);
    const bool lo = g & 1;
    const float* qz = qfu + hh * (RR + RS);
    const float* qr = qz + RR;
    auto word = [&](const float* src, int e) {
      if (hh >= G) return 0u;
      const float2 x = __ldcg(reinterpret_cast<const float2*>(src + e));
      float h0, l0, h1, l1;
      split_bf16(x.x, h0, l0);
      split_bf16(x.y, h1, l1);
      return lo ? pack_bf16(l0, l1) : pack_bf16(h0, h1);
    };
#pragma unroll
    for (int blk = 0; blk < Shape::ZB; ++blk) {
      fr[w++] = word(qz, k16_phys<Shape::Z32, Shape::Z16>(blk, t, 0));
      fr[w++] = word(qz, k16_phys<Shape::Z32, Shape::Z16>(blk, t, 1));
    }
    if (Shape::Z8) fr[w++] = word(qz, 32 * Shape::Z32 + 16 * Shape::Z16 + 2 * t);
#pragma unroll
    for (int blk = 0; blk < Shape::SB; ++blk) {
      fr[w++] = word(qr, k16_phys<Shape::S32, Shape::S16>(blk, t, 0));
      fr[w++] = word(qr, k16_phys<Shape::S32, Shape::S16>(blk, t, 1));
    }
    if (Shape::S8) fr[w++] = word(qr, 32 * Shape::S32 + 16 * Shape::S16 + 2 * t);
  }
}

template <int G, int RR, int RS, int P>
__global__ void __launch_bounds__(kRouteThreads) route_mma_kernel(const __grid_constant__ RouteArgs a) {
  using Shape = RouteMma<G, RR, RS>;
  constexpr int NT = Shape::NT;
  static_assert(P % 16 == 0, "page size must be a multiple of 16");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr uint32_t zbytes = P * RR * 2, rbytes = P * RS * 2;
  constexpr uint32_t page_bytes = zbytes + rbytes;
  constexpr int RPS = route_pages_per_stage(P, RR, RS);
  constexpr uint32_t stage_bytes = RPS * page_bytes;
  const int S = a.stages;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[kRouteWarps][kMaxStages];
  __shared__ float qsm_all[kRouteWarps][G * (RR + RS)];
  float* qsm = qsm_all[warp];
  uint8_t* ring = smem + (size_t)warp * S * stage_bytes;
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[warp][i], 1);
    mbar_init_fence();
  }
  __syncwarp();
  // The plan comes in the parameters (small batches) or from the prep grid
  // (then this grid waits for it first).  The query is folded by the warp
  // itself once its first copies are in flight.
  const int32_t* offsets = a.plan_n >= 0 ? a.plan_off : a.route_off;
  if (a.plan_n < 0) pdl_wait_primary();

  // this warp's contiguous share of the flat routed-page list
  const int W = gridDim.x * kRouteWarps, wg = blockIdx.x * kRouteWarps + warp;
  const long long T = offsets[a.batch];
  const int f0 = (int)(T * wg / W), f1 = (int)(T * (wg + 1) / W);
  const int count = f1 - f0;              // pages
  const int nst = (count + RPS - 1) / RPS;  // stages of up to RPS pages

  const __nv_bfloat16* zpool = static_cast<const __nv_bfloat16*>(a.z_pool);
  const __nv_bfloat16* rpool = static_cast<const __nv_bfloat16*>(a.r_pool);
  const uint64_t pol = policy_evict_first();
  RouteCursor ic;  // issue cursor (lane 0), runs S stages ahead
  if (count > 0) ic.seek(a, offsets, f0);
  RouteCursor cc = ic;  // compute cursor
  // Stage i holds pages [i*RPS, min((i+1)*RPS, count)) of this warp's share.
  // Lane 0 looks the slots of the next stage to issue up one iteration
  // early, so the page-table reads overlap the current stage's arithmetic.
  auto stage_pages = [&](int i) { return min(RPS, count - i * RPS); };
  int nslot[RPS];
  auto lookup = [&](int cnt) {
    RouteCursor c = ic;
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      nslot[k] = 0;
      if (k < cnt) {
        nslot[k] = __ldg(a.page_table + (size_t)c.b * a.ld_pt + c.j);
        c.advance(a);
      }
    }
  };
  // stage i goes to ring position s (= i mod S, tracked by the caller)
  auto issue = [&](int i, int s) {
    const int cnt = stage_pages(i);
    uint64_t* bar = &bars[warp][s];
    uint8_t* dst = ring + (size_t)s * stage_bytes;
    if (skip_issue_for_test(wg, i)) {
      for (int k = 0; k < cnt; ++k) ic.advance(a);
      return;
    }
    mbar_arrive_expect_tx(bar, cnt * page_bytes);
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      if (k < cnt) {
        int slot = nslot[k];
        if (slot < 0 || slot >= a.num_slots) {
          atomicOr(a.status, kStatusBadSlot);
          slot = 0;
        }
        const size_t row0 = ((size_t)slot * a.num_kv_heads + ic.kvh) * P;
        bulk_load(dst + k * page_bytes, zpool + row0 * RR, zbytes, bar, pol);
        if (RS > 0) bulk_load(dst + k * page_bytes + zbytes, rpool + row0 * RS, rbytes, bar, pol);
        ic.advance(a);
      }
    }
  };
  {
    // the first S stages: lane j looks page j up (all reads in parallel),
    // lane 0 issues
    const int first = min(S * RPS, count);
    int sl = 0;
    if (lane < first) {
      RouteCursor c = ic;
      for (int k = 0; k < lane; ++k) c.advance(a);
      sl = __ldg(a.page_table + (size_t)c.b * a.ld_pt + c.j);
    }
    for (int i = 0; i < S && i < nst; ++i) {
#pragma unroll
      for (int k = 0; k < RPS; ++k) nslot[k] = __shfl_sync(0xffffffffu, sl, (i * RPS + k) & 31);
      if (lane == 0) issue(i, i);
    }
  }
  pdl_launch_dependents();

  // route-prep spread over the warps: task (unit, slice) -> warp task mod W;
  // each writes its rows of the folded query and tags them with the call
  constexpr int NSL = (RR + RS + 32 / G - 1) / (32 / G);
  static_assert(NSL <= 32, "fold slices per unit must fit a warp");
  const int U = a.batch * a.num_kv_heads;
  for (int task = wg; task < U * NSL; task += W) {
    const int u = task / NSL;
    const int n = (a.seq_lens[u / a.num_kv_heads] + P - 1) / P;
    if (n == 0 || !(a.force || a.topk < n)) continue;
    if (a.head_dim == 128) fold_slice<G, RR, RS, 4>(a, u, task % NSL);
    else fold_slice<G, RR, RS, 2>(a, u, task % NSL);
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      *reinterpret_cast<volatile uint32_t*>(a.fold_flag + (size_t)u * 32 + task % NSL) = a.tag;
    }
  }
  if (count <= 0) return;

  constexpr int FR = NT * (2 * Shape::ZB + Shape::Z8 + 2 * Shape::SB + Shape::S8);
  uint32_t fr[FR];
  int cur_u = -1;

  bool ok = true;
  int i = 0;
  int s_i = 0;        // ring position of stage i (i mod S)
  uint32_t ph_i = 0;  // phase parity of that position's barrier for stage i
  for (; i < nst; ++i) {
    if (lane == 0 && i + S < nst) lookup(stage_pages(i + S));
    ok = mbar_wait(&bars[warp][s_i], ph_i, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const int cnt = stage_pages(i);
    const uint8_t* stage = ring + (size_t)s_i * stage_bytes;
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      if (k < cnt) {
        const int u = cc.unit(a);
        if (u != cur_u) {
          // this unit's folded query: its slices come from other warps; should
          // they be late (their CTA not yet resident), fold it here instead
          cur_u = u;
          bool ready = true;
          if (lane < NSL) ready = wait_tag(a.fold_flag + (size_t)u * 32 + lane, a.tag, kFoldWaitNs);
          if (__all_sync(0xffffffffu, ready)) {
            load_route_frags<G, RR, RS, FR>(a.qf + (size_t)u * G * (RR + RS), fr);
          } else if (a.head_dim == 128) {
            warp_fold_query<G, RR, RS, FR, 4>(a, cc.b, cc.kvh, qsm, fr);
          } else {
            warp_fold_query<G, RR, RS, FR, 2>(a, cc.b, cc.kvh, qsm, fr);
          }
        }
        const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(stage + k * page_bytes);
        const float best = route_page_score<G, RR, RS, P, FR>(zs, zs + P * RR, min(P, cc.L - cc.j * P), fr);
        if (lane == 0) a.scores[(size_t)cur_u * a.ld_pt + cc.j] = best;
        cc.advance(a);
      }
    }
    __syncwarp();
    if (lane == 0 && i + S < nst) issue(i + S, s_i);  // (i + S) mod S = i mod S
    if (++s_i == S) {
      s_i = 0;
      ph_i ^= 1u;
    }
  }
  if (!ok) {
    if (lane == 0)  // drain the copies still in flight, stages [i, min(i + S, nst))
      for (int j = i; j < nst && j < i + S; ++j)
        mbar_wait(&bars[warp][j % S], (uint32_t)((j / S) & 1), a.status);
  }
}

// ---------------------------------------------------------------------------
// CUDA-core routing for any shape and for fp32 pools: thread per (token,
// head) pair, rows read straight from global memory.
template <typename T>
__global__ void __launch_bounds__(kRouteThreads) route_generic_kernel(const __grid_constant__ RouteArgs a) {
  pdl_launch_dependents();
  const RouteUnit ru = route_unit(a);
  if (a.fill_tail && blockIdx.x == 0)
    for (int j = ru.n + threadIdx.x; j < a.ld_pt; j += blockDim.x)
      a.scores[(size_t)ru.u * a.ld_pt + j] = -INFINITY;
  if (!ru.active) return;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ TopkSmem tk;
  __shared__ int flag;
  __shared__ float red[kRouteWarps];
  const int G = a.gqa_group, r = a.rank_r, s = a.rank_s, P = a.page_size;
  float* qs = reinterpret_cast<float*>(smem);
  float* qz = qs + G * a.head_dim;
  float* qr = qz + G * r;
  route_prep<T>(a, ru, qs, qz, qr);

  const T* zpool = static_cast<const T*>(a.z_pool);
  const T* rpool = static_cast<const T*>(a.r_pool);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int p = ru.first; p < ru.last; ++p) {
    int slot = a.page_table[(size_t)ru.b * a.ld_pt + p];
    if (slot < 0 || slot >= a.num_slots) {
      if (threadIdx.x == 0) atomicOr(a.status, kStatusBadSlot);
      slot = 0;
    }
    const size_t row0 = ((size_t)slot * a.num_kv_heads + ru.kvh) * P;
    const int valid = min(P, ru.L - p * P);
    float best = -INFINITY;
    for (int idx = threadIdx.x; idx < valid * G; idx += blockDim.x) {
      const int tok = idx / G, h = idx % G;
      const T* zr = zpool + (row0 + tok) * r;
      float u = 0.f;
      for (int i = 0; i < r; ++i) u = fmaf(to_f32(zr[i]), qz[h * r + i], u);
      if (s > 0) {
        const T* rr = rpool + (row0 + tok) * s;
        for (int i = 0; i < s; ++i) u = fmaf(to_f32(rr[i]), qr[h * s + i], u);
      }
      best = fmaxf(best, u);
    }
    best = warp_max(best);
    if (lane == 0) red[warp] = best;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = red[0];
      for (int w = 1; w < kRouteWarps; ++w) m = fmaxf(m, red[w]);
      a.scores[(size_t)ru.u * a.ld_pt + p] = m;
    }
    __syncthreads();
  }
  route_finish<kRouteThreads>(a, ru, tk, &flag);
}

}  // namespace basiskv
