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
// Two kernels: route_mma_kernel (bf16 pools, tensor cores, persistent over
// a flat page list handed out as static shares plus chunks claimed at run
// time; the fold is spread over all warps as (unit, row slice) tasks whose
// results are written to global memory tagged with the call, and a warp
// entering a unit reads them back, folding locally only if they are late;
// the selection runs in the next grid) and route_generic_kernel (any
// dtype, grid (chunks of pages, Hkv, batch), fold once per CTA, the last
// CTA of each (sequence, KV head) runs the top-k).
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
  uint64_t* scores64;       // [B][Hkv][ld_pt] (tag << 32) | fp32 bits, when tagged_scores
  int tagged_scores;        // persistent kernel: write scores64 instead of scores
  int32_t* sel;             // [B][Hkv][ld_sel]
  int32_t* sel_out;         // [B][Hkv][topk] or null
  uint32_t* counters;       // [B][Hkv]
  uint32_t* sched;          // [2] chunk claims, finished warps (persistent kernel; zero between calls)
  uint32_t* status;
  int ld_pt, ld_sel, num_slots, num_kv_heads, head_dim, page_size;
  int rank_r, rank_s, gqa_group;
  int topk, pages_per_cta, stages;
  int static_pct;           // persistent kernel: percent of the pages handed out in static shares
  int force;                // route units whose every page would be selected
  int fill_tail;            // chunk 0 writes -inf to scores[n_b .. ld_pt)
  // persistent tensor-core kernel only
  int batch;
  const int32_t* route_off; // [B+1] prefix of routed pages x Hkv (from the prep grid)
  uint64_t* qf;             // [B*Hkv][G][r+s] folded queries: (tag << 32) | fp32 bits
  uint32_t tag;             // this call's tag (never 0)
  int plan_n;               // >= 0: plan_off holds route_off (batch <= kPlanMax)
  int32_t plan_off[kPlanMax + 1];
};

constexpr int kRouteThreads = 128;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kMaxStages = 8;
constexpr int kRouteChunkStages = 2;  // stages per claimed chunk of the persistent kernel

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
// Persistent: every warp streams chunks of the flat list of routed pages
// (sequence-major, then KV head, then page), claimed from a grid-wide
// counter, through its own ring of `stages` shared buffers filled by bulk
// copies (cp.async.bulk, L2 evict-first) completing on mbarriers, and writes
// one score per page (tagged with the call, so the selection grid can take
// a unit as soon as its pages are scored).  The selection runs in the next
// grid (topk_kernel).
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
  // sequence b's page count from the plan (its routed pages x Hkv), so the
  // page-table address never waits for the length, which is read beside it
  __device__ __forceinline__ void load(const RouteArgs& a) {
    n = (off[b + 1] - off[b]) / a.num_kv_heads;
    L = a.seq_lens[b];
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
    for (++b; b < a.batch; ++b)
      if (off[b + 1] > off[b]) {  // a routed sequence
        load(a);
        return;
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
template <int G>
struct FoldIn {
  float qv[G][4];       // this lane's query channels (d/32 of 4 used)
  float w[32 / G][4];   // this lane's channels of the slice's basis rows
};

template <int G, int RR, int RS, int CPL>
__device__ __forceinline__ void fold_load(const RouteArgs& a, int u, int slice, FoldIn<G>& in) {
  constexpr int RPB = 32 / G, ROWS = RR + RS, d = 32 * CPL;
  const int lane = threadIdx.x & 31;
  const int kvh = u % a.num_kv_heads;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + (size_t)u * G * d + lane * CPL;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if constexpr (CPL == 4) {
      const uint2 x = __ldg(reinterpret_cast<const uint2*>(q + h * d));
      in.qv[h][0] = __uint_as_float(x.x << 16);
      in.qv[h][1] = __uint_as_float(x.x & 0xffff0000u);
      in.qv[h][2] = __uint_as_float(x.y << 16);
      in.qv[h][3] = __uint_as_float(x.y & 0xffff0000u);
    } else {
      const uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(q + h * d));
      in.qv[h][0] = __uint_as_float(x << 16);
      in.qv[h][1] = __uint_as_float(x & 0xffff0000u);
    }
  }
  const int row0 = slice * RPB;
#pragma unroll
  for (int rl = 0; rl < RPB; ++rl) {
    const int row = row0 + rl;
    const float* src = row < RR ? a.w_zk + ((size_t)kvh * RR + row) * d
                                : a.b_r + ((size_t)kvh * RS + (row - RR)) * d;
    src += lane * CPL;
    if constexpr (CPL == 4) {
      const float4 x = row < ROWS ? __ldg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
      in.w[rl][0] = x.x;
      in.w[rl][1] = x.y;
      in.w[rl][2] = x.z;
      in.w[rl][3] = x.w;
    } else {
      const float2 x = row < ROWS ? __ldg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
      in.w[rl][0] = x.x;
      in.w[rl][1] = x.y;
    }
  }
}

// The slice's sums, stored tagged with the call: word (u, h, row) of qf is
// (tag << 32) | bits of the float, written by one 8-byte relaxed store, so a
// reader that sees the tag sees the value (no fence, no flag).
template <int G, int RR, int RS, int CPL>
__device__ __forceinline__ void fold_store(const RouteArgs& a, int u, int slice, const FoldIn<G>& in) {
  constexpr int RPB = 32 / G, ROWS = RR + RS;
  const int lane = threadIdx.x & 31;
  float v[32];
#pragma unroll
  for (int rl = 0; rl < RPB; ++rl)
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < CPL; ++j) acc = fmaf(in.w[rl][j], in.qv[h][j], acc);
      v[rl * G + h] = acc;
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
  const int row = slice * RPB + lane / G, h = lane % G;
  if (row < ROWS)
    st_relaxed_u64(a.qf + ((size_t)u * G + h) * ROWS + row, ((uint64_t)a.tag << 32) | __float_as_uint(v[0]));
}

// This lane's routing B-fragment words for unit u from the tagged folded
// query (split into bf16 hi + lo columns; same order as route_mma_kernel).
// Returns false when a word does not carry this call's tag yet.
template <int G, int RR, int RS, int FR>
__device__ bool load_route_frags(const uint64_t* qfu, uint32_t tag, uint32_t (&fr)[FR]) {
  using Shape = RouteMma<G, RR, RS>;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  bool ready = true;
  int w = 0;
#pragma unroll
  for (int j = 0; j < Shape::NT; ++j) {
    const int hh = 4 * j + (g >> 1);
    const bool lo = g & 1;
    const uint64_t* qz = qfu + hh * (RR + RS);
    const uint64_t* qr = qz + RR;
    auto word = [&](const uint64_t* src, int e) {
      if (hh >= G) return 0u;
      uint64_t x0, x1;
      ld_relaxed_v2u64(src + e, x0, x1);
      ready = ready && (uint32_t)(x0 >> 32) == tag && (uint32_t)(x1 >> 32) == tag;
      float h0, l0, h1, l1;
      split_bf16(__uint_as_float((uint32_t)x0), h0, l0);
      split_bf16(__uint_as_float((uint32_t)x1), h1, l1);
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
  return ready;
}

// Stage bookkeeping of route_mma_kernel: the position of a stage's first
// page (sequence b, KV head, page j, length L of sequence b) and its page
// count, written by the issuing lane next to the copies.
struct RouteStageMeta {
  int b, kvh_cnt, j, L;  // kvh_cnt = kvh | pages << 16
};

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
  __shared__ RouteStageMeta smeta[kRouteWarps][kMaxStages];
  __shared__ float qsm_all[kRouteWarps][G * (RR + RS)];
  float* qsm = qsm_all[warp];
  uint8_t* ring = smem + (size_t)warp * S * stage_bytes;
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[warp][i], 1);
    mbar_init_fence();
  }
  __syncwarp();
  // The plan comes in the parameters (small batches) or from the prep grid
  // (then this grid waits for it first).
  const int32_t* offsets = a.plan_n >= 0 ? a.plan_off : a.route_off;
  if (a.plan_n < 0) pdl_wait_primary();

  // Work: the first Ts pages of the flat list go to the warps in equal
  // contiguous shares; the rest is cut into chunks of CP pages that warps
  // done with their share claim from a grid-wide counter, so the warps the
  // memory system serves faster take more of it and all finish close
  // together.  Scores land at fixed places: the order changes no result.
  constexpr int CP = RPS * kRouteChunkStages;
  const int W = gridDim.x * kRouteWarps, wg = blockIdx.x * kRouteWarps + warp;
  const int T = offsets[a.batch];
  const int Ts = (int)((long long)T * a.static_pct / 100);
  const int ndyn = (T - Ts + CP - 1) / CP;

  // Route-prep first: tasks (unit, slice) -> warp task mod W, each writing
  // its rows of the folded query tagged with the call.  Done before any page
  // copy is queued, their reads do not wait behind the copies (a warp with
  // tasks starts streaming a little later; the claimed chunks even it out).
  constexpr int NSL = (RR + RS + 32 / G - 1) / (32 / G);
  static_assert(NSL <= 32, "fold slices per unit must fit a warp");
  const int U = a.batch * a.num_kv_heads;
  auto task_routed = [&](int task) {
    const int b = task / NSL / a.num_kv_heads;
    return offsets[b + 1] > offsets[b];
  };
  for (int task = wg; task < U * NSL; task += W) {
    if (!task_routed(task)) continue;
    FoldIn<G> fin;
    if (a.head_dim == 128) {
      fold_load<G, RR, RS, 4>(a, task / NSL, task % NSL, fin);
      fold_store<G, RR, RS, 4>(a, task / NSL, task % NSL, fin);
    } else {
      fold_load<G, RR, RS, 2>(a, task / NSL, task % NSL, fin);
      fold_store<G, RR, RS, 2>(a, task / NSL, task % NSL, fin);
    }
  }

  const __nv_bfloat16* zpool = static_cast<const __nv_bfloat16*>(a.z_pool);
  const __nv_bfloat16* rpool = static_cast<const __nv_bfloat16*>(a.r_pool);
  const uint64_t pol = policy_evict_first();
  // Lane 0 runs the issue side: it looks the next stage up one iteration
  // before issuing it (the page-table reads overlap the current stage's
  // arithmetic) and claims the next chunk when it looks up the last stage
  // of the current piece of work, one iteration before it needs it.
  RouteCursor ic;                                      // lane 0: next page to look up
  int lk_flat = (int)((long long)Ts * wg / W);         // its flat index
  int lk_end = (int)((long long)Ts * (wg + 1) / W);    // end of the current piece
  int nxt = 0;                                         // the claimed dynamic chunk
  int nslot[RPS], nkvh[RPS];
  RouteStageMeta nmeta;  // the looked-up stage (pages 0: none)
  nmeta.kvh_cnt = 0;
  if (lane == 0) {
    if (lk_flat < lk_end) ic.seek(a, offsets, lk_flat);
    else nxt = (int)atomicAdd(a.sched, 1u);  // no static share
  }
  auto lookup = [&]() {
    nmeta.kvh_cnt = 0;
    if (lk_flat == lk_end) {
      if (nxt >= ndyn) return;
      lk_flat = Ts + nxt * CP;
      lk_end = min(T, lk_flat + CP);
      ic.seek(a, offsets, lk_flat);
    }
    const int cnt = min(RPS, lk_end - lk_flat);
    nmeta.b = ic.b;
    nmeta.kvh_cnt = ic.kvh | (cnt << 16);
    nmeta.j = ic.j;
    nmeta.L = ic.L;
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      nslot[k] = 0;
      nkvh[k] = 0;
      if (k < cnt) {
        nslot[k] = __ldg(a.page_table + (size_t)ic.b * a.ld_pt + ic.j);
        nkvh[k] = ic.kvh;
        ic.advance(a);
      }
    }
    lk_flat += cnt;
    if (lk_flat == lk_end) nxt = (int)atomicAdd(a.sched, 1u);  // the piece after this one
  };
  // issue the looked-up stage, the i-th of this warp, into ring position s
  auto issue = [&](int i, int s) {
    const int cnt = nmeta.kvh_cnt >> 16;
    uint64_t* bar = &bars[warp][s];
    uint8_t* dst = ring + (size_t)s * stage_bytes;
    smeta[warp][s] = nmeta;
    if (skip_issue_for_test(wg, i)) return;
    mbar_arrive_expect_tx(bar, cnt * page_bytes);
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      if (k < cnt) {
        int slot = nslot[k];
        if (slot < 0 || slot >= a.num_slots) {
          atomicOr(a.status, kStatusBadSlot);
          slot = 0;
        }
        const size_t row0 = BASISKV_DEBUG_INDEX(((long long)slot * a.num_kv_heads + nkvh[k]) * P,
                                                (long long)a.num_slots * a.num_kv_heads * P, a.status);
        bulk_load(dst + k * page_bytes, zpool + row0 * RR, zbytes, bar, pol);
        if (RS > 0) bulk_load(dst + k * page_bytes + zbytes, rpool + row0 * RS, rbytes, bar, pol);
      }
    }
  };
  int nissued = 0;  // stages issued by this warp (uniform)
  {
    // the first stages of the static share: lane k looks page k up (all
    // page-table reads in flight together), lane 0 issues
    const int first = min(min(S * RPS, 32), lk_end - lk_flat);
    int sl = 0;
    RouteStageMeta m;
    m.b = m.kvh_cnt = m.j = m.L = 0;
    if (lane < first) {
      RouteCursor c;
      c.seek(a, offsets, lk_flat);
      for (int k = 0; k < lane; ++k) c.advance(a);
      sl = __ldg(a.page_table + (size_t)c.b * a.ld_pt + c.j);
      m.b = c.b;
      m.kvh_cnt = c.kvh;
      m.j = c.j;
      m.L = c.L;
    }
    for (int s = 0; s * RPS < first; ++s) {
      const int cnt = min(RPS, first - s * RPS);
      RouteStageMeta ms;
      ms.b = __shfl_sync(0xffffffffu, m.b, s * RPS);
      ms.kvh_cnt = __shfl_sync(0xffffffffu, m.kvh_cnt, s * RPS) | (cnt << 16);
      ms.j = __shfl_sync(0xffffffffu, m.j, s * RPS);
      ms.L = __shfl_sync(0xffffffffu, m.L, s * RPS);
#pragma unroll
      for (int k = 0; k < RPS; ++k) {
        const int src = min(s * RPS + k, 31);
        nslot[k] = __shfl_sync(0xffffffffu, sl, src);
        nkvh[k] = __shfl_sync(0xffffffffu, m.kvh_cnt, src);
      }
      if (lane == 0) {
        nmeta = ms;
        issue(nissued, s);
      }
      ++nissued;
    }
    if (lane == 0) {
      for (int k = 0; k < first; ++k) ic.advance(a);
      lk_flat += first;
      if (first > 0 && lk_flat == lk_end) nxt = (int)atomicAdd(a.sched, 1u);
      for (int s = nissued; s < S; ++s) {
        lookup();
        if (nmeta.kvh_cnt == 0) break;
        issue(nissued, s);
        ++nissued;
      }
      nmeta.kvh_cnt = 0;
    }
  }
  nissued = __shfl_sync(0xffffffffu, nissued, 0);
  pdl_launch_dependents();


  constexpr int FR = NT * (2 * Shape::ZB + Shape::Z8 + 2 * Shape::SB + Shape::S8);
  uint32_t fr[FR];
  int cur_u = -1;
  RouteCursor cc;  // compute cursor, set from each stage's bookkeeping
  cc.off = offsets;  // (it steps across sequences within a stage)

  bool ok = true;
  int i = 0;
  int s_i = 0;        // ring position of stage i (i mod S)
  uint32_t ph_i = 0;  // phase parity of that position's barrier for stage i
  for (; i < nissued; ++i) {
    if (lane == 0) lookup();  // the stage to issue at the end of this iteration
    ok = mbar_wait(&bars[warp][s_i], ph_i, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const RouteStageMeta m = smeta[warp][s_i];
    const int cnt = m.kvh_cnt >> 16;
    cc.b = m.b;
    cc.kvh = m.kvh_cnt & 0xffff;
    cc.j = m.j;
    cc.L = m.L;
    cc.n = (m.L + P - 1) / P;
    const uint8_t* stage = ring + (size_t)s_i * stage_bytes;
#pragma unroll
    for (int k = 0; k < RPS; ++k) {
      if (k < cnt) {
        const int u = cc.unit(a);
        if (u != cur_u) {
          // this unit's folded query comes from other warps; should it be
          // late (their CTA not yet resident), fold it here instead
          cur_u = u;
          const uint64_t* qfu = a.qf + (size_t)u * G * (RR + RS);
          bool ready = __all_sync(0xffffffffu, load_route_frags<G, RR, RS, FR>(qfu, a.tag, fr));
          if (!ready) {
            const uint64_t t0 = global_timer_ns();
            uint32_t pause = 64;
            while (!ready && global_timer_ns() - t0 < kFoldWaitNs) {
              __nanosleep(pause);
              pause = pause < 1024u ? 2 * pause : 1024u;
              ready = __all_sync(0xffffffffu, load_route_frags<G, RR, RS, FR>(qfu, a.tag, fr));
            }
          }
          if (!ready) {
            if (a.head_dim == 128) warp_fold_query<G, RR, RS, FR, 4>(a, cc.b, cc.kvh, qsm, fr);
            else warp_fold_query<G, RR, RS, FR, 2>(a, cc.b, cc.kvh, qsm, fr);
          }
        }
        const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(stage + k * page_bytes);
        const float best = route_page_score<G, RR, RS, P, FR>(zs, zs + P * RR, min(P, cc.L - cc.j * P), fr);
        if (lane == 0) {
          const size_t e = BASISKV_DEBUG_INDEX((long long)cur_u * a.ld_pt + cc.j,
                                               (long long)a.batch * a.num_kv_heads * a.ld_pt, a.status);
          if (a.tagged_scores)
            st_relaxed_u64(a.scores64 + e,
                           ((uint64_t)a.tag << 32) | __float_as_uint(best));
          else
            a.scores[e] = best;
        }
        cc.advance(a);
      }
    }
    __syncwarp();
    if (lane == 0 && nmeta.kvh_cnt != 0) {
      issue(nissued, s_i);  // stage nissued = i + S goes where stage i was
      ++nissued;
    }
    nissued = __shfl_sync(0xffffffffu, nissued, 0);
    if (++s_i == S) {
      s_i = 0;
      ph_i ^= 1u;
    }
  }
  if (!ok) {
    if (lane == 0)  // drain the copies still in flight, stages [i, nissued)
      for (int j = i; j < nissued; ++j) mbar_wait(&bars[warp][j % S], (uint32_t)((j / S) & 1), a.status);
  }
  // The last warp to finish resets the claim counter for the next call (a
  // warp's last claim has returned before it arrives here).
  if (lane == 0) {
    __threadfence();
    if (atomicAdd(a.sched + 1, 1u) == (uint32_t)W - 1) {
      a.sched[0] = 0u;
      a.sched[1] = 0u;
    }
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
