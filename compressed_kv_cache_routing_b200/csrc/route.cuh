// Page routing for BasisKV decode attention ("the compressed Value cache is
// further reused to help identify which Key pages should be accessed: it
// predicts part of the Key information needed for routing, while a
// Key-specific residual stores what cannot be recovered from Value").
//
// Routing key  Khat_t = Z_t.W_zk + R_t.B_r  is never formed: the kernels fold
// the bases into the query once per CTA (route-prep),
//     qz_h = W_zk.q_h  (r floats),   qr_h = B_r.q_h  (s floats),
// so that  q_h.Khat_t = Z_t.qz_h + R_t.qr_h  costs r + s multiply-adds per
// token and head and reads only the r + s stored values of each token.
// Page score S_j = max over the G heads and page j's valid tokens; the last
// CTA of each (sequence, KV head) runs the top-k over the page scores.
//
// Grid: (chunks of pages, Hkv, batch); each CTA owns pages
// [chunk*ppc, min((chunk+1)*ppc, n_b)) of one (sequence, KV head).
#pragma once

#include "common.cuh"
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
};

constexpr int kRouteThreads = 128;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kMaxStages = 8;

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
// Pages stream through per-warp rings of `stages` shared buffers filled by
// bulk copies (cp.async.bulk, L2 evict-first) completing on mbarriers; each
// warp owns pages first+w, first+w+4, ... of the CTA.
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

template <int G, int RR, int RS>
__global__ void __launch_bounds__(kRouteThreads) route_mma_kernel(const RouteArgs a) {
  using Shape = RouteMma<G, RR, RS>;
  constexpr int NT = Shape::NT;
  pdl_launch_dependents();
  const RouteUnit ru = route_unit(a);
  if (a.fill_tail && blockIdx.x == 0)
    for (int j = ru.n + threadIdx.x; j < a.ld_pt; j += blockDim.x)
      a.scores[(size_t)ru.u * a.ld_pt + j] = -INFINITY;
  if (!ru.active) return;

  const int P = a.page_size;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t zbytes = (uint32_t)P * RR * 2, rbytes = (uint32_t)P * RS * 2;
  const uint32_t stage_bytes = zbytes + rbytes;
  const int S = a.stages;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[kRouteWarps][kMaxStages];
  __shared__ TopkSmem tk;
  __shared__ int flag;
  uint8_t* ring = smem + (size_t)warp * S * stage_bytes;
  float* qs = reinterpret_cast<float*>(smem + (size_t)kRouteWarps * S * stage_bytes);
  float* qz = qs + G * a.head_dim;
  float* qr = qz + G * RR;

  const int npg = ru.last - ru.first;
  const int mine = npg > warp ? (npg - warp + kRouteWarps - 1) / kRouteWarps : 0;
  const __nv_bfloat16* zpool = static_cast<const __nv_bfloat16*>(a.z_pool);
  const __nv_bfloat16* rpool = static_cast<const __nv_bfloat16*>(a.r_pool);
  const int32_t* ptab = a.page_table + (size_t)ru.b * a.ld_pt;
  uint64_t pol = policy_evict_first();

  auto issue = [&](int i) {  // lane 0 only: my i-th page into stage i % S
    const int p = ru.first + warp + i * kRouteWarps;
    int slot = ptab[p];
    if (slot < 0 || slot >= a.num_slots) {
      atomicOr(a.status, kStatusBadSlot);
      slot = 0;
    }
    const size_t row0 = ((size_t)slot * a.num_kv_heads + ru.kvh) * P;
    uint64_t* bar = &bars[warp][i % S];
    uint8_t* dst = ring + (size_t)(i % S) * stage_bytes;
    mbar_arrive_expect_tx(bar, stage_bytes);
    bulk_load(dst, zpool + row0 * RR, zbytes, bar, pol);
    if (RS > 0) bulk_load(dst + zbytes, rpool + row0 * RS, rbytes, bar, pol);
  };

  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[warp][i], 1);
    mbar_init_fence();
    for (int i = 0; i < S && i < mine; ++i) issue(i);
  }
  __syncwarp();

  route_prep<__nv_bfloat16>(a, ru, qs, qz, qr);

  // B fragments of the split query: column n = 8j + g -> head 4j + g/2,
  // hi (g even) or lo (g odd) half.
  uint32_t bz[NT][Shape::ZB > 0 ? Shape::ZB : 1][2];
  uint32_t bz8[NT];
  uint32_t bs[NT][Shape::SB > 0 ? Shape::SB : 1][2];
  uint32_t bs8[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    const int h = 4 * j + (g >> 1);
    const bool lo = g & 1;
    auto part = [&](const float* v, int idx) {
      if (h >= G) return 0.f;
      float hi, lw;
      split_bf16(v[idx], hi, lw);
      return lo ? lw : hi;
    };
    const float* qzh = qz + h * RR;
    const float* qrh = qr + h * RS;
#pragma unroll
    for (int blk = 0; blk < Shape::ZB; ++blk) {
      const int e0 = k16_phys<Shape::Z32, Shape::Z16>(blk, t, 0);
      const int e1 = k16_phys<Shape::Z32, Shape::Z16>(blk, t, 1);
      bz[j][blk][0] = pack_bf16(part(qzh, e0), part(qzh, e0 + 1));
      bz[j][blk][1] = pack_bf16(part(qzh, e1), part(qzh, e1 + 1));
    }
    if (Shape::Z8) {
      const int e = 32 * Shape::Z32 + 16 * Shape::Z16 + 2 * t;
      bz8[j] = pack_bf16(part(qzh, e), part(qzh, e + 1));
    }
#pragma unroll
    for (int blk = 0; blk < Shape::SB; ++blk) {
      const int e0 = k16_phys<Shape::S32, Shape::S16>(blk, t, 0);
      const int e1 = k16_phys<Shape::S32, Shape::S16>(blk, t, 1);
      bs[j][blk][0] = pack_bf16(part(qrh, e0), part(qrh, e0 + 1));
      bs[j][blk][1] = pack_bf16(part(qrh, e1), part(qrh, e1 + 1));
    }
    if (Shape::S8) {
      const int e = 32 * Shape::S32 + 16 * Shape::S16 + 2 * t;
      bs8[j] = pack_bf16(part(qrh, e), part(qrh, e + 1));
    }
  }

  float* scores = a.scores + (size_t)ru.u * a.ld_pt;
  bool ok = true;
  int i = 0;
  for (; i < mine; ++i) {
    const int p = ru.first + warp + i * kRouteWarps;
    ok = mbar_wait(&bars[warp][i % S], (uint32_t)((i / S) & 1), a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(ring + (size_t)(i % S) * stage_bytes);
    const __nv_bfloat16* rs = zs + P * RR;
    const int valid = min(P, ru.L - p * P);
    float best = -INFINITY;
    for (int mt = 0; mt * 16 < valid; ++mt) {
      float acc[NT][4];
#pragma unroll
      for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      const __nv_bfloat16* z0 = zs + (mt * 16 + g) * RR;
      const __nv_bfloat16* z1 = z0 + 8 * RR;
#pragma unroll
      for (int sp = 0; sp < Shape::Z32; ++sp) {
        const uint4 v0 = lds128(z0 + 32 * sp + 8 * t), v1 = lds128(z1 + 32 * sp + 8 * t);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, bz[j][2 * sp][0], bz[j][2 * sp][1]);
          mma_k16(acc[j], v0.z, v1.z, v0.w, v1.w, bz[j][2 * sp + 1][0], bz[j][2 * sp + 1][1]);
        }
      }
      if (Shape::Z16) {
        const uint2 v0 = lds64(z0 + 32 * Shape::Z32 + 4 * t), v1 = lds64(z1 + 32 * Shape::Z32 + 4 * t);
#pragma unroll
        for (int j = 0; j < NT; ++j)
          mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, bz[j][Shape::ZB - 1][0], bz[j][Shape::ZB - 1][1]);
      }
      if (Shape::Z8) {
        const int o = 32 * Shape::Z32 + 16 * Shape::Z16 + 2 * t;
        const uint32_t v0 = lds32(z0 + o), v1 = lds32(z1 + o);
#pragma unroll
        for (int j = 0; j < NT; ++j) mma_k8(acc[j], v0, v1, bz8[j]);
      }
      if (RS > 0) {
        const __nv_bfloat16* r0 = rs + (mt * 16 + g) * RS;
        const __nv_bfloat16* r1 = r0 + 8 * RS;
#pragma unroll
        for (int sp = 0; sp < Shape::S32; ++sp) {
          const uint4 v0 = lds128(r0 + 32 * sp + 8 * t), v1 = lds128(r1 + 32 * sp + 8 * t);
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, bs[j][2 * sp][0], bs[j][2 * sp][1]);
            mma_k16(acc[j], v0.z, v1.z, v0.w, v1.w, bs[j][2 * sp + 1][0], bs[j][2 * sp + 1][1]);
          }
        }
        if (Shape::S16) {
          const uint2 v0 = lds64(r0 + 32 * Shape::S32 + 4 * t), v1 = lds64(r1 + 32 * Shape::S32 + 4 * t);
#pragma unroll
          for (int j = 0; j < NT; ++j)
            mma_k16(acc[j], v0.x, v1.x, v0.y, v1.y, bs[j][Shape::SB - 1][0], bs[j][Shape::SB - 1][1]);
        }
        if (Shape::S8) {
          const int o = 32 * Shape::S32 + 16 * Shape::S16 + 2 * t;
          const uint32_t v0 = lds32(r0 + o), v1 = lds32(r1 + o);
#pragma unroll
          for (int j = 0; j < NT; ++j) mma_k8(acc[j], v0, v1, bs8[j]);
        }
      }
      // D fragment: rows g, g+8 = tokens; columns 2t, 2t+1 = (hi, lo) of head 4j + t
      const int tok0 = mt * 16 + g, tok1 = tok0 + 8;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (4 * j + t < G) {
          if (tok0 < valid) best = fmaxf(best, acc[j][0] + acc[j][1]);
          if (tok1 < valid) best = fmaxf(best, acc[j][2] + acc[j][3]);
        }
      }
    }
    best = warp_max(best);
    __syncwarp();
    if (lane == 0) {
      scores[p] = best;
      if (i + S < mine) issue(i + S);
    }
  }
  if (!ok && lane == 0) {
    // a copy never completed: wait (bounded) for the pages still in flight,
    // [i, min(i + S, mine)), before the CTA's shared memory is released
    for (int j = i; j < mine && j < i + S; ++j)
      mbar_wait(&bars[warp][j % S], (uint32_t)((j / S) & 1), a.status);
  }
  route_finish<kRouteThreads>(a, ru, tk, &flag);
}

// ---------------------------------------------------------------------------
// CUDA-core routing for any shape and for fp32 pools: thread per (token,
// head) pair, rows read straight from global memory.
template <typename T>
__global__ void __launch_bounds__(kRouteThreads) route_generic_kernel(const RouteArgs a) {
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
