// Exact attention over the selected pages with a shared ring per CTA
// (BasisKV decode: "the original Keys are then retrieved only for the
// selected pages to compute exact QK scores"; values stay rank-r latents Z
// and the weighted latent is expanded by B_v at the end).
//
// attn_coop_kernel is persistent over the flat list of attention items
// (sequence-major, then KV head, selected entry, stage of the page), cut
// into chunks of chunk_items consecutive items: CTA c takes chunks c,
// c + gridDim.x, ... (one each as the host sizes them).  Its warps have
// four roles:
//  - the lookup warp looks items up 32 at a time, one per lane (selected
//    entry, then page-table slot), numbers the segments and queues the items
//    in shared memory;
//  - the issuing warp: lane j owns ring slot j and hands out the stages
//    j, j + NST, ...: it waits until the slot is free, writes the stage's
//    descriptor (unit, valid tokens, segment number) and starts the bulk
//    copies of TPS tokens of one selected page (K rows, Z rows and, for
//    int8 keys, the token scales);
//  - kCoopWarps consumer warps take the stages round-robin (stage n goes to
//    warp n mod kCoopWarps), so they share one deep ring and advance
//    together; a warp computes exact QK for its stage and the whole GQA
//    group, the online softmax and P.Z (attn_stage) into its own state;
//  - a segment is the run of one unit's items inside one chunk; at each
//    segment end every consumer warp leaves its state in a shared-memory
//    buffer (an empty state if none of the segment's stages was its) and
//    one of two merge warps (segments alternate between them) merges the
//    warp states in warp order; a unit inside one chunk is finished from
//    that state at once (B_v applied), otherwise the merge becomes the
//    segment's partial (slot = chunk index - the unit's first chunk), its
//    items are counted, and whoever completes the unit merges its partials
//    in slot order and applies B_v, while the consumers stream on.
// The partition into segments and every merge order follow from the
// chunking alone, so the results do not depend on timing.
#pragma once

#include "attn.cuh"

namespace basiskv {

// Ring stages: a multiple of kCoopWarps, so that stage n and stage n - NST
// of a slot belong to the same consumer warp (it has consumed the earlier one
// before it waits for the later, and a barrier's parity never aliases).
constexpr int kCoopMaxStages = 32;
constexpr int kCoopWarps = 8;   // consumer warps
// segment-state buffers between the consumers and the merge warp (fewer
// where one warp state is large)
__host__ __device__ constexpr int coop_bufs(int g, int rr) { return g * rr >= 256 ? 2 : 4; }
constexpr int kCoopMaxBufs = 4;
constexpr int kCoopLookQ = 64;  // looked-up items between the lookup warp and the issuing lanes
// Segment descriptors in flight: the lookup warp runs at most kCoopLookQ
// stages ahead of the issuing lanes, which run at most kCoopMaxStages ahead
// of the slowest consumer (plus one round of kCoopWarps), which runs at most
// kCoopMaxBufs segments ahead of the merge warps; a segment has a stage.
constexpr int kCoopSegs = 128;
constexpr int kCoopMergeWarps = 2;  // merge warps: segment f goes to merge warp f mod 2
constexpr int kCoopThreads = (kCoopWarps + 2 + kCoopMergeWarps) * 32;

// Descriptor of one staged item, written by the issuing warp before the
// copies are started (the barrier's completion makes it visible).
struct __align__(16) CoopMeta {
  int u;      // unit b * Hkv + kvh; -1 marks the end of the CTA's work
  int valid;  // tokens of the stage inside the sequence (<= 0: none)
  int sid;    // segment number within the CTA
  int pad;
};

// One looked-up item, passed from the lookup warp to the issuing lane of its
// stage through a shared-memory queue (seq = the stage number once filled).
struct __align__(16) CoopLook {
  unsigned long long row0;  // first pool row of the stage
  int u;                    // unit; -1: end marker stage; -2: no more stages for this lane
  int valid;                // tokens of the stage inside the sequence
  int sid;                  // segment number within the CTA
  uint32_t seq;
};

// Spin until *p == want (shared memory, bounded like mbar_wait; gives up
// when another warp has set *abort).
__device__ __forceinline__ bool poll_equal(const uint32_t* p, uint32_t want, uint32_t* status, volatile int* abort) {
  const volatile uint32_t* v = p;
  if (*v == want) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    __nanosleep(64);
    if (*v == want) return true;
    if ((it & 15u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(status, kStatusTimeout);
        *abort = 1;
        return false;
      }
    }
  }
}

// Descriptor of one segment, written by the lookup warp with the segment's
// first item, read by the merge warps.
struct __align__(16) CoopSeg {
  int u;          // unit; -1: no more segments
  int kvh;
  int slot;       // the segment's partial slot within its unit
  int seg_items;  // items of the segment
  int np;         // partial slots of the unit
  int nu;         // items of the unit
  int pad[2];
};


// Merge NW warp states of one segment (shared memory, [NW][MW] floats: the
// [G][RR] latent sum, then (m, l) per head) in warp order, into the
// MergeOut layout: every lane holds M, L of head lane % G and the float4
// slices v = lane + 32k of the [G][RR] sum.
template <int G, int RR, int NW>
__device__ __forceinline__ void merge_warp_states(const float* st, MergeOut<G, RR>& o) {
  constexpr int MW = G * RR + 16, V = MergeOut<G, RR>::V, VPL = MergeOut<G, RR>::VPL;
  const int lane = threadIdx.x & 31;
  const int hl = lane % G;
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) M = fmaxf(M, st[w * MW + G * RR + 2 * hl]);
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const float m = st[w * MW + G * RR + 2 * hl];
    if (m != -INFINITY) L = fmaf(exp2f(m - M), st[w * MW + G * RR + 2 * hl + 1], L);
  }
  o.M = M;
  o.L = L;
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    const int v = lane + 32 * k;
    const int h = min((4 * v) / RR, G - 1);
    const float Mh = __shfl_sync(0xffffffffu, M, h);
    float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
    if (v < V) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float m = st[w * MW + G * RR + 2 * h];
        const float wt = m == -INFINITY ? 0.f : exp2f(m - Mh);
        const float4 x = *reinterpret_cast<const float4*>(st + w * MW + 4 * v);
        s.x = fmaf(wt, x.x, s.x);
        s.y = fmaf(wt, x.y, s.y);
        s.z = fmaf(wt, x.z, s.z);
        s.w = fmaf(wt, x.w, s.w);
      }
    }
    o.acc[k] = s;
  }
}

// TS: the selection comes as tagged entries (sel64) from a selection grid
// that this grid does not wait for as a whole.
template <int G, int D, int RR, int TPS, bool K8 = false, bool TS = false>
__global__ void __launch_bounds__(kCoopThreads, 1) attn_coop_kernel(const __grid_constant__ AttnArgs a) {
  static_assert(G >= 1 && G <= 8, "GQA group must be 1..8");
  static_assert(D % 64 == 0 && RR % 8 == 0 && TPS % 16 == 0, "shape");
  constexpr int NW = kCoopWarps;
  constexpr int RT = RR / 8;
  constexpr int KB = K8 ? 1 : 2;
  constexpr uint32_t kbytes = TPS * D * KB, zbytes = TPS * RR * 2, sbytes = K8 ? TPS * 4 : 0;
  constexpr uint32_t stage_bytes = kbytes + zbytes + sbytes;
  constexpr int MW = G * RR + 16;  // floats of one warp's state: [G][RR] sum, then (m, l) per head
  constexpr int kCoopBufs = coop_bufs(G, RR);

  const int P = a.page_size, NST = a.stages;  // a multiple of NW
  const int sub = P / TPS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kCoopMaxStages], empty[kCoopMaxStages], mfull[kCoopMaxBufs], mempty[kCoopMaxBufs];
  __shared__ CoopMeta meta[kCoopMaxStages];
  __shared__ CoopSeg segs[kCoopSegs];
  __shared__ CoopLook lookq[kCoopLookQ];     // looked-up items, lookup warp -> issuing lanes
  __shared__ uint32_t lookd[kCoopLookQ];     // the stage whose entry each queue position last gave out
  __shared__ int abort_flag;
  uint8_t* ring = smem;
  float* mrg = reinterpret_cast<float*>(smem + (size_t)NST * stage_bytes);  // [kCoopBufs][NW][MW]
  float* zbar = mrg + kCoopBufs * NW * MW;                                  // [kCoopMergeWarps][G][RR]

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kCoopLookQ; ++i) lookq[i].seq = lookd[i] = 0xffffffffu;
    for (int i = 0; i < kCoopBufs; ++i) {
      mbar_init(&mfull[i], NW);
      mbar_init(&mempty[i], 1);
    }
    abort_flag = 0;
    mbar_init_fence();
  }
  __syncthreads();
  volatile int* abort = &abort_flag;

  if (warp == NW) {
    // ---- the lookup warp ---------------------------------------------------
    // the selection is written by the previous grid: wait for that grid, or,
    // with a tagged selection, for each unit's entries as they are looked up
    if constexpr (!TS) pdl_wait_primary();
    // the plan comes in the parameters, or from the prep grid, which
    // finished before the routing grid let this one launch
    const int32_t* offsets = a.plan_n >= 0 ? a.plan_off : a.attn_off;
    const long long T = offsets[a.batch];
    const long long CH = a.chunk_items > 0 ? a.chunk_items : max(1LL, (T + gridDim.x - 1) / gridDim.x);
    const long long nch = (T + CH - 1) / CH;
    uint32_t n = 0;  // next stage number (the same in every lane)
    int sid = -1;    // number of the last segment begun
    bool ok = true;
    // lane l waits until queue entry n + l is free, then fills it
    auto put = [&](uint32_t nn, const CoopLook& lk) -> bool {
      CoopLook* e = &lookq[nn % kCoopLookQ];
      if (nn >= (uint32_t)kCoopLookQ && !poll_equal(&lookd[nn % kCoopLookQ], nn - kCoopLookQ, a.status, abort))
        return false;
      e->row0 = lk.row0;
      e->u = lk.u;
      e->valid = lk.valid;
      e->sid = lk.sid;
      __threadfence_block();
      *reinterpret_cast<volatile uint32_t*>(&e->seq) = nn;
      return true;
    };
    for (long long c = blockIdx.x; ok && c < nch; c += gridDim.x) {
      const long long c0 = c * CH, c1 = min(T, c0 + CH);
      for (long long g0 = c0; ok && g0 < c1; g0 += 32) {
        const int n_in = (int)min(32LL, c1 - g0);
        // lane j looks up item g0 + j: its selected page and the page's slot
        CoopLook lk;
        bool new_seg = false;
        CoopSeg sg;
        if (lane < n_in) {
          // the item's place from the plan alone (sequence, KV head, selected
          // entry, stage), so that the length and the selected entry are
          // read together; the entry is used only where the unit is routed
          const int f = (int)(g0 + lane);
          int lo = 0, hi = a.batch;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (offsets[mid] <= f) lo = mid + 1;
            else hi = mid;
          }
          const int b = lo - 1;
          const int per_unit = (offsets[b + 1] - offsets[b]) / a.num_kv_heads;  // kb * sub
          const int rel = f - offsets[b];
          const int kvh = rel / per_unit, jj = (rel % per_unit) / sub, ts = (rel % per_unit) % sub;
          const int u = b * a.num_kv_heads + kvh;
          const size_t e = (size_t)u * a.ld_sel + jj;
          const int L = a.seq_lens[b];
          uint64_t w = TS ? ld_relaxed_u64(a.sel64 + e) : (uint64_t)(uint32_t)__ldcg(a.sel + e);
          const int n = (L + P - 1) / P;
          int page = jj;
          if (a.topk < n) {
            if (TS && (uint32_t)(w >> 32) != a.sel_tag) w = wait_selected(a.sel64 + e, a.sel_tag, a.status);
            page = (int)(uint32_t)w;
            if (page < 0 || page >= n) {
              atomicOr(a.status, kStatusBadPage);
              page = 0;
            }
          }
          int slot = __ldg(a.page_table + (size_t)b * a.ld_pt + page);
          if (slot < 0 || slot >= a.num_slots) {
            atomicOr(a.status, kStatusBadSlot);
            slot = 0;
          }
          const long long uo = offsets[b] + (long long)kvh * per_unit, nu = per_unit;
          lk.row0 = ((unsigned long long)slot * a.num_kv_heads + kvh) * P + (unsigned long long)ts * TPS;
          lk.u = u;
          lk.valid = L - (page * P + ts * TPS);
          new_seg = f == c0 || f == uo;
          sg.u = lk.u;
          sg.kvh = kvh;
          sg.slot = (int)(c - uo / CH);
          sg.seg_items = (int)(min(c1, uo + nu) - max(c0, uo));
          sg.np = (int)((uo + nu - 1) / CH - uo / CH + 1);
          sg.nu = (int)nu;
        }
        const unsigned starts = __ballot_sync(0xffffffffu, new_seg);
        lk.sid = sid + __popc(starts & (0xffffffffu >> (31 - lane)));
        bool lok = true;
        if (lane < n_in) {
          if (new_seg) segs[lk.sid % kCoopSegs] = sg;
          lok = put(n + lane, lk);
        }
        ok = __all_sync(0xffffffffu, lok);
        n += n_in;
        sid += __popc(starts);
      }
    }
    if (ok) {
      // the end: one closing segment number per merge warp, one stage without
      // copies for every consumer warp, and a stop for the other issuing lanes
      if (lane < kCoopMergeWarps) segs[(sid + 1 + lane) % kCoopSegs].u = -1;
      __syncwarp();
      if (lane < NST) {
        CoopLook lk;
        lk.row0 = 0;
        lk.u = lane < NW ? -1 : -2;
        lk.valid = 0;
        lk.sid = sid + 1;
        put(n + lane, lk);
      }
    }
    return;
  }

  if (warp == NW + 1) {
    // ---- the issuing warp: lane j hands out the stages of ring slot j ------
    if (lane >= NST) return;
    const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
    const __nv_bfloat16* zpool = static_cast<const __nv_bfloat16*>(a.z_pool);
    const uint64_t pol = policy_evict_first();
    const int s = lane;
    uint32_t pend = 0xffffffffu;  // the last stage this slot received copies for
    bool ok = true;
    for (uint32_t n = lane;; n += NST) {
      const CoopLook* e = &lookq[n % kCoopLookQ];
      if (!poll_equal(&e->seq, n, a.status, abort)) {
        ok = false;
        break;
      }
      __threadfence_block();
      const CoopLook lk = *e;
      if (lk.u == -2) break;
      // this slot's previous stage (n - NST) was handed out by this lane, so
      // the barrier is at most one phase behind the one waited for
      if (!mbar_wait_or_abort(&empty[s], ((n / NST) & 1u) ^ 1u, a.status, abort)) {
        ok = false;
        break;
      }
      meta[s] = CoopMeta{lk.u, lk.valid, lk.sid, 0};
      __threadfence_block();
      *reinterpret_cast<volatile uint32_t*>(&lookd[n % kCoopLookQ]) = n;
      if (lk.u == -1) {
        mbar_arrive(&full[s]);  // the end marker of one consumer warp
        break;
      }
      if (skip_issue_for_test((int)blockIdx.x, (int)n)) continue;
      uint8_t* dst = ring + (size_t)s * stage_bytes;
      pend = n;
      const unsigned long long row0 = BASISKV_DEBUG_INDEX(
          (long long)lk.row0, (long long)a.num_slots * a.num_kv_heads * P - TPS + 1, a.status);
      mbar_arrive_expect_tx(&full[s], stage_bytes);
      bulk_load(dst, kpool + row0 * D * KB, kbytes, &full[s], pol);
      bulk_load(dst + kbytes, zpool + row0 * RR, zbytes, &full[s], pol);
      if constexpr (K8) bulk_load(dst + kbytes + zbytes, a.k_scale + row0, sbytes, &full[s], pol);
    }
    // given up: let this slot's copies still in flight land before the CTA exits
    if (!ok && pend != 0xffffffffu) mbar_wait(&full[s], (pend / NST) & 1u, a.status);
    return;
  }

  if (warp > NW + 1) {
    // ---- the merge warps: segments mw, mw + 2, ... ----------------------------
    const int mw = warp - NW - 2;
    float* zb = zbar + mw * G * RR;
    // sequences no warp visits: without pages they get out = 0 and a -1
    // selection; with every page used (no routing) the identity selection
    const int ow = a.latent ? RR : D;
    for (int u = blockIdx.x * kCoopMergeWarps + mw; u < a.batch * a.num_kv_heads; u += gridDim.x * kCoopMergeWarps) {
      const int n = (a.seq_lens[u / a.num_kv_heads] + a.page_size - 1) / a.page_size;
      if (n == 0)
        for (int i = lane; i < G * ow; i += 32) a.out[(size_t)u * G * ow + i] = 0.f;
      if (a.sel_out && a.topk >= n)
        for (int i = lane; i < a.topk; i += 32) a.sel_out[(size_t)u * a.topk + i] = i < n ? i : -1;
    }
    for (uint32_t f = mw;; f += kCoopMergeWarps) {
      const int b = (int)(f % kCoopBufs);
      if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&mfull[b], (f / kCoopBufs) & 1u, a.status, abort))) return;
      CoopSeg sg = segs[f % kCoopSegs];
      if (sg.u < 0) return;
      sg.u = (int)BASISKV_DEBUG_INDEX(sg.u, a.batch * a.num_kv_heads, a.status);
      sg.kvh = (int)BASISKV_DEBUG_INDEX(sg.kvh, a.num_kv_heads, a.status);
      MergeOut<G, RR> mo;
      merge_warp_states<G, RR, NW>(mrg + (size_t)b * NW * MW, mo);
      __syncwarp();
      if (lane == 0) mbar_arrive(&mempty[b]);
      const int u = sg.u;
      if (sg.np == 1) {
        // the unit lies inside this chunk: this is its whole state
        if (a.latent) finish_unit_latent<G, RR>(mo, a.out + (size_t)u * G * RR);
        else finish_unit<G, RR, D>(mo, a.b_v + (size_t)sg.kvh * RR * D, a.out + (size_t)u * G * D, zb);
        continue;
      }
      if (sg.slot < a.np_cap) {
        const size_t part = (size_t)u * a.np_cap + sg.slot;
        if (lane < G) *reinterpret_cast<float2*>(a.part_ml + (part * G + lane) * 2) = make_float2(mo.M, mo.L);
#pragma unroll
        for (int k = 0; k < MergeOut<G, RR>::VPL; ++k) {
          const int v = lane + 32 * k;
          if (v < MergeOut<G, RR>::V) reinterpret_cast<float4*>(a.part_acc + part * G * RR)[v] = mo.acc[k];
        }
      } else if (lane == 0) {
        atomicOr(a.status, kStatusPartOverflow);  // more partials than slots: result invalid
      }
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        // release this partial, acquire the unit's others
        const uint32_t prevc = atomic_add_acq_rel(a.counters + u, (uint32_t)sg.seg_items);
        last = prevc + sg.seg_items == (uint32_t)sg.nu;
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        MergeOut<G, RR> fo;
        merge_all<G, RR>(a.part_ml + (size_t)u * a.np_cap * G * 2, a.part_acc + (size_t)u * a.np_cap * G * RR,
                         min(sg.np, a.np_cap), fo);
        if (a.latent) finish_unit_latent<G, RR>(fo, a.out + (size_t)u * G * RR);
        else finish_unit<G, RR, D>(fo, a.b_v + (size_t)sg.kvh * RR * D, a.out + (size_t)u * G * D, zb);
        if (lane == 0) a.counters[u] = 0u;
      }
    }
  }

  // ---- consumer warps: stages warp, warp + NW, warp + 2 NW, ... ----------
  uint32_t qa[D / 32][2][2];
  int q_u = -1;
  float m_run = -INFINITY, l_run = 0.f;
  float acc[RT][4];
#pragma unroll
  for (int c = 0; c < RT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
  uint32_t seg = 0;  // the segment this warp's state belongs to

  // leave the state of segment `seg` for the merge warp, then start afresh
  auto flush = [&]() -> bool {
    const int b = (int)(seg % kCoopBufs);
    if (!__all_sync(0xffffffffu,
                    mbar_wait_or_abort(&mempty[b], ((seg / kCoopBufs) & 1u) ^ 1u, a.status, abort)))
      return false;
    float l = l_run;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    float* w = mrg + (size_t)(b * NW + warp) * MW;
    if (g < G) {
      if (t == 0) {
        w[G * RR + 2 * g] = m_run;
        w[G * RR + 2 * g + 1] = l;
      }
#pragma unroll
      for (int c = 0; c < RT; ++c)
        *reinterpret_cast<float2*>(w + g * RR + 8 * c + 2 * t) = make_float2(acc[c][0] + acc[c][2], acc[c][1] + acc[c][3]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&mfull[b]);
    ++seg;
    m_run = -INFINITY;
    l_run = 0.f;
#pragma unroll
    for (int c = 0; c < RT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
    return true;
  };

  for (uint32_t n = warp;; n += NW) {
    const int s = (int)(n % NST);
    if (!__all_sync(0xffffffffu, mbar_wait_or_abort(&full[s], (n / NST) & 1u, a.status, abort))) return;
    const CoopMeta m = meta[s];
    // segments that ended before this stage (with or without stages of this warp)
    bool ok = true;
    while (ok && seg < (uint32_t)m.sid) ok = flush();
    if (!ok) return;
    if (m.u < 0) {
      // the closing segment numbers: one tells each merge warp to stop
      for (int j = 0; j < kCoopMergeWarps && flush(); ++j) {
      }
      return;
    }
    if (m.u != q_u) {
      load_q_frags<G, D, K8>(a, (int)BASISKV_DEBUG_INDEX(m.u, a.batch * a.num_kv_heads, a.status), qa);
      q_u = m.u;
    }
    if (m.valid > 0)
      attn_stage<G, D, RR, TPS, K8>(ring + (size_t)s * stage_bytes, m.valid, qa, a.scale_log2, m_run, l_run, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace basiskv
