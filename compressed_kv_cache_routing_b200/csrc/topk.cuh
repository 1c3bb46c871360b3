// Deterministic block-wide top-k page selection (BasisKV routing, "selected
// pages": the k pages of largest routing score per (sequence, KV head);
// equal scores go to the lower page index; the result is listed ascending).
//
// Scores are mapped to order-preserving unsigned keys; an MSB-first radix
// select (four 8-bit digits) finds the k-th largest key T and how many keys
// equal to T must be taken; a block scan in page order then takes every key
// above T plus the lowest-index keys equal to T.  The scores are read from
// global memory (L2) on every pass, so no shared buffer bounds the page count.
#pragma once

#include "common.cuh"

namespace basiskv {

// Order-preserving map float -> uint32 (larger float -> larger key).  -inf
// maps below every finite score; a NaN with the sign bit clear ranks above
// +inf.
__device__ __forceinline__ uint32_t score_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkSmem {
  int hist[256];
  int scan_tmp[32];
  int digit;
  int remaining;
  int whole;  // the digit's whole bucket is selected: later passes cannot change the set
};

// Select min(k, n) of the n scores at `scores` (global, written by other
// CTAs of this grid: read through L2).  Writes the ascending page list to
// sel[0 .. min(k,n)) and, when sel_out is not null, the same list padded with
// -1 to sel_out[0 .. out_len).  All NT threads of the block must call it.
template <int NT>
__device__ void block_topk(const float* scores, int n, int k, int32_t* sel, int32_t* sel_out,
                           int out_len, TopkSmem& sm) {
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int kb = k < n ? k : n;

  uint32_t thr = 0u;      // the kb-th largest key
  int need = 0;           // keys equal to thr to take, lowest page first
  if (kb < n) {
    uint32_t prefix = 0u, mask = 0u;
    int remaining = kb;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += NT) sm.hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += NT) {
        const uint32_t key = score_key(__ldcg(scores + i));
        if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns digits [8l, 8l+8); count keys in higher digits
        int local = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) local += sm.hist[8 * lane + q];
        int incl = local;  // keys in digits >= 8l
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += y;
        }
        const int above = incl - local;
        if (above < remaining && remaining <= incl) {
          int acc = above;
          for (int q = 7; q >= 0; --q) {
            const int c = sm.hist[8 * lane + q];
            if (acc + c >= remaining) {
              sm.digit = 8 * lane + q;
              sm.remaining = remaining - acc;
              break;
            }
            acc += c;
          }
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sm.digit) << shift;
      mask |= 0xFFu << shift;
      remaining = sm.remaining;
      __syncthreads();
    }
    thr = prefix;
    need = remaining;
  }

  // each thread owns a contiguous run of pages, so scans follow page order
  const int per = (n + NT - 1) / NT;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int total;
  int eq_before = 0;
  if (kb < n) {
    int eq = 0;
    for (int i = i0; i < i1; ++i) eq += score_key(__ldcg(scores + i)) == thr;
    eq_before = block_exclusive_scan<NT>(eq, sm.scan_tmp, &total);
  }
  int taken = 0;
  {
    int e = eq_before;
    for (int i = i0; i < i1; ++i) {
      bool take = true;
      if (kb < n) {
        const uint32_t key = score_key(__ldcg(scores + i));
        take = key > thr || (key == thr && e < need);
        e += key == thr;
      }
      taken += take;
    }
  }
  int pos = block_exclusive_scan<NT>(taken, sm.scan_tmp, &total);
  {
    int e = eq_before;
    for (int i = i0; i < i1; ++i) {
      bool take = true;
      if (kb < n) {
        const uint32_t key = score_key(__ldcg(scores + i));
        take = key > thr || (key == thr && e < need);
        e += key == thr;
      }
      if (take) {
        sel[pos] = i;
        if (sel_out) sel_out[pos] = i;
        ++pos;
      }
    }
  }
  if (sel_out)
    for (int i = kb + tid; i < out_len; i += NT) sel_out[i] = -1;
  (void)lane;
}

}  // namespace basiskv

namespace basiskv {

// ---------------------------------------------------------------------------
// Selection kernel: one CTA per (sequence, KV head) whose pages are routed.
// The scores are staged once in shared memory (up to keys_cap of them), the
// radix passes and the page-ordered compaction run there; units with more
// pages read the scores from L2 on every pass (block_topk).  The passes stop
// once the bucket holding the k-th key is taken whole: every key above the
// leading bits fixed so far and every key of the bucket is selected, so the
// compaction compares keys on those bits only and the set is the same.
struct TopkArgs {
  const float* scores;     // [B][Hkv][ld_pt]
  const uint64_t* scores64;  // [B][Hkv][ld_pt] (tag << 32) | fp32 bits, when poll
  const int32_t* seq_lens; // [B]
  int32_t* sel;            // [B][Hkv][ld_sel]
  int32_t* sel_out;        // [B][Hkv][topk] or null
  uint64_t* sel64;         // [B][Hkv][ld_sel] the selection tagged with the call, or null
  uint32_t* status;
  int num_kv_heads, page_size, ld_pt, ld_sel, topk, force, keys_cap;
  int poll;                // read tagged scores as they come, without waiting for the routing grid
  uint32_t tag;            // the routing call's tag (poll)
};

constexpr int kTopkThreads = 256;

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkArgs a) {
  pdl_launch_dependents();  // the attention grid waits for this one anyway
  __shared__ TopkSmem sm;
  extern __shared__ uint32_t keys[];
  const int b = blockIdx.y, kvh = blockIdx.x, u = b * a.num_kv_heads + kvh;
  const int n = (a.seq_lens[b] + a.page_size - 1) / a.page_size;
  if (n == 0 || !(a.force || a.topk < n)) return;
  // The scores come from the routing grid.  When they carry the call's tag
  // (poll) a CTA does not wait for the whole routing grid: it reads its
  // unit's scores until every one carries the tag, so units whose pages
  // are all scored are selected while the routing grid still streams
  // others.  Each 8-byte word is written and read atomically, so a tagged
  // word holds this call's score.
  if (!a.poll) pdl_wait_primary();
  const float* sc = a.scores + (size_t)u * a.ld_pt;
  int32_t* sel = a.sel + (size_t)u * a.ld_sel;
  uint64_t* sel64 = a.sel64 ? a.sel64 + (size_t)u * a.ld_sel : nullptr;
  int32_t* so = a.sel_out ? a.sel_out + (size_t)u * a.topk : nullptr;
  if (n > a.keys_cap) {
    block_topk<kTopkThreads>(sc, n, a.topk, sel, so, a.topk, sm);
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (a.poll) {
    const uint64_t* sc64 = a.scores64 + (size_t)u * a.ld_pt;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
      bool ok = true;
      for (int i = tid; i < n; i += kTopkThreads) {
        const uint64_t w = ld_relaxed_u64(sc64 + i);
        ok = ok && (uint32_t)(w >> 32) == a.tag;
        keys[i] = score_key(__uint_as_float((uint32_t)w));
      }
      if (__syncthreads_and(ok)) break;
      if (__syncthreads_or(global_timer_ns() - t0 > kWaitLimitNs)) {
        if (tid == 0) atomicOr(a.status, kStatusTimeout);
        break;
      }
      __nanosleep(512);
    }
  } else {
    for (int i = tid; i < n; i += kTopkThreads) keys[i] = score_key(__ldcg(sc + i));
  }
  __syncthreads();
  const int kb = a.topk < n ? a.topk : n;
  uint32_t thr = 0u, tmask = 0xFFFFFFFFu;  // keys compare on their bits under tmask
  int need = 0;
  if (kb < n) {
    uint32_t prefix = 0u, mask = 0u;
    int remaining = kb;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kTopkThreads) sm.hist[i] = 0;
      __syncthreads();
      for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + tid;
        const uint32_t key = i < n ? keys[i] : 0u;
        const bool in = i < n && (key & mask) == prefix;
        const uint32_t act = __ballot_sync(0xffffffffu, in);
        if (in) {
          const uint32_t digit = (key >> shift) & 255u;
          const uint32_t grp = __match_any_sync(act, digit);
          if ((int)(__ffs(grp) - 1) == lane) atomicAdd(&sm.hist[digit], __popc(grp));
        }
      }
      __syncthreads();
      if (warp == 0) {
        int local = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) local += sm.hist[8 * lane + q];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_down_sync(0xffffffffu, incl, o);
          if (lane + o < 32) incl += y;
        }
        const int above = incl - local;
        if (above < remaining && remaining <= incl) {
          int acc = above;
          for (int q = 7; q >= 0; --q) {
            const int c = sm.hist[8 * lane + q];
            if (acc + c >= remaining) {
              sm.digit = 8 * lane + q;
              sm.remaining = remaining - acc;
              sm.whole = remaining - acc == c;
              break;
            }
            acc += c;
          }
        }
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(sm.digit) << shift;
      mask |= 0xFFu << shift;
      remaining = sm.remaining;
      const bool whole = sm.whole;
      __syncthreads();
      if (whole) break;  // every key of the bucket is taken: the set is decided
    }
    thr = prefix;
    tmask = mask;
    need = remaining;
  }
  // page-ordered compaction: each thread owns a contiguous run
  const int per = (n + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
  int total;
  int eq = 0, take = 0;
  for (int i = i0; i < i1; ++i) eq += (keys[i] & tmask) == thr;
  const int eq_before = kb < n ? block_exclusive_scan<kTopkThreads>(eq, sm.scan_tmp, &total) : 0;
  {
    int e = eq_before;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[i] & tmask;
      take += kb >= n || key > thr || (key == thr && e < need);
      e += key == thr;
    }
  }
  int pos = block_exclusive_scan<kTopkThreads>(take, sm.scan_tmp, &total);
  {
    int e = eq_before;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[i] & tmask;
      if (kb >= n || key > thr || (key == thr && e < need)) {
        pos = (int)BASISKV_DEBUG_INDEX(pos, a.ld_sel, a.status);
        sel[pos] = i;
        if (sel64) st_relaxed_u64(sel64 + pos, ((uint64_t)a.tag << 32) | (uint32_t)i);
        if (so) so[pos] = i;
        ++pos;
      }
      e += key == thr;
    }
  }
  if (so)
    for (int i = kb + tid; i < a.topk; i += kTopkThreads) so[i] = -1;
}

}  // namespace basiskv
