// Exact attention over the selected pages for BasisKV decode ("the original
// Keys are then retrieved only for the selected pages to compute exact QK
// scores"); values stay rank-r latents Z, and the weighted latent is
// expanded by B_v in the fused combine.
//
// Two kernels.  attn_mma_kernel (bf16 pools, tensor cores; bf16 or int8
// keys) is persistent over the flat list of selected-page stages and is
// described above its definition.  attn_generic_kernel (any dtype or shape)
// runs a grid (splits, Hkv, batch): split sp of a (sequence, KV head)
// handles selected entries [sp*pps, min((sp+1)*pps, k_b)), keeps an online
// softmax state (running max m in log2 units, sum l, latent accumulator
// acc[r]) for the G query heads and writes it as one partial; the last CTA
// of the unit merges all partials and applies B_v.
#pragma once

#include <cuda_fp16.h>

#include "combine.cuh"
#include "common.cuh"

namespace basiskv {

// ---- f16 tensor-core helpers for int8 keys -----------------------------------
// The same product with f16 operands (A and B both f16).
__device__ __forceinline__ void mma_k16_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Pack two floats into an f16x2 register (first argument in the low half).
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// The four int8 codes of w (two's complement, byte i = code i) as f16 pairs
// (c0, c1) and (c2, c3), exactly.  Flipping a byte's top bit gives
// u = c + 128 in [0, 255]; the f16 whose bits are 0x64 in the high byte and
// u in the low byte is 1024 + u, because f16 values in [1024, 2048) are the
// integers; subtracting 1152 = 1024 + 128 (0x6480) then leaves c, exactly.
__device__ __forceinline__ void codes_to_f16x2(uint32_t w, uint32_t& c01, uint32_t& c23) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t p01 = __byte_perm(u, 0x64646464u, 0x4140);
  const uint32_t p23 = __byte_perm(u, 0x64646464u, 0x4342);
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(c01) : "r"(p01), "r"(0x64806480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(c23) : "r"(p23), "r"(0x64806480u));
}


struct AttnArgs {
  const void* q;             // [B][Hkv*G][d]
  const void* k_pool;        // [slots][Hkv][P][d]: pool dtype, or int8 codes when k_int8
  const float* k_scale;      // [slots][Hkv][P] per-token key scale (k_int8 only)
  const void* z_pool;        // [slots][Hkv][P][r]
  const float* b_v;          // [Hkv][r][d]
  const int32_t* page_table; // [B][ld_pt]
  const int32_t* seq_lens;   // [B]
  const int32_t* sel;        // [B][Hkv][ld_sel] (routed units)
  const uint64_t* sel64;     // [B][Hkv][ld_sel] (tag << 32) | page, or null (persistent kernel)
  uint32_t sel_tag;          // the tag of this call's selection (sel64)
  int32_t* sel_out;          // [B][Hkv][topk] or null
  float* part_ml;            // [B*Hkv][np_cap][G][2]
  float* part_acc;           // [B*Hkv][np_cap][G][r]
  uint32_t* counters;        // [B*Hkv]
  uint32_t* status;
  float* out;                // [B][Hkv*G][d]; [B][Hkv*G][r] when latent
  int ld_pt, ld_sel, num_slots, num_kv_heads, head_dim, page_size, rank_r, gqa_group;
  int topk, pages_per_split, stages, np_cap;
  float scale_log2;          // softmax_scale * log2(e)
  int latent;                // write the weighted latent zbar, before B_v
  int k_int8;                // keys are int8 codes: K_t = k_scale[t] * code_t
  // persistent tensor-core kernel only
  int batch;
  const int32_t* attn_off;   // [B+1] prefix of attention items x Hkv (from the prep grid)
  int chunk_items;           // cooperative kernel: items per chunk (0: one chunk per CTA)
  int plan_n;                // >= 0: plan_off holds attn_off (batch <= kPlanMax)
  int32_t plan_off[kPlanMax + 1];
};

constexpr int kAttnThreads = 128;
constexpr int kAttnWarps = kAttnThreads / 32;

struct AttnUnit {
  int b, kvh, u, L, n, kb, j0, j1;
  bool routed;
};

__device__ __forceinline__ AttnUnit attn_unit(const AttnArgs& a) {
  AttnUnit au;
  au.b = blockIdx.z;
  au.kvh = blockIdx.y;
  au.u = au.b * a.num_kv_heads + au.kvh;
  au.L = a.seq_lens[au.b];
  au.n = (au.L + a.page_size - 1) / a.page_size;
  if (au.n > a.ld_pt || au.L < 0) {
    // a length the page-table row cannot hold (only callers that pass
    // device lengths unchecked can get here): clamp to the row
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.status, kStatusBadLength);
    au.L = au.L < 0 ? 0 : a.ld_pt * a.page_size;
    au.n = au.L / a.page_size;
  }
  au.routed = a.topk < au.n;
  au.kb = au.routed ? a.topk : au.n;
  au.j0 = blockIdx.x * a.pages_per_split;
  au.j1 = min(au.kb, au.j0 + a.pages_per_split);
  return au;
}

// Logical page of selected entry jj, checked against [0, n).
__device__ __forceinline__ int selected_page(const AttnArgs& a, const AttnUnit& au, int jj) {
  if (!au.routed) return jj;
  int p = __ldcg(a.sel + (size_t)au.u * a.ld_sel + jj);
  if (p < 0 || p >= au.n) {
    atomicOr(a.status, kStatusBadPage);
    p = 0;
  }
  return p;
}

__device__ __forceinline__ int page_slot(const AttnArgs& a, const AttnUnit& au, int page) {
  int slot = a.page_table[(size_t)au.b * a.ld_pt + page];
  if (slot < 0 || slot >= a.num_slots) {
    atomicOr(a.status, kStatusBadSlot);
    slot = 0;
  }
  return slot;
}

// Units whose every page is used were not routed: list their pages.
__device__ __forceinline__ void write_identity_selection(const AttnArgs& a, const AttnUnit& au) {
  if (au.routed || blockIdx.x != 0 || a.sel_out == nullptr) return;
  int32_t* so = a.sel_out + (size_t)au.u * a.topk;
  for (int i = threadIdx.x; i < a.topk; i += blockDim.x) so[i] = i < au.n ? i : -1;
}

template <int NT>
__device__ __forceinline__ void attn_finish(const AttnArgs& a, const AttnUnit& au, int parts_per_cta,
                                            float* smem_f, int* flag) {
  if (!arrive_last(a.counters + au.u, gridDim.x, flag)) return;
  const int G = a.gqa_group;
  CombineArgs c;
  c.part_ml = a.part_ml + (size_t)au.u * a.np_cap * G * 2;
  c.part_acc = a.part_acc + (size_t)au.u * a.np_cap * G * a.rank_r;
  c.b_v = a.b_v + (size_t)au.kvh * a.rank_r * a.head_dim;
  c.out = a.out + (size_t)au.u * G * (a.latent ? a.rank_r : a.head_dim);
  c.latent = a.latent;
  c.np = gridDim.x * parts_per_cta;
  c.g = G;
  c.r = a.rank_r;
  c.d = a.head_dim;
  combine_unit<NT>(c, smem_f);
}

// One staged attention item of TPS tokens of one selected page: exact QK for
// the group (heads as M, tokens as N, k permuted so each B fragment is one
// 16-byte shared load), the online softmax in fp32 (log2 units) and the
// latent sum P.Z with the probabilities split into bf16 hi (rows g) and lo
// (rows g + 8).  `stage` holds the K rows (bf16, or int8 codes when K8),
// then the Z rows, then (K8) the TPS fp32 token scales; tokens at or past
// `valid` are masked.  qa: this lane's query fragments.
template <int G, int D, int RR, int TPS, bool K8>
__device__ __forceinline__ void attn_stage(const uint8_t* stage, int valid, const uint32_t (&qa)[D / 32][2][2],
                                           float scale_log2, float& m_run, float& l_run, float (&acc)[RR / 8][4]) {
  constexpr int DS = D / 32;
  constexpr int RT = RR / 8;
  constexpr int NTS = TPS / 8;
  constexpr int KBS = TPS / 16;
  constexpr int KB = K8 ? 1 : 2;
  constexpr uint32_t kbytes = TPS * D * KB, zbytes = TPS * RR * 2;
  (void)DS;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int trow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const __nv_bfloat16* zs = reinterpret_cast<const __nv_bfloat16*>(stage + kbytes);

  // exact QK for the group
  float s[NTS][2];
#pragma unroll
  for (int nt = 0; nt < NTS; ++nt) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    const uint8_t* krow = stage + (nt * 8 + g) * D * KB;
    const int tok = nt * 8 + 2 * t;
    if constexpr (K8) {
      // 128-byte code rows: odd rows take their two 64-channel spans in the
      // other order, so a quarter-warp's two rows fall on disjoint banks
      uint4 kv[D / 64];
      if constexpr (D / 64 == 2) {
        const int odd = g & 1;
        const uint4 u0 = lds128(krow + 64 * odd + 16 * t), u1 = lds128(krow + 64 * (1 - odd) + 16 * t);
        kv[0] = odd ? u1 : u0;
        kv[1] = odd ? u0 : u1;
      } else {
#pragma unroll
        for (int sp = 0; sp < D / 64; ++sp) kv[sp] = lds128(krow + 64 * sp + 16 * t);
      }
#pragma unroll
      for (int sp = 0; sp < D / 64; ++sp) {
        const uint4 v = kv[sp];
        uint32_t b0, b1;
        codes_to_f16x2(v.x, b0, b1);
        mma_k16_f16(d, qa[2 * sp][0][0], 0u, qa[2 * sp][0][1], 0u, b0, b1);
        codes_to_f16x2(v.y, b0, b1);
        mma_k16_f16(d, qa[2 * sp][1][0], 0u, qa[2 * sp][1][1], 0u, b0, b1);
        codes_to_f16x2(v.z, b0, b1);
        mma_k16_f16(d, qa[2 * sp + 1][0][0], 0u, qa[2 * sp + 1][0][1], 0u, b0, b1);
        codes_to_f16x2(v.w, b0, b1);
        mma_k16_f16(d, qa[2 * sp + 1][1][0], 0u, qa[2 * sp + 1][1][1], 0u, b0, b1);
      }
      const uint2 sc = lds64(stage + kbytes + zbytes + 4 * tok);
      d[0] *= __uint_as_float(sc.x);
      d[1] *= __uint_as_float(sc.y);
    } else {
      // 64-channel halves: thread t holds channels 16t .. 16t+15 of each
      // (16-byte chunks 2t and 2t+1); odd rows read the two chunks in the
      // other order, so the even and odd rows of a quarter-warp use even and
      // odd chunks (disjoint banks), and a select puts them back in place
#pragma unroll
      for (int h = 0; h < D / 64; ++h) {
        const int odd = g & 1;
        const uint4 u0 = lds128(krow + 2 * (64 * h + 16 * t + 8 * odd));
        const uint4 u1 = lds128(krow + 2 * (64 * h + 16 * t + 8 * (1 - odd)));
        const uint4 v0 = odd ? u1 : u0, v1 = odd ? u0 : u1;
        mma_k16(d, qa[2 * h][0][0], 0u, qa[2 * h][0][1], 0u, v0.x, v0.y);
        mma_k16(d, qa[2 * h][1][0], 0u, qa[2 * h][1][1], 0u, v0.z, v0.w);
        mma_k16(d, qa[2 * h + 1][0][0], 0u, qa[2 * h + 1][0][1], 0u, v1.x, v1.y);
        mma_k16(d, qa[2 * h + 1][1][0], 0u, qa[2 * h + 1][1][1], 0u, v1.z, v1.w);
      }
    }
    s[nt][0] = tok < valid ? d[0] * scale_log2 : -INFINITY;
    s[nt][1] = tok + 1 < valid ? d[1] * scale_log2 : -INFINITY;
  }
  // online softmax for head g (the quad 4g..4g+3 shares the row)
  float mloc = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NTS; ++nt) mloc = fmaxf(mloc, fmaxf(s[nt][0], s[nt][1]));
  mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 1));
  mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, 2));
  const float m_new = fmaxf(m_run, mloc);
  const float corr = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);
  const float base = (m_new == -INFINITY) ? 0.f : m_new;
  float lsum = 0.f;
#pragma unroll
  for (int nt = 0; nt < NTS; ++nt) {
    s[nt][0] = exp2f(s[nt][0] - base);
    s[nt][1] = exp2f(s[nt][1] - base);
    lsum += s[nt][0] + s[nt][1];
  }
  l_run = l_run * corr + lsum;
  m_run = m_new;
#pragma unroll
  for (int c = 0; c < RT; ++c) {
    acc[c][0] *= corr;
    acc[c][1] *= corr;
    acc[c][2] *= corr;
    acc[c][3] *= corr;
  }
  // latent sum P.Z
#pragma unroll
  for (int kb = 0; kb < KBS; ++kb) {
    float h0, l0, h1, l1, h2, l2, h3, l3;
    split_bf16(s[2 * kb][0], h0, l0);
    split_bf16(s[2 * kb][1], h1, l1);
    split_bf16(s[2 * kb + 1][0], h2, l2);
    split_bf16(s[2 * kb + 1][1], h3, l3);
    const uint32_t a0 = pack_bf16(h0, h1), a1 = pack_bf16(l0, l1);
    const uint32_t a2 = pack_bf16(h2, h3), a3 = pack_bf16(l2, l3);
    const __nv_bfloat16* zrow = zs + (kb * 16 + trow) * RR + 8 * (lane >> 4);
#pragma unroll
    for (int c2 = 0; c2 < RT / 2; ++c2) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(b0, b1, b2, b3, zrow + 16 * c2);
      mma_k16(acc[2 * c2], a0, a1, a2, a3, b0, b1);
      mma_k16(acc[2 * c2 + 1], a0, a1, a2, a3, b2, b3);
    }
    if (RT & 1) {
      uint32_t b0, b1;
      ldsm_x2_trans(b0, b1, zs + (kb * 16 + trow) * RR + 8 * (RT - 1));
      mma_k16(acc[RT - 1], a0, a1, a2, a3, b0, b1);
    }
  }
}

// ---------------------------------------------------------------------------
// Tensor-core attention for bf16 pools, persistent over the flat list of
// attention items (sequence-major, then KV head, selected entry, stage of
// the page); every warp streams one contiguous share of it.
//
// QK: S(16 x 8 tokens) = Qg(16 x d) . K^T, rows 0..G-1 of Qg hold the group's
// queries (rows G..15 zero), K rows come from shared memory; the k index is
// permuted so that thread t holds channels 16t .. 16t+15 of each 64-channel
// half of a key row (two 16-byte loads; MMA j of half h takes channels
// 64h + 16t + 4j .. +3 on both operands), and odd rows load the two chunks
// in swapped order, so the two rows a quarter-warp reads use disjoint
// banks.  The S fragment (row g = head, columns 2t, 2t+1 = tokens) is
// already the A fragment layout of the next product, so the probabilities
// never leave registers.
// PV: acc(16 x r) += Pg(16 x 16 tokens) . Z(16 tokens x r); row g of Pg holds
// bf16 hi(p) of head g and row g+8 holds lo(p) = bf16(p - hi(p)), so
// acc[g] + acc[g+8] is the latent sum with ~16-bit weights; Z fragments come
// from ldmatrix.trans.
// Each stage carries TPS tokens of one selected page (K then Z), staged by
// bulk copies into a per-warp ring.
// Int8 keys (K8): a stage carries the codes, Z, then the TPS token scales.
// Codes become f16 exactly in registers (codes_to_f16x2) and meet the query
// rounded to f16 in an f16 MMA; the 16-byte load of a token row covers 64
// channels, so the k index runs over channel 64*sp + 16*t + 4*j + e for MMA
// j of span sp (the query fragments follow the same order), and the token's
// scale multiplies its dot product before the softmax.  At the end of its segment of a unit a
// warp writes one partial (m, l, acc); the warp that completes the unit
// merges the partials and applies B_v.
// This lane's query fragments for unit u (the group's G heads as rows g < G
// of the A operand, zero rows for g >= G), in the k order of the key loads:
// MMA j of 64-channel span h takes channels (c, c+1) and (c+2, c+3) with
// c = 64*h + 16*t + 4*j.  Int8 keys meet the query rounded to f16.
template <int G, int D, bool K8>
__device__ __forceinline__ void load_q_frags(const AttnArgs& a, int u, uint32_t (&qa)[D / 32][2][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)u * G + (g < G ? g : 0)) * D;
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
    if (g < G) {
      v0 = __ldg(reinterpret_cast<const uint4*>(qrow + 64 * h + 16 * t));
      v1 = __ldg(reinterpret_cast<const uint4*>(qrow + 64 * h + 16 * t + 8));
    }
    if constexpr (K8) {
      auto h2 = [](uint32_t w) { return pack_f16(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)); };
      v0 = make_uint4(h2(v0.x), h2(v0.y), h2(v0.z), h2(v0.w));
      v1 = make_uint4(h2(v1.x), h2(v1.y), h2(v1.z), h2(v1.w));
    }
    qa[2 * h][0][0] = v0.x;
    qa[2 * h][0][1] = v0.y;
    qa[2 * h][1][0] = v0.z;
    qa[2 * h][1][1] = v0.w;
    qa[2 * h + 1][0][0] = v1.x;
    qa[2 * h + 1][0][1] = v1.y;
    qa[2 * h + 1][1][0] = v1.z;
    qa[2 * h + 1][1][1] = v1.w;
  }
}

// A tagged selection entry whose unit is still being selected: wait for it
// (bounded; on expiry the status says TIMEOUT and entry 0 is used).
__device__ __noinline__ uint64_t wait_selected(const uint64_t* src, uint32_t tag, uint32_t* status) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(256);
    const uint64_t w = ld_relaxed_u64(src);
    if ((uint32_t)(w >> 32) == tag) return w;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicOr(status, kStatusTimeout);
      return 0;
    }
  }
}

struct AttnCursor {
  int b, kvh, jj, ts, n, kb, L;
  int uoff;            // flat index of the unit's first item
  const int32_t* off;  // prefix of attention items x Hkv over sequences
  __device__ __forceinline__ void load(const AttnArgs& a) {
    L = a.seq_lens[b];
    n = (L + a.page_size - 1) / a.page_size;
    kb = min(a.topk, n);
    uoff = off[b];
  }
  __device__ void seek(const AttnArgs& a, const int32_t* offsets, int f, int sub) {
    off = offsets;
    int lo = 0, hi = a.batch;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= f) lo = mid + 1;
      else hi = mid;
    }
    b = lo - 1;
    load(a);
    const int per_unit = kb * sub;
    const int rel = f - uoff;
    kvh = rel / per_unit;
    const int r2 = rel % per_unit;
    jj = r2 / sub;
    ts = r2 % sub;
    uoff += kvh * per_unit;
  }
  __device__ __forceinline__ void advance(const AttnArgs& a, int sub) {
    if (++ts < sub) return;
    ts = 0;
    if (++jj < kb) return;
    jj = 0;
    if (++kvh < a.num_kv_heads) {
      uoff += kb * sub;
      return;
    }
    kvh = 0;
    for (++b; b < a.batch; ++b) {
      load(a);
      if (kb > 0) return;
    }
  }
  __device__ __forceinline__ int unit(const AttnArgs& a) const { return b * a.num_kv_heads + kvh; }
  template <bool TS>
  __device__ __forceinline__ int page(const AttnArgs& a) const { return checked<TS>(a, page_raw<TS>(a)); }
  // The selected entry, unchecked: the load stays in flight until the value
  // is used (check it with checked() when the item is issued).  A tagged
  // entry (TS: sel64) carries the tag of the call whose selection wrote it.
  template <bool TS>
  __device__ __forceinline__ auto page_raw(const AttnArgs& a) const {
    if constexpr (TS) {
      if (a.topk >= n) return (uint64_t)jj;
      return ld_relaxed_u64(a.sel64 + (size_t)unit(a) * a.ld_sel + jj);
    } else {
      if (a.topk >= n) return jj;
      return __ldcg(a.sel + (size_t)unit(a) * a.ld_sel + jj);
    }
  }
  template <bool TS, typename Word>
  __device__ __forceinline__ int checked(const AttnArgs& a, Word w) const {
    if constexpr (TS) {
      if (a.topk < n && (uint32_t)(w >> 32) != a.sel_tag)
        w = wait_selected(a.sel64 + (size_t)unit(a) * a.ld_sel + jj, a.sel_tag, a.status);
    }
    int p = (int)(uint32_t)w;
    if (p < 0 || p >= n) {
      atomicOr(a.status, kStatusBadPage);
      p = 0;
    }
    return p;
  }
};

// TS: the selection comes as tagged entries (sel64) from a selection grid
// that this grid does not wait for as a whole.
template <int G, int D, int RR, int TPS, bool K8 = false, bool TS = false>
__global__ void __launch_bounds__(kAttnThreads) attn_mma_kernel(const __grid_constant__ AttnArgs a) {
  static_assert(G >= 1 && G <= 8, "GQA group must be 1..8");
  static_assert(D % 32 == 0 && RR % 8 == 0 && TPS % 16 == 0, "shape");
  static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
  constexpr int DS = D / 32;     // 32-wide spans of the head dim
  constexpr int RT = RR / 8;     // n8 tiles of the latent
  constexpr int KB = K8 ? 1 : 2; // bytes per key element
  constexpr uint32_t kbytes = TPS * D * KB, zbytes = TPS * RR * 2, sbytes = K8 ? TPS * 4 : 0;
  constexpr uint32_t stage_bytes = kbytes + zbytes + sbytes;

  const int P = a.page_size, S = a.stages;
  const int sub = P / TPS;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t bars[kAttnWarps][8];
  __shared__ int tok0s[kAttnWarps][8];
  // sequences no warp visits: without pages they get out = 0 and a -1
  // selection; with every page used (no routing) the identity selection
  const int ow = a.latent ? RR : D;  // output row width
  for (int u = blockIdx.x; u < a.batch * a.num_kv_heads; u += gridDim.x) {
    const int n = (a.seq_lens[u / a.num_kv_heads] + a.page_size - 1) / a.page_size;
    if (n == 0)
      for (int i = threadIdx.x; i < G * ow; i += blockDim.x) a.out[(size_t)u * G * ow + i] = 0.f;
    if (a.sel_out && a.topk >= n)
      for (int i = threadIdx.x; i < a.topk; i += blockDim.x) a.sel_out[(size_t)u * a.topk + i] = i < n ? i : -1;
  }
  uint8_t* ring = smem + (size_t)warp * S * stage_bytes;
  float* zbar = reinterpret_cast<float*>(smem + (size_t)kAttnWarps * S * stage_bytes) + warp * G * RR;
  if (lane == 0) {
    for (int i = 0; i < S; ++i) mbar_init(&bars[warp][i], 1);
    mbar_init_fence();
  }
  __syncwarp();

  // the plan comes in the parameters, or from the prep grid, which finished
  // before the routing grid let this one launch
  const int32_t* offsets = a.plan_n >= 0 ? a.plan_off : a.attn_off;
  const long long W = (long long)gridDim.x * kAttnWarps;
  const int wg = blockIdx.x * kAttnWarps + warp;
  const long long T = offsets[a.batch];
  const int f0 = (int)(T * wg / W), f1 = (int)(T * (wg + 1) / W);
  const int count = f1 - f0;
  AttnCursor ic;
  if (count > 0) ic.seek(a, offsets, f0, sub);
  (void)f1;
  AttnCursor cc = ic;

  uint32_t qa[DS][2][2];
  auto load_q = [&](int u) { load_q_frags<G, D, K8>(a, u, qa); };
  int cur_u = -1;
  if (count > 0) {
    cur_u = cc.unit(a);
    load_q(cur_u);
  }
  // The selection is written by the previous grid: wait for that grid, or,
  // with a tagged selection, for each unit's entries as they are needed.
  if constexpr (!TS) pdl_wait_primary();
  if (count <= 0) return;

  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const __nv_bfloat16* zpool = static_cast<const __nv_bfloat16*>(a.z_pool);
  const uint64_t pol = policy_evict_first();
  // lane 0 issues item i of this warp into ring position s = i mod S; the selection and
  // page-table reads for an item are made one iteration before its issue so
  // they overlap the arithmetic of the current stage
  auto slot_of = [&](int page) { return __ldg(a.page_table + (size_t)ic.b * a.ld_pt + page); };
  auto issue = [&](int i, int s, int page, int slot) {
    if (slot < 0 || slot >= a.num_slots) {
      atomicOr(a.status, kStatusBadSlot);
      slot = 0;
    }
    const size_t row0 = BASISKV_DEBUG_INDEX(((long long)slot * a.num_kv_heads + ic.kvh) * P + (long long)ic.ts * TPS,
                                            (long long)a.num_slots * a.num_kv_heads * P - TPS + 1, a.status);
    tok0s[warp][s] = page * P + ic.ts * TPS;
    uint64_t* bar = &bars[warp][s];
    uint8_t* dst = ring + (size_t)s * stage_bytes;
    if (skip_issue_for_test(wg, i)) {
      ic.advance(a, sub);
      return;
    }
    mbar_arrive_expect_tx(bar, stage_bytes);
    bulk_load(dst, kpool + row0 * D * KB, kbytes, bar, pol);
    bulk_load(dst + kbytes, zpool + row0 * RR, zbytes, bar, pol);
    if constexpr (K8) bulk_load(dst + kbytes + zbytes, a.k_scale + row0, sbytes, bar, pol);
    ic.advance(a, sub);
  };
  AttnCursor ia;       // lane 0: the item after the next one to issue
  using SelWord = decltype(ic.page_raw<TS>(a));
  SelWord next_page = 0;  // lane 0: selected entry of the next item to issue (loaded, unchecked)
  {
    // the first S items: lane j looks item j up (all lookups in parallel),
    // lane 0 issues them in order
    const int first = min(S, count);
    int pg = 0, sl = 0;
    if (lane < first) {
      AttnCursor c = ic;
      for (int k = 0; k < lane; ++k) c.advance(a, sub);
      pg = c.page<TS>(a);
      sl = __ldg(a.page_table + (size_t)c.b * a.ld_pt + pg);
    }
    for (int i = 0; i < first; ++i) {
      const int pgi = __shfl_sync(0xffffffffu, pg, i), sli = __shfl_sync(0xffffffffu, sl, i);
      if (lane == 0) issue(i, i, pgi, sli);
    }
  }
  if (lane == 0) {
    if (S < count) {
      next_page = ic.page_raw<TS>(a);
      ia = ic;
      ia.advance(a, sub);
    }
  }

  float m_run = -INFINITY, l_run = 0.f;
  float acc[RT][4];
#pragma unroll
  for (int c = 0; c < RT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
  int seg = 0;
  AttnCursor prev = cc;

  // end of this warp's segment of unit u: write its partial, count the
  // items; the warp completing the unit merges everything and applies B_v
  // Warp w streams items [floor(T*w/W), floor(T*(w+1)/W)); the warp holding
  // item o is ceil((o+1)*W/T) - 1.  A unit's partial slot is the warp's rank
  // among the warps holding its items, so the merge order never changes.
  auto owner = [&](long long o) { return (int)(((o + 1) * W + T - 1) / T) - 1; };
  // end of this warp's segment of unit u: write its partial, count the
  // items; the warp completing the unit merges everything and applies B_v
  auto flush = [&](const AttnCursor& at) {
    const int u = cur_u;
    float l = l_run;
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int items = at.kb * sub;
    const int w_first = owner(at.uoff);
    const int np = owner((long long)at.uoff + items - 1) - w_first + 1;
    const int slot = wg - w_first;
    if (slot < a.np_cap) {
      if (g < G) {
        const size_t part = ((size_t)u * a.np_cap + slot) * G + g;
        if (t == 0) {
          a.part_ml[part * 2] = m_run;
          a.part_ml[part * 2 + 1] = l;
        }
        float* pa = a.part_acc + part * RR;
#pragma unroll
        for (int c = 0; c < RT; ++c) {
          pa[8 * c + 2 * t] = acc[c][0] + acc[c][2];
          pa[8 * c + 2 * t + 1] = acc[c][1] + acc[c][3];
        }
      }
    } else if (lane == 0) {
      atomicOr(a.status, kStatusPartOverflow);  // more partials than slots: result invalid
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence();
      const uint32_t prevc = atomicAdd(a.counters + u, (uint32_t)seg);
      last = prevc + seg == (uint32_t)items;
      __threadfence();
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      const float* bv = a.b_v + (size_t)at.kvh * RR * D;
      MergeOut<G, RR> mo;
      merge_all<G, RR>(a.part_ml + (size_t)u * a.np_cap * G * 2, a.part_acc + (size_t)u * a.np_cap * G * RR,
                       min(np, a.np_cap), mo);
      if (a.latent) finish_unit_latent<G, RR>(mo, a.out + (size_t)u * G * RR);
      else finish_unit<G, RR, D>(mo, bv, a.out + (size_t)u * G * D, zbar);
      if (lane == 0) a.counters[u] = 0u;
    }
  };

  bool ok = true;
  int i = 0;
  int s_i = 0;        // ring position of item i (i mod S)
  uint32_t ph_i = 0;  // phase parity of that position's barrier for item i
  for (; i < count; ++i) {
    int next_pg = 0, next_slot = 0;
    SelWord page_after = 0;
    if (lane == 0) {
      // the page of item i + S was read one iteration ago: check it and read
      // its slot now; the page of the item after it stays in flight
      if (i + S < count) {
        next_pg = ic.checked<TS>(a, next_page);
        next_slot = slot_of(next_pg);
      }
      if (i + S + 1 < count) page_after = ia.page_raw<TS>(a);
    }
    const int u = cc.unit(a);
    if (u != cur_u) {
      flush(prev);
      cur_u = u;
      seg = 0;
      m_run = -INFINITY;
      l_run = 0.f;
#pragma unroll
      for (int c = 0; c < RT; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
      load_q(u);
    }
    ok = mbar_wait(&bars[warp][s_i], ph_i, a.status);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    const int valid = cc.L - tok0s[warp][s_i];  // tokens of this stage inside the sequence
    attn_stage<G, D, RR, TPS, K8>(ring + (size_t)s_i * stage_bytes, valid, qa, a.scale_log2, m_run, l_run, acc);
    ++seg;
    __syncwarp();
    if (lane == 0 && i + S < count) {
      issue(i + S, s_i, next_pg, next_slot);  // (i + S) mod S = i mod S
      next_page = page_after;
      ia.advance(a, sub);
    }
    prev = cc;
    cc.advance(a, sub);
    if (++s_i == S) {
      s_i = 0;
      ph_i ^= 1u;
    }
  }
  if (!ok) {
    if (lane == 0)
      for (int j = i; j < count && j < i + S; ++j)
        mbar_wait(&bars[warp][j % S], (uint32_t)((j / S) & 1), a.status);
    return;
  }
  flush(prev);
}

// ---------------------------------------------------------------------------
// CUDA-core attention for any shape and for fp32 pools: one partial per CTA.
template <typename T>
__global__ void __launch_bounds__(kAttnThreads) attn_generic_kernel(const __grid_constant__ AttnArgs a) {
  const AttnUnit au = attn_unit(a);
  const int G = a.gqa_group, D = a.head_dim, RR = a.rank_r, P = a.page_size;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int flag;
  float* qs = reinterpret_cast<float*>(smem);  // [G][D]
  float* sc = qs + G * D;                      // [G][P]
  float* accs = sc + G * P;                    // [G][RR]
  float* corr = accs + G * RR;                 // [G]
  float* mrun = corr + G;                      // [G]
  float* lrun = mrun + G;                      // [G]
  const T* q = static_cast<const T*>(a.q) + (size_t)au.u * G * D;
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) qs[i] = to_f32(q[i]);
  for (int i = threadIdx.x; i < G * RR; i += blockDim.x) accs[i] = 0.f;
  for (int i = threadIdx.x; i < G; i += blockDim.x) {
    mrun[i] = -INFINITY;
    lrun[i] = 0.f;
  }
  pdl_wait_primary();
  __syncthreads();
  const T* kpool = static_cast<const T*>(a.k_pool);
  const T* zpool = static_cast<const T*>(a.z_pool);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int jj = au.j0; jj < au.j1; ++jj) {
    const int page = selected_page(a, au, jj);
    const int slot = page_slot(a, au, page);
    const size_t row0 = ((size_t)slot * a.num_kv_heads + au.kvh) * P;
    const int valid = min(P, au.L - page * P);
    for (int idx = threadIdx.x; idx < valid * G; idx += blockDim.x) {
      const int tok = idx / G, h = idx % G;
      float dot = 0.f;
      if (a.k_int8) {
        const int8_t* kc = static_cast<const int8_t*>(a.k_pool) + (row0 + tok) * D;
        for (int c = 0; c < D; ++c) dot = fmaf(qs[h * D + c], (float)kc[c], dot);
        dot *= a.k_scale[row0 + tok];
      } else {
        const T* kr = kpool + (row0 + tok) * D;
        for (int c = 0; c < D; ++c) dot = fmaf(qs[h * D + c], to_f32(kr[c]), dot);
      }
      sc[h * P + tok] = dot * a.scale_log2;
    }
    __syncthreads();
    for (int h = warp; h < G; h += kAttnWarps) {
      float m = -INFINITY;
      for (int tk = lane; tk < valid; tk += 32) m = fmaxf(m, sc[h * P + tk]);
      m = warp_max(m);
      const float m_new = fmaxf(mrun[h], m);
      float sum = 0.f;
      for (int tk = lane; tk < valid; tk += 32) {
        const float p = exp2f(sc[h * P + tk] - m_new);
        sc[h * P + tk] = p;
        sum += p;
      }
      sum = warp_sum(sum);
      if (lane == 0) {
        const float cr = exp2f(mrun[h] - m_new);
        corr[h] = cr;
        lrun[h] = lrun[h] * cr + sum;
        mrun[h] = m_new;
      }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * RR; idx += blockDim.x) {
      const int h = idx / RR, i = idx % RR;
      float acc = accs[idx] * corr[h];
      for (int tk = 0; tk < valid; ++tk) acc = fmaf(sc[h * P + tk], to_f32(zpool[(row0 + tk) * RR + i]), acc);
      accs[idx] = acc;
    }
    __syncthreads();
  }
  const size_t part0 = ((size_t)au.u * a.np_cap + blockIdx.x) * G;
  for (int h = threadIdx.x; h < G; h += blockDim.x) {
    a.part_ml[(part0 + h) * 2] = mrun[h];
    a.part_ml[(part0 + h) * 2 + 1] = lrun[h];
  }
  for (int idx = threadIdx.x; idx < G * RR; idx += blockDim.x) a.part_acc[part0 * RR + idx] = accs[idx];
  write_identity_selection(a, au);
  attn_finish<kAttnThreads>(a, au, 1, reinterpret_cast<float*>(smem), &flag);
}

}  // namespace basiskv
