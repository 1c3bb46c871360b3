// Host side of the BasisKV decode-attention library: argument validation,
// library-owned state, launch shapes and the C ABI declared in basiskv.h.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/basiskv.h"
#include "attn.cuh"
#include "attn_coop.cuh"
#include "encode.cuh"
#include "plan.cuh"
#include "route.cuh"

using namespace basiskv;

namespace {

thread_local std::string g_last_error;

// An NVTX range over the host side of a library call or grid launch, so a
// timeline tool shows which call and which grid each launch belongs to
// (header-only NVTX: without a tool attached a push and a pop cost a branch).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define CUDA_TRY(call)                                                                      \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(BASISKV_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

constexpr int kMaxSplits = 16;
constexpr int kProfEvents = 5;  // start, after prep, after routing, after selection, after attention
constexpr int kPartsCap = kMaxSplits * kAttnWarps;  // partials per unit
constexpr size_t kSchedWords = 2;  // work-claim counters of the persistent routing grid
constexpr int kRouteStaticPct = 75;  // routing pages in static shares when units are long
// Ring bytes per CTA: small rings let several CTAs (and so many warps, each
// with copies in flight) share an SM.
constexpr size_t kRouteSmemBudget = 48 * 1024;
constexpr size_t kAttnSmemBudget = 100 * 1024;
constexpr size_t kAttnSmemBudgetWide = 64 * 1024;  // attention rings when r >= 64
// Cooperative attention: one CTA per SM; its ring takes what is left of the
// SM's shared memory after the merge buffers.
constexpr size_t kCoopSmemPerSm = 212 * 1024;
constexpr long long kCoopMinItems = 8;       // items per CTA at least
constexpr long long kCoopMinUnitItems = 64;  // stages per unit from which the shared ring is used

using KernelFn = void (*)(const RouteArgs);
using AttnFn = void (*)(const AttnArgs);
// A persistent attention kernel chosen at create for this shape.
struct AttnKernel {
  AttnFn plain = nullptr;   // waits for the selection grid
  AttnFn tagged = nullptr;  // reads tagged selection entries as they come
  bool coop = false;        // attn_coop_kernel (shared ring), else attn_mma_kernel (a ring per warp)
  int threads = kAttnThreads, tps = 0, stages = 0, occ = 1;
  size_t smem = 0;
};
struct AttnFns {
  AttnFn plain;   // waits for the selection grid
  AttnFn tagged;  // reads tagged selection entries as they come
};

// ---- compiled tensor-core shapes ------------------------------------------
struct RouteKey {
  int g, r, s, p;
  bool operator<(const RouteKey& o) const { return std::tie(g, r, s, p) < std::tie(o.g, o.r, o.s, o.p); }
};
struct AttnKey {
  int g, d, r, tps;
  bool k8;  // int8 keys
  bool operator<(const AttnKey& o) const {
    return std::tie(g, d, r, tps, k8) < std::tie(o.g, o.d, o.r, o.tps, o.k8);
  }
};

const std::map<RouteKey, KernelFn>& route_table() {
  static const std::map<RouteKey, KernelFn> t = {
#define RK(G, R, S, P) {RouteKey{G, R, S, P}, &route_mma_kernel<G, R, S, P>}
#define RK2(G, R, S) RK(G, R, S, 32), RK(G, R, S, 64)
#ifdef BASISKV_WAIT_TEST
      RK(4, 32, 16, 64),  // the wait-expiry test build holds one shape
#else
      RK2(4, 16, 8),  RK2(4, 24, 8),  RK2(4, 32, 8),  RK2(4, 32, 16), RK2(4, 64, 16),
      RK2(4, 64, 32), RK2(4, 128, 0), RK2(4, 32, 0),  RK2(8, 32, 16), RK2(8, 24, 8),
      RK2(8, 64, 32), RK2(2, 32, 16), RK2(1, 32, 16), RK(4, 32, 16, 16), RK(4, 32, 16, 128),
      RK(4, 24, 8, 16),
#endif
#undef RK2
#undef RK
  };
  return t;
}

const std::map<AttnKey, AttnFns>& attn_table() {
  static const std::map<AttnKey, AttnFns> t = {
#define AK(G, D, R, T) \
  {AttnKey{G, D, R, T, false}, AttnFns{&attn_mma_kernel<G, D, R, T, false, false>, &attn_mma_kernel<G, D, R, T, false, true>}}
#define AK8(G, D, R, T) \
  {AttnKey{G, D, R, T, true}, AttnFns{&attn_mma_kernel<G, D, R, T, true, false>, &attn_mma_kernel<G, D, R, T, true, true>}}
#ifdef BASISKV_WAIT_TEST
      AK(4, 128, 32, 32), AK(4, 128, 32, 64),
#else
      AK(4, 128, 32, 64), AK(4, 128, 32, 32), AK(4, 128, 24, 32), AK(4, 128, 24, 16),
      AK(4, 128, 16, 64), AK(4, 128, 64, 32), AK(4, 128, 128, 32), AK(4, 128, 128, 16),
      AK(4, 64, 16, 16),  AK(4, 64, 32, 32),  AK(8, 128, 32, 64), AK(8, 128, 32, 32),
      AK(8, 128, 24, 32), AK(8, 128, 64, 32), AK(2, 128, 32, 64), AK(1, 128, 32, 64),
      AK8(4, 128, 32, 64), AK8(4, 128, 32, 32), AK8(4, 128, 24, 32), AK8(4, 128, 24, 16),
      AK8(4, 128, 128, 32), AK8(4, 128, 128, 16), AK8(4, 64, 16, 16), AK8(4, 64, 32, 32),
      AK8(8, 128, 32, 32), AK8(1, 128, 32, 64),
#endif
#undef AK8
#undef AK
  };
  return t;
}

// Cooperative attention kernels: key (G, d, r, tokens per stage, int8 keys).
const std::map<AttnKey, AttnFns>& coop_table() {
  static const std::map<AttnKey, AttnFns> t = {
#define CK(G, D, R, T, K8) \
  {AttnKey{G, D, R, T, K8}, AttnFns{&attn_coop_kernel<G, D, R, T, K8, false>, &attn_coop_kernel<G, D, R, T, K8, true>}}
#ifdef BASISKV_WAIT_TEST
      CK(4, 128, 32, 64, false), CK(4, 128, 32, 32, false),
#else
      CK(4, 128, 32, 64, false), CK(4, 128, 32, 32, false), CK(4, 128, 24, 32, false),
      CK(4, 128, 128, 64, false), CK(4, 128, 128, 32, false), CK(4, 64, 16, 16, false),
      CK(4, 128, 32, 64, true), CK(4, 128, 32, 32, true), CK(4, 128, 24, 32, true),
      CK(4, 128, 128, 64, true), CK(4, 128, 128, 32, true), CK(4, 64, 16, 16, true),
#endif
#undef CK
  };
  return t;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A = B^T (B B^T)^-1, the pseudo-inverse of a full-row-rank B [m][d], as
// A [d][m]; double precision, Gauss-Jordan with partial pivoting on the
// Gram matrix.  False when the rows of B are numerically dependent.
bool right_pinv(const float* B, int m, int d, float* A) {
  std::vector<double> G((size_t)m * m), Gi((size_t)m * m, 0.0);
  double gmax = 0.0;
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < m; ++j) {
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += (double)B[(size_t)i * d + c] * B[(size_t)j * d + c];
      G[(size_t)i * m + j] = acc;
      gmax = std::max(gmax, std::fabs(acc));
    }
  for (int i = 0; i < m; ++i) Gi[(size_t)i * m + i] = 1.0;
  for (int col = 0; col < m; ++col) {
    int piv = col;
    for (int row = col + 1; row < m; ++row)
      if (std::fabs(G[(size_t)row * m + col]) > std::fabs(G[(size_t)piv * m + col])) piv = row;
    const double pv = G[(size_t)piv * m + col];
    if (!(std::fabs(pv) > 1e-10 * gmax)) return false;
    for (int c = 0; c < m; ++c) {
      std::swap(G[(size_t)col * m + c], G[(size_t)piv * m + c]);
      std::swap(Gi[(size_t)col * m + c], Gi[(size_t)piv * m + c]);
    }
    for (int c = 0; c < m; ++c) {
      G[(size_t)col * m + c] /= pv;
      Gi[(size_t)col * m + c] /= pv;
    }
    for (int row = 0; row < m; ++row) {
      if (row == col) continue;
      const double f = G[(size_t)row * m + col];
      if (f == 0.0) continue;
      for (int c = 0; c < m; ++c) {
        G[(size_t)row * m + c] -= f * G[(size_t)col * m + c];
        Gi[(size_t)row * m + c] -= f * Gi[(size_t)col * m + c];
      }
    }
  }
  for (int c = 0; c < d; ++c)
    for (int j = 0; j < m; ++j) {
      double acc = 0.0;
      for (int i = 0; i < m; ++i) acc += (double)B[(size_t)i * d + c] * Gi[(size_t)i * m + j];
      A[(size_t)c * m + j] = (float)acc;
    }
  return true;
}

}  // namespace

struct basiskv_handle {
  basiskv_params p;
  int device = 0;
  int num_sms = 148;
  size_t elem = 2;
  // device state
  int32_t* d_page_table = nullptr;  // [max_batch][max_pages]
  int32_t* d_seq_lens = nullptr;    // [max_batch]
  float* d_scores = nullptr;        // [max_batch][Hkv][max_pages]
  uint64_t* d_scores64 = nullptr;   // [max_batch][Hkv][max_pages] scores tagged with the routing call
  uint64_t* d_sel64 = nullptr;      // [max_batch][Hkv][max_topk] selection tagged with the routing call
  int32_t* d_sel = nullptr;         // [max_batch][Hkv][max_topk]
  float* d_part_ml = nullptr;       // [max_batch*Hkv][kPartsCap][G][2]
  float* d_part_acc = nullptr;      // [max_batch*Hkv][kPartsCap][G][r]
  uint32_t* d_counters = nullptr;   // [3][max_batch*Hkv]: route, attention, partial count; then kSchedWords
  uint64_t* d_qf = nullptr;         // [max_batch*Hkv][G][r+s] folded routing queries, tagged with the call
  uint32_t route_tag = 0;           // tag of the last routing launch
  float* d_enc = nullptr;           // pinv(B_v) [Hkv][d][r], then pinv(B_r) [Hkv][d][s] (basiskv_encode_rows)
  bool enc_ready = false;
  uint32_t* d_status = nullptr;
  int32_t* d_route_off = nullptr;   // [max_batch+1]
  int32_t* d_attn_off = nullptr;    // [max_batch+1]
  // host-buffer entry point staging
  void* d_q_stage = nullptr;
  float* d_out_stage = nullptr;
  int32_t* d_sel_stage = nullptr;
  // host mirror (launch sizing, validation)
  std::vector<int32_t> h_table;
  std::vector<int32_t> h_lens;
  std::vector<int32_t> h_npages;
  // kernels chosen at create
  KernelFn route_fn = nullptr;
  AttnKernel attn_warp;  // a ring per warp: every shape it is compiled for
  AttnKernel attn_coop;  // a shared ring per CTA: long units
  int route_stages = 0;
  size_t route_smem = 0;
  int topk_keys = 0;  // scores staged in shared memory by the selection kernel
  int route_occ = 1;  // resident CTAs per SM of the persistent routing kernel
  // profiling
  std::vector<cudaEvent_t> events;  // kProfEvents per recorded call
  int prof_cap = 0, prof_calls = 0;
  int last_launch[6] = {0, 0, 0, 0, 0, 0};
};

namespace {

__global__ void set_entry_kernel(int32_t* table, int32_t* lens, int idx, int slot, int len) {
  if (idx >= 0) table[idx] = slot;
  *lens = len;
}

size_t combine_smem_floats(int np, int g, int r) { return (size_t)np * g + 3 * (size_t)g + (size_t)g * r; }

int validate_params(const basiskv_params* p) {
  if (!p) return fail(BASISKV_ERR_INVALID_ARG, "params is NULL");
  if (p->max_batch <= 0 || p->num_kv_heads <= 0 || p->gqa_group < 1 || p->gqa_group > 8 ||
      p->head_dim <= 0 || p->page_size <= 0 || p->rank_r <= 0 || p->rank_r > p->head_dim ||
      p->rank_s < 0 || p->max_pages_per_seq <= 0 || p->max_topk <= 0 || p->num_slots <= 0)
    return fail(BASISKV_ERR_INVALID_ARG,
                "bad shape: need max_batch, Hkv, d, P, r, max_pages, max_topk, num_slots > 0, "
                "1 <= G <= 8, r <= d, s >= 0");
  if (p->max_batch > 65535 || p->num_kv_heads > 65535)
    return fail(BASISKV_ERR_INVALID_ARG, "max_batch and num_kv_heads must be <= 65535");
  if (p->dtype != BASISKV_DTYPE_BF16 && p->dtype != BASISKV_DTYPE_F32)
    return fail(BASISKV_ERR_INVALID_ARG, "dtype must be BASISKV_DTYPE_BF16 or BASISKV_DTYPE_F32");
  if (p->k_format != BASISKV_KEYS_NATIVE && p->k_format != BASISKV_KEYS_INT8)
    return fail(BASISKV_ERR_INVALID_ARG, "k_format must be BASISKV_KEYS_NATIVE or BASISKV_KEYS_INT8");
  if (p->k_format == BASISKV_KEYS_INT8 && (!p->k_scale || !aligned16(p->k_scale)))
    return fail(BASISKV_ERR_INVALID_ARG, "int8 keys need a 16-byte aligned k_scale");
  if (!p->z_pool || !p->k_pool || !p->w_zk || !p->b_v || (p->rank_s > 0 && (!p->r_pool || !p->b_r)))
    return fail(BASISKV_ERR_INVALID_ARG, "pool or basis pointer is NULL");
  const void* ptrs[] = {p->z_pool, p->k_pool, p->w_zk, p->b_v};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(BASISKV_ERR_INVALID_ARG, "pools and bases must be 16-byte aligned");
  if (p->rank_s > 0 && (!aligned16(p->r_pool) || !aligned16(p->b_r)))
    return fail(BASISKV_ERR_INVALID_ARG, "pools and bases must be 16-byte aligned");
  if ((size_t)p->max_batch * p->max_pages_per_seq * p->num_kv_heads * (p->page_size / 16 + 1) >=
      ((size_t)1 << 31))
    return fail(BASISKV_ERR_INVALID_ARG, "page table too large (work lists must index in 32 bits)");
  return BASISKV_OK;
}

// Pick the tensor-core kernels for this shape when the pools are bf16.
void choose_kernels(basiskv_handle* h) {
  const basiskv_params& p = h->p;
  if (p.dtype != BASISKV_DTYPE_BF16) return;
  const size_t es = 2;
  auto rit = route_table().find(RouteKey{p.gqa_group, p.rank_r, p.rank_s, p.page_size});
  if (rit != route_table().end() && p.page_size % 16 == 0 && (p.head_dim == 128 || p.head_dim == 64)) {
    const size_t stage = (size_t)route_pages_per_stage(p.page_size, p.rank_r, p.rank_s) * p.page_size *
                         (p.rank_r + p.rank_s) * es;
    int st = (int)std::min<size_t>(4, kRouteSmemBudget / (kRouteWarps * stage));
    if (st >= 2) {
      h->route_fn = rit->second;
      h->route_stages = st;
      h->route_smem = kRouteWarps * st * stage;
    }
  }
  const bool k8 = p.k_format == BASISKV_KEYS_INT8;
  // the shared-ring kernel where a shape of it is compiled: 32-token stages
  // where pages allow, one CTA per SM, a ring of a multiple of eight stages
  for (int tps : {32, 64, 16}) {
    if (p.page_size % tps) continue;
    auto cit = coop_table().find(AttnKey{p.gqa_group, p.head_dim, p.rank_r, tps, k8});
    if (cit == coop_table().end()) continue;
    const size_t stage = (size_t)tps * (p.head_dim * (k8 ? 1 : es) + p.rank_r * es + (k8 ? 4 : 0));
    const size_t gr = (size_t)p.gqa_group * p.rank_r;
    const size_t extra =
        sizeof(float) * ((size_t)coop_bufs(p.gqa_group, p.rank_r) * kCoopWarps * (gr + 16) + kCoopMergeWarps * gr);
    if (kCoopSmemPerSm < extra + 2 * kCoopWarps * stage) continue;
    // a multiple of the consumer warps (each warp's stages keep their slots)
    const int st = (int)std::min<size_t>(kCoopMaxStages, (kCoopSmemPerSm - extra) / stage) / kCoopWarps * kCoopWarps;
    AttnKernel& k = h->attn_coop;
    k.plain = cit->second.plain;
    k.tagged = cit->second.tagged;
    k.coop = true;
    k.threads = kCoopThreads;
    k.tps = tps;
    k.stages = st;
    k.smem = st * stage + extra;
    break;
  }
  // Where P.Z is heavy (r >= 64) more resident warps pay for shallower
  // rings: a 64 KB ring lets three CTAs share an SM (dense limit, r = 128:
  // 120 us against 123 us, 111 against 115 with int8 keys); at r = 32 the
  // deeper rings are faster.  The default budget applies when no compiled
  // shape fits the smaller one.
  for (size_t budget : {p.rank_r >= 64 ? kAttnSmemBudgetWide : kAttnSmemBudget, kAttnSmemBudget}) {
    for (int tps : {64, 32, 16}) {
      if (p.page_size % tps) continue;
      auto ait = attn_table().find(AttnKey{p.gqa_group, p.head_dim, p.rank_r, tps, k8});
      if (ait == attn_table().end()) continue;
      const size_t stage = (size_t)tps * (p.head_dim * (k8 ? 1 : es) + p.rank_r * es + (k8 ? 4 : 0));
      int st = (int)std::min<size_t>(4, budget / (kAttnWarps * stage));
      if (st < 1) continue;
      if (st < 2 && tps > 16) continue;  // prefer a smaller stage with double buffering
      AttnKernel& k = h->attn_warp;
      k.plain = ait->second.plain;
      k.tagged = ait->second.tagged;
      k.tps = tps;
      k.stages = st;
      k.smem = kAttnWarps * st * stage + sizeof(float) * kAttnWarps * p.gqa_group * p.rank_r;
      return;
    }
  }
}

// Dynamic shared memory of encode_kernel: the row buffers, plus the KV
// head's A_v, W_zk and A_r when they fit (*stage).
constexpr size_t kEncodeStageMax = 200 * 1024;
size_t encode_smem(const basiskv_params& p, bool* stage) {
  const size_t d = p.head_dim, r = p.rank_r, s = p.rank_s;
  const size_t rows = sizeof(float) * (3 * d + r), bases = sizeof(float) * (2 * d * r + d * s);
  *stage = rows + bases <= kEncodeStageMax;
  return rows + (*stage ? bases : 0);
}

size_t generic_route_smem(const basiskv_params& p) {
  return sizeof(float) * (size_t)p.gqa_group * (p.head_dim + p.rank_r + p.rank_s);
}
size_t generic_attn_smem(const basiskv_params& p) {
  const size_t g = p.gqa_group;
  const size_t own = g * (p.head_dim + p.page_size + p.rank_r) + 3 * g;
  return sizeof(float) * std::max(own, combine_smem_floats(kMaxSplits, p.gqa_group, p.rank_r));
}

// Dynamic shared memory limit, and the largest shared-memory carveout: SMs
// then keep one L1/shared split for all of this library's grids, so a grid
// launched early (programmatic dependent launch) can share SMs with the one
// still finishing.
// The limit belongs to the function, not to a handle, so it is only ever
// raised: a handle with smaller shapes must not lower it under another's.
int set_smem_attr(const void* fn, size_t bytes) {
  cudaFuncAttributes fa;
  CUDA_TRY(cudaFuncGetAttributes(&fa, fn));
  if ((size_t)fa.maxDynamicSharedSizeBytes < bytes)
    CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared));
  return BASISKV_OK;
}

template <typename T>
int set_generic_attrs(const basiskv_params& p) {
  int rc = set_smem_attr((const void*)&route_generic_kernel<T>, generic_route_smem(p));
  if (rc) return rc;
  return set_smem_attr((const void*)&attn_generic_kernel<T>, generic_attn_smem(p));
}

struct LaunchPlan {
  int batch = 0;
  bool any_routed = false;
  long long route_pages = 0;  // routed pages x Hkv (persistent routing work list)
  long long attn_items = 0;   // selected pages x stages x Hkv (persistent attention work list)
  int max_unit_items = 0;
  int sub = 1;                // attention stages per page
  // generic kernels
  int route_ppc = 0, route_chunks = 0;
  int attn_pps = 0, attn_splits = 0;
  // persistent kernels
  int route_ctas = 0, attn_ctas = 0;
  long long attn_chunk = 0;   // shared-ring attention: items per CTA
  const AttnKernel* ak = nullptr;  // the persistent attention kernel, or none (generic)
  int route_static_pct = 100;  // pages of the persistent routing grid handed out in static shares
  int max_routed = 0;          // pages of the longest routed sequence
  // work plans (prefix over sequences), when batch <= kPlanMax
  std::vector<int32_t> route_off, attn_off;
};

LaunchPlan plan(const basiskv_handle* h, int batch, int topk, bool force_route) {
  LaunchPlan lp;
  lp.batch = batch;
  const basiskv_params& p = h->p;
  long long route_pages = 0, pages = 0;
  int max_routed = 0, max_kb = 0;
  for (int b = 0; b < batch; ++b) {
    const int n = h->h_npages[b];
    if (n > 0 && (force_route || topk < n)) {
      route_pages += n;
      max_routed = std::max(max_routed, n);
    }
    const int kb = std::min(topk, n);
    max_kb = std::max(max_kb, kb);
    pages += kb;
  }
  // The shared-ring kernel where units are long; with short units (a few
  // dozen stages) a CTA finishes many units, and the per-warp rings, whose
  // warps each finish their own, end sooner.
  const AttnKernel& co = h->attn_coop;
  if (co.plain && (long long)max_kb * (p.page_size / co.tps) >= kCoopMinUnitItems) lp.ak = &co;
  else if (h->attn_warp.plain) lp.ak = &h->attn_warp;
  lp.sub = lp.ak ? p.page_size / lp.ak->tps : 1;
  const long long items = pages * lp.sub;
  lp.route_pages = route_pages * p.num_kv_heads;
  lp.attn_items = items * p.num_kv_heads;
  if (batch <= kPlanMax) {
    lp.route_off.assign(batch + 1, 0);
    lp.attn_off.assign(batch + 1, 0);
    for (int b = 0; b < batch; ++b) {
      const int n = h->h_npages[b];
      const bool routed = n > 0 && (force_route || topk < n);
      lp.route_off[b + 1] = lp.route_off[b] + (routed ? n : 0) * p.num_kv_heads;
      lp.attn_off[b + 1] = lp.attn_off[b] + std::min(topk, n) * lp.sub * p.num_kv_heads;
    }
  }
  lp.max_unit_items = max_kb * lp.sub;
  lp.any_routed = max_routed > 0;
  // Long units (512 pages and more): a quarter of the routed pages is left
  // to warps that finish their static share early, which evens out the
  // ends of the warps.  Short units gain nothing from it (each claimed
  // chunk starts a new unit, whose folded query must be fetched first).
  lp.route_static_pct = max_routed >= 512 ? kRouteStaticPct : 100;
  lp.max_routed = max_routed;

  // generic kernels: a grid of (chunk | split, Hkv, batch)
  if (lp.any_routed) {
    const long long target = (long long)h->num_sms * 8;
    long long ppc = (lp.route_pages + target - 1) / target;
    ppc = std::max<long long>(kRouteWarps * 2, std::min<long long>(ppc, 512));
    const int chunks = (int)((max_routed + ppc - 1) / ppc);
    lp.route_ppc = (max_routed + chunks - 1) / chunks;
    lp.route_chunks = (max_routed + lp.route_ppc - 1) / lp.route_ppc;
  }
  const long long units = (long long)batch * p.num_kv_heads;
  int splits = (int)std::max<long long>(1, ((long long)h->num_sms * 3 + units - 1) / std::max(1LL, units));
  splits = std::min(splits, kMaxSplits);
  splits = std::max(1, std::min(splits, std::max(1, max_kb)));
  lp.attn_pps = std::max(1, (max_kb + splits - 1) / splits);
  lp.attn_splits = std::max(1, (max_kb + lp.attn_pps - 1) / lp.attn_pps);

  // persistent kernels: every warp streams an equal contiguous share
  const long long min_per_warp = 4;
  lp.route_ctas = (int)std::max<long long>(1, std::min<long long>(
      (long long)h->num_sms * h->route_occ, (lp.route_pages + kRouteWarps * min_per_warp - 1) /
                                                (kRouteWarps * min_per_warp)));
  if (lp.ak && lp.ak->coop) {
    // one chunk of consecutive items per CTA; a unit must meet at most
    // kPartsCap - 2 chunks
    long long ctas = std::min<long long>((long long)h->num_sms * lp.ak->occ,
                                         std::max<long long>(1, lp.attn_items / kCoopMinItems));
    if (lp.max_unit_items > 0) {
      const long long per = (lp.max_unit_items + kPartsCap - 3) / (kPartsCap - 2);
      ctas = std::min<long long>(ctas, std::max<long long>(1, lp.attn_items / per));
    }
    lp.attn_ctas = (int)std::max<long long>(1, ctas);
    lp.attn_chunk = std::max<long long>(1, (lp.attn_items + lp.attn_ctas - 1) / lp.attn_ctas);
    return lp;
  }
  long long attn_warps = std::min<long long>((long long)h->num_sms * (lp.ak ? lp.ak->occ : 1) * kAttnWarps,
                                             std::max<long long>(1, lp.attn_items));
  if (lp.max_unit_items > 0) {
    // a unit must meet at most kPartsCap - 2 warps: each warp gets at least
    // ceil(max_unit_items / (kPartsCap - 2)) items
    const long long per = (lp.max_unit_items + kPartsCap - 3) / (kPartsCap - 2);
    attn_warps = std::min<long long>(attn_warps, std::max<long long>(1, lp.attn_items / per));
  }
  lp.attn_ctas = (int)std::max<long long>(1, (attn_warps + kAttnWarps - 1) / kAttnWarps);
  return lp;
}

int launch_prep(basiskv_handle* h, const LaunchPlan& lp, int topk, int force, float* out, int32_t* sel_out,
                float* fill_scores, int latent, cudaStream_t stream) {
  NvtxRange range("basiskv prep grid");
  const basiskv_params& p = h->p;
  PrepArgs a;
  a.seq_lens = h->d_seq_lens;
  a.route_off = h->d_route_off;
  a.attn_off = h->d_attn_off;
  a.sel_out = sel_out;
  a.out = out;
  a.scores = fill_scores;
  a.batch = lp.batch;
  a.num_kv_heads = p.num_kv_heads;
  a.gqa_group = p.gqa_group;
  a.head_dim = p.head_dim;
  a.page_size = p.page_size;
  a.topk = topk;
  a.force = force;
  a.attn_sub = lp.sub;
  a.ld_pt = p.max_pages_per_seq;
  a.fill_scores = fill_scores != nullptr;
  a.out_width = latent ? p.rank_r : p.head_dim;
  prep_kernel<<<dim3(p.num_kv_heads, lp.batch), kPrepThreads, 0, stream>>>(a);
  CUDA_TRY(cudaGetLastError());
  return BASISKV_OK;
}

RouteArgs route_args(basiskv_handle* h, const LaunchPlan& lp, const void* q, int topk, float* scores,
                     int32_t* sel_out, int force) {
  const basiskv_params& p = h->p;
  RouteArgs a;
  a.q = q;
  a.z_pool = p.z_pool;
  a.r_pool = p.r_pool;
  a.w_zk = p.w_zk;
  a.b_r = p.b_r;
  a.page_table = h->d_page_table;
  a.seq_lens = h->d_seq_lens;
  a.scores = scores;
  a.scores64 = h->d_scores64;
  a.tagged_scores = 0;
  a.sel = h->d_sel;
  a.sel_out = sel_out;
  a.counters = h->d_counters;
  a.sched = h->d_counters + 3 * (size_t)p.max_batch * p.num_kv_heads;
  a.status = h->d_status;
  a.ld_pt = p.max_pages_per_seq;
  a.ld_sel = p.max_topk;
  a.num_slots = p.num_slots;
  a.num_kv_heads = p.num_kv_heads;
  a.head_dim = p.head_dim;
  a.page_size = p.page_size;
  a.rank_r = p.rank_r;
  a.rank_s = p.rank_s;
  a.gqa_group = p.gqa_group;
  a.topk = topk;
  a.pages_per_cta = lp.route_ppc;
  a.stages = h->route_stages;
  a.static_pct = lp.route_static_pct;
  a.force = force;
  a.fill_tail = force;
  a.batch = lp.batch;
  a.route_off = h->d_route_off;
  a.qf = h->d_qf;
  if (++h->route_tag == 0) h->route_tag = 1;  // 0 never matches: the folded queries start zeroed
  a.tag = h->route_tag;
  a.plan_n = lp.route_off.empty() ? -1 : lp.batch;
  for (size_t i = 0; i < lp.route_off.size(); ++i) a.plan_off[i] = lp.route_off[i];
  return a;
}

cudaLaunchConfig_t launch_cfg(dim3 grid, int threads, size_t smem, cudaStream_t stream, bool pdl,
                              cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cfg;
}

// Routing after the prep grid: the persistent tensor-core kernel (PDL: it
// waits for the prep grid before reading the plan), else the generic one.
int launch_route(basiskv_handle* h, const LaunchPlan& lp, const RouteArgs& a, bool pdl, cudaStream_t stream) {
  NvtxRange range("basiskv routing grid");
  const basiskv_params& p = h->p;
  cudaLaunchAttribute attr[1];
  if (h->route_fn) {
    cudaLaunchConfig_t cfg = launch_cfg(dim3(lp.route_ctas), kRouteThreads, h->route_smem, stream, pdl, attr);
    CUDA_TRY(cudaLaunchKernelEx(&cfg, h->route_fn, a));
    return BASISKV_OK;
  }
  dim3 grid(lp.route_chunks, p.num_kv_heads, lp.batch);
  if (p.dtype == BASISKV_DTYPE_BF16)
    route_generic_kernel<__nv_bfloat16><<<grid, kRouteThreads, generic_route_smem(p), stream>>>(a);
  else
    route_generic_kernel<float><<<grid, kRouteThreads, generic_route_smem(p), stream>>>(a);
  CUDA_TRY(cudaGetLastError());
  return BASISKV_OK;
}

// Selection for the persistent routing kernel (PDL behind it).
int launch_topk(basiskv_handle* h, const LaunchPlan& lp, int topk, const float* scores, int32_t* sel_out,
                int force, bool pdl, bool poll, cudaStream_t stream) {
  NvtxRange range("basiskv selection grid");
  const basiskv_params& p = h->p;
  TopkArgs a;
  a.scores = scores;
  a.scores64 = h->d_scores64;
  a.poll = poll;
  a.sel64 = poll ? h->d_sel64 : nullptr;
  a.tag = h->route_tag;
  a.status = h->d_status;
  a.seq_lens = h->d_seq_lens;
  a.sel = h->d_sel;
  a.sel_out = sel_out;
  a.num_kv_heads = p.num_kv_heads;
  a.page_size = p.page_size;
  a.ld_pt = p.max_pages_per_seq;
  a.ld_sel = p.max_topk;
  a.topk = topk;
  a.force = force;
  a.keys_cap = h->topk_keys;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_cfg(dim3(p.num_kv_heads, lp.batch), kTopkThreads,
                                      sizeof(uint32_t) * (size_t)h->topk_keys, stream, pdl, attr);
  CUDA_TRY(cudaLaunchKernelEx(&cfg, &topk_kernel, a));
  return BASISKV_OK;
}

int launch_attn(basiskv_handle* h, const LaunchPlan& lp, const void* q, int topk, float scale, int latent,
                float* out, int32_t* sel_out, bool pdl, bool tagged_sel, cudaStream_t stream) {
  NvtxRange range("basiskv attention grid");
  const basiskv_params& p = h->p;
  const size_t U = (size_t)p.max_batch * p.num_kv_heads;
  AttnArgs a;
  a.q = q;
  a.k_pool = p.k_pool;
  a.k_scale = p.k_scale;
  a.k_int8 = p.k_format == BASISKV_KEYS_INT8;
  a.z_pool = p.z_pool;
  a.b_v = p.b_v;
  a.page_table = h->d_page_table;
  a.seq_lens = h->d_seq_lens;
  a.sel = h->d_sel;
  a.sel64 = tagged_sel ? h->d_sel64 : nullptr;
  a.sel_tag = h->route_tag;
  a.sel_out = sel_out;
  a.part_ml = h->d_part_ml;
  a.part_acc = h->d_part_acc;
  a.counters = h->d_counters + U;
  a.status = h->d_status;
  a.out = out;
  a.ld_pt = p.max_pages_per_seq;
  a.ld_sel = p.max_topk;
  a.num_slots = p.num_slots;
  a.num_kv_heads = p.num_kv_heads;
  a.head_dim = p.head_dim;
  a.page_size = p.page_size;
  a.rank_r = p.rank_r;
  a.gqa_group = p.gqa_group;
  a.topk = topk;
  a.pages_per_split = lp.attn_pps;
  a.stages = lp.ak ? lp.ak->stages : 0;
  a.np_cap = kPartsCap;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.latent = latent;
  a.batch = lp.batch;
  a.attn_off = h->d_attn_off;
  a.plan_n = lp.attn_off.empty() ? -1 : lp.batch;
  a.chunk_items = (int)lp.attn_chunk;
  for (size_t i = 0; i < lp.attn_off.size(); ++i) a.plan_off[i] = lp.attn_off[i];

  cudaLaunchAttribute attr[1];
  if (lp.ak) {
    cudaLaunchConfig_t cfg = launch_cfg(dim3(lp.attn_ctas), lp.ak->threads, lp.ak->smem, stream, pdl, attr);
    CUDA_TRY(cudaLaunchKernelEx(&cfg, tagged_sel ? lp.ak->tagged : lp.ak->plain, a));
    return BASISKV_OK;
  }
  cudaLaunchConfig_t cfg = launch_cfg(dim3(lp.attn_splits, p.num_kv_heads, lp.batch), kAttnThreads,
                                      generic_attn_smem(p), stream, false, attr);
  if (p.dtype == BASISKV_DTYPE_BF16)
    CUDA_TRY(cudaLaunchKernelEx(&cfg, &attn_generic_kernel<__nv_bfloat16>, a));
  else
    CUDA_TRY(cudaLaunchKernelEx(&cfg, &attn_generic_kernel<float>, a));
  return BASISKV_OK;
}

int check_handle(basiskv_handle* h) {
  if (!h) return fail(BASISKV_ERR_INVALID_ARG, "handle is NULL");
  int dev = -1;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev != h->device) return fail(BASISKV_ERR_INVALID_ARG, "handle belongs to device %d, current is %d", h->device, dev);
  return BASISKV_OK;
}

int check_call(basiskv_handle* h, int batch, const void* q, int topk) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (batch < 0 || batch > h->p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "batch %d outside [0, %d]", batch, h->p.max_batch);
  if (topk <= 0 || topk > h->p.max_topk) return fail(BASISKV_ERR_INVALID_ARG, "topk %d outside [1, %d]", topk, h->p.max_topk);
  if (!q || !aligned16(q)) return fail(BASISKV_ERR_INVALID_ARG, "q must be a 16-byte aligned device pointer");
  return BASISKV_OK;
}

}  // namespace

extern "C" {

int basiskv_version(void) { return BASISKV_VERSION; }

const char* basiskv_last_error(void) { return g_last_error.c_str(); }

int basiskv_create(const basiskv_params* p, basiskv_handle** out) {
  if (!out) return fail(BASISKV_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  int rc = validate_params(p);
  if (rc) return rc;
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10)
    return fail(BASISKV_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                prop.major, prop.minor);

  basiskv_handle* h = new basiskv_handle();
  h->p = *p;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->elem = p->dtype == BASISKV_DTYPE_BF16 ? 2 : 4;
  const size_t B = p->max_batch, Hkv = p->num_kv_heads, U = B * Hkv, G = p->gqa_group;
  auto cleanup_fail = [&](int code, const char* what) {
    basiskv_destroy(h);
    return fail(code, "%s", what);
  };
  struct A {
    void** ptr;
    size_t bytes;
  } allocs[] = {
      {(void**)&h->d_page_table, sizeof(int32_t) * B * p->max_pages_per_seq},
      {(void**)&h->d_seq_lens, sizeof(int32_t) * B},
      {(void**)&h->d_scores, sizeof(float) * U * p->max_pages_per_seq},
      {(void**)&h->d_scores64, sizeof(uint64_t) * U * p->max_pages_per_seq},
      {(void**)&h->d_sel64, sizeof(uint64_t) * U * p->max_topk},
      {(void**)&h->d_sel, sizeof(int32_t) * U * p->max_topk},
      {(void**)&h->d_part_ml, sizeof(float) * U * kPartsCap * G * 2},
      {(void**)&h->d_part_acc, sizeof(float) * U * kPartsCap * G * p->rank_r},
      {(void**)&h->d_counters, sizeof(uint32_t) * (3 * U + kSchedWords)},
      {(void**)&h->d_qf, sizeof(uint64_t) * U * G * (p->rank_r + p->rank_s)},
      {(void**)&h->d_enc, sizeof(float) * Hkv * p->head_dim * (p->rank_r + p->rank_s)},
      {(void**)&h->d_status, sizeof(uint32_t)},
      {(void**)&h->d_route_off, sizeof(int32_t) * (B + 1)},
      {(void**)&h->d_attn_off, sizeof(int32_t) * (B + 1)},
      {(void**)&h->d_q_stage, h->elem * B * Hkv * G * p->head_dim},
      {(void**)&h->d_out_stage, sizeof(float) * B * Hkv * G * p->head_dim},
      {(void**)&h->d_sel_stage, sizeof(int32_t) * U * p->max_topk},
  };
  for (auto& a : allocs) {
    if (cudaMalloc(a.ptr, a.bytes) != cudaSuccess) {
      cudaGetLastError();
      return cleanup_fail(BASISKV_ERR_OOM, "device allocation failed");
    }
  }
  if (cudaMemset(h->d_page_table, 0, sizeof(int32_t) * B * p->max_pages_per_seq) != cudaSuccess ||
      cudaMemset(h->d_seq_lens, 0, sizeof(int32_t) * B) != cudaSuccess ||
      cudaMemset(h->d_counters, 0, sizeof(uint32_t) * (3 * U + kSchedWords)) != cudaSuccess ||
      cudaMemset(h->d_qf, 0, sizeof(uint64_t) * U * G * (p->rank_r + p->rank_s)) != cudaSuccess ||
      cudaMemset(h->d_scores64, 0, sizeof(uint64_t) * U * p->max_pages_per_seq) != cudaSuccess ||
      cudaMemset(h->d_sel64, 0, sizeof(uint64_t) * U * p->max_topk) != cudaSuccess ||
      cudaMemset(h->d_status, 0, sizeof(uint32_t)) != cudaSuccess)
    return cleanup_fail(BASISKV_ERR_CUDA, "cudaMemset failed");
  h->h_table.assign(B * p->max_pages_per_seq, 0);
  h->h_lens.assign(B, 0);
  h->h_npages.assign(B, 0);

  h->topk_keys = std::min(p->max_pages_per_seq, 16384);
  choose_kernels(h);
  int arc = h->route_fn ? set_smem_attr((const void*)h->route_fn, h->route_smem) : BASISKV_OK;
  for (AttnKernel* k : {&h->attn_warp, &h->attn_coop}) {
    if (!arc && k->plain) arc = set_smem_attr((const void*)k->plain, k->smem);
    if (!arc && k->tagged) arc = set_smem_attr((const void*)k->tagged, k->smem);
  }
  if (!arc)
    arc = set_smem_attr((const void*)&prep_kernel, 0);
  if (!arc) arc = set_smem_attr((const void*)&topk_kernel, sizeof(uint32_t) * (size_t)h->topk_keys);
  if (!arc && h->route_fn &&
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&h->route_occ, h->route_fn, kRouteThreads, h->route_smem) != cudaSuccess)
    arc = fail(BASISKV_ERR_CUDA, "occupancy query failed");
  for (AttnKernel* k : {&h->attn_warp, &h->attn_coop}) {
    if (arc || !k->plain) continue;
    // one grid size for both variants: the smaller residency of the two
    int occ = 0, occ_ts = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k->plain, k->threads, k->smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_ts, k->tagged, k->threads, k->smem) != cudaSuccess)
      arc = fail(BASISKV_ERR_CUDA, "occupancy query failed");
    else
      k->occ = std::max(1, std::min(occ, occ_ts));
  }
  if (!arc)
    arc = p->dtype == BASISKV_DTYPE_BF16 ? set_generic_attrs<__nv_bfloat16>(*p) : set_generic_attrs<float>(*p);
  if (!arc) {
    bool stage = false;
    const size_t esmem = encode_smem(*p, &stage);
    arc = p->dtype == BASISKV_DTYPE_BF16 ? set_smem_attr((const void*)&encode_kernel<__nv_bfloat16>, esmem)
                                        : set_smem_attr((const void*)&encode_kernel<float>, esmem);
  }
  if (arc) {
    std::string msg = g_last_error;
    basiskv_destroy(h);
    return fail(arc, "%s", msg.c_str());
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return cleanup_fail(BASISKV_ERR_CUDA, "device synchronize failed");
  *out = h;
  return BASISKV_OK;
}

int basiskv_destroy(basiskv_handle* h) {
  if (!h) return BASISKV_OK;
  cudaDeviceSynchronize();
  void* ptrs[] = {h->d_page_table, h->d_seq_lens, h->d_scores, h->d_sel, h->d_part_ml, h->d_part_acc,
                  h->d_counters, h->d_status, h->d_q_stage, h->d_out_stage, h->d_sel_stage,
                  h->d_route_off, h->d_attn_off, h->d_qf, h->d_scores64, h->d_sel64, h->d_enc};
  for (void* q : ptrs)
    if (q) cudaFree(q);
  for (cudaEvent_t e : h->events) cudaEventDestroy(e);
  delete h;
  return BASISKV_OK;
}

int basiskv_append_page(basiskv_handle* h, int seq, int slot, int n_tokens, basiskv_stream_t stream) {
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  if (seq < 0 || seq >= p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "seq %d outside [0, %d)", seq, p.max_batch);
  if (slot < 0 || slot >= p.num_slots) return fail(BASISKV_ERR_INVALID_ARG, "slot %d outside [0, %d)", slot, p.num_slots);
  if (n_tokens < 1 || n_tokens > p.page_size)
    return fail(BASISKV_ERR_INVALID_ARG, "n_tokens %d outside [1, %d]", n_tokens, p.page_size);
  const int n = h->h_npages[seq];
  if (n > 0 && h->h_lens[seq] != n * p.page_size)
    return fail(BASISKV_ERR_STATE, "sequence %d ends in a partial page", seq);
  if (n >= p.max_pages_per_seq) return fail(BASISKV_ERR_CAPACITY, "sequence %d already has %d pages", seq, n);
  const int idx = seq * p.max_pages_per_seq + n;
  const int len = h->h_lens[seq] + n_tokens;
  set_entry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(h->d_page_table, h->d_seq_lens + seq, idx, slot, len);
  CUDA_TRY(cudaGetLastError());
  h->h_table[idx] = slot;
  h->h_lens[seq] = len;
  h->h_npages[seq] = n + 1;
  return BASISKV_OK;
}

int basiskv_append_page_copy(basiskv_handle* h, int seq, int slot, int n_tokens, const void* z, const void* r,
                             const void* k, const float* k_scale, basiskv_stream_t stream) {
  NvtxRange range("basiskv_append_page_copy");
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  const bool int8 = p.k_format == BASISKV_KEYS_INT8;
  if (!z || !k || (p.rank_s > 0 && !r) || (int8 && !k_scale))
    return fail(BASISKV_ERR_INVALID_ARG, "z, k (and r when s > 0, k_scale with int8 keys) are required");
  // the checks of basiskv_append_page, before anything is copied
  if (seq < 0 || seq >= p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "seq %d outside [0, %d)", seq, p.max_batch);
  if (slot < 0 || slot >= p.num_slots) return fail(BASISKV_ERR_INVALID_ARG, "slot %d outside [0, %d)", slot, p.num_slots);
  if (n_tokens < 1 || n_tokens > p.page_size)
    return fail(BASISKV_ERR_INVALID_ARG, "n_tokens %d outside [1, %d]", n_tokens, p.page_size);
  const int n = h->h_npages[seq];
  if (n > 0 && h->h_lens[seq] != n * p.page_size)
    return fail(BASISKV_ERR_STATE, "sequence %d ends in a partial page", seq);
  if (n >= p.max_pages_per_seq) return fail(BASISKV_ERR_CAPACITY, "sequence %d already has %d pages", seq, n);
  // one strided copy per pool: source [Hkv][n_tokens][w], destination rows
  // [0, n_tokens) of the slot's page of every KV head
  cudaStream_t st = (cudaStream_t)stream;
  auto copy = [&](void* pool, const void* src, size_t row_bytes) -> int {
    uint8_t* dst = static_cast<uint8_t*>(pool) + (size_t)slot * p.num_kv_heads * p.page_size * row_bytes;
    CUDA_TRY(cudaMemcpy2DAsync(dst, p.page_size * row_bytes, src, n_tokens * row_bytes, n_tokens * row_bytes,
                               p.num_kv_heads, cudaMemcpyDeviceToDevice, st));
    return BASISKV_OK;
  };
  rc = copy(const_cast<void*>(p.z_pool), z, h->elem * p.rank_r);
  if (!rc && p.rank_s > 0) rc = copy(const_cast<void*>(p.r_pool), r, h->elem * p.rank_s);
  if (!rc) rc = copy(const_cast<void*>(p.k_pool), k, (int8 ? 1 : h->elem) * p.head_dim);
  if (!rc && int8) rc = copy(const_cast<float*>(p.k_scale), k_scale, sizeof(float));
  if (rc) return rc;
  return basiskv_append_page(h, seq, slot, n_tokens, stream);
}

int basiskv_append_tokens(basiskv_handle* h, int seq, int n_tokens, basiskv_stream_t stream) {
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  if (seq < 0 || seq >= p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "seq %d outside [0, %d)", seq, p.max_batch);
  if (n_tokens < 1) return fail(BASISKV_ERR_INVALID_ARG, "n_tokens must be >= 1");
  const int n = h->h_npages[seq];
  if (n == 0) return fail(BASISKV_ERR_STATE, "sequence %d has no page", seq);
  const int len = h->h_lens[seq] + n_tokens;
  if (len > n * p.page_size) return fail(BASISKV_ERR_STATE, "last page of sequence %d would overflow", seq);
  set_entry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(h->d_page_table, h->d_seq_lens + seq, -1, 0, len);
  CUDA_TRY(cudaGetLastError());
  h->h_lens[seq] = len;
  return BASISKV_OK;
}

int basiskv_reset_seq(basiskv_handle* h, int seq, basiskv_stream_t stream) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (seq < 0 || seq >= h->p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "seq %d outside [0, %d)", seq, h->p.max_batch);
  set_entry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(h->d_page_table, h->d_seq_lens + seq, -1, 0, 0);
  CUDA_TRY(cudaGetLastError());
  h->h_lens[seq] = 0;
  h->h_npages[seq] = 0;
  return BASISKV_OK;
}

int basiskv_load_page_table(basiskv_handle* h, int batch, const int32_t* page_table, int ld,
                            const int32_t* seq_lens, basiskv_stream_t stream) {
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  if (batch < 0 || batch > p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "batch %d outside [0, %d]", batch, p.max_batch);
  if (batch > 0 && (!page_table || !seq_lens || ld <= 0)) return fail(BASISKV_ERR_INVALID_ARG, "NULL table or lens");
  std::vector<int32_t> tab((size_t)batch * p.max_pages_per_seq, 0), lens(batch), np(batch);
  for (int b = 0; b < batch; ++b) {
    const int L = seq_lens[b];
    if (L < 0) return fail(BASISKV_ERR_INVALID_ARG, "seq_lens[%d] = %d", b, L);
    const int n = (L + p.page_size - 1) / p.page_size;
    if (n > p.max_pages_per_seq || n > ld)
      return fail(BASISKV_ERR_CAPACITY, "sequence %d needs %d pages (max %d, ld %d)", b, n, p.max_pages_per_seq, ld);
    for (int j = 0; j < n; ++j) {
      const int s = page_table[(size_t)b * ld + j];
      if (s < 0 || s >= p.num_slots) return fail(BASISKV_ERR_INVALID_ARG, "page_table[%d][%d] = %d outside [0, %d)", b, j, s, p.num_slots);
      tab[(size_t)b * p.max_pages_per_seq + j] = s;
    }
    lens[b] = L;
    np[b] = n;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (batch > 0) {
    CUDA_TRY(cudaMemcpyAsync(h->d_page_table, tab.data(), sizeof(int32_t) * tab.size(), cudaMemcpyHostToDevice, st));
    CUDA_TRY(cudaMemcpyAsync(h->d_seq_lens, lens.data(), sizeof(int32_t) * batch, cudaMemcpyHostToDevice, st));
  }
  CUDA_TRY(cudaStreamSynchronize(st));
  std::copy(tab.begin(), tab.end(), h->h_table.begin());
  std::copy(lens.begin(), lens.end(), h->h_lens.begin());
  std::copy(np.begin(), np.end(), h->h_npages.begin());
  return BASISKV_OK;
}

// The decode step behind basiskv_decode_attn (latent = 0: out = zbar.B_v,
// [batch][Hq][d]) and basiskv_decode_attn_latent (latent = 1: out = zbar,
// [batch][Hq][r]).
static int decode_step(basiskv_handle* h, int batch, const void* q, int topk, float softmax_scale, float* out,
                       int32_t* sel_out, basiskv_stream_t stream, int latent) {
  NvtxRange range(latent ? "basiskv_decode_attn_latent" : "basiskv_decode_attn");
  int rc = check_call(h, batch, q, topk);
  if (rc) return rc;
  if (!out) return fail(BASISKV_ERR_INVALID_ARG, "out is NULL");
  if (!std::isfinite(softmax_scale)) return fail(BASISKV_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (batch == 0) return BASISKV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const LaunchPlan lp = plan(h, batch, topk, false);
  const bool prof = h->prof_calls < h->prof_cap;
  cudaEvent_t* ev = prof ? &h->events[kProfEvents * h->prof_calls] : nullptr;
  if (prof) CUDA_TRY(cudaEventRecord(ev[0], st));
  const bool route_tc = lp.any_routed && h->route_fn;
  // the persistent grids read the work plan from their parameters; only a
  // batch too large for that needs the prep grid to write it
  const bool use_prep = (route_tc || lp.ak) && lp.route_off.empty();
  if (use_prep) {
    rc = launch_prep(h, lp, topk, 0, out, sel_out, nullptr, latent, st);
    if (rc) return rc;
  }
  if (prof) CUDA_TRY(cudaEventRecord(ev[1], st));
  // the first grid of a call never overlaps the caller's previous work
  // The tensor-core routing grid tags its scores with the call, and the
  // selection grid then takes each unit as soon as its scores are all
  // there (the selection kernel's shared memory holds the longest unit).
  const bool poll = route_tc && lp.max_routed <= h->topk_keys;
  if (lp.any_routed) {
    RouteArgs ra = route_args(h, lp, q, topk, h->d_scores, sel_out, 0);
    ra.tagged_scores = poll;
    rc = launch_route(h, lp, ra, use_prep && !prof, st);
    if (rc) return rc;
  }
  if (prof) CUDA_TRY(cudaEventRecord(ev[2], st));
  if (route_tc) {
    rc = launch_topk(h, lp, topk, h->d_scores, sel_out, 0, !prof, poll, st);
    if (rc) return rc;
  }
  if (prof) CUDA_TRY(cudaEventRecord(ev[3], st));
  // PDL only behind a routing grid (which signals after any prep grid has
  // finished, so the plan is complete when this grid starts)
  rc = launch_attn(h, lp, q, topk, softmax_scale, latent, out, sel_out, lp.any_routed && !prof, poll, st);
  if (rc) return rc;
  if (prof) {
    CUDA_TRY(cudaEventRecord(ev[4], st));
    ++h->prof_calls;
  }
  h->last_launch[0] = lp.any_routed ? (h->route_fn ? 0 : lp.route_ppc) : 0;
  h->last_launch[1] = lp.any_routed ? (h->route_fn ? lp.route_ctas : lp.route_chunks * h->p.num_kv_heads * batch) : 0;
  h->last_launch[2] = lp.ak ? 0 : lp.attn_splits;
  h->last_launch[3] = lp.ak ? lp.attn_ctas : lp.attn_splits * h->p.num_kv_heads * batch;
  h->last_launch[4] = h->route_fn != nullptr;
  h->last_launch[5] = lp.ak ? (lp.ak->coop ? 2 : 1) : 0;
  return BASISKV_OK;
}

int basiskv_decode_attn(basiskv_handle* h, int batch, const void* q, int topk, float softmax_scale,
                        float* out, int32_t* sel_out, basiskv_stream_t stream) {
  return decode_step(h, batch, q, topk, softmax_scale, out, sel_out, stream, 0);
}

int basiskv_decode_attn_latent(basiskv_handle* h, int batch, const void* q, int topk, float softmax_scale,
                               float* zbar_out, int32_t* sel_out, basiskv_stream_t stream) {
  return decode_step(h, batch, q, topk, softmax_scale, zbar_out, sel_out, stream, 1);
}

}  // extern "C"

namespace {

// The pseudo-inverses of the bases, once per handle, on the host (a set-up
// step, synchronous).
int ensure_encode_bases(basiskv_handle* h) {
  if (h->enc_ready) return BASISKV_OK;
  const basiskv_params& p = h->p;
  const int Hkv = p.num_kv_heads, d = p.head_dim, r = p.rank_r, s = p.rank_s;
  std::vector<float> bv((size_t)Hkv * r * d), br((size_t)Hkv * s * d), enc((size_t)Hkv * d * (r + s));
  CUDA_TRY(cudaMemcpy(bv.data(), p.b_v, sizeof(float) * bv.size(), cudaMemcpyDeviceToHost));
  if (s > 0) CUDA_TRY(cudaMemcpy(br.data(), p.b_r, sizeof(float) * br.size(), cudaMemcpyDeviceToHost));
  for (int kvh = 0; kvh < Hkv; ++kvh) {
    if (!right_pinv(bv.data() + (size_t)kvh * r * d, r, d, enc.data() + (size_t)kvh * d * r))
      return fail(BASISKV_ERR_INVALID_ARG, "the rows of B_v of KV head %d are linearly dependent", kvh);
    if (s > 0 && !right_pinv(br.data() + (size_t)kvh * s * d, s, d,
                             enc.data() + (size_t)Hkv * d * r + (size_t)kvh * d * s))
      return fail(BASISKV_ERR_INVALID_ARG, "the rows of B_r of KV head %d are linearly dependent", kvh);
  }
  CUDA_TRY(cudaMemcpy(h->d_enc, enc.data(), sizeof(float) * enc.size(), cudaMemcpyHostToDevice));
  h->enc_ready = true;
  return BASISKV_OK;
}


// Fill the pool fields of `a`, size the grid (a few tokens per CTA once
// there are more token-heads than two waves of CTAs) and launch.
int launch_encode(basiskv_handle* h, EncodeArgs& a, cudaStream_t st) {
  int rc = ensure_encode_bases(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  const int Hkv = p.num_kv_heads, d = p.head_dim, r = p.rank_r, s = p.rank_s;
  a.k_pool = const_cast<void*>(p.k_pool);
  a.k_scale = const_cast<float*>(p.k_scale);
  a.k_int8 = p.k_format == BASISKV_KEYS_INT8;
  a.z_pool = const_cast<void*>(p.z_pool);
  a.r_pool = const_cast<void*>(p.r_pool);
  a.a_v = h->d_enc;
  a.a_r = h->d_enc + (size_t)Hkv * d * r;
  a.w_zk = p.w_zk;
  a.num_kv_heads = Hkv;
  a.page_size = p.page_size;
  a.head_dim = d;
  a.rank_r = r;
  a.rank_s = s;
  a.num_slots = p.num_slots;
  a.status = h->d_status;
  const long long heads = (long long)a.n * Hkv, wave = 2LL * h->num_sms;
  a.tokens_per_cta = (int)std::max<long long>(1, (heads + wave - 1) / wave);
  bool stage = false;
  const size_t smem = encode_smem(p, &stage);
  a.stage = stage;
  const dim3 grid((a.n + a.tokens_per_cta - 1) / a.tokens_per_cta, Hkv);
  if (p.dtype == BASISKV_DTYPE_BF16) encode_kernel<__nv_bfloat16><<<grid, kEncodeThreads, smem, st>>>(a);
  else encode_kernel<float><<<grid, kEncodeThreads, smem, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return BASISKV_OK;
}

}  // namespace

extern "C" {

int basiskv_encode_rows(basiskv_handle* h, int slot, int row0, int n_rows, const void* k, const void* v,
                        basiskv_stream_t stream) {
  NvtxRange range("basiskv_encode_rows");
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  if (slot < 0 || slot >= p.num_slots) return fail(BASISKV_ERR_INVALID_ARG, "slot %d outside [0, %d)", slot, p.num_slots);
  if (n_rows < 1 || row0 < 0 || row0 + n_rows > p.page_size)
    return fail(BASISKV_ERR_INVALID_ARG, "rows [%d, %d) outside a page of %d", row0, row0 + n_rows, p.page_size);
  if (!k || !v) return fail(BASISKV_ERR_INVALID_ARG, "k or v is NULL");
  EncodeArgs a{};
  a.k = k;
  a.v = v;
  a.tok_stride = p.head_dim;
  a.head_stride = (long long)n_rows * p.head_dim;
  a.slot = slot;
  a.row0 = row0;
  a.n = n_rows;
  return launch_encode(h, a, (cudaStream_t)stream);
}

int basiskv_encode_tokens(basiskv_handle* h, int n, const int32_t* slots, const int32_t* rows, const void* k,
                          const void* v, basiskv_stream_t stream) {
  NvtxRange range("basiskv_encode_tokens");
  int rc = check_handle(h);
  if (rc) return rc;
  if (n < 0) return fail(BASISKV_ERR_INVALID_ARG, "n %d < 0", n);
  if (n == 0) return BASISKV_OK;
  if (!slots || !rows || !k || !v) return fail(BASISKV_ERR_INVALID_ARG, "slots, rows, k or v is NULL");
  const basiskv_params& p = h->p;
  EncodeArgs a{};
  a.k = k;
  a.v = v;
  a.tok_stride = (long long)p.num_kv_heads * p.head_dim;
  a.head_stride = p.head_dim;
  a.slots = slots;
  a.rows = rows;
  a.n = n;
  return launch_encode(h, a, (cudaStream_t)stream);
}

int basiskv_quantize_keys(basiskv_handle* h, const void* k, int64_t row0, int64_t n_rows,
                          basiskv_stream_t stream) {
  NvtxRange range("basiskv_quantize_keys");
  int rc = check_handle(h);
  if (rc) return rc;
  const basiskv_params& p = h->p;
  if (p.k_format != BASISKV_KEYS_INT8) return fail(BASISKV_ERR_INVALID_ARG, "the handle's keys are not int8");
  const long long rows = (long long)p.num_slots * p.num_kv_heads * p.page_size;
  if (!k || !aligned16(k)) return fail(BASISKV_ERR_INVALID_ARG, "k must be a 16-byte aligned device pointer");
  if (n_rows < 0 || row0 < 0 || row0 + n_rows > rows)
    return fail(BASISKV_ERR_INVALID_ARG, "rows [%lld, %lld) outside the pool's %lld", (long long)row0,
                (long long)(row0 + n_rows), rows);
  if (n_rows == 0) return BASISKV_OK;
  QuantizeArgs a;
  a.k = k;
  a.codes = static_cast<int8_t*>(const_cast<void*>(p.k_pool));
  a.scales = const_cast<float*>(p.k_scale);
  a.row0 = row0;
  a.n = n_rows;
  a.head_dim = p.head_dim;
  constexpr int rows_per_cta = kEncodeThreads / 32 * kQuantRowsPerWarp;
  const long long ctas = (n_rows + rows_per_cta - 1) / rows_per_cta;
  if (ctas > 0x7fffffffLL) return fail(BASISKV_ERR_INVALID_ARG, "too many rows for one call");
  cudaStream_t st = (cudaStream_t)stream;
  if (p.dtype == BASISKV_DTYPE_BF16)
    quantize_rows_kernel<__nv_bfloat16><<<(unsigned)ctas, kEncodeThreads, 0, st>>>(a);
  else
    quantize_rows_kernel<float><<<(unsigned)ctas, kEncodeThreads, 0, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return BASISKV_OK;
}

int basiskv_decode_attn_host(basiskv_handle* h, int batch, const void* q_host, int topk, float softmax_scale,
                             float* out_host, int32_t* sel_host, basiskv_stream_t stream) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (!q_host || !out_host) return fail(BASISKV_ERR_INVALID_ARG, "q_host or out_host is NULL");
  if (batch < 0 || batch > h->p.max_batch) return fail(BASISKV_ERR_INVALID_ARG, "batch %d outside [0, %d]", batch, h->p.max_batch);
  cudaStream_t st = (cudaStream_t)stream;
  const size_t rows = (size_t)batch * h->p.num_kv_heads * h->p.gqa_group;
  CUDA_TRY(cudaMemcpyAsync(h->d_q_stage, q_host, h->elem * rows * h->p.head_dim, cudaMemcpyHostToDevice, st));
  // Pinned (page-locked) result buffers are written by the kernels through
  // their device mapping, so no copy follows the step; pageable ones go
  // through the library's staging buffers.
  auto mapped = [](void* host) -> void* {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
  };
  float* dout = static_cast<float*>(mapped(out_host));
  int32_t* dsel = sel_host ? static_cast<int32_t*>(mapped(sel_host)) : nullptr;
  rc = basiskv_decode_attn(h, batch, h->d_q_stage, topk, softmax_scale, dout ? dout : h->d_out_stage,
                           sel_host ? (dsel ? dsel : h->d_sel_stage) : nullptr, stream);
  if (rc) return rc;
  if (!dout)
    CUDA_TRY(cudaMemcpyAsync(out_host, h->d_out_stage, sizeof(float) * rows * h->p.head_dim, cudaMemcpyDeviceToHost,
                             st));
  if (sel_host && !dsel)
    CUDA_TRY(cudaMemcpyAsync(sel_host, h->d_sel_stage, sizeof(int32_t) * batch * h->p.num_kv_heads * topk,
                             cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  return BASISKV_OK;
}

int basiskv_route(basiskv_handle* h, int batch, const void* q, int topk, float* scores_out, int32_t* sel_out,
                  basiskv_stream_t stream) {
  NvtxRange range("basiskv_route");
  int rc = check_call(h, batch, q, topk);
  if (rc) return rc;
  if (batch == 0) return BASISKV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  const LaunchPlan lp = plan(h, batch, topk, true);
  float* scores = scores_out ? scores_out : h->d_scores;
  // the prep grid writes -inf past n_b, the -1 rows of empty sequences and,
  // for large batches, the plan
  rc = launch_prep(h, lp, topk, 1, nullptr, sel_out, scores, 0, st);
  if (rc) return rc;
  if (!lp.any_routed) return BASISKV_OK;
  RouteArgs ra = route_args(h, lp, q, topk, scores, sel_out, 1);
  rc = launch_route(h, lp, ra, true, st);
  if (rc || !h->route_fn) return rc;
  return launch_topk(h, lp, topk, scores, sel_out, 1, true, false, st);
}

int basiskv_get_status(basiskv_handle* h, uint32_t* status, int clear) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (!status) return fail(BASISKV_ERR_INVALID_ARG, "status is NULL");
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(status, h->d_status, sizeof(uint32_t), cudaMemcpyDeviceToHost));
  if (clear && *status) {
    // a call that gave up part way can leave arrival counts behind: start
    // the next call from zero
    CUDA_TRY(cudaMemset(h->d_counters, 0,
                        sizeof(uint32_t) * (3 * (size_t)h->p.max_batch * h->p.num_kv_heads + kSchedWords)));
    CUDA_TRY(cudaMemset(h->d_status, 0, sizeof(uint32_t)));
  }
  return BASISKV_OK;
}

int basiskv_profile_begin(basiskv_handle* h, int max_calls) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (max_calls < 0) return fail(BASISKV_ERR_INVALID_ARG, "max_calls < 0");
  while ((int)h->events.size() < kProfEvents * max_calls) {
    cudaEvent_t e;
    CUDA_TRY(cudaEventCreate(&e));
    h->events.push_back(e);
  }
  h->prof_cap = max_calls;
  h->prof_calls = 0;
  return BASISKV_OK;
}

int basiskv_profile_end(basiskv_handle* h, float* ms, int* ncalls) {
  int rc = check_handle(h);
  if (rc) return rc;
  for (int i = 0; i < h->prof_calls; ++i) {
    cudaEvent_t* ev = &h->events[kProfEvents * i];
    CUDA_TRY(cudaEventSynchronize(ev[kProfEvents - 1]));
    for (int k = 0; k + 1 < kProfEvents && ms; ++k)
      CUDA_TRY(cudaEventElapsedTime(&ms[i * kProfEvents + k], ev[k], ev[k + 1]));
    if (ms) CUDA_TRY(cudaEventElapsedTime(&ms[i * kProfEvents + kProfEvents - 1], ev[0], ev[kProfEvents - 1]));
  }
  if (ncalls) *ncalls = h->prof_calls;
  h->prof_cap = 0;
  h->prof_calls = 0;
  return BASISKV_OK;
}

int basiskv_last_launch(basiskv_handle* h, int info[6]) {
  int rc = check_handle(h);
  if (rc) return rc;
  if (!info) return fail(BASISKV_ERR_INVALID_ARG, "info is NULL");
  for (int i = 0; i < 6; ++i) info[i] = h->last_launch[i];
  return BASISKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode.  Some callers may not allocate device memory at
// all: code running inside a framework that owns every allocation, or code
// inside a region where cudaMalloc is not allowed.  This entry point runs
// the decode step without a handle and without allocating: its scratch
// (page scores, selection, split partials, arrival counters, a status word)
// is one fixed-size __device__ array in this file, which every GPU that
// loads the library keeps until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mutex;

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The status word sits at the start of the array, where every call finds it
// whatever its shapes.
constexpr size_t kNoAllocStatusOffset = 0;

// Device address of the scratch array on the current device.  The symbol's
// host-side name is not a device address, so it is resolved here once per
// device with cudaGetSymbolAddress.
int noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(BASISKV_ERR_UNSUPPORTED, "device %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(BASISKV_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BASISKV_OK;
}

}  // namespace

extern "C" int basiskv_decode_attn_noalloc(const basiskv_params* p, int batch, const int32_t* page_table,
                                           const int32_t* seq_lens, const void* q, int topk,
                                           float softmax_scale, float* out, int32_t* sel_out,
                                           basiskv_stream_t stream) {
  int rc = validate_params(p);
  if (rc) return rc;
  if (batch < 0 || batch > p->max_batch) return fail(BASISKV_ERR_INVALID_ARG, "batch %d outside [0, %d]", batch, p->max_batch);
  if (topk <= 0 || topk > p->max_topk) return fail(BASISKV_ERR_INVALID_ARG, "topk %d outside [1, %d]", topk, p->max_topk);
  if (!q || !aligned16(q) || !out || !page_table || !seq_lens)
    return fail(BASISKV_ERR_INVALID_ARG, "q (16-byte aligned), out, page_table and seq_lens are required");
  if (!std::isfinite(softmax_scale)) return fail(BASISKV_ERR_INVALID_ARG, "softmax_scale must be finite");
  if (batch == 0) return BASISKV_OK;

  // scratch layout: status | counters | scores | selection | partial (m, l) | partial acc
  const size_t U = (size_t)batch * p->num_kv_heads, G = p->gqa_group;
  const int splits = std::min(kMaxSplits, std::max(1, topk));
  const size_t off_status = kNoAllocStatusOffset;
  const size_t off_counters = align256(off_status + sizeof(uint32_t));
  const size_t off_scores = align256(off_counters + sizeof(uint32_t) * 2 * U);
  const size_t off_sel = align256(off_scores + sizeof(float) * U * p->max_pages_per_seq);
  const size_t off_ml = align256(off_sel + sizeof(int32_t) * U * topk);
  const size_t off_acc = align256(off_ml + sizeof(float) * U * splits * G * 2);
  const size_t need = align256(off_acc + sizeof(float) * U * splits * G * p->rank_r);
  if (need > kNoAllocScratchBytes)
    return fail(BASISKV_ERR_CAPACITY,
                "this call needs %zu bytes of scratch; the allocation-free path has %zu (reduce batch, "
                "pages per sequence or top-k, or use basiskv_create)", need, kNoAllocScratchBytes);

  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  unsigned char* scratch = nullptr;
  rc = noalloc_scratch(dev, reinterpret_cast<void**>(&scratch));
  if (rc) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  // the status word and the arrival counters must start at zero
  CUDA_TRY(cudaMemsetAsync(scratch, 0, off_scores, st));

  // routing: a grid of (page chunk, KV head, sequence) sized by the table's
  // row length; chunks past a sequence's pages exit at once
  const int ppc = std::max(kRouteWarps * 2, std::min(64, p->max_pages_per_seq));
  RouteArgs ra{};
  ra.q = q;
  ra.z_pool = p->z_pool;
  ra.r_pool = p->r_pool;
  ra.w_zk = p->w_zk;
  ra.b_r = p->b_r;
  ra.page_table = page_table;
  ra.seq_lens = seq_lens;
  ra.scores = reinterpret_cast<float*>(scratch + off_scores);
  ra.sel = reinterpret_cast<int32_t*>(scratch + off_sel);
  ra.sel_out = sel_out;
  ra.counters = reinterpret_cast<uint32_t*>(scratch + off_counters);
  ra.status = reinterpret_cast<uint32_t*>(scratch + off_status);
  ra.ld_pt = p->max_pages_per_seq;
  ra.ld_sel = topk;
  ra.num_slots = p->num_slots;
  ra.num_kv_heads = p->num_kv_heads;
  ra.head_dim = p->head_dim;
  ra.page_size = p->page_size;
  ra.rank_r = p->rank_r;
  ra.rank_s = p->rank_s;
  ra.gqa_group = p->gqa_group;
  ra.topk = topk;
  ra.pages_per_cta = ppc;
  ra.batch = batch;
  ra.plan_n = -1;
  const dim3 rgrid((p->max_pages_per_seq + ppc - 1) / ppc, p->num_kv_heads, batch);
  const size_t rsmem = generic_route_smem(*p);
  if (p->dtype == BASISKV_DTYPE_BF16) {
    rc = set_smem_attr((const void*)&route_generic_kernel<__nv_bfloat16>, rsmem);
    if (rc) return rc;
    route_generic_kernel<__nv_bfloat16><<<rgrid, kRouteThreads, rsmem, st>>>(ra);
  } else {
    rc = set_smem_attr((const void*)&route_generic_kernel<float>, rsmem);
    if (rc) return rc;
    route_generic_kernel<float><<<rgrid, kRouteThreads, rsmem, st>>>(ra);
  }
  CUDA_TRY(cudaGetLastError());

  // attention: (split, KV head, sequence), one partial per CTA
  AttnArgs aa{};
  aa.q = q;
  aa.k_pool = p->k_pool;
  aa.k_scale = p->k_scale;
  aa.k_int8 = p->k_format == BASISKV_KEYS_INT8;
  aa.z_pool = p->z_pool;
  aa.b_v = p->b_v;
  aa.page_table = page_table;
  aa.seq_lens = seq_lens;
  aa.sel = ra.sel;
  aa.sel_out = sel_out;
  aa.part_ml = reinterpret_cast<float*>(scratch + off_ml);
  aa.part_acc = reinterpret_cast<float*>(scratch + off_acc);
  aa.counters = ra.counters + U;
  aa.status = ra.status;
  aa.out = out;
  aa.ld_pt = p->max_pages_per_seq;
  aa.ld_sel = topk;
  aa.num_slots = p->num_slots;
  aa.num_kv_heads = p->num_kv_heads;
  aa.head_dim = p->head_dim;
  aa.page_size = p->page_size;
  aa.rank_r = p->rank_r;
  aa.gqa_group = p->gqa_group;
  aa.topk = topk;
  aa.pages_per_split = (topk + splits - 1) / splits;
  aa.np_cap = splits;
  aa.scale_log2 = softmax_scale * 1.4426950408889634f;
  aa.batch = batch;
  aa.plan_n = -1;
  const dim3 agrid((topk + aa.pages_per_split - 1) / aa.pages_per_split, p->num_kv_heads, batch);
  const size_t g = p->gqa_group;
  const size_t asmem = sizeof(float) * std::max(g * (p->head_dim + p->page_size + p->rank_r) + 3 * g,
                                                combine_smem_floats(splits, p->gqa_group, p->rank_r));
  if (p->dtype == BASISKV_DTYPE_BF16) {
    rc = set_smem_attr((const void*)&attn_generic_kernel<__nv_bfloat16>, asmem);
    if (rc) return rc;
    attn_generic_kernel<__nv_bfloat16><<<agrid, kAttnThreads, asmem, st>>>(aa);
  } else {
    rc = set_smem_attr((const void*)&attn_generic_kernel<float>, asmem);
    if (rc) return rc;
    attn_generic_kernel<float><<<agrid, kAttnThreads, asmem, st>>>(aa);
  }
  CUDA_TRY(cudaGetLastError());
  return BASISKV_OK;
}

extern "C" int basiskv_noalloc_status(uint32_t* status) {
  if (!status) return fail(BASISKV_ERR_INVALID_ARG, "status is NULL");
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  unsigned char* scratch = nullptr;
  int rc = noalloc_scratch(dev, reinterpret_cast<void**>(&scratch));
  if (rc) return rc;
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(status, scratch + kNoAllocStatusOffset, sizeof(uint32_t), cudaMemcpyDeviceToHost));
  return BASISKV_OK;
}
