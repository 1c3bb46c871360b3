// Encode incoming keys and values into the compressed pools ("BasisKV: Value
// Latents for Communication and Key Routing", English abstract: the Value
// cache is held as rank-r latents, and a Key-specific residual stores what
// the Value latent cannot predict).  Least squares, per KV head:
//     Z = V . A_v                      A_v = pinv(B_v)  [d][r]
//     R = (K - Z_stored . W_zk) . A_r  A_r = pinv(B_r)  [d][s]
// The residual is taken against the stored (rounded) latent, so that
// Z.W_zk + R.B_r predicts K from exactly what routing will read.  K rows
// are stored as given, or as int8 codes with a per-token scale (the lossy
// key compression of "PackKV: Reducing KV Cache Memory Footprint through
// LLM-Aware Lossy Compression", abstract, read as symmetric int8):
//     scale = max_c |k_c| / 127,   code_c = rint(k_c / scale)
// in float32 with IEEE division, ties to even; a zero row gets scale 0.
#pragma once

#include "common.cuh"

namespace basiskv {

struct EncodeArgs {
  // incoming keys and values, pool dtype: element (token i, KV head h, channel c)
  // at i * tok_stride + h * head_stride + c
  const void* k;
  const void* v;
  long long tok_stride, head_stride;
  void* k_pool;       // [slots][Hkv][P][d]: pool dtype, or int8 codes when k_int8
  float* k_scale;     // [slots][Hkv][P] (k_int8 only)
  int k_int8;
  void* z_pool;       // [slots][Hkv][P][r]
  void* r_pool;       // [slots][Hkv][P][s]
  const float* a_v;   // [Hkv][d][r]
  const float* a_r;   // [Hkv][d][s]
  const float* w_zk;  // [Hkv][r][d]
  int num_kv_heads, page_size, head_dim, rank_r, rank_s, num_slots;
  // destinations: token i goes to row (row0 + i) of pool slot `slot`, or,
  // when `slots` is not null, to row rows[i] of slot slots[i]
  int slot, row0, n;
  const int32_t* slots;
  const int32_t* rows;
  int tokens_per_cta;
  int stage;          // copy the KV head's A_v, W_zk, A_r to shared memory first
  uint32_t* status;
};

constexpr int kEncodeThreads = 128;

// One key row of d values to int8 codes and its scale, by one warp.
template <typename T>
__device__ __forceinline__ void warp_quantize_row(const T* k, int d, int8_t* codes, float* scale, int lane) {
  float amax = 0.f;
  for (int c = lane; c < d; c += 32) amax = fmaxf(amax, fabsf(to_f32(k[c])));
  amax = warp_max(amax);
  const float sc = __fdiv_rn(amax, 127.f);
  for (int c = lane; c < d; c += 32) {
    int q = 0;
    if (sc > 0.f) q = __float2int_rn(__fdiv_rn(to_f32(k[c]), sc));
    codes[c] = (int8_t)max(-127, min(127, q));
  }
  if (lane == 0) *scale = sc;
}

// Rows [row0, row0 + n) of a key pool in its flat row order
// ((slot * Hkv + kvh) * P + token), from keys k [n][d] in the pool dtype.
struct QuantizeArgs {
  const void* k;
  int8_t* codes;   // the int8 key pool
  float* scales;   // [rows]
  long long row0, n;
  int head_dim;
};

// Rows per warp of quantize_rows_kernel: their loads are issued together so
// that each warp keeps several rows in flight.
constexpr int kQuantRowsPerWarp = 4;

// code of x for scale sc (as warp_quantize_row)
__device__ __forceinline__ uint32_t quant_code(float x, float sc) {
  const int q = sc > 0.f ? __float2int_rn(__fdiv_rn(x, sc)) : 0;
  return (uint32_t)(uint8_t)(int8_t)max(-127, min(127, q));
}

template <typename T>
__global__ void __launch_bounds__(kEncodeThreads) quantize_rows_kernel(const QuantizeArgs a) {
  const int lane = threadIdx.x & 31;
  const long long i0 = ((long long)blockIdx.x * (kEncodeThreads / 32) + (threadIdx.x >> 5)) * kQuantRowsPerWarp;
  if (i0 >= a.n) return;
  if constexpr (sizeof(T) == 2) {
    if (a.head_dim == 128) {
      // bf16 rows of 128: four values per lane, one 8-byte load per row
      uint2 v[kQuantRowsPerWarp];
#pragma unroll
      for (int r = 0; r < kQuantRowsPerWarp; ++r)
        v[r] = i0 + r < a.n ? __ldg(reinterpret_cast<const uint2*>(static_cast<const T*>(a.k) + (i0 + r) * 128) + lane)
                            : make_uint2(0u, 0u);
#pragma unroll
      for (int r = 0; r < kQuantRowsPerWarp; ++r) {
        if (i0 + r >= a.n) break;
        const float x0 = __uint_as_float(v[r].x << 16), x1 = __uint_as_float(v[r].x & 0xffff0000u);
        const float x2 = __uint_as_float(v[r].y << 16), x3 = __uint_as_float(v[r].y & 0xffff0000u);
        const float amax = warp_max(fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3))));
        const float sc = __fdiv_rn(amax, 127.f);
        const long long row = a.row0 + i0 + r;
        reinterpret_cast<uint32_t*>(a.codes + row * 128)[lane] =
            quant_code(x0, sc) | quant_code(x1, sc) << 8 | quant_code(x2, sc) << 16 | quant_code(x3, sc) << 24;
        if (lane == 0) a.scales[row] = sc;
      }
      return;
    }
  }
  for (int r = 0; r < kQuantRowsPerWarp && i0 + r < a.n; ++r) {
    const long long i = i0 + r, row = a.row0 + i;
    warp_quantize_row(static_cast<const T*>(a.k) + i * a.head_dim, a.head_dim, a.codes + row * a.head_dim,
                      a.scales + row, lane);
  }
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Grid (ceil(n / tokens_per_cta), Hkv): a CTA encodes tokens_per_cta
// consecutive tokens of one KV head, in fp32, outputs rounded to the pool
// dtype.  With `stage`, the head's A_v [d][r], W_zk [r][d] and A_r [d][s]
// are first copied to shared memory (coalesced) and every product reads
// them there; otherwise they are read from global memory.  Dynamic shared
// memory: (3d + r) floats, plus (2dr + ds) floats with `stage`.
// Destinations outside the pool set BAD_SLOT and are skipped.
template <typename T>
__global__ void __launch_bounds__(kEncodeThreads) encode_kernel(const EncodeArgs a) {
  extern __shared__ float esm[];
  const int kvh = blockIdx.y, tid = threadIdx.x;
  const int d = a.head_dim, r = a.rank_r, s = a.rank_s;
  float* kr = esm;      // [d] incoming key
  float* vr = kr + d;   // [d] incoming value
  float* z = vr + d;    // [r] stored latent, widened back
  float* res = z + r;   // [d] key minus its prediction from the stored latent
  const float* Av = a.a_v + (size_t)kvh * d * r;
  const float* W = a.w_zk + (size_t)kvh * r * d;
  const float* Ar = a.a_r + (size_t)kvh * d * s;
  if (a.stage) {
    float* sav = res + d;
    float* sw = sav + d * r;
    float* sar = sw + r * d;
    const bool vec = ((d * r) % 4 == 0) && ((d * s) % 4 == 0) &&
                     ((reinterpret_cast<uintptr_t>(Av) | reinterpret_cast<uintptr_t>(W) |
                       reinterpret_cast<uintptr_t>(Ar) | reinterpret_cast<uintptr_t>(sav)) & 15u) == 0;
    if (vec) {  // 16-byte loads: a quarter of the load instructions
      for (int e = tid; e < d * r / 4; e += kEncodeThreads) {
        reinterpret_cast<float4*>(sav)[e] = __ldg(reinterpret_cast<const float4*>(Av) + e);
        reinterpret_cast<float4*>(sw)[e] = __ldg(reinterpret_cast<const float4*>(W) + e);
      }
      for (int e = tid; e < d * s / 4; e += kEncodeThreads)
        reinterpret_cast<float4*>(sar)[e] = __ldg(reinterpret_cast<const float4*>(Ar) + e);
    } else {
      for (int e = tid; e < d * r; e += kEncodeThreads) {
        sav[e] = Av[e];
        sw[e] = W[e];
      }
      for (int e = tid; e < d * s; e += kEncodeThreads) sar[e] = Ar[e];
    }
    Av = sav;
    W = sw;
    Ar = sar;
  }
  const int i_end = min(a.n, (int)(blockIdx.x + 1) * a.tokens_per_cta);
  for (int i = blockIdx.x * a.tokens_per_cta; i < i_end; ++i) {
    int slot = a.slot, prow = a.row0 + i;
    if (a.slots) {
      slot = a.slots[i];
      prow = a.rows[i];
    }
    if (slot < 0 || slot >= a.num_slots || prow < 0 || prow >= a.page_size) {
      if (tid == 0) atomicOr(a.status, kStatusBadSlot);
      continue;  // uniform over the CTA: the same token for every thread
    }
    const size_t in = (size_t)i * a.tok_stride + (size_t)kvh * a.head_stride;
    const size_t row = ((size_t)slot * a.num_kv_heads + kvh) * a.page_size + prow;
    const T* k = static_cast<const T*>(a.k) + in;
    const T* v = static_cast<const T*>(a.v) + in;
    __syncthreads();  // the previous token's buffers (and the staged bases) are settled
    for (int c = tid; c < d; c += kEncodeThreads) {
      kr[c] = to_f32(k[c]);
      vr[c] = to_f32(v[c]);
      if (!a.k_int8) static_cast<T*>(a.k_pool)[row * d + c] = k[c];
    }
    if (a.k_int8 && tid < 32)
      warp_quantize_row(k, d, static_cast<int8_t*>(a.k_pool) + row * d, a.k_scale + row, tid);
    __syncthreads();
    T* zp = static_cast<T*>(a.z_pool) + row * r;
    for (int j = tid; j < r; j += kEncodeThreads) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(vr[c], Av[(size_t)c * r + j], acc);
      const T zt = from_f32<T>(acc);
      zp[j] = zt;
      z[j] = to_f32(zt);
    }
    if (s == 0) continue;
    __syncthreads();
    for (int c = tid; c < d; c += kEncodeThreads) {
      float acc = kr[c];
      for (int t = 0; t < r; ++t) acc = fmaf(-z[t], W[(size_t)t * d + c], acc);
      res[c] = acc;
    }
    __syncthreads();
    T* rp = static_cast<T*>(a.r_pool) + row * s;
    for (int j = tid; j < s; j += kEncodeThreads) {
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(res[c], Ar[(size_t)c * s + j], acc);
      rp[j] = from_f32<T>(acc);
    }
  }
}

}  // namespace basiskv
