// Encode incoming keys and values into the compressed pools ("BasisKV: Value
// Latents for Communication and Key Routing", English abstract: the Value
// cache is held as rank-r latents, and a Key-specific residual stores what
// the Value latent cannot predict).  Least squares, per KV head:
//     Z = V . A_v                      A_v = pinv(B_v)  [d][r]
//     R = (K - Z_stored . W_zk) . A_r  A_r = pinv(B_r)  [d][s]
// The residual is taken against the stored (rounded) latent, so that
// Z.W_zk + R.B_r predicts K from exactly what routing will read.  K rows
// are stored as given.
#pragma once

#include "common.cuh"

namespace basiskv {

struct EncodeArgs {
  const void* k;      // [Hkv][n][d] pool dtype
  const void* v;      // [Hkv][n][d] pool dtype
  void* k_pool;       // [slots][Hkv][P][d]
  void* z_pool;       // [slots][Hkv][P][r]
  void* r_pool;       // [slots][Hkv][P][s]
  const float* a_v;   // [Hkv][d][r]
  const float* a_r;   // [Hkv][d][s]
  const float* w_zk;  // [Hkv][r][d]
  int num_kv_heads, page_size, head_dim, rank_r, rank_s;
  int slot, row0, n;  // rows [row0, row0 + n) of pool slot `slot`
};

constexpr int kEncodeThreads = 128;

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

// One CTA per (row, KV head); fp32 arithmetic, outputs rounded to the pool
// dtype.  Dynamic shared memory: (3d + r) floats.
template <typename T>
__global__ void __launch_bounds__(kEncodeThreads) encode_rows_kernel(const EncodeArgs a) {
  extern __shared__ float esm[];
  const int i = blockIdx.x, kvh = blockIdx.y, tid = threadIdx.x;
  const int d = a.head_dim, r = a.rank_r, s = a.rank_s;
  float* kr = esm;      // [d] incoming key
  float* vr = kr + d;   // [d] incoming value
  float* z = vr + d;    // [r] stored latent, widened back
  float* res = z + r;   // [d] key minus its prediction from the stored latent
  const size_t in = ((size_t)kvh * a.n + i) * d;
  const size_t row = ((size_t)a.slot * a.num_kv_heads + kvh) * a.page_size + a.row0 + i;
  const T* k = static_cast<const T*>(a.k) + in;
  const T* v = static_cast<const T*>(a.v) + in;
  T* kp = static_cast<T*>(a.k_pool) + row * d;
  for (int c = tid; c < d; c += kEncodeThreads) {
    kr[c] = to_f32(k[c]);
    vr[c] = to_f32(v[c]);
    kp[c] = k[c];
  }
  __syncthreads();
  const float* Av = a.a_v + (size_t)kvh * d * r;
  T* zp = static_cast<T*>(a.z_pool) + row * r;
  for (int j = tid; j < r; j += kEncodeThreads) {
    float acc = 0.f;
    for (int c = 0; c < d; ++c) acc = fmaf(vr[c], Av[(size_t)c * r + j], acc);
    const T zt = from_f32<T>(acc);
    zp[j] = zt;
    z[j] = to_f32(zt);
  }
  if (s == 0) return;
  __syncthreads();
  const float* W = a.w_zk + (size_t)kvh * r * d;
  for (int c = tid; c < d; c += kEncodeThreads) {
    float acc = kr[c];
    for (int t = 0; t < r; ++t) acc = fmaf(-z[t], W[(size_t)t * d + c], acc);
    res[c] = acc;
  }
  __syncthreads();
  const float* Ar = a.a_r + (size_t)kvh * d * s;
  T* rp = static_cast<T*>(a.r_pool) + row * s;
  for (int j = tid; j < s; j += kEncodeThreads) {
    float acc = 0.f;
    for (int c = 0; c < d; ++c) acc = fmaf(res[c], Ar[(size_t)c * s + j], acc);
    rp[j] = from_f32<T>(acc);
  }
}

}  // namespace basiskv
