// Cache-write step: the new token's row of the latent cache, before decode
// attention reads it ("Multi-Head Low-Rank Attention": Methodology, third
// paragraph — the latent states are RMS-normalised before the up-projection;
// Main Findings, variance bullet — the KV latent is scaled by alpha_kv; Key
// Contributions #2 — one decoupled RoPE key per token).
//
// Per sequence s, with p = positions[s]:
//   row[b * d_cb + i] = alpha_kv * gamma[b * d_cb + i] * c[b * d_cb + i]
//                       / sqrt(mean_i c[b * d_cb + i]^2 + eps)      (each block b)
//   row[nb * d_cb + i], row[nb * d_cb + i + d_r/2] = the pair (i, i + d_r/2) of
//                       k_rope rotated by p * theta^(-2 i / d_r)
// written (in the cache dtype) at token p of sequence s: page_table[s][p / 64]
// row p % 64 (paged) or row s * max_len + p (contiguous).
// One CTA per sequence: warps 0-3 normalise the latent blocks (one block per
// warp at a time), warp 4 rotates the RoPE key.  The rotation angle and its
// sine and cosine are taken in fp64: at positions near 2^17 an fp32 angle is
// off by ~1e-2 rad.
#include "dispatch.h"

#include <math.h>

namespace mlra {
namespace {

constexpr int kCacheThreads = 160;

template <typename T> __device__ __forceinline__ float load_f(const T* p);
template <> __device__ __forceinline__ float load_f<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float load_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(kCacheThreads)
    cache_append_kernel(const T* __restrict__ c_new, const T* __restrict__ k_rope_new,
                        const float* __restrict__ gamma, float alpha_kv, float eps, double theta,
                        T* __restrict__ cache, int64_t num_pages, const int32_t* __restrict__ page_table,
                        int max_pages, int cap, const int32_t* __restrict__ positions, int nb,
                        int d_cb, int d_r, int32_t* status) {
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos = __ldg(positions + s);
  if (pos < 0 || pos >= cap) {
    if (threadIdx.x == 0 && status) set_error(status, MLRA_ERR_INVALID_ARG);
    return;
  }
  int64_t row;
  if (page_table) {
    const int pg = __ldg(page_table + size_t(s) * max_pages + pos / kPageSize);
    if (pg < 0 || pg >= num_pages) {
      if (threadIdx.x == 0 && status) set_error(status, MLRA_ERR_BAD_PAGE);
      return;
    }
    row = int64_t(pg) * kPageSize + pos % kPageSize;
  } else {
    row = int64_t(s) * max_pages + pos;
  }
  const int K = nb * d_cb, D = K + d_r;
  T* dst = cache + row * D;
  if (warp < 4) {
    for (int b = warp; b < nb; b += 4) {
      const T* src = c_new + size_t(s) * K + size_t(b) * d_cb;
      float ss = 0.f;
      for (int i = lane; i < d_cb; i += 32) {
        const float v = load_f(src + i);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float scale = alpha_kv / sqrtf(ss / float(d_cb) + eps);
      for (int i = lane; i < d_cb; i += 32)
        dst[b * d_cb + i] = from_f<T>(load_f(src + i) * scale * __ldg(gamma + b * d_cb + i));
    }
  } else {
    const int half = d_r / 2;
    const T* src = k_rope_new + size_t(s) * d_r;
    for (int i = lane; i < half; i += 32) {
      const double ang = double(pos) * pow(theta, -2.0 * i / d_r);
      double sn, cs;
      sincos(ang, &sn, &cs);
      const float a = load_f(src + i), bv = load_f(src + i + half);
      const float c32 = float(cs), s32 = float(sn);
      dst[K + i] = from_f<T>(a * c32 - bv * s32);
      dst[K + i + half] = from_f<T>(a * s32 + bv * c32);
    }
  }
}

// Query side of the same step (Main Findings, variance bullet: the query is
// scaled by alpha_q; Key Contributions #2: the decoupled RoPE query meets the
// shared RoPE key): for every sequence s and head h,
//   out[s, h, i], out[s, h, i + d_r/2] = the pair (i, i + d_r/2) of
//   alpha * q_rope[s, h, :] rotated by positions[s] * theta^(-2 i / d_r),
// the same rotation as the cache write's, so that the RoPE logit depends on the
// distance between the query's and the key's positions only.  One CTA per
// sequence: the d_r / 2 angles are taken once in fp64 (shared memory), then
// every (head, pair) of the sequence is rotated in fp32 and rounded once to the
// storage dtype.
constexpr int kQRopeThreads = 256;
constexpr int kMaxHalf = 256;

template <typename T>
__global__ void __launch_bounds__(kQRopeThreads)
    query_rope_kernel(const T* __restrict__ q_rope, const int32_t* __restrict__ positions,
                      float alpha, double theta, T* __restrict__ out, int heads, int d_r) {
  __shared__ float cs_sm[kMaxHalf], sn_sm[kMaxHalf];
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x;
  const int half = d_r / 2;
  const int pos = __ldg(positions + s);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double ang = double(pos) * pow(theta, -2.0 * i / d_r);
    double sn, cs;
    sincos(ang, &sn, &cs);
    cs_sm[i] = float(cs);
    sn_sm[i] = float(sn);
  }
  __syncthreads();
  const size_t base = size_t(s) * heads * d_r;
  for (int x = threadIdx.x; x < heads * half; x += blockDim.x) {
    const int h = x / half, i = x - h * half;
    const T* src = q_rope + base + size_t(h) * d_r;
    const float a = load_f(src + i) * alpha, b = load_f(src + i + half) * alpha;
    T* dst = out + base + size_t(h) * d_r;
    dst[i] = from_f<T>(a * cs_sm[i] - b * sn_sm[i]);
    dst[i + half] = from_f<T>(a * sn_sm[i] + b * cs_sm[i]);
  }
}

}  // namespace

cudaError_t launch_query_rope(const mlra_config_t& c, const void* q_rope, const int32_t* positions,
                              float alpha, double theta, void* q_rope_out, int batch,
                              cudaStream_t st) {
  if (c.d_r % 2 != 0 || c.d_r / 2 > kMaxHalf) return cudaErrorInvalidValue;
  if (c.dtype == MLRA_BF16)
    return launch_pdl(query_rope_kernel<__nv_bfloat16>, dim3(batch), dim3(kQRopeThreads), 0, st,
                      (const __nv_bfloat16*)q_rope, positions, alpha, theta,
                      (__nv_bfloat16*)q_rope_out, c.n_heads, c.d_r);
  return launch_pdl(query_rope_kernel<float>, dim3(batch), dim3(kQRopeThreads), 0, st,
                    (const float*)q_rope, positions, alpha, theta, (float*)q_rope_out, c.n_heads,
                    c.d_r);
}

cudaError_t launch_cache_append(const mlra_config_t& c, const void* c_new, const void* k_rope_new,
                                const float* gamma, float alpha_kv, float eps, double theta,
                                void* kv_cache, int64_t num_pages, const int32_t* page_table,
                                int max_pages, int cap, const int32_t* positions, int batch,
                                int32_t* status, cudaStream_t st) {
  if (c.dtype == MLRA_BF16)
    return launch_pdl(cache_append_kernel<__nv_bfloat16>, dim3(batch), dim3(kCacheThreads), 0, st,
                      (const __nv_bfloat16*)c_new, (const __nv_bfloat16*)k_rope_new, gamma,
                      alpha_kv, eps, theta, (__nv_bfloat16*)kv_cache, num_pages, page_table,
                      max_pages, cap, positions, c.n_blocks, c.d_cb, c.d_r, status);
  return launch_pdl(cache_append_kernel<float>, dim3(batch), dim3(kCacheThreads), 0, st,
                    (const float*)c_new, (const float*)k_rope_new, gamma, alpha_kv, eps, theta,
                    (float*)kv_cache, num_pages, page_table, max_pages, cap, positions,
                    c.n_blocks, c.d_cb, c.d_r, status);
}

}  // namespace mlra
