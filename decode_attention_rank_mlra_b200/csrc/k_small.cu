// Small kernels of the decode step: split plan, query absorption, split-KV
// combine and output up-projection.  All fp32 SIMT: together they move well
// under 5% of the bytes of the attention kernel (see the layer description in
// include/mlra.h for the maths).
#include "mlra_internal.cuh"

#include <math.h>

namespace mlra {

template <typename T> __device__ __forceinline__ float ld_f32(const T* p);
template <> __device__ __forceinline__ float ld_f32<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// ---------------------------------------------------------------------------
// Plan: tile stream offsets and split slots from the per-sequence lengths.
// One block of 1024 threads; each thread scans a contiguous run of sequences.
// ---------------------------------------------------------------------------
__device__ int block_inclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  int r = v + (warp > 0 ? warp_tot[warp - 1] : 0);
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ seqlens, int batch,
                                                    int cap, int ctas_per_group, int max_slots,
                                                    WsHeader* hdr, int32_t* tile_off,
                                                    int32_t* slot_off) {
  __shared__ int warp_tot[32];
  __shared__ int s_total, s_share, s_bad;
  if (threadIdx.x == 0) { hdr->error = 0; s_bad = 0; }
  __syncthreads();
  const int per = (batch + blockDim.x - 1) / blockDim.x;
  const int b0 = min(batch, (int)threadIdx.x * per), b1 = min(batch, b0 + per);
  auto tiles_of = [&](int s) {
    int L = __ldg(seqlens + s);
    if (L < 0 || L > cap) { s_bad = 1; L = L < 0 ? 0 : cap; }
    return (L + kTile - 1) / kTile;
  };
  int local = 0;
  for (int s = b0; s < b1; ++s) local += tiles_of(s);
  int incl = block_inclusive_scan(local, warp_tot);
  int run = incl - local;
  for (int s = b0; s < b1; ++s) { tile_off[s] = run; run += tiles_of(s); }
  if (threadIdx.x == blockDim.x - 1) {
    tile_off[batch] = incl;
    s_total = incl;
    s_share = max(1, (incl + ctas_per_group - 1) / ctas_per_group);
  }
  __syncthreads();
  const int share = s_share;
  local = 0;
  for (int s = b0; s < b1; ++s) {
    int a = tile_off[s], e = tile_off[s + 1];
    local += (e > a) ? ((e - 1) / share - a / share + 1) : 0;
  }
  incl = block_inclusive_scan(local, warp_tot);
  run = incl - local;
  for (int s = b0; s < b1; ++s) {
    slot_off[s] = run;
    int a = tile_off[s], e = tile_off[s + 1];
    run += (e > a) ? ((e - 1) / share - a / share + 1) : 0;
  }
  if (threadIdx.x == blockDim.x - 1) {
    slot_off[batch] = incl;
    hdr->total_tiles = s_total;
    hdr->share = share;
    hdr->n_slots = incl;
    hdr->ctas_per_group = ctas_per_group;
    hdr->batch = batch;
    hdr->max_slots = max_slots;
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) set_error(&hdr->error, MLRA_ERR_INVALID_ARG);
}

cudaError_t launch_plan(const int32_t* seqlens, int batch, int cap, int ctas_per_group, void* ws,
                        const WsLayout& L, cudaStream_t st) {
  char* base = static_cast<char*>(ws);
  plan_kernel<<<1, 1024, 0, st>>>(seqlens, batch, cap, ctas_per_group, L.max_slots,
                                  reinterpret_cast<WsHeader*>(base),
                                  reinterpret_cast<int32_t*>(base + L.tile_off),
                                  reinterpret_cast<int32_t*>(base + L.slot_off));
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Absorption: q_abs[s,h,b,i] = sum_j W_uk[b,h,i,j] q_nope[s,h,j]
// Block (head h, 8 sequences); warp w takes latent rows (b,i) = w, w+8, ...;
// lanes split j and reduce with shuffles.  W_uk is streamed once per block.
// ---------------------------------------------------------------------------
constexpr int kSeqBlk = 8;

template <typename T>
__global__ void __launch_bounds__(256) absorb_kernel(const T* __restrict__ q_nope,
                                                     const T* __restrict__ w_uk,
                                                     float* __restrict__ q_abs, int batch,
                                                     int heads, int nb, int d_cb, int d_h) {
  extern __shared__ float sq[];  // [kSeqBlk][d_h]
  const int h = blockIdx.x, s0 = blockIdx.y * kSeqBlk;
  const int ns = min(kSeqBlk, batch - s0);
  for (int x = threadIdx.x; x < kSeqBlk * d_h; x += blockDim.x) {
    int s = x / d_h, j = x % d_h;
    sq[x] = (s < ns) ? ld_f32(q_nope + (size_t(s0 + s) * heads + h) * d_h + j) : 0.f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows = nb * d_cb;
  for (int r = warp; r < rows; r += 8) {
    const int b = r / d_cb, i = r % d_cb;
    const T* wrow = w_uk + ((size_t(b) * heads + h) * d_cb + i) * d_h;
    float acc[kSeqBlk];
#pragma unroll
    for (int s = 0; s < kSeqBlk; ++s) acc[s] = 0.f;
    for (int j = lane; j < d_h; j += 32) {
      float w = ld_f32(wrow + j);
#pragma unroll
      for (int s = 0; s < kSeqBlk; ++s) acc[s] = fmaf(w, sq[s * d_h + j], acc[s]);
    }
#pragma unroll
    for (int s = 0; s < kSeqBlk; ++s) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[s] += __shfl_xor_sync(0xffffffffu, acc[s], o);
    }
    if (lane < ns) {
      float v = acc[0];
#pragma unroll
      for (int s = 1; s < kSeqBlk; ++s) if (lane == s) v = acc[s];
      q_abs[((size_t(s0 + lane) * heads + h) * nb + b) * d_cb + i] = v;
    }
  }
}

cudaError_t launch_absorb(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                          float* q_abs, int batch, cudaStream_t st) {
  dim3 grid(c.n_heads, (batch + kSeqBlk - 1) / kSeqBlk);
  size_t sm = sizeof(float) * kSeqBlk * c.d_h;
  if (c.dtype == MLRA_BF16)
    absorb_kernel<__nv_bfloat16><<<grid, 256, sm, st>>>(
        (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)w_uk, q_abs, batch, c.n_heads,
        c.n_blocks, c.d_cb, c.d_h);
  else
    absorb_kernel<float><<<grid, 256, sm, st>>>((const float*)q_nope, (const float*)w_uk, q_abs,
                                                batch, c.n_heads, c.n_blocks, c.d_cb, c.d_h);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Split-KV combine: one warp per (sequence, head, branch).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const char* __restrict__ ws, WsLayout L,
                                                      int batch, int heads, int nb, int d_cb,
                                                      float* __restrict__ o_latent,
                                                      float* __restrict__ lse_out) {
  const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int total = batch * heads * nb;
  if (warp_g >= total) return;
  const int b = warp_g % nb, h = (warp_g / nb) % heads, s = warp_g / (nb * heads);
  const int32_t* slot_off = reinterpret_cast<const int32_t*>(ws + L.slot_off);
  const float* o_part = reinterpret_cast<const float*>(ws + L.o_part);
  const float* lse_part = reinterpret_cast<const float*>(ws + L.lse_part);
  const int k0 = __ldg(slot_off + s), k1 = __ldg(slot_off + s + 1);
  const size_t row = (size_t(h) * nb + b);
  const size_t slot_stride = size_t(heads) * nb;
  float* dst = o_latent + ((size_t(s) * heads + h) * nb + b) * d_cb;
  if (k1 <= k0) {
    for (int i = lane; i < d_cb; i += 32) dst[i] = 0.f;
    if (lse_out && lane == 0) lse_out[(size_t(s) * heads + h) * nb + b] = -INFINITY;
    return;
  }
  float m = -INFINITY;
  for (int k = k0; k < k1; ++k) m = fmaxf(m, __ldg(lse_part + size_t(k) * slot_stride + row));
  if (m == -INFINITY) {  // every token of the sequence was rejected (bad page)
    for (int i = lane; i < d_cb; i += 32) dst[i] = 0.f;
    if (lse_out && lane == 0) lse_out[(size_t(s) * heads + h) * nb + b] = -INFINITY;
    return;
  }
  float den = 0.f;
  for (int k = k0; k < k1; ++k) den += expf(__ldg(lse_part + size_t(k) * slot_stride + row) - m);
  const float inv = 1.f / den;
  for (int i = lane; i < d_cb; i += 32) {
    float acc = 0.f;
    for (int k = k0; k < k1; ++k) {
      float w = expf(__ldg(lse_part + size_t(k) * slot_stride + row) - m);
      acc = fmaf(w, __ldg(o_part + (size_t(k) * slot_stride + row) * d_cb + i), acc);
    }
    dst[i] = acc * inv;
  }
  if (lse_out && lane == 0) lse_out[(size_t(s) * heads + h) * nb + b] = m + logf(den);
}

cudaError_t launch_combine(const mlra_config_t& c, const void* ws, const WsLayout& L, int batch,
                           float* o_latent, float* lse, cudaStream_t st) {
  const int rows = batch * c.n_heads * c.n_blocks;
  const int blocks = (rows * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  combine_kernel<<<blocks, 256, 0, st>>>(static_cast<const char*>(ws), L, batch, c.n_heads,
                                         c.n_blocks, c.d_cb, o_latent, lse);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Output up-projection: out[s,h,j] = branch_scale * sum_{b,i} o[s,h,b,i] W_uv[b,h,i,j]
// Block (head h, 8 sequences); W_uv rows are staged through shared memory in
// chunks of 32 latent rows; warp w owns sequence s0+w, lanes own columns j.
// ---------------------------------------------------------------------------
constexpr int kKChunk = 32;

template <typename T>
__global__ void __launch_bounds__(256) out_proj_kernel(const float* __restrict__ o_lat,
                                                       const T* __restrict__ w_uv,
                                                       float* __restrict__ out, int batch,
                                                       int heads, int nb, int d_cb, int d_h,
                                                       float branch_scale) {
  extern __shared__ float sm[];
  float* sw = sm;                       // [kKChunk][d_h]
  float* so = sm + kKChunk * d_h;       // [kSeqBlk][kKChunk]
  const int h = blockIdx.x, s0 = blockIdx.y * kSeqBlk;
  const int ns = min(kSeqBlk, batch - s0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = nb * d_cb;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};  // columns lane + 32 q, q < d_h / 32 (d_h <= 128)
  for (int k0 = 0; k0 < K; k0 += kKChunk) {
    __syncthreads();
    for (int x = threadIdx.x; x < kKChunk * d_h; x += blockDim.x) {
      int kk = x / d_h, j = x % d_h, k = k0 + kk;
      int b = k / d_cb, i = k % d_cb;
      sw[x] = ld_f32(w_uv + ((size_t(b) * heads + h) * d_cb + i) * d_h + j);
    }
    for (int x = threadIdx.x; x < kSeqBlk * kKChunk; x += blockDim.x) {
      int s = x / kKChunk, kk = x % kKChunk, k = k0 + kk;
      so[x] = (s < ns) ? __ldg(o_lat + (size_t(s0 + s) * heads + h) * K + k) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKChunk; ++kk) {
      const float o = so[warp * kKChunk + kk];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int j = lane + 32 * q;
        if (j < d_h) acc[q] = fmaf(o, sw[kk * d_h + j], acc[q]);
      }
    }
  }
  if (warp < ns) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int j = lane + 32 * q;
      if (j < d_h) out[(size_t(s0 + warp) * heads + h) * d_h + j] = branch_scale * acc[q];
    }
  }
}

cudaError_t launch_out_proj(const mlra_config_t& c, const float* o_latent, const void* w_uv,
                            float* out, int batch, cudaStream_t st) {
  dim3 grid(c.n_heads, (batch + kSeqBlk - 1) / kSeqBlk);
  size_t sm = sizeof(float) * (kKChunk * c.d_h + kSeqBlk * kKChunk);
  if (c.dtype == MLRA_BF16)
    out_proj_kernel<__nv_bfloat16><<<grid, 256, sm, st>>>(
        o_latent, (const __nv_bfloat16*)w_uv, out, batch, c.n_heads, c.n_blocks, c.d_cb, c.d_h,
        c.branch_scale);
  else
    out_proj_kernel<float><<<grid, 256, sm, st>>>(o_latent, (const float*)w_uv, out, batch,
                                                  c.n_heads, c.n_blocks, c.d_cb, c.d_h,
                                                  c.branch_scale);
  return cudaGetLastError();
}

}  // namespace mlra
