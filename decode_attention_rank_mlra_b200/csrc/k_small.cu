// Small kernels of the decode step: split plan, query absorption, split-KV
// combine and output up-projection.  All fp32 SIMT: together they move well
// under 5% of the bytes of the attention kernel (see the layer description in
// include/mlra.h for the maths).
#include "dispatch.h"

#include <math.h>

#include <algorithm>

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
  pdl_wait();
  // the error word is clear before the dependent attention kernel can start
  // (it does not wait for this kernel and may record an error at once)
  if (threadIdx.x == 0) {
    hdr->error = 0;
    hdr->fallback_error = 0;
    hdr->fallback_done = 0;
    __threadfence();
    s_bad = 0;
  }
  __syncthreads();
  pdl_trigger();
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
    const int a = tile_off[s], e = tile_off[s + 1];
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
  return launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, st, seqlens, batch, cap, ctas_per_group,
                    L.max_slots, reinterpret_cast<WsHeader*>(base),
                    reinterpret_cast<int32_t*>(base + L.tile_off),
                    reinterpret_cast<int32_t*>(base + L.slot_off));
}

// ---------------------------------------------------------------------------
// Absorption: q_abs[s,h,b,i] = sum_j W_uk[b,h,i,j] q_nope[s,h,j]
// Block = (head h, 256 latent rows, 8 sequences), one thread per latent row
// (b,i).  The thread issues every 16-byte load of its W_uk row (d_h contiguous
// values) for a 64-wide chunk at once, then multiplies with q_nope of the 8
// sequences read from shared memory as float4 (one address per warp:
// broadcast).
// ---------------------------------------------------------------------------
constexpr int kSeqBlk = 8;
constexpr int kAbsThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& u, float (&w)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(h[k]);
    w[2 * k] = f.x;
    w[2 * k + 1] = f.y;
  }
}

template <typename T> struct Chunk8;
template <> struct Chunk8<__nv_bfloat16> {  // 8 bf16 = one 16-byte load
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void get(float (&w)[8]) const { unpack8(u, w); }
};
template <> struct Chunk8<float> {  // 8 fp32 = two 16-byte loads
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p + 4));
  }
  __device__ __forceinline__ void get(float (&w)[8]) const {
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w; w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  }
};

template <typename T>
__global__ void __launch_bounds__(kAbsThreads) absorb_kernel(const T* __restrict__ q_nope,
                                                             const T* __restrict__ w_uk,
                                                             float* __restrict__ q_abs, int batch,
                                                             int heads, int nb, int d_cb, int d_h,
                                                             float alpha) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float4 sq4[];  // [kSeqBlk][d_h / 4]
  float* sq = reinterpret_cast<float*>(sq4);
  const int h = blockIdx.x, s0 = blockIdx.z * kSeqBlk;
  const int ns = min(kSeqBlk, batch - s0);
  for (int x = threadIdx.x; x < kSeqBlk * d_h; x += blockDim.x) {
    const int s = x / d_h, j = x - s * d_h;
    sq[x] = (s < ns) ? ld_f32(q_nope + (size_t(s0 + s) * heads + h) * d_h + j) : 0.f;
  }
  __syncthreads();
  const int K = nb * d_cb;
  const int r = blockIdx.y * kAbsThreads + threadIdx.x;
  if (r >= K) return;
  const int b = r / d_cb, i = r - b * d_cb;
  const T* wrow = w_uk + ((size_t(b) * heads + h) * d_cb + i) * d_h;
  float acc[kSeqBlk];
#pragma unroll
  for (int s = 0; s < kSeqBlk; ++s) acc[s] = 0.f;
  const int q4 = d_h / 4;
  for (int j0 = 0; j0 < d_h; j0 += 64) {
    const int nc = min(8, (d_h - j0) / 8);
    Chunk8<T> c[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < nc) c[k].load(wrow + j0 + 8 * k);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k >= nc) break;
      float w[8];
      c[k].get(w);
      const int jq = (j0 + 8 * k) / 4;
#pragma unroll
      for (int s = 0; s < kSeqBlk; ++s) {
        const float4 qa = sq4[s * q4 + jq], qb = sq4[s * q4 + jq + 1];
        acc[s] = fmaf(w[0], qa.x, acc[s]); acc[s] = fmaf(w[1], qa.y, acc[s]);
        acc[s] = fmaf(w[2], qa.z, acc[s]); acc[s] = fmaf(w[3], qa.w, acc[s]);
        acc[s] = fmaf(w[4], qb.x, acc[s]); acc[s] = fmaf(w[5], qb.y, acc[s]);
        acc[s] = fmaf(w[6], qb.z, acc[s]); acc[s] = fmaf(w[7], qb.w, acc[s]);
      }
    }
  }
  for (int s = 0; s < ns; ++s) q_abs[(size_t(s0 + s) * heads + h) * K + r] = acc[s] * alpha;
}

cudaError_t launch_absorb(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                          float* q_abs, int batch, float alpha, cudaStream_t st) {
  dim3 grid(c.n_heads, (c.n_blocks * c.d_cb + kAbsThreads - 1) / kAbsThreads,
            (batch + kSeqBlk - 1) / kSeqBlk);
  size_t sm = sizeof(float) * kSeqBlk * c.d_h;
  if (c.dtype == MLRA_BF16)
    return launch_pdl(absorb_kernel<__nv_bfloat16>, grid, dim3(kAbsThreads), sm, st,
                      (const __nv_bfloat16*)q_nope, (const __nv_bfloat16*)w_uk, q_abs, batch,
                      c.n_heads, c.n_blocks, c.d_cb, c.d_h, alpha);
  return launch_pdl(absorb_kernel<float>, grid, dim3(kAbsThreads), sm, st, (const float*)q_nope,
                    (const float*)w_uk, q_abs, batch, c.n_heads, c.n_blocks, c.d_cb, c.d_h, alpha);
}

// ---------------------------------------------------------------------------
// Split-KV combine: one warp per (sequence, head, branch).  Lane k reads the
// lse of split k (32 splits per round), the merge weights come from warp
// reductions, and each lane accumulates 4 consecutive latent values per split
// with 16-byte loads (d_cb a multiple of 128 uses the vector path).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) combine_kernel(const char* __restrict__ ws, WsLayout L,
                                                      int batch, int heads, int nb, int d_cb,
                                                      float* __restrict__ o_latent,
                                                      float* __restrict__ lse_out) {
  pdl_wait();
  pdl_trigger();
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
  float* lse_dst = lse_out ? lse_out + (size_t(s) * heads + h) * nb + b : nullptr;
  // max and sum of exp over the splits
  float m = -INFINITY;
  for (int k = k0 + lane; k < k1; k += 32) m = fmaxf(m, __ldg(lse_part + size_t(k) * slot_stride + row));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (k1 <= k0 || m == -INFINITY) {  // no token (empty sequence / every page rejected)
    for (int i = lane; i < d_cb; i += 32) dst[i] = 0.f;
    if (lse_dst && lane == 0) *lse_dst = -INFINITY;
    return;
  }
  float den = 0.f;
  for (int k = k0 + lane; k < k1; k += 32) den += expf(__ldg(lse_part + size_t(k) * slot_stride + row) - m);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  const float inv = 1.f / den;
  if ((d_cb & 127) == 0) {
    for (int i0 = 0; i0 < d_cb; i0 += 128) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int kb = k0; kb < k1; kb += 32) {
        const int k = kb + lane;
        const float wl = (k < k1) ? expf(__ldg(lse_part + size_t(k) * slot_stride + row) - m) * inv : 0.f;
        const int nk = min(32, k1 - kb);
        for (int j = 0; j < nk; ++j) {
          const float w = __shfl_sync(0xffffffffu, wl, j);
          const float4 o = __ldg(reinterpret_cast<const float4*>(
              o_part + (size_t(kb + j) * slot_stride + row) * d_cb + i0 + 4 * lane));
          acc.x = fmaf(w, o.x, acc.x); acc.y = fmaf(w, o.y, acc.y);
          acc.z = fmaf(w, o.z, acc.z); acc.w = fmaf(w, o.w, acc.w);
        }
      }
      *reinterpret_cast<float4*>(dst + i0 + 4 * lane) = acc;
    }
  } else {
    for (int i = lane; i < d_cb; i += 32) {
      float acc = 0.f;
      for (int k = k0; k < k1; ++k) {
        const float w = expf(__ldg(lse_part + size_t(k) * slot_stride + row) - m) * inv;
        acc = fmaf(w, __ldg(o_part + (size_t(k) * slot_stride + row) * d_cb + i), acc);
      }
      dst[i] = acc;
    }
  }
  if (lse_dst && lane == 0) *lse_dst = m + logf(den);
}

cudaError_t launch_combine(const mlra_config_t& c, const void* ws, const WsLayout& L, int batch,
                           float* o_latent, float* lse, cudaStream_t st) {
  const int rows = batch * c.n_heads * c.n_blocks;
  const int blocks = (rows * 32 + 255) / 256;
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, st, static_cast<const char*>(ws), L,
                    batch, c.n_heads, c.n_blocks, c.d_cb, o_latent, lse);
}

// ---------------------------------------------------------------------------
// Output up-projection: out[s,h,j] = branch_scale * sum_{b,i} o[s,h,b,i] W_uv[b,h,i,j]
// Block = (head h, 8 sequences), 8 warps.  Warp w sums the latent rows k=(b,i)
// of its eighth of K = nb*d_cb; lane l owns output columns 4l..4l+3 (one
// coalesced row segment of W_uv per warp and k, read as 4 values per lane).
// o of the 8 sequences is kept transposed in shared memory ([k][s], two
// float4 per k, broadcast across the warp); the eight warps' partial sums are
// added through shared memory.
// ---------------------------------------------------------------------------
constexpr int kOpWarps = 8;

__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}

template <typename T>
__global__ void __launch_bounds__(kOpWarps * 32) out_proj_kernel(const float* __restrict__ o_lat,
                                                                 const T* __restrict__ w_uv,
                                                                 float* __restrict__ out, int batch,
                                                                 int heads, int nb, int d_cb,
                                                                 int d_h, float branch_scale) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float4 sm4[];
  const int K = nb * d_cb;
  float* so = reinterpret_cast<float*>(sm4);    // [K][kSeqBlk]
  float* red = so + size_t(K) * kSeqBlk;        // [kOpWarps][kSeqBlk][d_h]
  const int h = blockIdx.x, s0 = blockIdx.y * kSeqBlk;
  const int ns = min(kSeqBlk, batch - s0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int x = threadIdx.x; x < kSeqBlk * K; x += blockDim.x) {
    const int s = x / K, k = x - s * K;
    so[k * kSeqBlk + s] = (s < ns) ? __ldg(o_lat + (size_t(s0 + s) * heads + h) * K + k) : 0.f;
  }
  __syncthreads();
  const int c0 = 4 * lane;
  const bool cok = c0 < d_h;
  float4 acc[kSeqBlk];
#pragma unroll
  for (int s = 0; s < kSeqBlk; ++s) acc[s] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int per = K / kOpWarps;  // K is a multiple of 8
  const int k0 = warp * per, k1 = k0 + per;
  int b = k0 / d_cb, i = k0 - b * d_cb;
  const T* wp = w_uv + ((size_t(b) * heads + h) * d_cb + i) * d_h + c0;
  for (int k = k0; k < k1; k += 8) {
    float4 w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {  // 8 rows in flight
      w[u] = cok ? load4(wp) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (++i == d_cb) { i = 0; ++b; wp = w_uv + (size_t(b) * heads + h) * d_cb * d_h + c0; }
      else wp += d_h;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 oa = *reinterpret_cast<const float4*>(so + (k + u) * kSeqBlk);
      const float4 ob = *reinterpret_cast<const float4*>(so + (k + u) * kSeqBlk + 4);
      const float o[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
#pragma unroll
      for (int s = 0; s < kSeqBlk; ++s) {
        acc[s].x = fmaf(o[s], w[u].x, acc[s].x); acc[s].y = fmaf(o[s], w[u].y, acc[s].y);
        acc[s].z = fmaf(o[s], w[u].z, acc[s].z); acc[s].w = fmaf(o[s], w[u].w, acc[s].w);
      }
    }
  }
  if (cok) {
#pragma unroll
    for (int s = 0; s < kSeqBlk; ++s)
      *reinterpret_cast<float4*>(red + (size_t(warp) * kSeqBlk + s) * d_h + c0) = acc[s];
  }
  __syncthreads();
  for (int x = threadIdx.x; x < kSeqBlk * d_h; x += blockDim.x) {
    const int s = x / d_h, j = x - s * d_h;
    if (s >= ns) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kOpWarps; ++w) v += red[(size_t(w) * kSeqBlk + s) * d_h + j];
    out[(size_t(s0 + s) * heads + h) * d_h + j] = branch_scale * v;
  }
}

cudaError_t launch_out_proj(const mlra_config_t& c, const float* o_latent, const void* w_uv,
                            float* out, int batch, cudaStream_t st) {
  if ((c.n_blocks * c.d_cb) % 64 != 0 || c.d_h % 4 != 0) return cudaErrorInvalidValue;
  dim3 grid(c.n_heads, (batch + kSeqBlk - 1) / kSeqBlk);
  const size_t sm = sizeof(float) * (size_t(c.n_blocks) * c.d_cb * kSeqBlk +
                                     size_t(kOpWarps) * kSeqBlk * c.d_h);
  if (sm > 48 * 1024) {
    // opt in once per device to the shared memory a wide latent needs
    static int set_for[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || set_for[dev] < (int)sm) {
      cudaError_t e = cudaFuncSetAttribute(out_proj_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(out_proj_kernel<float>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) set_for[dev] = (int)sm;
    }
  }
  if (c.dtype == MLRA_BF16)
    return launch_pdl(out_proj_kernel<__nv_bfloat16>, grid, dim3(kOpWarps * 32), sm, st, o_latent,
                      (const __nv_bfloat16*)w_uv, out, batch, c.n_heads, c.n_blocks, c.d_cb,
                      c.d_h, c.branch_scale);
  return launch_pdl(out_proj_kernel<float>, grid, dim3(kOpWarps * 32), sm, st, o_latent,
                    (const float*)w_uv, out, batch, c.n_heads, c.n_blocks, c.d_cb, c.d_h,
                    c.branch_scale);
}

// ---------------------------------------------------------------------------
// Staging of a step's inputs from page-locked host memory: the kernel reads
// the mapped host ranges directly (bypassing the cache, the host rewrites them
// between steps) and writes the workspace.  At decode sizes (tens of KB) one
// launch costs a PCIe round trip, where each copy-engine transfer carries a
// fixed cost several times larger.
namespace {

struct StageArgs {
  StageCopy c[3];
  int n;
};

template <typename U>
__device__ __forceinline__ void stage_units(const void* src, void* dst, size_t n, size_t tid,
                                            size_t nth) {
  const U* s = static_cast<const U*>(src);
  U* d = static_cast<U*>(dst);
  size_t i = tid;
  // four loads in flight per thread before the first store
  for (; i + 3 * nth < n; i += 4 * nth) {
    const U v0 = __ldcv(s + i), v1 = __ldcv(s + i + nth), v2 = __ldcv(s + i + 2 * nth),
            v3 = __ldcv(s + i + 3 * nth);
    d[i] = v0;
    d[i + nth] = v1;
    d[i + 2 * nth] = v2;
    d[i + 3 * nth] = v3;
  }
  for (; i < n; i += nth) d[i] = __ldcv(s + i);
}

__host__ __device__ inline int stage_unit(const StageCopy& c) {
  const uintptr_t m = reinterpret_cast<uintptr_t>(c.src) | reinterpret_cast<uintptr_t>(c.dst) |
                      uintptr_t(c.bytes);
  return (m & 15) == 0 ? 16 : (m & 7) == 0 ? 8 : (m & 3) == 0 ? 4 : (m & 1) == 0 ? 2 : 1;
}

__global__ void __launch_bounds__(256) stage_kernel(StageArgs a) {
  // the previous step's kernels may still read the destination
  pdl_wait();
  pdl_trigger();
  const size_t tid = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t nth = size_t(gridDim.x) * blockDim.x;
  for (int k = 0; k < a.n; ++k) {
    const StageCopy& c = a.c[k];
    switch (stage_unit(c)) {
      case 16: stage_units<uint4>(c.src, c.dst, c.bytes / 16, tid, nth); break;
      case 8: stage_units<uint2>(c.src, c.dst, c.bytes / 8, tid, nth); break;
      case 4: stage_units<unsigned int>(c.src, c.dst, c.bytes / 4, tid, nth); break;
      case 2: stage_units<unsigned short>(c.src, c.dst, c.bytes / 2, tid, nth); break;
      default: stage_units<unsigned char>(c.src, c.dst, c.bytes, tid, nth); break;
    }
  }
}

}  // namespace

cudaError_t launch_stage(const StageCopy* copies, int n, cudaStream_t st) {
  if (n < 1 || n > 3) return cudaErrorInvalidValue;
  StageArgs a{};
  a.n = n;
  size_t units = 0;
  for (int k = 0; k < n; ++k) {
    a.c[k] = copies[k];
    units = std::max(units, copies[k].bytes / size_t(stage_unit(copies[k])));
  }
  // one unit per thread up to 4 waves of 148 CTAs; beyond that each thread
  // loops, four loads at a time
  const size_t blocks = std::min<size_t>(std::max<size_t>((units + 255) / 256, 1), 592);
  return launch_pdl(stage_kernel, dim3(unsigned(blocks)), dim3(256), 0, st, a);
}

}  // namespace mlra
