// Tensor-core weight contractions of the decode step (sm_100a): the query
// absorption q_abs = W_uk q_nope and the output up-projection
// out = branch_scale * W_uv^T o, the latter optionally fused with the split-KV
// combine that produces o ("Multi-Head Low-Rank Attention", Main Findings:
// the absorbable steps of the MQA-style decode; Methodology: the per-branch
// outputs are concatenated and projected by W_uv with the 1/sqrt(n_blocks)
// branch scale).
//
// Both are per-head batched GEMMs with a tiny batch (the decode batch), so the
// weights are the traffic: each CTA streams one head's weight tile with TMA and
// runs a 128-row tcgen05 product with the sequences on the N side.
//  * absorb:  D[r, s] = sum_j W_uk[r, j] q_nope[s, j]   (A = W_uk K-major,
//             B = q_nope K-major, both bf16 from global);
//  * out_proj: D[j, s] = sum_k W_uv[k, j] o[s, k]        (A = W_uv MN-major,
//             B = o as bf16 hi + lo pairs written by the CTA's threads, so the
//             fp32 o enters with ~16 significant bits).
#include "dispatch.h"
#include "sm100_ptx.cuh"

#include <cudaTypedefs.h>
#include <math.h>

namespace mlra {
namespace {

using namespace ptx;

constexpr uint64_t kWaitNs = 2000000000ull;

// Bounded wait on an mbarrier phase: false once 2 s have passed.
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitNs) return false;
  return true;
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
  return n <= 32 ? 32u : n <= 64 ? 64u : n <= 128 ? 128u : 256u;
}

// ---------------------------------------------------------------------------
// Absorption.  CTA = (head h, 128 latent rows r0.., NT sequences s0..).
// q_abs[s, h, r] for r = b * d_cb + i; the 128 rows of a CTA lie in one branch
// (d_cb is a multiple of 128) and are consecutive rows of W_uk viewed as
// [nb * H * d_cb, d_h].
// ---------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(128, 1)
    absorb_tc_kernel(const __grid_constant__ CUtensorMap map_w,
                     const __grid_constant__ CUtensorMap map_q, float* __restrict__ q_abs,
                     int batch, int heads, int nb, int d_cb, float alpha) {
  constexpr int kA = 128 * 128;  // bytes of one 64-column box of 128 rows
  constexpr int kB = NT * 128;   // bytes of one 64-column box of NT rows
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int loaded;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, r0 = blockIdx.y * 128, s0 = blockIdx.z * NT;
  const int K = nb * d_cb;
  const uint32_t bar_load = smem_addr(&bars[0]), bar_mma = smem_addr(&bars[1]);
  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    loaded = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(&tmem_slot), tmem_cols_for(NT));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    const uint32_t a = smem_addr(sm), b = a + 2 * kA;
    if (lane == 0) {
      const int row = (r0 / d_cb * heads + h) * d_cb + r0 % d_cb;
      mbar_arrive_expect_tx(bar_load, 2 * kA + 2 * kB);
      tma_load_2d(a, &map_w, 0, row, bar_load);
      tma_load_2d(a + kA, &map_w, 64, row, bar_load);
      tma_load_3d(b, &map_q, 0, h, s0, bar_load);
      tma_load_3d(b + kB, &map_q, 64, h, s0, bar_load);
    }
    __syncwarp();
    if (wait_phase(bar_load, 0)) {
      if (lane == 0) loaded = 1;
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
      const uint64_t da = smem_desc(a, 16, 1024, kSwizzle128B);
      const uint64_t db = smem_desc(b, 16, 1024, kSwizzle128B);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_ss_warp(tmem, da + uint64_t(((k >> 2) * kA + (k & 3) * 32) >> 4),
                    db + uint64_t(((k >> 2) * kB + (k & 3) * 32) >> 4), idesc, k > 0 ? 1u : 0u);
    }
    mma_commit_warp(bar_mma);  // also completes at once when nothing was issued
  }
  const bool done = wait_phase(bar_mma, 0);
  tc_fence_after();
  __syncthreads();
  // a load or product that never finished leaves NaN rather than stale values
  const bool good = done && loaded;
  const int r = r0 + 32 * warp + lane;
  const uint32_t row_t = tmem + (uint32_t(32 * warp) << 16);
#pragma unroll 1
  for (int c = 0; c < NT; c += 32) {
    uint32_t v[32];
    if (NT >= 32) {
      tmem_ld32(row_t + c, v);
    } else {
      uint32_t w[16];
      tmem_ld16(row_t + c, w);
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = w[k];
    }
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < (NT < 32 ? NT : 32); ++k) {
      const int s = s0 + c + k;
      if (s < batch)
        q_abs[(size_t(s) * heads + h) * K + r] =
            good ? __uint_as_float(v[k]) * alpha : __int_as_float(0x7fc00000);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols_for(NT));
  }
}

// ---------------------------------------------------------------------------
// Output projection, optionally fused with the split-KV combine.
// A cluster of C = K / 64 CTAs per (head h, NT sequences s0..): CTA c of the
// cluster owns the 64 rows k = 64c.. of K = nb * d_cb (all inside one branch)
// and computes the partial product D_c[j, s] = sum_{k in chunk} W_uv[k, j] o[s, k]
// (128 TMEM lanes = the d_h = 128 features, NT columns):
//   A: W_uv rows of the chunk, all 128 features, one TMA load (MN-major);
//   B: o[s, h, chunk] split into bf16 hi and lo, written by the CTA's threads
//      (K-major, 128-byte swizzle).  With COMBINE, o is the log-sum-exp merge
//      of the sequence's split partials: o = sum_k exp(lse_k - lse) o_k.
// The C partials are then summed in a fixed order through distributed shared
// memory, each CTA producing NT / C of the sequences' outputs (deterministic).
// ---------------------------------------------------------------------------
constexpr int kOpChunk = 64;              // K rows per CTA
constexpr int kOpA = kOpChunk * 256;      // A bytes (64 rows x 128 bf16)

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162 t;
  t = __floats2bfloat162_rn(v[0], v[1]); u.x = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[2], v[3]); u.y = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[4], v[5]); u.z = *reinterpret_cast<uint32_t*>(&t);
  t = __floats2bfloat162_rn(v[6], v[7]); u.w = *reinterpret_cast<uint32_t*>(&t);
  return u;
}
__device__ __forceinline__ void unpack8_bf16(const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    v[2 * k] = __uint_as_float(w[k] << 16);
    v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}
__device__ __forceinline__ void fma8(float (&v)[8], float w, const float4& x, const float4& y) {
  v[0] = fmaf(w, x.x, v[0]); v[1] = fmaf(w, x.y, v[1]);
  v[2] = fmaf(w, x.z, v[2]); v[3] = fmaf(w, x.w, v[3]);
  v[4] = fmaf(w, y.x, v[4]); v[5] = fmaf(w, y.y, v[5]);
  v[6] = fmaf(w, y.z, v[6]); v[7] = fmaf(w, y.w, v[7]);
}

struct OpArgs {
  const float* o_latent_in;  // !COMBINE: [B, H, K]
  const char* ws;            // COMBINE: workspace (plan + split partials)
  WsLayout L;
  float* o_latent_out;       // COMBINE: optional [B, H, K]
  float* lse_out;            // COMBINE: optional [B, H, nb]
  float* out;                // [B, H, d_h]
  int batch, heads, nb, d_cb;
  float branch_scale;
};

template <int NT>
struct OpShape {
  static constexpr int kB = NT * 128;               // hi (or lo) operand bytes
  static constexpr int kRed = NT * 128 * 4;         // fp32 partial D, [s][j]
  static constexpr int kOperands = kOpA + 2 * kB;   // A + B hi + B lo
  static constexpr int kMain = kOperands > kRed ? kOperands : kRed;
};

template <bool COMBINE, int NT>
__global__ void __launch_bounds__(128, 8)
    out_proj_tc_kernel(const __grid_constant__ CUtensorMap map_w, const OpArgs a) {
  using S = OpShape<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  uint8_t* smA = sm;
  uint8_t* smB = sm + kOpA;                      // hi at +0, lo at +kB
  float* red = reinterpret_cast<float*>(sm);     // after the product: partial D [s][j]
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int s_fail;
  const uint32_t AFULL = smem_addr(&bars[0]), DONE = smem_addr(&bars[1]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = (a.nb * a.d_cb) / kOpChunk;      // CTAs per cluster
  const int kc = int(cluster_rank());
  const int h = blockIdx.x / C, s0 = blockIdx.y * NT;
  const int H = a.heads, nb = a.nb, K = nb * a.d_cb;
  const int k0 = kc * kOpChunk, b = k0 / a.d_cb, i0 = k0 % a.d_cb;
  if (threadIdx.x == 0) {
    mbar_init(AFULL, 1);
    mbar_init(DONE, 1);
    s_fail = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(&tmem_slot), tmem_cols_for(NT));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (threadIdx.x == 0) {
    const int row = (b * H + h) * a.d_cb + i0;
    mbar_arrive_expect_tx(AFULL, kOpA);
    tma_load_2d(smem_addr(smA), &map_w, 0, row, AFULL);
    tma_load_2d(smem_addr(smA) + kOpA / 2, &map_w, 64, row, AFULL);
  }
  const int n_seq = min(NT, a.batch - s0);
  const int32_t* slot_off = COMBINE ? reinterpret_cast<const int32_t*>(a.ws + a.L.slot_off) : nullptr;
  const float* o_part = COMBINE ? reinterpret_cast<const float*>(a.ws + a.L.o_part) : nullptr;
  const float* lse_part = COMBINE ? reinterpret_cast<const float*>(a.ws + a.L.lse_part) : nullptr;
  // ---- B operand: o[s, h, k0 + 8 part ..] as bf16 hi / lo, 8 values per group
#pragma unroll
  for (int u = 0; u < NT / 16; ++u) {
    const int g = threadIdx.x + 128 * u;
    const int sl = g >> 3, part = g & 7;
    const int s = s0 + sl, kk = k0 + 8 * part;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (sl < n_seq) {
      const size_t orow = (size_t(s) * H + h) * K + kk;  // o[s, h, kk..kk+7]
      if (COMBINE) {
        // online log-sum-exp merge over the splits, four per round: each
        // split's lse and partial are loaded together, so a round costs one
        // memory round trip
        const int q0 = __ldg(slot_off + s), q1 = __ldg(slot_off + s + 1);
        const size_t lstride = size_t(H) * nb, pstride = lstride * a.d_cb;
        const float* l0 = lse_part + size_t(h) * nb + b;
        const float* p0 = o_part + (size_t(h) * nb + b) * a.d_cb + i0 + 8 * part;
        float m = -INFINITY, den = 0.f;
        for (int q = q0; q < q1; q += 4) {
          float lz[4];
          float4 x[4], y[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const bool in = q + r < q1;
            const size_t qq = size_t(in ? q + r : q0);
            lz[r] = in ? __ldg(l0 + qq * lstride) : -INFINITY;
            const float4* p = reinterpret_cast<const float4*>(p0 + qq * pstride);
            x[r] = __ldg(p);
            y[r] = __ldg(p + 1);
          }
          const float mr = fmaxf(fmaxf(lz[0], lz[1]), fmaxf(lz[2], lz[3]));
          const float mn = fmaxf(m, mr);
          if (mn == -INFINITY) continue;  // splits without tokens
          const float sc = expf(m - mn);  // 0 while m is still -inf
          den *= sc;
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] *= sc;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float w = expf(lz[r] - mn);
            den += w;
            fma8(v, w, x[r], y[r]);
          }
          m = mn;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] *= inv;
        if (a.lse_out && i0 == 0 && part == 0)
          a.lse_out[(size_t(s) * H + h) * nb + b] = den > 0.f ? m + logf(den) : -INFINITY;
        if (a.o_latent_out) {
          float4* d = reinterpret_cast<float4*>(a.o_latent_out + orow);
          d[0] = make_float4(v[0], v[1], v[2], v[3]);
          d[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
      } else {
        const float4* p = reinterpret_cast<const float4*>(a.o_latent_in + orow);
        const float4 x = __ldg(p), y = __ldg(p + 1);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
        v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
      }
    }
    const uint4 hi = pack8_bf16(v);
    float vh[8];
    unpack8_bf16(hi, vh);
#pragma unroll
    for (int e = 0; e < 8; ++e) vh[e] = v[e] - vh[e];
    const uint4 lo = pack8_bf16(vh);
    const int off = sl * 128 + ((part ^ (sl & 7)) << 4);  // 128-byte swizzle
    *reinterpret_cast<uint4*>(smB + off) = hi;
    *reinterpret_cast<uint4*>(smB + S::kB + off) = lo;
  }
  fence_proxy_async_smem();
  __syncthreads();

  // ---- partial product of this chunk
  if (warp == 0) {
    if (wait_phase(AFULL, 0)) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(128, NT, true, false);
      const uint32_t a0 = smem_addr(smA), b0 = smem_addr(smB);
#pragma unroll
      for (int ks = 0; ks < kOpChunk / 16; ++ks) {
        const uint64_t da = smem_desc(a0 + ks * 2048, kOpA / 2, 1024, kSwizzle128B);
        const uint64_t dh = smem_desc(b0 + ks * 32, 16, 1024, kSwizzle128B);
        const uint64_t dl = smem_desc(b0 + S::kB + ks * 32, 16, 1024, kSwizzle128B);
        mma_ss_warp(tmem, da, dh, idesc, ks > 0 ? 1u : 0u);
        mma_ss_warp(tmem, da, dl, idesc, 1u);
      }
    } else if (lane == 0) {
      s_fail = 1;
    }
    __syncwarp();
    mma_commit_warp(DONE);  // completes at once when nothing was issued
  }
  if (!wait_phase(DONE, 0)) s_fail = 1;
  tc_fence_after();
  __syncthreads();
  const bool good = !s_fail;
  // D_c -> red[s][j] (thread = feature j = its TMEM lane); A / B are dead now
  {
    const int j = threadIdx.x;
    const uint32_t row_t = tmem + (uint32_t(32 * warp) << 16);
#pragma unroll 1
    for (int c = 0; c < NT; c += 32) {
      uint32_t v[32];
      if (NT >= 32) {
        tmem_ld32(row_t + c, v);
      } else {
        uint32_t w[16];
        tmem_ld16(row_t + c, w);
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = w[k];
      }
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < (NT < 32 ? NT : 32); ++k)
        red[(c + k) * 128 + j] = good ? __uint_as_float(v[k]) : __int_as_float(0x7fc00000);
    }
  }
  cluster_sync_all();  // every CTA's partial is in its shared memory
  // out[s, h, j] = branch_scale * sum_c D_c[j, s], summed in cluster-rank order;
  // CTA kc produces sequences kc * NT / C ..
  {
    const int per = NT / C;
    const uint32_t red0 = smem_addr(red);
    for (int e = threadIdx.x; e < per * 128; e += 128) {
      const int sl = kc * per + e / 128, j = e % 128;
      const uint32_t off = uint32_t((sl * 128 + j) * 4);
      float acc = 0.f;
      for (int r = 0; r < C; ++r) acc += dsmem_ld_f32(dsmem_addr(red0 + off, uint32_t(r)));
      if (s0 + sl < a.batch) a.out[(size_t(s0 + sl) * H + h) * 128 + j] = a.branch_scale * acc;
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its partial
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols_for(NT));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor map with 128-byte swizzle over `rank` dims (innermost first).
bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
             strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Kern>
cudaError_t set_smem_once(Kern kern, int bytes, int* done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && done[dev] >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = bytes;
  return e;
}

template <int NT>
cudaError_t absorb_t(const mlra_config_t& c, const CUtensorMap& mw, const CUtensorMap& mq,
                     float* q_abs, int batch, float alpha, cudaStream_t st) {
  static int done[64] = {0};
  const int smem = 1024 + 2 * 128 * 128 + 2 * NT * 128;
  cudaError_t e = set_smem_once(absorb_tc_kernel<NT>, smem, done);
  if (e != cudaSuccess) return e;
  dim3 grid(c.n_heads, c.n_blocks * c.d_cb / 128, (batch + NT - 1) / NT);
  return launch_pdl(absorb_tc_kernel<NT>, grid, dim3(128), smem, st, mw, mq, q_abs, batch,
                    c.n_heads, c.n_blocks, c.d_cb, alpha);
}

template <bool COMBINE, int NT>
cudaError_t out_proj_t(const mlra_config_t& c, const CUtensorMap& mw, const OpArgs& a,
                       cudaStream_t st) {
  static int done[64] = {0};
  const int C = c.n_blocks * c.d_cb / kOpChunk;
  const int smem = 1024 + OpShape<NT>::kMain;
  if (smem > 232448 || C < 1 || C > 8 || NT % C != 0) return cudaErrorInvalidValue;
  auto kern = out_proj_tc_kernel<COMBINE, NT>;
  cudaError_t e = set_smem_once(kern, smem, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c.n_heads * C, (a.batch + NT - 1) / NT);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, mw, a);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool proj_tc_supported(const mlra_config_t& c) {
  return c.dtype == MLRA_BF16 && c.d_h == 128 && c.d_cb % 128 == 0 &&
         c.n_blocks * c.d_cb <= 512;
}

cudaError_t launch_absorb_tc(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                             float* q_abs, int batch, float alpha, cudaStream_t st) {
  if (!proj_tc_supported(c) || !aligned16(q_nope) || !aligned16(w_uk)) return cudaErrorNotSupported;
  const int NT = batch <= 16 ? 16 : batch <= 32 ? 32 : batch <= 64 ? 64 : batch <= 128 ? 128 : 256;
  CUtensorMap mw, mq;
  const cuuint64_t wd[2] = {128, cuuint64_t(c.n_blocks) * c.n_heads * c.d_cb};
  const cuuint64_t ws[1] = {256};
  const cuuint32_t wb[2] = {64, 128};
  const cuuint64_t qd[3] = {128, cuuint64_t(c.n_heads), cuuint64_t(batch)};
  const cuuint64_t qs[2] = {256, cuuint64_t(c.n_heads) * 256};
  const cuuint32_t qb[3] = {64, 1, cuuint32_t(NT)};
  if (!encode_bf16(&mw, w_uk, 2, wd, ws, wb) || !encode_bf16(&mq, q_nope, 3, qd, qs, qb))
    return cudaErrorInvalidValue;
  switch (NT) {
    case 16: return absorb_t<16>(c, mw, mq, q_abs, batch, alpha, st);
    case 32: return absorb_t<32>(c, mw, mq, q_abs, batch, alpha, st);
    case 64: return absorb_t<64>(c, mw, mq, q_abs, batch, alpha, st);
    case 128: return absorb_t<128>(c, mw, mq, q_abs, batch, alpha, st);
    default: return absorb_t<256>(c, mw, mq, q_abs, batch, alpha, st);
  }
}

// o_latent_in != nullptr: plain projection of o_latent.  Otherwise the split
// partials of `ws` are merged on the way (o_latent_out / lse_out optional).
cudaError_t launch_out_proj_tc(const mlra_config_t& c, const float* o_latent_in, const void* ws,
                               const WsLayout& L, float* o_latent_out,
                               float* lse_out, const void* w_uv, float* out, int batch,
                               cudaStream_t st) {
  if (!proj_tc_supported(c) || !aligned16(w_uv)) return cudaErrorNotSupported;
  if (o_latent_in && !aligned16(o_latent_in)) return cudaErrorNotSupported;
  if (o_latent_out && !aligned16(o_latent_out)) return cudaErrorNotSupported;
  CUtensorMap mw;
  const cuuint64_t wd[2] = {128, cuuint64_t(c.n_blocks) * c.n_heads * c.d_cb};
  const cuuint64_t wsb[1] = {256};
  const cuuint32_t wb[2] = {64, kOpChunk};
  if (!encode_bf16(&mw, w_uv, 2, wd, wsb, wb)) return cudaErrorInvalidValue;
  OpArgs a;
  a.o_latent_in = o_latent_in;
  a.ws = static_cast<const char*>(ws);
  a.L = L;
  a.o_latent_out = o_latent_out;
  a.lse_out = lse_out;
  a.out = out;
  a.batch = batch;
  a.heads = c.n_heads;
  a.nb = c.n_blocks;
  a.d_cb = c.d_cb;
  a.branch_scale = c.branch_scale;
  // small N tiles keep many clusters in flight; W_uv is re-read per tile from L2
  const int NT = batch <= 64 ? 16 : batch <= 256 ? 32 : 64;
  if (o_latent_in) {
    switch (NT) {
      case 16: return out_proj_t<false, 16>(c, mw, a, st);
      case 32: return out_proj_t<false, 32>(c, mw, a, st);
      default: return out_proj_t<false, 64>(c, mw, a, st);
    }
  }
  switch (NT) {
    case 16: return out_proj_t<true, 16>(c, mw, a, st);
    case 32: return out_proj_t<true, 32>(c, mw, a, st);
    default: return out_proj_t<true, 64>(c, mw, a, st);
  }
}

}  // namespace mlra
