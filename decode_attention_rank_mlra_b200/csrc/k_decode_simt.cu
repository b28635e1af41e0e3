// fp32 SIMT split-KV decode attention over the latent cache.
//
// Computes, for one split of one sequence and every (head, branch) of the
// CTA's group, the latent output o = softmax(z) . c_b and lse = log sum exp(z)
// with z = (q_abs . c_b[t] + q_rope . k_rope[t]) * scale (one softmax per
// branch: "Multi-Head Low-Rank Attention", Methodology, second paragraph).
// Everything is fp32 FFMA, so this path meets a 1e-5 relative bound; it is the
// path of fp32 caches and handles every shape the tensor-core kernel does not.
//
// CTA work: group g = (head group of 16, branch b); the CTA walks its share of
// the tile stream, in sub-tiles of 32 tokens staged in shared memory as fp32.
// 128 threads: head slot i = tid / 8, sub = tid % 8.
#include "dispatch.h"

#include <math.h>

namespace mlra {
namespace {

constexpr int kSub = 32;      // tokens per shared-memory sub-tile
constexpr int kHeadSlots = 16;
constexpr int kThreads = 128;

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// Four consecutive cache elements as fp32 (16-byte load for fp32, 8-byte for
// bf16: every row offset and column used is a multiple of 4 elements).
template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

template <typename T, int DCB, int DR>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(DecodeArgs a) {
  constexpr int DK = DCB + DR;       // per-branch key width in the latent space
  constexpr int RS = DK + 1;         // padded shared-memory row (odd: conflict-free)
  constexpr int FPT = DCB / 8;       // latent features per thread
  extern __shared__ float smem[];
  float* sq = smem;                         // [16][RS]  q_abs | q_rope of the head slots
  float* sc = sq + kHeadSlots * RS;         // [32][RS]  c_b | k_rope of the sub-tile
  float* sp = sc + kSub * RS;               // [16][32]  probabilities

  pdl_wait();
  pdl_trigger();
  const mlra_config_t& cfg = a.cfg;
  const int nb = cfg.n_blocks, H = cfg.n_heads, D = nb * DCB + DR;
  const int g = blockIdx.x / a.ctas_per_group;
  const int c = blockIdx.x % a.ctas_per_group;
  const int b = g % nb, hg = g / nb;
  const int tid = threadIdx.x, slot = tid / 8, sub = tid % 8;
  const int head = hg * kHeadSlots + slot;
  const bool head_ok = head < H;

  const char* ws = static_cast<const char*>(a.ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  const int32_t* tile_off = reinterpret_cast<const int32_t*>(ws + a.L.tile_off);
  const int32_t* slot_off = reinterpret_cast<const int32_t*>(ws + a.L.slot_off);
  float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
  const int total = hdr->total_tiles, share = hdr->share;
  const T* cache = static_cast<const T*>(a.kv_cache);
  const T* q_rope = static_cast<const T*>(a.q_rope);
  const float sl2 = cfg.softmax_scale * 1.4426950408889634f;  // scale * log2(e)

  int t_begin = c * share, t_end = min(total, t_begin + share);
  int cur_seq = -1;
  while (t_begin < t_end) {
    const int s = find_seq(tile_off, a.batch, t_begin);
    const int s_t0 = __ldg(tile_off + s), s_t1 = __ldg(tile_off + s + 1);
    const int piece_end = min(t_end, s_t1);
    const int split = t_begin / share - s_t0 / share;
    const int L = min(max(__ldg(a.seqlens + s), 0), a.cap);
    const int tok0 = (t_begin - s_t0) * kTile;
    const int tok1 = min(L, (piece_end - s_t0) * kTile);

    // queries of this sequence, head group and branch
    if (s != cur_seq) {
      __syncthreads();
      for (int x = tid; x < kHeadSlots * DK; x += kThreads) {
        int i = x / DK, k = x % DK, hh = hg * kHeadSlots + i;
        float v = 0.f;
        if (hh < H) {
          if (k < DCB) v = __ldg(a.q_abs + ((size_t(s) * H + hh) * nb + b) * DCB + k);
          else v = to_f32(q_rope[(size_t(s) * H + hh) * DR + (k - DCB)]);
        }
        sq[i * RS + k] = v;
      }
      cur_seq = s;
    }

    float m = -INFINITY, l = 0.f;
    float acc[FPT];
#pragma unroll
    for (int k = 0; k < FPT; ++k) acc[k] = 0.f;

    for (int t0 = tok0; t0 < tok1; t0 += kSub) {
      const int nt = min(kSub, tok1 - t0);
      __syncthreads();
      // stage c_b | k_rope of tokens [t0, t0 + nt) (zeros past the end), four
      // elements per load, the loads of a thread independent of one another
      constexpr int DK4 = DK / 4;
#pragma unroll 2
      for (int x = tid; x < kSub * DK4; x += kThreads) {
        const int tt = x / DK4, k = (x - tt * DK4) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (tt < nt) {
          const int t = t0 + tt;
          long long row;
          bool ok = true;
          if (a.page_table) {
            const int pg = __ldg(a.page_table + size_t(s) * a.max_pages + t / kPageSize);
            if (pg < 0 || pg >= a.num_pages) { ok = false; set_error(&hdr->error, MLRA_ERR_BAD_PAGE); }
            row = (long long)pg * kPageSize + (t % kPageSize);
          } else {
            row = (long long)s * a.max_pages + t;
          }
          if (ok) {
            const int col = (k < DCB) ? (b * DCB + k) : (nb * DCB + (k - DCB));
            v = load4<T>(cache + row * D + col);
          }
        }
        float* dst = sc + tt * RS + k;
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
      }
      __syncthreads();
      // logits of 4 tokens per thread
      float z[4];
      float mt = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int tt = sub + 8 * q;
        float d = 0.f;
        const float* qr = sq + slot * RS;
        const float* cr = sc + tt * RS;
#pragma unroll 8
        for (int k = 0; k < DK; ++k) d = fmaf(qr[k], cr[k], d);
        z[q] = (tt < nt) ? d * sl2 : -INFINITY;
        mt = fmaxf(mt, z[q]);
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
      const float m_new = fmaxf(m, mt);
      const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - m_new);
      float ls = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float p = (z[q] == -INFINITY) ? 0.f : exp2f(z[q] - m_new);
        sp[slot * kSub + sub + 8 * q] = p;
        ls += p;
      }
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      l = l * alpha + ls;
      m = m_new;
      __syncwarp();
      // O = alpha * O + P . c_b
#pragma unroll
      for (int k = 0; k < FPT; ++k) acc[k] *= alpha;
      for (int tt = 0; tt < nt; ++tt) {
        const float p = sp[slot * kSub + tt];
        const float* cr = sc + tt * RS;
#pragma unroll
        for (int k = 0; k < FPT; ++k) acc[k] = fmaf(p, cr[sub + 8 * k], acc[k]);
      }
    }

    // write the split partial
    const int slot_idx = __ldg(slot_off + s) + split;
    if (head_ok && tok1 > tok0) {
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      float* dst = o_part + ((size_t(slot_idx) * H + head) * nb + b) * DCB;
#pragma unroll
      for (int k = 0; k < FPT; ++k) dst[sub + 8 * k] = acc[k] * inv;
      if (sub == 0)
        lse_part[(size_t(slot_idx) * H + head) * nb + b] =
            (l > 0.f) ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
    t_begin = piece_end;
  }
}

template <typename T, int DCB, int DR>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  constexpr int RS = DCB + DR + 1;
  const size_t smem = sizeof(float) * (size_t(kHeadSlots) * RS + size_t(kSub) * RS + kHeadSlots * kSub);
  auto kern = decode_simt_kernel<T, DCB, DR>;
  static bool attr_set[64] = {false};  // once per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int grid = a.n_groups * a.ctas_per_group;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, a);
}

}  // namespace

bool simt_supported(const mlra_config_t& c) {
  const bool shape = (c.d_cb == 64 && c.d_r == 32) || (c.d_cb == 128 && c.d_r == 64) ||
                     (c.d_cb == 512 && c.d_r == 64);
  return shape && c.n_heads >= 1 && c.n_blocks >= 1;
}

void simt_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group) {
  const int hgroups = (c.n_heads + kHeadSlots - 1) / kHeadSlots;
  *n_groups = hgroups * c.n_blocks;
  // about 4 resident CTAs per SM over all groups
  *ctas_per_group = (num_sms * 4 + *n_groups - 1) / *n_groups;
}

cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st) {
  const mlra_config_t& c = a.cfg;
  const bool bf = c.dtype == MLRA_BF16;
  if (c.d_cb == 64 && c.d_r == 32)
    return bf ? launch_t<__nv_bfloat16, 64, 32>(a, st) : launch_t<float, 64, 32>(a, st);
  if (c.d_cb == 128 && c.d_r == 64)
    return bf ? launch_t<__nv_bfloat16, 128, 64>(a, st) : launch_t<float, 128, 64>(a, st);
  if (c.d_cb == 512 && c.d_r == 64)
    return bf ? launch_t<__nv_bfloat16, 512, 64>(a, st) : launch_t<float, 512, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace mlra
