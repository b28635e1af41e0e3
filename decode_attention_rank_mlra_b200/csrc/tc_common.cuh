// Helpers shared by the tensor-core attention kernels (k_decode_tc.cu and
// k_decode_tc_mla.cu): bounded mbarrier waits, bf16 packing, and the tensor
// map through which TMA reads the latent cache.
#pragma once

#include "mlra_internal.cuh"
#include "sm100_ptx.cuh"

#include <cudaTypedefs.h>
#include <cuda_fp16.h>

namespace mlra {
namespace tc {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kBoxCols = 64;             // bf16 columns per TMA box (128 B)
constexpr int kBoxBytes = kTile * 128;   // 64 rows x 128 B
constexpr int kSmemLimit = 232448;       // max dynamic shared memory per block

// Bounded mbarrier wait: false on timeout (error recorded) or when another role aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* err) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (ptx::globaltimer() - t0 > kTimeoutNs) {
      set_error(err, MLRA_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// The same wait for a warp whose lanes go on to .sync.aligned instructions
// (TMEM loads and stores): every lane tests the barrier (one instruction for
// the warp) and gets the same answer, so on a timeout the whole warp leaves
// together instead of a part of it issuing them.  (Measured: a single lane
// that waits and then hands its answer to the others made the kernels
// 15-25 % slower.)
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity,
                                              volatile int* abort_flag, int32_t* err) {
  const bool good = wait_bar(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, good);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// Eight bf16 values (one 16-byte chunk) -> fp16 in place, round to nearest:
// exact for 2^-17 <= |c| < 65520 (bf16's 8 significant bits fit fp16's), a
// smaller magnitude lands on fp16's subnormal grid of 2^-24.  Returns bits 15 /
// 31 set when a value became inf or NaN, i.e. left the fp16 range.
__device__ __forceinline__ uint32_t bf16x8_to_f16(uint4& w) {
  uint32_t over = 0;
  uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __half2 h = __floats2half2_rn(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xffff0000u));
    const uint32_t h2 = *reinterpret_cast<uint32_t*>(&h);
    over |= (h2 & 0x7fff7fffu) + 0x04000400u;  // inf / NaN carries into bit 15
    wv[e] = h2;
  }
  return over;
}

// Converter step over one stage: the chunks q = ct, ct + kConvThreads, ... <
// kChunks of the latent boxes at shared address `base` (64 rows of 128 bytes
// per box, chunk q in row (q / 8) mod 64), bf16 -> fp16 in place; rows at or
// past `valid` become zeros.  Two chunks in flight per thread.
template <int kChunks, int kConvThreads>
__device__ __forceinline__ uint32_t convert_stage(uint32_t base, int ct, int valid) {
  uint32_t over = 0;
  if (valid >= 64) {
    if constexpr (kChunks % (2 * kConvThreads) == 0) {
#pragma unroll
      for (int i = 0; i < kChunks / kConvThreads; i += 2) {
        const uint32_t a0 = base + 16u * uint32_t(ct + kConvThreads * i);
        const uint32_t a1 = a0 + 16u * kConvThreads;
        uint4 w0 = ptx::lds128(a0), w1 = ptx::lds128(a1);
        over |= bf16x8_to_f16(w0);
        over |= bf16x8_to_f16(w1);
        ptx::sts128(a0, w0);
        ptx::sts128(a1, w1);
      }
    } else {  // a share that does not split into pairs: the last pair may be one chunk
#pragma unroll
      for (int q = ct; q < kChunks; q += 2 * kConvThreads) {
        const uint32_t a0 = base + 16u * uint32_t(q);
        const bool two = q + kConvThreads < kChunks;
        uint4 w0 = ptx::lds128(a0), w1 = make_uint4(0u, 0u, 0u, 0u);
        if (two) w1 = ptx::lds128(a0 + 16u * kConvThreads);
        over |= bf16x8_to_f16(w0);
        if (two) over |= bf16x8_to_f16(w1);
        ptx::sts128(a0, w0);
        if (two) ptx::sts128(a0 + 16u * kConvThreads, w1);
      }
    }
  } else {
#pragma unroll 1
    for (int q = ct; q < kChunks; q += kConvThreads) {
      const uint32_t a0 = base + 16u * uint32_t(q);
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (((q >> 3) & 63) < valid) {
        w = ptx::lds128(a0);
        over |= bf16x8_to_f16(w);
      }
      ptx::sts128(a0, w);
    }
  }
  return over;
}

// Zero the rows at or past `valid` of the 64 x 128-byte box at `base`.
template <int kConvThreads>
__device__ __forceinline__ void zero_box_rows(uint32_t base, int ct, int valid) {
#pragma unroll 1
  for (int q = ct; q < 512; q += kConvThreads)
    if (((q >> 3) & 63) >= valid) ptx::sts128(base + 16u * uint32_t(q), make_uint4(0u, 0u, 0u, 0u));
}

// The cache as a 2-D bf16 tensor [rows, D] (rows = pages * 64, or batch *
// max_len when contiguous), read in 64 x 64 boxes with the 128-byte swizzle.
inline cudaError_t make_cache_map(const DecodeArgs& a, CUtensorMap* map) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  if (!enc) return cudaErrorNotSupported;
  const mlra_config_t& c = a.cfg;
  const int D = c.n_blocks * c.d_cb + c.d_r;
  const uint64_t rows = a.page_table ? uint64_t(a.num_pages) * kPageSize
                                     : uint64_t(a.batch) * uint64_t(a.max_pages);
  if (rows >= (uint64_t(1) << 31)) return cudaErrorInvalidValue;
  cuuint64_t dims[2] = {cuuint64_t(D), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(D) * 2};
  cuuint32_t box[2] = {kBoxCols, kTile};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.kv_cache), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// MLA (one latent block of 512, k_decode_tc_mla.cu): CTAs of 64 heads x one
// 256-feature half of the latent output.
inline bool mla_supported(const mlra_config_t& c) {
  return c.n_blocks == 1 && c.d_cb == 512 && c.d_r == 64 && c.n_heads % 64 == 0;
}
inline int mla_groups(const mlra_config_t& c) { return (c.n_heads / 64) * 2; }
cudaError_t launch_decode_tc_mla(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st);

// MLA with a multiple of 128 heads (k_decode_mla_pair.cu): clusters of two
// CTAs, each holding half of the latent channels; ctas_per_group counts
// clusters.
bool mla_pair_supported(const mlra_config_t& c);
int mla_pair_clusters(const mlra_config_t& c, int num_sms);
cudaError_t launch_decode_mla_pair(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st);

// Latent blocks of 128 channels, 128 heads x one branch per CTA
// (k_decode_wide.cu): head counts that are multiples of 128.
bool wide_supported(const mlra_config_t& c);
int wide_groups(const mlra_config_t& c);
cudaError_t launch_decode_wide(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st);

}  // namespace tc
}  // namespace mlra
