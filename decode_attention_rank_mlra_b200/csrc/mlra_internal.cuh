// Internal declarations shared by the kernels and the host API of libmlra.
// Nothing here is part of the C ABI (include/mlra.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/mlra.h"

namespace mlra {

// Tokens per tile of the KV stream: the unit of planning and of one TMA stage.
constexpr int kTile = 64;
constexpr int kPageSize = 64;

// ---------------------------------------------------------------------------
// Workspace layout (all segments 256-byte aligned, in this order):
//   Header                       256 B
//   tile_off  [batch + 1] int32   first tile of each sequence in the tile stream
//   slot_off  [batch + 1] int32   first split slot of each sequence
//   o_part    [max_slots, h, nb, d_cb] fp32   normalised latent output of a split
//   lse_part  [max_slots, h, nb]       fp32   natural-log sum of exp of a split
// ---------------------------------------------------------------------------
struct WsHeader {
  int32_t error;          // first device-side error code (0 = none)
  int32_t total_tiles;    // tiles in the whole stream
  int32_t share;          // tiles per CTA of one branch group
  int32_t n_slots;        // split slots used
  int32_t ctas_per_group; // persistent CTAs per branch group
  int32_t batch;
  int32_t max_slots;
  int32_t pad[57];
};
static_assert(sizeof(WsHeader) == 256, "header must be 256 bytes");

struct WsLayout {
  size_t tile_off, slot_off, o_part, lse_part, total;
  int32_t max_slots;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int batch, int heads, int nb, int d_cb, int max_slots) {
  WsLayout L;
  size_t off = sizeof(WsHeader);
  L.tile_off = off; off = align256(off + sizeof(int32_t) * (batch + 1));
  L.slot_off = off; off = align256(off + sizeof(int32_t) * (batch + 1));
  L.o_part = off;   off = align256(off + sizeof(float) * size_t(max_slots) * heads * nb * d_cb);
  L.lse_part = off; off = align256(off + sizeof(float) * size_t(max_slots) * heads * nb);
  L.total = off;
  L.max_slots = max_slots;
  return L;
}

// Record the first device-side error (later ones are dropped).
__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
  atomicCAS(err, 0, code);
}

// Split bookkeeping shared by the decode kernels: the tile stream of all
// sequences is cut into `share`-tile pieces, one per CTA of a branch group.
struct Plan {
  const int32_t* tile_off;  // [batch+1]
  const int32_t* slot_off;  // [batch+1]
  const int32_t* seqlens;   // [batch]
  int32_t batch;
  int32_t total_tiles;
  int32_t share;
};

// Sequence containing global tile `t` (tile_off is non-decreasing).
__device__ __forceinline__ int find_seq(const int32_t* tile_off, int batch, int t) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(tile_off + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Dispatch entry points of the individual kernel files (host side).
cudaError_t launch_plan(const int32_t* seqlens, int batch, int cap, int ctas_per_group, void* ws,
                        const WsLayout& L, cudaStream_t st);
cudaError_t launch_absorb(const mlra_config_t& c, const void* q_nope, const void* w_uk,
                          float* q_abs, int batch, cudaStream_t st);
cudaError_t launch_combine(const mlra_config_t& c, const void* ws, const WsLayout& L, int batch,
                           float* o_latent, float* lse, cudaStream_t st);
cudaError_t launch_out_proj(const mlra_config_t& c, const float* o_latent, const void* w_uv,
                            float* out, int batch, cudaStream_t st);

struct DecodeArgs {
  mlra_config_t cfg;
  const float* q_abs;
  const void* q_rope;
  const void* kv_cache;
  int64_t num_pages;
  const int32_t* page_table;
  int32_t max_pages;        // paged: table stride; contiguous: max_len
  int32_t cap;              // largest valid sequence length (tokens)
  const int32_t* seqlens;
  int32_t batch;
  void* ws;
  WsLayout L;
  int32_t ctas_per_group;
  int32_t n_groups;
};

// fp32 SIMT decode (any supported shape / dtype).
bool simt_supported(const mlra_config_t& c);
void simt_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group);
cudaError_t launch_decode_simt(const DecodeArgs& a, cudaStream_t st);

// Tensor-core decode (tcgen05 / TMEM / TMA), bf16 cache.
bool tc_supported(const mlra_config_t& c);
void tc_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group);
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st);

}  // namespace mlra
