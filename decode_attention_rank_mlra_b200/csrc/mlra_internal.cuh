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
  // A launch that recomputes the call on the head-rows (or 64-head MLA) kernel
  // after a 128-head kernel reported MLRA_ERR_RANGE records its own errors
  // here, and its CTAs count themselves out here.
  int32_t fallback_error;
  int32_t fallback_done;
  int32_t pad[55];
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
  L.tile_off = off;  off = align256(off + sizeof(int32_t) * (batch + 1));
  L.slot_off = off;  off = align256(off + sizeof(int32_t) * (batch + 1));
  L.o_part = off;    off = align256(off + sizeof(float) * size_t(max_slots) * heads * nb * d_cb);
  L.lse_part = off;  off = align256(off + sizeof(float) * size_t(max_slots) * heads * nb);
  L.total = off;
  L.max_slots = max_slots;
  return L;
}

// Record the first device-side error (later ones are dropped).
__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
  atomicCAS(err, 0, code);
}

// Split bookkeeping of the decode kernels: the tile stream of all sequences
// is cut into `share`-tile pieces, one per CTA of a branch group.
// Sequence containing global tile `t` (tile_off is non-decreasing).
__device__ __forceinline__ int find_seq(const int32_t* tile_off, int batch, int t) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(tile_off + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One piece of a CTA's share: tiles [t0, t1) of sequence s (tile indices
// within the sequence), written to split slot `slot`; L = the sequence length.
struct Piece {
  int s, t0, t1, slot, L;
};

// Programmatic dependent launch: every kernel of the library is launched so
// that the next kernel on the stream may start its prologue early; each one
// waits for its predecessor's completion (and memory) before it reads what the
// predecessor writes, and lets its dependents launch right after.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Exclusive prefix sum of one int per thread over a block of NT threads;
// `scratch` holds NT / 32 + 1 ints of shared memory.  *total = block sum.
template <int NT>
__device__ int block_exclusive_scan(int v, int* scratch, int* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += n;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int w = 0; w < NW; ++w) {
      const int t = scratch[w];
      scratch[w] = run;
      run += t;
    }
    scratch[NW] = run;
  }
  __syncthreads();
  const int r = x - v + scratch[warp];
  *total = scratch[NW];
  __syncthreads();
  return r;
}

// The split plan of persistent CTA c, computed by its whole block from the
// sequence lengths with the same arithmetic as the plan kernel, so that the CTA
// can start streaming without waiting for that kernel.  Writes to shared
// memory: out[0] = tiles in the stream, out[1] = tiles per CTA (share), then
// the CTA's first two pieces as {s, s0, s1, slot, L} at out[2] and out[7]
// (s = -1: the share has no such piece).
template <int NT>
__device__ void plan_first_pieces(const int32_t* __restrict__ seqlens, int batch, int cap, int cpg,
                                  int c, int* out, int* scratch) {
  const int per = (batch + NT - 1) / NT;
  const int b0 = min(batch, int(threadIdx.x) * per), b1 = min(batch, b0 + per);
  auto len_of = [&](int s) { return min(max(__ldg(seqlens + s), 0), cap); };
  int loc = 0;
  for (int s = b0; s < b1; ++s) loc += (len_of(s) + kTile - 1) / kTile;
  int total;
  const int a0 = block_exclusive_scan<NT>(loc, scratch, &total);
  const int share = max(1, (total + cpg - 1) / cpg);
  int sloc = 0;
  for (int s = b0, a = a0; s < b1; ++s) {
    const int e = a + (len_of(s) + kTile - 1) / kTile;
    sloc += (e > a) ? (e - 1) / share - a / share + 1 : 0;
    a = e;
  }
  int stot;
  const int q0 = block_exclusive_scan<NT>(sloc, scratch, &stot);
  const int g0 = c * share, gend = min(total, g0 + share);
  if (threadIdx.x == 0) {
    out[0] = total;
    out[1] = share;
    out[2] = -1;
    out[7] = -1;
  }
  __syncthreads();
  for (int pass = 0; pass < 2; ++pass) {
    // pass 0: the sequence holding tile g0; pass 1: the next non-empty one,
    // which starts where the first piece's sequence ends
    const int want = pass == 0 ? g0 : (out[2] >= 0 ? out[4] : gend);
    if (want < gend) {
      for (int s = b0, a = a0, q = q0; s < b1; ++s) {
        const int L = len_of(s);
        const int e = a + (L + kTile - 1) / kTile;
        if (e > a && a <= want && want < e) {
          int* r = out + 2 + 5 * pass;
          r[0] = s;
          r[1] = a;
          r[2] = e;
          r[3] = q + want / share - a / share;
          r[4] = L;
        }
        q += (e > a) ? (e - 1) / share - a / share + 1 : 0;
        a = e;
      }
    }
    __syncthreads();
  }
}

// Walks the pieces of one persistent CTA's share [gt, end) of the tile stream.
// The first two pieces come from the CTA's own plan (plan_first_pieces); later
// ones from the plan kernel's records, after waiting for that kernel, each
// starting a new sequence whose bounds are loaded one piece ahead.
struct Walker {
  const int32_t* tile_off;
  const int32_t* slot_off;
  const int32_t* seqlens;
  const int* pre;  // shared memory: two {s, s0, s1, slot, L} records
  int batch, cap, gt, end;
  int used = 0;
  int cur = -1, cur_s1 = 0;
  bool ahead = false;
  int n_s1 = 0, n_slot = 0, n_L = 0;  // sequence cur + 1, loaded ahead

  __device__ void load_ahead() {
    const int s = cur + 1;
    ahead = s < batch;
    if (ahead) {
      n_s1 = __ldg(tile_off + s + 1);
      n_slot = __ldg(slot_off + s);
      n_L = __ldg(seqlens + s);
    }
  }
  __device__ bool next(Piece& p) {
    if (gt >= end) return false;
    int s, s0, s1, slot, L;
    const bool own = used < 2;
    if (own) {
      const int* r = pre + 5 * used;
      ++used;
      s = r[0]; s0 = r[1]; s1 = r[2]; slot = r[3]; L = r[4];
    } else {
      if (!ahead) {
        pdl_wait();  // the plan kernel's records
        load_ahead();
      }
      s = cur + 1;
      s0 = cur_s1;  // == gt: a later piece opens its sequence (split 0)
      if (n_s1 > gt) {
        s1 = n_s1; slot = n_slot; L = n_L;
      } else {  // empty sequences in between
        while (__ldg(tile_off + s + 1) <= gt) ++s;
        s0 = __ldg(tile_off + s);
        s1 = __ldg(tile_off + s + 1);
        slot = __ldg(slot_off + s);
        L = __ldg(seqlens + s);
      }
    }
    const int pe = min(end, s1);
    p.s = s;
    p.t0 = gt - s0;
    p.t1 = pe - s0;
    p.slot = slot;
    p.L = min(max(L, 0), cap);
    gt = pe;
    cur = s;
    cur_s1 = s1;
    if (!own && gt < end) load_ahead();  // (the plan kernel is complete here)
    else ahead = false;
    return true;
  }
};

template <typename... K, typename... A>
cudaError_t launch_pdl(void (*kern)(K...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<A&&>(args)...);
}

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
  // Test of the failure path: the TMA producer of CTA 0 leaves the full
  // barrier of this tile (its count in that CTA's stream) unsignalled, so the
  // MMA warp's bounded wait runs out (MLRA_ERR_TIMEOUT).  -1: none.  Set only
  // from MLRA_TEST_STALL_TILE; honoured by the head-rows kernel.
  int32_t stall_tile = -1;
  // 1: this launch runs only if the 128-head kernel launched just before it
  // left MLRA_ERR_RANGE in the error word, and then recomputes every output of
  // the call (same plan, same slots); otherwise each CTA returns at once.
  int32_t range_fallback = 0;
};

}  // namespace mlra
