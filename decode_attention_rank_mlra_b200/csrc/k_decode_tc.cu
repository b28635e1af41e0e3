// Tensor-core split-KV decode attention over the bf16 latent cache (sm_100a).
//
// What it computes is the same as the SIMT kernel: for one split of one
// sequence and every (head, branch) of the CTA's branch group,
//   z_t = (q_abs . c_b[t] + q_rope . k_rope[t]) * scale,
//   o = softmax(z) . c_b,  lse = log sum exp z
// with one softmax per latent branch ("Multi-Head Low-Rank Attention",
// Methodology, second paragraph) over the shared latent cache, the absorbed
// "MQA-style" step of Main Findings ("three absorbable steps").
//
// How (one CTA per SM, persistent over a share of the tile stream):
//  * warp 4 streams 64-token tiles of the cache with TMA (SWIZZLE_128B boxes of
//    64 rows x 64 columns): the two boxes of each latent block c_b of the
//    group and the RoPE box, into a multi-stage shared-memory ring;
//  * warp 5 issues tcgen05.mma: S = Q . C^T (A = queries in TMEM, B = cache tile
//    K-major) and O += P . C (A = probabilities in TMEM, B = the same tile,
//    MN-major).  The 128 MMA rows are (branch, head, hi|lo): every head of the
//    group is an M row, and per-branch MMAs write only their own rows through
//    the disable-output-lane mask, so one tile in shared memory feeds every
//    branch;
//  * warps 0-3 (one per TMEM lane quadrant) run the online softmax of their
//    rows and write P back into TMEM.
// Precision: queries and probabilities are carried as bf16 hi + lo pairs (two
// MMA rows per head), so both enter the fp32-accumulated products with about
// 16 significant bits while the cache stays the bf16 it is stored as.
#include "dispatch.h"
#include "tc_common.cuh"

#include <math.h>
#include <stdlib.h>
#include <string.h>

namespace mlra {
namespace {

using namespace ptx;
using tc::kBoxBytes;
using tc::kBoxCols;
using tc::kSmemLimit;
using tc::pack_bf16;
using tc::wait_bar;
using tc::wait_bar_warp;

constexpr int kThreadsTC = 192;              // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kPrefetchAhead = 6;            // tiles before a piece's end
constexpr int kPrefetchTiles = 4;            // first tiles of the next sequence
constexpr uint32_t kTmemCols = 512;
// Queries are double-buffered by piece: buffer b at b * kQBuf holds the q_abs
// rows (bf16 pairs, 64 columns) and then the q_rope rows (32 columns).
constexpr uint32_t kQBuf = 96;
constexpr uint32_t kColQr = 64;              // q_rope offset inside a query buffer
constexpr uint32_t kColS = 2 * kQBuf;        // S / P double buffer: 2 x 64 columns
constexpr uint32_t kColO = kColS + 128;      // O accumulator: 128 columns

template <int G>
struct TcShape {
  static constexpr int kBoxes = 2 * G + 1;
  static constexpr int kStage = kBoxes * kBoxBytes;
  static constexpr int kStagesRaw = (kSmemLimit - 2048) / kStage;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kBars = 2 * kStages + 9;
  static constexpr int kSmem = 1024 + kStages * kStage + kBars * 8 + 64;
  static_assert(kStages >= 3, "too few pipeline stages");
};

// G branches x HPC heads per CTA (rows = G * HPC * 2 <= 128).  The grid is
// (branch groups x head groups) x CTAs per group; one CTA per SM.
template <int G, int HPC>
__global__ void __launch_bounds__(kThreadsTC, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  using S = TcShape<G>;
  constexpr int NST = S::kStages;
  constexpr int STAGE = S::kStage;
  constexpr int WPB = HPC / 16;  // TMEM lane quadrants per branch
  static_assert(G * WPB <= 4, "rows exceed 128");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NST * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_addr(bars);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (NST + i); };
  auto SFULL = [&](int i) { return bar0 + 8u * (2 * NST + i); };
  auto PREADY = [&](int i) { return bar0 + 8u * (2 * NST + 2 + i); };
  // PV of tile k commits to PVDONE(k & 1): a waiter for PV(k) has always seen
  // S(k) or later, which implies PV(k-2) is complete, so parity waits are exact.
  auto PVDONE = [&](int i) { return bar0 + 8u * (2 * NST + 4 + i); };
  auto QREADY = [&](int i) { return bar0 + 8u * (2 * NST + 6 + i); };
  const uint32_t DRAIN = bar0 + 8u * (2 * NST + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  if (a.range_fallback) {
    // after the 128-head kernel's grid: every thread reads its final error word
    pdl_wait();
    if (*reinterpret_cast<volatile int32_t*>(&hdr->error) != MLRA_ERR_RANGE) return;
  }
  int32_t* err = a.range_fallback ? &hdr->fallback_error : &hdr->error;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(SFULL(i), 1);
      mbar_init(PREADY(i), 4);
      mbar_init(PVDONE(i), 1);
    }
    mbar_init(QREADY(0), 4);
    mbar_init(QREADY(1), 4);
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // No wait for the plan kernel launched just before: this kernel starts only
  // after that kernel passed its own griddepcontrol.wait (so the queries, the
  // lengths, the page table and the cache are final) and reset the error word;
  // the CTA plans its first two pieces itself.
  pdl_trigger();

  const char* wsc = static_cast<const char*>(a.ws);
  const int nb = a.cfg.n_blocks, H = a.cfg.n_heads;
  const int grp = blockIdx.x / a.ctas_per_group;
  const int c = blockIdx.x % a.ctas_per_group;
  const int g = grp % (nb / G);            // branch group
  const int head0 = (grp / (nb / G)) * HPC;  // first head of this CTA's head group
  __shared__ int plan_sm[12], scan_sm[kThreadsTC / 32 + 1];
  plan_first_pieces<kThreadsTC>(a.seqlens, a.batch, a.cap, a.ctas_per_group, c, plan_sm, scan_sm);
  const int total = plan_sm[0], share = plan_sm[1];
  Walker walk{reinterpret_cast<const int32_t*>(wsc + a.L.tile_off),
              reinterpret_cast<const int32_t*>(wsc + a.L.slot_off),
              a.seqlens, plan_sm + 2,
              a.batch, a.cap, c * share, min(total, (c + 1) * share)};

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      const uint64_t evict_first = policy_evict_first();  // the cache is streamed once
      // The first tiles of a new sequence arrive slowly (cold pages): a few
      // tiles before a piece that another piece follows ends, the first tiles
      // of the next sequence are prefetched into L2.
      const size_t row_bytes = size_t(a.cfg.n_blocks * a.cfg.d_cb + a.cfg.d_r) * 2;
      auto prefetch_head = [&](int s2) {
        if (s2 >= a.batch) return;
        const int L2 = min(max(__ldg(a.seqlens + s2), 0), a.cap);
        const int nt = min((L2 + kTile - 1) / kTile, kPrefetchTiles);
        for (int j = 0; j < nt; ++j) {
          int64_t row;
          int rows = kTile;
          if (a.page_table) {
            const int pg = __ldg(a.page_table + size_t(s2) * a.max_pages + j);
            if (pg < 0 || pg >= a.num_pages) continue;
            row = int64_t(pg) * kPageSize;
          } else {
            row = int64_t(s2) * a.max_pages + int64_t(j) * kTile;
            rows = min(kTile, a.max_pages - j * kTile);  // the allocation ends with the last row
          }
          bulk_prefetch_l2(static_cast<const char*>(a.kv_cache) + row * row_bytes,
                           uint32_t(rows * row_bytes));
        }
      };
      Piece p;
      int it = 0;
      bool ok = true;
      while (ok && walk.next(p)) {
        const bool more = walk.gt < walk.end;  // another piece follows in this share
        const int t_pf = max(p.t0, p.t1 - kPrefetchAhead);
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          const int st = it % NST;
          if (more && t == t_pf) prefetch_head(p.s + 1);
          if (!wait_bar(EMPTY(st), ((it / NST) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
          int row;
          if (a.page_table) {
            const int pg = __ldg(a.page_table + size_t(p.s) * a.max_pages + t);
            if (pg < 0 || pg >= a.num_pages) {
              set_error(err, MLRA_ERR_BAD_PAGE);
              row = -2 * kTile;  // out of bounds: the box is zero-filled
            } else {
              row = pg * kPageSize;
            }
          } else {
            row = p.s * a.max_pages + t * kTile;
          }
          if (it == a.stall_tile && blockIdx.x == 0) continue;  // failure-path test only
          mbar_arrive_expect_tx(FULL(st), STAGE);
          const uint32_t dst = smem_addr(stages + st * STAGE);
#pragma unroll
          for (int bx = 0; bx < G; ++bx) {
            const int br = g * G + bx;
            tma_load_2d_hint(dst + (2 * bx) * kBoxBytes, &tmap, br * 128, row, FULL(st), evict_first);
            tma_load_2d_hint(dst + (2 * bx + 1) * kBoxBytes, &tmap, br * 128 + kBoxCols, row,
                             FULL(st), evict_first);
          }
          tma_load_2d_hint(dst + 2 * G * kBoxBytes, &tmap, nb * 128, row, FULL(st), evict_first);
        }
      }
      if (!ok) {
        // let loads already in flight land before the CTA can exit
        for (int j = 0; j < NST; ++j) {
          const int k = it - 1 - j;
          if (k < 0) break;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(FULL(k % NST), (k / NST) & 1) && globaltimer() - t0 < 10000000ull) {}
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop; each MMA / commit is issued by one elected
    // lane with warp-uniform operands (compile-time offsets from per-stage
    // descriptors), which keeps the issue rate at the tensor core's pace.  The
    // lanes stay converged (the only divergent loop ends in __syncwarp), so
    // they poll each barrier together and leave a wait together.
    //  QK : S[rows, tokens] = Q[rows, K] . C[tokens, K]^T  (A: TMEM, B: smem K-major)
    //  PV : O[rows, features] += P[rows, tokens] . C_b[tokens, features]
    //       (A: probabilities in TMEM over the S buffer, B: the same tile, MN-major)
    // Rows of other branches are kept out of each branch's MMAs by the
    // disable-output-lane mask.
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);
    const uint32_t sbase0 = smem_addr(stages);
    const uint64_t dK = smem_desc(sbase0, 16, 1024, kSwizzle128B);
    const uint64_t dMN = smem_desc(sbase0, kBoxBytes, 1024, kSwizzle128B);
    Piece p;
    int it = 0, piece = 0;
    int prev = -1;            // tile whose PV is still to be issued
    bool prev_first = false;  // ...and whether it opens its piece
    bool ok = true;
    auto issue_pv = [&](int pit, bool first) {
      const uint64_t d = dMN + uint64_t(((pit % NST) * STAGE) >> 4);
      const uint32_t a_p = tmem + kColS + 64 * (pit & 1);
#pragma unroll
      for (int bx = 0; bx < G; ++bx) {
        if (g * G + bx >= nb) continue;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)
          mma_ts_warp(tmem + kColO, a_p + 8 * k,
                      d + uint64_t((2 * bx * kBoxBytes + k * 16 * 128) >> 4), kIdescPV,
                      (first && k == 0) ? 0u : 1u, (0 / WPB == bx) ? 0u : ~0u,
                      (1 / WPB == bx) ? 0u : ~0u, (2 / WPB == bx) ? 0u : ~0u,
                      (3 / WPB == bx) ? 0u : ~0u);
      }
      mma_commit_warp(EMPTY(pit % NST));
      mma_commit_warp(PVDONE(pit & 1));
    };
    while (ok && walk.next(p)) {
      if (!wait_bar_warp(QREADY(piece & 1), (piece >> 1) & 1, abort_flag, err)) { ok = false; break; }
      const uint32_t qbuf = tmem + uint32_t(piece & 1) * kQBuf;
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % NST, sb = it & 1;
        if (!wait_bar_warp(FULL(st), (it / NST) & 1, abort_flag, err)) { ok = false; break; }
        const int valid = min(kTile, p.L - t * kTile);
        if (valid < kTile) {
          // zero the rows past the sequence end (whatever the cache holds there)
          const int per_box = (kTile - valid) * 8;
          uint8_t* sp = stages + st * STAGE;
          for (int i = lane; i < per_box * S::kBoxes; i += 32) {
            const int bx = i / per_box, rem = i % per_box;
            *reinterpret_cast<uint4*>(sp + bx * kBoxBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        {
          const uint64_t d = dK + uint64_t((st * STAGE) >> 4);
          const uint32_t s_acc = tmem + kColS + 64 * sb;
#pragma unroll
          for (int bx = 0; bx < G; ++bx) {
            if (g * G + bx >= nb) continue;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ts_warp(s_acc, qbuf + 8 * k,
                          d + uint64_t(((2 * bx + (k >> 2)) * kBoxBytes + (k & 3) * 32) >> 4),
                          kIdescQK, k > 0 ? 1u : 0u, (0 / WPB == bx) ? 0u : ~0u,
                          (1 / WPB == bx) ? 0u : ~0u, (2 / WPB == bx) ? 0u : ~0u,
                          (3 / WPB == bx) ? 0u : ~0u);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_warp(s_acc, qbuf + kColQr + 8 * k,
                        d + uint64_t((2 * G * kBoxBytes + k * 32) >> 4), kIdescQK, 1u, 0u, 0u, 0u,
                        0u);
          mma_commit_warp(SFULL(sb));
        }
        if (prev >= 0) {
          if (!wait_bar_warp(PREADY(prev & 1), (prev >> 1) & 1, abort_flag, err)) { ok = false; break; }
          tc_fence_after();
          issue_pv(prev, prev_first);
        }
        prev = it;
        prev_first = (t == p.t0);
      }
      // the piece's last PV goes out before the next piece's first QK: the
      // epilogue waits for it, and must not wait for the next piece's data
      if (ok && prev >= 0) {
        if (!wait_bar_warp(PREADY(prev & 1), (prev >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        issue_pv(prev, prev_first);
        prev = -1;
      }
      ++piece;
    }
    if (ok && prev >= 0) {
      if (wait_bar_warp(PREADY(prev & 1), (prev >> 1) & 1, abort_flag, err)) {
        tc_fence_after();
        issue_pv(prev, prev_first);
      } else {
        ok = false;
      }
    }
    if (!ok) {
      // drain MMAs already issued before TMEM is released
      mma_commit_warp(DRAIN);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(DRAIN, 0) && globaltimer() - t0 < 10000000ull) {}
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    // Thread = one TMEM lane of the quadrant: branch bg, head, and x = lane / 16,
    // which is the row the thread writes the queries of (0: hi, 1: lo) and the
    // half of each tile's 64 tokens it takes the softmax of.
    const int bg = warp / WPB;
    const int branch = g * G + bg;
    const bool active = bg < G && branch < nb;
    const int x = lane >> 4;
    const int head = head0 + 16 * (warp % WPB) + (lane & 15);
    const uint32_t row_t = tmem + (uint32_t(32 * warp) << 16);
    const float sl2 = a.cfg.softmax_scale * 1.4426950408889634f;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
    const unsigned short* q_rope = static_cast<const unsigned short*>(a.q_rope);
    // (q_abs rows are 512 B and q_rope rows 128 B apart; both bases are 16-byte
    // aligned, so whole rows are read with 16-byte loads.)
    auto q_row = [&](const Piece& pc) {
      return reinterpret_cast<const float4*>(a.q_abs + ((size_t(pc.s) * H + head) * nb + branch) * 128);
    };
    auto qr_row = [&](const Piece& pc) {
      return reinterpret_cast<const uint4*>(q_rope + (size_t(pc.s) * H + head) * 64);
    };
    // Lanes 0-15 of the quadrant hold the hi rows and lanes 16-31 the lo rows of
    // the same 16 heads.  The .16x32bx2 TMEM accesses give thread t (< 16) both
    // rows of head t for tokens 0-31 and thread t + 16 both rows for tokens
    // 32-63, so S_hi + S_lo, the P_hi / P_lo write-back and O_hi + O_lo need no
    // shuffles.
    const uint32_t hi_t = row_t;                   // lane base 0 of the quadrant
    const uint32_t lo_t = row_t + (16u << 16);     // lane base 16
    // Queries of a piece into query buffer `buf`: thread t (x = 0) converts the
    // first half of head t's row, thread t + 16 the second half, and the
    // .16x32bx2 stores put the hi parts in the hi row and the lo parts in the
    // lo row (the lo row's RoPE columns are zero).
    auto write_q = [&](const Piece& pc, int buf) {
      const float4* q = q_row(pc) + 16 * x;
      float4 f[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) f[j] = active ? __ldg(q + j) : make_float4(0.f, 0.f, 0.f, 0.f);
      const uint4* qr = qr_row(pc) + 4 * x;
      uint4 u[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) u[j] = active ? __ldg(qr + j) : make_uint4(0u, 0u, 0u, 0u);
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v[4] = {f[j].x, f[j].y, f[j].z, f[j].w};
        float w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
        hi[2 * j] = pack_bf16(v[0], v[1]);
        hi[2 * j + 1] = pack_bf16(v[2], v[3]);
        lo[2 * j] = pack_bf16(w[0], w[1]);
        lo[2 * j + 1] = pack_bf16(w[2], w[3]);
      }
      const uint32_t qb = uint32_t(buf) * kQBuf;
      tmem_st_x2_32<32>(hi_t + qb, hi);
      tmem_st_x2_32<32>(lo_t + qb, lo);
      uint32_t rr[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rr[4 * j] = u[j].x; rr[4 * j + 1] = u[j].y; rr[4 * j + 2] = u[j].z; rr[4 * j + 3] = u[j].w;
      }
      tmem_st_x2_16<16>(hi_t + qb + kColQr, rr);
#pragma unroll
      for (int j = 0; j < 16; ++j) rr[j] = 0u;
      tmem_st_x2_16<16>(lo_t + qb + kColQr, rr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(QREADY(buf));
    };
    // pull the next piece's query rows into L2 while this piece streams
    auto prefetch_q = [&](const Piece& pc) {
      if (!active) return;
      const char* q = reinterpret_cast<const char*>(q_row(pc));
      prefetch_l2_evict_last(q + 256 * x);
      prefetch_l2_evict_last(q + 256 * x + 128);
      if (x == 0) prefetch_l2_evict_last(qr_row(pc));
    };
    Piece p, pn;
    int it = 0, pidx = 0;
    bool ok = walk.next(p);
    bool has_next = ok && walk.next(pn);
    // the first two pieces' queries go in before the cache stream saturates
    // memory; piece k + 1's go in during piece k's first tile (k >= 1)
    if (ok) write_q(p, 0);
    if (has_next) write_q(pn, 1);
    while (ok) {
      // m: the reference point of the exponentials, in log2 units.  It is the
      // first tile's max and moves only when a later tile would overflow
      // (2^64 above it); a stale m only shifts all weights by the same factor.
      float m = -INFINITY, l = 0.f;
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int sb = it & 1;
        if (!wait_bar_warp(SFULL(sb), (it >> 1) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        float raw[32];
        {
          uint32_t sh[32], sl[32];
          tmem_ld_x2_32<32>(hi_t + kColS + 64 * sb, sh);
          tmem_ld_x2_32<32>(lo_t + kColS + 64 * sb, sl);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) raw[k] = __uint_as_float(sh[k]) + __uint_as_float(sl[k]);
        }
        const int valid = min(kTile, p.L - t * kTile);
        if (valid < kTile) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (32 * x + k >= valid) raw[k] = -INFINITY;
        }
        auto tile_max = [&]() {
          float t16[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) t16[k] = fmaxf(raw[k], raw[k + 16]);
#pragma unroll
          for (int k = 0; k < 8; ++k) t16[k] = fmaxf(t16[k], t16[k + 8]);
#pragma unroll
          for (int k = 0; k < 4; ++k) t16[k] = fmaxf(t16[k], t16[k + 4]);
          const float mx = fmaxf(fmaxf(t16[0], t16[2]), fmaxf(t16[1], t16[3]));
          return fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16)) * sl2;
        };
        if (t == p.t0) m = tile_max();
        uint32_t whi[16], wlo[16];
        float ls;
        auto exps = [&]() {
          const float neg_m = -m;
          ls = 0.f;
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float p0 = ex2_approx(fmaf(raw[k], sl2, neg_m));
            const float p1 = ex2_approx(fmaf(raw[k + 1], sl2, neg_m));
            ls += p0 + p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const float2 hf = __bfloat1622float2(h2);
            whi[k / 2] = *reinterpret_cast<const uint32_t*>(&h2);
            wlo[k / 2] = pack_bf16(p0 - hf.x, p1 - hf.y);
          }
        };
        exps();
        if (__any_sync(0xffffffffu, !(ls <= 0x1p64f))) {
          // rare: a score far above m (or a NaN).  Raise m to this tile's max,
          // rescale l and the O rows once the previous PV is done, redo the tile.
          // The TMEM pass is taken by the whole warp (alpha = 1 for rows whose
          // m stays): its loads and stores are warp-wide instructions.
          const float mt = tile_max();
          float alpha = 1.f;
          if (mt > m) {
            alpha = ex2_approx(m - mt);
            m = mt;
            l *= alpha;
          }
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            const int pk = it - 1;
            if (!wait_bar_warp(PVDONE(pk & 1), (pk >> 1) & 1, abort_flag, err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t r[32];
              tmem_ld32(row_t + kColO + 32 * ch, r);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
              tmem_st32(row_t + kColO + 32 * ch, r);
            }
            tmem_wait_st();
          }
          exps();
        }
        l += ls;
        // P over S: the hi row of head t takes P_hi of all 64 tokens, the lo row P_lo
        tmem_st_x2_16<16>(hi_t + kColS + 64 * sb, whi);
        tmem_st_x2_16<16>(lo_t + kColS + 64 * sb, wlo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PREADY(sb));
        // every QK of the previous piece is done: its query buffer takes the next piece's
        if (t == p.t0 && pidx >= 1 && has_next) write_q(pn, (pidx + 1) & 1);
      }
      if (!ok) break;
      // ---- epilogue: o = (O_hi + O_lo) / l, lse
      {
        const int pk = it - 1;
        if (!wait_bar_warp(PVDONE(pk & 1), (pk >> 1) & 1, abort_flag, err)) { ok = false; break; }
      }
      tc_fence_after();
      const float l_tot = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      float* dst = o_part + ((size_t(p.slot) * H + head) * nb + branch) * 128;
#pragma unroll 1
      for (int j = 0; j < 2; ++j) {
        // thread t: features 32j.., thread t + 16: features 64 + 32j..
        uint32_t oh[32], ol[32];
        tmem_ld_x2_32<64>(hi_t + kColO + 32 * j, oh);
        tmem_ld_x2_32<64>(lo_t + kColO + 32 * j, ol);
        tmem_wait_ld();
        if (active) {
          // 32-byte stores: each one fills a whole sector
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            float o8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              o8[e] = (__uint_as_float(oh[8 * k + e]) + __uint_as_float(ol[8 * k + e])) * inv;
            st_global_v8(dst + 64 * x + 32 * j + 8 * k, o8);
          }
        }
      }
      if (active && x == 0)
        lse_part[(size_t(p.slot) * H + head) * nb + branch] =
            l_tot > 0.f ? (m + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
      if (!has_next) break;
      p = pn;
      ++pidx;
      has_next = walk.next(pn);
      if (has_next) prefetch_q(pn);
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_wait();  // complete only after the plan kernel (whose records the merge reads)
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (a.range_fallback && threadIdx.x == 0) {
    // the last CTA out replaces MLRA_ERR_RANGE by this launch's own outcome
    __threadfence();
    if (atomicAdd(&hdr->fallback_done, 1) == int(gridDim.x) - 1)
      atomicCAS(&hdr->error, MLRA_ERR_RANGE,
                *reinterpret_cast<volatile int32_t*>(&hdr->fallback_error));
  }
}

// Heads per CTA (a head group) and branches per CTA: the 128 MMA rows hold
// G branches x HPC heads x (hi, lo).
int hpc_of(const mlra_config_t& c) { return c.n_heads < 64 ? c.n_heads : 64; }
int g_of(const mlra_config_t& c) {
  const int per = 64 / hpc_of(c);
  return c.n_blocks < per ? c.n_blocks : per;
}

template <int G, int HPC>
cudaError_t launch_t(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st) {
  using S = TcShape<G>;
  auto kern = decode_tc_kernel<G, HPC>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  return launch_pdl(kern, dim3(a.n_groups * a.ctas_per_group), dim3(kThreadsTC), S::kSmem, st, map,
                    a);
}

// Head counts that are multiples of 128 go to the 128-head kernel
// (k_decode_wide.cu); MLRA_TC_LAYOUT=rows keeps them on the kernel above
// wherever it applies, for comparison.
bool use_rows_layout() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MLRA_TC_LAYOUT");
    v = (e && strcmp(e, "rows") == 0) ? 1 : 0;
  }
  return v == 1;
}

bool rows_supported(const mlra_config_t& c) {
  if (c.d_cb != 128) return false;
  if (c.n_heads != 16 && c.n_heads != 32 && c.n_heads != 64 && c.n_heads != 128) return false;
  if (c.n_blocks != 1 && c.n_blocks != 2 && c.n_blocks != 4) return false;
  return c.n_blocks % g_of(c) == 0;
}

bool use_wide(const mlra_config_t& c) {
  return tc::wide_supported(c) && !(use_rows_layout() && rows_supported(c));
}

}  // namespace

bool tc_supported(const mlra_config_t& c) {
  if (c.dtype != MLRA_BF16 || c.d_r != 64) return false;
  if (c.d_cb == 512) return tc::mla_supported(c);
  if (use_wide(c)) return true;
  if (c.d_cb != 128) return false;
  if (c.n_heads != 16 && c.n_heads != 32 && c.n_heads != 64 && c.n_heads != 128) return false;
  if (c.n_blocks != 1 && c.n_blocks != 2 && c.n_blocks != 4) return false;
  return c.n_blocks % g_of(c) == 0;
}

void tc_grid(const mlra_config_t& c, int num_sms, int* n_groups, int* ctas_per_group) {
  if (tc::mla_pair_supported(c)) {
    *n_groups = c.n_heads / 128;
    *ctas_per_group = tc::mla_pair_clusters(c, num_sms);
    return;
  }
  *n_groups = c.d_cb == 512 ? tc::mla_groups(c)
              : use_wide(c) ? tc::wide_groups(c)
                            : (c.n_blocks / g_of(c)) * (c.n_heads / hpc_of(c));
  *ctas_per_group = num_sms / *n_groups > 0 ? num_sms / *n_groups : 1;
}

cudaError_t launch_rows(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st) {
  const mlra_config_t& c = a.cfg;
  switch (hpc_of(c) * 10 + g_of(c)) {
    case 164: return launch_t<4, 16>(map, a, st);
    case 162: return launch_t<2, 16>(map, a, st);
    case 161: return launch_t<1, 16>(map, a, st);
    case 322: return launch_t<2, 32>(map, a, st);
    case 321: return launch_t<1, 32>(map, a, st);
    case 641: return launch_t<1, 64>(map, a, st);
  }
  return cudaErrorInvalidValue;
}

// The 128-head kernels carry the tile as fp16 and report a cache value of
// magnitude >= 65520 (MLRA_ERR_RANGE).  Each is followed by a launch of a
// kernel that keeps the tile in bf16 (head-rows for MLRA with 128 heads, the
// 64-head MLA kernel for MLA) on the same plan and slots: its CTAs return at
// once unless the word holds MLRA_ERR_RANGE, and otherwise recompute the call.
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const mlra_config_t& c = a.cfg;
  CUtensorMap map;
  cudaError_t e = tc::make_cache_map(a, &map);
  if (e != cudaSuccess) return e;
  DecodeArgs f = a;
  f.range_fallback = 1;
  f.stall_tile = -1;
  if (tc::mla_pair_supported(c)) {
    e = tc::launch_decode_mla_pair(map, a, st);
    if (e != cudaSuccess) return e;
    f.n_groups = tc::mla_groups(c);
    return tc::launch_decode_tc_mla(map, f, st);
  }
  if (c.d_cb == 512) return tc::launch_decode_tc_mla(map, a, st);
  if (use_wide(c)) {
    e = tc::launch_decode_wide(map, a, st);
    if (e != cudaSuccess || !rows_supported(c)) return e;
    f.n_groups = (c.n_blocks / g_of(c)) * (c.n_heads / hpc_of(c));
    return launch_rows(map, f, st);
  }
  return launch_rows(map, a, st);
}

}  // namespace mlra
