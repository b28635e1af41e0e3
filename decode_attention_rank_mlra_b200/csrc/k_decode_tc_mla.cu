// Tensor-core split-KV decode attention for MLA (one latent block of 512
// channels plus the shared RoPE key, sm_100a): the comparison mode of
// "Multi-Head Low-Rank Attention" (Main Findings: MLA caches one 4 d_h latent
// head; Methodology: MLRA partitions it into blocks).
//
// What it computes is the same as the other attention kernels with
// n_blocks = 1: z_t = (q_abs . c[t] + q_rope . k_rope[t]) * scale,
// o = softmax(z) . c, lse = log sum exp z, per head and split.
//
// How.  With 64 heads a CTA's MMA rows are (head, hi|lo) = 128.  The 512-wide
// output does not fit TMEM beside the queries, so a CTA owns one 256-feature
// half of the output, and the two half CTAs of a head group compute the same
// scores (bit for bit: same operands, same MMA order).  TMEM holds the hi/lo
// queries of latent channels 0-255 (128 columns), the RoPE query (32), S (64)
// and the O half (256); the queries of channels 256-511 sit in shared memory
// (64 KB, K-major, 128-byte swizzle) as the A operand of the second half of
// the scores.
//  * warp 4: TMA of the nine 64-column boxes of a 64-token tile (8 latent +
//    RoPE) into a 2-stage ring;
//  * warp 5: S = Q C^T over K = 512 + 64 (36 MMAs of M = 128, N = 64: 16 with
//    A in TMEM, 16 with A in shared memory, 4 for RoPE), then, once the
//    softmax has written P over S, O += P C_q over the half's four boxes
//    (MN-major B, two MMA groups of N = 128);
//  * warps 0-3: the softmax of the hi / lo rows exactly as in k_decode_tc.cu.
// S has a single 64-column buffer (TMEM is full), so the QK of tile i+1 is
// issued right after the PV of tile i.
#include "tc_common.cuh"

#include <math.h>

namespace mlra {
namespace tc {
namespace {

using namespace ptx;

constexpr int kThreads = 192;          // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kHeads = 64;             // heads per CTA (128 MMA rows with hi / lo)
constexpr int kLat = 512;              // latent channels
constexpr int kBoxes = kLat / kBoxCols + 1;  // 8 latent boxes + RoPE
constexpr int kStage = kBoxes * kBoxBytes;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;          // q_abs hi / lo rows, channels 0-255: 128 columns
constexpr uint32_t kColQr = 128;       // q_rope rows: 32 columns
constexpr uint32_t kColS = 160;        // S / P: 64 columns
constexpr uint32_t kColO = 224;        // O half: two 128-feature quarters, 256 columns
constexpr int kQsChunk = 128 * 128;    // 128 rows x 64 channels of bf16
constexpr int kQsBytes = 4 * kQsChunk; // q_abs hi / lo rows, channels 256-511
constexpr int kBars = 2 * kStages + 6;
constexpr int kSmem = 1024 + kQsBytes + kStages * kStage + kBars * 8 + 64;
static_assert(kSmem <= kSmemLimit, "shared memory");

__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_mla_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* q_sm = smem;                  // queries of channels 256-511
  uint8_t* stages = smem + kQsBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stages + kStages * kStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t bar0 = smem_addr(bars);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (kStages + i); };
  const uint32_t SFULL = bar0 + 8u * (2 * kStages);
  const uint32_t PREADY = bar0 + 8u * (2 * kStages + 1);
  // PV of tile k completes phase k of PVDONE; QK of tile k+1 is issued after
  // it, so anyone who has seen S(k+1) waits on an exact phase.
  const uint32_t PVDONE = bar0 + 8u * (2 * kStages + 2);
  const uint32_t QREADY = bar0 + 8u * (2 * kStages + 3);
  const uint32_t DRAIN = bar0 + 8u * (2 * kStages + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  if (a.range_fallback) {
    // after the 128-head kernel's grid: every thread reads its final error word
    pdl_wait();
    if (*reinterpret_cast<volatile int32_t*>(&hdr->error) != MLRA_ERR_RANGE) return;
  }
  int32_t* err = a.range_fallback ? &hdr->fallback_error : &hdr->error;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
    }
    mbar_init(SFULL, 1);
    mbar_init(PREADY, 4);
    mbar_init(PVDONE, 1);
    mbar_init(QREADY, 4);
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
  // As in k_decode_tc.cu: no wait for the plan kernel; the CTA plans its own
  // first two pieces.
  pdl_trigger();

  const char* wsc = static_cast<const char*>(a.ws);
  const int H = a.cfg.n_heads;
  const int grp = blockIdx.x / a.ctas_per_group;
  const int c = blockIdx.x % a.ctas_per_group;
  const int fh = grp & 1;                 // output half: features 256 fh ..
  const int head0 = (grp >> 1) * kHeads;  // first head of the CTA's head group
  __shared__ int plan_sm[12], scan_sm[kThreads / 32 + 1];
  plan_first_pieces<kThreads>(a.seqlens, a.batch, a.cap, a.ctas_per_group, c, plan_sm, scan_sm);
  const int total = plan_sm[0], share = plan_sm[1];
  Walker walk{reinterpret_cast<const int32_t*>(wsc + a.L.tile_off),
              reinterpret_cast<const int32_t*>(wsc + a.L.slot_off),
              a.seqlens, plan_sm + 2,
              a.batch, a.cap, c * share, min(total, (c + 1) * share)};

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      const uint64_t evict_first = policy_evict_first();
      Piece p;
      int it = 0;
      bool ok = true;
      while (ok && walk.next(p)) {
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          const int st = it % kStages;
          if (!wait_bar(EMPTY(st), ((it / kStages) & 1) ^ 1, abort_flag, err)) { ok = false; break; }
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
          mbar_arrive_expect_tx(FULL(st), kStage);
          const uint32_t dst = smem_addr(stages + st * kStage);
#pragma unroll
          for (int bx = 0; bx < kBoxes; ++bx)
            tma_load_2d_hint(dst + bx * kBoxBytes, &tmap, bx * kBoxCols, row, FULL(st), evict_first);
        }
      }
      if (!ok) {
        for (int j = 0; j < kStages; ++j) {
          const int k = it - 1 - j;
          if (k < 0) break;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(FULL(k % kStages), (k / kStages) & 1) &&
                 globaltimer() - t0 < 10000000ull) {}
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    // (converged lanes poll each barrier together, as in k_decode_tc.cu)
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);
    const uint32_t sbase0 = smem_addr(stages);
    const uint64_t dK = smem_desc(sbase0, 16, 1024, kSwizzle128B);
    const uint64_t dMN = smem_desc(sbase0, kBoxBytes, 1024, kSwizzle128B);
    const uint64_t dQs = smem_desc(smem_addr(q_sm), 16, 1024, kSwizzle128B);
    Piece p;
    int it = 0, piece = 0;
    bool ok = true;
    while (ok && walk.next(p)) {
      if (!wait_bar_warp(QREADY, piece & 1, abort_flag, err)) { ok = false; break; }
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % kStages;
        if (!wait_bar_warp(FULL(st), (it / kStages) & 1, abort_flag, err)) { ok = false; break; }
        const int valid = min(kTile, p.L - t * kTile);
        if (valid < kTile) {
          // zero the rows past the sequence end (whatever the cache holds there)
          const int per_box = (kTile - valid) * 8;
          uint8_t* sp = stages + st * kStage;
          for (int i = lane; i < per_box * kBoxes; i += 32) {
            const int bx = i / per_box, rem = i % per_box;
            *reinterpret_cast<uint4*>(sp + bx * kBoxBytes + (valid + rem / 8) * 128 + (rem % 8) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        const uint64_t d = dK + uint64_t((st * kStage) >> 4);
        // S = Q_lat C^T (32 K-steps over the 8 latent boxes: channels 0-255
        // with A in TMEM, 256-511 with A in shared memory) + Q_rope K_rope^T
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mma_ts_warp(tmem + kColS, tmem + kColQ + 8 * k,
                      d + uint64_t(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4), kIdescQK,
                      k > 0 ? 1u : 0u, 0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 16; k < kLat / 16; ++k)
          mma_ss_warp(tmem + kColS,
                      dQs + uint64_t((((k - 16) >> 2) * kQsChunk + ((k - 16) & 3) * 32) >> 4),
                      d + uint64_t(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4), kIdescQK, 1u);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts_warp(tmem + kColS, tmem + kColQr + 8 * k,
                      d + uint64_t(((kBoxes - 1) * kBoxBytes + k * 32) >> 4), kIdescQK, 1u, 0u, 0u,
                      0u, 0u);
        mma_commit_warp(SFULL);
        // O_q += P C_q once the probabilities are over S
        if (!wait_bar_warp(PREADY, it & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const uint64_t dv =
              dMN + uint64_t((st * kStage + 2 * (2 * fh + qq) * kBoxBytes) >> 4);
#pragma unroll
          for (int k = 0; k < kTile / 16; ++k)
            mma_ts_warp(tmem + kColO + 128 * qq, tmem + kColS + 8 * k,
                        dv + uint64_t((k * 16 * 128) >> 4), kIdescPV,
                        (t == p.t0 && k == 0) ? 0u : 1u, 0u, 0u, 0u, 0u);
        }
        mma_commit_warp(EMPTY(st));
        mma_commit_warp(PVDONE);
      }
      ++piece;
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
    // Quadrant w: lanes 0-15 the hi rows, lanes 16-31 the lo rows of heads
    // head0 + 16 w + (0..15).  x = lane / 16 picks the half of each tile's
    // tokens a thread takes the softmax of, and the half of the query row it
    // converts (see k_decode_tc.cu for the .16x32bx2 pairing).
    const int x = lane >> 4;
    const int head = head0 + 16 * warp + (lane & 15);
    const uint32_t row_t = tmem + (uint32_t(32 * warp) << 16);
    const uint32_t hi_t = row_t, lo_t = row_t + (16u << 16);
    const float sl2 = a.cfg.softmax_scale * 1.4426950408889634f;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
    const unsigned short* q_rope = static_cast<const unsigned short*>(a.q_rope);
    auto q_row = [&](const Piece& pc) {
      return reinterpret_cast<const float4*>(a.q_abs + (size_t(pc.s) * H + head) * kLat);
    };
    auto qr_row = [&](const Piece& pc) {
      return reinterpret_cast<const uint4*>(q_rope + (size_t(pc.s) * H + head) * 64);
    };
    // Thread (warp, lane) fills MMA row 32 warp + lane: the hi (x = 0) or lo
    // (x = 1) bf16 part of its head's query.  Channels 0-255 go to TMEM (32x32b
    // stores: a thread writes its own lane), channels 256-511 to the shared-
    // memory A operand: four 16 KB chunks of 64 channels, K-major with the
    // 128-byte swizzle (16-byte unit u of row r at u ^ (r & 7)).  The previous
    // piece's QK MMAs, the only readers of either, are complete when this runs.
    uint8_t* const q_srow = q_sm + (4 * warp + (lane >> 3)) * 1024 + (lane & 7) * 128;
    auto write_q = [&](const Piece& pc) {
      const float4* q = q_row(pc);
#pragma unroll 1
      for (int r = 0; r < 8; ++r) {  // 64 channels per round
        float4 f[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = __ldg(q + 16 * r + j);
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float v[4] = {f[j].x, f[j].y, f[j].z, f[j].w};
          float u[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            u[e] = x ? v[e] - __bfloat162float(__float2bfloat16_rn(v[e])) : v[e];
          w[2 * j] = pack_bf16(u[0], u[1]);
          w[2 * j + 1] = pack_bf16(u[2], u[3]);
        }
        if (r < 4) {
          tmem_st32(row_t + kColQ + 32 * r, w);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(q_srow + (r - 4) * kQsChunk + ((k ^ (lane & 7)) << 4)) =
                make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      // RoPE query: the hi row holds it, the lo row zeros
      uint32_t rr[32];
      if (x == 0) {
        const uint4* qr = qr_row(pc);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 u = __ldg(qr + j);
          rr[4 * j] = u.x; rr[4 * j + 1] = u.y; rr[4 * j + 2] = u.z; rr[4 * j + 3] = u.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) rr[j] = 0u;
      }
      tmem_st32(row_t + kColQr, rr);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(QREADY);
    };
    auto prefetch_q = [&](const Piece& pc) {
      const char* q = reinterpret_cast<const char*>(q_row(pc)) + 1024 * x;
#pragma unroll
      for (int k = 0; k < 8; ++k) prefetch_l2_evict_last(q + 128 * k);
      if (x == 0) prefetch_l2_evict_last(qr_row(pc));
    };
    Piece p, pn;
    int it = 0;
    bool ok = walk.next(p);
    bool has_next = ok && walk.next(pn);
    if (ok) write_q(p);
    if (has_next) prefetch_q(pn);
    while (ok) {
      // m: reference point of the exponentials (log2 units), the first tile's
      // max, moved only when a later tile would overflow (as in k_decode_tc.cu)
      float m = -INFINITY, l = 0.f;
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        if (!wait_bar_warp(SFULL, it & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        float raw[32];
        {
          uint32_t sh[32], sl[32];
          tmem_ld_x2_32<32>(hi_t + kColS, sh);
          tmem_ld_x2_32<32>(lo_t + kColS, sl);
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
          // rare: a score far above m (or a NaN): raise m, rescale l and the O
          // rows (the previous PV is complete: S of this tile was issued after it)
          // (the TMEM pass is warp-wide: alpha = 1 for rows whose m stays)
          const float mt = tile_max();
          float alpha = 1.f;
          if (mt > m) {
            alpha = ex2_approx(m - mt);
            m = mt;
            l *= alpha;
          }
          if (t > p.t0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            if (!wait_bar_warp(PVDONE, (it - 1) & 1, abort_flag, err)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 8; ++ch) {
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
        tmem_st_x2_16<16>(hi_t + kColS, whi);
        tmem_st_x2_16<16>(lo_t + kColS, wlo);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PREADY);
        // every QK of this piece is done: the next piece's queries can go in now
        if (t + 1 == p.t1 && has_next) write_q(pn);
      }
      if (!ok) break;
      // ---- epilogue: o = (O_hi + O_lo) / l for the half, lse
      if (!wait_bar_warp(PVDONE, (it - 1) & 1, abort_flag, err)) { ok = false; break; }
      tc_fence_after();
      const float l_tot = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      float* dst = o_part + (size_t(p.slot) * H + head) * kLat + 256 * fh;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        uint32_t oh[32], ol[32];
        tmem_ld_x2_32<128>(hi_t + kColO + 32 * j, oh);
        tmem_ld_x2_32<128>(lo_t + kColO + 32 * j, ol);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            o8[e] = (__uint_as_float(oh[8 * k + e]) + __uint_as_float(ol[8 * k + e])) * inv;
          st_global_v8(dst + 128 * x + 32 * j + 8 * k, o8);
        }
      }
      // the two half CTAs hold the same m and l: half 0 writes the lse
      if (fh == 0 && x == 0)
        lse_part[size_t(p.slot) * H + head] =
            l_tot > 0.f ? (m + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
      if (!has_next) break;
      p = pn;
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

}  // namespace

cudaError_t launch_decode_tc_mla(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_mla_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  return launch_pdl(decode_tc_mla_kernel, dim3(a.n_groups * a.ctas_per_group), dim3(kThreads),
                    kSmem, st, map, a);
}

}  // namespace tc
}  // namespace mlra
