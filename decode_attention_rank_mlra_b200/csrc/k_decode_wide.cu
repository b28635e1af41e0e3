// Tensor-core split-KV decode attention for 128 query heads per CTA and one
// latent branch of 128 channels (sm_100a): MLRA-4 / MLRA-2 / MLA-128 layers
// whose head count is a multiple of 128.
//
// What it computes is the same as the other attention kernels: for one split
// of one sequence, one branch b and 128 heads,
//   z_t = (q_abs . c_b[t] + q_rope . k_rope[t]) * scale,
//   o = softmax(z) . c_b,  lse = log sum exp z
// with one softmax per latent branch ("Multi-Head Low-Rank Attention",
// Methodology, second paragraph) over the shared latent cache, i.e. the
// absorbed "MQA-style" step of Main Findings ("three absorbable steps").
//
// How (one CTA per SM, persistent over a share of the tile stream):
//  * warp 13 streams 64-token tiles of the cache with TMA (SWIZZLE_128B boxes of
//    64 rows x 64 columns): the two boxes of latent block c_b and the RoPE box,
//    into a multi-stage shared-memory ring;
//  * warps 8, 10, 11 convert each arrived tile's two latent boxes from bf16 to fp16
//    in place and zero the rows past the sequence end (exact for
//    2^-17 <= |c| < 65520; larger magnitudes are reported as MLRA_ERR_RANGE, and
//    the head-rows kernel launched after this one then recomputes the call);
//  * warp 9 issues tcgen05.mma: S = Q . C^T with the 128 MMA rows = the 128
//    heads, the queries in TMEM (A) and the tile K-major in shared memory (B):
//    8 MMAs with the fp16 query against the fp16 latent block (one row per
//    head, scaled by a power of two that brings its largest magnitude to
//    [2^13, 2^14)), 4 with the bf16 RoPE query (scaled by the same power of
//    two, exactly) against the bf16 RoPE box; then O += P . C_b with P in TMEM
//    (A, fp16) and the fp16 tile MN-major (B);
//  * warps 0-7 (two per TMEM lane quadrant: thread = one head = one TMEM lane
//    and one half of the tile's 64 tokens) run the online softmax of their
//    row and write P as fp16 over S (an MMA's A and B share one type; fp16 P
//    carries 11 significant bits where bf16 P carries 8, which the bf16
//    tolerance needs).
#include "dispatch.h"
#include "tc_common.cuh"

#include <cuda_fp16.h>
#include <math.h>

namespace mlra {
namespace {

using namespace ptx;
using tc::kBoxBytes;
using tc::kSmemLimit;
using tc::wait_bar;
using tc::wait_bar_warp;

constexpr int kThreadsW = 448;  // warps 0-7 softmax, 8, 10, 11 convert, 9 MMA, 13 TMA, 12 idle
// Warp w runs on scheduler w % 4.  The softmax warps of the slowest scheduler
// gate every tile, so the other roles are spread thin: one converter on
// schedulers 0, 2 and 3 each, the MMA and TMA warps (light issue) on 1.
// (Measured: a converter beside the MMA warp, or two on one scheduler, left that
// scheduler's softmax warps 700-2,000 cycles behind the others.)
constexpr int kWarpTma = 13, kWarpMma = 9, kConvWarps = 3;
__device__ __forceinline__ bool is_conv(int w) { return w == 8 || w == 10 || w == 11; }
__device__ __forceinline__ int conv_index(int w) { return w == 8 ? 0 : w - 9; }
constexpr uint32_t kTmemColsW = 512;
constexpr uint32_t kColQ = 0;                 // fp16 query (64 cols) | bf16 RoPE query (32)
constexpr uint32_t kColQr = 64;
constexpr int kNS = 4;                        // S / P buffers (PV(k) follows QK(k + kLook))
constexpr int kLook = 2;                      // QKs issued ahead of the oldest pending PV
static_assert(kLook < kNS, "QK(k + kNS) reuses the buffer that PV(k) reads");
constexpr uint32_t kColS = 128;               // S / P buffers: kNS x 64 columns
constexpr uint32_t kColO = kColS + 64 * kNS;  // O accumulator: 128 columns
constexpr int kBoxesW = 3;                    // two latent boxes + the RoPE box
constexpr int kStageW = kBoxesW * kBoxBytes;
constexpr int kStagesRawW = (kSmemLimit - 2048) / kStageW;
constexpr int kStagesW = kStagesRawW > 8 ? 8 : kStagesRawW;
constexpr int kBarsW = 3 * kStagesW + 3 * kNS + 2;
constexpr int kSmemW = 1024 + kStagesW * kStageW + kBarsW * 8 + 64 + 4 * 128 * 4;
constexpr float kPMaxW = 32768.f;             // largest P kept before a rescale (fp16)
static_assert(kStagesW >= 3, "too few pipeline stages");

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// Grid: (branches x head groups of 128) x CTAs per group; one CTA per SM.
__global__ void __launch_bounds__(kThreadsW, 1)
    decode_wide_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  constexpr int NST = kStagesW;
  constexpr int STAGE = kStageW;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NST * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarsW);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xch = reinterpret_cast<float*>(tmem_slot + 16);  // [2 maxima | 2 sums][128 rows]
  const uint32_t bar0 = smem_addr(bars);
  auto FULL = [&](int i) { return bar0 + 8u * i; };
  auto EMPTY = [&](int i) { return bar0 + 8u * (NST + i); };
  auto CONV = [&](int i) { return bar0 + 8u * (2 * NST + i); };  // tile converted
  // S(k), P(k) and PV(k) use buffer k % kNS; phase parity (k / kNS) & 1.
  auto SFULL = [&](int i) { return bar0 + 8u * (3 * NST + i); };
  auto PREADY = [&](int i) { return bar0 + 8u * (3 * NST + kNS + i); };
  // PV of tile k commits to PVDONE(k % kNS): PV(k + kNS) cannot be issued
  // before this group signals P(k + kNS), so a waiter's parity is exact.
  auto PVDONE = [&](int i) { return bar0 + 8u * (3 * NST + 2 * kNS + i); };
  const uint32_t QREADY = bar0 + 8u * (3 * NST + 3 * kNS);  // one phase per piece
  const uint32_t DRAIN = bar0 + 8u * (3 * NST + 3 * kNS + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  int32_t* err = &hdr->error;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
      mbar_init(CONV(i), kConvWarps);
    }
    for (int i = 0; i < kNS; ++i) {
      mbar_init(SFULL(i), 1);
      mbar_init(PREADY(i), 8);
      mbar_init(PVDONE(i), 1);
    }
    mbar_init(QREADY, 8);
    mbar_init(DRAIN, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_addr(tmem_slot), kTmemColsW);
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
  const int branch = grp % nb;
  const int head0 = (grp / nb) * 128;
  __shared__ int plan_sm[12], scan_sm[kThreadsW / 32 + 1];
  plan_first_pieces<kThreadsW>(a.seqlens, a.batch, a.cap, a.ctas_per_group, c, plan_sm, scan_sm);
  const int total = plan_sm[0], share = plan_sm[1];
  Walker walk{reinterpret_cast<const int32_t*>(wsc + a.L.tile_off),
              reinterpret_cast<const int32_t*>(wsc + a.L.slot_off),
              a.seqlens, plan_sm + 2,
              a.batch, a.cap, c * share, min(total, (c + 1) * share)};

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      const uint64_t evict_first = policy_evict_first();  // the cache is streamed once
      Piece p;
      int it = 0;
      bool ok = true;
      while (ok && walk.next(p)) {
        for (int t = p.t0; t < p.t1; ++t, ++it) {
          const int st = it % NST;
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
          tma_load_2d_hint(dst, &tmap, branch * 128, row, FULL(st), evict_first);
          tma_load_2d_hint(dst + kBoxBytes, &tmap, branch * 128 + 64, row, FULL(st), evict_first);
          tma_load_2d_hint(dst + 2 * kBoxBytes, &tmap, nb * 128, row, FULL(st), evict_first);
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
  } else if (is_conv(warp)) {
    // ------------------------------------------------------------ converters
    // The tile's two latent boxes bf16 -> fp16 in place (16-byte chunks in
    // address order); rows past the valid tokens, latent and RoPE, become
    // zeros, so they never depend on what the cache holds there.
    const int ct = 32 * conv_index(warp) + lane;  // 0..95
    Piece p;
    int it = 0;
    bool ok = true;
    while (ok && walk.next(p)) {
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % NST;
        if (!wait_bar_warp(FULL(st), (it / NST) & 1, abort_flag, err)) { ok = false; break; }
        const int valid = min(kTile, p.L - t * kTile);
        const uint32_t base = smem_addr(stages + st * STAGE);
        const uint32_t over = tc::convert_stage<2 * 512, 32 * kConvWarps>(base, ct, valid);
        if (valid < kTile) tc::zero_box_rows<32 * kConvWarps>(base + 2 * kBoxBytes, ct, valid);
        if ((over & 0x80008000u) != 0) set_error(err, MLRA_ERR_RANGE);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(CONV(st));
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop; each MMA / commit is issued by one elected
    // lane, and every wait is warp-uniform.
    //  QK : S[heads, tokens] = Q . C^T (fp16) + Qr . Kr^T (bf16)
    //       (A: queries in TMEM, B: the tile K-major)
    //  PV : O[heads, features] += P[heads, tokens] . C_b[tokens, features]
    //       (A: fp16 probabilities in TMEM over the S buffer, B: the fp16 tile MN-major)
    constexpr uint32_t kIdescQK = idesc_f16_f32(128, kTile, false, false);
    constexpr uint32_t kIdescQR = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t kIdescPV = idesc_f16_f32(128, 128, false, true);
    const uint32_t sbase0 = smem_addr(stages);
    const uint64_t dK = smem_desc(sbase0, 16, 1024, kSwizzle128B);
    const uint64_t dMN = smem_desc(sbase0, kBoxBytes, 1024, kSwizzle128B);
    Piece p;
    int it = 0, piece = 0;
    // tiles whose PV is still to be issued: npend consecutive tiles from
    // `oldest`; bit j of first_mask: pending tile j opens its piece (its PV
    // then overwrites O)
    int oldest = 0, npend = 0;
    uint32_t first_mask = 0;
    bool ok = true;
    // PV of the oldest pending tile: issued after QK of the kLook tiles that
    // follow it, so those scores are ready while its softmax runs
    auto issue_pv = [&]() -> bool {
      const int k0 = oldest;
      if (!wait_bar_warp(PREADY(k0 % kNS), (k0 / kNS) & 1, abort_flag, err)) return false;
      tc_fence_after();
      const uint64_t d = dMN + uint64_t(((k0 % NST) * STAGE) >> 4);
      const uint32_t a_p = tmem + kColS + 64 * (k0 % kNS);
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k)
        mma_ts_warp(tmem + kColO, a_p + 8 * k, d + uint64_t((k * 16 * 128) >> 4), kIdescPV,
                    ((first_mask & 1u) && k == 0) ? 0u : 1u, 0u, 0u, 0u, 0u);
      mma_commit_warp(EMPTY(k0 % NST));
      mma_commit_warp(PVDONE(k0 % kNS));
      ++oldest;
      first_mask >>= 1;
      --npend;
      return true;
    };
    while (ok && walk.next(p)) {
      if (!wait_bar_warp(QREADY, piece & 1, abort_flag, err)) { ok = false; break; }
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % NST, sb = it % kNS;
        if (!wait_bar_warp(CONV(st), (it / NST) & 1, abort_flag, err)) { ok = false; break; }
        tc_fence_after();
        {
          const uint64_t d = dK + uint64_t((st * STAGE) >> 4);
          const uint32_t s_acc = tmem + kColS + 64 * sb;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts_warp(s_acc, tmem + kColQ + 8 * k,
                        d + uint64_t((((k >> 2) * kBoxBytes) + (k & 3) * 32) >> 4), kIdescQK,
                        k > 0 ? 1u : 0u, 0u, 0u, 0u, 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_warp(s_acc, tmem + kColQr + 8 * k,
                        d + uint64_t((2 * kBoxBytes + k * 32) >> 4), kIdescQR, 1u, 0u, 0u, 0u, 0u);
          mma_commit_warp(SFULL(sb));
        }
        if (npend == 0) oldest = it;
        first_mask |= uint32_t(t == p.t0) << npend;
        ++npend;
        if (npend > kLook && !issue_pv()) { ok = false; break; }
      }
      // the piece's last PVs go out before the next piece's first QK: the
      // epilogue waits for them, and the next piece's queries wait for the epilogue
      while (ok && npend > 0)
        if (!issue_pv()) ok = false;
      ++piece;
    }
    if (!ok) {
      // drain MMAs already issued before TMEM is released
      mma_commit_warp(DRAIN);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(DRAIN, 0) && globaltimer() - t0 < 10000000ull) {}
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax warps 0-7
    // Warps q and q + 4 share TMEM lane quadrant q: a thread owns one head
    // (lane = row) and one half of each tile's 64 tokens (x = warp / 4); the
    // two halves of a row meet at a 64-thread named barrier (id 1 + q) only to
    // combine the row's maxima and sums.  Every wait ends in a vote at that
    // barrier, so the pair leaves a failed wait together.
    const int q4 = warp & 3, x = warp >> 2;
    const int r = 32 * q4 + lane;
    const int head = head0 + r;
    const int pid = 1 + q4;
    const uint32_t row_t = tmem + (uint32_t(32 * q4) << 16);
    const float sl2_base = a.cfg.softmax_scale * 1.4426950408889634f;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
    const unsigned short* q_rope = static_cast<const unsigned short*>(a.q_rope);
    float* mx_sm = xch;          // [2][128] tile maxima of the two halves
    float* lx_sm = xch + 256;    // [2][128] sums of the two halves
    auto pair_fail = [&](bool good) { return bar_red_or(pid, 64, !good); };

    // This head's queries into TMEM, half x of the latent channels and of the
    // RoPE channels, both times 2^e (e from the largest |q_abs| of the row, so
    // that it lands in [2^13, 2^14) as fp16): fp16(q 2^e) | q_rope 2^e (bf16,
    // exact).  Returns 2^-e, which the softmax folds into its scale.
    auto write_q = [&](const Piece& pc) -> float {
      const float4* q0 = reinterpret_cast<const float4*>(
          a.q_abs + ((size_t(pc.s) * H + head) * nb + branch) * 128);
      float mx = 0.f;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const float4 g = __ldg(q0 + j);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(g.x), fabsf(g.y)), fmaxf(fabsf(g.z), fabsf(g.w))));
      }
      int e = 0;
      if (mx > 0.f && mx < INFINITY) {
        const int k = int((__float_as_uint(mx) >> 23) & 0xff) - 126;  // mx in [2^(k-1), 2^k)
        e = min(max(14 - k, -100), 100);
      }
      const float sc = __int_as_float((127 + e) << 23);
      uint32_t w[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float4 g = __ldg(q0 + 16 * x + j);
        w[2 * j] = pack_f16(g.x * sc, g.y * sc);
        w[2 * j + 1] = pack_f16(g.z * sc, g.w * sc);
      }
      tmem_st32(row_t + kColQ + 32 * x, w);
      const uint4* qr =
          reinterpret_cast<const uint4*>(q_rope + (size_t(pc.s) * H + head) * 64) + 4 * x;
      uint32_t rr[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 u = __ldg(qr + j);
        const uint32_t uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)  // bf16 pair times 2^e: exact
          rr[4 * j + e2] = tc::pack_bf16(__uint_as_float(uv[e2] << 16) * sc,
                                         __uint_as_float(uv[e2] & 0xffff0000u) * sc);
      }
      tmem_st16(row_t + kColQr + 16 * x, rr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(QREADY);
      return 1.f / sc;
    };

    Piece p, pn;
    int it = 0;
    bool ok = walk.next(p);
    float inv_sc = ok ? write_q(p) : 1.f;
    while (ok) {
      const float sl2 = sl2_base * inv_sc;
      // m: the reference point of the exponentials, in log2 units, the same in
      // both halves of a row.  It is the first tile's max and moves only when a
      // later tile would push P past 2^15 (fp16 keeps it exactly); a stale m
      // only scales all weights alike.  l: this half's sum.
      float m = -INFINITY, l = 0.f;
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int sb = it % kNS;
        bool good = wait_bar_warp(SFULL(sb), (it / kNS) & 1, abort_flag, err);
        tc_fence_after();
        float z[32];  // raw scores of tokens 32x.. ; the scale enters with the exponent
        {
          uint32_t sv[32];
          tmem_ld32(row_t + kColS + 64 * sb + 32 * x, sv);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) z[k] = __uint_as_float(sv[k]);
        }
        const int valid = min(kTile, p.L - t * kTile);
        if (valid < kTile) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (32 * x + k >= valid) z[k] = -INFINITY;
        }
        auto half_max = [&]() {
          float t16[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) t16[k] = fmaxf(z[k], z[k + 16]);
#pragma unroll
          for (int k = 0; k < 8; ++k) t16[k] = fmaxf(t16[k], t16[k + 8]);
#pragma unroll
          for (int k = 0; k < 4; ++k) t16[k] = fmaxf(t16[k], t16[k + 4]);
          return fmaxf(fmaxf(t16[0], t16[1]), fmaxf(t16[2], t16[3])) * sl2;
        };
        // the row's maximum over both halves (every wait of the pair has been
        // voted on before, so both halves reach this barrier)
        auto row_max = [&]() {
          mx_sm[x * 128 + r] = half_max();
          bar_sync(pid, 64);
          const float v = fmaxf(mx_sm[r], mx_sm[128 + r]);
          return v;
        };
        if (t == p.t0) {
          if (pair_fail(good)) { ok = false; break; }
          m = row_max();
        }
        uint32_t pw[16];
        float ls;
        auto exps = [&]() {
          ls = 0.f;
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float p0 = ex2_approx(fmaf(z[k], sl2, -m));
            const float p1 = ex2_approx(fmaf(z[k + 1], sl2, -m));
            ls += p0 + p1;
            pw[k / 2] = pack_f16(p0, p1);
          }
        };
        exps();
        // (ls bounds every P of this half: a P above 2^15 or a NaN fails the test)
        if (bar_red_or(pid, 64, !(ls <= kPMaxW) || !good)) {
          if (pair_fail(good)) { ok = false; break; }
          // rare: a score far above m (or a NaN).  Raise m to this tile's row
          // max, rescale l and the O row once the previous PV is done, redo the
          // tile.  Each warp of the pair rescales its half of the O columns; the
          // pass is taken by the whole warp (alpha = 1 for rows whose m stays).
          const float mt = row_max();
          float alpha = 1.f;
          if (mt > m) {
            alpha = ex2_approx(m - mt);
            m = mt;
            l *= alpha;
          }
          const bool any = __any_sync(0xffffffffu, alpha != 1.f);
          const int pk = it - 1;
          const bool g2 = !any || wait_bar_warp(PVDONE(pk % kNS), (pk / kNS) & 1, abort_flag, err);
          if (pair_fail(g2)) { ok = false; break; }
          if (any) {
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
              uint32_t ov[32];
              tmem_ld32(row_t + kColO + 64 * x + 32 * ch, ov);
              tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
              tmem_st32(row_t + kColO + 64 * x + 32 * ch, ov);
            }
            tmem_wait_st();
          }
          exps();
        }
        l += ls;
        tmem_st16(row_t + kColS + 64 * sb + 16 * x, pw);  // P over the first 32 columns of S
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PREADY(sb));
      }
      if (!ok) break;
      // every QK of this piece is done: the query columns take the next piece's
      const bool has_next = walk.next(pn);
      if (has_next) inv_sc = write_q(pn);
      // ---- epilogue: o = O / l, lse (this half: O columns 64x..64x+63)
      {
        const int pk = it - 1;
        const bool g = wait_bar_warp(PVDONE(pk % kNS), (pk / kNS) & 1, abort_flag, err);
        if (pair_fail(g)) { ok = false; break; }
      }
      tc_fence_after();
      lx_sm[x * 128 + r] = l;
      bar_sync(pid, 64);
      const float l_tot = lx_sm[r] + lx_sm[128 + r];
      const float inv = l_tot > 0.f ? 1.f / l_tot : 0.f;
      float* dst = o_part + ((size_t(p.slot) * H + head) * nb + branch) * 128 + 64 * x;
#pragma unroll 1
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t ov[32];
        tmem_ld32(row_t + kColO + 64 * x + 32 * ch, ov);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o8[e] = __uint_as_float(ov[8 * k + e]) * inv;
          st_global_v8(dst + 32 * ch + 8 * k, o8);
        }
      }
      if (x == 0)
        lse_part[(size_t(p.slot) * H + head) * nb + branch] =
            l_tot > 0.f ? (m + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
      // (the next piece's first PV overwrites O only after its first P is
      // ready, which this thread signals after these loads completed; lx_sm is
      // next written after the pair's next barriers)
      if (!has_next) break;
      p = pn;
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_wait();  // complete only after the plan kernel (whose records the merge reads)
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemColsW);
  }
}

}  // namespace

namespace tc {

bool wide_supported(const mlra_config_t& c) {
  return c.dtype == MLRA_BF16 && c.d_cb == 128 && c.d_r == 64 && c.n_heads % 128 == 0 &&
         (c.n_blocks == 1 || c.n_blocks == 2 || c.n_blocks == 4);
}

int wide_groups(const mlra_config_t& c) { return c.n_blocks * (c.n_heads / 128); }

cudaError_t launch_decode_wide(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_wide_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemW);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  return launch_pdl(decode_wide_kernel, dim3(a.n_groups * a.ctas_per_group), dim3(kThreadsW),
                    kSmemW, st, map, a);
}

}  // namespace tc
}  // namespace mlra
