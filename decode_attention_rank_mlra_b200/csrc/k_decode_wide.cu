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
//  * warp 4 streams 64-token tiles of the cache with TMA (SWIZZLE_128B boxes of
//    64 rows x 64 columns): the two boxes of latent block c_b and the RoPE box,
//    into a multi-stage shared-memory ring;
//  * warp 5 issues tcgen05.mma: S = Q . C^T with the 128 MMA rows = the 128
//    heads, the queries in TMEM (A) and the tile K-major in shared memory (B);
//    the fp32 absorbed query enters as bf16 hi and lo halves along K (16 MMAs
//    over the latent block, 4 over the RoPE box, whose bf16 query is exact);
//    then O += P . C_b with P in TMEM (A, fp16) and the tile MN-major (B);
//  * warps 0-7 (two per TMEM lane quadrant: thread = one head = one TMEM lane
//    and one half of the tile's 64 tokens) run the online softmax of their
//    row, write P as fp16 over S, and convert
//    the tile's latent boxes from bf16 to fp16 in place for the product with P
//    (an MMA's A and B share one type; fp16 P carries 11 significant bits where
//    bf16 P carries 8, which the bf16 tolerance needs); the conversion is exact
//    for |c| < 65520 and larger magnitudes are reported as MLRA_ERR_RANGE.
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

constexpr int kThreadsW = 320;                // warps 0-7 softmax, 8 TMA, 9 MMA
constexpr int kWarpTma = 8, kWarpMma = 9;
constexpr uint32_t kTmemColsW = 512;
constexpr uint32_t kColQ = 0;                 // q hi (64 cols) | q lo (64) | q_rope (32)
constexpr uint32_t kColQlo = 64;
constexpr uint32_t kColQr = 128;
constexpr int kNS = 2;                        // S / P buffers (PV(k) follows QK(k + 1))
constexpr uint32_t kColS = 160;               // S / P buffers: kNS x 64 columns
constexpr uint32_t kColO = kColS + 64 * kNS;  // O accumulator: 128 columns
constexpr int kBoxesW = 3;                    // two latent boxes + the RoPE box
constexpr int kStageW = kBoxesW * kBoxBytes;
constexpr int kStagesRawW = (kSmemLimit - 2048) / kStageW;
constexpr int kStagesW = kStagesRawW > 8 ? 8 : kStagesRawW;
constexpr int kBarsW = 2 * kStagesW + 3 * kNS + 2;
constexpr int kSmemW = 1024 + kStagesW * kStageW + kBarsW * 8 + 64 + 4 * 128 * 4;
constexpr float kPMaxW = 32768.f;             // largest P kept before a rescale (fp16)
static_assert(kStagesW >= 3, "too few pipeline stages");

// Instruction descriptor of kind::f16 with fp32 accumulation, fp16 A and B.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major,
                                                     bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

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
  // S(k), P(k) and PV(k) use buffer k % kNS; phase parity (k / kNS) & 1.
  auto SFULL = [&](int i) { return bar0 + 8u * (2 * NST + i); };
  auto PREADY = [&](int i) { return bar0 + 8u * (2 * NST + kNS + i); };
  // PV of tile k commits to PVDONE(k % kNS): PV(k + kNS) cannot be issued
  // before this group signals P(k + kNS), so a waiter's parity is exact.
  auto PVDONE = [&](int i) { return bar0 + 8u * (2 * NST + 2 * kNS + i); };
  const uint32_t QREADY = bar0 + 8u * (2 * NST + 3 * kNS);  // one phase per piece
  const uint32_t DRAIN = bar0 + 8u * (2 * NST + 3 * kNS + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  int32_t* err = &hdr->error;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(FULL(i), 1);
      mbar_init(EMPTY(i), 1);
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
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop; each MMA / commit is issued by one elected
    // lane, and every wait is warp-uniform.
    //  QK : S[heads, tokens] = Q_hi . C^T + Q_lo . C^T + Qr . Kr^T
    //       (A: queries in TMEM, B: the tile K-major)
    //  PV : O[heads, features] += P[heads, tokens] . C_b[tokens, features]
    //       (A: fp16 probabilities in TMEM over the S buffer, B: the fp16 tile MN-major)
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t kIdescPV = idesc_f16_f32(128, 128, false, true);
    const uint32_t sbase0 = smem_addr(stages);
    const uint64_t dK = smem_desc(sbase0, 16, 1024, kSwizzle128B);
    const uint64_t dMN = smem_desc(sbase0, kBoxBytes, 1024, kSwizzle128B);
    Piece p;
    int it = 0, piece = 0;
    int prev = -1;            // tile whose PV is still to be issued
    bool prev_first = false;  // ...and whether it opens its piece
    bool ok = true;
    // PV(prev): after QK(prev + 1), so the softmax of tile prev overlaps it
    auto issue_pv = [&]() -> bool {
      if (!wait_bar_warp(PREADY(prev % kNS), (prev / kNS) & 1, abort_flag, err)) return false;
      tc_fence_after();
      const uint64_t d = dMN + uint64_t(((prev % NST) * STAGE) >> 4);
      const uint32_t a_p = tmem + kColS + 64 * (prev % kNS);
#pragma unroll
      for (int k = 0; k < kTile / 16; ++k)
        mma_ts_warp(tmem + kColO, a_p + 8 * k, d + uint64_t((k * 16 * 128) >> 4), kIdescPV,
                    (prev_first && k == 0) ? 0u : 1u, 0u, 0u, 0u, 0u);
      mma_commit_warp(EMPTY(prev % NST));
      mma_commit_warp(PVDONE(prev % kNS));
      prev = -1;
      return true;
    };
    while (ok && walk.next(p)) {
      if (!wait_bar_warp(QREADY, piece & 1, abort_flag, err)) { ok = false; break; }
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % NST, sb = it % kNS;
        if (!wait_bar_warp(FULL(st), (it / NST) & 1, abort_flag, err)) { ok = false; break; }
        const int valid = min(kTile, p.L - t * kTile);
        if (valid < kTile) {
          // zero the rows past the sequence end (whatever the cache holds there)
          const int per_box = (kTile - valid) * 8;
          uint8_t* sp = stages + st * STAGE;
          for (int i = lane; i < per_box * kBoxesW; i += 32) {
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
          for (int k = 0; k < 8; ++k)
            mma_ts_warp(s_acc, tmem + kColQ + 8 * k,
                        d + uint64_t((((k >> 2) * kBoxBytes) + (k & 3) * 32) >> 4), kIdescQK,
                        k > 0 ? 1u : 0u, 0u, 0u, 0u, 0u);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts_warp(s_acc, tmem + kColQlo + 8 * k,
                        d + uint64_t((((k >> 2) * kBoxBytes) + (k & 3) * 32) >> 4), kIdescQK, 1u,
                        0u, 0u, 0u, 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_warp(s_acc, tmem + kColQr + 8 * k,
                        d + uint64_t((2 * kBoxBytes + k * 32) >> 4), kIdescQK, 1u, 0u, 0u, 0u, 0u);
          mma_commit_warp(SFULL(sb));
        }
        if (prev >= 0 && !issue_pv()) { ok = false; break; }
        prev = it;
        prev_first = (t == p.t0);
      }
      // the piece's last PV goes out before the next piece's first QK: the
      // epilogue waits for it, and the next piece's queries wait for the epilogue
      if (ok && prev >= 0 && !issue_pv()) ok = false;
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
    const float sl2 = a.cfg.softmax_scale * 1.4426950408889634f;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
    const unsigned short* q_rope = static_cast<const unsigned short*>(a.q_rope);
    float* mx_sm = xch;          // [2][128] tile maxima of the two halves
    float* lx_sm = xch + 256;    // [2][128] sums of the two halves
    auto pair_fail = [&](bool good) { return bar_red_or(pid, 64, !good); };

    // This head's queries into TMEM, half x of the latent channels and of the
    // RoPE channels: bf16(q) | bf16(q - bf16(q)) | q_rope.
    auto write_q = [&](const Piece& pc) {
      const float4* q = reinterpret_cast<const float4*>(
          a.q_abs + ((size_t(pc.s) * H + head) * nb + branch) * 128) + 16 * x;
      float4 f[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) f[j] = __ldg(q + j);
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v[4] = {f[j].x, f[j].y, f[j].z, f[j].w};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          const float2 hf = __bfloat1622float2(h2);
          hi[2 * j + e] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[2 * j + e] = tc::pack_bf16(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
        }
      }
      tmem_st32(row_t + kColQ + 32 * x, hi);
      tmem_st32(row_t + kColQlo + 32 * x, lo);
      const uint4* qr =
          reinterpret_cast<const uint4*>(q_rope + (size_t(pc.s) * H + head) * 64) + 4 * x;
      uint32_t rr[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 u = __ldg(qr + j);
        rr[4 * j] = u.x; rr[4 * j + 1] = u.y; rr[4 * j + 2] = u.z; rr[4 * j + 3] = u.w;
      }
      tmem_st16(row_t + kColQr + 16 * x, rr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(QREADY);
    };

    Piece p, pn;
    int it = 0;
    bool ok = walk.next(p);
    if (ok) write_q(p);
    while (ok) {
      // m: the reference point of the exponentials, in log2 units, the same in
      // both halves of a row.  It is the first tile's max and moves only when a
      // later tile would push P past 2^15 (fp16 keeps it exactly); a stale m
      // only scales all weights alike.  l: this half's sum.
      float m = -INFINITY, l = 0.f;
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int sb = it % kNS, st = it % NST;
        bool good = wait_bar(SFULL(sb), (it / kNS) & 1, abort_flag, err);
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
        // The scores are done with the tile: its latent boxes are converted to
        // fp16 (row r: box r / 64, token row r % 64; this thread takes pieces
        // 4x..4x+3 in swizzled order, so a quarter-warp touches different bank
        // groups).  Rows past the valid tokens are written as zeros here too,
        // so they never depend on which copy of the row this thread reads.
        auto convert = [&]() {
          uint4* row = reinterpret_cast<uint4*>(stages + st * STAGE + (r >> 6) * kBoxBytes +
                                                (r & 63) * 128);
          uint4 w[4];
          if ((r & 63) >= valid) {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = make_uint4(0u, 0u, 0u, 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = row[(4 * x + j) ^ (r & 7)];
          }
          // an fp16 half is inf / NaN iff (h & 0x7fff) + 0x0400 carries into bit 15
          uint32_t over = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w[j]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t h2 =
                  pack_f16(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xffff0000u));
              over |= (h2 & 0x7fff7fffu) + 0x04000400u;
              wv[e] = h2;
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) row[(4 * x + j) ^ (r & 7)] = w[j];
          if ((over & 0x80008000u) != 0) set_error(err, MLRA_ERR_RANGE);
        };
        // The two warps of a quadrant take the conversion and the exponentials
        // in opposite orders, so one uses the conversion path while the other
        // uses the XU pipe (the conversion has no barrier: both still meet the
        // pair's barriers in the same order).
        if (x == 0) convert();
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
        if (x == 1) convert();
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
          const bool g2 = !any || wait_bar(PVDONE(pk % kNS), (pk / kNS) & 1, abort_flag, err);
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
        fence_proxy_async_smem();  // the fp16 tile, for the PV's shared-memory reads
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(PREADY(sb));
      }
      if (!ok) break;
      // every QK of this piece is done: the query columns take the next piece's
      const bool has_next = walk.next(pn);
      if (has_next) write_q(pn);
      // ---- epilogue: o = O / l, lse (this half: O columns 64x..64x+63)
      {
        const int pk = it - 1;
        const bool g = wait_bar(PVDONE(pk % kNS), (pk / kNS) & 1, abort_flag, err);
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
