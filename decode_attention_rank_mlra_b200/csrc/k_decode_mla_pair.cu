// Tensor-core split-KV decode attention for MLA with 128 query heads per
// cluster of two CTAs (sm_100a): the comparison mode of "Multi-Head Low-Rank
// Attention" (Main Findings: MLA caches one 4 d_h latent head, 512 channels
// here, plus the shared RoPE key).
//
// What it computes is the same as the other attention kernels with
// n_blocks = 1: z_t = (q_abs . c[t] + q_rope . k_rope[t]) * scale,
// o = softmax(z) . c, lse = log sum exp z, per head and split.
//
// How.  128 heads x 512 output features in fp32 fill a whole SM's tensor
// memory, so a cluster of two CTAs shares each 64-token tile; CTA r (r = 0, 1)
// holds latent channels [256 r, 256 r + 256) of the tile and of the queries,
// which are at once the K half of the scores it computes and the N half of
// the output it accumulates:
//   S_r = Q[:, half r] C[:, half r]^T + (RoPE K-steps 2r, 2r + 1),
//   S   = S_0 + S_1   (no product is computed twice),
//   O[:, half r] += P C[:, half r].
// CTA r runs the softmax of heads [64 r, 64 r + 64): its "relay" warps (the
// TMEM quadrants of the partner's heads) store those rows of S_r into the
// partner's shared memory; its "own" warps add them to their own rows, take
// the online softmax, write their P rows (fp16) into TMEM over S and into the
// partner's shared memory, where the partner's relay warps move them into its
// TMEM.  Each CTA then multiplies the full P (A, TMEM) by its half of the tile
// (B, shared memory, MN-major).  Messages are bulk copies of each warp's rows
// (2-4 KB, staged in this CTA's shared memory) into the partner's, completing
// on its mbarrier; buffers return by remote arrivals once read.  The rescale
// factors of a moving softmax reference and the final 1 / l travel with the P
// rows.
//
// Precision: queries as fp16 (one row per head, scaled per head by a power of
// two that brings the row's largest magnitude to [2^13, 2^14)), the latent
// tile converted bf16 -> fp16 in place by four converter warps before the
// scores (exact for 2^-17 <= |c| < 65520; larger magnitudes are reported as
// MLRA_ERR_RANGE, and the 64-head MLA kernel launched after this one then
// recomputes the call), fp16 probabilities, fp32 accumulation; the RoPE part stays
// bf16 x bf16 (the query scaled by the same power of two, exactly).
//
// Warps: 0-7 softmax (warp w: TMEM quadrant w & 3, token half w >> 2; "own"
// in quadrants 2, 3, which hold this CTA's heads, "relay" in quadrants 0, 1),
// 8, 9, 12, 13 convert, 10 TMA, 11 MMA.
#include "tc_common.cuh"

#include <cuda_fp16.h>
#include <math.h>

namespace mlra {
namespace tc {
namespace {

using namespace ptx;

constexpr int kThreads = 448;
// Warp w runs on scheduler w % 4.  Each CTA keeps its own heads' rows in TMEM
// lanes 64-127 (quadrants 2, 3), so its softmax exponentials run on schedulers
// 2 and 3; the converters (whose bf16 -> fp16 conversions share the
// exponentials' unit) sit on schedulers 0 and 1 with the relay warps.
constexpr int kWarpTma = 10, kWarpMma = 11;
__device__ __forceinline__ bool is_conv(int w) { return w == 8 || w == 9 || w == 12 || w == 13; }
__device__ __forceinline__ int conv_index(int w) { return (w & 1) + 2 * ((w >> 2) & 1); }
constexpr int kBoxes = 5;                       // 4 latent boxes of this CTA's half + RoPE
constexpr int kStage = kBoxes * kBoxBytes;      // 40 KB
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;                   // fp16 queries, this half: 128 columns
constexpr uint32_t kColS = 128;                 // S partial: 2 x 64 columns
constexpr uint32_t kColO = 256;                 // O, this half's 256 features
constexpr int kQrBytes = 128 * 128;             // RoPE queries (bf16, K-major, 128-B swizzle)
constexpr int kSMsgBytes = 64 * 256;            // the partner's 64 rows of S: [half][row][32] fp32
constexpr int kPMsgBytes = 64 * 128 + 512;      // 64 rows of P: [half][row][32] fp16, then per
                                                // quadrant alpha[32], 1 / l [32]
constexpr float kPMax = 32768.f;                // largest P kept before a rescale (fp16)
// barriers
constexpr int kBFull = 0, kBConv = 3, kBEmpty = 6, kBSFull = 9, kBSMsgF = 11, kBSMsgE = 13,
              kBPMsgF = 15, kBPMsgE = 17, kBPReady = 19, kBPvDone = 21, kBQReady = 23,
              kBDrain = 24, kBars = 25;
constexpr int kOffStages = 0;
constexpr int kOffQr = kOffStages + kStages * kStage;
constexpr int kOffSMsg = kOffQr + kQrBytes;
constexpr int kOffSStage = kOffSMsg + 2 * kSMsgBytes;  // S rows to send: 4 warps x 4 KB
constexpr int kOffPMsg = kOffSStage + kSMsgBytes;        // P rows received
constexpr int kOffPOut = kOffPMsg + 2 * kPMsgBytes;      // P rows to send
constexpr int kOffBars = kOffPOut + 2 * kPMsgBytes;
constexpr int kOffMisc = kOffBars + kBars * 8;
constexpr int kSmem = 1024 + kOffMisc + 64 + 4 * 128 * 4;
static_assert(kSmem <= kSmemLimit, "shared memory");
static_assert(kOffQr % 1024 == 0, "swizzled operands need 1 KB alignment");

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low 16 bits)
  return *reinterpret_cast<uint32_t*>(&v);
}

// Bounded wait on a barrier whose phases other CTAs complete (acquire at
// cluster scope); false on timeout (error recorded) or abort.
__device__ __forceinline__ bool wait_cl(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        int32_t* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      set_error(err, MLRA_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// The same wait for a whole (converged) warp: every lane tests, every lane
// gets the same answer.
__device__ __forceinline__ bool wait_cl_warp(uint32_t bar, uint32_t parity,
                                             volatile int* abort_flag, int32_t* err) {
  const bool good = wait_cl(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, good);
}

// Row r of a 128-byte-swizzled K-major operand: 16-byte unit u at u ^ (r & 7).
__device__ __forceinline__ uint32_t sw128(uint32_t base, int r, int u) {
  return base + uint32_t(r) * 128u + uint32_t((u ^ (r & 7)) << 4);
}
// S message: token half x of row r (32 fp32 = 8 units of 16 bytes), unit u
// at u ^ (r & 7).
__device__ __forceinline__ uint32_t smsg_at(uint32_t base, int x, int r, int u) {
  return base + uint32_t(x) * 8192u + uint32_t(r) * 128u + uint32_t((u ^ (r & 7)) << 4);
}
// P message: token half x of row r (32 fp16 = 4 units), unit u at u ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t pmsg_at(uint32_t base, int x, int r, int u) {
  return base + uint32_t(x) * 4096u + uint32_t(r) * 64u + uint32_t((u ^ ((r >> 1) & 3)) << 4);
}
__global__ void __launch_bounds__(kThreads, 1)
    decode_mla_pair_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem + kOffStages;
  const uint32_t s_base = smem_addr(smem);
  const uint32_t qr_s = s_base + kOffQr;
  auto SMSG = [&](int i) { return s_base + kOffSMsg + uint32_t(i) * kSMsgBytes; };
  auto PMSG = [&](int i) { return s_base + kOffPMsg + uint32_t(i) * kPMsgBytes; };
  auto POUT = [&](int i) { return s_base + kOffPOut + uint32_t(i) * kPMsgBytes; };
  const uint32_t sstage = s_base + kOffSStage;
  const uint32_t bar0 = s_base + kOffBars;
  auto BAR = [&](int i) { return bar0 + 8u * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* xch = reinterpret_cast<float*>(smem + kOffMisc + 64);  // [2 maxima | 2 sums][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = int(cluster_rank());
  const uint32_t peer = uint32_t(rank ^ 1);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(a.ws);
  int32_t* err = &hdr->error;

  // this CTA's share of the tile stream (both CTAs of a cluster walk the same one)
  const char* wsc = static_cast<const char*>(a.ws);
  const int H = a.cfg.n_heads;
  const int cl = blockIdx.x >> 1;
  const int grp = cl / a.ctas_per_group;
  const int c = cl % a.ctas_per_group;
  const int head0 = grp * 128;
  __shared__ int plan_sm[12], scan_sm[kThreads / 32 + 1];
  plan_first_pieces<kThreads>(a.seqlens, a.batch, a.cap, a.ctas_per_group, c, plan_sm, scan_sm);
  const int total = plan_sm[0], share = plan_sm[1];
  const int g_begin = c * share, g_end = min(total, (c + 1) * share);
  const int n_my = max(0, g_end - g_begin);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(BAR(kBFull + i), 1);
      mbar_init(BAR(kBConv + i), 4);
      mbar_init(BAR(kBEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(kBSFull + i), 1);
      mbar_init(BAR(kBSMsgF + i), 1);   // armed with the bytes of the partner's copies
      mbar_init(BAR(kBSMsgE + i), 4);   // the partner's 4 own warps
      mbar_init(BAR(kBPMsgF + i), 1);   // armed with the bytes of the partner's copies
      mbar_init(BAR(kBPMsgE + i), 4);   // the partner's 4 relay warps
      mbar_init(BAR(kBPReady + i), 8);
      mbar_init(BAR(kBPvDone + i), 1);
    }
    mbar_init(BAR(kBQReady), 8);
    mbar_init(BAR(kBDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
    // the first two messages of each kind may come as soon as the partner starts
    for (int i = 0; i < 2 && i < n_my; ++i) {
      mbar_arrive_expect_tx(BAR(kBSMsgF + i), kSMsgBytes);
      mbar_arrive_expect_tx(BAR(kBPMsgF + i), kPMsgBytes);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_addr(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();

  Walker walk{reinterpret_cast<const int32_t*>(wsc + a.L.tile_off),
              reinterpret_cast<const int32_t*>(wsc + a.L.slot_off),
              a.seqlens, plan_sm + 2, a.batch, a.cap, g_begin, g_end};

  if (warp == kWarpTma) {
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
          if (!wait_bar(BAR(kBEmpty + st), ((it / kStages) & 1) ^ 1, abort_flag, err)) {
            ok = false;
            break;
          }
          int row;
          if (a.page_table) {
            const int pg = __ldg(a.page_table + size_t(p.s) * a.max_pages + t);
            if (pg < 0 || pg >= a.num_pages) {
              set_error(err, MLRA_ERR_BAD_PAGE);
              row = -2 * kTile;  // out of bounds: the boxes are zero-filled
            } else {
              row = pg * kPageSize;
            }
          } else {
            row = p.s * a.max_pages + t * kTile;
          }
          if (it == a.stall_tile && blockIdx.x == 0) continue;  // failure-path test only
          mbar_arrive_expect_tx(BAR(kBFull + st), kStage);
          const uint32_t dst = smem_addr(stages + st * kStage);
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_2d_hint(dst + bx * kBoxBytes, &tmap, 256 * rank + bx * kBoxCols, row,
                             BAR(kBFull + st), evict_first);
          tma_load_2d_hint(dst + 4 * kBoxBytes, &tmap, 512, row, BAR(kBFull + st), evict_first);
        }
      }
      if (!ok) {
        for (int j = 0; j < kStages; ++j) {
          const int k = it - 1 - j;
          if (k < 0) break;
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(BAR(kBFull + k % kStages), (k / kStages) & 1) &&
                 globaltimer() - t0 < 10000000ull) {}
        }
      }
    }
  } else if (is_conv(warp)) {
    // ------------------------------------------------------------ converters
    // Each tile's four latent boxes bf16 -> fp16 in place (16-byte chunks, any
    // order); rows past the valid tokens (latent and RoPE) become zeros, so
    // they never depend on what the cache holds there.
    const int ct = 32 * conv_index(warp) + lane;  // 0..127
    Piece p;
    int it = 0;
    bool ok = true;
    while (ok && walk.next(p)) {
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % kStages;
        if (!wait_bar_warp(BAR(kBFull + st), (it / kStages) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        const int valid = min(kTile, p.L - t * kTile);
        const uint32_t base = smem_addr(stages + st * kStage);
        const uint32_t over = convert_stage<4 * 512, 128>(base, ct, valid);
        if (valid < kTile) zero_box_rows<128>(base + 4 * kBoxBytes, ct, valid);
        if ((over & 0x80008000u) != 0) set_error(err, MLRA_ERR_RANGE);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(kBConv + st));
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    //  QK : S_r = Q_half . C_half^T (16 MMAs, A fp16 in TMEM, B the converted
    //       boxes K-major) + this CTA's two RoPE K-steps (bf16, A in shared memory)
    //  PV : O_half += P . C_half (8 MMAs of N = 128, A = P fp16 in TMEM over S)
    // S(k + 2) overwrites P(k): PV(k) is issued before QK(k + 2) and tensor
    // operations run in issue order, so no barrier guards the buffer.
    constexpr uint32_t kIdQK = idesc_f16_f32(128, kTile, false, false);
    constexpr uint32_t kIdQR = idesc_bf16_f32(128, kTile, false, false);
    constexpr uint32_t kIdPV = idesc_f16_f32(128, 128, false, true);
    const uint32_t sbase0 = smem_addr(stages);
    const uint64_t dK = smem_desc(sbase0, 16, 1024, kSwizzle128B);
    const uint64_t dMN = smem_desc(sbase0, kBoxBytes, 1024, kSwizzle128B);
    const uint64_t dQr = smem_desc(qr_s, 16, 1024, kSwizzle128B);
    Piece p;
    int it = 0, piece = 0;
    int prev = -1;
    bool prev_first = false;
    bool ok = true;
    auto issue_pv = [&]() -> bool {
      const int pb = prev & 1;
      if (!wait_bar_warp(BAR(kBPReady + pb), (prev >> 1) & 1, abort_flag, err)) return false;
      tc_fence_after();
      const int st = prev % kStages;
      const uint64_t dv = dMN + uint64_t((st * kStage) >> 4);
      const uint32_t a_p = tmem + kColS + 64 * pb;
#pragma unroll
      for (int hq = 0; hq < 2; ++hq)
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)
          mma_ts_warp(tmem + kColO + 128 * hq, a_p + 8 * k,
                      dv + uint64_t((2 * hq * kBoxBytes + k * 16 * 128) >> 4), kIdPV,
                      (prev_first && k == 0) ? 0u : 1u, 0u, 0u, 0u, 0u);
      mma_commit_warp(BAR(kBEmpty + st));
      mma_commit_warp(BAR(kBPvDone + pb));
      prev = -1;
      return true;
    };
    while (ok && walk.next(p)) {
      if (!wait_bar_warp(BAR(kBQReady), piece & 1, abort_flag, err)) { ok = false; break; }
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int st = it % kStages, sb = it & 1;
        if (!wait_bar_warp(BAR(kBConv + st), (it / kStages) & 1, abort_flag, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t d = dK + uint64_t((st * kStage) >> 4);
        const uint32_t s_acc = tmem + kColS + 64 * sb;
#pragma unroll
        for (int k = 0; k < 16; ++k)
          mma_ts_warp(s_acc, tmem + kColQ + 8 * k,
                      d + uint64_t(((k >> 2) * kBoxBytes + (k & 3) * 32) >> 4), kIdQK,
                      k > 0 ? 1u : 0u, 0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int kk = 2 * rank + j;
          mma_ss_warp(s_acc, dQr + uint64_t((kk * 32) >> 4),
                      d + uint64_t((4 * kBoxBytes + kk * 32) >> 4), kIdQR, 1u);
        }
        mma_commit_warp(BAR(kBSFull + sb));
        if (prev >= 0 && !issue_pv()) { ok = false; break; }
        prev = it;
        prev_first = (t == p.t0);
      }
      if (ok && prev >= 0 && !issue_pv()) ok = false;
      ++piece;
    }
    if (!ok) {
      mma_commit_warp(BAR(kBDrain));
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(BAR(kBDrain), 0) && globaltimer() - t0 < 10000000ull) {}
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int qd = warp & 3, x = warp >> 2;
    // TMEM lane r holds head (r + 64 (1 - rank)) mod 128 of the group: this
    // CTA's own heads in lanes 64-127, the partner's in lanes 0-63
    const bool own = (qd >> 1) == 1;
    const int r = 32 * qd + lane;         // TMEM lane = MMA row
    const int rl = r & 63;                // row within the 64 heads of one CTA
    const int head = head0 + ((r + 64 * (1 - rank)) & 127);
    const int pid = 1 + qd;               // named barrier of the quadrant's two warps
    const uint32_t row_t = tmem + (uint32_t(32 * qd) << 16);
    const float sl2_base = a.cfg.softmax_scale * 1.4426950408889634f;
    float* o_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.o_part);
    float* lse_part = reinterpret_cast<float*>(static_cast<char*>(a.ws) + a.L.lse_part);
    const unsigned short* q_rope = static_cast<const unsigned short*>(a.q_rope);
    float* mx_sm = xch;
    float* lx_sm = xch + 256;
    auto pair_fail = [&](bool good) { return bar_red_or(pid, 64, !good); };
    const uint32_t peer_smsg0 = dsmem_addr(SMSG(0), peer);
    const uint32_t peer_pmsg0 = dsmem_addr(PMSG(0), peer);
    const uint32_t peer_smsgf0 = dsmem_addr(BAR(kBSMsgF), peer);
    const uint32_t peer_smsge0 = dsmem_addr(BAR(kBSMsgE), peer);
    const uint32_t peer_pmsgf0 = dsmem_addr(BAR(kBPMsgF), peer);
    const uint32_t peer_pmsge0 = dsmem_addr(BAR(kBPMsgE), peer);
    const bool arm_s = own && x == 0 && (qd & 1) == 0 && lane == 0;   // one thread per CTA
    const bool arm_p = !own && x == 0 && (qd & 1) == 0 && lane == 0;

    // The queries of piece pc into TMEM (this CTA's 256 channels as fp16, half
    // x of them) and shared memory (the RoPE query, half x of its 64 channels),
    // both times 2^e, e from the row's largest |q_abs| over all 512 channels
    // (both CTAs find the same e).  Returns 2^-e.
    auto write_q = [&](const Piece& pc) -> float {
      const float4* q = reinterpret_cast<const float4*>(a.q_abs + (size_t(pc.s) * H + head) * 512);
      float mx = 0.f;
#pragma unroll 4
      for (int j = 0; j < 128; ++j) {
        const float4 f = __ldg(q + j);
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
      }
      int e = 0;
      if (mx > 0.f && mx < INFINITY) {
        const int k = int((__float_as_uint(mx) >> 23) & 0xff) - 126;  // mx in [2^(k-1), 2^k)
        e = min(max(14 - k, -100), 100);
      }
      const float sc = __int_as_float((127 + e) << 23);
      const float4* qh = q + 64 * rank + 32 * x;
#pragma unroll 1
      for (int j2 = 0; j2 < 2; ++j2) {
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float4 f = __ldg(qh + 16 * j2 + j);
          w[2 * j] = pack_h2(f.x * sc, f.y * sc);
          w[2 * j + 1] = pack_h2(f.z * sc, f.w * sc);
        }
        tmem_st32(row_t + kColQ + 64 * x + 32 * j2, w);
      }
      const uint4* qr = reinterpret_cast<const uint4*>(q_rope + (size_t(pc.s) * H + head) * 64) + 4 * x;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 u = __ldg(qr + j);
        uint32_t* uv = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)  // bf16 pair times 2^e: exact
          uv[e2] = tc::pack_bf16(__uint_as_float(uv[e2] << 16) * sc,
                                 __uint_as_float(uv[e2] & 0xffff0000u) * sc);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sw128(qr_s, r, 4 * x + j)),
                     "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w)
                     : "memory");
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(kBQReady));
      return 1.f / sc;
    };
    // O rows of this warp (its quadrant, columns 128 x ..) times alpha (the
    // caller has seen the previous PV complete)
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ov[32];
        tmem_ld32(row_t + kColO + 128 * x + 32 * ch, ov);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
        tmem_st32(row_t + kColO + 128 * x + 32 * ch, ov);
      }
      tmem_wait_st();
    };

    // relay: this CTA's partial S rows of the partner's heads, tile itx -> partner
    auto send_s = [&](int itx) -> bool {
      const int sb = itx & 1;
      if (!wait_bar_warp(BAR(kBSFull + sb), (itx >> 1) & 1, abort_flag, err)) return false;
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld32(row_t + kColS + 64 * sb + 32 * x, sv);
      tmem_wait_ld();
      // the staging block is free once the partner has read message itx - 1
      // (its copy has landed: the partner waited for all of its bytes)
      if (itx >= 1) {
        const int pk = itx - 1;
        if (!wait_cl_warp(BAR(kBSMsgE + (pk & 1)), (pk >> 1) & 1, abort_flag, err)) return false;
      }
      const uint32_t stg = sstage + uint32_t(2 * (qd & 1) + x) * 4096u;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                         stg + uint32_t(lane) * 128u + uint32_t((j ^ (lane & 7)) << 4)),
                     "r"(sv[4 * j]), "r"(sv[4 * j + 1]), "r"(sv[4 * j + 2]), "r"(sv[4 * j + 3])
                     : "memory");
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        bulk_copy_to_peer(peer_smsg0 + uint32_t(sb) * kSMsgBytes + uint32_t(x) * 8192u +
                              uint32_t(32 * (qd & 1)) * 128u,
                          stg, 4096u, peer_smsgf0 + 8u * sb);
      return true;
    };
    // relay: the partner's P rows of tile itx for these heads, into TMEM over S
    auto recv_p = [&](int itx, bool last, bool may_rescale, float& inv_l) -> bool {
      const int sb = itx & 1;
      if (!wait_cl_warp(BAR(kBPMsgF + sb), (itx >> 1) & 1, abort_flag, err)) return false;
      if (arm_p && itx + 2 < n_my) mbar_arrive_expect_tx(BAR(kBPMsgF + sb), kPMsgBytes);
      const uint32_t src = PMSG(sb);
      uint32_t pw[16];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(pw[4 * j]), "=r"(pw[4 * j + 1]), "=r"(pw[4 * j + 2]), "=r"(pw[4 * j + 3])
                     : "r"(pmsg_at(src, x, rl, j)));
      const float* side = reinterpret_cast<const float*>(smem + kOffPMsg + sb * kPMsgBytes + 8192) +
                          64 * (qd & 1);
      const float alpha = side[lane];
      if (last) inv_l = side[32 + lane];
      tmem_st16(row_t + kColS + 64 * sb + 16 * x, pw);
      // (the store above and the vote below consume every value read from the
      // message: the buffer may go back to the partner; inv_l is never negative)
      const bool resc = __any_sync(0xffffffffu, alpha != 1.f || inv_l < 0.f);
      if (lane == 0) mbar_arrive_remote(peer_pmsge0 + 8u * sb);  // buffer read
      if (resc && may_rescale) {
        const int pk = itx - 1;
        if (!wait_bar_warp(BAR(kBPvDone + (pk & 1)), (pk >> 1) & 1, abort_flag, err)) return false;
        tc_fence_after();
        rescale_o(alpha);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(kBPReady + sb));
      return true;
    };

    Piece p, pn;
    int it = 0;
    bool ok = walk.next(p);
    float inv_sc = ok ? write_q(p) : 1.f;
    while (ok) {
      float m = -INFINITY, l = 0.f;   // own rows: reference point (log2 units) and sum
      float inv_l = 0.f;
      const float sl2 = sl2_base * inv_sc;
      if (!own && p.t0 < p.t1 && !send_s(it)) { ok = false; break; }
      for (int t = p.t0; t < p.t1; ++t, ++it) {
        const int sb = it & 1;
        const bool last = t + 1 == p.t1;
        const int valid = min(kTile, p.L - t * kTile);
        if (!own) {
          // ---- relay: S of tile it + 1 to the partner ahead of the P of tile it
          if (t + 1 < p.t1 && !send_s(it + 1)) { ok = false; break; }
          if (!recv_p(it, last, t > p.t0, inv_l)) { ok = false; break; }
        } else {
          // ---- own rows: S = S_r + S_(1-r), online softmax, P to TMEM and the partner
          const bool good = wait_bar_warp(BAR(kBSFull + sb), (it >> 1) & 1, abort_flag, err) &&
                            wait_cl_warp(BAR(kBSMsgF + sb), (it >> 1) & 1, abort_flag, err);
          if (pair_fail(good)) { ok = false; break; }
          if (arm_s && it + 2 < n_my) mbar_arrive_expect_tx(BAR(kBSMsgF + sb), kSMsgBytes);
          tc_fence_after();
          float z[32];
          {
            uint32_t sv[32];
            tmem_ld32(row_t + kColS + 64 * sb + 32 * x, sv);
            const uint32_t src = SMSG(sb);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              uint4 u;
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                           : "r"(smsg_at(src, x, rl, j)));
              z[4 * j] = __uint_as_float(u.x);
              z[4 * j + 1] = __uint_as_float(u.y);
              z[4 * j + 2] = __uint_as_float(u.z);
              z[4 * j + 3] = __uint_as_float(u.w);
            }
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) z[k] += __uint_as_float(sv[k]);
          }
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
          auto row_max = [&]() {
            mx_sm[x * 128 + r] = half_max();
            bar_sync(pid, 64);
            return fmaxf(mx_sm[r], mx_sm[128 + r]);
          };
          if (t == p.t0) m = row_max();
          uint32_t pw[16];
          float ls;
          auto exps = [&]() {
            ls = 0.f;
#pragma unroll
            for (int k = 0; k < 32; k += 2) {
              const float p0 = ex2_approx(fmaf(z[k], sl2, -m));
              const float p1 = ex2_approx(fmaf(z[k + 1], sl2, -m));
              ls += p0 + p1;
              pw[k / 2] = pack_h2(p0, p1);
            }
          };
          exps();
          float alpha = 1.f;
          const bool over = bar_red_or(pid, 64, !(ls <= kPMax));
          // (ls, an input of the vote, depends on every value read from the
          // message: the buffer may go back to the partner)
          if (lane == 0) mbar_arrive_remote(peer_smsge0 + 8u * sb);  // message read
          if (over) {
            // rare: a score far above m (or a NaN): raise m to this tile's row
            // max, rescale l and this CTA's O rows of these heads (the partner
            // rescales its own from alpha), redo the tile
            const float mt = row_max();
            if (mt > m) {
              alpha = ex2_approx(m - mt);
              m = mt;
              l *= alpha;
            }
            if (t == p.t0) alpha = 1.f;  // nothing accumulated yet in either CTA
            const bool any = __any_sync(0xffffffffu, alpha != 1.f);
            const int pk = it - 1;
            bool g2 = true;
            if (any) g2 = wait_bar_warp(BAR(kBPvDone + (pk & 1)), (pk >> 1) & 1, abort_flag, err);
            if (pair_fail(g2)) { ok = false; break; }
            if (any) {
              tc_fence_after();
              rescale_o(alpha);
            }
            exps();
          }
          l += ls;
          if (last) {
            lx_sm[x * 128 + r] = l;
            bar_sync(pid, 64);
            const float l_tot = lx_sm[r] + lx_sm[128 + r];
            inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
            if (x == 0)
              lse_part[size_t(p.slot) * H + head] =
                  l_tot > 0.f ? (m + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
          }
          {  // the partner's relay has read P(it - 2): both copies of buffer sb are free
            const bool g3 = wait_cl_warp(BAR(kBPMsgE + sb), ((it >> 1) & 1) ^ 1, abort_flag, err);
            if (pair_fail(g3)) { ok = false; break; }
          }
          const uint32_t pout = POUT(sb);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(pmsg_at(pout, x, rl, j)),
                         "r"(pw[4 * j]), "r"(pw[4 * j + 1]), "r"(pw[4 * j + 2]), "r"(pw[4 * j + 3])
                         : "memory");
          const uint32_t so = pout + 8192u + uint32_t(qd & 1) * 256u;
          if (x == 0) {
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(so + 4u * lane), "r"(__float_as_uint(alpha))
                         : "memory");
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(so + 128u + 4u * lane),
                         "r"(__float_as_uint(inv_l))
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const uint32_t fb = peer_pmsgf0 + 8u * sb;
            const uint32_t off = uint32_t(x) * 4096u + uint32_t(32 * (qd & 1)) * 64u;
            bulk_copy_to_peer(peer_pmsg0 + uint32_t(sb) * kPMsgBytes + off, pout + off, 2048u, fb);
            if (x == 0)
              bulk_copy_to_peer(peer_pmsg0 + uint32_t(sb) * kPMsgBytes + 8192u +
                                    uint32_t(qd & 1) * 256u,
                                so, 256u, fb);
          }
          tmem_st16(row_t + kColS + 64 * sb + 16 * x, pw);  // P over S
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(kBPReady + sb));
        }
      }
      if (!ok) break;
      // every QK of this piece is done: the queries take the next piece's
      const bool has_next = walk.next(pn);
      if (has_next) inv_sc = write_q(pn);
      // ---- epilogue: o = O / l for this CTA's 256 features (half x of them)
      {
        // (own warps leave a failed wait with their quadrant's partner warp:
        // they meet at named barriers; relay warps have none)
        const int pk = it - 1;
        const bool g = wait_bar_warp(BAR(kBPvDone + (pk & 1)), (pk >> 1) & 1, abort_flag, err);
        if (own ? pair_fail(g) : !g) { ok = false; break; }
      }
      tc_fence_after();
      float* dst = o_part + (size_t(p.slot) * H + head) * 512 + 256 * rank + 128 * x;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t ov[32];
        tmem_ld32(row_t + kColO + 128 * x + 32 * ch, ov);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float o8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o8[e] = __uint_as_float(ov[8 * k + e]) * inv_l;
          st_global_v8(dst + 32 * ch + 8 * k, o8);
        }
      }
      if (!has_next) break;
      p = pn;
    }
  }

  tc_fence_before();
  __syncthreads();
  // Both CTAs reach this point after bounded waits only, and no message leaves
  // a CTA after it.  After a failure, copies already on their way into this
  // CTA's shared memory are given a bounded time to land before it exits.
  cluster_sync_all();
  if (*abort_flag) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) {}
  }
  __syncthreads();
  pdl_wait();  // complete only after the plan kernel (whose records the merge reads)
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool mla_pair_supported(const mlra_config_t& c) {
  return c.dtype == MLRA_BF16 && c.n_blocks == 1 && c.d_cb == 512 && c.d_r == 64 &&
         c.n_heads % 128 == 0;
}

// Clusters of two CTAs the device runs at once (every SM pair of a GPC), per
// head group of 128.
int mla_pair_clusters(const mlra_config_t& c, int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int n = (dev >= 0 && dev < 64) ? cached[dev] : 0;
  if (n == 0) {
    n = num_sms / 2;
    if (cudaFuncSetAttribute(decode_mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmem) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(num_sms);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int m = 0;
      if (cudaOccupancyMaxActiveClusters(&m, decode_mla_pair_kernel, &cfg) == cudaSuccess && m > 0)
        n = m < n ? m : n;
    }
    (void)cudaGetLastError();
    if (dev >= 0 && dev < 64) cached[dev] = n;
  }
  const int groups = c.n_heads / 128;
  return n / groups > 0 ? n / groups : 1;
}

cudaError_t launch_decode_mla_pair(const CUtensorMap& map, const DecodeArgs& a, cudaStream_t st) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_mla_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * a.n_groups * a.ctas_per_group);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_mla_pair_kernel, map, a);
}

}  // namespace tc
}  // namespace mlra
