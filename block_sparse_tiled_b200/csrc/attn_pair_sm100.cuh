// Attention of query row blocks that share their key list, two 64-row blocks (128 queries) per work
// item, on sm_100a.
//
// A prefix query tile attends to every key tile ("Mike0021/FastH3-4step-Preview-VSA", section "Video
// Sparse Attention is not optional here": prefix queries attend densely), so any two prefix query row
// blocks of one head share every key block; and with 128-token tiles ("FastH3 OmniRef inference",
// section "Device profiles") the two 64-row halves of a video query tile share that tile's key list.
// This kernel runs such pairs together in the standard orientation
//     S [128 queries x 128 keys] = Q_pair (M = 128, K-major) * K_blk^T (N = 128, K-major)
//     O [128 queries x D]       += P (M = 128, read from TMEM) * V_blk (N = D, MN-major)
// so one tcgen05.mma covers twice the work of the transposed N = 64 form that the other video query
// tiles use (vsa_attn_kernel), and P reaches the tensor core through TMEM: no shared-memory P, no proxy
// fence.  Work item = (b, h, pair j): query row blocks 2j and 2j + 1 of the launch's range [0, r_end)
// (the second one absent when r_end is odd: its rows are computed from zero-filled or neighbouring rows
// and never stored).  Key blocks: for a prefix query tile, row blocks (2n, 2n + 1) of the whole
// sequence, all of them; for a 128-token video query tile, the tiles of its key list (the always-kept
// prefix tiles, then the kept reference and selected video tiles), one tile per block.
//
// The softmax is row-wise: two threads per query row, one per 64-key half of every block, each keeping
// its half-row's sum in registers.  The running maximum follows the lazy rule of vsa_attn_kernel: a
// block is exponentiated against the current row maximum m; the first block of an item takes the exact
// row maximum (the two halves exchange theirs through shared memory), and a later block takes it again
// only when some logit exceeds m by more than kRescaleLog2 (then O and the sums are rescaled).  The
// check of later blocks is skipped for the rest of an item when the first block already shows, by the
// Cauchy-Schwarz bound |q . k| <= |q| max|k|, that no later logit can overflow.
//
// Roles (512 threads, 16 warps):
//   warp 0       Q + K producer (TMA; claims items from the global counter, publishes them in a ring)
//   warp 1       V producer
//   warp 2       S issuer (one thread) and TMEM owner
//   warp 3       P.V issuer (one thread)
//   warps 4..11  softmax: warp w reads TMEM lane quadrant w % 4 (query rows 32 (w % 4) ..) and key half
//                (w - 4) / 4 of every block
//   warps 12..15 epilogue: 1 / l, O from TMEM, the gated compression term, bf16 rows in sequence order
// TMEM (512 columns): S double buffer (2 x 128), O (D columns from 256), P double buffer (2 x 64 columns,
// two bf16 per 32-bit cell, from 384).  Every mbarrier wait is bounded (see ptx.cuh).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_sm100.cuh"

namespace vsa {

constexpr int kPairSoftWarps = 8;
constexpr int kPairEpiWarp0 = 4 + kPairSoftWarps;
constexpr int kPairThreads = 32 * (kPairEpiWarp0 + 4);
constexpr uint32_t kPairS0 = 0, kPairO0 = 256, kPairP0 = 384;  // TMEM columns

template <int D>
struct PairLayout {
  static constexpr int kHalves = (D + 63) / 64;             // 64-column halves of a row (D = 96: two)
  static constexpr int kRowsBytes = kHalves * 128 * 128;    // 128 rows of one operand
  static constexpr int kKStages = 2, kVStages = 3, kRing = 8;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kRowsBytes;
  static constexpr int oV = oK + kKStages * kRowsBytes;
  static constexpr int oBar = oV + kVStages * kRowsBytes;
  static constexpr int bQFull = 0, bQEmpty = 1;
  static constexpr int bKFull = 2, bKEmpty = bKFull + kKStages;
  static constexpr int bVFull = bKEmpty + kKStages, bVEmpty = bVFull + kVStages;
  static constexpr int bSFull = bVEmpty + kVStages, bSEmpty = bSFull + 2;
  static constexpr int bPFull = bSEmpty + 2, bPEmpty = bPFull + 2;
  static constexpr int bOFull = bPEmpty + 2, bOEmpty = bOFull + 1;
  static constexpr int bLFull = bOEmpty + 1;
  static constexpr int bRFull = bLFull + 2, bREmpty = bRFull + kRing;
  static constexpr int bDoneS = bREmpty + kRing, bDonePV = bDoneS + 1;
  static constexpr int kNumBars = bDonePV + 1;
  static constexpr int oMisc = oBar + kNumBars * 8;            // tmem base, abort flag
  static constexpr int oRing = ((oMisc + 8 + 15) / 16) * 16;   // int ring[kRing]
  static constexpr int oRed = oRing + kRing * 4;               // float red[2 halves][128 rows]
  static constexpr int oLsum = oRed + 1024;                    // float lsum[2 items][2 halves][128 rows]
  static constexpr int oEnd = oLsum + 2048;
  static size_t bytes() { return 1024 /*alignment slack*/ + oEnd; }
};

// a.s_lo, a.r_end: the launch's query row blocks [r_lo, r_end) (the prefix row blocks; with 128-token
// tiles any tile-aligned range); a.n_s: pairs per (b, h); the other fields as for vsa_attn_kernel
// (tile-order inputs).  kF8: Q and K are 8-bit E4M3 code rows (128 bytes whatever D) with one scale per
// row (a.q_scale, a.k_scale); S is then a kind::f8f6f4 product (32 codes per K-step) of the codes, and the
// softmax multiplies each logit by its key row's scale and its query row's scale (times the softmax
// scale) before the exponent; P.V stays bf16 ("FastH3 OmniRef inference", section "Device profiles":
// 8-bit Q/K for the dense prefix query tiles, bf16 P.V).
template <int D, bool kF8 = false>
__global__ void __launch_bounds__(kPairThreads, 1)
    vsa_attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using Ly = PairLayout<D>;
  constexpr int kQKSteps = kF8 ? (D + 31) / 32 : D / 16;
  constexpr int kQKHalves = kF8 ? 1 : Ly::kHalves;                  // 8 KB boxes per 64 rows of Q or K
  constexpr uint32_t kQKRowsBytes = kQKHalves * 128 * 128;           // bytes of 128 rows of Q or K
  constexpr int kPVSteps = 128 / 16;
  constexpr uint32_t kIdescS = kF8 ? umma_idesc_e4m3(128, 128) : umma_idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kIdescPV = umma_idesc_bf16(128, D, 0, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::oBar);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::oMisc + 4);
  int* ring_s = reinterpret_cast<int*>(sm + Ly::oRing);
  float* red_s = reinterpret_cast<float*>(sm + Ly::oRed);
  float* lsum_s = reinterpret_cast<float*>(sm + Ly::oLsum);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_t = a.n_t, sh = a.sub_shift, n_sel = n_t >> sh;
  const int r_lo = a.s_lo, r_end = a.r_end;  // query row blocks of the launch: [r_lo, r_end), in pairs
  const int npairs = a.n_s;                  // items per (b, h)
  const int P = a.P, V = n_sel - P, E = a.n_exempt, W = a.kr + a.topk;
  // Key blocks of the item whose first query row block is s0: for a prefix query tile every row block,
  // two at a time; for a video query tile of 128 tokens (sh = 1; both row blocks are that tile) the E
  // always-kept and the kr + topk listed tiles, one 128-key block each.
  auto item_blocks = [&](int s0) -> int { return ((s0 >> sh) < P) ? (n_t + 1) / 2 : E + W; };
  // first key row block of block n; the block's second half is the next row block (or, past the last
  // row block, a masked repeat)
  auto block_row = [&](int64_t bh, int s0, int n) -> int {
    const int i = s0 >> sh;
    if (i < P) return 2 * n;
    const int sel = (n < E) ? (a.exempt ? __ldg(a.exempt + n) : n) : __ldg(a.idx + (bh * V + (i - P)) * W + (n - E));
    return sel << 1;
  };
  const WaitCtl ctl{abort_flag, a.status, kWaitTimeoutNs};

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(&bars[Ly::bQFull], 1);
    mbar_init(&bars[Ly::bQEmpty], 1);
    for (int s = 0; s < Ly::kKStages; ++s) {
      mbar_init(&bars[Ly::bKFull + s], 1);
      mbar_init(&bars[Ly::bKEmpty + s], 1);
    }
    for (int s = 0; s < Ly::kVStages; ++s) {
      mbar_init(&bars[Ly::bVFull + s], 1);
      mbar_init(&bars[Ly::bVEmpty + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[Ly::bSFull + s], 1);
      mbar_init(&bars[Ly::bSEmpty + s], kPairSoftWarps * 32);  // every softmax thread arrives
      mbar_init(&bars[Ly::bPFull + s], kPairSoftWarps * 32);
      mbar_init(&bars[Ly::bPEmpty + s], 1);
      mbar_init(&bars[Ly::bLFull + s], kPairSoftWarps);
    }
    mbar_init(&bars[Ly::bOFull], 1);
    mbar_init(&bars[Ly::bOEmpty], 4);
    for (int s = 0; s < Ly::kRing; ++s) {
      mbar_init(&bars[Ly::bRFull + s], 1);
      mbar_init(&bars[Ly::bREmpty + s], 3 + kPairSoftWarps + 4);  // V producer, two issuers, softmax, epilogue
    }
    mbar_init(&bars[Ly::bDoneS], 1);
    mbar_init(&bars[Ly::bDonePV], 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 2) {
    tmem_alloc(tmem_base_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  // claimed item it of this CTA (-1: none left), read by one thread of a consumer warp
  auto ring_take = [&](int it, int site) -> int {
    const int slot = it % Ly::kRing;
    const bool ok = mbar_wait(&bars[Ly::bRFull + slot], (it / Ly::kRing) & 1, ctl, site);
    const int w = ok ? ring_s[slot] : -1;
    mbar_arrive(&bars[Ly::bREmpty + slot]);
    return w;
  };

  if (warp <= 1) {
    // ============================================================ TMA producers (warp 0: Q + K, warp 1: V)
    const bool is_k = (warp == 0);
    const int nstages = is_k ? Ly::kKStages : Ly::kVStages;
    const int b_full = is_k ? Ly::bKFull : Ly::bVFull;
    const int b_empty = is_k ? Ly::bKEmpty : Ly::bVEmpty;
    uint8_t* ring = sm + (is_k ? Ly::oK : Ly::oV);
    const void* tmap = is_k ? static_cast<const void*>(&tm_k) : static_cast<const void*>(&tm_v);
    uint32_t g = 0;
    int it = 0, pub = 0;
    bool ok = true, more = true;
    // lane 0 of the K producer claims items two ahead of its own use (item = (b*H + h) * npairs + j)
    auto publish_next = [&]() {
      if (!more) return;
      const int slot = pub % Ly::kRing;
      if (!mbar_wait(&bars[Ly::bREmpty + slot], ((pub / Ly::kRing) & 1) ^ 1, ctl, 44)) {
        more = false;
        return;
      }
      const int claimed = atomicAdd(a.sched, 1);
      const int v = (claimed < a.n_items) ? claimed : -1;
      ring_s[slot] = v;
      mbar_arrive(&bars[Ly::bRFull + slot]);
      ++pub;
      if (v < 0) more = false;
    };
    if (is_k && lane == 0) {
      publish_next();
      publish_next();
    }
    for (;; ++it) {
      int w = -1;
      if (lane == 0) {
        if (is_k) {
          w = (it < pub) ? ring_s[it % Ly::kRing] : -1;
          publish_next();
        } else {
          w = ring_take(it, 45);
        }
      }
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w < 0 || !ok) break;
      const int64_t bh = w / npairs;
      const int s0 = r_lo + 2 * static_cast<int>(w - bh * npairs);
      if (is_k) {
        // the item's 128 query rows: row blocks s0 and s0 + 1 (rows past the tensor read as zeros)
        if (lane == 0) {
          ok = mbar_wait(&bars[Ly::bQEmpty], (it & 1) ^ 1, ctl, 31);
          if (ok) mbar_arrive_expect_tx(&bars[Ly::bQFull], kQKRowsBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok && lane < 2 * kQKHalves) {
          const int hh = lane >> 1, second = lane & 1;
          const int row = static_cast<int>((bh * n_t + s0 + second) * 64);
          tma_load_2d(sm + Ly::oQ + hh * 16384 + second * 8192, &tm_q, &bars[Ly::bQFull], hh * 64, row);
        }
        __syncwarp();
      }
      const int nb = item_blocks(s0);
      int rows = 0;  // lane j: the first key row block of block 32 * (n / 32) + j
      for (int n = 0; n < nb && ok; ++n, ++g) {
        if ((n & 31) == 0) rows = (n + lane < nb) ? block_row(bh, s0, n + lane) : 0;
        const int ka = __shfl_sync(0xffffffffu, rows, n & 31);
        const int kb = (ka + 1 < n_t) ? ka + 1 : ka;  // past the last row block: a masked repeat
        const int st = g % nstages;
        const uint32_t u = g / nstages;
        if (lane == 0) {
          ok = mbar_wait(&bars[b_empty + st], (u & 1) ^ 1, ctl, is_k ? 32 : 33);
          if (ok) mbar_arrive_expect_tx(&bars[b_full + st], is_k ? kQKRowsBytes : Ly::kRowsBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane < 2 * (is_k ? kQKHalves : Ly::kHalves)) {
          const int hh = lane >> 1, second = lane & 1;
          const int row = static_cast<int>((bh * n_t + (second ? kb : ka)) * 64);
          tma_load_2d(ring + st * Ly::kRowsBytes + hh * 16384 + second * 8192, tmap, &bars[b_full + st], hh * 64,
                      row);
        }
        __syncwarp();
      }
    }
    // drain: every load this warp issued must land before the CTA exits
    if (lane == 0) {
      const WaitCtl drain{abort_flag, a.status, kWaitTimeoutNs};
      for (int s = 0; s < nstages && static_cast<uint32_t>(s) < g; ++s) {
        const uint32_t last = g - 1 - s;
        mbar_wait_drain(&bars[b_full + (last % nstages)], (last / nstages) & 1, drain, 40);
      }
      if (is_k && it > 0) mbar_wait_drain(&bars[Ly::bQFull], (it - 1) & 1, drain, 41);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ============================================================ S issuer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int it = 0;; ++it) {
        const int w = ring_take(it, 46);
        if (w < 0 || !ok) break;
        const int64_t bh = w / npairs;
        const int nb = item_blocks(r_lo + 2 * static_cast<int>(w - bh * npairs));
        ok = mbar_wait(&bars[Ly::bQFull], it & 1, ctl, 34);
        const uint64_t qd0 = umma_desc_sw128(smem_u32(sm + Ly::oQ), 16, 1024);
        for (int n = 0; n < nb && ok; ++n, ++g) {
          const int kst = g % Ly::kKStages;
          const int sb = g & 1;
          ok = mbar_wait(&bars[Ly::bKFull + kst], (g / Ly::kKStages) & 1, ctl, 35);
          ok = ok && mbar_wait(&bars[Ly::bSEmpty + sb], ((g >> 1) & 1) ^ 1, ctl, 36);
          if (!ok) break;
          tc_fence_after();
          const uint64_t bd0 = umma_desc_sw128(smem_u32(sm + Ly::oK + kst * Ly::kRowsBytes), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kQKSteps; ++kk) {
            // 16 elements (32 bytes) of every row per step, the next 64-column half every 4 steps
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
            if constexpr (kF8)
              umma_ss_f8(tmem + kPairS0 + sb * 128, qd0 + off, bd0 + off, kIdescS, kk > 0 ? 1u : 0u);
            else
              umma_ss(tmem + kPairS0 + sb * 128, qd0 + off, bd0 + off, kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[Ly::bKEmpty + kst]);
          umma_commit(&bars[Ly::bSFull + sb]);
          if (n == nb - 1) umma_commit(&bars[Ly::bQEmpty]);
        }
      }
      umma_commit(&bars[Ly::bDoneS]);
      mbar_wait_drain(&bars[Ly::bDoneS], 0, ctl, 42);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ============================================================ P.V issuer
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int it = 0;; ++it) {
        const int w = ring_take(it, 47);
        if (w < 0 || !ok) break;
        const int64_t bh = w / npairs;
        const int nb = item_blocks(r_lo + 2 * static_cast<int>(w - bh * npairs));
        for (int n = 0; n < nb && ok; ++n, ++g) {
          const int vst = g % Ly::kVStages;
          const int pb = g & 1;
          ok = mbar_wait(&bars[Ly::bVFull + vst], (g / Ly::kVStages) & 1, ctl, 37);
          ok = ok && mbar_wait(&bars[Ly::bPFull + pb], (g >> 1) & 1, ctl, 38);
          ok = ok && (n > 0 || mbar_wait(&bars[Ly::bOEmpty], (it & 1) ^ 1, ctl, 39));
          if (!ok) break;
          tc_fence_after();
          // V [keys x d] in 64-column halves: d contiguous (MN-major B), halves 16 KB apart, 8-key groups
          // 1 KB apart; a K-step is 16 keys = 2 KB further
          const uint64_t bd0 = umma_desc_sw128(smem_u32(sm + Ly::oV + vst * Ly::kRowsBytes), 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < kPVSteps; ++kk) {
            umma_ts(tmem + kPairO0, tmem + kPairP0 + pb * 64 + kk * 8, bd0 + static_cast<uint64_t>(kk * 128),
                    kIdescPV, (n > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars[Ly::bVEmpty + vst]);
          umma_commit(&bars[Ly::bPEmpty + pb]);
          if (n == nb - 1) umma_commit(&bars[Ly::bOFull]);
        }
      }
      umma_commit(&bars[Ly::bDonePV]);
      mbar_wait_drain(&bars[Ly::bDonePV], 0, ctl, 43);
    }
    __syncwarp();
  } else if (warp < kPairEpiWarp0) {
    // ============================================================ softmax
    const int qd = warp & 3;
    const int hf = (warp - 4) >> 2;          // key half of every block
    const int r = qd * 32 + lane;            // query row of the pair (TMEM lane)
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const float cl = a.scale_log2;
    uint32_t g = 0;
    for (int it = 0;; ++it) {
      int w = (lane == 0) ? ring_take(it, 48) : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (named_bar_or(1, 256, w < 0)) break;  // the softmax warps stop together
      const int64_t bh = w / npairs;
      const int s0 = r_lo + 2 * static_cast<int>(w - bh * npairs);
      const int s = s0 + (r >> 6);             // this row's query row block
      const bool row_ok = s < r_end;
      const int nb = item_blocks(s0);
      // overflow bound of this row: cl |q| max|k| + ceil(log2 max|v|)+ - skip_cap (rows not stored: none)
      float lim = -INFINITY;
      if (a.q_norm != nullptr && row_ok) {
        const float qn = __ldg(a.q_norm + (bh * n_t + s) * 64 + (r & 63));
        const float kmax = __ldg(a.kv_max + 2 * bh), vmax = __ldg(a.kv_max + 2 * bh + 1);
        const int ev = max(0, static_cast<int>((__float_as_uint(vmax) >> 23) & 0xffu) - 126);
        lim = cl * qn * kmax + static_cast<float>(ev) - a.skip_cap;
      }
      // the factor that turns this row's raw scores into log2 units: cl, or with 8-bit Q/K the row's scale
      // times cl (each key's scale is applied to its column first)
      float xs = cl;
      if constexpr (kF8) xs = row_ok ? __ldg(a.q_scale + (bh * n_t + s) * 64 + (r & 63)) * cl : 0.0f;
      float m = 0.0f;        // running row maximum, log2 units
      float lacc[8];         // partial sums of this half-row
#pragma unroll
      for (int j = 0; j < 8; ++j) lacc[j] = 0.0f;
      bool skip = false;
      uint32_t mlo = 0, mhi = 0;  // lane j: the key-mask word of this half of block 32 * (n / 32) + j
      [[maybe_unused]] int kro = 0;  // 8-bit Q/K: lane j, that half's first key-scale index (b, h, block) * 64
      for (int n = 0; n < nb; ++n, ++g) {
        const int sb = g & 1;
        if ((n & 31) == 0) {
          uint64_t m = 0ull;
          if (n + lane < nb) {
            const int kt = block_row(bh, s0, n + lane) + hf;  // key row block of this half
            m = (kt < n_t) ? __ldg(a.key_mask + kt) : 0ull;
            if constexpr (kF8) kro = static_cast<int>((bh * n_t + min(kt, n_t - 1)) * 64);
          }
          mlo = static_cast<uint32_t>(m);
          mhi = static_cast<uint32_t>(m >> 32);
        }
        const uint64_t kmask = static_cast<uint64_t>(__shfl_sync(0xffffffffu, mlo, n & 31)) |
                               (static_cast<uint64_t>(__shfl_sync(0xffffffffu, mhi, n & 31)) << 32);
        // 8-bit Q/K: scale column j of chunk c by its key's scale (the same addresses in every lane); the
        // 32 scales of a chunk are loaded before its S columns are waited for, so their latency overlaps
        [[maybe_unused]] const float* ksc = nullptr;
        if constexpr (kF8) ksc = a.k_scale + __shfl_sync(0xffffffffu, kro, n & 31);
        [[maybe_unused]] float4 k4[4];
        [[maybe_unused]] int kc = 0;
        auto load_ks = [&](int c) {  // the chunk's first 16 scales
          if constexpr (kF8) {
            kc = c;
#pragma unroll
            for (int j = 0; j < 4; ++j) k4[j] = __ldg(reinterpret_cast<const float4*>(ksc + c) + j);
          }
        };
        auto key_scale = [&](float* x) {
          if constexpr (kF8) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 k = j < 4 ? k4[j] : __ldg(reinterpret_cast<const float4*>(ksc + kc) + j);
              mul2(x[4 * j], x[4 * j + 1], x[4 * j], x[4 * j + 1], k.x, k.y);
              mul2(x[4 * j + 2], x[4 * j + 3], x[4 * j + 2], x[4 * j + 3], k.z, k.w);
            }
          }
        };
        const uint32_t s_col = t_lane + kPairS0 + sb * 128 + 64 * hf;
        mbar_wait(&bars[Ly::bSFull + sb], (g >> 1) & 1, ctl, 50);
        tc_fence_after();
        // the half-row's largest logit (log2 units, less m), read first when this block may rescale:
        // fl(s * xs - m) is monotone in s (xs >= 0), so the largest scaled score gives it
        bool slow = (n == 0);
        float t = -INFINITY;
        if (n == 0 || !skip) {
          float smax = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; c += 32) {
            float x[32];
            load_ks(c);
            tmem_ld32(s_col + c, x);
            tmem_wait_ld();
            key_scale(x);
            if (kmask != ~0ull) {  // the same word in every lane of the warp
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (!((kmask >> (c + j)) & 1ull)) x[j] = -INFINITY;
            }
#pragma unroll
            for (int j = 0; j < 32; j += 2) smax = max3(smax, x[j], x[j + 1]);
          }
          t = (smax == -INFINITY) ? -INFINITY : fmaf(smax, xs, -m);
          if (n > 0) slow = named_bar_or(1, 256, t > kRescaleLog2);
        }
        float d = 0.0f;  // the increase of m in this block
        if (slow) {
          // exact row maximum of this block over both halves; raise m by it
          red_s[hf * 128 + r] = t;
          named_bar_sync(2, 256);
          const float c = fmaxf(red_s[r], red_s[128 + r]);
          if (n == 0) {
            d = (c == -INFINITY) ? 0.0f : c;
            m = d;
            // no later block can overflow when every row's bound is within reach of its first maximum
            skip = (a.q_norm != nullptr) && !named_bar_or(1, 256, !(lim <= d));
          } else {
            d = fmaxf(c, 0.0f);
            m += d;
            named_bar_sync(2, 256);  // red_s read by both halves before a later block rewrites it
          }
          if (n > 0) {
            // d differs from row to row, so every lane takes this path (a factor of 1 where d = 0): the
            // TMEM loads and stores below are warp-collective
            const float f = ex2_approx(-d);
#pragma unroll
            for (int j = 0; j < 8; ++j) lacc[j] *= f;
            // O holds blocks < n of this item: wait for the last P.V, then rescale this half-row's columns
            const uint32_t gp = g - 1;
            mbar_wait(&bars[Ly::bPEmpty + (gp & 1)], (gp >> 1) & 1, ctl, 51);
            tc_fence_after();
            constexpr int kHalfD = D / 2;  // 32, 48 or 64 columns of O per thread
#pragma unroll
            for (int c0 = 0; c0 < kHalfD; c0 += 16) {
              float o[16];
              tmem_ld16(t_lane + kPairO0 + hf * kHalfD + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] *= f;
              tmem_st16(t_lane + kPairO0 + hf * kHalfD + c0, o);
            }
            tmem_wait_st();
            tc_fence_before();
          }
        }
        // probabilities against the (new) m, partial row sums, P (bf16 pairs) into TMEM, 32 keys at a time
        const int pb = g & 1;
        mbar_wait(&bars[Ly::bPEmpty + pb], ((g >> 1) & 1) ^ 1, ctl, 52);
        tc_fence_after();
        const float nm = -m;
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          float x[32];
          load_ks(c);
          tmem_ld32(s_col + c, x);
          tmem_wait_ld();
          if (c == 32) {  // S^T of this block fully read
            tc_fence_before();
            mbar_arrive(&bars[Ly::bSEmpty + sb]);
          }
          key_scale(x);
#pragma unroll
          for (int j = 0; j < 32; j += 2) fma2(x[j], x[j + 1], x[j], x[j + 1], xs, xs, nm, nm);
          if (kmask != ~0ull) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (!((kmask >> (c + j)) & 1ull)) x[j] = -INFINITY;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] = ex2_approx(x[j]);
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
#pragma unroll
            for (int e = 0; e < 8; e += 2) add2(lacc[e], lacc[e + 1], lacc[e], lacc[e + 1], x[j + e], x[j + e + 1]);
          }
          uint32_t pw[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) pw[q] = pack_bf16x2(x[2 * q], x[2 * q + 1]);
          tmem_st16(t_lane + kPairP0 + pb * 64 + 32 * hf + c / 2, reinterpret_cast<const float*>(pw));
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[Ly::bPFull + pb]);
      }
      // this half-row's sum for the epilogue (buffer it & 1 is free once item it-2 is stored)
      const float lsum = ((lacc[0] + lacc[1]) + (lacc[2] + lacc[3])) + ((lacc[4] + lacc[5]) + (lacc[6] + lacc[7]));
      lsum_s[((it & 1) * 2 + hf) * 128 + r] = lsum;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Ly::bLFull + (it & 1)]);
    }
  } else {
    // ============================================================ epilogue: one thread per query row
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    const bool use_oc = (a.gate_nonzero == nullptr) || (*a.gate_nonzero != 0);
    for (int it = 0;; ++it) {
      int w = (lane == 0) ? ring_take(it, 49) : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w < 0) break;  // every epilogue warp reads the same ring, so all stop at the same item
      const int64_t bh = w / npairs;
      const int s0 = r_lo + 2 * static_cast<int>(w - bh * npairs);
      const int s = s0 + (r >> 6);
      const int64_t b = bh / a.H;
      const int h = static_cast<int>(bh - b * a.H);
      const int32_t tok = (s < r_end) ? __ldg(a.tile_token + static_cast<int64_t>(s) * 64 + (r & 63)) : -1;
      uint16_t* dst = nullptr;
      const uint16_t* gsrc = nullptr;
      float gq = 0.0f;
      if (tok >= 0) {
        int part = 0;
        int64_t lt = tok;
        if (a.io.table != nullptr) {
          part = static_cast<int>(tok / a.io.Ls);
          lt = tok - part * a.io.Ls;
        }
        const int64_t row = b * a.io.Ls + lt;
        uint16_t* obase = a.io.table ? static_cast<uint16_t*>(const_cast<void*>(a.io.table[kPartOut * a.io.nparts + part]))
                                     : a.out;
        dst = obase + (row * a.io.Htot + a.io.h0 + h) * D;
        const uint16_t* gb =
            a.io.table ? static_cast<const uint16_t*>(a.io.table[kPartGate * a.io.nparts + part]) : a.gate;
        if (a.gate_pc)
          gsrc = gb + row * a.gate_ld + static_cast<int64_t>(a.io.h0 + h) * D;
        else if (use_oc)
          gq = bf16_bits_to_f32(__ldg(gb + row * a.gate_ld + a.io.h0 + h));
      }
      const float* oc = a.o_c + (bh * n_sel + (s >> sh)) * D;
      mbar_wait(&bars[Ly::bLFull + (it & 1)], (it >> 1) & 1, ctl, 53);
      const float* lp = lsum_s + (it & 1) * 256;
      const float rl = rcp_approx(lp[r] + lp[128 + r]);
      mbar_wait(&bars[Ly::bOFull], it & 1, ctl, 54);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        tmem_ld32(t_lane + kPairO0 + c0, o);
        tmem_wait_ld();
        if (dst != nullptr) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            U128 v;
            uint32_t* pv = &v.x;
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const int d = c0 + c + e;
              float g0 = gq, g1 = gq;
              if (a.gate_pc && use_oc) {
                g0 = bf16_bits_to_f32(__ldg(gsrc + d));
                g1 = bf16_bits_to_f32(__ldg(gsrc + d + 1));
              }
              const float oc0 = use_oc ? __ldg(oc + d) : 0.0f, oc1 = use_oc ? __ldg(oc + d + 1) : 0.0f;
              pv[e >> 1] = pack_bf16x2(fmaf(o[c + e], rl, g0 * oc0), fmaf(o[c + e + 1], rl, g1 * oc1));
            }
            *reinterpret_cast<U128*>(dst + c0 + c) = v;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Ly::bOEmpty]);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace vsa
