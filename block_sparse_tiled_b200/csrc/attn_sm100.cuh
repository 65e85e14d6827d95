// Block-sparse VSA-H3 attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Work item = (b, h, 64-row block s of the query tiles), numbered (b*H + h)*n_rb + s.
// With 64-token tiles a row block is a tile; with 128-token tiles (sub_shift = 1)
// tile i is row blocks 2i and 2i+1, which share its key list.  The key list of
// query tile i is every tile for a prefix query tile, else the P prefix tiles
// followed by the tile's selected video tiles (ascending), taken as row blocks
// and walked two row blocks (128 keys) at a time.  With reference segments the
// always-kept prefix tiles are the non-reference ones, and the kept reference
// tiles come first in the idx row.  CTAs claim items in order from a global counter
// (one per SM, persistent), so the items in flight stay within a head or two
// and that head's K/V stays resident in L2 even though prefix query tiles cost
// many times a video query tile.
//
// A query tile is only 64 rows, so the kernel works in the transposed form,
// which keeps every row of the 128-row tcgen05 MMA busy:
//     S^T [128 keys x 64 queries]  = K_blk (M=128, K-major) * Q_tile^T (N=64, K-major)
//     O^T [D x 64 queries]        += V_blk^T (M=D, MN-major) * P^T (N=64, MN-major)
// S^T and O^T live in TMEM (lane = key or d, column = query).  The softmax
// statistics are per query, i.e. per TMEM column, across lanes:
//   - the running maximum m[q] is kept lazily: a block is exponentiated
//     against the current m, and only when some logit exceeds m by more than
//     kRescaleLog2 (or on an item's first super-block, below) is the exact column
//     maximum taken across the 128 lanes and O^T, l rescaled.  Any m with no
//     overflow gives the same softmax, so this is exact up to rounding.
//     Deciding "exceeds" takes a vote of the column group every super-block,
//     unless the first one already shows that no later logit can overflow: a
//     logit is at most |q| max|k| (Cauchy-Schwarz), so when that
//     bound is within skip_cap - log2(max|v|) of the first maximum for
//     every column, P, l and O^T stay finite without further rescaling and the
//     group skips the votes for the rest of the item;
//   - l[q] is kept as per-lane partial sums and reduced once per item.
// Blocks go two at a time through one handshake (a super-block of 256 keys): the
// S^T issuer fills both 64-column halves of one S^T buffer and signals once, the
// softmax exponentiates both halves against one m (a super-block that needs the
// exact maximum takes it over both halves in a first pass over S^T), writes both
// 128-key halves of one P^T buffer and releases S^T and P^T with one arrival
// each, and the P.V issuer runs both halves' MMAs on one P^T-full wait.
// O^T is double-buffered in TMEM, so one item's epilogue (in its own warps)
// overlaps the next item's blocks.
// D = 64 uses the same M = 128 PV product with a zero upper half of V^T, and
// D = 96 one whose upper 32 rows TMA fills with zeros.
//
// Roles (768 threads, 24 warps):
//   warp 0  K producer: TMA for the query tile of each item and the K tiles
//           of each block (4 lanes issue the four 8 KB boxes in parallel);
//   warp 1  V producer: TMA for the V tiles of each block;
//   warp 2  S^T issuer (one thread) and TMEM owner;
//   warp 3  P.V issuer (one thread);
//   warps 4..19  softmax, four groups of four warps; group g owns query
//           columns [16g, 16g + 16), warp w reads TMEM lane quadrant w % 4
//           (four softmax warps per SM sub-partition hide each other's latency);
//           each warp derives its blocks' valid-key counts from the key list,
//           32 blocks at a time, and shuffles them out per block;
//   warps 20..23 epilogue: 1/l, O^T from TMEM, the gated compression term
//           and the bf16 store in sequence order.
// Two issuing threads keep two tcgen05 streams in flight (one thread alone is
// limited by its issue latency), and several issuing lanes keep enough TMA
// loads in flight.  Every mbarrier wait is bounded; after a timeout the kernel
// stops issuing work, finishes its loops without waiting, drains what it
// issued and returns with the status word set.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "prep_kernels.cuh"
#include "ptx.cuh"

namespace vsa {

// Optional per-role cycle accounting (build with -DVSA_ROLE_TIMERS): each role
// of each CTA adds clock64() deltas into up to 8 counters, read back with
// vsa_role_timers().  Compiled out otherwise.
#ifdef VSA_ROLE_TIMERS
constexpr int kRoleTimerCtas = 160;
__device__ unsigned long long g_role_cycles[kRoleTimerCtas][8][8];
#define ROLE_TIMER_START() \
  unsigned long long rt_acc_[8] = {0, 0, 0, 0, 0, 0, 0, 0}; \
  unsigned long long rt_t_ = clock64()
#define ROLE_MARK(c)                         \
  do {                                       \
    const unsigned long long n_ = clock64(); \
    rt_acc_[c] += n_ - rt_t_;                \
    rt_t_ = n_;                              \
  } while (0)
#define ROLE_TIMER_SAVE(role)                                                               \
  do {                                                                                      \
    if (blockIdx.x < kRoleTimerCtas)                                                        \
      for (int c_ = 0; c_ < 8; ++c_) g_role_cycles[blockIdx.x][role][c_] = rt_acc_[c_];     \
  } while (0)
#else
#define ROLE_TIMER_START() \
  do {                     \
  } while (0)
#define ROLE_MARK(c) \
  do {               \
  } while (0)
#define ROLE_TIMER_SAVE(role) \
  do {                        \
  } while (0)
#endif

constexpr int kSoftGroups = 4;                    // softmax column groups
constexpr int kGroupCols = 64 / kSoftGroups;       // query columns per group
constexpr int kSoftWarps = 4 * kSoftGroups;        // one warp per TMEM lane quadrant per group
constexpr int kEpiWarp0 = 4 + kSoftWarps;          // first epilogue warp
constexpr int kAttnThreads = 32 * (kEpiWarp0 + 4);
// Lazy-max threshold: probabilities stay <= 2^24 between exact rescales.  With
// at most 2^23 keys per row, row sums stay below 2^47 and P.V partial sums far
// below the binary32 range.
constexpr float kRescaleLog2 = 24.0f;
constexpr int kSBufs = 2;             // S^T buffers in TMEM, one per super-block (two 64-column halves)
constexpr int kOCol0 = 128 * kSBufs;  // O^T double buffer follows (2 x 64 columns)
constexpr uint32_t kTmemCols = 512;

struct AttnArgs {
  const int32_t* idx;         // [B, H, V, kr + topk]: kept reference tiles, then video tiles (each ascending)
  const int32_t* exempt;      // NULL: every prefix tile is always kept; else the n_exempt always-kept ones
  int n_exempt, kr;           // always-kept prefix tiles (P without reference tiles); reference tiles kept
  const int32_t* tile_token;  // [n_rb * 64]: token of each row of each 64-row block
  const int32_t* tile_valid;  // [n_t]
  const float* o_c;           // [B, H, n_t, D] (per tile)
  const uint16_t* gate;       // [B, L, gate_ld] bf16: the gate of head h at gate[(b*L + t)*gate_ld + h]
  uint16_t* out;              // [B, L, H, D] bf16
  int* status;                // [2] device status word
  int* sched;                 // item counter, zero at launch
  int64_t L;
  int H, n_t, P, topk;  // n_t here: 64-row blocks per (b, h) (tiles << sub_shift); P, topk in tiles
  int sub_shift;         // log2(tile size / 64): 0 for 64-token tiles, 1 for 128
  int gate_ld;  // gate elements between consecutive tokens (H or H*D, or more when a head slice is processed)
  int gate_pc;  // 0: one gate per (token, head) at h; 1: one per channel, at h*D + d
  const int* gate_nonzero;  // NULL, or a flag that is 0 when every gate is zero (o_c then unread)
  const uint64_t* key_mask;  // [n_rb]: bit r set when row r of the block as loaded is a key (a token)
  const int32_t* coord;      // [n_rb][4] TMA coordinates of a block read from sequence order
  PartIO io;                 // where gate and out live (one tensor, or sequence parts, possibly on peers)
  const float* q_scale;      // 8-bit Q/K only: [B, H, n_rb, 64] scale of each query row (tile order)
  const float* k_scale;      // 8-bit Q/K only: [B, H, n_rb, 64] scale of each key row
  // Overflow bound (NULL: none, every block votes on a rescale): the Euclidean norm of each query row
  // [B, H, n_rb, 64] in tile-order rows (8-bit Q/K: of the dequantised row, scale times code norm), and
  // per (b, h) the largest key norm and |v| (float pairs); skip_cap = 124 - ceil(log2(keys of the
  // longest list)).
  const float* q_norm;
  const float* kv_max;
  float skip_cap;
  float scale_log2;  // softmax scale * log2(e)
  int s_lo, n_s;     // the launch covers row blocks [s_lo, s_lo + n_s) of every (b, h)
  int r_end;         // pair kernel: its pairs cover [s_lo, s_lo + 2 n_s); rows >= r_end are not queries
  int64_t n_items;   // B * H * n_s
};

// Tensor maps for loading tiles straight from sequence order (q, k, v): a 4-D map over [b, token, head, d]
// for prefix runs and, per batch, a 5-D map over [t, y, x, head, d] of the video grid.
constexpr int kSeqMaxBatch = 4;
struct SeqMaps {
  CUtensorMap prefix[3];
  CUtensorMap video[3][kSeqMaxBatch];
};

template <int D, bool kF8 = false>
struct AttnLayout {
  // 128-byte swizzle atoms along D.  D = 96 uses two, the second half-empty: TMA fills columns 96..127
  // with zeros, the S^T product stops after D/16 K-steps and O^T rows 96..127 are never stored.
  // kF8: Q and K are 8-bit codes, one 128-byte atom per row for any D (the S^T product runs D/32
  // K-steps of 32 bytes); V stays bf16.
  static constexpr int kHalves = (D + 63) / 64;
  static constexpr int kQBytes = kF8 ? 64 * 128 : 64 * 64 * kHalves * 2;    // one query tile
  static constexpr int kKVBytes = 128 * 64 * kHalves * 2;                  // 128 keys of V (bf16)
  static constexpr int kKBytes = kF8 ? 128 * 128 : kKVBytes;               // 128 keys of K
  static constexpr int kHalfBytes = 128 * 128;  // one 64-column half of a 128-row block
  static constexpr int kPHalfBytes = 128 * 64 * 2;  // P^T of one 128-key block
  static constexpr int kPBytes = 2 * kPHalfBytes;    // P^T of one super-block (256 keys)
  static constexpr int kQBufs = 1;
  static constexpr int kKStages = kF8 ? 4 : 2;
  static constexpr int kVStages = 2;
  static constexpr int kPBufs = 2;  // P^T buffers in shared memory
  static constexpr int kRing = 8;  // claimed items in flight
  static constexpr int kZeroBytes = (D == 64) ? 16384 : 0;
  // kF8: the query scales of the two items in flight in the softmax (64 floats each, times the
  // softmax scale * log2 e)
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQBufs * kQBytes;
  static constexpr int oV = oK + kKStages * kKBytes;
  static constexpr int oP = oV + kVStages * kKVBytes;
  static constexpr int oZ = oP + kPBufs * kPBytes;
  static constexpr int oQS = oZ + kZeroBytes;
  static constexpr int oBar = oQS + (kF8 ? 512 : 0);
  // barrier indices (8 bytes each)
  static constexpr int bQFull = 0, bQEmpty = bQFull + kQBufs;
  static constexpr int bKFull = bQEmpty + kQBufs, bKEmpty = bKFull + kKStages;
  static constexpr int bVFull = bKEmpty + kKStages, bVEmpty = bVFull + kVStages;
  static constexpr int bSFull = bVEmpty + kVStages, bSEmpty = bSFull + kSBufs;
  static constexpr int bPFull = bSEmpty + kSBufs, bPEmpty = bPFull + kPBufs;
  static constexpr int bOFull = bPEmpty + kPBufs, bOEmpty = bOFull + 2;
  static constexpr int bLFull = bOEmpty + 2;
  static constexpr int bRFull = bLFull + 2, bREmpty = bRFull + kRing;
  static constexpr int bDoneS = bREmpty + kRing, bDonePV = bDoneS + 1;
  static constexpr int kNumBars = bDonePV + 1;
  static constexpr int oMisc = oBar + kNumBars * 8;          // tmem base, abort flag
  static constexpr int oRing = ((oMisc + 8 + 15) / 16) * 16;  // int ring[kRing]: claimed items, -1 = none left
  static constexpr int oM = oRing + kRing * 4;               // float -m[64]: negated running max (log2 units)
  static constexpr int oDelta = oM + 256;                    // float delta[64]: m increase of a rescale
  static constexpr int oRed = oDelta + 256;                  // float red[groups][4 quadrants][group columns]
  static constexpr int oLsum = oRed + 1024;                  // float lpart[2 buffers][4 quadrants][64]
  static constexpr int oRg = oLsum + 2048;                   // float2 {1 / l, gate}[64]   (epilogue)
  static constexpr int oDst = oRg + 512;                     // bf16* dst[64]: out row of each query (epilogue)
  static constexpr int oGsrc = oDst + 512;                   // const bf16* gsrc[64]: its per-channel gate row
  static constexpr int oSkip = oGsrc + 512;                  // int skip[groups]: the item needs no votes
  static constexpr int oRows = oSkip + 16;                   // uint32 rows[2]: token rows of the item (ballots)
  static constexpr int oEnd = oRows + 8;
  static size_t bytes(int /*n_t*/) { return 1024 /*alignment slack*/ + oEnd; }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// In-warp reduce-scatter (sum) of 32 per-lane columns: afterwards v[0] holds the
// sum over the warp's 32 lanes of column `lane`.  The input array is consumed.
__device__ __forceinline__ void warp_sum_scatter32(float* v, int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step;  // 16, 8, 4, 2, 1
    const int bit = 4 - step;     // lane bit that picks the kept half
    const bool upper = (lane >> bit) & 1;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float lo = v[i], hi = v[i + half];
      const float send = upper ? lo : hi;
      const float keep = upper ? hi : lo;
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << bit);
    }
  }
}

// kSeq = false: Q/K/V come from tile-order copies through 2-D maps (tm_q/k/v).  kSeq = true: they come
// straight from the sequence-order tensors through `seq`, one box per tile (a 64-token prefix run or a
// 4x4x4 video cube); rows outside the tile are masked by key_mask and not stored.
// kF8 (tile-order copies only): Q and K are E4M3 codes with one scale per row (a.q_scale, a.k_scale).
// S^T is then an 8-bit product (kind::f8f6f4, K = 32 per instruction: half the instructions of bf16)
// of the codes; the softmax multiplies each logit by its key row's scale and its query column's scale
// before the exponent.  P.V is unchanged (bf16).
template <int D, bool kSeq, bool kF8>
__global__ void __launch_bounds__(kAttnThreads, 1)
    vsa_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a, const __grid_constant__ SeqMaps seq) {
  static_assert(!(kSeq && kF8), "8-bit Q/K reads tile-order copies");
  using Ly = AttnLayout<D, kF8>;
  constexpr int kQKSteps = kF8 ? (D + 31) / 32 : D / 16;
  constexpr int kPVSteps = 128 / 16;
  constexpr uint32_t kIdescS = kF8 ? umma_idesc_e4m3(128, 64) : umma_idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 64, 1, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::oBar);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::oMisc + 4);
  int* ring_s = reinterpret_cast<int*>(sm + Ly::oRing);
  float* m_s = reinterpret_cast<float*>(sm + Ly::oM);
  float* delta_s = reinterpret_cast<float*>(sm + Ly::oDelta);
  float* red_s = reinterpret_cast<float*>(sm + Ly::oRed);
  float* lpart_s = reinterpret_cast<float*>(sm + Ly::oLsum);
  float2* rg_s = reinterpret_cast<float2*>(sm + Ly::oRg);
  uint16_t** dst_s = reinterpret_cast<uint16_t**>(sm + Ly::oDst);
  const uint16_t** gsrc_s = reinterpret_cast<const uint16_t**>(sm + Ly::oGsrc);
  uint32_t* rows_s = reinterpret_cast<uint32_t*>(sm + Ly::oRows);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // n_t: 64-row blocks per (b, h); n_sel: tiles (the selection's unit), P and topk count tiles
  const int n_t = a.n_t, sh = a.sub_shift, n_sel = n_t >> sh, P = a.P, topk = a.topk, V = n_sel - P;
  const WaitCtl ctl{abort_flag, a.status, kWaitTimeoutNs};

  // ---------------------------------------------------------------- setup
  if (Ly::kZeroBytes > 0) {
    uint32_t* z = reinterpret_cast<uint32_t*>(sm + Ly::oZ);
    for (int t = threadIdx.x; t < Ly::kZeroBytes / 4; t += blockDim.x) z[t] = 0u;
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < Ly::kQBufs; ++s) {
      mbar_init(&bars[Ly::bQFull + s], 1);
      mbar_init(&bars[Ly::bQEmpty + s], 1);
    }
    for (int s = 0; s < Ly::kKStages; ++s) {
      mbar_init(&bars[Ly::bKFull + s], 1);
      mbar_init(&bars[Ly::bKEmpty + s], 1);
    }
    for (int s = 0; s < Ly::kVStages; ++s) {
      mbar_init(&bars[Ly::bVFull + s], 1);
      mbar_init(&bars[Ly::bVEmpty + s], 1);
    }
    for (int s = 0; s < 4; ++s) {
      if (s < kSBufs) {
        mbar_init(&bars[Ly::bSFull + s], 1);
        mbar_init(&bars[Ly::bSEmpty + s], kSoftWarps * 32);  // every softmax thread arrives
      }
      if (s < Ly::kPBufs) {
        mbar_init(&bars[Ly::bPFull + s], kSoftWarps * 32);
        mbar_init(&bars[Ly::bPEmpty + s], 1);
      }
    }
    for (int s = 0; s < Ly::kRing; ++s) {
      mbar_init(&bars[Ly::bRFull + s], 1);
      mbar_init(&bars[Ly::bREmpty + s], 3 + kSoftWarps + 4);  // V producer, two issuers, softmax, epilogue
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[Ly::bOFull + s], 1);
      mbar_init(&bars[Ly::bOEmpty + s], 4);
      mbar_init(&bars[Ly::bLFull + s], kSoftWarps);
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
    tmem_alloc(tmem_base_s, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  // key list of query tile i, in 64-row blocks: all tiles, or the E always-kept prefix tiles and the
  // kr + topk entries of the tile's idx row
  const int E = a.n_exempt, W = a.kr + topk;
  auto list_len = [&](int i) { return ((i < P) ? n_sel : E + W) << sh; };
  // row block of list position t (in row blocks) of query tile i
  auto key_tile = [&](int64_t bh, int i, int t) -> int {
    const int ts = t >> sh;
    int sel;
    if (i < P)
      sel = ts;
    else if (ts < E)
      sel = a.exempt ? __ldg(a.exempt + ts) : ts;
    else
      sel = __ldg(a.idx + (bh * V + (i - P)) * W + (ts - E));
    return (sel << sh) | (t & ((1 << sh) - 1));
  };
  // Claimed item number `it` of this CTA (-1: none left), read by one thread of a consumer warp.
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
    int it = 0;
    bool ok = true;
    ROLE_TIMER_START();
    // Lane 0 of the K producer claims items (global counter) two ahead of its own use and
    // publishes them in the ring; -1 marks the end.  The other roles read the ring.
    int pub = 0;       // items published so far
    bool more = true;  // the counter may still have items
    auto publish_next = [&]() {
      if (!more) return;
      const int slot = pub % Ly::kRing;
      if (!mbar_wait(&bars[Ly::bREmpty + slot], ((pub / Ly::kRing) & 1) ^ 1, ctl, 24)) {
        more = false;
        return;
      }
      const int claimed = atomicAdd(a.sched, 1);  // items fit in an int (the plan checks B*H*n_t*64 < 2^31)
      // claimed -> item (b*H + h)*n_t + s of the launch's row blocks
      const int v = (claimed < a.n_items) ? (claimed / a.n_s) * n_t + a.s_lo + claimed % a.n_s : -1;
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
          w = ring_take(it, 25);
        }
      }
      w = __shfl_sync(0xffffffffu, w, 0);
      if (w < 0 || !ok) break;
      const int64_t bh = w / n_t;
      const int s = static_cast<int>(w - bh * n_t);  // query row block
      const int i = s >> sh;                          // its tile
      const int nk = list_len(i), nb = (nk + 1) / 2;
      if (is_k) {
        // the query tile of this item (loaded by the K warp, which runs ahead with the S^T issuer)
        const int qb = it % Ly::kQBufs;
        const uint32_t qu = it / Ly::kQBufs;
        if (lane == 0) {
          ROLE_MARK(3);
          ok = mbar_wait(&bars[Ly::bQEmpty + qb], (qu & 1) ^ 1, ctl, 1);
          ROLE_MARK(0);
          if (ok) mbar_arrive_expect_tx(&bars[Ly::bQFull + qb], Ly::kQBytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok && lane < (kF8 ? 1 : Ly::kHalves)) {
          void* dst = sm + Ly::oQ + qb * Ly::kQBytes + lane * 8192;
          if constexpr (kSeq) {
            const int4 c = __ldg(reinterpret_cast<const int4*>(a.coord) + s);
            const int bb = static_cast<int>(bh / a.H), hh = static_cast<int>(bh - static_cast<int64_t>(bb) * a.H);
            if (c.x == 0)
              tma_load_4d(dst, &seq.prefix[0], &bars[Ly::bQFull + qb], lane * 64, hh, c.y, bb);
            else
              tma_load_5d(dst, &seq.video[0][bb], &bars[Ly::bQFull + qb], lane * 64, hh, c.y, c.z, c.w);
          } else {
            const int row = static_cast<int>((bh * n_t + s) * 64);
            tma_load_2d(dst, &tm_q, &bars[Ly::bQFull + qb], lane * 64, row);
          }
        }
      }
      for (int n0 = 0; n0 < nb && ok; n0 += 32) {
        const int n = n0 + lane;
        int ta = 0, tb = -1;
        if (n < nb) {
          ta = key_tile(bh, i, 2 * n);
          tb = (2 * n + 1 < nk) ? key_tile(bh, i, 2 * n + 1) : -1;
        }
        const int cnt = min(32, nb - n0);
        for (int j = 0; j < cnt; ++j, ++g) {
          const int ka = __shfl_sync(0xffffffffu, ta, j);
          const int kb_raw = __shfl_sync(0xffffffffu, tb, j);
          const int kb = kb_raw < 0 ? ka : kb_raw;  // an odd list repeats its last tile; the softmax masks it
          const int st = g % nstages;
          const uint32_t u = g / nstages;
          // bytes of one stage: K (8-bit: one 8 KB box per tile), or V plus, with 8-bit Q/K, the key scales
          const int stage_bytes = is_k ? Ly::kKBytes : Ly::kKVBytes;
          const int halves = (is_k && kF8) ? 1 : Ly::kHalves;
          if (lane == 0) {
            ROLE_MARK(3);
            ok = mbar_wait(&bars[b_empty + st], (u & 1) ^ 1, ctl, is_k ? 2 : 3);
            ROLE_MARK(1);
            if (ok) mbar_arrive_expect_tx(&bars[b_full + st], stage_bytes);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          // lanes [0, 2*halves) issue one 8 KB box each: (half, tile a|b)
          if (lane < 2 * halves) {
            const int hh = lane >> 1, second = lane & 1;
            const int t = second ? kb : ka;
            void* dst = ring + st * stage_bytes + hh * Ly::kHalfBytes + second * 8192;
            if constexpr (kSeq) {
              const int4 c = __ldg(reinterpret_cast<const int4*>(a.coord) + t);
              const int bb = static_cast<int>(bh / a.H), head = static_cast<int>(bh - static_cast<int64_t>(bb) * a.H);
              const int ti = is_k ? 1 : 2;
              if (c.x == 0)
                tma_load_4d(dst, &seq.prefix[ti], &bars[b_full + st], hh * 64, head, c.y, bb);
              else
                tma_load_5d(dst, &seq.video[ti][bb], &bars[b_full + st], hh * 64, head, c.y, c.z, c.w);
            } else {
              const int row = static_cast<int>((bh * n_t + t) * 64);
              tma_load_2d(dst, tmap, &bars[b_full + st], hh * 64, row);
            }
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) {
      ROLE_MARK(3);
      ROLE_TIMER_SAVE(warp);
    }
    // drain: every load this warp issued must land before the CTA exits
    if (lane == 0) {
      const WaitCtl drain{abort_flag, a.status, kWaitTimeoutNs};
      for (int s = 0; s < nstages && static_cast<uint32_t>(s) < g; ++s) {
        const uint32_t last = g - 1 - s;
        mbar_wait_drain(&bars[b_full + (last % nstages)], (last / nstages) & 1, drain, 20);
      }
      if (is_k && it > 0) {
        for (int s = 0; s < Ly::kQBufs && s < it; ++s) {
          const int lastq = it - 1 - s;
          mbar_wait_drain(&bars[Ly::bQFull + (lastq % Ly::kQBufs)], (lastq / Ly::kQBufs) & 1, drain, 21);
        }
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ============================================================ S^T issuer
    // Super-block j of an item = its 128-key blocks 2j and 2j + 1 (the second absent at an odd end): both
    // go into S^T buffer sb (two 64-column halves), which the softmax releases with one arrival.
    if (lane == 0) {
      uint32_t g = 0, G = 0;  // 128-key blocks (K stages) and super-blocks (S^T buffers) so far
      int it = 0;
      bool ok = true;
      ROLE_TIMER_START();
      for (;; ++it) {
        const int w = ring_take(it, 26);
        if (w < 0 || !ok) break;
        const int64_t bh = w / n_t;
        const int i = static_cast<int>(w - bh * n_t) >> sh;  // the item's tile
        const int nb = (list_len(i) + 1) / 2, nsb = (nb + 1) / 2;
        const int qb = it % Ly::kQBufs;
        ROLE_MARK(3);
        ok = mbar_wait(&bars[Ly::bQFull + qb], (it / Ly::kQBufs) & 1, ctl, 5);
        ROLE_MARK(0);
        const uint64_t qd0 = umma_desc_sw128(smem_u32(sm + Ly::oQ + qb * Ly::kQBytes), 16, 1024);
        for (int j = 0; j < nsb && ok; ++j, ++G) {
          const int sb = G % kSBufs;
          ROLE_MARK(3);
          ok = mbar_wait(&bars[Ly::bSEmpty + sb], ((G / kSBufs) & 1) ^ 1, ctl, 7);
          ROLE_MARK(2);
          const int nh = min(2, nb - 2 * j);
          for (int h = 0; h < nh && ok; ++h, ++g) {
            const int kst = g % Ly::kKStages;
            ROLE_MARK(3);
            ok = mbar_wait(&bars[Ly::bKFull + kst], (g / Ly::kKStages) & 1, ctl, 6);
            ROLE_MARK(1);
            if (!ok) break;
            tc_fence_after();
            // descriptors of the block's first K-step; a step moves the start address (bits 0..13, 16-byte
            // units, no carry: shared memory addresses stay below 256 KB) by a compile-time offset
            const uint64_t ad0 = umma_desc_sw128(smem_u32(sm + Ly::oK + kst * Ly::kKBytes), 16, 1024);
            const uint32_t dcol = tmem + sb * 128 + h * 64;
#pragma unroll
            for (int kk = 0; kk < kQKSteps; ++kk) {
              // 32 bytes of every row per step: 16 bf16 or 32 8-bit elements
              const uint64_t ad = ad0 + static_cast<uint64_t>(((kk >> 2) * Ly::kHalfBytes + (kk & 3) * 32) >> 4);
              const uint64_t bd = qd0 + static_cast<uint64_t>(((kk >> 2) * 8192 + (kk & 3) * 32) >> 4);
              if constexpr (kF8)
                umma_ss_f8(dcol, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
              else
                umma_ss(dcol, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
            }
            umma_commit(&bars[Ly::bKEmpty + kst]);
          }
          if (!ok) break;
          umma_commit(&bars[Ly::bSFull + sb]);
          if (j == nsb - 1) umma_commit(&bars[Ly::bQEmpty + qb]);
        }
      }
      ROLE_MARK(3);
      ROLE_TIMER_SAVE(2);
      umma_commit(&bars[Ly::bDoneS]);
      mbar_wait_drain(&bars[Ly::bDoneS], 0, ctl, 22);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ============================================================ P.V issuer
    if (lane == 0) {
      uint32_t g = 0, G = 0;  // 128-key blocks (V stages) and super-blocks (P^T buffers) so far
      int it = 0;
      bool ok = true;
      ROLE_TIMER_START();
      for (;; ++it) {
        const int w = ring_take(it, 27);
        if (w < 0 || !ok) break;
        const int64_t bh = w / n_t;
        const int i = static_cast<int>(w - bh * n_t) >> sh;  // the item's tile
        const int nb = (list_len(i) + 1) / 2, nsb = (nb + 1) / 2;
        const int ob = it & 1;
        for (int j = 0; j < nsb && ok; ++j, ++G) {
          const int pb = G % Ly::kPBufs;
          ROLE_MARK(3);
          ok = mbar_wait(&bars[Ly::bPFull + pb], (G / Ly::kPBufs) & 1, ctl, 9);
          ROLE_MARK(1);
          ok = ok && (j > 0 || mbar_wait(&bars[Ly::bOEmpty + ob], ((it >> 1) & 1) ^ 1, ctl, 10));
          ROLE_MARK(2);
          const int nh = min(2, nb - 2 * j);
          for (int h = 0; h < nh && ok; ++h, ++g) {
            const int vst = g % Ly::kVStages;
            ROLE_MARK(3);
            ok = mbar_wait(&bars[Ly::bVFull + vst], (g / Ly::kVStages) & 1, ctl, 8);
            ROLE_MARK(0);
            if (!ok) break;
            tc_fence_after();
            // V^T atoms along M (= d): the other 64-column half, or the zero region for D = 64
            const uint32_t lbo_v = (D > 64) ? Ly::kHalfBytes
                                              : static_cast<uint32_t>(Ly::oZ - (Ly::oV + vst * Ly::kKVBytes));
            const uint64_t ad0 = umma_desc_sw128(smem_u32(sm + Ly::oV + vst * Ly::kKVBytes), lbo_v, 1024);
            // rows 128 h .. 128 h + 127 of the super-block's P^T (one 128-key block, 16 KB)
            const uint64_t bd0 =
                umma_desc_sw128(smem_u32(sm + Ly::oP + pb * Ly::kPBytes + h * Ly::kPHalfBytes), 8192, 1024);
#pragma unroll
            for (int kk = 0; kk < kPVSteps; ++kk) {
              // a K-step is 16 keys = 2048 bytes further (start address in 16-byte units)
              umma_ss(tmem + kOCol0 + ob * 64, ad0 + static_cast<uint64_t>(kk * 128),
                      bd0 + static_cast<uint64_t>(kk * 128), kIdescPV, (j > 0 || h > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&bars[Ly::bVEmpty + vst]);
          }
          if (!ok) break;
          umma_commit(&bars[Ly::bPEmpty + pb]);
          if (j == nsb - 1) umma_commit(&bars[Ly::bOFull + ob]);
        }
      }
      ROLE_MARK(3);
      ROLE_TIMER_SAVE(3);
      umma_commit(&bars[Ly::bDonePV]);
      mbar_wait_drain(&bars[Ly::bDonePV], 0, ctl, 23);
    }
    __syncwarp();
  } else if (warp < kEpiWarp0) {
    // ============================================================ softmax
    constexpr int CG = kGroupCols;
    const int grp = (warp - 4) >> 2;                   // column group: queries [CG grp, CG grp + CG)
    const int tid = threadIdx.x - 128 * (grp + 1);     // 0..127 within the group
    const int qd = warp & 3;                           // TMEM lane quadrant this warp may access
    const int kl = qd * 32 + lane;                     // key lane (S^T) / d lane (O^T)
    const int c0 = grp * CG;
    const int bar_vote = 1 + 2 * grp, bar_sync = 2 + 2 * grp;  // named barriers of this group
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    float* m_g = m_s + c0;   // the group's columns of the running maximum area, which holds -m
    float* nm_g = m_g;
    float* delta_g = delta_s + c0;
    float* red_g = red_s + grp * 4 * CG;
    const float cl = a.scale_log2;
    // 8-bit Q/K: query scales (times cl) of the group's columns, one buffer per item parity (at a fixed
    // offset from m_g); the group's first warp fills the buffer before the item's first barrier
    constexpr int kQscFromM = (Ly::oQS - Ly::oM) / 4;
    int* skip_s = reinterpret_cast<int*>(sm + Ly::oSkip);
    // With an overflow bound, lanes 0..15 of the group's first warp hold, per item, the least
    // first-block maximum m1 of their column for which no later block can overflow:
    //   cl |q| max|k| + ceil(log2 max|v|)+ - skip_cap   (compared with m1 in log2 units; NaN: never)
    // Tile-order rows are the query rows of the block; boxes read from sequence order hold a partial
    // tile's rows at their cube positions, in the same order, so there the tile-order row is the rank
    // of the position among the valid ones.
    float lim = 0.0f;
    auto item_limit = [&](int w, int r) -> float {
      const int64_t bhw = w / n_t;
      float qn;
      if constexpr (kSeq) {
        const uint64_t m = __ldg(a.key_mask + (w - bhw * n_t));
        qn = ((m >> r) & 1ull) ? __ldg(a.q_norm + static_cast<int64_t>(w) * 64 + __popcll(m & ((1ull << r) - 1ull)))
                               : 0.0f;
      } else {
        qn = __ldg(a.q_norm + static_cast<int64_t>(w) * 64 + r);
      }
      const float kmax = __ldg(a.kv_max + 2 * bhw), vmax = __ldg(a.kv_max + 2 * bhw + 1);
      const int ev = max(0, static_cast<int>((__float_as_uint(vmax) >> 23) & 0xffu) - 126);
      return cl * qn * kmax + static_cast<float>(ev) - a.skip_cap;
    };
    uint32_t G = 0;  // super-blocks so far (S^T and P^T buffers)
    int it = 0;
    ROLE_TIMER_START();
    for (;; ++it) {
      int w = (lane == 0) ? ring_take(it, 28) : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      if constexpr (kF8) {
        if (qd == 0 && lane < CG && w >= 0)
          m_g[kQscFromM + (it & 1) * 64 + lane] = __ldg(a.q_scale + static_cast<int64_t>(w) * 64 + c0 + lane) * cl;
      }
      if (a.q_norm != nullptr && qd == 0 && lane < CG && w >= 0) lim = item_limit(w, c0 + lane);
      if (named_bar_or(bar_vote, 128, w < 0)) break;  // the group stops together
      const int64_t bh = w / n_t;
      const int i = static_cast<int>(w - bh * n_t) >> sh;  // the item's tile
      const int nk = list_len(i), nb = (nk + 1) / 2;
      const int ob = it & 1;
      const float* qsc_g = m_g + kQscFromM + ob * 64;
      // lane j: the key-mask word of block n0 + j for this warp's TMEM lane quadrant (rows
      // 32*qd .. 32*qd + 31 of the block: tile a for qd < 2, tile b otherwise); with 8-bit Q/K also
      // that tile's row-scale offset (b, h, tile) * 64.  Refilled every 32 blocks (16 super-blocks).
      uint32_t vcache = 0;
      int kcache = 0;  // B*H*n_t*64 < 2^31 (checked when the plan is made)
      auto refill = [&](int n0) {
        const int nn = n0 + lane;
        vcache = 0;
        if (nn < nb) {
          const int t = 2 * nn + (qd >> 1);
          const int kt = (t < nk) ? key_tile(bh, i, t) : -1;
          const uint64_t m = (kt >= 0) ? __ldg(a.key_mask + kt) : 0ull;
          vcache = static_cast<uint32_t>(m >> (32 * (qd & 1)));
          if constexpr (kF8) kcache = static_cast<int>((bh * n_t + max(kt, 0)) * 64);
        }
      };

      float l[CG];
#pragma unroll
      for (int j = 0; j < CG; ++j) l[j] = 0.0f;
      bool skip = false;  // set by the first super-block: the item's later ones take no vote
      const int nsb = (nb + 1) / 2;

      // Super-block j of the item: its 128-key blocks 2j and 2j + 1 (nh of them), in S^T buffer sb and
      // P^T buffer pb, with one S^T-full wait, one S^T-empty and one P^T-full arrival for both.  The
      // first super-block (kFirst) and one whose vote fires take the exact column maximum over both
      // blocks first (a first pass over S^T), then exponentiate in a second pass, so that both blocks'
      // probabilities share one m.
      auto sblock = [&](auto first_c, const int j) {
        constexpr bool kFirst = decltype(first_c)::value;
        const int sb = G % kSBufs;
        const uint32_t su = G / kSBufs;
        const int pb = G % Ly::kPBufs;
        const uint32_t pu = G / Ly::kPBufs;
        const int nh = min(2, nb - 2 * j);
        ROLE_MARK(7);
        if (((2 * j) & 31) == 0) refill(2 * j);
        uint32_t km[2];
        [[maybe_unused]] float ks[2] = {1.0f, 1.0f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          km[h] = __shfl_sync(0xffffffffu, vcache, (2 * j + h) & 31);
          if constexpr (kF8) ks[h] = __ldg(a.k_scale + __shfl_sync(0xffffffffu, kcache, (2 * j + h) & 31) + (kl & 63));
        }
        ROLE_MARK(0);
        mbar_wait(&bars[Ly::bSFull + sb], su & 1, ctl, 12);
        ROLE_MARK(1);
        tc_fence_after();
        const uint32_t s_col = t_lane + sb * 128 + c0;
        // x = logit * log2(e) - m (m = 0 before the first super-block: nm_g is not read then); with 8-bit
        // Q/K the logit is the code product times the key and query scales (two columns per instruction:
        // fma2/mul2 round each lane as fmaf/fmul do; nm_g holds -m); rows that are not keys get -inf
        auto load_scaled = [&](auto use_m_c, int h, float* x) {
          constexpr bool kUseM = decltype(use_m_c)::value;
          tmem_ld16(s_col + h * 64, x);
          tmem_wait_ld();
          if constexpr (kF8) {
#pragma unroll
            for (int jj = 0; jj < CG; jj += 2) mul2(x[jj], x[jj + 1], x[jj], x[jj + 1], ks[h], ks[h]);
#pragma unroll
            for (int jj = 0; jj < CG; jj += 4) {
              const float4 c4 = *reinterpret_cast<const float4*>(qsc_g + jj);
              if constexpr (kUseM) {
                const float4 m4 = *reinterpret_cast<const float4*>(nm_g + jj);
                fma2(x[jj], x[jj + 1], x[jj], x[jj + 1], c4.x, c4.y, m4.x, m4.y);
                fma2(x[jj + 2], x[jj + 3], x[jj + 2], x[jj + 3], c4.z, c4.w, m4.z, m4.w);
              } else {
                mul2(x[jj], x[jj + 1], x[jj], x[jj + 1], c4.x, c4.y);
                mul2(x[jj + 2], x[jj + 3], x[jj + 2], x[jj + 3], c4.z, c4.w);
              }
            }
          } else if constexpr (kUseM) {
#pragma unroll
            for (int jj = 0; jj < CG; jj += 4) {
              const float4 m4 = *reinterpret_cast<const float4*>(nm_g + jj);
              fma2(x[jj], x[jj + 1], x[jj], x[jj + 1], cl, cl, m4.x, m4.y);
              fma2(x[jj + 2], x[jj + 3], x[jj + 2], x[jj + 3], cl, cl, m4.z, m4.w);
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < CG; jj += 2) mul2(x[jj], x[jj + 1], x[jj], x[jj + 1], cl, cl);
          }
          if (km[h] != 0xffffffffu) {  // the same word in every lane: a uniform branch
            if (!((km[h] >> lane) & 1u)) {  // not a key: a pad or out-of-tile row
#pragma unroll
              for (int jj = 0; jj < CG; ++jj) x[jj] = -INFINITY;
            }
          }
        };
        bool slow = kFirst;
        if constexpr (!kFirst) {
          if (!skip) {  // the same in all 128 threads of the group
            // the vote: does any logit of the super-block exceed m by more than kRescaleLog2?
            static_assert(CG == 16, "the vote's maximum is written for 16 columns");
            float t = -INFINITY;
            for (int h = 0; h < nh; ++h) {
              float x[CG];
              load_scaled(std::true_type{}, h, x);
              t = max3(t, max3(max3(max3(x[0], x[1], x[2]), max3(x[3], x[4], x[5]), max3(x[6], x[7], x[8])),
                               max3(x[9], x[10], x[11]), max3(max3(x[12], x[13], x[14]), x[15], x[15])),
                       t);
            }
            slow = named_bar_or(bar_vote, 128, t > kRescaleLog2);
          }
        }
        ROLE_MARK(3);
        if (slow) {
          // exact column maximum of the super-block over the group's 128 lanes (lane c keeps column c's
          // maximum over this warp's rows of both blocks); raise m by it
          float cm = -INFINITY;
          for (int h = 0; h < nh; ++h) {
            float x[CG];
            load_scaled(std::integral_constant<bool, !kFirst>{}, h, x);
#pragma unroll
            for (int jj = 0; jj < CG; ++jj) {
              float r;
              asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x[jj]));
              if (jj == lane) cm = fmaxf(cm, r);
            }
          }
          if (lane < CG) red_g[qd * CG + lane] = cm;
          named_bar_sync(bar_sync, 128);
          if (tid < CG) {
            const float c = fmaxf(fmaxf(red_g[tid], red_g[CG + tid]), fmaxf(red_g[2 * CG + tid], red_g[3 * CG + tid]));
            float d;
            if constexpr (kFirst) {
              d = (c == -INFINITY) ? 0.0f : c;
              nm_g[tid] = -d;
              if (a.q_norm != nullptr) {  // lanes 0..15 of the group's first warp
                const uint32_t ok = __ballot_sync(0xffffu, lim <= d);
                if (tid == 0) skip_s[grp] = (ok == 0xffffu) ? 1 : 0;
              }
            } else {
              d = fmaxf(c, 0.0f);
              nm_g[tid] -= d;  // -(m + d), rounded as m + d would be
            }
            delta_g[tid] = d;
          }
          named_bar_sync(bar_sync, 128);
          if constexpr (kFirst) skip = (a.q_norm != nullptr) && skip_s[grp] != 0;
          if constexpr (!kFirst) {
#pragma unroll
            for (int jj = 0; jj < CG; ++jj) l[jj] *= ex2_approx(-delta_g[jj]);
            // O^T holds the super-blocks < j of this item: wait for the last one's P.V, then rescale this
            // group's columns
            const uint32_t gp = G - 1;
            mbar_wait(&bars[Ly::bPEmpty + (gp % Ly::kPBufs)], (gp / Ly::kPBufs) & 1, ctl, 13);
            tc_fence_after();
            float o[CG];
            tmem_ld16(t_lane + kOCol0 + ob * 64 + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int jj = 0; jj < CG; ++jj) o[jj] *= ex2_approx(-delta_g[jj]);
            tmem_st16(t_lane + kOCol0 + ob * 64 + c0, o);
            tmem_wait_st();
            tc_fence_before();
          }
        }
        ROLE_MARK(4);
        // probabilities against the (new) m, partial row sums, this group's part of the P^T rows of both
        // blocks (bf16, 128-byte swizzle)
        mbar_wait(&bars[Ly::bPEmpty + pb], (pu & 1) ^ 1, ctl, 14);
        ROLE_MARK(6);
        for (int h = 0; h < nh; ++h) {
          float x[CG];
          // the first super-block's m is in nm_g now (its slow path always runs)
          load_scaled(std::true_type{}, h, x);
          if (h == nh - 1) {
            tc_fence_before();
            mbar_arrive(&bars[Ly::bSEmpty + sb]);  // per thread: no warp-level branch or sync
          }
#pragma unroll
          for (int jj = 0; jj < CG; ++jj) x[jj] = ex2_approx(x[jj]);
#pragma unroll
          for (int jj = 0; jj < CG; jj += 2) add2(l[jj], l[jj + 1], l[jj], l[jj + 1], x[jj], x[jj + 1]);
          uint8_t* prow = sm + Ly::oP + pb * Ly::kPBytes + h * Ly::kPHalfBytes + kl * 128;
#pragma unroll
          for (int cc = 0; cc < CG / 8; ++cc) {
            const int c = grp * (CG / 8) + cc;  // 16-byte chunk = queries 8c .. 8c+7
            U128 w4;
            w4.x = pack_bf16x2(x[8 * cc + 0], x[8 * cc + 1]);
            w4.y = pack_bf16x2(x[8 * cc + 2], x[8 * cc + 3]);
            w4.z = pack_bf16x2(x[8 * cc + 4], x[8 * cc + 5]);
            w4.w = pack_bf16x2(x[8 * cc + 6], x[8 * cc + 7]);
            *reinterpret_cast<U128*>(prow + ((c ^ (kl & 7)) << 4)) = w4;
          }
        }
        ROLE_MARK(5);
        fence_proxy_async_smem();
        mbar_arrive(&bars[Ly::bPFull + pb]);
      };
      if (nsb > 0) {
        sblock(std::true_type{}, 0);
        ++G;
      }
      for (int j = 1; j < nsb; ++j, ++G) sblock(std::false_type{}, j);


      // hand this warp's partial row sums to the epilogue (buffer ob is free once item it-2 is stored):
      // reduce-scatter over the warp's 32 lanes, lane j (j < CG) then holds column c0 + j
#pragma unroll
      for (int step = 0; step < 4; ++step) {
        const int half = (CG / 2) >> step;
        const int bit = 3 - step;
        const bool upper = (lane >> bit) & 1;
#pragma unroll
        for (int j = 0; j < half; ++j) {
          const float lo = l[j], hi = l[j + half];
          const float send = upper ? lo : hi;
          const float keep = upper ? hi : lo;
          l[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1 << bit);
        }
      }
      l[0] += __shfl_xor_sync(0xffffffffu, l[0], 16);
      if (it >= 2) mbar_wait(&bars[Ly::bOEmpty + ob], ((it >> 1) & 1) ^ 1, ctl, 15);
      if (lane < CG) lpart_s[(ob * 4 + qd) * 64 + c0 + lane] = l[0];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Ly::bLFull + ob]);
    }
    ROLE_MARK(7);
    if (tid == 0) ROLE_TIMER_SAVE(4 + (grp & 1));
  } else {
    // ============================================================ epilogue
    const int tid = threadIdx.x - 32 * kEpiWarp0;  // 0..127
    const int qd = warp & 3;
    const int d = qd * 32 + lane;                  // O^T lane = d
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    // with every gate zero the compression term vanishes and o_c was not computed
    const bool use_oc = (a.gate_nonzero == nullptr) || (*a.gate_nonzero != 0);
    int it = 0;
    ROLE_TIMER_START();
    for (;; ++it) {
      int w = (lane == 0) ? ring_take(it, 29) : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (named_bar_or(9, 128, w < 0)) break;  // the epilogue warps stop together
      const int64_t bh = w / n_t;
      const int s = static_cast<int>(w - bh * n_t);  // query row block
      const int i = s >> sh;                          // its tile
      const int64_t b = bh / a.H;
      const int h = static_cast<int>(bh - b * a.H);
      const int ob = it & 1;
      if (tid < 64) {
        // per query row: where its output row starts (NULL: a pad, not stored), its per-token gate or
        // the start of its per-channel gate row
        const int32_t tok = __ldg(a.tile_token + static_cast<int64_t>(s) * 64 + tid);
        uint16_t* dst = nullptr;
        const uint16_t* gsrc = nullptr;
        float g = 0.0f;
        if (tok >= 0) {
          int part = 0;
          int64_t lt = tok;
          if (a.io.table != nullptr) {
            part = static_cast<int>(tok / a.io.Ls);
            lt = tok - part * a.io.Ls;
          }
          const int64_t row = b * a.io.Ls + lt;  // row of the token in its part (or in the one tensor)
          uint16_t* obase = a.io.table ? static_cast<uint16_t*>(const_cast<void*>(a.io.table[kPartOut * a.io.nparts + part]))
                                       : a.out;
          dst = obase + (row * a.io.Htot + a.io.h0 + h) * D;
          const uint16_t* gb =
              a.io.table ? static_cast<const uint16_t*>(a.io.table[kPartGate * a.io.nparts + part]) : a.gate;
          if (a.gate_pc)
            gsrc = gb + row * a.gate_ld + static_cast<int64_t>(a.io.h0 + h) * D;
          else if (use_oc)
            g = bf16_bits_to_f32(__ldg(gb + row * a.gate_ld + a.io.h0 + h));
        }
        dst_s[tid] = dst;
        gsrc_s[tid] = gsrc;
        rg_s[tid].y = g;
        const uint32_t tokens = __ballot_sync(0xffffffffu, tok >= 0);  // tid < 64: two whole warps
        if (lane == 0) rows_s[tid >> 5] = tokens;
      }
      const float oc = (d < D && use_oc) ? __ldg(a.o_c + (bh * n_sel + i) * D + d) : 0.0f;
      ROLE_MARK(3);
      mbar_wait(&bars[Ly::bLFull + ob], (it >> 1) & 1, ctl, 16);
      ROLE_MARK(0);
      if (tid < 64) {
        const float* lp = lpart_s + ob * 4 * 64 + tid;
        rg_s[tid].x = rcp_approx((lp[0] + lp[64]) + (lp[128] + lp[192]));
      }
      mbar_wait(&bars[Ly::bOFull + ob], (it >> 1) & 1, ctl, 17);
      ROLE_MARK(1);
      named_bar_sync(9, 128);  // rl, gate, row pointers ready
      const bool full = (rows_s[0] & rows_s[1]) == ~0u;  // all 64 query rows are tokens
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tc_fence_after();
        float o[32];
        tmem_ld32(t_lane + kOCol0 + ob * 64 + 32 * half, o);
        tmem_wait_ld();
        if (half == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[Ly::bOEmpty + ob]);
        }
        // out = O^T / l + gate * o_c (per-channel gate: gate[d]); a block of 64 tokens (every block but
        // a tile's ragged end) stores without a per-row test
        auto store = [&](int j, uint16_t* dst) {
          const int q = 32 * half + j;
          const float2 rg = rg_s[q];
          const float gq = (a.gate_pc && use_oc) ? bf16_bits_to_f32(__ldg(gsrc_s[q] + d)) : rg.y;
          dst[d] = __bfloat16_as_ushort(__float2bfloat16_rn(fmaf(o[j], rg.x, gq * oc)));
        };
        if (d < D) {
          if (full) {
#pragma unroll
            for (int j = 0; j < 32; ++j) store(j, dst_s[32 * half + j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              uint16_t* dst = dst_s[32 * half + j];
              if (dst != nullptr) store(j, dst);
            }
          }
        }
      }
      named_bar_sync(9, 128);  // smem of this item no longer read
    }
    ROLE_MARK(3);
    if (tid == 0) ROLE_TIMER_SAVE(6);
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace vsa
