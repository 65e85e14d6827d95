// Block-sparse VSA-H3 attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Work item = (b, h, query tile i).  Its key list is every tile for a prefix
// query tile, else the P prefix tiles followed by the tile's selected video
// tiles (ascending).  The list is walked two key tiles (128 keys) at a time.
//
// A query tile is only 64 rows, so the kernel works in the transposed form,
// which keeps every row of the 128-row tcgen05 MMA busy:
//     S^T [128 keys x 64 queries]  = K_blk (M=128, K-major) * Q_tile^T (N=64, K-major)
//     O^T [D x 64 queries]        += V_blk^T (M=D, MN-major) * P^T (N=64, MN-major)
// S^T and O^T live in TMEM (lane = key or d, column = query).  The softmax
// statistics are per query, i.e. per TMEM column, across lanes:
//   - the running maximum m[q] is kept lazily: a block is exponentiated
//     against the current m, and only when some logit exceeds m by more than
//     kRescaleLog2 (or on the first block of an item) is the exact column
//     maximum taken across the 128 lanes and O^T, l rescaled.  Any m with no
//     overflow gives the same softmax, so this is exact up to rounding;
//   - l[q] is kept as per-lane partial sums and reduced once per item.
// D = 64 uses the same M = 128 PV product with a zero upper half of V^T.
//
// Roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner + MMA
// issuer (one thread), warps 2..5 = softmax + epilogue (TMEM lane quadrant =
// warp % 4).  Every mbarrier wait is bounded; after a timeout the kernel
// stops issuing work, finishes its loops without waiting, drains what it
// issued and returns with the status word set.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "prep_kernels.cuh"
#include "ptx.cuh"

namespace vsa {

constexpr int kAttnThreads = 192;
constexpr float kRescaleLog2 = 8.0f;  // lazy-max threshold: exponents stay <= 2^8
constexpr uint32_t kTmemCols = 256;   // S^T double buffer (2 x 64) + O^T (64), rounded to a power of 2

struct AttnArgs {
  const int32_t* idx;         // [B, H, V, topk] global key-tile indices (ascending per row)
  const int32_t* tile_token;  // [n_t * 64]
  const int32_t* tile_valid;  // [n_t]
  const float* o_c;           // [B, H, n_t, D]
  const uint16_t* gate;       // [B, L, H] bf16
  uint16_t* out;              // [B, L, H, D] bf16
  int* status;                // [2] device status word
  int64_t L;
  int H, n_t, P, topk;
  float scale_log2;  // softmax scale * log2(e)
  int64_t n_items;   // B * H * n_t
};

template <int D>
struct AttnLayout {
  static constexpr int kHalves = D / 64;          // 128-byte swizzle atoms along D
  static constexpr int kQBytes = 64 * D * 2;      // one query tile
  static constexpr int kKVBytes = 128 * D * 2;    // 128 keys of K (or of V)
  static constexpr int kHalfBytes = 128 * 128;    // one 64-column half of a 128-row block
  static constexpr int kPBytes = 128 * 64 * 2;    // P^T of one block
  static constexpr int kStages = 2;
  static constexpr int kZeroBytes = (D == 64) ? 16384 : 0;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + 2 * kQBytes;
  static constexpr int oV = oK + kStages * kKVBytes;
  static constexpr int oP = oV + kStages * kKVBytes;
  static constexpr int oZ = oP + 2 * kPBytes;
  static constexpr int oBar = oZ + kZeroBytes;
  // barriers (8 bytes each)
  enum {
    bQFull = 0, bQEmpty = 2, bKFull = 4, bVFull = 6, bKVEmpty = 8, bSFull = 10, bSEmpty = 12,
    bPFull = 14, bPEmpty = 16, bOFull = 18, bOEmpty = 19, bDone = 20, kNumBars = 21
  };
  static constexpr int oMisc = oBar + kNumBars * 8;             // tmem base, abort flag
  static constexpr int oM = ((oMisc + 8 + 15) / 16) * 16;       // float m[64]
  static constexpr int oAlpha = oM + 256;                       // float alpha[64]
  static constexpr int oRed = oAlpha + 256;                     // float red[4][64]
  static constexpr int oLsum = oRed + 1024;                     // float lsum[64]
  static constexpr int oGate = oLsum + 256;                     // float gate[64]
  static constexpr int oQtok = oGate + 256;                     // int qtok[64]
  static constexpr int oTileValid = oQtok + 256;                // uint8 [n_t]
  static size_t bytes(int n_t) {
    const size_t tv = ((static_cast<size_t>(n_t) + 15) / 16) * 16;
    return 1024 /*alignment slack*/ + oTileValid + 2 * tv;
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// In-warp reduce-scatter of 64 per-lane columns: afterwards v[0], v[1] hold the
// reduction over the warp's 32 lanes for columns 2*lane and 2*lane + 1.  The
// input array is consumed.
template <bool kMax>
__device__ __forceinline__ void warp_reduce_scatter64(float* v, int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 32 >> step;      // 32, 16, 8, 4, 2
    const int bit = 4 - step;         // lane bit that picks the kept half
    const bool upper = (lane >> bit) & 1;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float lo = v[i], hi = v[i + half];
      const float send = upper ? lo : hi;
      const float keep = upper ? hi : lo;
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1 << bit);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    vsa_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using Ly = AttnLayout<D>;
  constexpr int kQKSteps = D / 16;
  constexpr int kPVSteps = 128 / 16;
  constexpr uint32_t kIdescS = umma_idesc_bf16(128, 64, 0, 0);
  constexpr uint32_t kIdescPV = umma_idesc_bf16(128, 64, 1, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Ly::oBar);
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(sm + Ly::oMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Ly::oMisc + 4);
  float* m_s = reinterpret_cast<float*>(sm + Ly::oM);
  float* alpha_s = reinterpret_cast<float*>(sm + Ly::oAlpha);
  float* red_s = reinterpret_cast<float*>(sm + Ly::oRed);
  float* lsum_s = reinterpret_cast<float*>(sm + Ly::oLsum);
  float* gate_s = reinterpret_cast<float*>(sm + Ly::oGate);
  int32_t* qtok_s = reinterpret_cast<int32_t*>(sm + Ly::oQtok);
  uint8_t* tile_valid_s = sm + Ly::oTileValid;
  uint8_t* kvalid_s = tile_valid_s + ((a.n_t + 15) / 16) * 16;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_t = a.n_t, P = a.P, topk = a.topk, V = n_t - P;
  const WaitCtl ctl{abort_flag, a.status};

  // ---------------------------------------------------------------- setup
  for (int t = threadIdx.x; t < n_t; t += blockDim.x) tile_valid_s[t] = static_cast<uint8_t>(a.tile_valid[t]);
  if (Ly::kZeroBytes > 0) {
    uint32_t* z = reinterpret_cast<uint32_t*>(sm + Ly::oZ);
    for (int t = threadIdx.x; t < Ly::kZeroBytes / 4; t += blockDim.x) z[t] = 0u;
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[Ly::bQFull + s], 1);
      mbar_init(&bars[Ly::bQEmpty + s], 1);
      mbar_init(&bars[Ly::bKFull + s], 1);
      mbar_init(&bars[Ly::bVFull + s], 1);
      mbar_init(&bars[Ly::bKVEmpty + s], 1);
      mbar_init(&bars[Ly::bSFull + s], 1);
      mbar_init(&bars[Ly::bSEmpty + s], 4);
      mbar_init(&bars[Ly::bPFull + s], 4);
      mbar_init(&bars[Ly::bPEmpty + s], 1);
    }
    mbar_init(&bars[Ly::bOFull], 1);
    mbar_init(&bars[Ly::bOEmpty], 4);
    mbar_init(&bars[Ly::bDone], 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_s, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_s;

  auto list_len = [&](int i) { return (i < P) ? n_t : P + topk; };
  auto key_tile = [&](int64_t bh, int i, int t) -> int {
    if (i < P || t < P) return t;
    return __ldg(a.idx + (bh * V + (i - P)) * topk + (t - P));
  };

  if (warp == 0) {
    // ============================================================ TMA producer
    uint32_t g = 0;
    int it = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; w < a.n_items && ok; w += gridDim.x, ++it) {
      const int64_t bh = w / n_t;
      const int i = static_cast<int>(w - bh * n_t);
      const int nk = list_len(i), nb = (nk + 1) / 2;
      if (lane == 0) {
        const int qb = it & 1;
        ok = mbar_wait(&bars[Ly::bQEmpty + qb], ((it >> 1) & 1) ^ 1, ctl, 1);
        if (ok) {
          mbar_arrive_expect_tx(&bars[Ly::bQFull + qb], Ly::kQBytes);
          const int row = static_cast<int>((bh * n_t + i) * 64);
          for (int hh = 0; hh < Ly::kHalves; ++hh)
            tma_load_2d(sm + Ly::oQ + qb * Ly::kQBytes + hh * 8192, &tm_q, &bars[Ly::bQFull + qb], hh * 64, row);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int n0 = 0; n0 < nb && ok; n0 += 32) {
        const int n = n0 + lane;
        int ta = 0, tb = 0;
        if (n < nb) {
          ta = key_tile(bh, i, 2 * n);
          tb = (2 * n + 1 < nk) ? key_tile(bh, i, 2 * n + 1) : ta;
        }
        const int cnt = min(32, nb - n0);
        for (int j = 0; j < cnt; ++j) {
          const int ka = __shfl_sync(0xffffffffu, ta, j);
          const int kb = __shfl_sync(0xffffffffu, tb, j);
          if (lane == 0 && ok) {
            const int st = g & 1;
            const uint32_t u = g >> 1;
            ok = mbar_wait(&bars[Ly::bKVEmpty + st], (u & 1) ^ 1, ctl, 2);
            if (ok) {
              const int ra = static_cast<int>((bh * n_t + ka) * 64);
              const int rb = static_cast<int>((bh * n_t + kb) * 64);
              uint8_t* kdst = sm + Ly::oK + st * Ly::kKVBytes;
              uint8_t* vdst = sm + Ly::oV + st * Ly::kKVBytes;
              mbar_arrive_expect_tx(&bars[Ly::bKFull + st], Ly::kKVBytes);
              for (int hh = 0; hh < Ly::kHalves; ++hh) {
                tma_load_2d(kdst + hh * Ly::kHalfBytes, &tm_k, &bars[Ly::bKFull + st], hh * 64, ra);
                tma_load_2d(kdst + hh * Ly::kHalfBytes + 8192, &tm_k, &bars[Ly::bKFull + st], hh * 64, rb);
              }
              mbar_arrive_expect_tx(&bars[Ly::bVFull + st], Ly::kKVBytes);
              for (int hh = 0; hh < Ly::kHalves; ++hh) {
                tma_load_2d(vdst + hh * Ly::kHalfBytes, &tm_v, &bars[Ly::bVFull + st], hh * 64, ra);
                tma_load_2d(vdst + hh * Ly::kHalfBytes + 8192, &tm_v, &bars[Ly::bVFull + st], hh * 64, rb);
              }
            }
          }
          ++g;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
      }
    }
    // drain: every load issued must have landed before the CTA may exit
    if (lane == 0) {
      for (int s = 0; s < 2; ++s) {
        if (g > static_cast<uint32_t>(s)) {
          const uint32_t last = (g - 1 - s) >> 1;  // last use of stage ((g - 1 - s) & 1)
          const int st = (g - 1 - s) & 1;
          wait_slow(&bars[Ly::bKFull + st], last & 1, WaitCtl{abort_flag, a.status}, 3);
          wait_slow(&bars[Ly::bVFull + st], last & 1, WaitCtl{abort_flag, a.status}, 3);
        }
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      uint32_t g = 0;
      int it = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t gp, bool first) -> bool {
        const int st = gp & 1;
        const uint32_t u = gp >> 1;
        if (!mbar_wait(&bars[Ly::bVFull + st], u & 1, ctl, 4)) return false;
        if (!mbar_wait(&bars[Ly::bPFull + st], u & 1, ctl, 5)) return false;
        if (first && !mbar_wait(&bars[Ly::bOEmpty], (it & 1) ^ 1, ctl, 6)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sm + Ly::oV + st * Ly::kKVBytes);
        const uint32_t pbase = smem_u32(sm + Ly::oP + st * Ly::kPBytes);
        // V^T atoms along M (= d): the other 64-column half, or the zero region for D = 64
        const uint32_t lbo_v = (D == 128) ? Ly::kHalfBytes
                                          : static_cast<uint32_t>(Ly::oZ - (Ly::oV + st * Ly::kKVBytes));
#pragma unroll
        for (int kk = 0; kk < kPVSteps; ++kk) {
          const uint64_t ad = umma_desc_sw128(vbase + kk * 2048, lbo_v, 1024);
          const uint64_t bd = umma_desc_sw128(pbase + kk * 2048, 8192, 1024);
          umma_ss(tmem + 128, ad, bd, kIdescPV, (!first || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars[Ly::bKVEmpty + st]);
        umma_commit(&bars[Ly::bPEmpty + st]);
        return true;
      };
      for (int64_t w = blockIdx.x; w < a.n_items && ok; w += gridDim.x, ++it) {
        const int64_t bh = w / n_t;
        const int i = static_cast<int>(w - bh * n_t);
        const int nb = (list_len(i) + 1) / 2;
        const int qb = it & 1;
        ok = mbar_wait(&bars[Ly::bQFull + qb], (it >> 1) & 1, ctl, 7);
        const uint32_t qbase = smem_u32(sm + Ly::oQ + qb * Ly::kQBytes);
        for (int n = 0; n < nb && ok; ++n, ++g) {
          const int st = g & 1;
          const uint32_t u = g >> 1;
          ok = mbar_wait(&bars[Ly::bKFull + st], u & 1, ctl, 8) &&
               mbar_wait(&bars[Ly::bSEmpty + st], (u & 1) ^ 1, ctl, 9);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kbase = smem_u32(sm + Ly::oK + st * Ly::kKVBytes);
#pragma unroll
          for (int kk = 0; kk < kQKSteps; ++kk) {
            const uint64_t ad = umma_desc_sw128(kbase + (kk >> 2) * Ly::kHalfBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bd = umma_desc_sw128(qbase + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
            umma_ss(tmem + st * 64, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(&bars[Ly::bSFull + st]);
          if (n == nb - 1) umma_commit(&bars[Ly::bQEmpty + qb]);
          if (n > 0) ok = issue_pv(g - 1, n == 1);
        }
        if (ok) ok = issue_pv(g - 1, nb == 1);
        if (ok) umma_commit(&bars[Ly::bOFull]);
      }
      // drain: all issued tcgen05 work completes before TMEM is released
      umma_commit(&bars[Ly::bDone]);
      wait_slow(&bars[Ly::bDone], 0, WaitCtl{abort_flag, a.status}, 10);
    }
    __syncwarp();
  } else {
    // ============================================================ softmax + epilogue
    const int tid = threadIdx.x - 64;  // 0..127
    const int qd = warp & 3;           // TMEM lane quadrant this warp may access
    const int kl = qd * 32 + lane;     // key lane (S^T) / d lane (O^T)
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
    uint32_t g = 0;
    int it = 0;
    for (int64_t w = blockIdx.x; w < a.n_items; w += gridDim.x, ++it) {
      const int64_t bh = w / n_t;
      const int i = static_cast<int>(w - bh * n_t);
      const int64_t b = bh / a.H;
      const int h = static_cast<int>(bh - b * a.H);
      const int nk = list_len(i), nb = (nk + 1) / 2;
      const int valid_i = tile_valid_s[i];
      for (int t = tid; t < nk; t += 128) kvalid_s[t] = tile_valid_s[key_tile(bh, i, t)];
      if (tid < 64) {
        const int32_t tok = a.tile_token[static_cast<int64_t>(i) * 64 + tid];
        qtok_s[tid] = tok;
        gate_s[tid] = (tok >= 0) ? bf16_bits_to_f32(a.gate[(b * a.L + tok) * a.H + h]) : 0.0f;
      }
      named_bar_sync(1, 128);

      float l[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) l[j] = 0.0f;

      for (int n = 0; n < nb; ++n, ++g) {
        const int sb = g & 1;
        const uint32_t su = g >> 1;
        mbar_wait(&bars[Ly::bSFull + sb], su & 1, ctl, 11);
        tc_fence_after();
        float y[64];
        tmem_ld32(t_lane + sb * 64, y);
        tmem_ld32(t_lane + sb * 64 + 32, y + 32);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Ly::bSEmpty + sb]);

        const int pos = 2 * n + (kl >> 6);
        const int vcount = (pos < nk) ? kvalid_s[pos] : 0;
        const bool valid = (kl & 63) < vcount;
#pragma unroll
        for (int j = 0; j < 64; ++j) y[j] = valid ? y[j] * a.scale_log2 : -INFINITY;

        bool slow = true;
        if (n > 0) {
          float xm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; j += 4) {
            const float4 m4 = *reinterpret_cast<const float4*>(m_s + j);
            xm = fmaxf(xm, fmaxf(fmaxf(y[j] - m4.x, y[j + 1] - m4.y), fmaxf(y[j + 2] - m4.z, y[j + 3] - m4.w)));
          }
          slow = named_bar_or(2, 128, xm > kRescaleLog2);
        }
        if (slow) {
          // exact column maximum of this block: butterfly per column, lane (j % 32) keeps column j
          float cm0 = -INFINITY, cm1 = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            float c = y[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c = fmaxf(c, __shfl_xor_sync(0xffffffffu, c, o));
            if ((j & 31) == lane) {
              if (j < 32) cm0 = c; else cm1 = c;
            }
          }
          red_s[qd * 64 + lane] = cm0;
          red_s[qd * 64 + 32 + lane] = cm1;
          named_bar_sync(3, 128);
          if (tid < 64) {
            const float cm = fmaxf(fmaxf(red_s[tid], red_s[64 + tid]), fmaxf(red_s[128 + tid], red_s[192 + tid]));
            const float mo = (n == 0) ? -INFINITY : m_s[tid];
            float mn = fmaxf(mo, cm);
            if (mn == -INFINITY) mn = 0.0f;
            alpha_s[tid] = (mo == -INFINITY) ? 0.0f : ex2_approx(mo - mn);
            m_s[tid] = mn;
          }
          named_bar_sync(3, 128);
          if (n > 0) {
#pragma unroll
            for (int j = 0; j < 64; ++j) l[j] *= alpha_s[j];
            // O^T holds blocks < n of this item: wait for the last P.V, then rescale its columns
            const uint32_t gp = g - 1;
            mbar_wait(&bars[Ly::bPEmpty + (gp & 1)], (gp >> 1) & 1, ctl, 12);
            tc_fence_after();
#pragma unroll
            for (int hc = 0; hc < 64; hc += 32) {
              float o[32];
              tmem_ld32(t_lane + 128 + hc, o);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= alpha_s[hc + j];
              tmem_st32(t_lane + 128 + hc, o);
            }
            tmem_wait_st();
            tc_fence_before();
          }
        }
        // probabilities, partial row sums, P^T row of this key lane (bf16, 128-byte swizzle)
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(m_s + j);
          y[j] = ex2_approx(y[j] - m4.x);
          y[j + 1] = ex2_approx(y[j + 1] - m4.y);
          y[j + 2] = ex2_approx(y[j + 2] - m4.z);
          y[j + 3] = ex2_approx(y[j + 3] - m4.w);
          l[j] += y[j];
          l[j + 1] += y[j + 1];
          l[j + 2] += y[j + 2];
          l[j + 3] += y[j + 3];
        }
        mbar_wait(&bars[Ly::bPEmpty + sb], (su & 1) ^ 1, ctl, 13);
        uint8_t* prow = sm + Ly::oP + sb * Ly::kPBytes + kl * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          U128 w4;
          w4.x = pack_bf16x2(y[8 * c + 0], y[8 * c + 1]);
          w4.y = pack_bf16x2(y[8 * c + 2], y[8 * c + 3]);
          w4.z = pack_bf16x2(y[8 * c + 4], y[8 * c + 5]);
          w4.w = pack_bf16x2(y[8 * c + 6], y[8 * c + 7]);
          *reinterpret_cast<U128*>(prow + ((c ^ (kl & 7)) << 4)) = w4;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[Ly::bPFull + sb]);
      }

      // ---------------------------------------------------------- epilogue
      warp_reduce_scatter64<false>(l, lane);
      red_s[qd * 64 + 2 * lane] = l[0];
      red_s[qd * 64 + 2 * lane + 1] = l[1];
      named_bar_sync(3, 128);
      if (tid < 64) lsum_s[tid] = (red_s[tid] + red_s[64 + tid]) + (red_s[128 + tid] + red_s[192 + tid]);
      mbar_wait(&bars[Ly::bOFull], it & 1, ctl, 14);
      tc_fence_after();
      float o[64];
      tmem_ld32(t_lane + 128, o);
      tmem_ld32(t_lane + 128 + 32, o + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[Ly::bOEmpty]);
      named_bar_sync(3, 128);  // lsum_s ready
      uint16_t* stage = reinterpret_cast<uint16_t*>(sm + Ly::oP);  // [64 q][D] bf16; P buffers are idle now
      if (kl < D) {
        const float oc = a.o_c[(bh * n_t + i) * D + kl];
#pragma unroll
        for (int q = 0; q < 64; ++q) {
          const float val = o[q] / lsum_s[q] + gate_s[q] * oc;
          stage[q * D + kl] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
        }
      }
      named_bar_sync(3, 128);
      constexpr int kChunks = D / 8;
      for (int e = tid; e < 64 * kChunks; e += 128) {
        const int q = e / kChunks, c = e - q * kChunks;
        if (q < valid_i) {
          const int32_t tok = qtok_s[q];
          uint16_t* dst = a.out + ((b * a.L + tok) * a.H + h) * D + c * 8;
          *reinterpret_cast<U128*>(dst) = *reinterpret_cast<const U128*>(stage + q * D + c * 8);
        }
      }
      named_bar_sync(3, 128);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace vsa
