// Tile gather, pooling, pooled tile scores, top-k selection and the
// compression branch of the VSA-H3 forward.  All of these are bound by HBM or
// L2 traffic, not by arithmetic; the pooled scores keep a pinned binary32
// order so the selection is reproducible bit for bit:
//   pooled = (((+0 + x_0) + x_1) + ... ) / n_valid       (rows in tile order)
//   score  = fl(fma(pq_{D-1}, pk_{D-1}, ... fma(pq_0, pk_0, +0)) * scale)
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace vsa {

constexpr int kTile = 64;

struct alignas(16) U128 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ---------------------------------------------------------------------------
// S2 (+ S3 pooling): sequence order [B, L, H, D] -> tile order [B, H, n_t, 64, D]
// One CTA per (tile, head, batch) moves the tile of Q, K and V with 16-byte
// loads/stores (each 256-byte token row is read by 16 consecutive threads),
// keeps the three tiles in shared memory and, if asked, pools them there.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(384) gather_pool_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    uint16_t* __restrict__ q_t, uint16_t* __restrict__ k_t, uint16_t* __restrict__ v_t,
    float* __restrict__ pq, float* __restrict__ pk, float* __restrict__ pv,
    const int32_t* __restrict__ tile_token, const int32_t* __restrict__ tile_valid, int64_t L, int H,
    int n_t) {
  constexpr int kChunks = D / 8;  // 16-byte chunks per row
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* tiles = reinterpret_cast<uint16_t*>(smem_raw);  // [3][64][D]
  __shared__ int32_t tok_s[kTile];

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const bool pool = (pq != nullptr);
  if (threadIdx.x < kTile) tok_s[threadIdx.x] = tile_token[static_cast<int64_t>(tile) * kTile + threadIdx.x];
  __syncthreads();

  const int64_t dst_base = ((static_cast<int64_t>(b) * H + h) * n_t + tile) * kTile * D;
  const uint16_t* srcs[3] = {q, k, v};
  uint16_t* dsts[3] = {q_t, k_t, v_t};
  for (int e = threadIdx.x; e < 3 * kTile * kChunks; e += blockDim.x) {
    const int tsr = e / (kTile * kChunks);
    const int rem = e - tsr * (kTile * kChunks);
    const int r = rem / kChunks, c = rem - r * kChunks;
    const int32_t tok = tok_s[r];
    U128 val = {0u, 0u, 0u, 0u};
    if (tok >= 0) {
      const uint4* src = reinterpret_cast<const uint4*>(srcs[tsr] + ((static_cast<int64_t>(b) * L + tok) * H + h) * D);
      const uint4 t4 = __ldg(src + c);
      val = U128{t4.x, t4.y, t4.z, t4.w};
    }
    reinterpret_cast<U128*>(dsts[tsr] + dst_base)[r * kChunks + c] = val;
    if (pool) reinterpret_cast<U128*>(tiles + tsr * kTile * D)[r * kChunks + c] = val;
  }
  if (!pool) return;
  __syncthreads();
  const int n = tile_valid[tile];
  float* outs[3] = {pq, pk, pv};
  for (int e = threadIdx.x; e < 3 * D; e += blockDim.x) {
    const int tsr = e / D, d = e - tsr * D;
    const uint16_t* col = tiles + tsr * kTile * D + d;
    float sum = 0.0f;
    for (int r = 0; r < n; ++r) sum = __fadd_rn(sum, bf16_bits_to_f32(col[r * D]));
    outs[tsr][((static_cast<int64_t>(b) * H + h) * n_t + tile) * D + d] = __fdiv_rn(sum, static_cast<float>(n));
  }
}

// ---------------------------------------------------------------------------
// S3 pooling from tile order (the standalone entry point): one CTA per
// (tile, head, batch), one thread per (tensor, d), rows added in tile order.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(384) pool_tiles_kernel(const uint16_t* __restrict__ q_t,
                                                          const uint16_t* __restrict__ k_t,
                                                          const uint16_t* __restrict__ v_t,
                                                          float* __restrict__ pq, float* __restrict__ pk,
                                                          float* __restrict__ pv,
                                                          const int32_t* __restrict__ tile_valid, int H,
                                                          int n_t) {
  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t row0 = ((static_cast<int64_t>(b) * H + h) * n_t + tile);
  const int n = tile_valid[tile];
  const uint16_t* srcs[3] = {q_t, k_t, v_t};
  float* outs[3] = {pq, pk, pv};
  for (int e = threadIdx.x; e < 3 * D; e += blockDim.x) {
    const int tsr = e / D, d = e - tsr * D;
    const uint16_t* col = srcs[tsr] + row0 * kTile * D + d;
    float sum = 0.0f;
    for (int r = 0; r < n; ++r) sum = __fadd_rn(sum, bf16_bits_to_f32(__ldg(col + r * D)));
    outs[tsr][row0 * D + d] = __fdiv_rn(sum, static_cast<float>(n));
  }
}

// ---------------------------------------------------------------------------
// S3 scores: S[bh, i, j] = fl(fma-chain_d(pq[i,d] pk[j,d]) * scale).
// A 64 x 64 block of S per CTA, 4 x 4 outputs per thread, d staged through
// shared memory 32 at a time; every output's chain runs d = 0..D-1 in order.
// ---------------------------------------------------------------------------
constexpr int kScoreBlk = 64;
constexpr int kScoreDk = 32;

__global__ void __launch_bounds__(256) scores_kernel(const float* __restrict__ pq, const float* __restrict__ pk,
                                                      float* __restrict__ S, int n_t, int D, float scale) {
  __shared__ __align__(16) float As[kScoreDk][kScoreBlk + 4];
  __shared__ __align__(16) float Bs[kScoreDk][kScoreBlk + 4];
  const int bh = blockIdx.z;
  const int i0 = blockIdx.y * kScoreBlk, j0 = blockIdx.x * kScoreBlk;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const float* A = pq + static_cast<int64_t>(bh) * n_t * D;
  const float* Bm = pk + static_cast<int64_t>(bh) * n_t * D;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.0f;

  for (int d0 = 0; d0 < D; d0 += kScoreDk) {
    // stage pq[i0..i0+63][d0..d0+31] and pk[j0..][d0..] transposed (d-major)
    for (int e = threadIdx.x; e < kScoreBlk * kScoreDk; e += 256) {
      const int r = e / kScoreDk, dd = e - r * kScoreDk;
      const int i = i0 + r, j = j0 + r;
      As[dd][r] = (i < n_t) ? A[static_cast<int64_t>(i) * D + d0 + dd] : 0.0f;
      Bs[dd][r] = (j < n_t) ? Bm[static_cast<int64_t>(j) * D + d0 + dd] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int dd = 0; dd < kScoreDk; ++dd) {
      const float4 a4 = *reinterpret_cast<const float4*>(&As[dd][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Bs[dd][tx * 4]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = __fmaf_rn(av[a], bv[c], acc[a][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty * 4 + a;
    if (i >= n_t) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + tx * 4 + c;
      if (j < n_t) S[(static_cast<int64_t>(bh) * n_t + i) * n_t + j] = __fmul_rn(acc[a][c], scale);
    }
  }
}

// ---------------------------------------------------------------------------
// S4 top-k: one warp per (bh, video query tile).  The row's video scores go to
// shared memory as order-preserving 32-bit keys; a 32-step bitwise search
// finds the k-th largest key T; the tiles with key > T, plus the lowest-index
// ones with key == T up to k, are emitted in ascending index order.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;  // -0.0 ranks equal to +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_sum(int x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ S, int32_t* __restrict__ idx,
                                                    int BH, int n_t, int P, int k, int rows_per_block) {
  extern __shared__ uint32_t keys_s[];  // [rows_per_block][V]
  const int V = n_t - P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * rows_per_block + warp;
  if (warp >= rows_per_block || row >= static_cast<int64_t>(BH) * V) return;
  const int bh = static_cast<int>(row / V), iv = static_cast<int>(row - static_cast<int64_t>(bh) * V);
  uint32_t* keys = keys_s + static_cast<int64_t>(warp) * V;
  const float* srow = S + (static_cast<int64_t>(bh) * n_t + (P + iv)) * n_t + P;
  for (int j = lane; j < V; j += 32) keys[j] = order_key(__ldg(srow + j));
  __syncwarp();

  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < V; j += 32) cnt += (keys[j] >= cand) ? 1 : 0;
    if (warp_sum(cnt) >= k) T = cand;
  }
  int gt = 0;
  for (int j = lane; j < V; j += 32) gt += (keys[j] > T) ? 1 : 0;
  const int need = k - warp_sum(gt);  // how many of the tiles equal to T to take, lowest index first

  int32_t* out = idx + row * k;
  int written = 0, eq_seen = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int j0 = 0; j0 < V; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = (j < V) ? keys[j] : 0u;
    const bool is_gt = (j < V) && key > T;
    const bool is_eq = (j < V) && key == T;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, is_eq);
    const int eq_before = eq_seen + __popc(eq_ballot & lt_mask);
    const bool take = is_gt || (is_eq && eq_before < need);
    const uint32_t take_ballot = __ballot_sync(0xffffffffu, take);
    if (take) out[written + __popc(take_ballot & lt_mask)] = P + j;
    written += __popc(take_ballot);
    eq_seen += __popc(eq_ballot);
  }
}

// ---------------------------------------------------------------------------
// S4 compression: o_c[bh, i, :] = sum_j softmax_j(S[bh, i, :]) pv[bh, j, :]
// over all n_t tiles, binary32.  A CTA owns 64 rows of one (b, h): first each
// row's max and exp-sum (4 threads per row), then the weighted sum of pooled
// V rows staged 32 tiles at a time.
// ---------------------------------------------------------------------------
constexpr int kCompRows = 64;
constexpr int kCompJ = 32;

template <int D>
__global__ void __launch_bounds__(256) compress_kernel(const float* __restrict__ S, const float* __restrict__ pv,
                                                        float* __restrict__ o_c, int n_t) {
  __shared__ float m_s[kCompRows], inv_s[kCompRows];
  __shared__ __align__(16) float W_s[kCompRows][kCompJ + 1];
  __shared__ __align__(16) float PV_s[kCompJ][D];
  const int bh = blockIdx.y, i0 = blockIdx.x * kCompRows;
  const float* Sb = S + static_cast<int64_t>(bh) * n_t * n_t;
  const float* PVb = pv + static_cast<int64_t>(bh) * n_t * D;

  {  // row statistics: 4 threads per row
    const int r = threadIdx.x >> 2, part = threadIdx.x & 3;
    const int i = i0 + r;
    float m = -INFINITY;
    if (i < n_t)
      for (int j = part; j < n_t; j += 4) m = fmaxf(m, Sb[static_cast<int64_t>(i) * n_t + j]);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float l = 0.0f;
    if (i < n_t)
      for (int j = part; j < n_t; j += 4) l += expf(Sb[static_cast<int64_t>(i) * n_t + j] - m);
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (part == 0) {
      m_s[r] = m;
      inv_s[r] = (i < n_t) ? 1.0f / l : 0.0f;
    }
  }
  __syncthreads();

  constexpr int kCols = D / 32;  // d values per thread: thread owns rows r0..r0+7 (step 8) and d = lane + 32c
  const int lane = threadIdx.x & 31, rgrp = threadIdx.x >> 5;  // 8 row groups of 8 rows
  float acc[8][kCols];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[a][c] = 0.0f;

  for (int j0 = 0; j0 < n_t; j0 += kCompJ) {
    for (int e = threadIdx.x; e < kCompRows * kCompJ; e += 256) {
      const int r = e / kCompJ, jj = e - r * kCompJ;
      const int i = i0 + r, j = j0 + jj;
      W_s[r][jj] = (i < n_t && j < n_t) ? expf(Sb[static_cast<int64_t>(i) * n_t + j] - m_s[r]) : 0.0f;
    }
    for (int e = threadIdx.x; e < kCompJ * D; e += 256) {
      const int jj = e / D, d = e - jj * D;
      const int j = j0 + jj;
      PV_s[jj][d] = (j < n_t) ? PVb[static_cast<int64_t>(j) * D + d] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < kCompJ; ++jj) {
      float pvv[kCols];
#pragma unroll
      for (int c = 0; c < kCols; ++c) pvv[c] = PV_s[jj][lane + 32 * c];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const float w = W_s[rgrp * 8 + a][jj];
#pragma unroll
        for (int c = 0; c < kCols; ++c) acc[a][c] = fmaf(w, pvv[c], acc[a][c]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int r = rgrp * 8 + a, i = i0 + r;
    if (i >= n_t) continue;
#pragma unroll
    for (int c = 0; c < kCols; ++c)
      o_c[(static_cast<int64_t>(bh) * n_t + i) * D + lane + 32 * c] = acc[a][c] * inv_s[r];
  }
}

}  // namespace vsa
