// libvsa: C ABI of the VSA-H3 forward (declared in include/vsa.h).
// Host side: tile plan, argument checks, workspace layout, TMA descriptors
// and the launch sequence.  No allocation happens per call; a plan owns its
// small device tables, the caller owns every tensor and workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>
#include <vector>

#include "attn_pair_sm100.cuh"
#include "attn_sm100.cuh"
#include "prep_kernels.cuh"
#include "vsa.h"

#ifndef VSA_PAIR_PREFIX
#define VSA_PAIR_PREFIX 1
#endif

namespace {

thread_local std::string g_last_error;

vsa_status fail(vsa_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

#define VSA_CUDA_TRY(call)                                                                  \
  do {                                                                                      \
    cudaError_t e_ = (call);                                                                \
    if (e_ != cudaSuccess) return fail(VSA_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

#define VSA_TRY(expr)                 \
  do {                                \
    vsa_status s_ = (expr);           \
    if (s_ != VSA_OK) return s_;      \
  } while (0)

constexpr int kTile = VSA_TILE_SIZE;  // rows of a block in the tile-order copies and the attention kernel

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The resolved problem: prefix segments, video grid and derived counts.
struct Resolved {
  std::vector<int64_t> segments;
  int64_t T = 0, Hg = 0, W = 0;
  int64_t L = 0;
  int64_t n_prefix = 0, n_video = 0;
  int32_t topk = 0;
  float scale = 0.0f;
  int32_t tile = 64;             // tokens per tile (64 or 128)
  int32_t ct = 4, ch = 4, cw = 4;  // video cube shape
  int32_t sh = 0;                // log2(tile / 64): 64-row blocks per tile = 1 << sh
  // reference keep: per prefix tile, 1 for a tile of a reference segment; R of them; kr kept per video
  // query tile
  std::vector<uint8_t> tile_ref;
  int64_t n_ref = 0;
  int32_t kr = 0;
};

// Reference tiles kept per video query tile: max(1, min(ceil(keep * R), R)) in binary64; 0 without any.
int32_t ref_keep_for(double keep, int64_t R) {
  if (R <= 0) return 0;
  double k = std::ceil(keep * static_cast<double>(R));
  if (k > static_cast<double>(R)) k = static_cast<double>(R);
  if (k < 1.0) k = 1.0;
  return static_cast<int32_t>(k);
}

// topk = max(1, min(ceil((1 - sparsity) * V), V)), evaluated in binary64; 0 without video tiles.
int32_t topk_for(double sparsity, int64_t V) {
  if (V <= 0) return 0;
  double k = std::ceil((1.0 - sparsity) * static_cast<double>(V));
  if (k > static_cast<double>(V)) k = static_cast<double>(V);
  if (k < 1.0) k = 1.0;
  return static_cast<int32_t>(k);
}

vsa_status resolve(const vsa_geometry* g, Resolved* r) {
  if (g == nullptr) return fail(VSA_ERR_INVALID_ARG, "geometry is NULL");
  if (g->batch < 1 || g->heads < 1) return fail(VSA_ERR_INVALID_ARG, "batch and heads must be >= 1");
  if (g->gate_per_channel != 0 && g->gate_per_channel != 1)
    return fail(VSA_ERR_INVALID_ARG, "gate_per_channel must be 0 or 1");
  if (g->seq_tiles != 0 && g->seq_tiles != 1) return fail(VSA_ERR_INVALID_ARG, "seq_tiles must be 0 or 1");
  if (g->seq_tiles && g->batch > 4)
    return fail(VSA_ERR_UNSUPPORTED, "seq_tiles needs batch <= 4 (one 5-D tensor map per batch)");
  if (g->qk_fp8 < 0 || g->qk_fp8 > 3) return fail(VSA_ERR_INVALID_ARG, "qk_fp8 must be 0, 1, 2 or 3");
  if (g->qk_fp8 && g->seq_tiles)
    return fail(VSA_ERR_UNSUPPORTED, "qk_fp8 reads 8-bit tile-order copies: it needs seq_tiles = 0");
  if (g->head_dim != 64 && g->head_dim != 96 && g->head_dim != 128)
    return fail(VSA_ERR_UNSUPPORTED, "head_dim must be 64, 96 or 128, got " + std::to_string(g->head_dim));
  if (g->tile_size != 64 && g->tile_size != 128)
    return fail(VSA_ERR_UNSUPPORTED, "tile_size must be 64 or 128, got " + std::to_string(g->tile_size));
  r->tile = g->tile_size;
  r->sh = (g->tile_size == 128) ? 1 : 0;
  if (g->cube_t == 0 && g->cube_h == 0 && g->cube_w == 0) {
    r->ct = 4;
    r->ch = 4;
    r->cw = (g->tile_size == 128) ? 8 : 4;
  } else {
    if (g->cube_t < 1 || g->cube_h < 1 || g->cube_w < 1 ||
        static_cast<int64_t>(g->cube_t) * g->cube_h * g->cube_w != g->tile_size)
      return fail(VSA_ERR_INVALID_ARG, "cube_t * cube_h * cube_w must equal tile_size (or all be 0)");
    r->ct = g->cube_t;
    r->ch = g->cube_h;
    r->cw = g->cube_w;
  }
  if (g->seq_tiles && g->tile_size != 64) return fail(VSA_ERR_UNSUPPORTED, "seq_tiles needs 64-token tiles");
  if (!(g->sparsity >= 0.0 && g->sparsity <= 1.0)) return fail(VSA_ERR_INVALID_ARG, "sparsity must lie in [0, 1]");
  if (g->grid_t < 0 || g->grid_h < 0 || g->grid_w < 0) return fail(VSA_ERR_INVALID_ARG, "negative grid size");
  const bool any_zero = g->grid_t == 0 || g->grid_h == 0 || g->grid_w == 0;
  const bool all_zero = g->grid_t == 0 && g->grid_h == 0 && g->grid_w == 0;
  if (any_zero && !all_zero) return fail(VSA_ERR_SHAPE, "grid sides must be all positive or all zero");
  r->T = g->grid_t;
  r->Hg = g->grid_h;
  r->W = g->grid_w;
  const int64_t n_video_tokens = r->T * r->Hg * r->W;

  r->segments.clear();
  if (g->token_tags != nullptr) {
    if (g->seq_len <= 0) return fail(VSA_ERR_INVALID_ARG, "token_tags needs seq_len > 0");
    // every maximal run of equal tags is one segment
    std::vector<std::pair<int32_t, int64_t>> runs;
    for (int64_t t = 0; t < g->seq_len; ++t) {
      if (runs.empty() || runs.back().first != g->token_tags[t]) runs.push_back({g->token_tags[t], 0});
      runs.back().second += 1;
    }
    size_t n_pre = runs.size();
    if (n_video_tokens > 0) {
      if (runs.back().first != g->video_tag || runs.back().second != n_video_tokens)
        return fail(VSA_ERR_SHAPE, "the last tag run must be the video tokens (T*H*W of video_tag)");
      n_pre -= 1;
    }
    for (size_t s = 0; s < n_pre; ++s) {
      if (runs[s].first == g->video_tag) return fail(VSA_ERR_SHAPE, "video_tag appears before the last run");
      r->segments.push_back(runs[s].second);
    }
  } else {
    if (g->n_segments < 0) return fail(VSA_ERR_INVALID_ARG, "n_segments < 0");
    if (g->n_segments > 0 && g->segment_len == nullptr) return fail(VSA_ERR_INVALID_ARG, "segment_len is NULL");
    for (int s = 0; s < g->n_segments; ++s) {
      if (g->segment_len[s] < 0) return fail(VSA_ERR_INVALID_ARG, "negative segment length");
      r->segments.push_back(g->segment_len[s]);
    }
  }
  int64_t prefix_tokens = 0;
  r->n_prefix = 0;
  for (int64_t n : r->segments) {
    prefix_tokens += n;
    r->n_prefix += (n + r->tile - 1) / r->tile;
  }
  r->L = prefix_tokens + n_video_tokens;
  if (g->token_tags == nullptr && g->seq_len != 0 && g->seq_len != r->L)
    return fail(VSA_ERR_SHAPE, "seq_len " + std::to_string(g->seq_len) + " != prefix + T*H*W = " +
                                   std::to_string(r->L));
  r->n_video = all_zero ? 0 : ((r->T + r->ct - 1) / r->ct) * ((r->Hg + r->ch - 1) / r->ch) *
                                  ((r->W + r->cw - 1) / r->cw);
  const int64_t n_t = r->n_prefix + r->n_video;
  if (n_t > (1 << 24)) return fail(VSA_ERR_UNSUPPORTED, "too many tiles");
  r->topk = topk_for(g->sparsity, r->n_video);
  r->tile_ref.clear();
  r->n_ref = 0;
  r->kr = 0;
  if (g->segment_reference != nullptr) {
    if (g->token_tags != nullptr) return fail(VSA_ERR_INVALID_ARG, "segment_reference needs segment_len, not tags");
    if (!(g->reference_keep > 0.0 && g->reference_keep <= 1.0))
      return fail(VSA_ERR_INVALID_ARG, "reference_keep must lie in (0, 1]");
    for (size_t s = 0; s < r->segments.size(); ++s) {
      const int32_t f = g->segment_reference[s];
      if (f != 0 && f != 1) return fail(VSA_ERR_INVALID_ARG, "segment_reference flags must be 0 or 1");
      const int64_t nt = (r->segments[s] + r->tile - 1) / r->tile;
      r->tile_ref.insert(r->tile_ref.end(), static_cast<size_t>(nt), static_cast<uint8_t>(f));
      if (f) r->n_ref += nt;
    }
    r->kr = (r->n_video > 0) ? ref_keep_for(g->reference_keep, r->n_ref) : 0;
  }
  r->scale = (g->softmax_scale != 0.0f) ? g->softmax_scale
                                        : static_cast<float>(1.0 / std::sqrt(static_cast<double>(g->head_dim)));
  if (!(std::isfinite(r->scale)) || r->scale <= 0.0f) return fail(VSA_ERR_INVALID_ARG, "softmax_scale must be > 0");
  const int64_t rows = static_cast<int64_t>(g->batch) * g->heads * n_t * r->tile;
  if (rows >= (int64_t(1) << 31)) return fail(VSA_ERR_UNSUPPORTED, "B*H*n_tiles*tile_size must stay below 2^31");
  if (static_cast<int64_t>(g->batch) * g->heads > 65535 || g->heads > 65535)
    return fail(VSA_ERR_UNSUPPORTED, "B*H must not exceed 65535");
  return VSA_OK;
}

// Token table of every tile (-1 = pad), valid rows first: tok[tile * r.tile + row].
void build_tables(const Resolved& r, std::vector<int32_t>* tok, std::vector<int32_t>* valid) {
  const int64_t n_t = r.n_prefix + r.n_video, T = r.tile;
  tok->assign(static_cast<size_t>(n_t * T), -1);
  valid->assign(static_cast<size_t>(n_t), 0);
  int64_t tile = 0, base = 0;
  for (int64_t n : r.segments) {
    for (int64_t s = 0; s < n; s += T) {
      const int64_t cnt = std::min<int64_t>(T, n - s);
      for (int64_t j = 0; j < cnt; ++j) (*tok)[tile * T + j] = static_cast<int32_t>(base + s + j);
      (*valid)[tile++] = static_cast<int32_t>(cnt);
    }
    base += n;
  }
  const int64_t nct = (r.T + r.ct - 1) / r.ct, nch = (r.Hg + r.ch - 1) / r.ch, ncw = (r.W + r.cw - 1) / r.cw;
  for (int64_t a = 0; a < nct && r.n_video > 0; ++a)
    for (int64_t bb = 0; bb < nch; ++bb)
      for (int64_t c = 0; c < ncw; ++c) {
        int cnt = 0;
        const int64_t t1 = std::min(r.T, r.ct * a + r.ct), h1 = std::min(r.Hg, r.ch * bb + r.ch),
                      w1 = std::min(r.W, r.cw * c + r.cw);
        for (int64_t t = r.ct * a; t < t1; ++t)
          for (int64_t h = r.ch * bb; h < h1; ++h)
            for (int64_t w = r.cw * c; w < w1; ++w)
              (*tok)[tile * T + cnt++] = static_cast<int32_t>(base + (t * r.Hg + h) * r.W + w);
        (*valid)[tile++] = cnt;
      }
}

// Key mask of every 64-row block of the tile-order copies: the low `valid rows of the block` bits
// (a tile holds its valid rows first, so block j of a tile holds min(64, max(0, valid - 64 j))).
void build_block_masks(const Resolved& r, const std::vector<int32_t>& valid, std::vector<uint64_t>* mask) {
  const int sub = 1 << r.sh;
  mask->assign(valid.size() * sub, 0);
  for (size_t i = 0; i < valid.size(); ++i)
    for (int j = 0; j < sub; ++j) {
      const int v = std::min(64, std::max(0, valid[i] - 64 * j));
      (*mask)[i * sub + j] = v >= 64 ? ~0ull : ((1ull << v) - 1);
    }
}

// Tables for reading tiles straight from sequence order with TMA: a tile is one box, a 64-token run of
// a prefix segment (4-D map over [b, token, head, d]) or a 4x4x4 cube of the video grid (5-D map over
// [t, y, x, head, d] per batch).  Box row r is the token at position r of the run, or cube position
// ((t - t0)*4 + (y - y0))*4 + (x - x0); rows outside the segment or the grid are masked.
//   row_token[tile*64 + r]: token of box row r, -1 if masked
//   mask_seq[tile]: bit r set when box row r is a token of the tile
//   coord[tile]: {0, first token, 0, 0} for a prefix run, {1, x0, y0, t0} for a cube
// (64-token tiles only.)
void build_seq_tables(const Resolved& r, const std::vector<uint64_t>& mask_tiled, std::vector<int32_t>* row_token,
                      std::vector<uint64_t>* mask_seq, std::vector<int32_t>* coord) {
  const int64_t n_t = r.n_prefix + r.n_video;
  row_token->assign(static_cast<size_t>(n_t * kTile), -1);
  mask_seq->assign(static_cast<size_t>(n_t), 0);
  coord->assign(static_cast<size_t>(n_t * 4), 0);
  int64_t tile = 0, base = 0;
  for (int64_t n : r.segments) {
    for (int64_t s = 0; s < n; s += kTile) {
      const int64_t cnt = std::min<int64_t>(kTile, n - s);
      for (int64_t j = 0; j < cnt; ++j) (*row_token)[tile * kTile + j] = static_cast<int32_t>(base + s + j);
      (*mask_seq)[tile] = mask_tiled[tile];
      (*coord)[tile * 4 + 1] = static_cast<int32_t>(base + s);
      ++tile;
    }
    base += n;
  }
  const int64_t ct = (r.T + 3) / 4, ch = (r.Hg + 3) / 4, cw = (r.W + 3) / 4;
  for (int64_t a = 0; a < ct && r.n_video > 0; ++a)
    for (int64_t bb = 0; bb < ch; ++bb)
      for (int64_t c = 0; c < cw; ++c) {
        uint64_t m = 0;
        for (int64_t t = 0; t < 4; ++t)
          for (int64_t h = 0; h < 4; ++h)
            for (int64_t w = 0; w < 4; ++w) {
              const int64_t tt = 4 * a + t, hh = 4 * bb + h, ww = 4 * c + w;
              if (tt >= r.T || hh >= r.Hg || ww >= r.W) continue;
              const int64_t row = (t * 4 + h) * 4 + w;
              (*row_token)[tile * kTile + row] = static_cast<int32_t>(base + (tt * r.Hg + hh) * r.W + ww);
              m |= 1ull << row;
            }
        (*mask_seq)[tile] = m;
        int32_t* cd = coord->data() + tile * 4;
        cd[0] = 1;
        cd[1] = static_cast<int32_t>(4 * c);
        cd[2] = static_cast<int32_t>(4 * bb);
        cd[3] = static_cast<int32_t>(4 * a);
        ++tile;
      }
}

// seq_tiles: no tile-order copies (their regions are empty).
// qk_fp8: q_t and k_t hold 8-bit codes, 128 bytes per row whatever D, and q_s, k_s one float per row.
// tile: tokens per tile (the copies hold n_t * tile rows per (b, h)).
// q_n and kv_max hold the attention's overflow-bound statistics: the norm of every query row (tile-order
// rows; with qk_fp8 of the dequantised row) and, per (b, h), the largest key norm and |v| (two floats).
vsa_workspace_layout make_layout(int64_t B, int64_t H, int64_t D, int64_t n_t, int64_t tile, int64_t V, int64_t topk,
                                 bool seq_tiles,
                                 bool qk_fp8, bool qk_split = false, bool fp4 = false) {
  vsa_workspace_layout w{};
  size_t off = 0;
  const size_t rows = static_cast<size_t>(B * H * n_t * tile);
  const size_t tiles = seq_tiles ? 0 : rows * D * 2;
  const size_t qk_tiles = qk_fp8 ? rows * vsa::kF8RowBytes : tiles;
  const bool scales = qk_fp8 || qk_split;
  const size_t pooled = static_cast<size_t>(B * H * n_t * D * 4);
  w.q_t = off; off += align256(qk_tiles);
  w.k_t = off; off += align256(qk_tiles);
  w.v_t = off; off += align256(tiles);
  w.q_s = off; off += align256(scales ? rows * 4 : 0);
  w.k_s = off; off += align256(scales ? rows * 4 : 0);
  w.q_n = off; off += align256(rows * 4);
  w.kv_max = off; off += align256(static_cast<size_t>(B * H * 8));
  w.pq = off; off += align256(pooled);
  w.pk = off; off += align256(pooled);
  w.pv = off; off += align256(pooled);
  w.scores = off; off += align256(static_cast<size_t>(B * H * n_t * n_t * 4));
  w.idx = off; off += align256(static_cast<size_t>(B * H * V * topk * 4));
  w.o_c = off; off += align256(pooled);
  // prefix split: 8-bit codes of Q and K beside the bf16 copies, and their overflow-bound statistics
  w.q_c = off; off += align256(qk_split ? rows * vsa::kF8RowBytes : 0);
  w.k_c = off; off += align256(qk_split ? rows * vsa::kF8RowBytes : 0);
  w.q_n8 = off; off += align256(qk_split ? rows * 4 : 0);
  w.kv_max8 = off; off += align256(qk_split ? static_cast<size_t>(B * H * 8) : 0);
  // FP4 video query tiles: the binary64 key column sums and the key means
  w.k_sum = off; off += align256(fp4 ? static_cast<size_t>(B * H * D * 8) : 0);
  w.k_mu = off; off += align256(fp4 ? static_cast<size_t>(B * H * D * 4) : 0);
  w.total = off;
  return w;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

vsa_status get_encoder(EncodeTiledFn* out) {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  static std::string err;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || p == nullptr)
      err = "cuTensorMapEncodeTiled is not available from the driver";
    else
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (fn == nullptr) return fail(VSA_ERR_CUDA, err);
  *out = fn;
  return VSA_OK;
}

// Tile-order tensor [rows, D] bf16 as a 2-D map with 64 x 64 boxes, 128-byte swizzle.
vsa_status make_tile_map(CUtensorMap* m, const void* base, int64_t rows, int D) {
  EncodeTiledFn enc;
  VSA_TRY(get_encoder(&enc));
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string(r));
  return VSA_OK;
}

// 8-bit tile-order codes [rows, 128 bytes] as a 2-D map with 128-byte x 64-row boxes, 128-byte swizzle.
vsa_status make_code_map(CUtensorMap* m, const void* base, int64_t rows) {
  EncodeTiledFn enc;
  VSA_TRY(get_encoder(&enc));
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(vsa::kF8RowBytes), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(vsa::kF8RowBytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(vsa::kF8RowBytes), 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled (8-bit map) failed with code " + std::to_string(r));
  return VSA_OK;
}

// Maps for reading q, k or v [B, L, H, D] straight from sequence order (SeqMaps): the prefix as a 4-D
// tensor [B][L][H][D] with one box per 64-token run (box 64 d x 1 head x 64 tokens x 1 batch), the video
// of batch b as a 5-D tensor [T][Hg][W][H][D] starting at token b*L + P with one box per 4x4x4 cube.
// Out-of-range box rows (past the sequence or the grid) are filled with zeros and masked.
vsa_status make_seq_maps(CUtensorMap* prefix, CUtensorMap* video, const void* base, int64_t B, int64_t L, int64_t H,
                         int64_t D, int64_t P, int64_t T, int64_t Hg, int64_t W) {
  EncodeTiledFn enc;
  VSA_TRY(get_encoder(&enc));
  const cuuint64_t e = 2;  // bytes per element
  {
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L),
                          static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {D * e, H * D * e, L * H * D * e};
    cuuint32_t box[4] = {64, 1, 64, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(prefix, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled (prefix map) failed: " + std::to_string(r));
  }
  if (T * Hg * W == 0) return VSA_OK;
  for (int64_t b = 0; b < B; ++b) {
    const auto* vbase = static_cast<const uint8_t*>(base) + ((b * L + P) * H * D) * e;
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(W),
                          static_cast<cuuint64_t>(Hg), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[4] = {D * e, H * D * e, W * H * D * e, Hg * W * H * D * e};
    cuuint32_t box[5] = {64, 1, 4, 4, 4};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(video + b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<uint8_t*>(vbase), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VSA_ERR_CUDA, "cuTensorMapEncodeTiled (video map) failed: " + std::to_string(r));
  }
  return VSA_OK;
}

}  // namespace

// Scratch of vsa_forward_noalloc: one array per device, alive until the
// process exits, shared by every call on that device.  Host code never uses
// its name as an address; the device address is looked up once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[VSA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 128;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on `device` (the current device).
vsa_status noalloc_scratch_address(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return fail(VSA_ERR_DEVICE, "device ordinal out of range");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[device] == nullptr) {
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
    if (e != cudaSuccess || addr == nullptr)
      return fail(VSA_ERR_CUDA, std::string("cudaGetSymbolAddress of the no-alloc scratch: ") + cudaGetErrorString(e));
    g_noalloc_addr[device] = addr;
  }
  *out = g_noalloc_addr[device];
  return VSA_OK;
}

}  // namespace

struct vsa_plan_s {
  int device = 0;
  int num_sms = 0;
  size_t max_smem = 0;
  int32_t B = 0, H = 0, D = 0;
  int32_t gate_pc = 0;  // gate [B, L, H*D] (1) or [B, L, H] (0)
  // vsa_forward_parts: the part pointer table (host copy and device copy, 5 operands x kMaxParts)
  std::vector<const void*> part_table;
  const void** d_part_table = nullptr;
  bool seq_tiles = false;  // the attention reads tiles from sequence order (no tile-order copies)
  bool qk_fp8 = false;     // 8-bit Q/K (E4M3 codes, one scale per token and head) for the fine logits
  bool qk_split = false;   // the same for the dense prefix query tiles only; video query tiles keep bf16
  bool fp4 = false;        // with qk_split: the video query tiles' logits from FP4 Q and smoothed FP4 K
  // bf16 attention: the dense prefix query row blocks run two at a time on vsa_attn_pair_kernel (built
  // with VSA_PAIR_PREFIX=0 they stay on vsa_attn_kernel, one at a time)
  bool pair_prefix = VSA_PAIR_PREFIX != 0;
  Resolved r;
  int32_t n_t = 0, P = 0, V = 0, topk = 0;
  // reference keep: kr of the n_ref reference tiles kept per video query tile (idx rows hold kr + topk);
  // the always-kept prefix tiles and the reference tiles (device copies only when n_ref > 0)
  int32_t kr = 0, n_ref = 0;
  std::vector<int32_t> exempt_tiles, ref_tiles;
  int32_t* d_exempt = nullptr;
  int32_t* d_refs = nullptr;
  std::vector<int32_t> tile_token, tile_valid;
  int32_t* d_tile_token = nullptr;
  int32_t* d_tile_valid = nullptr;
  // key masks of the 64-row blocks of the tile-order copies (build_block_masks), and the tables for
  // TMA loads straight from sequence order (build_seq_tables, 64-token tiles)
  std::vector<int32_t> row_token, coord;
  std::vector<uint64_t> mask_seq, mask_tiled;
  int32_t* d_row_token = nullptr;
  int32_t* d_coord = nullptr;  // [n_t][4]
  uint64_t* d_mask_seq = nullptr;
  uint64_t* d_mask_tiled = nullptr;
  // vsa_sparse_attn_fwd (bf16 plans): the overflow-bound statistics of its tile-order inputs, query row
  // norms then the (b, h) maxima
  float* d_stats = nullptr;
  // [0] error code, [1] failure site, [2] attention item counter, [3] gate nonzero, [4] pair-kernel item
  // counter, [5] and [6] the two counters of a second attention launch running concurrently
  int* d_status = nullptr;
  vsa_workspace_layout ws{};
  // Head-slice plans share the parent's device tables and status word and own nothing on the device.
  bool owns_device = true;
  // vsa_forward_host: head-slice plans for chunks of `hc` heads (and the remainder), and the copy streams
  // and events of its pipeline.  Created on first use, released with the plan.
  struct HostPipe {
    int32_t hc = 0;
    vsa_plan_s* sub = nullptr;       // hc heads
    vsa_plan_s* sub_last = nullptr;  // H % hc heads, when H is not a multiple of hc
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t ev_in[2] = {}, ev_comp[2] = {}, ev_out[2] = {}, ev_gate = nullptr, ev_start = nullptr;
  } pipe;
  // the prefix pair kernel runs on `side`, forked from and joined back to the caller's stream, so that
  // vsa_attn_kernel starts on the SMs its last items leave idle (created on first use)
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr, ev_split = nullptr;
};

namespace {

vsa_status check_plan(vsa_plan p) {
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  int dev = -1;
  VSA_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != p->device) return fail(VSA_ERR_INVALID_ARG, "the current device is not the plan's device");
  return VSA_OK;
}

vsa_status check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs) {
    if (q == nullptr) return fail(VSA_ERR_INVALID_ARG, "a required device pointer is NULL");
    if (!aligned16(q)) return fail(VSA_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  }
  return VSA_OK;
}

vsa_status launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(VSA_ERR_CUDA, std::string(what) + " launch: " + cudaGetErrorString(e));
  return VSA_OK;
}

// Opt in to `bytes` of dynamic shared memory (static shared memory counts
// against the same default 48 KB, so the attribute is always set).
template <typename K>
vsa_status allow_smem(K kernel, size_t bytes) {
  if (bytes > 0)
    VSA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)));
  return VSA_OK;
}

// Calls f(std::integral_constant<int, D>{}) for the plan's head dimension (64, 96 or 128).
template <typename F>
vsa_status with_head_dim(int D, F&& f) {
  switch (D) {
    case 64: return f(std::integral_constant<int, 64>{});
    case 96: return f(std::integral_constant<int, 96>{});
    case 128: return f(std::integral_constant<int, 128>{});
    default: return fail(VSA_ERR_UNSUPPORTED, "head_dim must be 64, 96 or 128");
  }
}

// One sequence-order tensor per operand, all heads of the plan.
vsa::PartIO single_io(vsa_plan p) { return vsa::PartIO{nullptr, 1, p->r.L, p->H, 0}; }

// qs/ks: with an 8-bit plan, the per-row scales (qt/kt then receive codes).
// qn/kv (with pooling): the overflow-bound statistics of the staged tiles (8-bit Q/K: Q/K norms from the
// codes); kv must hold zeros on entry (the kernel raises it with atomicMax).
// f8: write Q and K as 8-bit codes (qt, kt: 128-byte code rows, qs, ks: row scales); vt NULL without
// pooling: V is not read.
vsa_status run_gather(vsa_plan p, const void* q, const void* k, const void* v, void* qt, void* kt, void* vt, float* pq,
                      float* pk, float* pv, cudaStream_t s, const vsa::PartIO* io = nullptr, float* qs = nullptr,
                      float* ks = nullptr, float* qn = nullptr, uint32_t* kv = nullptr, int f8 = -1,
                      int q_tiles = -1) {
  const bool codes = (f8 < 0) ? p->qk_fp8 : (f8 != 0);
  const vsa::PartIO pio = io ? *io : single_io(p);
  if (p->n_t == 0) return VSA_OK;
  const bool pool = pq != nullptr;
  // q_tiles: a codes-only pass (no pooling, no V) writes Q for tiles [0, q_tiles) only
  if (q_tiles < 0) q_tiles = p->n_t;
  if (q_tiles < p->n_t && (pool || vt != nullptr)) return fail(VSA_ERR_INVALID_ARG, "partial Q needs a codes-only pass");
  const size_t smem = pool ? static_cast<size_t>(3) * p->r.tile * p->D * 2 : 0;
  dim3 grid(p->n_t, p->H, p->B);
  const auto* qq = static_cast<const uint16_t*>(q);
  const auto* kk = static_cast<const uint16_t*>(k);
  const auto* vv = static_cast<const uint16_t*>(v);
  auto* vo = static_cast<uint16_t*>(vt);
  auto launch = [&](auto kernel) -> vsa_status {
    VSA_TRY(allow_smem(kernel, smem));
    kernel<<<grid, 384, smem, s>>>(qq, kk, vv, qt, kt, vo, qs, ks, pq, pk, pv, p->d_tile_token, p->d_tile_valid,
                                   p->r.L, p->H, p->n_t, pio, qn, kv, q_tiles);
    return VSA_OK;
  };
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    const bool parts = pio.table != nullptr;
    auto by_tile = [&](auto k64, auto k128) { return p->r.sh ? launch(k128) : launch(k64); };
    if (codes)
      return parts ? by_tile(vsa::gather_pool_kernel<D, true, true, 1>, vsa::gather_pool_kernel<D, true, true, 2>)
                   : by_tile(vsa::gather_pool_kernel<D, false, true, 1>, vsa::gather_pool_kernel<D, false, true, 2>);
    return parts ? by_tile(vsa::gather_pool_kernel<D, true, false, 1>, vsa::gather_pool_kernel<D, true, false, 2>)
                 : by_tile(vsa::gather_pool_kernel<D, false, false, 1>, vsa::gather_pool_kernel<D, false, false, 2>);
  }));
  return launch_check("gather_pool");
}

// Plan-owned statistics of the step attention: row norms (256-aligned), then B*H float pairs.
size_t stats_rows_bytes(const vsa_plan_s* p) {
  return align256(static_cast<size_t>(p->B) * p->H * p->n_t * p->r.tile * 4);
}
size_t stats_bytes(const vsa_plan_s* p) { return stats_rows_bytes(p) + static_cast<size_t>(p->B) * p->H * 8; }

// The overflow-bound statistics of tile-order copies (what the gather computes while pooling); kv is
// zeroed here.
vsa_status run_tile_stats(vsa_plan p, const void* qt, const void* kt, const void* vt, float* qn, uint32_t* kv,
                          cudaStream_t s) {
  VSA_CUDA_TRY(cudaMemsetAsync(kv, 0, static_cast<size_t>(p->B) * p->H * 8, s));
  if (p->n_t == 0) return VSA_OK;
  const size_t smem = static_cast<size_t>(3) * p->r.tile * p->D * 2;
  dim3 grid(p->n_t, p->H, p->B);
  const auto* a = static_cast<const uint16_t*>(qt);
  const auto* b = static_cast<const uint16_t*>(kt);
  const auto* c = static_cast<const uint16_t*>(vt);
  auto launch = [&](auto kernel) -> vsa_status {
    VSA_TRY(allow_smem(kernel, smem));
    kernel<<<grid, 384, smem, s>>>(a, b, c, qn, kv, p->H, p->n_t);
    return VSA_OK;
  };
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    return p->r.sh ? launch(vsa::tile_stats_kernel<D, 128>) : launch(vsa::tile_stats_kernel<D, 64>);
  }));
  return launch_check("tile statistics");
}

// FP4 video query tiles: the key means of the key copy (binary64 column sums, then / L), the FP4 rounding
// of the video query tiles of qt and of every key tile of kt (smoothed) in place, and the overflow-bound
// statistics of the rounded copies.
vsa_status run_fp4(vsa_plan p, void* qt, void* kt, const void* vt, double* ksum, float* mu, float* qn, uint32_t* kv,
                   cudaStream_t s) {
  if (p->n_t == 0) return VSA_OK;
  const int64_t BH = static_cast<int64_t>(p->B) * p->H;
  if (BH > 65535) return fail(VSA_ERR_UNSUPPORTED, "FP4 key means: batch * heads must be <= 65535");
  const int64_t rows = static_cast<int64_t>(p->n_t) * p->r.tile;  // key rows per (b, h)
  const int per_cta = 512;
  VSA_CUDA_TRY(cudaMemsetAsync(ksum, 0, static_cast<size_t>(BH) * p->D * sizeof(double), s));
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    const dim3 grid(static_cast<unsigned>((rows + per_cta - 1) / per_cta), static_cast<unsigned>(BH));
    vsa::key_sum_kernel<D><<<grid, 128, 0, s>>>(static_cast<const uint16_t*>(kt), ksum, rows, per_cta);
    return VSA_OK;
  }));
  VSA_TRY(launch_check("key sums"));
  const int64_t nm = BH * p->D;
  vsa::key_mean_kernel<<<static_cast<unsigned>((nm + 255) / 256), 256, 0, s>>>(ksum, mu, nm,
                                                                               static_cast<double>(p->r.L));
  VSA_TRY(launch_check("key means"));
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    const int64_t n_rows = BH * rows;
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((n_rows * (D / 16) + 255) / 256, 16LL * p->num_sms));
    vsa::fp4_round_tiles_kernel<D><<<dim3(static_cast<unsigned>(blocks), 2), 256, 0, s>>>(
        static_cast<uint16_t*>(qt), static_cast<uint16_t*>(kt), mu, p->d_tile_valid, p->n_t, p->r.tile, p->P, n_rows);
    return VSA_OK;
  }));
  VSA_TRY(launch_check("FP4 rounding"));
  return run_tile_stats(p, qt, kt, vt, qn, kv, s);
}

vsa_status run_pool(vsa_plan p, const void* qt, const void* kt, const void* vt, float* pq, float* pk, float* pv,
                    cudaStream_t s) {
  if (p->n_t == 0) return VSA_OK;
  dim3 grid(p->n_t, p->H, p->B);
  const auto* a = static_cast<const uint16_t*>(qt);
  const auto* b = static_cast<const uint16_t*>(kt);
  const auto* c = static_cast<const uint16_t*>(vt);
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    vsa::pool_tiles_kernel<D><<<grid, 384, 0, s>>>(a, b, c, pq, pk, pv, p->d_tile_valid, p->H, p->n_t, p->r.tile);
    return VSA_OK;
  }));
  return launch_check("pool_tiles");
}

vsa_status run_scores(vsa_plan p, const float* pq, const float* pk, float* S, cudaStream_t s) {
  if (p->n_t == 0) return VSA_OK;
  const int nb = (p->n_t + vsa::kScoreBlk - 1) / vsa::kScoreBlk;
  dim3 grid(nb, nb, p->B * p->H);
  vsa::scores_kernel<<<grid, 256, 0, s>>>(pq, pk, S, p->n_t, p->D, p->r.scale);
  return launch_check("scores");
}

vsa_status run_topk(vsa_plan p, const float* S, const float* pv, int32_t* idx, float* o_c, cudaStream_t s,
                    const int* gate_nonzero = nullptr) {
  if (p->n_t == 0) return VSA_OK;
  const int64_t BH = static_cast<int64_t>(p->B) * p->H;
  // one selection per video query tile over `ncols` candidates (the video tiles, or the listed reference
  // tiles), written at column `off` of idx rows kr + topk wide
  auto select = [&](const int32_t* cols, int ncols, int k, int off) -> vsa_status {
    const size_t row_bytes = static_cast<size_t>(ncols) * 4;
    int rows = static_cast<int>(std::min<size_t>(8, std::max<size_t>(1, (200 * 1024) / row_bytes)));
    const size_t smem = row_bytes * rows;
    if (smem > p->max_smem) return fail(VSA_ERR_UNSUPPORTED, "too many candidate tiles for the top-k kernel");
    VSA_TRY(allow_smem(vsa::topk_kernel, smem));
    const int64_t nrows = BH * p->V;
    const int64_t blocks = (nrows + rows - 1) / rows;
    if (blocks > 0x7fffffff) return fail(VSA_ERR_UNSUPPORTED, "top-k grid too large");
    vsa::topk_kernel<<<static_cast<unsigned>(blocks), 256, smem, s>>>(S, idx, static_cast<int>(BH), p->n_t, p->P,
                                                                     k, rows, cols, ncols, p->kr + p->topk, off);
    return launch_check("topk");
  };
  if (p->V > 0 && p->kr > 0) VSA_TRY(select(p->d_refs, p->n_ref, p->kr, 0));
  dim3 grid((p->n_t + vsa::kCompRows - 1) / vsa::kCompRows, static_cast<unsigned>(BH));
  // Up to 40 x 32 tiles: the video top-k and the compression in one pass over each score row (a row's
  // keys held in registers); longer rows: the top-k kernel, then the compression kernel.
  const int J = (p->n_t + 31) / 32;
  const int k = (p->V > 0) ? p->topk : 0;
  if (J <= 40) {
    VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
      constexpr int D = decltype(dc)::value;
      auto launch = [&](auto kernel) {
        VSA_TRY(allow_smem(kernel, vsa::kTcSmem));
        kernel<<<grid, 256, vsa::kTcSmem, s>>>(S, pv, o_c, idx, p->n_t, p->P, k, p->kr + p->topk, p->kr, gate_nonzero,
                                               p->d_status);
        return VSA_OK;
      };
      if (J <= 8) return launch(vsa::select_compress_kernel<D, 8>);
      if (J <= 16) return launch(vsa::select_compress_kernel<D, 16>);
      if (J <= 24) return launch(vsa::select_compress_kernel<D, 24>);
      return launch(vsa::select_compress_kernel<D, 40>);
    }));
    return launch_check("select_compress");
  }
  if (k > 0) VSA_TRY(select(nullptr, p->V, p->topk, p->kr));
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    vsa::compress_kernel<D><<<grid, 256, 0, s>>>(S, pv, o_c, p->n_t, gate_nonzero);
    return VSA_OK;
  }));
  return launch_check("compress");
}

// qt/kt/vt: tile-order copies; or, with seq_qkv (q, k, v in sequence order), the kernel reads the
// tiles itself (needs B <= kSeqMaxBatch).
// Makes the plan's side stream (and its events) on first use and orders it after the work queued on s.
vsa_status fork_side(vsa_plan p, cudaStream_t s) {
  if (p->side == nullptr) {
    VSA_CUDA_TRY(cudaStreamCreateWithFlags(&p->side, cudaStreamNonBlocking));
    VSA_CUDA_TRY(cudaEventCreateWithFlags(&p->ev_fork, cudaEventDisableTiming));
    VSA_CUDA_TRY(cudaEventCreateWithFlags(&p->ev_join, cudaEventDisableTiming));
    VSA_CUDA_TRY(cudaEventCreateWithFlags(&p->ev_split, cudaEventDisableTiming));
  }
  VSA_CUDA_TRY(cudaEventRecord(p->ev_fork, s));
  VSA_CUDA_TRY(cudaStreamWaitEvent(p->side, p->ev_fork, 0));
  return VSA_OK;
}

vsa_status run_attn(vsa_plan p, const void* qt, const void* kt, const void* vt, const int32_t* idx, const float* o_c,
                    const void* gate, void* out, cudaStream_t s, int gate_ld = 0, const int* gate_nonzero = nullptr,
                    const void* const* seq_qkv = nullptr, const vsa::PartIO* io = nullptr, const float* qs = nullptr,
                    const float* ks = nullptr, const float* qn = nullptr, const uint32_t* kv = nullptr, int f8 = -1,
                    int s_lo = 0, int n_s = -1, bool alt_counters = false) {
  if (p->n_t == 0) return VSA_OK;
  const bool seq = (seq_qkv != nullptr);
  const bool codes = (f8 < 0) ? p->qk_fp8 : (f8 != 0);  // Q and K as 8-bit codes (8-bit S^T product)
  // the kernel works in 64-row blocks: one per tile, or two per 128-token tile
  const int64_t n_rb = static_cast<int64_t>(p->n_t) << p->r.sh;
  const int64_t rows = static_cast<int64_t>(p->B) * p->H * n_rb * kTile;
  CUtensorMap mq{}, mk{}, mv{};
  vsa::SeqMaps sm{};
  if (seq) {
    if (p->B > vsa::kSeqMaxBatch) return fail(VSA_ERR_UNSUPPORTED, "sequence-order attention needs batch <= 4");
    const int64_t vid = p->r.T * p->r.Hg * p->r.W;
    for (int t = 0; t < 3; ++t)
      VSA_TRY(make_seq_maps(&sm.prefix[t], sm.video[t], seq_qkv[t], p->B, p->r.L, p->H, p->D, p->r.L - vid, p->r.T,
                            p->r.Hg, p->r.W));
  } else if (codes) {
    VSA_TRY(make_code_map(&mq, qt, rows));
    VSA_TRY(make_code_map(&mk, kt, rows));
    VSA_TRY(make_tile_map(&mv, vt, rows, p->D));
  } else {
    VSA_TRY(make_tile_map(&mq, qt, rows, p->D));
    VSA_TRY(make_tile_map(&mk, kt, rows, p->D));
    VSA_TRY(make_tile_map(&mv, vt, rows, p->D));
  }
  if (codes && (qs == nullptr || ks == nullptr)) return fail(VSA_ERR_INVALID_ARG, "8-bit Q/K needs its scales");
  vsa::AttnArgs a{};
  a.idx = idx;
  a.tile_token = seq ? p->d_row_token : p->d_tile_token;  // query row -> token (-1: not stored)
  a.tile_valid = p->d_tile_valid;
  a.key_mask = seq ? p->d_mask_seq : p->d_mask_tiled;
  a.coord = p->d_coord;
  a.o_c = o_c;
  a.gate = static_cast<const uint16_t*>(gate);
  a.out = static_cast<uint16_t*>(out);
  a.status = p->d_status;
  // item counters: [2] (video kernel) and [4] (pair kernel), or [5] and [6] for a launch that runs
  // concurrently with another run_attn on the same plan
  a.sched = p->d_status + (alt_counters ? 5 : 2);
  a.L = p->r.L;
  a.H = p->H;
  a.gate_pc = p->gate_pc;
  a.gate_nonzero = gate_nonzero;
  a.io = io ? *io : single_io(p);
  a.q_scale = qs;
  a.k_scale = ks;
  // overflow bound: P <= 2^gap per key, so l <= keys * 2^gap < 2^126 (its reciprocal stays normal) and
  // |O| <= keys * 2^gap * max|v| < 2^125 when gap <= 124 - ceil(log2 keys) - ceil(log2 max|v|)+
  if (qn != nullptr && kv != nullptr) {
    int lg = 0;
    while ((int64_t{1} << lg) < static_cast<int64_t>(p->n_t) * p->r.tile) ++lg;
    a.q_norm = qn;
    a.kv_max = reinterpret_cast<const float*>(kv);
    a.skip_cap = static_cast<float>(124 - lg);
  }
  a.gate_ld = gate_ld > 0 ? gate_ld : (p->gate_pc ? p->H * p->D : p->H);
  a.n_t = static_cast<int>(n_rb);
  a.sub_shift = p->r.sh;
  a.P = p->P;
  a.topk = p->topk;
  a.kr = p->kr;
  a.n_exempt = p->n_ref > 0 ? static_cast<int>(p->exempt_tiles.size()) : p->P;
  a.exempt = p->n_ref > 0 ? p->d_exempt : nullptr;
  a.scale_log2 = static_cast<float>(static_cast<double>(p->r.scale) * 1.4426950408889634);
  // the row blocks this launch covers: [s_lo, s_lo + n_s) of every (b, h)
  if (n_s < 0) n_s = static_cast<int>(n_rb) - s_lo;
  if (s_lo < 0 || n_s < 0 || s_lo + n_s > n_rb) return fail(VSA_ERR_INVALID_ARG, "attention row-block range");
  if (n_s == 0) return VSA_OK;
  // tile-order attention (bf16 or 8-bit Q/K): query row blocks that share their key list go two at a time
  // (128 queries per key block) to the pair kernel -- the prefix row blocks of a launch that covers them,
  // when their pairs fill the SMs, and with 128-token tiles every tile of the range (its two row blocks)
  // -- and the other video row blocks to vsa_attn_kernel
  const int pre_rb = p->P << p->r.sh;
  int pair_lo = 0, pair_hi = 0;  // row blocks [pair_lo, pair_hi) go in pairs
  if (!seq && p->pair_prefix) {
    if (p->r.sh == 1 && s_lo % 2 == 0 && n_s % 2 == 0) {
      pair_lo = s_lo;
      pair_hi = s_lo + n_s;
    } else if (s_lo == 0 && n_s >= pre_rb &&
               static_cast<int64_t>(p->B) * p->H * ((pre_rb + 1) / 2) >= p->num_sms) {
      // 64-token tiles: the prefix pairs go to the pair kernel only when there are enough of them to fill
      // the GPU; with a few heads (a head chunk of the host pipeline, a sequence-parallel rank) a handful of
      // long dense items would hold their SMs while the video launch waits, and vsa_attn_kernel's item
      // schedule spreads the prefix row blocks among the video ones instead
      pair_hi = pre_rb;
    }
  }
  bool joined = true;  // no side-stream work to join back
  if (pair_hi > pair_lo) {
    vsa::AttnArgs ap = a;
    ap.s_lo = pair_lo;
    ap.r_end = pair_hi;
    ap.n_s = (pair_hi - pair_lo + 1) / 2;
    ap.n_items = static_cast<int64_t>(p->B) * p->H * ap.n_s;
    ap.sched = p->d_status + (alt_counters ? 6 : 4);  // its own item counter
    n_s = s_lo + n_s - pair_hi;  // what is left: [pair_hi, s_lo + n_s)
    s_lo = pair_hi;
    // with video row blocks to run too, the pair kernel goes on the side stream (forked from s)
    cudaStream_t ps = s;
    if (n_s > 0) {
      VSA_TRY(fork_side(p, s));
      ps = p->side;
      joined = false;
    }
    VSA_CUDA_TRY(cudaMemsetAsync(ap.sched, 0, sizeof(int), ps));
    VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
      constexpr int D = decltype(dc)::value;
      const size_t smem = vsa::PairLayout<D>::bytes();
      if (smem > p->max_smem) return fail(VSA_ERR_UNSUPPORTED, "attention shared memory exceeds the device limit");
      const int64_t gp = std::min<int64_t>(ap.n_items, p->num_sms);
      if (codes) {
        VSA_TRY(allow_smem(vsa::vsa_attn_pair_kernel<D, true>, smem));
        vsa::vsa_attn_pair_kernel<D, true><<<static_cast<unsigned>(gp), vsa::kPairThreads, smem, ps>>>(mq, mk, mv, ap);
      } else {
        VSA_TRY(allow_smem(vsa::vsa_attn_pair_kernel<D>, smem));
        vsa::vsa_attn_pair_kernel<D><<<static_cast<unsigned>(gp), vsa::kPairThreads, smem, ps>>>(mq, mk, mv, ap);
      }
      return VSA_OK;
    }));
    VSA_TRY(launch_check("pair attention"));
    if (!joined) VSA_CUDA_TRY(cudaEventRecord(p->ev_join, p->side));
    if (n_s == 0) return VSA_OK;
  }
  a.s_lo = s_lo;
  a.n_s = n_s;
  a.n_items = static_cast<int64_t>(p->B) * p->H * n_s;
  const int64_t grid = std::min<int64_t>(a.n_items, p->num_sms);
  // the item counter of the persistent schedule starts at zero for every launch
  VSA_CUDA_TRY(cudaMemsetAsync(a.sched, 0, sizeof(int), s));
  auto launch = [&](auto kernel, size_t smem) -> vsa_status {
    if (smem > p->max_smem) return fail(VSA_ERR_UNSUPPORTED, "attention shared memory exceeds the device limit");
    VSA_TRY(allow_smem(kernel, smem));
    kernel<<<static_cast<unsigned>(grid), vsa::kAttnThreads, smem, s>>>(mq, mk, mv, a, sm);
    return VSA_OK;
  };
  VSA_TRY(with_head_dim(p->D, [&](auto dc) -> vsa_status {
    constexpr int D = decltype(dc)::value;
    if (seq) return launch(vsa::vsa_attn_kernel<D, true, false>, vsa::AttnLayout<D>::bytes(p->n_t));
    if (codes) return launch(vsa::vsa_attn_kernel<D, false, true>, vsa::AttnLayout<D, true>::bytes(p->n_t));
    return launch(vsa::vsa_attn_kernel<D, false, false>, vsa::AttnLayout<D>::bytes(p->n_t));
  }));
  VSA_TRY(launch_check("attention"));
  if (!joined) VSA_CUDA_TRY(cudaStreamWaitEvent(s, p->ev_join, 0));  // the caller's stream sees both kernels
  return VSA_OK;
}

// ---------------------------------------------------------------- host pipeline helpers
void release_side(vsa_plan_s* p) {
  if (p->side) cudaStreamDestroy(p->side);
  if (p->ev_fork) cudaEventDestroy(p->ev_fork);
  if (p->ev_join) cudaEventDestroy(p->ev_join);
  if (p->ev_split) cudaEventDestroy(p->ev_split);
  p->side = nullptr;
  p->ev_fork = p->ev_join = p->ev_split = nullptr;
}

void release_host_pipe(vsa_plan_s* p) {
  auto& h = p->pipe;
  for (vsa_plan_s* sub : {h.sub, h.sub_last})
    if (sub) release_side(sub);
  delete h.sub;
  delete h.sub_last;
  h.sub = h.sub_last = nullptr;
  if (h.h2d) cudaStreamDestroy(h.h2d);
  if (h.d2h) cudaStreamDestroy(h.d2h);
  h.h2d = h.d2h = nullptr;
  for (cudaEvent_t* e : {&h.ev_in[0], &h.ev_in[1], &h.ev_comp[0], &h.ev_comp[1], &h.ev_out[0], &h.ev_out[1], &h.ev_gate,
                         &h.ev_start}) {
    if (*e) cudaEventDestroy(*e);
    *e = nullptr;
  }
  h.hc = 0;
}

// A plan for heads [h0, h0 + heads) of `p`'s geometry: same tables and status word, its own workspace layout.
vsa_plan_s* make_head_slice_plan(const vsa_plan_s* p, int32_t heads) {
  auto* q = new vsa_plan_s();
  q->device = p->device;
  q->num_sms = p->num_sms;
  q->max_smem = p->max_smem;
  q->B = p->B;
  q->H = heads;
  q->D = p->D;
  q->gate_pc = p->gate_pc;
  q->r = p->r;
  q->n_t = p->n_t;
  q->P = p->P;
  q->V = p->V;
  q->topk = p->topk;
  q->d_tile_token = p->d_tile_token;
  q->d_tile_valid = p->d_tile_valid;
  q->d_row_token = p->d_row_token;
  q->d_coord = p->d_coord;
  q->d_mask_seq = p->d_mask_seq;
  q->d_mask_tiled = p->d_mask_tiled;
  q->d_status = p->d_status;
  q->seq_tiles = p->seq_tiles;
  q->qk_fp8 = p->qk_fp8;
  q->qk_split = p->qk_split;
  q->fp4 = p->fp4;
  q->pair_prefix = p->pair_prefix;
  q->kr = p->kr;
  q->n_ref = p->n_ref;
  q->exempt_tiles = p->exempt_tiles;
  q->ref_tiles = p->ref_tiles;
  q->d_exempt = p->d_exempt;
  q->d_refs = p->d_refs;
  q->ws = make_layout(q->B, q->H, q->D, q->n_t, q->r.tile, q->V, q->topk + q->kr, q->seq_tiles, q->qk_fp8,
                      q->qk_split, q->fp4);
  q->owns_device = false;
  return q;
}

// Workspace of vsa_forward_host with chunks of hc heads: one head-slice forward workspace, two staging
// slots (q, k, v and out of one chunk each) and the whole gate.
struct HostLayout {
  size_t fwd = 0, slot[2] = {0, 0}, gate = 0, total = 0;
  size_t chunk_bytes = 0;  // one [B, L, hc, D] bf16 tensor, 256-aligned
};
HostLayout host_layout(const vsa_plan_s* p, int32_t hc) {
  HostLayout h;
  const size_t tokens = static_cast<size_t>(p->B) * static_cast<size_t>(p->r.L);
  h.chunk_bytes = align256(tokens * static_cast<size_t>(hc) * p->D * 2);
  h.fwd = 0;
  size_t off =
      align256(make_layout(p->B, hc, p->D, p->n_t, p->r.tile, p->V, p->topk + p->kr, p->seq_tiles, p->qk_fp8,
                           p->qk_split, p->fp4)
                   .total);
  for (int s = 0; s < 2; ++s) {
    h.slot[s] = off;
    off += 4 * h.chunk_bytes;  // q, k, v, out
  }
  h.gate = off;
  off += align256(tokens * static_cast<size_t>(p->gate_pc ? p->H * p->D : p->H) * 2);
  h.total = off;
  return h;
}

// The four steps on one stream; `w` holds p->ws.total bytes.  gate_ld: gate elements between tokens.
vsa_status forward_impl(vsa_plan p, const void* q, const void* k, const void* v, const void* gate, int gate_ld, void* out,
                        uint8_t* w, cudaStream_t s, const vsa::PartIO* io = nullptr) {
  auto* qt = w + p->ws.q_t;
  auto* kt = w + p->ws.k_t;
  auto* vt = w + p->ws.v_t;
  auto* pq = reinterpret_cast<float*>(w + p->ws.pq);
  auto* pk = reinterpret_cast<float*>(w + p->ws.pk);
  auto* pv = reinterpret_cast<float*>(w + p->ws.pv);
  auto* S = reinterpret_cast<float*>(w + p->ws.scores);
  auto* idx = reinterpret_cast<int32_t*>(w + p->ws.idx);
  auto* oc = reinterpret_cast<float*>(w + p->ws.o_c);
  auto* qsc = p->qk_fp8 ? reinterpret_cast<float*>(w + p->ws.q_s) : nullptr;
  auto* ksc = p->qk_fp8 ? reinterpret_cast<float*>(w + p->ws.k_s) : nullptr;
  auto* qn = reinterpret_cast<float*>(w + p->ws.q_n);
  auto* kv = reinterpret_cast<uint32_t*>(w + p->ws.kv_max);
  VSA_CUDA_TRY(cudaMemsetAsync(kv, 0, static_cast<size_t>(p->B) * p->H * 8, s));
  // does any gate differ from zero?  (if not, the compression branch is skipped on the device)
  int* gate_nz = p->d_status + 3;
  // sequence parts: the gate is spread over the parts and is not scanned; the branch is kept
  const bool parts = (io != nullptr && io->table != nullptr);
  VSA_CUDA_TRY(cudaMemsetAsync(gate_nz, parts ? 1 : 0, sizeof(int), s));
  if (p->n_t > 0 && !parts) {
    // scan from the 16-byte boundary at or below the gate (a head slice of a wider gate need not be
    // aligned) to this plan's last gate element; values of other heads in between can only make the
    // check say "nonzero", which keeps the branch
    const int64_t width = p->gate_pc ? static_cast<int64_t>(p->H) * p->D : p->H;  // this plan's gate per token
    const int64_t last = (static_cast<int64_t>(p->B) * p->r.L - 1) * gate_ld + width;  // one past, in elements
    const uintptr_t g = reinterpret_cast<uintptr_t>(gate);
    const uintptr_t g16 = g & ~static_cast<uintptr_t>(15);
    const int64_t ng = last + static_cast<int64_t>((g - g16) / 2);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((ng / 8 + 255) / 256, 8LL * p->num_sms));
    vsa::gate_any_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(reinterpret_cast<const uint16_t*>(g16), ng,
                                                                         gate_nz);
    VSA_TRY(launch_check("gate check"));
  }
  // With seq_tiles the attention reads Q/K/V straight from sequence order and the gather only pools;
  // otherwise the gather writes tile-order copies, which the attention reads with better DRAM locality.
  const bool seq = p->seq_tiles;
  VSA_TRY(run_gather(p, q, k, v, seq ? nullptr : qt, seq ? nullptr : kt, seq ? nullptr : vt, pq, pk, pv, s, io, qsc, ksc,
                     qn, kv));
  // prefix split: a second gather writes the 8-bit codes of K and of the prefix tiles' Q (no pooling, V
  // not read) with their own overflow-bound statistics; the value maximum comes from the first gather's
  // statistics
  auto* qc = w + p->ws.q_c;
  auto* kc = w + p->ws.k_c;
  auto* qn8 = reinterpret_cast<float*>(w + p->ws.q_n8);
  auto* kv8 = reinterpret_cast<uint32_t*>(w + p->ws.kv_max8);
  if (p->qk_split) {
    auto* qs2 = reinterpret_cast<float*>(w + p->ws.q_s);
    auto* ks2 = reinterpret_cast<float*>(w + p->ws.k_s);
    VSA_CUDA_TRY(cudaMemsetAsync(kv8, 0, static_cast<size_t>(p->B) * p->H * 8, s));
    VSA_TRY(run_gather(p, q, k, v, qc, kc, nullptr, nullptr, nullptr, nullptr, s, io, qs2, ks2, qn8, kv8, 1, p->P));
    VSA_CUDA_TRY(cudaMemcpy2DAsync(kv8 + 1, 8, kv + 1, 8, 4, static_cast<size_t>(p->B) * p->H,
                                   cudaMemcpyDeviceToDevice, s));
  }
  // FP4 video query tiles: the bf16 copies (already pooled) become their FP4 roundings, with new statistics
  if (p->fp4)
    VSA_TRY(run_fp4(p, qt, kt, vt, reinterpret_cast<double*>(w + p->ws.k_sum), reinterpret_cast<float*>(w + p->ws.k_mu),
                    qn, kv, s));
  VSA_TRY(run_scores(p, pq, pk, S, s));
  VSA_TRY(run_topk(p, S, pv, idx, oc, s, gate_nz));
  const void* qkv[3] = {q, k, v};
  if (p->qk_split) {
    // the dense prefix query row blocks on the 8-bit kernel, the video ones on the bf16 kernel; the two
    // launches write disjoint output rows and run concurrently: the prefix one on the plan's side stream
    // (forked from s, with its own item counters), the video one on s, which then waits for the side
    const int pre = p->P << p->r.sh;
    if (pre == 0)
      return run_attn(p, qt, kt, vt, idx, oc, gate, out, s, gate_ld, gate_nz, nullptr, io, nullptr, nullptr, qn, kv,
                      0);
    VSA_TRY(fork_side(p, s));
    VSA_TRY(run_attn(p, qc, kc, vt, idx, oc, gate, out, p->side, gate_ld, gate_nz, nullptr, io,
                     reinterpret_cast<float*>(w + p->ws.q_s), reinterpret_cast<float*>(w + p->ws.k_s), qn8, kv8, 1, 0,
                     pre, true));
    VSA_CUDA_TRY(cudaEventRecord(p->ev_split, p->side));
    VSA_TRY(run_attn(p, qt, kt, vt, idx, oc, gate, out, s, gate_ld, gate_nz, nullptr, io, nullptr, nullptr, qn, kv, 0,
                     pre));
    VSA_CUDA_TRY(cudaStreamWaitEvent(s, p->ev_split, 0));
    return VSA_OK;
  }
  return run_attn(p, qt, kt, vt, idx, oc, gate, out, s, gate_ld, gate_nz, seq ? qkv : nullptr, io, qsc, ksc, qn, kv);
}

// Gate elements per token: H, or H*D for a per-channel gate.
int64_t gate_width(const vsa_plan_s* p) { return p->gate_pc ? static_cast<int64_t>(p->H) * p->D : p->H; }

void fill_dims(const vsa_geometry* g, const Resolved& r, vsa_plan_dims* d) {
  d->n_tiles = static_cast<int32_t>(r.n_prefix + r.n_video);
  d->n_prefix_tiles = static_cast<int32_t>(r.n_prefix);
  d->n_video_tiles = static_cast<int32_t>(r.n_video);
  d->topk = r.topk;
  d->seq_len = r.L;
  d->softmax_scale = r.scale;
  d->workspace_bytes =
      make_layout(g->batch, g->heads, g->head_dim, d->n_tiles, r.tile, r.n_video, r.topk + r.kr, g->seq_tiles != 0,
                  g->qk_fp8 == 1, g->qk_fp8 >= 2, g->qk_fp8 == 3)
          .total;
  d->selected_pairs = r.n_video * (r.n_prefix - r.n_ref + r.kr + r.topk) + r.n_prefix * (r.n_prefix + r.n_video);
  d->tile_size = r.tile;
  d->n_ref_tiles = static_cast<int32_t>(r.n_ref);
  d->ref_topk = r.kr;
}

}  // namespace

extern "C" {

const char* vsa_last_error(void) { return g_last_error.c_str(); }

const char* vsa_version(void) { return "vsa-b200 0.1 (sm_100a)"; }

#ifdef VSA_ROLE_TIMERS
// Per-role cycle counters of the last attention launch (timer builds only):
// host[cta][role][counter], 160 x 8 x 8 unsigned 64-bit values.
vsa_status vsa_role_timers(void* host) {
  VSA_CUDA_TRY(cudaDeviceSynchronize());
  VSA_CUDA_TRY(cudaMemcpyFromSymbol(host, vsa::g_role_cycles, sizeof(vsa::g_role_cycles)));
  return VSA_OK;
}
#endif

vsa_status vsa_plan_query(const vsa_geometry* g, vsa_plan_dims* out) {
  if (out == nullptr) return fail(VSA_ERR_INVALID_ARG, "out is NULL");
  Resolved r;
  VSA_TRY(resolve(g, &r));
  fill_dims(g, r, out);
  return VSA_OK;
}

vsa_status vsa_plan_tables_host(const vsa_geometry* g, int32_t* tile_token, int32_t* tile_valid) {
  Resolved r;
  VSA_TRY(resolve(g, &r));
  std::vector<int32_t> tok, val;
  build_tables(r, &tok, &val);
  if (tile_token) std::memcpy(tile_token, tok.data(), tok.size() * 4);
  if (tile_valid) std::memcpy(tile_valid, val.data(), val.size() * 4);
  return VSA_OK;
}

vsa_status vsa_plan_tiles(const vsa_geometry* g, void* stream, vsa_plan* out) {
  if (out == nullptr) return fail(VSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  Resolved r;
  VSA_TRY(resolve(g, &r));
  int dev = 0;
  VSA_CUDA_TRY(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  VSA_CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10 || prop.minor != 0)
    return fail(VSA_ERR_DEVICE, "libvsa is built for sm_100a; device " + std::to_string(dev) + " is sm_" +
                                    std::to_string(prop.major) + std::to_string(prop.minor));
  auto* p = new vsa_plan_s();
  p->device = dev;
  p->num_sms = prop.multiProcessorCount;
  p->max_smem = prop.sharedMemPerBlockOptin;
  p->B = g->batch;
  p->H = g->heads;
  p->D = g->head_dim;
  p->gate_pc = g->gate_per_channel;
  p->r = r;
  p->n_t = static_cast<int32_t>(r.n_prefix + r.n_video);
  p->P = static_cast<int32_t>(r.n_prefix);
  p->V = static_cast<int32_t>(r.n_video);
  p->topk = r.topk;
  build_tables(r, &p->tile_token, &p->tile_valid);
  build_block_masks(r, p->tile_valid, &p->mask_tiled);
  if (r.tile == kTile) build_seq_tables(r, p->mask_tiled, &p->row_token, &p->mask_seq, &p->coord);
  p->seq_tiles = g->seq_tiles != 0;
  p->qk_fp8 = g->qk_fp8 == 1;
  p->qk_split = g->qk_fp8 >= 2;  // 3: the split with FP4 video query tiles
  p->fp4 = g->qk_fp8 == 3;
  p->kr = r.kr;
  p->n_ref = static_cast<int32_t>(r.n_ref);
  for (int32_t j = 0; j < p->P && p->n_ref > 0; ++j) (r.tile_ref[j] ? p->ref_tiles : p->exempt_tiles).push_back(j);
  p->ws = make_layout(p->B, p->H, p->D, p->n_t, r.tile, p->V, p->topk + p->kr, p->seq_tiles, p->qk_fp8,
                      p->qk_split, p->fp4);
  auto cleanup = [p] {
    cudaFree(p->d_tile_token);
    cudaFree(p->d_tile_valid);
    cudaFree(p->d_row_token);
    cudaFree(p->d_coord);
    cudaFree(p->d_mask_seq);
    cudaFree(p->d_mask_tiled);
    cudaFree(p->d_status);
    cudaFree(p->d_exempt);
    cudaFree(p->d_refs);
    cudaFree(p->d_stats);
    delete p;
  };
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tok_bytes = std::max<size_t>(4, p->tile_token.size() * 4);
  const size_t val_bytes = std::max<size_t>(4, p->tile_valid.size() * 4);
  const size_t mask_bytes = std::max<size_t>(8, p->mask_seq.size() * 8);
  const size_t block_mask_bytes = std::max<size_t>(8, p->mask_tiled.size() * 8);
  const size_t coord_bytes = std::max<size_t>(16, p->coord.size() * 4);
  if (cudaMalloc(&p->d_tile_token, tok_bytes) != cudaSuccess || cudaMalloc(&p->d_tile_valid, val_bytes) != cudaSuccess ||
      cudaMalloc(&p->d_row_token, tok_bytes) != cudaSuccess || cudaMalloc(&p->d_coord, coord_bytes) != cudaSuccess ||
      cudaMalloc(&p->d_mask_seq, mask_bytes) != cudaSuccess ||
      cudaMalloc(&p->d_mask_tiled, block_mask_bytes) != cudaSuccess ||
      cudaMalloc(&p->d_status, 8 * sizeof(int)) != cudaSuccess ||
      (p->n_ref > 0 && (cudaMalloc(&p->d_exempt, std::max<size_t>(4, p->exempt_tiles.size() * 4)) != cudaSuccess ||
                        cudaMalloc(&p->d_refs, p->ref_tiles.size() * 4) != cudaSuccess)) ||
      (!p->qk_fp8 && !p->qk_split && cudaMalloc(&p->d_stats, stats_bytes(p)) != cudaSuccess)) {
    cleanup();
    return fail(VSA_ERR_CUDA, "cudaMalloc of the plan tables failed");
  }
  cudaError_t e = cudaSuccess;
  if (!p->tile_token.empty())
    e = cudaMemcpyAsync(p->d_tile_token, p->tile_token.data(), p->tile_token.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->tile_valid.empty())
    e = cudaMemcpyAsync(p->d_tile_valid, p->tile_valid.data(), p->tile_valid.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->row_token.empty())
    e = cudaMemcpyAsync(p->d_row_token, p->row_token.data(), p->row_token.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->coord.empty())
    e = cudaMemcpyAsync(p->d_coord, p->coord.data(), p->coord.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->mask_seq.empty())
    e = cudaMemcpyAsync(p->d_mask_seq, p->mask_seq.data(), p->mask_seq.size() * 8, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->mask_tiled.empty())
    e = cudaMemcpyAsync(p->d_mask_tiled, p->mask_tiled.data(), p->mask_tiled.size() * 8, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->exempt_tiles.empty() && p->d_exempt)
    e = cudaMemcpyAsync(p->d_exempt, p->exempt_tiles.data(), p->exempt_tiles.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && !p->ref_tiles.empty())
    e = cudaMemcpyAsync(p->d_refs, p->ref_tiles.data(), p->ref_tiles.size() * 4, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(p->d_status, 0, 8 * sizeof(int), s);
  if (e != cudaSuccess) {
    cleanup();
    return fail(VSA_ERR_CUDA, std::string("plan upload: ") + cudaGetErrorString(e));
  }
  *out = p;
  return VSA_OK;
}

vsa_status vsa_plan_info(vsa_plan p, vsa_plan_dims* out) {
  if (p == nullptr || out == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  out->n_tiles = p->n_t;
  out->n_prefix_tiles = p->P;
  out->n_video_tiles = p->V;
  out->topk = p->topk;
  out->seq_len = p->r.L;
  out->softmax_scale = p->r.scale;
  out->workspace_bytes = p->ws.total;
  out->selected_pairs =
      static_cast<int64_t>(p->V) * (p->P - p->n_ref + p->kr + p->topk) + static_cast<int64_t>(p->P) * p->n_t;
  out->tile_size = p->r.tile;
  out->n_ref_tiles = p->n_ref;
  out->ref_topk = p->kr;
  return VSA_OK;
}

vsa_status vsa_plan_tables(vsa_plan p, int32_t* tile_token, int32_t* tile_valid) {
  if (p == nullptr) return fail(VSA_ERR_INVALID_ARG, "plan is NULL");
  if (tile_token) std::memcpy(tile_token, p->tile_token.data(), p->tile_token.size() * 4);
  if (tile_valid) std::memcpy(tile_valid, p->tile_valid.data(), p->tile_valid.size() * 4);
  return VSA_OK;
}

vsa_status vsa_plan_workspace(vsa_plan p, vsa_workspace_layout* out) {
  if (p == nullptr || out == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  *out = p->ws;
  return VSA_OK;
}

vsa_status vsa_plan_destroy(vsa_plan p) {
  if (p == nullptr) return VSA_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(p->device);
  cudaDeviceSynchronize();
  release_host_pipe(p);
  release_side(p);
  cudaFree(p->d_part_table);
  if (p->owns_device) {
    cudaFree(p->d_tile_token);
    cudaFree(p->d_tile_valid);
    cudaFree(p->d_row_token);
    cudaFree(p->d_coord);
    cudaFree(p->d_mask_seq);
    cudaFree(p->d_mask_tiled);
    cudaFree(p->d_status);
    cudaFree(p->d_exempt);
    cudaFree(p->d_refs);
    cudaFree(p->d_stats);
  }
  if (prev >= 0) cudaSetDevice(prev);
  delete p;
  return VSA_OK;
}

vsa_status vsa_gather_tiles(vsa_plan p, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, vsa_bf16* q_t,
                            vsa_bf16* k_t, vsa_bf16* v_t, float* pq, float* pk, float* pv, float* q_norm,
                            float* kv_max, void* stream) {
  VSA_TRY(check_plan(p));
  if (p->qk_fp8 || p->qk_split)
    return fail(VSA_ERR_UNSUPPORTED, "the step entry points take bf16 tiles: use vsa_forward with qk_fp8");
  VSA_TRY(check_ptrs({q, k, v, q_t, k_t, v_t}));
  const int npool = (pq != nullptr) + (pk != nullptr) + (pv != nullptr);
  if (npool != 0 && npool != 3) return fail(VSA_ERR_INVALID_ARG, "pq, pk, pv must be all NULL or all set");
  if (npool == 3) VSA_TRY(check_ptrs({pq, pk, pv}));
  if ((q_norm == nullptr) != (kv_max == nullptr))
    return fail(VSA_ERR_INVALID_ARG, "q_norm and kv_max must be both NULL or both set");
  if (q_norm != nullptr && npool != 3) return fail(VSA_ERR_INVALID_ARG, "the statistics are taken while pooling");
  if (q_norm != nullptr) VSA_TRY(check_ptrs({q_norm, kv_max}));
  const auto s = static_cast<cudaStream_t>(stream);
  auto* kv = reinterpret_cast<uint32_t*>(kv_max);
  if (kv != nullptr) VSA_CUDA_TRY(cudaMemsetAsync(kv, 0, static_cast<size_t>(p->B) * p->H * 8, s));
  return run_gather(p, q, k, v, q_t, k_t, v_t, pq, pk, pv, s, nullptr, nullptr, nullptr, q_norm, kv);
}

vsa_status vsa_pool_and_score(vsa_plan p, const vsa_bf16* q_t, const vsa_bf16* k_t, const vsa_bf16* v_t, float* pq,
                              float* pk, float* pv, float* scores, void* stream) {
  VSA_TRY(check_plan(p));
  VSA_TRY(check_ptrs({pq, pk, pv, scores}));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (q_t != nullptr) {
    if (p->qk_fp8 || p->qk_split)
    return fail(VSA_ERR_UNSUPPORTED, "the step entry points take bf16 tiles: use vsa_forward with qk_fp8");
    VSA_TRY(check_ptrs({q_t, k_t, v_t}));
    VSA_TRY(run_pool(p, q_t, k_t, v_t, pq, pk, pv, s));
  }
  return run_scores(p, pq, pk, scores, s);
}

vsa_status vsa_topk_select(vsa_plan p, const float* scores, const float* pv, int32_t* idx, float* o_c,
                           void* stream) {
  VSA_TRY(check_plan(p));
  VSA_TRY(check_ptrs({scores, pv, o_c}));
  if (p->V > 0) VSA_TRY(check_ptrs({idx}));
  return run_topk(p, scores, pv, idx, o_c, static_cast<cudaStream_t>(stream));
}

vsa_status vsa_sparse_attn_fwd(vsa_plan p, const vsa_bf16* q_t, const vsa_bf16* k_t, const vsa_bf16* v_t,
                               const int32_t* idx, const float* o_c, const vsa_bf16* gate, vsa_bf16* out,
                               const float* q_norm, const float* kv_max, void* stream) {
  VSA_TRY(check_plan(p));
  if (p->qk_fp8 || p->qk_split)
    return fail(VSA_ERR_UNSUPPORTED, "the step entry points take bf16 tiles: use vsa_forward with qk_fp8");
  VSA_TRY(check_ptrs({q_t, k_t, v_t, o_c, gate, out}));
  if (p->V > 0) VSA_TRY(check_ptrs({idx}));
  const auto s = static_cast<cudaStream_t>(stream);
  if ((q_norm == nullptr) != (kv_max == nullptr))
    return fail(VSA_ERR_INVALID_ARG, "q_norm and kv_max must be both NULL or both set");
  if (q_norm != nullptr) {  // the caller's statistics of these tiles (vsa_gather_tiles with statistics)
    VSA_TRY(check_ptrs({q_norm, kv_max}));
    return run_attn(p, q_t, k_t, v_t, idx, o_c, gate, out, s, 0, nullptr, nullptr, nullptr, nullptr, nullptr, q_norm,
                    reinterpret_cast<const uint32_t*>(kv_max));
  }
  // otherwise the overflow bound from these inputs' own statistics, into the plan's buffer
  float* qn = p->d_stats;
  auto* kv = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p->d_stats) + stats_rows_bytes(p));
  VSA_TRY(run_tile_stats(p, q_t, k_t, v_t, qn, kv, s));
  return run_attn(p, q_t, k_t, v_t, idx, o_c, gate, out, s, 0, nullptr, nullptr, nullptr, nullptr, nullptr, qn, kv);
}

vsa_status vsa_forward(vsa_plan p, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const vsa_bf16* gate,
                       vsa_bf16* out, void* workspace, size_t workspace_bytes, void* stream) {
  VSA_TRY(check_plan(p));
  VSA_TRY(check_ptrs({q, k, v, gate, out, workspace}));
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < p->ws.total)
    return fail(VSA_ERR_WORKSPACE, "workspace holds " + std::to_string(workspace_bytes) + " bytes, needs " +
                                       std::to_string(p->ws.total));
  return forward_impl(p, q, k, v, gate, static_cast<int>(gate_width(p)), out, static_cast<uint8_t*>(workspace),
                      static_cast<cudaStream_t>(stream));
}

vsa_status vsa_forward_noalloc(vsa_plan p, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v,
                               const vsa_bf16* gate, vsa_bf16* out, void* stream) {
  VSA_TRY(check_plan(p));
  if (p->ws.total > VSA_NOALLOC_SCRATCH_BYTES)
    return fail(VSA_ERR_WORKSPACE, "vsa_forward_noalloc: this geometry needs " + std::to_string(p->ws.total) +
                                       " bytes of scratch; the static scratch array holds " +
                                       std::to_string(VSA_NOALLOC_SCRATCH_BYTES) + " bytes (use vsa_forward)");
  void* scratch = nullptr;
  VSA_TRY(noalloc_scratch_address(p->device, &scratch));
  return vsa_forward(p, q, k, v, gate, out, scratch, VSA_NOALLOC_SCRATCH_BYTES, stream);
}

vsa_status vsa_forward_parts(vsa_plan p, const vsa_seq_parts* parts, void* workspace, size_t workspace_bytes,
                             void* stream) {
  VSA_TRY(check_plan(p));
  if (parts == nullptr) return fail(VSA_ERR_INVALID_ARG, "parts is NULL");
  const int n = parts->nparts;
  if (n < 1 || n > VSA_MAX_PARTS) return fail(VSA_ERR_INVALID_ARG, "nparts must lie in [1, VSA_MAX_PARTS]");
  if (parts->tokens_per_part < 1 || parts->tokens_per_part * n != p->r.L)
    return fail(VSA_ERR_SHAPE, "nparts * tokens_per_part must equal the sequence length " + std::to_string(p->r.L));
  if (parts->head_offset < 0 || parts->head_offset + p->H > parts->heads_total)
    return fail(VSA_ERR_SHAPE, "head_offset + the plan's heads must not exceed heads_total");
  if (p->seq_tiles) return fail(VSA_ERR_UNSUPPORTED, "sequence parts need a plan without seq_tiles");
  if (parts->q == nullptr || parts->k == nullptr || parts->v == nullptr || parts->gate == nullptr || parts->out == nullptr)
    return fail(VSA_ERR_INVALID_ARG, "a pointer array is NULL");
  for (int i = 0; i < n; ++i)
    VSA_TRY(check_ptrs({parts->q[i], parts->k[i], parts->v[i], parts->gate[i], parts->out[i]}));
  VSA_TRY(check_ptrs({workspace}));
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VSA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (workspace_bytes < p->ws.total)
    return fail(VSA_ERR_WORKSPACE, "workspace holds " + std::to_string(workspace_bytes) + " bytes, needs " +
                                       std::to_string(p->ws.total));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p->d_part_table == nullptr)
    VSA_CUDA_TRY(cudaMalloc(reinterpret_cast<void**>(&p->d_part_table), 5 * VSA_MAX_PARTS * sizeof(void*)));
  // table layout: operand-major, nparts entries each (q, k, v, gate, out)
  p->part_table.assign(5 * static_cast<size_t>(n), nullptr);
  for (int i = 0; i < n; ++i) {
    p->part_table[0 * n + i] = parts->q[i];
    p->part_table[1 * n + i] = parts->k[i];
    p->part_table[2 * n + i] = parts->v[i];
    p->part_table[3 * n + i] = parts->gate[i];
    p->part_table[4 * n + i] = parts->out[i];
  }
  VSA_CUDA_TRY(cudaMemcpyAsync(p->d_part_table, p->part_table.data(), p->part_table.size() * sizeof(void*),
                               cudaMemcpyHostToDevice, s));
  const vsa::PartIO io{p->d_part_table, n, parts->tokens_per_part, parts->heads_total, parts->head_offset};
  const int gate_ld = p->gate_pc ? parts->heads_total * p->D : parts->heads_total;
  return forward_impl(p, parts->q[0], parts->k[0], parts->v[0], parts->gate[0], gate_ld, parts->out[0],
                      static_cast<uint8_t*>(workspace), s, &io);
}

vsa_status vsa_forward_host_workspace(vsa_plan p, int32_t head_chunk, size_t* bytes) {
  if (p == nullptr || bytes == nullptr) return fail(VSA_ERR_INVALID_ARG, "NULL argument");
  if (head_chunk < 1 || head_chunk > p->H) return fail(VSA_ERR_INVALID_ARG, "head_chunk must lie in [1, heads]");
  *bytes = host_layout(p, head_chunk).total;
  return VSA_OK;
}

vsa_status vsa_forward_host(vsa_plan p, const vsa_bf16* q, const vsa_bf16* k, const vsa_bf16* v, const vsa_bf16* gate,
                            vsa_bf16* out, int32_t head_chunk, void* workspace, size_t workspace_bytes, void* stream) {
  VSA_TRY(check_plan(p));
  if (!p->owns_device) return fail(VSA_ERR_INVALID_ARG, "not a plan made by vsa_plan_tiles");
  if (q == nullptr || k == nullptr || v == nullptr || gate == nullptr || out == nullptr)
    return fail(VSA_ERR_INVALID_ARG, "a required host pointer is NULL");
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(VSA_ERR_INVALID_ARG, "workspace must be a 256-byte aligned device pointer");
  if (head_chunk < 1 || head_chunk > p->H) return fail(VSA_ERR_INVALID_ARG, "head_chunk must lie in [1, heads]");
  const HostLayout hl = host_layout(p, head_chunk);
  if (workspace_bytes < hl.total)
    return fail(VSA_ERR_WORKSPACE, "workspace holds " + std::to_string(workspace_bytes) + " bytes, needs " +
                                       std::to_string(hl.total));
  auto& hp = p->pipe;
  if (hp.hc != head_chunk) {  // (re)build the head-slice plans, copy streams and events
    release_host_pipe(p);
    hp.sub = make_head_slice_plan(p, head_chunk);
    if (p->H % head_chunk != 0) hp.sub_last = make_head_slice_plan(p, p->H % head_chunk);
    cudaError_t e = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking);
    for (cudaEvent_t* ev : {&hp.ev_in[0], &hp.ev_in[1], &hp.ev_comp[0], &hp.ev_comp[1], &hp.ev_out[0], &hp.ev_out[1],
                            &hp.ev_gate, &hp.ev_start})
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      release_host_pipe(p);
      return fail(VSA_ERR_CUDA, std::string("host pipeline setup: ") + cudaGetErrorString(e));
    }
    hp.hc = head_chunk;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* w = static_cast<uint8_t*>(workspace);
  const size_t tokens = static_cast<size_t>(p->B) * static_cast<size_t>(p->r.L);
  const size_t row = static_cast<size_t>(p->H) * p->D * 2;  // bytes of one token's heads on the host
  const int nchunks = (p->H + head_chunk - 1) / head_chunk;
  auto* dgate = reinterpret_cast<uint16_t*>(w + hl.gate);

  // everything earlier on the caller's stream (including a previous call's use of the staging slots)
  // comes before this call's copies
  VSA_CUDA_TRY(cudaEventRecord(hp.ev_start, s));
  VSA_CUDA_TRY(cudaStreamWaitEvent(hp.h2d, hp.ev_start, 0));
  VSA_CUDA_TRY(cudaStreamWaitEvent(hp.d2h, hp.ev_start, 0));
  const int64_t gw = gate_width(p);  // gate elements per token
  VSA_CUDA_TRY(cudaMemcpyAsync(dgate, gate, tokens * static_cast<size_t>(gw) * 2, cudaMemcpyHostToDevice, hp.h2d));
  VSA_CUDA_TRY(cudaEventRecord(hp.ev_gate, hp.h2d));
  VSA_CUDA_TRY(cudaStreamWaitEvent(s, hp.ev_gate, 0));

  for (int c = 0; c < nchunks; ++c) {
    const int slot = c & 1;
    const int h0 = c * head_chunk;
    const int hn = std::min(head_chunk, p->H - h0);
    vsa_plan_s* sp = (hn == head_chunk) ? hp.sub : hp.sub_last;
    uint8_t* base = w + hl.slot[slot];
    uint8_t* dq = base;
    uint8_t* dk = base + hl.chunk_bytes;
    uint8_t* dv = base + 2 * hl.chunk_bytes;
    uint8_t* dout = base + 3 * hl.chunk_bytes;
    const size_t width = static_cast<size_t>(hn) * p->D * 2;  // bytes of one token's heads in the chunk
    const size_t hoff = static_cast<size_t>(h0) * p->D * 2;
    // host -> device: the chunk's heads of q, k, v (slot free once chunk c-2 has been computed)
    if (c >= 2) VSA_CUDA_TRY(cudaStreamWaitEvent(hp.h2d, hp.ev_comp[slot], 0));
    VSA_CUDA_TRY(cudaMemcpy2DAsync(dq, width, reinterpret_cast<const uint8_t*>(q) + hoff, row, width, tokens,
                                   cudaMemcpyHostToDevice, hp.h2d));
    VSA_CUDA_TRY(cudaMemcpy2DAsync(dk, width, reinterpret_cast<const uint8_t*>(k) + hoff, row, width, tokens,
                                   cudaMemcpyHostToDevice, hp.h2d));
    VSA_CUDA_TRY(cudaMemcpy2DAsync(dv, width, reinterpret_cast<const uint8_t*>(v) + hoff, row, width, tokens,
                                   cudaMemcpyHostToDevice, hp.h2d));
    VSA_CUDA_TRY(cudaEventRecord(hp.ev_in[slot], hp.h2d));
    // the forward of the chunk on the caller's stream (output slot free once chunk c-2 is back on the host)
    VSA_CUDA_TRY(cudaStreamWaitEvent(s, hp.ev_in[slot], 0));
    if (c >= 2) VSA_CUDA_TRY(cudaStreamWaitEvent(s, hp.ev_out[slot], 0));
    // the chunk's first head in the whole gate: element h0 of each token, or channel h0*D
    VSA_TRY(forward_impl(sp, dq, dk, dv, dgate + (p->gate_pc ? static_cast<int64_t>(h0) * p->D : h0), static_cast<int>(gw),
                         dout, w + hl.fwd, s));
    VSA_CUDA_TRY(cudaEventRecord(hp.ev_comp[slot], s));
    // device -> host: the chunk's heads of the output
    VSA_CUDA_TRY(cudaStreamWaitEvent(hp.d2h, hp.ev_comp[slot], 0));
    VSA_CUDA_TRY(cudaMemcpy2DAsync(reinterpret_cast<uint8_t*>(out) + hoff, row, dout, width, width, tokens,
                                   cudaMemcpyDeviceToHost, hp.d2h));
    VSA_CUDA_TRY(cudaEventRecord(hp.ev_out[slot], hp.d2h));
  }
  // the caller's stream ends after the last copy back (the d2h stream runs its copies in order)
  VSA_CUDA_TRY(cudaStreamWaitEvent(s, hp.ev_out[(nchunks - 1) & 1], 0));
  return VSA_OK;
}

vsa_status vsa_wait_selftest(vsa_plan p, int64_t timeout_ns, void* stream, int32_t* code, int32_t* where) {
  VSA_TRY(check_plan(p));
  if (timeout_ns < 1000 || timeout_ns > 10000000000ll)
    return fail(VSA_ERR_INVALID_ARG, "timeout_ns must lie in [1e3, 1e10]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  VSA_CUDA_TRY(cudaMemsetAsync(p->d_status, 0, 2 * sizeof(int), s));
  vsa::wait_selftest_kernel<<<1, 64, 0, s>>>(p->d_status, static_cast<uint64_t>(timeout_ns));
  VSA_TRY(launch_check("wait self-test"));
  return vsa_device_status(p, stream, code, where);
}

vsa_status vsa_device_status(vsa_plan p, void* stream, int32_t* code, int32_t* where) {
  VSA_TRY(check_plan(p));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h[2] = {0, 0};
  VSA_CUDA_TRY(cudaMemcpyAsync(h, p->d_status, sizeof h, cudaMemcpyDeviceToHost, s));
  VSA_CUDA_TRY(cudaStreamSynchronize(s));
  VSA_CUDA_TRY(cudaMemsetAsync(p->d_status, 0, sizeof h, s));
  VSA_CUDA_TRY(cudaStreamSynchronize(s));
  if (code) *code = h[0];
  if (where) *where = h[1];
  return VSA_OK;
}

}  // extern "C"
