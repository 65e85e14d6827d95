/*
 * VSA-H3 forward -- plain CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline / reference arm use it.  It shares no code, header, table or
 * constant with the CUDA library; it is written straight from the method's
 * statement and is meant to be read against it line by line.
 *
 * Source of the method (the only place the pages state what VSA-H3 computes):
 *   "Mike0021/FastH3-4step-Preview-VSA", section "Video Sparse Attention is
 *   not optional here": the latent video grid is cut into 4x4x4 cubes of 64
 *   tokens and each prefix segment into runs that never cross a segment;
 *   tiles are scored per head in fp32 from their pooled (mean) Q and K;
 *   topk = max(1, min(ceil((1 - sparsity) * n_video_tiles), n_video_tiles))
 *   video key tiles are kept per video query tile, prefix keys are kept for
 *   all of them and prefix queries see every key; a compression branch
 *   softmax(scores) @ pool(v) gives one vector per tile that is multiplied by
 *   the gate (no activation) and added to each row of the tile.
 * Supporting passages:
 *   "FastH3 NVFP4 on RTX PRO 6000 (sm_120)", section "Block-sparse FP4
 *   attention for VSA tiles": per-query-block lists of key blocks, partially
 *   filled tiles carry valid counts, exempt mode gives every query the first
 *   prefix tile; section "Model integration": pad rows are zero.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   R1 video tokens follow the prefix in raster (t, h, w) order, w fastest;
 *   R2 a grid side that is not a multiple of 4 gives partial edge cubes
 *      (ceil-divided cube grid);
 *   R3 inside a tile the valid tokens come first, pads last;
 *   R4 a pooled tile is the mean over its valid tokens (divisor = count);
 *   R5 pooled scores use the same softmax scale as the fine branch;
 *   R6 the fp32 arithmetic order is pinned: pooling adds rows in tile order
 *      starting from +0.0f, then one IEEE division; a score is a chain of
 *      fmaf over d = 0..D-1 starting from +0.0f, then one multiply by scale;
 *   R7 ties in the top-k order go to the lower video tile index; the chosen
 *      tiles are listed in ascending index;
 *   R8 topk uses binary64 arithmetic for (1 - sparsity) * V and its ceiling,
 *      and is 0 when there are no video tiles;
 *   R9 the compression softmax runs over ALL tiles (prefix and video)
 *      -- parity unpinned;
 *   R10 the compression branch is added to every tile row, prefix tiles
 *      included -- parity unpinned;
 *   R11 the gate is one scalar per (batch, token, head).
 *   R12 the per-channel variant: one gate per (batch, token, channel h*D + d), [B, L, H*D].
 *   R16 the 8-bit Q/K variant ("FastH3 OmniRef inference", section "The Blackwell stack" and
 *      "Fallbacks": query/key rounding to 8 bits with bf16 P.V, per-token FP8 Q/K; the
 *      multi-GPU notes of "FastH3 NVFP4 on RTX PRO 6000": a scale for each token of each head):
 *      8 bits = OCP FP8 E4M3 ("E4M3FN": bias 7, no infinities, largest 448); one binary32
 *      scale per (batch, token, head), s = amax / 448 in binary32 where amax is the largest
 *      |x_d| of the token's head row; code_d = E4M3 round-to-nearest-even of the binary32
 *      quotient x_d / s, saturating at +-448; a row with amax = 0 has s = 0 and all codes
 *      +0.  The dequantised value code * s replaces Q and K in the fine branch's logits
 *      only: selection, compression and P.V keep the bf16 inputs.  The variant covers
 *      every query tile.
 *   R17 128-token tiles ("FastH3 OmniRef inference", section "The Blackwell stack": VSA
 *      with 128-token tiles; the cube shape is not stated): a prefix tile is a
 *      segment-pure run of up to 128 tokens and a video tile a ct x ch x cw cube with
 *      ct*ch*cw = 128, by default 4 x 4 x 8 (the 4 x 4 x 4 cube doubled along w, the
 *      fastest axis); every other step is the 64-token method with "64" read as the
 *      tile size.
 *   R18 "reference keep" (same passage: "reference keep 0.1"): a prefix segment may be a
 *      reference segment (the reference vision tokens and reference audio of the
 *      conditioning prefix).  Its tiles are not always-kept prefix keys: each video query
 *      tile keeps the kr reference tiles with the highest pooled scores S[i, j] (ties to
 *      the lower index), kr = max(1, min(ceil(keep * R), R)) in binary64 for R reference
 *      tiles (0 when R = 0), listed ascending before its topk video tiles.  The other
 *      prefix tiles stay always kept; prefix query tiles (reference ones included) stay
 *      dense; the compression still runs over all tiles.
 *   R20 FP4 video query tiles ("FastH3 OmniRef inference", sections "Device profiles",
 *      "Environment" and "Fallbacks": the video query tiles run on an FP4 kernel; key
 *      smoothing removes each head's mean key before the FP4 rounding; the emulator fallback
 *      fixes the numerics: FP4 Q and K for the video query tiles, 8-bit per-token Q and K for
 *      the prefix tiles, bf16 P.V, smoothed K; "FastH3 NVFP4 on RTX PRO 6000", model
 *      integration and "What was tried": activations carry a global scale of 1 and one scale
 *      per 16 values computed per call; values are E2M1 with E4M3 block scales):
 *      FP4 = OCP E2M1 (bit 3 sign, 2-bit exponent with bias 1, 1-bit mantissa; magnitudes
 *      0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN).  Rows of D are cut into blocks of
 *      16 consecutive elements; a block's scale is the E4M3 code e4m3_round(amax / 6)
 *      (binary32 division, amax the largest |x| of the block) and each element's code is
 *      e2m1_round(x / value(scale)) (binary32 division; nearest, ties to the even code,
 *      saturating at 6); a scale of value 0 gives codes +0.  The global scale is 1.
 *      Key smoothing: mu[b, h, d] = the binary64 sum of k[b, t, h, d] over the L tokens in
 *      token order, divided by L in binary64, rounded to binary32; the quantised key is
 *      x = k - mu in binary32.  Queries are not smoothed.  The dequantised values code *
 *      scale (at most 6 significant bits, magnitudes 2^-10 .. 2688) are bf16 numbers, and
 *      they replace Q and K in the video query tiles' logits; the prefix query tiles follow
 *      R16 on the unsmoothed inputs (the split); selection, compression and P.V keep bf16.
 *      Subtracting mu from every key changes each query row's logits by one constant,
 *      which the softmax removes: only the rounding changes.  The native kernel's
 *      quantised P.V ("two-level P") is not defined on the pages and is not modelled.
 *
 * Precision: selection (pool, score, top-k) in IEEE binary32 with the pinned
 * order above; fine attention, compression and the output in binary64.
 *
 * Build: gcc -O2 -fno-fast-math -ffp-contract=off -fopenmp -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Tile size and cube shape are arguments: 64-token (4,4,4) tiles, or the
 * 128-token tiles of reading R17. */

/* ------------------------------------------------------------------ */
/* helpers                                                             */
/* ------------------------------------------------------------------ */

static float bf16_to_float(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------ */
/* O0 8-bit Q/K: E4M3 codes with one scale per (batch, token, head)   */
/* (reading R16)                                                       */
/* ------------------------------------------------------------------ */

/* Value of an E4M3 code: bit 7 sign, bits 6..3 exponent field e (bias 7),
 * bits 2..0 mantissa m.  e = 0: subnormal, m/8 * 2^-6; otherwise
 * (1 + m/8) * 2^(e-7).  e = 15 with m = 7 is NaN; there is no infinity. */
double vsa_oracle_e4m3_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* E4M3 code nearest to y; a tie goes to the even code (even mantissa); a
 * magnitude at or above 448 (the largest finite value, code 0x7E) gives
 * +-448.  The sign bit is the sign of y, so -0 and negative values that
 * round to zero give 0x80. */
int vsa_oracle_e4m3_round(float y) {
    int sign = signbit(y) ? 0x80 : 0;
    double a = fabs((double)y);
    int lo = 0, hi = 126; /* codes 0..126 hold the finite magnitudes in increasing order */
    double dl, dh;
    if (a >= 448.0) return sign | 126;
    /* largest code lo with value(lo) <= a (binary search over 0..126) */
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (vsa_oracle_e4m3_value(mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    dl = a - vsa_oracle_e4m3_value(lo);
    if (dl == 0.0) return sign | lo;
    dh = vsa_oracle_e4m3_value(lo + 1) - a;
    if (dl < dh) return sign | lo;
    if (dh < dl) return sign | (lo + 1);
    return sign | ((lo & 1) ? lo + 1 : lo);
}

void vsa_oracle_e4m3_round_array(const float *y, int64_t n, uint8_t *code) {
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n; ++e) code[e] = (uint8_t)vsa_oracle_e4m3_round(y[e]);
}

/* Per-row quantisation of x [N, D] (bf16 bits), one row = one (batch, token,
 * head): amax = max_d |x_d|; s = amax / 448 (binary32 division); code_d =
 * e4m3_round(x_d / s) (binary32 division); amax = 0 gives s = 0 and codes +0. */
void vsa_oracle_quant_e4m3(const uint16_t *x, int64_t N, int D, uint8_t *code, float *scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < N; ++r) {
        const uint16_t *xr = x + r * D;
        float amax = 0.0f, s;
        for (int d = 0; d < D; ++d) {
            float a = fabsf(bf16_to_float(xr[d]));
            if (a > amax) amax = a;
        }
        s = amax / 448.0f;
        scale[r] = s;
        for (int d = 0; d < D; ++d) {
            float q = (amax == 0.0f) ? 0.0f : bf16_to_float(xr[d]) / s;
            code[r * D + d] = (uint8_t)((amax == 0.0f) ? 0 : vsa_oracle_e4m3_round(q));
        }
    }
}

/* ------------------------------------------------------------------ */
/* O1 FP4 (E2M1) codes with one E4M3 scale per 16 values, key          */
/* smoothing (reading R20)                                             */
/* ------------------------------------------------------------------ */

/* Value of an E2M1 code: bit 3 sign, bits 2..1 exponent field e (bias 1), bit 0
 * mantissa m.  e = 0: subnormal, m/2; otherwise (1 + m/2) * 2^(e-1). */
double vsa_oracle_e2m1_value(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* E2M1 code nearest to y; a tie goes to the even code; magnitudes at or above 6 give
 * +-6 (code 7).  The sign bit is the sign of y (-0 and small negatives give 0x8). */
int vsa_oracle_e2m1_round(float y) {
    int sign = signbit(y) ? 8 : 0;
    double a = fabs((double)y);
    int lo = 0;
    double dl, dh;
    if (a >= 6.0) return sign | 7;
    while (lo < 7 && vsa_oracle_e2m1_value(lo + 1) <= a) ++lo; /* largest code with value <= a */
    dl = a - vsa_oracle_e2m1_value(lo);
    if (dl == 0.0) return sign | lo;
    dh = vsa_oracle_e2m1_value(lo + 1) - a;
    if (dl < dh) return sign | lo;
    if (dh < dl) return sign | (lo + 1);
    return sign | ((lo & 1) ? lo + 1 : lo);
}

void vsa_oracle_e2m1_round_array(const float *y, int64_t n, uint8_t *code) {
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n; ++e) code[e] = (uint8_t)vsa_oracle_e2m1_round(y[e]);
}

/* Block quantisation of rows x [N, D] (binary32; D a multiple of 16): for each block of 16
 * consecutive elements, amax = max |x|, scale code sc = e4m3_round(amax / 6) (binary32
 * division), sv = value(sc), code = e2m1_round(x / sv) (binary32 division), or +0 when
 * sv = 0.  code [N, D], scale [N, D / 16]. */
void vsa_oracle_quant_fp4(const float *x, int64_t N, int D, uint8_t *code, uint8_t *scale) {
    const int nb = D / 16;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < N; ++r) {
        for (int blk = 0; blk < nb; ++blk) {
            const float *xb = x + r * D + blk * 16;
            uint8_t *cb = code + r * D + blk * 16;
            float amax = 0.0f, sv;
            int sc;
            for (int j = 0; j < 16; ++j) {
                float a = fabsf(xb[j]);
                if (a > amax) amax = a;
            }
            sc = vsa_oracle_e4m3_round(amax / 6.0f);
            sv = (float)vsa_oracle_e4m3_value(sc);
            scale[r * nb + blk] = (uint8_t)sc;
            for (int j = 0; j < 16; ++j) cb[j] = (uint8_t)((sv == 0.0f) ? 0 : vsa_oracle_e2m1_round(xb[j] / sv));
        }
    }
}

/* Key smoothing: mu [B, H, D] = (binary64 sum over t of k[b, t, h, d], token order) / L,
 * rounded to binary32; ks [B, L, H, D] = k - mu in binary32. */
void vsa_oracle_smooth_keys(const uint16_t *k, int64_t B, int64_t L, int H, int D, float *mu, float *ks) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int d = 0; d < D; ++d) {
                double sum = 0.0;
                float m;
                for (int64_t t = 0; t < L; ++t) sum += (double)bf16_to_float(k[((b * L + t) * H + h) * D + d]);
                m = (float)(sum / (double)L);
                mu[(b * H + h) * D + d] = m;
                for (int64_t t = 0; t < L; ++t) {
                    int64_t e = ((b * L + t) * H + h) * D + d;
                    ks[e] = bf16_to_float(k[e]) - m;
                }
            }
}

/* One operand of the fine branch's logits (Q or K), [B, L, H, D]: bf16 bits,
 * or (code != NULL) E4M3 codes with one binary32 scale per row of D. */
typedef struct {
    const uint16_t *bf16;
    const uint8_t *code;
    const float *scale;
} qk_operand;

static double e4m3_table[256];
static int e4m3_table_ready = 0;

static double qk_value(const qk_operand *x, int64_t row, int D, int d) {
    if (x->code) return e4m3_table[x->code[row * D + d]] * (double)x->scale[row];
    return (double)bf16_to_float(x->bf16[row * D + d]);
}

static void qk_tables(void) {
    if (e4m3_table_ready) return;
    for (int c = 0; c < 256; ++c) e4m3_table[c] = vsa_oracle_e4m3_value(c);
    e4m3_table_ready = 1;
}

/* ------------------------------------------------------------------ */
/* O1 geometry                                                         */
/* ------------------------------------------------------------------ */

/* Tile counts of a packed sequence with `tile`-token tiles whose video cubes are
 * ct x ch x cw (ct*ch*cw == tile; 64 = 4x4x4 as the method states, R17 for 128):
 * each prefix segment of n tokens gives ceil(n/tile) segment-pure tiles; the
 * T x H x W video grid gives ceil(T/ct) * ceil(H/ch) * ceil(W/cw) cubes (R2).
 * Returns 0, or -1 on a bad argument. */
int vsa_oracle_geometry(int n_seg, const int32_t *seg_len, int T, int Hg, int W, int tile, int ct, int ch,
                        int cw, int32_t *n_tiles, int32_t *n_prefix, int32_t *n_video) {
    if (n_seg < 0 || T < 0 || Hg < 0 || W < 0) return -1;
    if (tile < 1 || ct < 1 || ch < 1 || cw < 1 || ct * ch * cw != tile) return -1;
    int64_t p = 0;
    for (int s = 0; s < n_seg; ++s) {
        if (seg_len[s] < 0) return -1;
        p += ceil_div(seg_len[s], tile);
    }
    int64_t v = (T > 0 && Hg > 0 && W > 0)
                    ? ceil_div(T, ct) * ceil_div(Hg, ch) * ceil_div(W, cw)
                    : 0;
    *n_prefix = (int32_t)p;
    *n_video = (int32_t)v;
    *n_tiles = (int32_t)(p + v);
    return 0;
}

/* Token table: tile_token[i*tile + r] is the packed-sequence index of row r
 * of tile i, or -1 for a pad row; tile_valid[i] counts the valid rows.
 * Prefix tiles first, in sequence order; then the cubes in raster (a,b,c)
 * order; inside a cube, raster (t,h,w) (readings R1, R3). */
int vsa_oracle_tiles(int n_seg, const int32_t *seg_len, int T, int Hg, int W, int tile, int ct, int ch, int cw,
                     int32_t *tile_token, int32_t *tile_valid) {
    int32_t nt, np, nv;
    if (vsa_oracle_geometry(n_seg, seg_len, T, Hg, W, tile, ct, ch, cw, &nt, &np, &nv)) return -1;
    for (int64_t i = 0; i < (int64_t)nt * tile; ++i) tile_token[i] = -1;

    int i = 0;
    int64_t offset = 0; /* first token of the current segment */
    for (int s = 0; s < n_seg; ++s) {
        int64_t n = seg_len[s];
        for (int64_t first = 0; first < n; first += tile) {
            int cnt = 0;
            for (int64_t t = first; t < n && t < first + tile; ++t)
                tile_token[(int64_t)i * tile + cnt++] = (int32_t)(offset + t);
            tile_valid[i++] = cnt;
        }
        offset += n;
    }
    if (nv > 0) {
        int64_t video_base = offset;
        for (int a = 0; a < ceil_div(T, ct); ++a)
            for (int b = 0; b < ceil_div(Hg, ch); ++b)
                for (int c = 0; c < ceil_div(W, cw); ++c) {
                    int cnt = 0;
                    for (int t = ct * a; t < ct * a + ct && t < T; ++t)
                        for (int h = ch * b; h < ch * b + ch && h < Hg; ++h)
                            for (int w = cw * c; w < cw * c + cw && w < W; ++w)
                                tile_token[(int64_t)i * tile + cnt++] =
                                    (int32_t)(video_base + ((int64_t)t * Hg + h) * W + w);
                    tile_valid[i++] = cnt;
                }
    }
    return 0;
}

/* O4 count: topk = max(1, min(ceil((1 - s) * V), V)) in binary64 (R8). */
int vsa_oracle_topk_count(double sparsity, int n_video) {
    if (n_video <= 0) return 0;
    double k = ceil((1.0 - sparsity) * (double)n_video);
    if (k > (double)n_video) k = (double)n_video;
    if (k < 1.0) k = 1.0;
    return (int)k;
}

/* ------------------------------------------------------------------ */
/* O2 pooling (binary32, pinned order)                                 */
/* ------------------------------------------------------------------ */

/* x: [B, L, H, D] bf16 bits.  pooled: [B, H, n_t, D] float.
 * pooled = (((0 + x_0) + x_1) + ... + x_{n-1}) / n  over the valid rows in
 * tile order, every step one IEEE binary32 rounding (R4, R6). */
void vsa_oracle_pool(const uint16_t *x, int B, int64_t L, int H, int D, int n_t, int tile,
                     const int32_t *tile_token, const int32_t *tile_valid, float *pooled) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n_t; ++i)
                for (int d = 0; d < D; ++d) {
                    float sum = 0.0f;
                    for (int r = 0; r < tile_valid[i]; ++r) {
                        int64_t tok = tile_token[(int64_t)i * tile + r];
                        sum = sum + bf16_to_float(x[(((int64_t)b * L + tok) * H + h) * D + d]);
                    }
                    pooled[(((int64_t)b * H + h) * n_t + i) * D + d] =
                        sum / (float)tile_valid[i];
                }
}

/* ------------------------------------------------------------------ */
/* O3 pooled tile scores (binary32, pinned order)                      */
/* ------------------------------------------------------------------ */

/* S[bh, i, j] = fl(fmaf-chain_{d=0..D-1}(pq[bh,i,d] * pk[bh,j,d]) * scale). */
void vsa_oracle_scores(const float *pq, const float *pk, int BH, int n_t, int D,
                       float scale, float *S) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        for (int i = 0; i < n_t; ++i)
            for (int j = 0; j < n_t; ++j) {
                const float *a = pq + ((int64_t)bh * n_t + i) * D;
                const float *b = pk + ((int64_t)bh * n_t + j) * D;
                float acc = 0.0f;
                for (int d = 0; d < D; ++d) acc = fmaf(a[d], b[d], acc);
                S[((int64_t)bh * n_t + i) * n_t + j] = acc * scale;
            }
}

/* ------------------------------------------------------------------ */
/* O4 top-k selection                                                  */
/* ------------------------------------------------------------------ */

typedef struct {
    float s;
    int32_t j;
} scored_tile;

/* order: higher score first; equal scores -> lower tile index first (R7) */
static int by_score_then_index(const void *pa, const void *pb) {
    const scored_tile *a = (const scored_tile *)pa, *b = (const scored_tile *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_index(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* For each (bh, video query tile iv) pick the k video key tiles with the
 * highest S[bh, P+iv, P+j]; write their GLOBAL tile indices (P + j) in
 * ascending order to idx[bh, iv, 0..k-1].  Returns -1 if any compared score
 * is NaN (inputs with NaN are rejected), else 0. */
int vsa_oracle_select(const float *S, int BH, int n_t, int P, int k, int32_t *idx) {
    int V = n_t - P;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : bad)
    for (int bh = 0; bh < BH; ++bh)
        for (int iv = 0; iv < V; ++iv) {
            scored_tile *row = (scored_tile *)malloc(sizeof(scored_tile) * (size_t)(V > 0 ? V : 1));
            const float *srow = S + ((int64_t)bh * n_t + (P + iv)) * n_t;
            for (int j = 0; j < V; ++j) {
                row[j].s = srow[P + j];
                row[j].j = j;
                if (isnan(row[j].s)) bad = 1;
            }
            qsort(row, (size_t)V, sizeof(scored_tile), by_score_then_index);
            int32_t *out = idx + ((int64_t)bh * V + iv) * k;
            for (int t = 0; t < k; ++t) out[t] = P + row[t].j;
            qsort(out, (size_t)k, sizeof(int32_t), by_index);
            free(row);
        }
    return bad ? -1 : 0;
}

/* Reference keep (R18): kr = max(1, min(ceil(keep * R), R)) in binary64; 0 without reference tiles. */
int vsa_oracle_ref_count(double keep, int n_ref) {
    double k;
    if (n_ref <= 0) return 0;
    k = ceil(keep * (double)n_ref);
    if (k > (double)n_ref) k = (double)n_ref;
    if (k < 1.0) k = 1.0;
    return (int)k;
}

/* Selection with reference tiles (R18): for each (bh, video query tile iv), idx[bh, iv, 0..kr)
 * = the kr reference tiles (prefix tiles j with is_ref[j]) with the highest S[bh, P+iv, j],
 * ascending; idx[bh, iv, kr..kr+k) = the k video tiles as vsa_oracle_select picks them.  Ties go
 * to the lower index.  Returns -1 if a compared score is NaN. */
int vsa_oracle_select_ref(const float *S, int BH, int n_t, int P, const uint8_t *is_ref, int kr, int k,
                          int32_t *idx) {
    int V = n_t - P, R = 0, w = kr + k;
    int bad = 0;
    for (int j = 0; j < P; ++j) R += is_ref[j] ? 1 : 0;
#pragma omp parallel for collapse(2) schedule(static) reduction(| : bad)
    for (int bh = 0; bh < BH; ++bh)
        for (int iv = 0; iv < V; ++iv) {
            int n = (V > R ? V : R);
            scored_tile *row = (scored_tile *)malloc(sizeof(scored_tile) * (size_t)(n > 0 ? n : 1));
            const float *srow = S + ((int64_t)bh * n_t + (P + iv)) * n_t;
            int32_t *out = idx + ((int64_t)bh * V + iv) * w;
            int m = 0;
            for (int j = 0; j < P; ++j)
                if (is_ref[j]) {
                    row[m].s = srow[j];
                    row[m].j = j;
                    if (isnan(row[m].s)) bad = 1;
                    ++m;
                }
            qsort(row, (size_t)m, sizeof(scored_tile), by_score_then_index);
            for (int t = 0; t < kr; ++t) out[t] = row[t].j;
            qsort(out, (size_t)kr, sizeof(int32_t), by_index);
            for (int j = 0; j < V; ++j) {
                row[j].s = srow[P + j];
                row[j].j = j;
                if (isnan(row[j].s)) bad = 1;
            }
            qsort(row, (size_t)V, sizeof(scored_tile), by_score_then_index);
            for (int t = 0; t < k; ++t) out[kr + t] = P + row[t].j;
            qsort(out + kr, (size_t)k, sizeof(int32_t), by_index);
            free(row);
        }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------ */
/* O6 compression branch (binary64)                                    */
/* ------------------------------------------------------------------ */

/* o_c[bh, i, :] = sum_j softmax_j(S[bh, i, :]) * pv[bh, j, :], j over all
 * n_t tiles (reading R9). */
void vsa_oracle_compress(const float *S, const float *pv, int BH, int n_t, int D, double *o_c) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        for (int i = 0; i < n_t; ++i) {
            const float *srow = S + ((int64_t)bh * n_t + i) * n_t;
            double m = -INFINITY;
            for (int j = 0; j < n_t; ++j)
                if ((double)srow[j] > m) m = (double)srow[j];
            double denom = 0.0;
            for (int j = 0; j < n_t; ++j) denom += exp((double)srow[j] - m);
            double *o = o_c + ((int64_t)bh * n_t + i) * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int j = 0; j < n_t; ++j) {
                double w = exp((double)srow[j] - m) / denom;
                const float *pvj = pv + ((int64_t)bh * n_t + j) * D;
                for (int d = 0; d < D; ++d) o[d] += w * (double)pvj[d];
            }
        }
}

/* ------------------------------------------------------------------ */
/* O5 fine branch, list formulation (binary64)                         */
/* ------------------------------------------------------------------ */

/* The key set of query tile i: every tile for a prefix query tile (dense
 * prefix queries); the P prefix tiles plus idx[b,h,i-P,:] for a video query
 * tile (exempt prefix keys).  Writes the set into keys[] and returns its size. */
/* Key tiles of query tile i: every tile for a prefix query tile; otherwise the always-kept prefix
 * tiles (all P, or those with is_ref[j] == 0 when is_ref is given, R18) followed by the w = kr + k
 * entries of its idx row. */
static int key_set(int i, int n_t, int P, const uint8_t *is_ref, int w, const int32_t *idx_row,
                   int32_t *keys) {
    int n = 0;
    if (i < P) {
        for (int j = 0; j < n_t; ++j) keys[j] = j;
        return n_t;
    }
    for (int j = 0; j < P; ++j)
        if (!is_ref || !is_ref[j]) keys[n++] = j;
    for (int t = 0; t < w; ++t) keys[n++] = idx_row[t];
    return n;
}

/* Fine branch of one query tile (b, h, i): for each valid query row r,
 *   logit_c = scale * <q_r, k_c> over the valid key rows c of its key set,
 *   o_f[r] = sum_c softmax(logit)_c * v_c,
 * written to rows[r * D + d] in tile row order (pad rows left untouched). */
static void fine_one_tile(const qk_operand *q, const qk_operand *kk, const uint16_t *v, int b, int h, int i,
                          int64_t L, int H, int D, int n_t, int P, int k, const uint8_t *is_ref, int kr, int tile,
                          const int32_t *tile_token, const int32_t *tile_valid, const int32_t *idx, double scale,
                          double *rows) {
    int V = n_t - P, w = kr + k;
    int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_t);
    const int32_t *idx_row = (i >= P) ? idx + (((int64_t)b * H + h) * V + (i - P)) * w : NULL;
    int nk = key_set(i, n_t, P, is_ref, w, idx_row, keys);
    /* every valid key row of the key set, in list order */
    int64_t max_rows = (int64_t)nk * tile;
    int64_t *ktok = (int64_t *)malloc(sizeof(int64_t) * (size_t)max_rows);
    double *logit = (double *)malloc(sizeof(double) * (size_t)max_rows);
    int64_t nrows = 0;
    for (int t = 0; t < nk; ++t)
        for (int c = 0; c < tile_valid[keys[t]]; ++c)
            ktok[nrows++] = tile_token[(int64_t)keys[t] * tile + c];

    for (int r = 0; r < tile_valid[i]; ++r) {
        int64_t qt = tile_token[(int64_t)i * tile + r];
        int64_t qrow = ((int64_t)b * L + qt) * H + h;
        double m = -INFINITY;
        for (int64_t c = 0; c < nrows; ++c) {
            int64_t krow = ((int64_t)b * L + ktok[c]) * H + h;
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += qk_value(q, qrow, D, d) * qk_value(kk, krow, D, d);
            logit[c] = scale * dot;
            if (logit[c] > m) m = logit[c];
        }
        double denom = 0.0;
        for (int64_t c = 0; c < nrows; ++c) {
            logit[c] = exp(logit[c] - m);
            denom += logit[c];
        }
        double *o = rows + (int64_t)r * D;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (int64_t c = 0; c < nrows; ++c) {
            const uint16_t *vc = v + (((int64_t)b * L + ktok[c]) * H + h) * D;
            double w = logit[c] / denom;
            for (int d = 0; d < D; ++d) o[d] += w * (double)bf16_to_float(vc[d]);
        }
    }
    free(logit);
    free(ktok);
    free(keys);
}

/* o_f[b, tok, h, :] for every valid query token tok of every (b, h, i) with
 * todo[(b*H + h)*n_t + i] != 0 (todo == NULL: all).
 * q, k, v: [B, L, H, D] bf16 bits; idx: [B, H, V, k] global tile indices.
 * q8/qs and k8/ks (both NULL, or both set): the 8-bit variant (R16), E4M3
 * codes [B, L, H, D] and scales [B, L, H] used for the logits instead of q, k. */
void vsa_oracle_fine(const uint16_t *q, const uint16_t *kk, const uint16_t *v, const uint8_t *q8,
                     const float *qs, const uint8_t *k8, const float *ks, int B, int64_t L,
                     int H, int D, int n_t, int P, int k, const uint8_t *is_ref, int kr, int tile,
                     const int32_t *tile_token, const int32_t *tile_valid, const int32_t *idx, double scale,
                     const uint8_t *todo, double *o_f) {
    qk_operand qo = {q, q8, qs}, ko = {kk, k8, ks};
    qk_tables();
#pragma omp parallel for collapse(3) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n_t; ++i) {
                int64_t bhi = ((int64_t)b * H + h) * n_t + i;
                if (todo && !todo[bhi]) continue;
                double *rows = (double *)malloc(sizeof(double) * (size_t)tile * (size_t)D);
                fine_one_tile(&qo, &ko, v, b, h, i, L, H, D, n_t, P, k, is_ref, kr, tile, tile_token, tile_valid,
                              idx, scale, rows);
                for (int r = 0; r < tile_valid[i]; ++r) {
                    int64_t tok = tile_token[(int64_t)i * tile + r];
                    memcpy(o_f + (((int64_t)b * L + tok) * H + h) * D, rows + (int64_t)r * D,
                           sizeof(double) * (size_t)D);
                }
                free(rows);
            }
}

/* The fine branch of selected query tiles only: items[n] = (b*H + h)*n_t + i;
 * out[n, r, :] for the tile's rows r in tile order (pad rows set to 0). */
void vsa_oracle_fine_tiles(const uint16_t *q, const uint16_t *kk, const uint16_t *v, const uint8_t *q8,
                           const float *qs, const uint8_t *k8, const float *ks, int B, int64_t L,
                           int H, int D, int n_t, int P, int k, const uint8_t *is_ref, int kr, int tile,
                           const int32_t *tile_token,
                           const int32_t *tile_valid, const int32_t *idx, double scale, int n_items,
                           const int64_t *items, double *out) {
    qk_operand qo = {q, q8, qs}, ko = {kk, k8, ks};
    (void)B;
    qk_tables();
#pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_items; ++n) {
        int64_t bhi = items[n];
        int i = (int)(bhi % n_t);
        int64_t bh = bhi / n_t;
        int h = (int)(bh % H), b = (int)(bh / H);
        double *rows = out + (int64_t)n * tile * D;
        for (int64_t e = 0; e < (int64_t)tile * D; ++e) rows[e] = 0.0;
        fine_one_tile(&qo, &ko, v, b, h, i, L, H, D, n_t, P, k, is_ref, kr, tile, tile_token, tile_valid, idx, scale,
                      rows);
    }
}

/* ------------------------------------------------------------------ */
/* O5' fine branch, mask formulation (binary64, second definition)     */
/* ------------------------------------------------------------------ */

/* Dense softmax attention over the packed sequence in token order, where
 * query token a may attend key token c iff c's tile is in the key set of a's
 * tile (the "masked reference" the pages compare the block-sparse kernel
 * against).  Tokens outside every tile do not occur.  Used on small inputs
 * only: builds an L x L mask per (b, h). */
void vsa_oracle_fine_masked(const uint16_t *q, const uint16_t *kk, const uint16_t *v, int B,
                            int64_t L, int H, int D, int n_t, int P, int k, const uint8_t *is_ref, int kr,
                            int tile, const int32_t *tile_token, const int32_t *tile_valid,
                            const int32_t *idx, double scale, double *o_f) {
    int V = n_t - P, w = kr + k;
    int32_t *tile_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)L);
    for (int i = 0; i < n_t; ++i)
        for (int r = 0; r < tile_valid[i]; ++r) tile_of[tile_token[(int64_t)i * tile + r]] = i;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            /* allowed[i * n_t + j]: key tile j in the key set of query tile i */
            uint8_t *allowed = (uint8_t *)calloc((size_t)n_t * n_t, 1);
            int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_t);
            for (int i = 0; i < n_t; ++i) {
                const int32_t *idx_row =
                    (i >= P) ? idx + (((int64_t)b * H + h) * V + (i - P)) * w : NULL;
                int nk = key_set(i, n_t, P, is_ref, w, idx_row, keys);
                for (int t = 0; t < nk; ++t) allowed[(int64_t)i * n_t + keys[t]] = 1;
            }
            double *logit = (double *)malloc(sizeof(double) * (size_t)L);
            for (int64_t a = 0; a < L; ++a) {
                int ti = tile_of[a];
                const uint16_t *qa = q + (((int64_t)b * L + a) * H + h) * D;
                double m = -INFINITY;
                for (int64_t c = 0; c < L; ++c) {
                    if (!allowed[(int64_t)ti * n_t + tile_of[c]]) {
                        logit[c] = -INFINITY;
                        continue;
                    }
                    const uint16_t *kc = kk + (((int64_t)b * L + c) * H + h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += (double)bf16_to_float(qa[d]) * (double)bf16_to_float(kc[d]);
                    logit[c] = scale * dot;
                    if (logit[c] > m) m = logit[c];
                }
                double denom = 0.0;
                for (int64_t c = 0; c < L; ++c) {
                    logit[c] = (logit[c] == -INFINITY) ? 0.0 : exp(logit[c] - m);
                    denom += logit[c];
                }
                double *o = o_f + (((int64_t)b * L + a) * H + h) * D;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int64_t c = 0; c < L; ++c) {
                    if (logit[c] == 0.0) continue;
                    const uint16_t *vc = v + (((int64_t)b * L + c) * H + h) * D;
                    double w = logit[c] / denom;
                    for (int d = 0; d < D; ++d) o[d] += w * (double)bf16_to_float(vc[d]);
                }
            }
            free(logit);
            free(keys);
            free(allowed);
        }
    free(tile_of);
}

/* ------------------------------------------------------------------ */
/* O7 output                                                           */
/* ------------------------------------------------------------------ */

/* out[b, tok, h, d] = o_f[b, tok, h, d] + gate * o_c[b, h, tile(tok), d] for the valid rows of
 * every tile with todo set (NULL: all), no activation (R10, R11).  gate: bf16 bits, either
 * [B, L, H], one scalar per token and head (gate_per_channel = 0), or [B, L, H*D], one per
 * channel h*D + d of the token (gate_per_channel = 1, R12). */
void vsa_oracle_output(const double *o_f, const double *o_c, const uint16_t *gate, int gate_per_channel,
                       int B, int64_t L, int H, int D, int n_t, int tile, const int32_t *tile_token,
                       const int32_t *tile_valid, const uint8_t *todo, double *out) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < n_t; ++i) {
                if (todo && !todo[((int64_t)b * H + h) * n_t + i]) continue;
                const double *oc = o_c + (((int64_t)b * H + h) * n_t + i) * D;
                for (int r = 0; r < tile_valid[i]; ++r) {
                    int64_t tok = tile_token[(int64_t)i * tile + r];
                    int64_t row = (((int64_t)b * L + tok) * H + h);
                    for (int d = 0; d < D; ++d) {
                        uint16_t gbits = gate_per_channel ? gate[row * D + d] : gate[row];
                        double g = (double)bf16_to_float(gbits);
                        out[row * D + d] = o_f[row * D + d] + g * oc[d];
                    }
                }
            }
}
