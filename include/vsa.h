/*
 * vsa.h -- C ABI of libvsa, the VSA-H3 Video Sparse Attention forward on
 * NVIDIA B200 (sm_100a).
 *
 * What the library computes (the method as "Mike0021/FastH3-4step-Preview-VSA"
 * states it in its section "Video Sparse Attention is not optional here"):
 * the packed [text | cond | audio | video] sequence is cut into 64-token
 * tiles -- segment-pure prefix tiles and (4,4,4) cubes of the post-patchify
 * video grid; Q, K and V are pooled per tile; per-head fp32 pooled tile
 * scores pick, for every video query tile, the top-k video key tiles with
 *     topk = max(1, min(ceil((1 - sparsity) * n_video_tiles), n_video_tiles));
 * prefix key tiles are always kept and prefix query tiles attend densely;
 * block-sparse softmax attention runs over the kept tiles; and the
 * compression term -- the pooled V tiles weighted by the softmax of the
 * query tile's scores -- is added to each of the tile's rows, times the
 * per-token gate (no activation).
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev are CUDA device pointers; the caller owns every
 *    tensor and every workspace and must keep them alive until the work on
 *    `stream` has finished.  The library never frees caller memory and never
 *    allocates device memory per call; a plan allocates its own small tables
 *    once, in vsa_plan_tiles, and frees them in vsa_plan_destroy.
 *  - bf16 tensors are raw IEEE bfloat16 bit patterns (vsa_bf16).  Every
 *    device pointer must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  All device work is asynchronous on it; no entry point but
 *    vsa_device_status synchronises.
 *  - Layouts (row-major, last index fastest):
 *      sequence order : q, k, v, out  [B, L, H, D];  gate [B, L, H], or [B, L, H*D]
 *                       with vsa_geometry.gate_per_channel
 *      tile order     : q_t, k_t, v_t [B, H, n_tiles, 64, D]  (pad rows zero)
 *      pooled         : pq, pk, pv    [B, H, n_tiles, D] float
 *      scores         : [B, H, n_tiles, n_tiles] float
 *      selection      : idx [B, H, n_video_tiles, topk] int32, global tile
 *                       indices (prefix tiles are 0..P-1, video tiles P..),
 *                       ascending in each row
 *      compression    : o_c [B, H, n_tiles, D] float
 *  - Tile geometry: prefix tiles in sequence order (a segment of n tokens
 *    gives ceil(n/64) tiles, the last one partial); then the video cubes in
 *    raster (t/4, h/4, w/4) order, edge cubes partial when a grid side is not
 *    a multiple of 4.  Video tokens follow the prefix in raster (t, h, w)
 *    order, w fastest.  Inside a tile the valid tokens come first, in
 *    sequence (prefix) or raster (cube) order, then zero pads.
 *  - A plan's device status word and the attention kernels' work counters are
 *    shared by every call made with that plan: calls with one plan must not
 *    overlap on the GPU (use one plan per concurrent stream).
 *  - The attention may run as two kernels: row blocks that share their key
 *    list (the dense prefix query tiles, when B * H * ceil(P/2) reaches the
 *    SM count; every query tile with 128-token tiles) go two at a time to a
 *    second kernel, on a stream the plan owns that is forked from the
 *    caller's stream with an event and joined back to it before the call
 *    returns, so the caller's stream still orders all of a call's work.
 *  - Errors: argument and shape errors are detected on the host and returned
 *    synchronously with nothing launched; a failed launch returns
 *    VSA_ERR_CUDA; device-side failures (a bounded wait that ran out) are
 *    recorded in the plan's device status word, read with vsa_device_status.
 *    vsa_last_error() returns a message for the calling thread's last error.
 *    There is no fallback path: an unsupported case is an error.
 */
#ifndef VSA_H_
#define VSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VSA_TILE_SIZE 64 /* tokens per tile by default; video tiles are then 4x4x4 cubes */

typedef uint16_t vsa_bf16; /* raw bfloat16 bits */

typedef enum vsa_status {
  VSA_OK = 0,
  VSA_ERR_INVALID_ARG = 1, /* NULL or misaligned pointer, value out of range */
  VSA_ERR_SHAPE = 2,       /* inconsistent sizes */
  VSA_ERR_UNSUPPORTED = 3, /* valid but not implemented (tile size, head_dim) */
  VSA_ERR_WORKSPACE = 4,   /* workspace smaller than vsa_plan_dims.workspace_bytes */
  VSA_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  VSA_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out */
  VSA_ERR_DEVICE = 7       /* no usable sm_100 device */
} vsa_status;

/* Problem statement.  Either `segment_len` (n_segments prefix segments in
 * order, e.g. {text, cond, audio}; zero lengths allowed) or `token_tags`
 * (seq_len tags, one per token; every maximal run of equal tags is one
 * segment; the video run must be last and tagged `video_tag`) describes the
 * prefix.  Host pointers; read only during vsa_plan_tiles. */
typedef struct vsa_geometry {
  int32_t batch;            /* B >= 1 */
  int32_t heads;            /* H >= 1 */
  int32_t head_dim;         /* D: 64, 96 or 128 */
  int32_t n_segments;       /* number of prefix segments (ignored with tags) */
  const int32_t* segment_len;
  const int32_t* token_tags; /* NULL to use segment_len */
  int64_t seq_len;           /* L: required with tags; checked otherwise */
  int32_t video_tag;         /* tag value of the video tokens (tags only) */
  int32_t grid_t, grid_h, grid_w; /* post-patchify video grid; 0 = no video */
  int32_t tile_size;         /* tokens per tile: 64, or 128 (the OmniRef variant: "FastH3
                                OmniRef inference", section "The Blackwell stack").  A prefix
                                tile is a segment-pure run of up to tile_size tokens, a video
                                tile a cube_t x cube_h x cube_w block of the grid. */
  double sparsity;           /* in [0, 1] */
  float softmax_scale;       /* 0 => (float)(1 / sqrt((double)head_dim)) */
  int32_t gate_per_channel;  /* 0: gate [B, L, H], one scalar per token and head;
                                1: gate [B, L, H*D], one per channel h*D + d */
  int32_t seq_tiles;         /* 0: vsa_forward copies Q/K/V to tile order first (faster on B200);
                                1: the attention reads each tile straight from sequence order
                                with 4-D/5-D TMA boxes: no tile-order copies, a workspace smaller
                                by 3*B*H*n_tiles*64*D*2 bytes, batch <= 4, 64-token tiles */
  int32_t qk_fp8;            /* 0: the fine branch's logits use the bf16 Q and K;
                                1: 8-bit Q/K: each (token, head) row of Q and K is quantised to
                                OCP FP8 E4M3 codes with one binary32 scale s = amax / 448
                                (code = E4M3(x / s), round to nearest even, saturating; an
                                all-zero row has s = 0), and the logits are the 8-bit product
                                times both scales.  Selection, compression and P.V keep bf16.
                                Every query tile is covered.  Passages: "FastH3 OmniRef
                                inference", sections "The Blackwell stack" and "Fallbacks"
                                (8-bit per-token Q/K with bf16 P.V); "FastH3 NVFP4 on RTX PRO
                                6000 (sm_120)", multi-GPU notes (one FP8 scale per token and
                                head);
                                2: the pages' prefix split: the dense prefix query tiles take the
                                8-bit logits of 1, the video query tiles keep bf16.  Passage:
                                "FastH3 OmniRef inference", section "Device profiles" (dense
                                prefix query tiles: Q and K rounded to 8 bits, bf16 P.V);
                                3: the prefix split of 2, and the video query tiles' logits use
                                FP4 Q and K: K smoothed first (mu[b, h, d] = the key mean over
                                the L tokens, a binary64 sum / L rounded to binary32, subtracted
                                in binary32), then every row of Q and K cut into blocks of 16
                                values, each block scaled by the E4M3 code of amax / 6 (binary32
                                division, nearest even, saturating) and each value rounded to
                                the nearest E2M1 value of x / scale (ties to even, saturating at
                                6); global scale 1.  The rounded values are bf16 numbers and
                                run through the bf16 attention.  The key mean's binary64 sum is
                                computed in parallel: it equals the token-order sum when that
                                sum is exact (a column's bf16 values within about 2^28 of one
                                another at L = 75,008), and otherwise may differ in its last
                                bits, which reaches the binary32 mean only near a rounding
                                boundary.  Passages: "FastH3 OmniRef inference", sections
                                "Device profiles", "Environment" and "Fallbacks"; "FastH3 NVFP4
                                on RTX PRO 6000 (sm_120)", model integration.
                                Modes 1 to 3 need seq_tiles = 0, and only the whole-forward
                                entry points accept such a plan. */
  int32_t cube_t, cube_h, cube_w; /* video cube shape, product = tile_size; all 0 = the default:
                                     4x4x4 for 64 tokens (the method's), 4x4x8 for 128 (the
                                     pages do not state it: the 64-token cube doubled along w) */
  const int32_t* segment_reference; /* NULL, or n_segments flags (segments only, not tags): 1 marks a
                                       reference segment ("FastH3 OmniRef inference", section "The
                                       Blackwell stack": "reference keep").  Its R tiles are not
                                       always-kept keys: each video query tile keeps the kr of them
                                       with the highest pooled scores (ties: lower index),
                                       kr = max(1, min(ceil(reference_keep * R), R)) in binary64;
                                       the other prefix tiles stay always kept and prefix query
                                       tiles stay dense.  idx rows then hold kr + topk entries: the
                                       kept reference tiles, then the video tiles, each ascending. */
  double reference_keep;            /* in (0, 1]; read when a segment is a reference segment */
} vsa_geometry;

typedef struct vsa_plan_s* vsa_plan; /* opaque, library-owned */

/* Sizes a plan resolved. */
typedef struct vsa_plan_dims {
  int32_t n_tiles;        /* P + V */
  int32_t n_prefix_tiles; /* P */
  int32_t n_video_tiles;  /* V */
  int32_t topk;           /* kept video key tiles per video query tile */
  int64_t seq_len;        /* L */
  float softmax_scale;    /* the scale actually used */
  size_t workspace_bytes; /* device scratch vsa_forward needs */
  int64_t selected_pairs; /* (query tile, key tile) pairs per (b, h):
                             V * (P - R + kr + topk) + P * n_tiles */
  int32_t tile_size;      /* tokens per tile (64 or 128) */
  int32_t n_ref_tiles;    /* R: prefix tiles of reference segments */
  int32_t ref_topk;       /* kr: reference tiles kept per video query tile (0 without any) */
} vsa_plan_dims;

/* ---- S1: tile plan (host) ------------------------------------------------
 * vsa_plan_tiles: resolve the tile geometry (segments -> segment-pure prefix
 * tiles, grid -> (4,4,4) cubes, the topk count), build the token table of
 * every tile and upload it to the current device, asynchronously on
 * `stream`.  Allocates the plan's device tables (a few hundred KB at most)
 * and its device status word.  On success *out owns them.
 * Passage: "Mike0021/FastH3-4step-Preview-VSA", section "Video Sparse
 * Attention is not optional here" (tile geometry, topk formula); "FastH3
 * NVFP4 on RTX PRO 6000 (sm_120)", section "Block-sparse FP4 attention for
 * VSA tiles" (partially filled tiles carry valid counts). */
vsa_status vsa_plan_tiles(const vsa_geometry* g, void* stream, vsa_plan* out);

/* Resolved sizes.  Host only; never blocks. */
vsa_status vsa_plan_info(vsa_plan p, vsa_plan_dims* out);

/* Host copies of the plan's tables: tile_token[n_tiles * tile_size] (sequence index
 * of each tile row, -1 for a pad) and tile_valid[n_tiles] (valid rows).
 * Either pointer may be NULL.  Host only. */
vsa_status vsa_plan_tables(vsa_plan p, int32_t* tile_token, int32_t* tile_valid);

/* Resolve sizes without a device (no plan, no allocation). */
vsa_status vsa_plan_query(const vsa_geometry* g, vsa_plan_dims* out);

/* The token table a plan would upload, computed on the host without a device:
 * tile_token[n_tiles * tile_size] and tile_valid[n_tiles] (caller-allocated host
 * arrays, sized from vsa_plan_query).  Either pointer may be NULL. */
vsa_status vsa_plan_tables_host(const vsa_geometry* g, int32_t* tile_token, int32_t* tile_valid);

/* Free the plan's device tables (synchronises with the device first). */
vsa_status vsa_plan_destroy(vsa_plan p);

/* ---- S2: gather to tile order --------------------------------------------
 * q_t/k_t/v_t[b,h,tile,r,:] = q/k/v[b, token(tile, r), h, :], pad rows zero.
 * If pq, pk and pv are all non-NULL the pooled tiles (S3's first half) are
 * written in the same pass, bit-identical to vsa_pool_and_score's.
 * If q_norm and kv_max are non-NULL too (both or neither; only with pooling),
 * the same pass writes the attention's overflow-bound statistics of the
 * tiles: q_norm [B, H, n_tiles, tile_size] float32, the Euclidean norm of
 * every query row (0 for pads), and kv_max [B, H, 2] float32, the largest
 * key-row norm and |v| of each (b, h) -- the values vsa_forward keeps in its
 * workspace (q_n, kv_max), to be passed on to vsa_sparse_attn_fwd.
 * Passage: "FastH3 NVFP4 on RTX PRO 6000 (sm_120)", section "Model
 * integration" (gather to tile order once; pad rows zero). */
vsa_status vsa_gather_tiles(vsa_plan p, const vsa_bf16* q_dev, const vsa_bf16* k_dev,
                            const vsa_bf16* v_dev, vsa_bf16* q_t_dev, vsa_bf16* k_t_dev,
                            vsa_bf16* v_t_dev, float* pq_dev, float* pk_dev, float* pv_dev,
                            float* q_norm_dev, float* kv_max_dev, void* stream);

/* ---- S3: pooling and pooled tile scores ----------------------------------
 * pooled[b,h,t,d] = (sum over the tile's valid rows r, in tile order, from
 * +0.0f, one binary32 rounding per add) / n_valid  (IEEE division);
 * scores[b,h,i,j] = fl(fmaf chain over d = 0..D-1 of pq[i,d]*pk[j,d], from
 * +0.0f) * softmax_scale.  Every (i, j) pair, prefix tiles included.
 * Inputs in tile order.  If q_t_dev is NULL the pooling is skipped and pq/pk
 * must already hold pooled tiles (e.g. from vsa_gather_tiles).
 * Passage: "Mike0021/FastH3-4step-Preview-VSA", section "Video Sparse
 * Attention is not optional here" (per-head fp32 pooled tile scores). */
vsa_status vsa_pool_and_score(vsa_plan p, const vsa_bf16* q_t_dev, const vsa_bf16* k_t_dev,
                              const vsa_bf16* v_t_dev, float* pq_dev, float* pk_dev,
                              float* pv_dev, float* scores_dev, void* stream);

/* ---- S4: top-k selection and the compression branch ---------------------
 * idx[b,h,iv,:] = the topk video key tiles with the highest scores[b,h,P+iv,
 * P+j] (ties: lower index first), as global indices in ascending order
 * (with reference segments: first the kr kept reference tiles, ascending, so a
 * row holds kr + topk entries);
 * o_c[b,h,i,:] = sum_j softmax_j(scores[b,h,i,:]) * pv[b,h,j,:] over all
 * n_tiles tiles, in binary32.
 * Passage: "Mike0021/FastH3-4step-Preview-VSA", section "Video Sparse
 * Attention is not optional here" (top-k; compression softmax(scores) @
 * pool(v)); "FastH3 NVFP4 on RTX PRO 6000 (sm_120)", section "Block-sparse
 * FP4 attention for VSA tiles" (per-query-block index lists). */
vsa_status vsa_topk_select(vsa_plan p, const float* scores_dev, const float* pv_dev,
                           int32_t* idx_dev, float* o_c_dev, void* stream);

/* ---- S5: block-sparse attention and the gated epilogue -------------------
 * For a video query tile: softmax attention over the keys of all prefix
 * tiles and of its idx row; for a prefix query tile: over every tile.  Pad
 * keys are masked.  Then out[b,l,h,:] = o_fine + gate[b,l,h] * o_c[b,h,
 * tile(l),:] (with a per-channel gate, gate[b,l,h*D+d] scales column d),
 * rounded to bf16 and written in sequence order (pad rows are not written).  Q/K/V in tile order; BF16 tensor-core products with fp32
 * accumulation; P rounded to bf16 before the P.V product.
 * Passage: "FastH3 NVFP4 on RTX PRO 6000 (sm_120)", section "Block-sparse FP4
 * attention for VSA tiles" (block lists, exempt prefix key tile visited
 * first); "Mike0021/FastH3-4step-Preview-VSA", section "Video Sparse
 * Attention is not optional here" (dense prefix queries; gated compression
 * branch with no activation).
 * The rescale checks of the softmax are bounded with the tiles' magnitude
 * statistics (see vsa_gather_tiles): pass those of exactly these q_t, k_t,
 * v_t as q_norm_dev and kv_max_dev (statistics of other tensors void the
 * bound, and the output may then overflow to infinity), or NULL for both:
 * the call then takes them itself first (one extra kernel reading the
 * tiles, into a buffer the plan owns, so such calls on one plan must not
 * overlap).  Either way the output is bit-identical to vsa_forward's. */
vsa_status vsa_sparse_attn_fwd(vsa_plan p, const vsa_bf16* q_t_dev, const vsa_bf16* k_t_dev,
                               const vsa_bf16* v_t_dev, const int32_t* idx_dev,
                               const float* o_c_dev, const vsa_bf16* gate_dev,
                               vsa_bf16* out_dev, const float* q_norm_dev,
                               const float* kv_max_dev, void* stream);

/* ---- the whole forward ---------------------------------------------------
 * S2..S5 in one call, sequence order in and out.  `workspace_dev` must hold
 * vsa_plan_dims.workspace_bytes bytes (256-byte aligned); its contents on
 * entry do not matter and on return are the intermediates (tile-order Q/K/V,
 * unless the plan has seq_tiles; pooled tiles, scores, idx, o_c) at offsets
 * vsa_workspace_layout gives.
 * When every gate value is zero (+0 or -0) the compression branch adds
 * nothing: a device-side check then skips its kernel and its epilogue term,
 * and the o_c region is left as it was. */
vsa_status vsa_forward(vsa_plan p, const vsa_bf16* q_dev, const vsa_bf16* k_dev,
                       const vsa_bf16* v_dev, const vsa_bf16* gate_dev, vsa_bf16* out_dev,
                       void* workspace_dev, size_t workspace_bytes, void* stream);

/* ---- the whole forward over sequence parts (sequence parallelism) ---------
 * The forward of vsa_forward for this plan's H heads, when the sequence-order
 * tensors are split by token into `nparts` parts, as a sequence-parallel
 * (Ulysses) layout has them: part p holds tokens [p*Ls, (p+1)*Ls) of q, k, v
 * and gate, and receives those tokens of out.  Each part is a [B, Ls, Htot, D]
 * tensor ([B, Ls, Htot] or [B, Ls, Htot*D] for the gate), and this call reads
 * and writes heads [head_offset, head_offset + H) of it.  Parts may be peer
 * mappings of other GPUs' memory (NVLink): then the seq->head exchange happens
 * inside the gather kernel's loads and the head->seq exchange inside the
 * attention epilogue's stores, with no separate all-to-all.  Passage: "FastH3
 * NVFP4 on RTX PRO 6000 (sm_120)", section "What was tried" (Ulysses sequence
 * parallelism: all-to-all of q/k/v/gate to heads and of the output back).
 *  - Requires nparts * tokens_per_part == L, head_offset + H <= heads_total,
 *    a plan without seq_tiles, and 16-byte aligned pointers.
 *  - The caller orders the call after the parts' producers (on every GPU
 *    whose memory a part lives in) and consumers of out after the call, e.g.
 *    with a barrier on each side; nothing inside the call waits on another
 *    GPU.  Calls with one plan must not overlap.
 *  - The all-zero-gate check is not run (the compression branch is kept).
 * Errors: VSA_ERR_INVALID_ARG, VSA_ERR_SHAPE, VSA_ERR_UNSUPPORTED,
 * VSA_ERR_WORKSPACE, VSA_ERR_CUDA. */
#define VSA_MAX_PARTS 64
typedef struct vsa_seq_parts {
  int32_t nparts;              /* 1..VSA_MAX_PARTS */
  int64_t tokens_per_part;     /* Ls */
  int32_t heads_total;         /* Htot of the parts' layout */
  int32_t head_offset;         /* first of this plan's heads within Htot */
  const vsa_bf16* const* q;    /* nparts device pointers each (local or peer-mapped) */
  const vsa_bf16* const* k;
  const vsa_bf16* const* v;
  const vsa_bf16* const* gate;
  vsa_bf16* const* out;
} vsa_seq_parts;
vsa_status vsa_forward_parts(vsa_plan p, const vsa_seq_parts* parts, void* workspace_dev,
                             size_t workspace_bytes, void* stream);

/* ---- the whole forward with inputs and output in host memory ---------------
 * The forward of vsa_forward for q, k, v [B, L, H, D], gate [B, L, H] (or [B, L, H*D]) and out
 * [B, L, H, D] that live in HOST memory (bf16, sequence order).  No
 * counterpart on the pages: the heads of the attention are independent, so
 * the call processes them in chunks of `head_chunk` heads and overlaps, on
 * three streams, the host->device copy of one chunk, the forward of the
 * previous one on `stream` and the device->host copy of the one before.
 * The result is bit-identical to vsa_forward on the same inputs.
 *  - Host buffers should be page-locked; pageable memory still gives the
 *    right result, but the copies then do not overlap.
 *  - `workspace_dev` (256-byte aligned) must hold the bytes that
 *    vsa_forward_host_workspace returns for the same head_chunk: a
 *    forward workspace for one chunk, two staging slots and the gate.
 *  - The call returns once everything is enqueued; `out` is complete when
 *    `stream` has drained (cudaStreamSynchronize).  Earlier work on `stream`
 *    finishes before the call's copies start.
 *  - The first call with a given head_chunk creates two copy streams, eight
 *    events and the head-slice plans; they belong to the plan and are
 *    released by vsa_plan_destroy.  Calls with one plan must not overlap.
 * Errors: VSA_ERR_INVALID_ARG (NULL pointer, head_chunk outside [1, H],
 * unaligned workspace), VSA_ERR_WORKSPACE (workspace too small), VSA_ERR_CUDA
 * (a copy or launch failed). */
vsa_status vsa_forward_host_workspace(vsa_plan p, int32_t head_chunk, size_t* bytes);
vsa_status vsa_forward_host(vsa_plan p, const vsa_bf16* q_host, const vsa_bf16* k_host,
                            const vsa_bf16* v_host, const vsa_bf16* gate_host, vsa_bf16* out_host,
                            int32_t head_chunk, void* workspace_dev, size_t workspace_bytes,
                            void* stream);

/* ---- the whole forward without a caller workspace -------------------------
 * No counterpart on the pages: this entry point exists for callers that
 * cannot allocate device memory on their call path -- for instance a plugin
 * running inside a host engine that owns all device memory, or a serving loop
 * whose memory budget is fixed after start-up -- and so cannot hand
 * vsa_forward a workspace.  It runs exactly vsa_forward's kernels, with the
 * scratch held in one file-scope device array of VSA_NOALLOC_SCRATCH_BYTES
 * (64 MiB) that every GPU which loads libvsa keeps until the process exits.
 * The caller still passes the inputs and the output.  It allocates nothing:
 * no cudaMalloc, cudaFree or allocating library routine.
 *  - A plan whose vsa_plan_dims.workspace_bytes exceeds the array is
 *    rejected with VSA_ERR_WORKSPACE before anything is launched.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture on the device.
 *  - Every call on a device uses the same array: calls whose work may
 *    overlap on the GPU (different streams, or several threads) race and
 *    must be serialised by the caller.  Nothing in the array needs to start
 *    at zero; each call overwrites what it reads.
 * On return the array holds the call's intermediates (not exposed). */
#define VSA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
vsa_status vsa_forward_noalloc(vsa_plan p, const vsa_bf16* q_dev, const vsa_bf16* k_dev,
                               const vsa_bf16* v_dev, const vsa_bf16* gate_dev, vsa_bf16* out_dev,
                               void* stream);

/* Byte offsets of the intermediates inside vsa_forward's workspace.  With
 * qk_fp8, q_t and k_t hold E4M3 codes [B, H, n_tiles, 64, 128] (128 bytes per
 * row whatever D; bytes D..127 zero) and q_s, k_s the row scales [B, H,
 * n_tiles, 64] float32 (0 for pad rows); otherwise q_s and k_s are empty.
 * q_n holds the Euclidean norm of every query row [B, H, n_tiles, tile_size]
 * float32 (tile-order rows, 0 for pad rows; with qk_fp8 the norm of the
 * dequantised row, scale times code norm) and kv_max, per (b, h), the largest
 * key-row norm (likewise) and the largest |v| (two float32); the attention
 * bounds its logits by them (Cauchy-Schwarz) to skip rescale checks that
 * cannot fire. */
/* With qk_fp8 = 2 (the prefix split) q_t and k_t hold the bf16 copies, q_c and k_c
 * the E4M3 codes [B, H, n_tiles, 64, 128] with their row scales in q_s, k_s, and
 * q_n8, kv_max8 the statistics of the dequantised rows (q_c .. kv_max8 are empty
 * otherwise).  Only the prefix tiles' query rows are quantised (the video query
 * tiles keep bf16 logits): the video tiles' part of q_c, q_s and q_n8 is left as
 * it was.  With qk_fp8 = 3 the same, and the video query tiles of q_t and every
 * valid key row of k_t hold their FP4 roundings (bf16 numbers), k_sum the binary64
 * key column sums [B, H, D] and k_mu the key means [B, H, D] float32 (k_sum and
 * k_mu are empty otherwise); q_n and kv_max are the statistics of the rounded
 * copies. */
typedef struct vsa_workspace_layout {
  size_t q_t, k_t, v_t, q_s, k_s, q_n, kv_max, pq, pk, pv, scores, idx, o_c;
  size_t q_c, k_c, q_n8, kv_max8, k_sum, k_mu, total;
} vsa_workspace_layout;
vsa_status vsa_plan_workspace(vsa_plan p, vsa_workspace_layout* out);

/* Failure-detection self-test.  No counterpart on the pages: it checks the
 * library's own safety net.  It launches one small kernel whose threads wait,
 * with the same bounded-wait code the attention kernel uses, on a barrier that
 * nothing ever arrives on, with a limit of timeout_ns (1e3 .. 1e10).  The first
 * wait to run out writes VSA_ERR_TIMEOUT and a site code to the plan's device
 * status word; the other threads give up when they see the abort.  The call
 * synchronises `stream`, returns the status word in *code and *where (NULL
 * allowed), and clears it.  A working build returns VSA_OK with *code ==
 * VSA_ERR_TIMEOUT, after about timeout_ns.  The GPU context stays usable. */
vsa_status vsa_wait_selftest(vsa_plan p, int64_t timeout_ns, void* stream, int32_t* code, int32_t* where);

/* Read (synchronising `stream`) and clear the plan's device status word.
 * *code receives VSA_OK or VSA_ERR_TIMEOUT; *where a kernel-specific site
 * code (0 if none). */
vsa_status vsa_device_status(vsa_plan p, void* stream, int32_t* code, int32_t* where);

/* Message for the calling thread's most recent error ("" if none). */
const char* vsa_last_error(void);

/* Library version string. */
const char* vsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H_ */
