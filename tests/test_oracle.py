"""Pins for the CPU oracle: what the pages and the mathematics fix, checked
against the oracle without reference to the CUDA library.

Each test states what pins it: a closed form, a special case that reduces to
a library routine (torch's scaled_dot_product_attention), brute force on tiny
inputs, an invariant, or an exact value within an error bound.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import synth

# ---------------------------------------------------------------------------
# helpers (independent of the oracle's code)
# ---------------------------------------------------------------------------


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return synth.as_bits(x.to(torch.bfloat16))


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def token_coords(w: synth.Workload, tok: int):
    """Decode a packed-sequence index into ('prefix', segment, offset) or
    ('video', t, h, w) -- written here from the packing statement alone."""
    off = 0
    for s, n in enumerate(w.segments):
        if tok < off + n:
            return ("prefix", s, tok - off)
        off += n
    v = tok - off
    T, H, W = w.grid
    return ("video", v // (H * W), (v // W) % H, v % W)


def dense_sdpa(q, k, v, scale):
    """torch SDPA in float64 over [L, D] operands (library routine)."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
        scale=scale)
    return out[0, 0].numpy()


def rand_bits(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return bf16_bits(torch.randn(*shape, generator=g, dtype=torch.float64) * scale)


# ---------------------------------------------------------------------------
# O1 geometry
# ---------------------------------------------------------------------------

# (n_tiles, n_prefix, n_video) by hand:
#   tiny : ceil(40/64)+ceil(24/64) = 2 ; (8/4)(8/4)(8/4) = 8
#   small: 256/64 + 64/64 + 192/64 = 8 ; (8/4)(16/4)(32/4) = 64
#   480p : 384/64 + 384/64 = 12 ; ceil(8/4) ceil(30/4) ceil(56/4) = 2*8*14 = 224
#   768p : 512/64 + 768/64 = 20 ; (24/4)(48/4)(64/4) = 6*12*16 = 1152
GEOMETRY = {
    "tiny": (10, 2, 8),
    "small": (72, 8, 64),
    "480p": (236, 12, 224),
    "768p_s0.8": (1172, 20, 1152),
    "768p_s0.9": (1172, 20, 1152),
}


@pytest.mark.parametrize("name", list(GEOMETRY))
def test_geometry_counts(oracle_mod, name):
    w = synth.workload(name)
    geo = oracle_mod.geometry(w.segments, w.grid)
    assert (geo.n_tiles, geo.n_prefix, geo.n_video) == GEOMETRY[name]
    assert geo.seq_len == w.seq_len


@pytest.mark.parametrize("name", ["tiny", "small", "480p"])
def test_geometry_partition(oracle_mod, name):
    """Every token sits in exactly one tile; valid rows first; prefix tiles are
    segment-pure runs of consecutive tokens; a video tile is one (4,4,4) cube
    with its tokens in raster (t,h,w) order."""
    w = synth.workload(name)
    geo = oracle_mod.geometry(w.segments, w.grid)
    tok, val = geo.tile_token, geo.tile_valid
    assert int(val.sum()) == w.seq_len
    seen = np.zeros(w.seq_len, np.int64)
    for i in range(geo.n_tiles):
        n = int(val[i])
        assert 1 <= n <= 64
        assert (tok[i, :n] >= 0).all() and (tok[i, n:] == -1).all()
        seen[tok[i, :n]] += 1
        coords = [token_coords(w, int(t)) for t in tok[i, :n]]
        if i < geo.n_prefix:
            assert all(c[0] == "prefix" for c in coords)
            assert len({c[1] for c in coords}) == 1  # segment-pure
            assert list(tok[i, :n]) == list(range(tok[i, 0], tok[i, 0] + n))
            assert coords[0][2] % 64 == 0
        else:
            assert all(c[0] == "video" for c in coords)
            cubes = {(c[1] // 4, c[2] // 4, c[3] // 4) for c in coords}
            assert len(cubes) == 1
            assert [c[1:] for c in coords] == sorted(c[1:] for c in coords)
    assert (seen == 1).all()
    # cubes appear in raster order of their (a, b, c) coordinates
    firsts = [token_coords(w, int(tok[i, 0]))[1:] for i in range(geo.n_prefix, geo.n_tiles)]
    cube_ids = [(t // 4, h // 4, x // 4) for (t, h, x) in firsts]
    assert cube_ids == sorted(cube_ids) and len(set(cube_ids)) == geo.n_video


def test_geometry_partial_cubes(oracle_mod):
    """480p: H = 30 is not a multiple of 4; the last cube row holds 4*2*4 = 32
    tokens, and there are 2 * 14 = 28 such cubes."""
    w = synth.workload("480p")
    geo = oracle_mod.geometry(w.segments, w.grid)
    v = geo.tile_valid[geo.n_prefix:]
    assert int((v == 32).sum()) == 28 and int((v == 64).sum()) == 224 - 28
    # tiny: the text tile holds 40 valid tokens, the audio tile 24
    t = synth.workload("tiny")
    g2 = oracle_mod.geometry(t.segments, t.grid)
    assert list(g2.tile_valid[:2]) == [40, 24]


def test_geometry_edge_cases(oracle_mod):
    # grid sides below 4 and empty segments
    geo = oracle_mod.geometry((0, 0, 1), (1, 2, 3))
    assert (geo.n_tiles, geo.n_prefix, geo.n_video) == (2, 1, 1)
    assert list(geo.tile_valid) == [1, 6]
    geo = oracle_mod.geometry((65,), (0, 0, 0))
    assert (geo.n_tiles, geo.n_prefix, geo.n_video) == (2, 2, 0)
    assert list(geo.tile_valid) == [64, 1]


# ---------------------------------------------------------------------------
# O4 topk count
# ---------------------------------------------------------------------------


def _golden_topk():
    rows = []
    with open(__file__.replace("test_oracle.py", "golden/topk_table.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                s, V, k = line.split()
                rows.append((float(s), int(V), int(k)))
    return rows


@pytest.mark.parametrize("s,V,k", _golden_topk())
def test_topk_count_table(oracle_mod, s, V, k):
    assert oracle_mod.topk_count(s, V) == k


# ---------------------------------------------------------------------------
# O2 pooling, O3 scores
# ---------------------------------------------------------------------------


def test_pool_special_cases(oracle_mod):
    """A tile whose valid rows are all equal pools to that value exactly; a
    one-token tile pools to its token; pads never count."""
    segments, grid = (40, 1), (4, 4, 8)
    geo = oracle_mod.geometry(segments, grid)
    L, H, D = geo.seq_len, 2, 16
    x = np.zeros((1, L, H, D), np.float32)
    x[0, :40] = 0.71875  # the 40-token text tile, constant (bf16-exact)
    x[0, 40] = -3.25  # the one-token cond tile
    rng = np.random.default_rng(0)
    x[0, 41:] = rng.standard_normal((L - 41, H, D))
    bits = bf16_bits(torch.from_numpy(x))
    p = oracle_mod.pool(bits, geo)
    assert (p[0, :, 0, :] == np.float32(0.71875)).all()
    assert (p[0, :, 1, :] == np.float32(-3.25)).all()


def test_pool_matches_exact_mean(oracle_mod):
    """fp32 pooled means agree with the exact mean (fp64) within the
    sequential-sum error bound n * eps32 * sum|x| / n + the division."""
    w = synth.workload("small")
    geo = oracle_mod.geometry(w.segments, w.grid)
    x = rand_bits((1, w.seq_len, 3, 128), 1)
    p = oracle_mod.pool(x, geo).astype(np.float64)
    xf = bits_to_f64(x)
    eps = 2.0 ** -24
    for i in range(geo.n_tiles):
        n = geo.tile_valid[i]
        rows = xf[0, geo.tile_token[i, :n]]  # [n, H, D]
        exact = rows.mean(axis=0)  # [H, D]
        bound = (n + 1) * eps * np.abs(rows).sum(axis=0) / n + eps * np.abs(exact)
        assert (np.abs(p[0, :, i, :] - exact) <= bound).all()


def test_scores_bound_and_symmetry(oracle_mod):
    rng = np.random.default_rng(2)
    pq = rng.standard_normal((1, 2, 12, 128)).astype(np.float32)
    pk = rng.standard_normal((1, 2, 12, 128)).astype(np.float32)
    scale = oracle_mod.default_scale(128)
    S = oracle_mod.scores(pq, pk, scale).astype(np.float64)
    exact = np.einsum("bhid,bhjd->bhij", pq.astype(np.float64), pk.astype(np.float64)) * scale
    absdot = np.einsum("bhid,bhjd->bhij", np.abs(pq).astype(np.float64), np.abs(pk).astype(np.float64))
    eps = 2.0 ** -24
    assert (np.abs(S - exact) <= (128 + 2) * eps * absdot * scale + eps * np.abs(exact)).all()
    # the fmaf chain is symmetric in its two operands
    Ss = oracle_mod.scores(pq, pq, scale)
    assert (Ss == np.swapaxes(Ss, -1, -2)).all()
    # a power-of-two scale multiplies exactly
    S1 = oracle_mod.scores(pq, pk, 1.0)
    S4 = oracle_mod.scores(pq, pk, 0.25)
    assert (S4 == S1 * np.float32(0.25)).all()
    # the default scale is 1/sqrt(D) rounded once to binary32
    assert np.float32(oracle_mod.default_scale(128)) == np.float32(1 / math.sqrt(128))
    assert oracle_mod.default_scale(64) == 0.125


# ---------------------------------------------------------------------------
# O4 selection
# ---------------------------------------------------------------------------


def _dominates(a, b):
    """Tile a ranks above tile b: higher score, or equal score and lower index."""
    return a[0] > b[0] or (a[0] == b[0] and a[1] < b[1])


def test_select_brute_force_tiny(oracle_mod):
    """Of all C(8,4)=70 subsets of the 8 video key tiles, exactly one has every
    member ranked above every non-member; it equals the oracle's pick."""
    w = synth.workload("tiny")
    x = synth.make_inputs(w)
    geo = oracle_mod.geometry(w.segments, w.grid)
    pq = oracle_mod.pool(synth.as_bits(x["q"]), geo)
    pk = oracle_mod.pool(synth.as_bits(x["k"]), geo)
    S = oracle_mod.scores(pq, pk, oracle_mod.default_scale(w.head_dim))
    k = oracle_mod.topk_count(w.sparsity, geo.n_video)
    idx = oracle_mod.select(S, geo.n_prefix, k)
    P, V = geo.n_prefix, geo.n_video
    for h in range(w.heads):
        for iv in range(V):
            row = [(float(S[0, h, P + iv, P + j]), P + j) for j in range(V)]
            winners = []
            for sub in itertools.combinations(range(V), k):
                ins = [row[j] for j in sub]
                outs = [row[j] for j in range(V) if j not in sub]
                if all(_dominates(a, b) for a in ins for b in outs):
                    winners.append([P + j for j in sub])
            assert len(winners) == 1
            assert list(idx[0, h, iv]) == winners[0]


def test_select_ties_go_to_lower_index(oracle_mod):
    P, V = 1, 6
    n_t = P + V
    S = np.zeros((1, 1, n_t, n_t), np.float32)
    S[0, 0, P:, P:] = np.array([1.0, 2.0, 2.0, 0.5, 2.0, 3.0], np.float32)
    idx = oracle_mod.select(S, P, 3)  # 3.0 (j=5), then the 2.0s at j=1, 2
    assert list(idx[0, 0, 0]) == [P + 1, P + 2, P + 5]
    idx = oracle_mod.select(S, P, 6)
    assert list(idx[0, 0, 0]) == [P + j for j in range(6)]
    S[0, 0, P:, P:] = 0.0  # all equal: the lowest k indices
    assert list(oracle_mod.select(S, P, 2)[0, 0, 3]) == [P, P + 1]


# ---------------------------------------------------------------------------
# O5 fine branch
# ---------------------------------------------------------------------------


def _tiny_case(sparsity, heads=2):
    w = synth.workload("tiny", sparsity=sparsity, heads=heads)
    x = synth.make_inputs(w)
    return w, {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}


def test_fine_sparsity0_equals_dense_attention(oracle_mod):
    """At sparsity 0 every query sees every token: the fine branch is plain
    softmax attention over the packed sequence (torch SDPA in float64)."""
    w, x = _tiny_case(0.0)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.0)
    assert r.topk == r.geo.n_video
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    for h in range(w.heads):
        ref = dense_sdpa(q[0, :, h], k[0, :, h], v[0, :, h], r.scale)
        assert np.abs(r.o_f[0, :, h] - ref).max() < 1e-12


def test_fine_prefix_queries_are_dense(oracle_mod):
    w, x = _tiny_case(0.5)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.5)
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    npre = sum(w.segments)
    for h in range(w.heads):
        ref = dense_sdpa(q[0, :npre, h], k[0, :, h], v[0, :, h], r.scale)
        assert np.abs(r.o_f[0, :npre, h] - ref).max() < 1e-12


def test_fine_video_query_sees_prefix_and_selected(oracle_mod):
    """A video query row attends exactly the tokens of the prefix tiles and of
    its selected tiles: SDPA over that token subset reproduces it."""
    w, x = _tiny_case(0.5)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.5)
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    geo = r.geo
    for h in range(w.heads):
        for iv in range(geo.n_video):
            i = geo.n_prefix + iv
            tiles = list(range(geo.n_prefix)) + list(r.idx[0, h, iv])
            assert len(set(tiles)) == geo.n_prefix + r.topk
            keys = np.concatenate([geo.tile_token[t, :geo.tile_valid[t]] for t in tiles])
            qs = geo.tile_token[i, :geo.tile_valid[i]]
            ref = dense_sdpa(q[0, qs, h], k[0, keys, h], v[0, keys, h], r.scale)
            assert np.abs(r.o_f[0, qs, h] - ref).max() < 1e-12


def test_fine_topk1_two_tiles_by_hand(oracle_mod):
    """No prefix, two video tiles, sparsity 0.5 -> topk = 1.  Make tile 0's
    pooled q/k strongly aligned with tile 1's k: both query tiles must pick
    tile 1, and each query row is softmax attention over tile 1 alone."""
    segments, grid = (), (4, 4, 8)
    geo = oracle_mod.geometry(segments, grid)
    assert (geo.n_prefix, geo.n_video, oracle_mod.topk_count(0.5, 2)) == (0, 2, 1)
    L, D = 128, 64
    rng = np.random.default_rng(3)
    qf = rng.standard_normal((1, L, 1, D)) * 0.1
    kf = rng.standard_normal((1, L, 1, D)) * 0.1
    vf = rng.standard_normal((1, L, 1, D))
    t1 = geo.tile_token[1, :64]
    qf[0, :, 0, :] += 1.0  # every query points along +1
    kf[0, t1, 0, :] += 1.0  # only tile 1's keys point along +1
    q, k, v = (bf16_bits(torch.from_numpy(a)) for a in (qf, kf, vf))
    gate = bf16_bits(torch.zeros(1, L, 1))
    r = oracle_mod.forward(q, k, v, gate, segments, grid, 0.5)
    assert r.idx[0, 0, :, 0].tolist() == [1, 1]
    qd, kd, vd = (bits_to_f64(a) for a in (q, k, v))
    ref = dense_sdpa(qd[0, :, 0], kd[0, t1, 0], vd[0, t1, 0], r.scale)
    assert np.abs(r.o_f[0, :, 0] - ref).max() < 1e-12


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.9])
def test_fine_list_equals_mask_formulation(oracle_mod, sparsity):
    """The block-list formulation and the dense L x L masked formulation of
    the same selection agree (the pages' "masked reference")."""
    w, x = _tiny_case(sparsity)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, sparsity)
    om = oracle_mod.fine_masked(x["q"], x["k"], x["v"], r.geo, r.idx, r.topk, r.scale)
    assert np.abs(om - r.o_f).max() < 1e-12


# ---------------------------------------------------------------------------
# O6 compression, O7 output
# ---------------------------------------------------------------------------


def test_compress_invariants(oracle_mod):
    rng = np.random.default_rng(4)
    pv = rng.standard_normal((1, 2, 5, 16)).astype(np.float32)
    # equal scores -> plain mean of the pooled values over all tiles
    S = np.full((1, 2, 5, 5), 0.375, np.float32)
    oc = oracle_mod.compress(S, pv)
    assert np.abs(oc - pv.astype(np.float64).mean(axis=2, keepdims=True)).max() < 1e-14
    # one dominant score -> that tile's pooled value
    S = np.zeros((1, 2, 5, 5), np.float32)
    S[..., 3] = 200.0
    oc = oracle_mod.compress(S, pv)
    assert np.abs(oc - pv[:, :, 3:4, :].astype(np.float64)).max() < 1e-12
    # a single tile -> its own pooled value
    oc = oracle_mod.compress(np.zeros((1, 2, 1, 1), np.float32), pv[:, :, :1])
    assert (oc == pv[:, :, :1].astype(np.float64)).all()
    # weights are a softmax: known two-tile closed form
    S2 = np.array([[[[0.0, math.log(3.0)]] * 2]], np.float32)
    pv2 = np.array([[[[1.0], [5.0]]]], np.float32)
    oc = oracle_mod.compress(S2, pv2)
    assert abs(oc[0, 0, 0, 0] - (0.25 * 1 + 0.75 * 5)) < 1e-6


def test_output_gate(oracle_mod):
    w, x = _tiny_case(0.5)
    zero = bf16_bits(torch.zeros(1, w.seq_len, w.heads))
    r0 = oracle_mod.forward(x["q"], x["k"], x["v"], zero, w.segments, w.grid, 0.5)
    assert (r0.out == r0.o_f).all()
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.5)
    g = bits_to_f64(x["gate"])
    geo = r.geo
    for i in range(geo.n_tiles):
        toks = geo.tile_token[i, :geo.tile_valid[i]]
        for h in range(w.heads):
            expect = r.o_f[0, toks, h] + g[0, toks, h][:, None] * r.o_c[0, h, i][None, :]
            assert np.abs(r.out[0, toks, h] - expect).max() < 1e-15


def test_output_gate_per_channel(oracle_mod):
    """Reading R12, the per-channel gate [B, L, H*D]: channel h*D + d of a token scales column d of
    head h's compression row.  Pins: a gate equal across the D channels of each (token, head)
    gives exactly the scalar-gate output; a one-hot gate (1 at one channel of every token, 0
    elsewhere) changes only that head and column, by the compression value; a zero gate gives
    o_f."""
    w, x = _tiny_case(0.5)
    B, L, H, D = 1, w.seq_len, w.heads, w.head_dim
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.5)
    wide = np.repeat(x["gate"][..., None], D, axis=-1).reshape(B, L, H * D)
    rw = oracle_mod.forward(x["q"], x["k"], x["v"], wide, w.segments, w.grid, 0.5)
    assert np.array_equal(rw.out, r.out)
    h1, d1 = 1, 37
    onehot = np.zeros((B, L, H * D), np.uint16)
    onehot[:, :, h1 * D + d1] = bf16_bits(torch.ones(1))[0]
    ro = oracle_mod.forward(x["q"], x["k"], x["v"], onehot, w.segments, w.grid, 0.5)
    diff = ro.out - ro.o_f
    mask = np.zeros_like(diff, bool)
    mask[:, :, h1, d1] = True
    assert (diff[~mask] == 0).all()
    geo = ro.geo
    for i in range(geo.n_tiles):
        toks = geo.tile_token[i, :geo.tile_valid[i]]
        assert np.abs(diff[0, toks, h1, d1] - ro.o_c[0, h1, i, d1]).max() < 1e-14  # (a + b) - a rounds
    rz = oracle_mod.forward(x["q"], x["k"], x["v"], np.zeros((B, L, H * D), np.uint16), w.segments, w.grid, 0.5)
    assert (rz.out == rz.o_f).all()


def test_scores_fused_chain_in_d_order(oracle_mod):
    """Reading R6 fixes the score arithmetic: one fused multiply-add per d,
    d ascending, from +0.  Two hand-worked cases pin it:
      [-1, 1+2^-12] . [1, 1+2^-12]: -1, then fma gives 2^-11 + 2^-24 exactly
        (an unfused multiply would round a*a first and give 2^-11);
      [2^-30, 1, -1] . [1, 1, 1]: 2^-30, then 1 + 2^-30 rounds to 1, then 0
        (the reverse order would give 2^-30)."""
    a = np.float32(1 + 2.0 ** -12)
    pq = np.zeros((1, 1, 2, 4), np.float32)
    pk = np.zeros((1, 1, 2, 4), np.float32)
    pq[0, 0, 0, :2] = [-1.0, a]
    pk[0, 0, 0, :2] = [1.0, a]
    pq[0, 0, 1, :3] = [2.0 ** -30, 1.0, -1.0]
    pk[0, 0, 1, :3] = [1.0, 1.0, 1.0]
    S = oracle_mod.scores(pq, pk, 1.0)
    assert S[0, 0, 0, 0] == np.float32(2.0 ** -11 + 2.0 ** -24)
    assert S[0, 0, 1, 1] == 0.0


def test_pool_adds_rows_in_tile_order(oracle_mod):
    """Reading R6 for pooling: rows are added in tile order from +0.  Rows
    (2^-30, 1, -1) give ((0 + 2^-30) + 1) - 1 = 0 in binary32; any other
    order that adds 2^-30 last would give 2^-30 / 3."""
    segments, grid = (3,), (0, 0, 0)
    geo = oracle_mod.geometry(segments, grid)
    x = np.zeros((1, 3, 1, 8), np.float32)
    x[0, :, 0, 0] = [2.0 ** -30, 1.0, -1.0]
    x[0, :, 0, 1] = [1.0, -1.0, 2.0 ** -30]
    p = oracle_mod.pool(bf16_bits(torch.from_numpy(x)), geo)
    assert p[0, 0, 0, 0] == 0.0
    assert p[0, 0, 0, 1] == np.float32(2.0 ** -30) / np.float32(3.0)
