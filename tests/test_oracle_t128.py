"""Pins for the oracle with 128-token tiles (reading R17: prefix runs of up to 128
tokens, ct x ch x cw video cubes with ct*ch*cw = 128, 4 x 4 x 8 by default).

What pins it, independently of the oracle's code: tile counts worked by hand;
the partition invariants; a 4x4x8 cube is exactly the union of two w-adjacent
4x4x4 cubes of the 64-token geometry; pooling of constant and one-token tiles;
and the fine branch against torch SDPA (sparsity 0, prefix rows, every video
row over its prefix + selected tokens), the mask formulation, and a
brute-force top-k on a tiny case."""
import itertools

import numpy as np
import pytest
import torch

import synth


def bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dense_sdpa(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
        scale=scale)
    return out[0, 0].numpy()


# (segments, grid, cube) -> (n_tiles, n_prefix, n_video), by hand
COUNTS = [
    ((512, 0, 768), (24, 48, 64), (4, 4, 8), (586, 10, 576)),    # 4 + 0 + 6 prefix; 6 * 12 * 8 cubes
    ((384, 0, 384), (8, 30, 56), (4, 4, 8), (118, 6, 112)),      # 2 * ceil(30/4)=8 * 7
    ((384, 0, 384), (8, 30, 56), (8, 4, 4), (118, 6, 112)),      # 1 * 8 * 14
    ((40, 0, 24), (8, 8, 8), (4, 4, 8), (6, 2, 4)),
    ((129,), (5, 6, 9), (4, 4, 8), (2 + 2 * 2 * 2, 2, 8)),       # 129 = 128 + 1; ceil(9/8) = 2
    ((), (4, 4, 8), (4, 4, 8), (1, 0, 1)),
]


@pytest.mark.parametrize("segments,grid,cube,expect", COUNTS)
def test_t128_counts(oracle_mod, segments, grid, cube, expect):
    geo = oracle_mod.geometry(segments, grid, tile=128, cube=cube)
    assert (geo.n_tiles, geo.n_prefix, geo.n_video) == expect
    assert geo.tile_token.shape == (expect[0], 128)


@pytest.mark.parametrize("segments,grid,cube,expect", COUNTS)
def test_t128_partition(oracle_mod, segments, grid, cube, expect):
    geo = oracle_mod.geometry(segments, grid, tile=128, cube=cube)
    L = sum(segments) + int(np.prod(grid))
    tok = geo.tile_token
    valid = tok >= 0
    # valid rows first, counted by tile_valid; every token exactly once
    assert (valid.sum(1) == geo.tile_valid).all()
    assert all(valid[i, :geo.tile_valid[i]].all() for i in range(geo.n_tiles))
    assert np.array_equal(np.sort(tok[valid]), np.arange(L))
    # prefix tiles are segment-pure runs of up to 128 in order
    off, i = 0, 0
    for n in segments:
        for first in range(0, n, 128):
            cnt = min(128, n - first)
            assert list(tok[i, :cnt]) == list(range(off + first, off + first + cnt))
            i += 1
        off += n
    # each video tile is one ct x ch x cw block of the grid in raster (t, h, w) order
    T, Hg, W = grid
    ct, ch, cw = cube
    P = sum(segments)
    for i in range(geo.n_prefix, geo.n_tiles):
        v = tok[i, :geo.tile_valid[i]] - P
        t, h, w = v // (Hg * W), (v // W) % Hg, v % W
        assert len(set(t // ct)) == len(set(h // ch)) == len(set(w // cw)) == 1
        assert list(v) == sorted(v)


def test_t128_cube_is_two_w_adjacent_64_cubes(oracle_mod):
    segments, grid = (), (8, 12, 16)
    g128 = oracle_mod.geometry(segments, grid, tile=128, cube=(4, 4, 8))
    g64 = oracle_mod.geometry(segments, grid)
    # 64-token cubes in raster (a, b, c) order: c runs over 16/4 = 4 w-blocks, the 128 cubes over 2
    for i in range(g128.n_tiles):
        a_b, c = divmod(i, 2)
        pair = [a_b * 4 + 2 * c, a_b * 4 + 2 * c + 1]
        assert set(g128.tile_token[i]) == set(g64.tile_token[pair].ravel())


def test_t128_pool_special_cases(oracle_mod):
    segments, grid = (1, 128), (4, 4, 8)
    geo = oracle_mod.geometry(segments, grid, tile=128)
    L = 1 + 128 + 128
    x = np.zeros((1, L, 1, 8), np.float32)
    x[0, 0] = 3.25            # the one-token prefix tile pools to itself
    x[0, 1:129] = -1.5        # a full constant prefix tile
    x[0, 129:] = np.arange(128, dtype=np.float32)[:, None, None] / 64.0  # 0 .. 127/64, exact mean 127/128
    xb = synth.as_bits(torch.from_numpy(x).to(torch.bfloat16))
    p = oracle_mod.pool(xb, geo)
    assert (p[0, 0, 0] == 3.25).all() and (p[0, 0, 1] == -1.5).all()
    assert (p[0, 0, 2] == np.float32(127.0 / 128.0)).all()


def _case(sparsity, seed=2):
    w = synth.Workload("tiny128", 1, 2, 64, (40, 0, 24), (8, 8, 8), sparsity)
    x = synth.make_inputs(w, seed=seed)
    return w, {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}


def test_t128_sparsity0_is_dense(oracle_mod):
    w, x = _case(0.0)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.0, tile=128)
    assert r.topk == r.geo.n_video == 4
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    for h in range(w.heads):
        ref = dense_sdpa(q[0, :, h], k[0, :, h], v[0, :, h], r.scale)
        assert np.abs(r.o_f[0, :, h] - ref).max() < 1e-12


@pytest.mark.parametrize("sparsity", [0.5, 0.75])
def test_t128_rows_attend_prefix_and_selected(oracle_mod, sparsity):
    w, x = _case(sparsity)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, sparsity, tile=128)
    q, k, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    geo = r.geo
    npre = sum(w.segments)
    for h in range(w.heads):
        ref = dense_sdpa(q[0, :npre, h], k[0, :, h], v[0, :, h], r.scale)
        assert np.abs(r.o_f[0, :npre, h] - ref).max() < 1e-12
        for iv in range(geo.n_video):
            i = geo.n_prefix + iv
            tiles = list(range(geo.n_prefix)) + list(r.idx[0, h, iv])
            keys = np.concatenate([geo.tile_token[t, :geo.tile_valid[t]] for t in tiles])
            qs = geo.tile_token[i, :geo.tile_valid[i]]
            ref = dense_sdpa(q[0, qs, h], k[0, keys, h], v[0, keys, h], r.scale)
            assert np.abs(r.o_f[0, qs, h] - ref).max() < 1e-12
    om = oracle_mod.fine_masked(x["q"], x["k"], x["v"], geo, r.idx, r.topk, r.scale)
    assert np.abs(om - r.o_f).max() < 1e-12


def test_t128_select_brute_force(oracle_mod):
    """Every C(4, 2) subset of video key tiles by its summed score: the pick is the unique best subset
    (the scores of a tiny random case have no ties)."""
    w, x = _case(0.5, seed=5)
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], w.segments, w.grid, 0.5, tile=128)
    P, V = r.geo.n_prefix, r.geo.n_video
    for h in range(w.heads):
        for iv in range(V):
            s = r.S[0, h, P + iv, P:]
            best = max(itertools.combinations(range(V), r.topk), key=lambda c: sum(s[list(c)]))
            assert list(r.idx[0, h, iv]) == [P + j for j in sorted(best)]
