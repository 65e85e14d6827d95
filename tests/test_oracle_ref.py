"""Pins for the oracle's reference keep (reading R18): reference prefix segments whose tiles each video
query tile keeps only kr of, chosen by pooled score like the video tiles.

What pins it, independently of the oracle's code: the kr formula worked by hand; no reference segment
reduces to the plain method exactly; keep = 1 keeps every reference tile, which is the plain method's
key set; the kept reference tiles are the best subset by brute force; every video row equals torch
SDPA over the always-kept prefix, kept reference and selected video tokens; prefix rows stay dense;
and the list and mask formulations agree."""
import itertools

import numpy as np
import pytest
import torch

import synth

SEGMENTS, FLAGS, GRID = (40, 200, 24), (False, True, False), (8, 8, 8)


def bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dense_sdpa(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
        scale=scale)
    return out[0, 0].numpy()


def inputs(seed=1, heads=2, D=64):
    w = synth.Workload("ref", 1, heads, D, SEGMENTS, GRID, 0.5)
    x = synth.make_inputs(w, seed=seed)
    return w, {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}


@pytest.mark.parametrize("keep,R,kr", [(0.1, 10, 1), (0.1, 24, 3), (0.1, 0, 0), (1.0, 7, 7), (1e-9, 5, 1),
                                       (0.5, 7, 4), (0.7, 10, 7), (0.35, 21, 8)])
def test_ref_count_table(oracle_mod, keep, R, kr):
    """max(1, min(ceil(keep * R), R)) in binary64, worked by hand (0.35 * 21 = 7.35 -> 8)."""
    assert oracle_mod.ref_count(keep, R) == kr


def test_ref_geometry_flags(oracle_mod):
    geo = oracle_mod.geometry(SEGMENTS, GRID, ref_segments=FLAGS)
    assert list(geo.is_ref) == [0, 1, 1, 1, 1, 0] and geo.n_ref == 4 and geo.n_prefix == 6
    geo128 = oracle_mod.geometry(SEGMENTS, GRID, tile=128, ref_segments=FLAGS)
    assert list(geo128.is_ref) == [0, 1, 1, 0]


def test_no_reference_is_the_plain_method(oracle_mod):
    w, x = inputs()
    plain = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], SEGMENTS, GRID, 0.5)
    none = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], SEGMENTS, GRID, 0.5, ref_segments=(0, 0, 0),
                              ref_keep=0.1)
    assert np.array_equal(plain.idx, none.idx)
    assert np.array_equal(plain.o_f, none.o_f) and np.array_equal(plain.out, none.out)


def test_keep_one_keeps_every_reference_tile(oracle_mod):
    w, x = inputs()
    plain = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], SEGMENTS, GRID, 0.5)
    full = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], SEGMENTS, GRID, 0.5, ref_segments=FLAGS,
                              ref_keep=1.0)
    assert (full.idx[..., :4] == np.array([1, 2, 3, 4])).all()
    assert np.array_equal(full.idx[..., 4:], plain.idx)
    assert np.abs(full.o_f - plain.o_f).max() < 1e-12  # same key set, another summation order


@pytest.mark.parametrize("keep", [0.1, 0.5])
def test_reference_selection_brute_force_and_sdpa(oracle_mod, keep):
    w, x = inputs(seed=4)
    sel = oracle_mod.selection(x["q"], x["k"], x["v"], SEGMENTS, GRID, 0.5, ref_segments=FLAGS, ref_keep=keep)
    geo, kr, k = sel["geo"], sel["kr"], sel["topk"]
    assert kr == oracle_mod.ref_count(keep, 4) and sel["idx"].shape[-1] == kr + k
    r = oracle_mod.forward(x["q"], x["k"], x["v"], x["gate"], SEGMENTS, GRID, 0.5, ref_segments=FLAGS, ref_keep=keep)
    assert np.array_equal(r.idx, sel["idx"])
    q, kk, v = (bits_to_f64(x[n]) for n in ("q", "k", "v"))
    refs = [1, 2, 3, 4]
    for h in range(w.heads):
        for iv in range(geo.n_video):
            i = geo.n_prefix + iv
            s = sel["S"][0, h, i]
            best = max(itertools.combinations(refs, kr), key=lambda c: sum(s[list(c)]))
            assert list(sel["idx"][0, h, iv, :kr]) == sorted(best)
            tiles = [0, 5] + list(sel["idx"][0, h, iv])
            keys = np.concatenate([geo.tile_token[t, :geo.tile_valid[t]] for t in tiles])
            qs = geo.tile_token[i, :geo.tile_valid[i]]
            ref = dense_sdpa(q[0, qs, h], kk[0, keys, h], v[0, keys, h], sel["scale"])
            assert np.abs(r.o_f[0, qs, h] - ref).max() < 1e-12
        npre = sum(SEGMENTS)
        dense = dense_sdpa(q[0, :npre, h], kk[0, :, h], v[0, :, h], sel["scale"])
        assert np.abs(r.o_f[0, :npre, h] - dense).max() < 1e-12
    om = oracle_mod.fine_masked(x["q"], x["k"], x["v"], geo, r.idx, r.topk, r.scale)
    assert np.abs(om - r.o_f).max() < 1e-12
