"""The C ABI without a GPU: the library loads, exports every symbol the
header declares, and its host-side plan (tile geometry, token tables, topk,
argument checks) agrees with the oracle's independent tiling."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def vsa():
    from block_sparse_tiled_b200 import build

    build.build()
    import block_sparse_tiled_b200 as m

    m.load_library()
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "vsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(vsa_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(vsa):
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(vsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(vsa.EXPORTED)
    dyn = subprocess.run(["nm", "-D", "--defined-only", vsa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (vsa_\w+)", dyn))
    assert set(names) <= exported
    assert vsa.load_library().vsa_version().decode().startswith("vsa-b200")


def _kw(w, **over):
    kw = dict(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
              sparsity=w.sparsity, tile_size=w.tile, cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    kw.update(over)
    return kw


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_plan_matches_oracle_geometry(vsa, oracle_mod, name):
    w = synth.workload(name)
    d = vsa.vsa_plan_query(**_kw(w))
    geo = oracle_mod.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments)
    assert (d["n_tiles"], d["n_prefix_tiles"], d["n_video_tiles"]) == (geo.n_tiles, geo.n_prefix, geo.n_video)
    assert d["topk"] == oracle_mod.topk_count(w.sparsity, geo.n_video)
    assert d["seq_len"] == w.seq_len
    assert d["softmax_scale"] == np.float32(oracle_mod.default_scale(w.head_dim))
    P, V, k, n = geo.n_prefix, geo.n_video, d["topk"], geo.n_tiles
    R = geo.n_ref
    kr = oracle_mod.ref_count(w.ref_keep, R) if R else 0
    assert (d["n_ref_tiles"], d["ref_topk"]) == (R, kr)
    assert d["selected_pairs"] == V * (P - R + kr + k) + P * n
    if name in ("tiny", "small", "480p"):
        tok, val = vsa.vsa_plan_tables_host(**_kw(w))
        assert np.array_equal(tok, geo.tile_token)
        assert np.array_equal(val, geo.tile_valid)


@pytest.mark.parametrize("segments,grid", [
    ((), (4, 4, 4)), ((1,), (1, 1, 1)), ((0, 0, 130), (3, 5, 7)), ((64, 64), (0, 0, 0)),
    ((17,), (9, 2, 13)), ((0,), (4, 8, 4)),
])
def test_plan_edge_geometries(vsa, oracle_mod, segments, grid):
    kw = dict(batch=2, heads=3, head_dim=64, segments=segments, grid=grid, sparsity=0.7)
    d = vsa.vsa_plan_query(**kw)
    geo = oracle_mod.geometry(segments, grid)
    assert (d["n_tiles"], d["n_prefix_tiles"], d["n_video_tiles"]) == (geo.n_tiles, geo.n_prefix, geo.n_video)
    tok, val = vsa.vsa_plan_tables_host(**kw)
    assert np.array_equal(tok, geo.tile_token) and np.array_equal(val, geo.tile_valid)


@pytest.mark.parametrize("s", [0.0, 0.5, 0.8, 0.9, 0.95, 1.0])
def test_plan_topk_sweep(vsa, oracle_mod, s):
    w = synth.workload("768p_s0.9")
    assert vsa.vsa_plan_query(**_kw(w, sparsity=s))["topk"] == oracle_mod.topk_count(s, 1152)


def test_token_tags_match_segments(vsa):
    # text 40, cond 0 (absent), audio 24, then 8x8x8 video tagged 9
    tags = [1] * 40 + [3] * 24 + [9] * 512
    a = vsa.vsa_plan_query(batch=1, heads=2, head_dim=64, token_tags=tags, video_tag=9, grid=(8, 8, 8), sparsity=0.5)
    b = vsa.vsa_plan_query(batch=1, heads=2, head_dim=64, segments=(40, 24), grid=(8, 8, 8), sparsity=0.5)
    assert a == b
    # interleaved runs of one tag are separate segments
    tags2 = [1] * 10 + [2] * 10 + [1] * 10 + [9] * 64
    t2, _ = vsa.vsa_plan_tables_host(batch=1, heads=1, head_dim=64, token_tags=tags2, video_tag=9, grid=(4, 4, 4))
    assert t2.shape[0] == 4


@pytest.mark.parametrize("over,status", [
    (dict(sparsity=1.5), "VSA_ERR_INVALID_ARG"),
    (dict(sparsity=-0.1), "VSA_ERR_INVALID_ARG"),
    (dict(sparsity=float("nan")), "VSA_ERR_INVALID_ARG"),
    (dict(tile_size=32), "VSA_ERR_UNSUPPORTED"),
    (dict(tile_size=128, cube=(4, 4, 4)), "VSA_ERR_INVALID_ARG"),
    (dict(tile_size=128, seq_tiles=True), "VSA_ERR_UNSUPPORTED"),
    (dict(head_dim=80), "VSA_ERR_UNSUPPORTED"),
    (dict(grid=(8, 0, 8)), "VSA_ERR_SHAPE"),
    (dict(batch=0), "VSA_ERR_INVALID_ARG"),
    (dict(segments=(-1,)), "VSA_ERR_INVALID_ARG"),
])
def test_plan_rejects_bad_arguments(vsa, over, status):
    w = synth.workload("tiny")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(**_kw(w, **over))
    assert vsa.STATUS_NAMES[e.value.status] == status
    assert vsa.load_library().vsa_last_error().decode() != ""


def test_token_tags_video_not_last(vsa):
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(batch=1, heads=1, head_dim=64, token_tags=[9] * 64 + [1] * 3, video_tag=9,
                           grid=(4, 4, 4))
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_SHAPE"


def test_workspace_size(vsa):
    w = synth.workload("768p_s0.9")
    d = vsa.vsa_plan_query(**_kw(w))
    n_t, D, H = 1172, 128, 56
    tiles = H * n_t * 64 * D * 2
    assert d["workspace_bytes"] >= 3 * tiles + 4 * H * n_t * D * 4 + H * n_t * n_t * 4 + H * 1152 * 116 * 4
    assert d["workspace_bytes"] < 3 * tiles * 1.2


def test_seq_tiles_workspace_and_limits(vsa):
    """seq_tiles drops the three tile-order copies from the workspace and needs batch <= 4."""
    kw = dict(batch=1, heads=56, head_dim=128, segments=(512, 0, 768), grid=(24, 48, 64), sparsity=0.9)
    a = vsa.vsa_plan_query(**kw)["workspace_bytes"]
    b = vsa.vsa_plan_query(seq_tiles=True, **kw)["workspace_bytes"]
    tiles = 3 * 56 * 1172 * 64 * 128 * 2
    assert a - b == tiles
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(batch=5, heads=2, head_dim=64, segments=(64,), grid=(4, 4, 4), seq_tiles=True)
    assert e.value.status == 3  # VSA_ERR_UNSUPPORTED


def test_qk_fp8_workspace_and_limits(vsa):
    """8-bit Q/K: q_t/k_t hold one 128-byte code row per tile row (instead of D bf16 values) plus one float32
    scale per row each; it needs tile-order copies (no seq_tiles)."""
    kw = dict(batch=1, heads=56, head_dim=128, segments=(512, 0, 768), grid=(24, 48, 64), sparsity=0.9)
    a = vsa.vsa_plan_query(**kw)["workspace_bytes"]
    b = vsa.vsa_plan_query(qk_fp8=True, **kw)["workspace_bytes"]
    rows = 56 * 1172 * 64
    assert a - b == 2 * rows * 128 * 2 - (2 * rows * 128 + 2 * rows * 4)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(qk_fp8=True, seq_tiles=True, **kw)
    assert e.value.status == 3  # VSA_ERR_UNSUPPORTED
    g, keep = vsa.make_geometry(**kw)
    g.qk_fp8 = 4
    import ctypes

    d = vsa.PlanDims()
    assert vsa.load_library().vsa_plan_query(ctypes.byref(g), ctypes.byref(d)) == 1  # VSA_ERR_INVALID_ARG


def test_qk_prefix_split_workspace(vsa):
    """The prefix split (qk_fp8 = 2) keeps the bf16 copies and adds 8-bit code rows of Q and K (128 bytes
    per tile row each), their scales and the dequantised rows' norms and (b, h) maxima."""
    kw = dict(batch=1, heads=56, head_dim=128, segments=(512, 0, 768), grid=(24, 48, 64), sparsity=0.9)
    a = vsa.vsa_plan_query(**kw)["workspace_bytes"]
    c = vsa.vsa_plan_query(qk_fp8="prefix", **kw)["workspace_bytes"]
    rows = 56 * 1172 * 64
    assert c - a == 2 * rows * 128 + 2 * rows * 4 + rows * 4 + 512  # codes, scales, norms, maxima (aligned)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(qk_fp8="prefix", seq_tiles=True, **kw)
    assert e.value.status == 3  # VSA_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        vsa.make_geometry(qk_fp8="video", **kw)


def test_qk_fp4_workspace(vsa):
    """FP4 video query tiles (qk_fp8 = 3): the prefix split's workspace plus the binary64 key column sums
    and the binary32 key means, one per (b, h, d); it needs tile-order copies too."""
    kw = dict(batch=1, heads=56, head_dim=128, segments=(512, 0, 768), grid=(24, 48, 64), sparsity=0.9)
    c = vsa.vsa_plan_query(qk_fp8="prefix", **kw)["workspace_bytes"]
    f = vsa.vsa_plan_query(qk_fp8="fp4", **kw)["workspace_bytes"]
    assert f - c == 56 * 128 * 8 + 56 * 128 * 4
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_plan_query(qk_fp8="fp4", seq_tiles=True, **kw)
    assert e.value.status == 3  # VSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("segments,grid,cube", [
    ((512, 0, 768), (24, 48, 64), None),
    ((384, 0, 384), (8, 30, 56), (8, 4, 4)),
    ((40, 0, 24), (8, 8, 8), None),
    ((129, 3), (5, 6, 9), (2, 8, 8)),
])
def test_plan_tile128_matches_oracle_geometry(vsa, oracle_mod, segments, grid, cube):
    """128-token tiles: the host token table equals the oracle's, and the workspace holds 128-row tiles."""
    kw = dict(batch=1, heads=2, head_dim=128, segments=segments, grid=grid, sparsity=0.9, tile_size=128, cube=cube)
    d = vsa.vsa_plan_query(**kw)
    geo = oracle_mod.geometry(segments, grid, tile=128, cube=cube)
    assert (d["n_tiles"], d["n_prefix_tiles"], d["n_video_tiles"], d["tile_size"]) == (
        geo.n_tiles, geo.n_prefix, geo.n_video, 128)
    assert d["topk"] == oracle_mod.topk_count(0.9, geo.n_video)
    tok, val = vsa.vsa_plan_tables_host(**kw)
    assert np.array_equal(tok, geo.tile_token) and np.array_equal(val, geo.tile_valid)
    d64 = vsa.vsa_plan_query(**dict(kw, tile_size=64, cube=None))
    assert d["workspace_bytes"] > 0 and d64["n_tiles"] >= d["n_tiles"]


def test_reference_keep_plan_and_limits(vsa, oracle_mod):
    """Reference segments: counts as the oracle's, an idx row of kr + topk entries, and the argument checks."""
    kw = dict(batch=1, heads=4, head_dim=128, segments=(40, 200, 24), grid=(8, 8, 8), sparsity=0.5,
              ref_segments=(0, 1, 0), ref_keep=0.5)
    d = vsa.vsa_plan_query(**kw)
    geo = oracle_mod.geometry(kw["segments"], kw["grid"], ref_segments=kw["ref_segments"])
    assert (d["n_ref_tiles"], d["ref_topk"], d["topk"]) == (4, 2, 4)
    assert d["selected_pairs"] == geo.n_video * (6 - 4 + 2 + 4) + 6 * geo.n_tiles
    plain = vsa.vsa_plan_query(**dict(kw, ref_segments=None))
    assert d["workspace_bytes"] - plain["workspace_bytes"] >= 0  # idx rows grow by kr entries
    for bad in (dict(ref_keep=0.0), dict(ref_keep=1.5), dict(ref_segments=(0, 2, 0))):
        with pytest.raises(vsa.VsaError) as e:
            vsa.vsa_plan_query(**dict(kw, **bad))
        assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_INVALID_ARG"
    # no video tiles: no reference selection either
    d0 = vsa.vsa_plan_query(**dict(kw, grid=(0, 0, 0)))
    assert d0["ref_topk"] == 0 and d0["n_ref_tiles"] == 4
