"""Reference keep on the GPU against the oracle (reading R18): reference prefix segments whose tiles each
video query tile keeps only kr of, chosen by pooled score.

Bar, as for the plain method: pooled tiles, scores and the selection (kept reference tiles, then video
tiles, in one idx row) bit-exact; compression within 1e-5 relative; the output within max-abs 2e-2 and
mean-abs 2e-3 of the float64 oracle.  Small shapes are compared in full for 64- and 128-token tiles,
several keep ratios, an all-reference prefix and 8-bit Q/K; the OmniRef-shaped 1344x768 workload on the
whole selection and sampled query tiles."""
import dataclasses

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module")
def vsa():
    from block_sparse_tiled_b200 import build

    build.build()
    import block_sparse_tiled_b200 as m

    m.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    return m


def plan_for(vsa, w, qk_fp8=False):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel,
                              tile_size=w.tile, cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep,
                              qk_fp8=qk_fp8)


def compare_out(got, ref):
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def full_parity(vsa, oracle_mod, w, seed=0, qk_fp8=False):
    x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, tile=w.tile,
                             cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep, qk8=qk_fp8)
    plan = plan_for(vsa, w, qk_fp8)
    kr = plan.dims["ref_topk"]
    assert kr == (oracle_mod.ref_count(w.ref_keep, ref.geo.n_ref) if ref.geo.n_video else 0)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    for n in ("pq", "pk", "pv"):
        assert np.array_equal(views[n].cpu().numpy(), getattr(ref, n)), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    g = views["o_c"].cpu().numpy().astype(np.float64)
    assert np.abs(g - ref.o_c).max() <= 1e-5 * max(1.0, np.abs(ref.o_c).max())
    compare_out(out.float().cpu().numpy().astype(np.float64), ref.out)
    plan.destroy()
    return ref


BASE = synth.Workload("ref", 1, 4, 128, (40, 200, 24), (8, 8, 16), 0.5, ref_segments=(False, True, False),
                      ref_keep=0.1)


@pytest.mark.parametrize("over", [
    dict(),                                          # keep 0.1: one of 4 reference tiles
    dict(ref_keep=0.5),
    dict(ref_keep=1.0),                              # every reference tile: the plain key set
    dict(segments=(300,), ref_segments=(True,)),     # the whole prefix is reference: no always-kept tile
    dict(segments=(70, 130, 5, 64), ref_segments=(True, False, True, False), ref_keep=0.3, head_dim=96),
    dict(tile=128, segments=(40, 520, 24), ref_keep=0.25),   # 128-token tiles
    dict(tile=128, segments=(200, 300), ref_segments=(True, True), grid=(5, 6, 7), batch=2, heads=3),
])
def test_ref_full_parity(vsa, oracle_mod, over):
    w = dataclasses.replace(BASE, **over)
    full_parity(vsa, oracle_mod, w, seed=3)


def test_ref_fp8(vsa, oracle_mod):
    full_parity(vsa, oracle_mod, dataclasses.replace(BASE, ref_keep=0.5), seed=5, qk_fp8=True)


def test_omniref_768p_sampled(vsa, oracle_mod):
    """The OmniRef-shaped workload: 1344x768 video in 128-token tiles, text 512 + 6144 reference tokens
    (48 reference tiles, keep 0.1 -> 5) + audio 768, sparsity 0.9."""
    w = synth.workload("omniref_768p")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan = plan_for(vsa, w)
    assert (plan.dims["n_ref_tiles"], plan.dims["ref_topk"]) == (48, 5)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity, tile=128,
                               ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    geo = sel["geo"]
    assert np.array_equal(views["scores"].cpu().numpy(), sel["S"])
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    tiles = sorted({0, 5, 53, geo.n_prefix, geo.n_tiles - 1, *range(geo.n_prefix, geo.n_tiles, 113)})
    items = np.array([h * geo.n_tiles + i for h in (0, 55) for i in tiles], np.int64)
    of = oracle_mod.fine_tiles(xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items)
    ref = oracle_mod.output_tiles(of, sel["o_c"], xb["gate"], geo, items, w.heads)
    got = np.zeros_like(ref)
    for n, bhi in enumerate(items):
        i, h = int(bhi % geo.n_tiles), int(bhi // geo.n_tiles)
        nv = int(geo.tile_valid[i])
        rows = torch.from_numpy(geo.tile_token[i, :nv].astype(np.int64)).cuda()
        got[n, :nv] = out[0][rows, h].double().cpu().numpy()
    compare_out(got, ref)
    plan.destroy()
