"""128-token tiles (tile_size = 128) on the GPU against the oracle with the same tiling.

The library runs each 128-token query tile as two 64-row blocks that share the tile's key list, and
walks each listed 128-token key tile as one 128-key block.  Bar, as for 64-token tiles: tile-order
copies (128 rows per tile), pooled tiles, scores and the selection bit-exact; compression within
1e-5 relative; the output within max-abs 2e-2 and mean-abs 2e-3 of the float64 oracle.  Small
workloads are compared in full (through vsa_forward and through the step entry points), the
1344x768 workload on the whole selection and sampled query tiles."""
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


def plan_for(vsa, w, heads=None, qk_fp8=False):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=heads or w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel,
                              tile_size=w.tile, cube=w.cube, qk_fp8=qk_fp8)


def t128(name, **over):
    return dataclasses.replace(synth.workload(name), tile=128, name=f"{name}_t128", **over)


def expected_tiles(xbits, geo):
    B, L, H, D = xbits.shape
    tok = geo.tile_token
    res = np.zeros((B, H, geo.n_tiles, geo.tile, D), np.uint16)
    valid = tok >= 0
    for b in range(B):
        res[b][:, valid] = xbits[b].transpose(1, 0, 2)[:, tok[valid]]
    return res


def compare_out(got, ref):
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def full_parity(vsa, oracle_mod, w, seed=0, stepwise=True):
    x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, tile=w.tile,
                             cube=w.cube)
    plan = plan_for(vsa, w)
    assert plan.dims["tile_size"] == w.tile and plan.dims["n_tiles"] == ref.geo.n_tiles
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    for n in ("q", "k", "v"):
        assert np.array_equal(synth.as_bits(views[n + "_t"]), expected_tiles(xb[n], ref.geo)), n
    for n in ("pq", "pk", "pv"):
        assert np.array_equal(views[n].cpu().numpy(), getattr(ref, n)), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    g = views["o_c"].cpu().numpy().astype(np.float64)
    assert np.abs(g - ref.o_c).max() <= 1e-5 * max(1.0, np.abs(ref.o_c).max())
    compare_out(out.float().cpu().numpy().astype(np.float64), ref.out)
    if stepwise:
        B, H, D, n_t = w.batch, w.heads, w.head_dim, ref.geo.n_tiles
        V, k = ref.geo.n_video, ref.topk
        bf = dict(dtype=torch.bfloat16, device="cuda")
        f32 = dict(dtype=torch.float32, device="cuda")
        t = {n: torch.empty(B, H, n_t, 128, D, **bf) for n in ("q_t", "k_t", "v_t")}
        vsa.vsa_gather_tiles(plan, x["q"], x["k"], x["v"], t["q_t"], t["k_t"], t["v_t"])
        pq, pk, pv = (torch.empty(B, H, n_t, D, **f32) for _ in range(3))
        S = torch.empty(B, H, n_t, n_t, **f32)
        vsa.vsa_pool_and_score(plan, t["q_t"], t["k_t"], t["v_t"], pq, pk, pv, S)
        idx = torch.empty(B, H, max(V, 1), max(k, 1), dtype=torch.int32, device="cuda")
        o_c = torch.empty(B, H, n_t, D, **f32)
        vsa.vsa_topk_select(plan, S, pv, idx, o_c)
        out2 = torch.empty_like(x["q"])
        vsa.vsa_sparse_attn_fwd(plan, t["q_t"], t["k_t"], t["v_t"], idx, o_c, x["gate"], out2)
        torch.cuda.synchronize()
        assert np.array_equal(pq.cpu().numpy(), ref.pq) and np.array_equal(S.cpu().numpy(), ref.S)
        assert np.array_equal(idx[:, :, :V, :k].cpu().numpy(), ref.idx)
        assert torch.equal(out2, out)
    plan.destroy()
    return ref


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_t128_full_parity(vsa, oracle_mod, name):
    full_parity(vsa, oracle_mod, t128(name))


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D,cube", [
    ((), (8, 8, 16), 0.5, 1, 2, 64, None),              # no prefix
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128, None),       # prefix only: every query tile dense
    ((10,), (3, 2, 5), 0.5, 1, 3, 128, None),           # grid below one cube: one partial tile
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128, None),      # ragged everywhere, batch 2
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 96, None),       # head_dim 96
    ((129,), (4, 8, 8), 1.0, 1, 2, 128, None),          # topk = 1; a one-token prefix tile half
    ((200, 0, 60), (8, 8, 8), 0.5, 1, 2, 128, (8, 4, 4)),  # temporal cube
    ((40, 0, 24), (6, 12, 8), 0.5, 3, 2, 64, (2, 8, 8)),   # flat cube, batch 3
])
def test_t128_edge_cases(vsa, oracle_mod, segments, grid, sparsity, B, H, D, cube):
    w = synth.Workload("edge128", B, H, D, tuple(segments), tuple(grid), sparsity, tile=128, cube=cube)
    full_parity(vsa, oracle_mod, w, seed=3)


def test_t128_gate_per_channel(vsa, oracle_mod):
    full_parity(vsa, oracle_mod, t128("small", gate_per_channel=True), seed=7, stepwise=False)


def test_t128_768p_sampled(vsa, oracle_mod):
    """The 1344x768 workload with 128-token tiles (586 tiles, topk 58): selection in full, sampled output."""
    w = synth.workload("768p_t128_s0.9")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan = plan_for(vsa, w)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity, tile=128)
    geo = sel["geo"]
    assert (geo.n_tiles, sel["topk"]) == (586, 58)
    assert np.array_equal(views["pq"].cpu().numpy(), sel["pq"])
    assert np.array_equal(views["scores"].cpu().numpy(), sel["S"])
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    tiles = sorted({0, geo.n_prefix - 1, geo.n_prefix, geo.n_tiles - 1, *range(geo.n_prefix, geo.n_tiles, 97)})
    items = np.array([h * geo.n_tiles + i for h in (0, 29, 55) for i in tiles], np.int64)
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


def test_t128_fp8_parts_and_host_routes(vsa, oracle_mod):
    """128-token tiles with 8-bit Q/K against the oracle's 8-bit variant, and the sequence-part and
    host-pipeline routes bit-identical to the device forward."""
    w = t128("small")
    x = synth.make_inputs(w, seed=8, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, qk8=True,
                             tile=128)
    plan = plan_for(vsa, w, qk_fp8=True)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=vsa.alloc_workspace(plan))
    torch.cuda.synchronize()
    compare_out(out.float().cpu().numpy().astype(np.float64), ref.out)
    plan.destroy()
    plan = plan_for(vsa, w)
    dev = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=vsa.alloc_workspace(plan))
    torch.cuda.synchronize()
    hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "gate")}
    assert torch.equal(vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=3), dev.cpu())
    plan.destroy()
    world = 2
    parts = {n: [c.contiguous() for c in torch.chunk(x[n], world, dim=1)] for n in ("q", "k", "v", "gate")}
    outs = [torch.full_like(p, float("nan")) for p in parts["q"]]
    for rank in range(world):
        ls, hn, h0 = vsa.ulysses_partition(w.seq_len, w.heads, world, rank)
        p = plan_for(vsa, w, heads=hn)
        vsa.vsa_forward_parts(p, parts["q"], parts["k"], parts["v"], parts["gate"], outs, h0)
        torch.cuda.synchronize()
        p.destroy()
    assert torch.equal(torch.cat(outs, dim=1), dev)
