"""vsa_forward_parts: the forward over a sequence split by token into parts,
as a sequence-parallel (Ulysses) layout holds it.

On several GPUs each rank's parts are peer mappings and the gather kernel's
loads and the epilogue's stores carry the all-to-all exchanges.  Here every
part lives on one GPU: the ranks' forwards run one after another (no kernel
waits on another), each for its head group over all parts.  The assembled
output is checked against the CPU oracle (selection of each rank's heads bit
for bit, the output within max-abs 2e-2 and mean-abs 2e-3), and must also
equal vsa_forward on the whole tensors bit for bit (every head's computation
is the same; only where its rows are read from and written to differs) --
except on the prefix query rows of 64-token tiles when a rank has too few
heads for the pair kernel and the whole forward enough, where the two agree
within the output tolerance."""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from conftest import assert_routes_agree

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


def plan_for(vsa, w, heads=None, **kw):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=heads or w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, **kw)


def split(t, n):
    return [c.contiguous() for c in torch.chunk(t, n, dim=1)]


def run_ranks(vsa, w, x, world):
    """The emulated ranks' forwards; returns the assembled output and each rank's idx (its heads)."""
    L, H = w.seq_len, w.heads
    parts = {n: split(x[n], world) for n in ("q", "k", "v", "gate")}
    out_parts = [torch.full_like(p, float("nan")) for p in parts["q"]]
    idx = []
    for rank in range(world):
        ls, hn, h0 = vsa.ulysses_partition(L, H, world, rank)
        assert ls * world == L and parts["q"][0].shape[1] == ls
        plan = plan_for(vsa, w, heads=hn)
        ws = vsa.alloc_workspace(plan)
        vsa.vsa_forward_parts(plan, parts["q"], parts["k"], parts["v"], parts["gate"], out_parts, h0, workspace=ws)
        torch.cuda.synchronize()
        assert vsa.device_status(plan) == (0, 0)
        idx.append(vsa.workspace_views(plan, ws)["idx"].cpu().numpy())
        plan.destroy()
    return torch.cat(out_parts, dim=1), np.concatenate(idx, axis=1)


def reference(vsa, w, x):
    plan = plan_for(vsa, w)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=vsa.alloc_workspace(plan))
    torch.cuda.synchronize()
    plan.destroy()
    return out


@pytest.mark.parametrize("name,world,over", [
    ("small", 2, {}), ("small", 4, {}), ("small", 8, {}),
    ("small", 4, dict(head_dim=96, gate_per_channel=True)),
    ("tiny", 2, {}),
    ("480p", 4, {}), ("480p", 8, {}),
])
def test_parts_match_oracle_and_whole_forward(vsa, oracle_mod, name, world, over):
    w = dataclasses.replace(synth.workload(name), **over)
    x = synth.make_inputs(w, seed=21, device="cuda")
    got, idx = run_ranks(vsa, w, x, world)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity)
    geo = sel["geo"]
    assert np.array_equal(idx, sel["idx"])
    # the output against the oracle: every query tile at the small shapes, a sample of tiles of every
    # rank's heads at 480p
    if w.seq_len * w.heads <= 64 * 1024:
        tiles = list(range(geo.n_tiles))
    else:
        tiles = sorted({0, geo.n_prefix - 1, geo.n_tiles - 1, *range(geo.n_prefix, geo.n_tiles, 37)})
    heads = sorted({h for r in range(world) for h in (r * (w.heads // world), (r + 1) * (w.heads // world) - 1)})
    items = np.array([h * geo.n_tiles + i for h in heads for i in tiles], np.int64)
    of = oracle_mod.fine_tiles(xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items)
    ref = oracle_mod.output_tiles(of, sel["o_c"], xb["gate"], geo, items, w.heads)
    g = np.zeros_like(ref)
    for n, hi in enumerate(items):
        i, h = int(hi % geo.n_tiles), int(hi // geo.n_tiles)
        nv = int(geo.tile_valid[i])
        rows = torch.from_numpy(geo.tile_token[i, :nv].astype(np.int64)).cuda()
        g[n, :nv] = got[0][rows, h].double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    assert_routes_agree(w, got, reference(vsa, w, x), w.heads // world)


def test_parts_argument_errors(vsa):
    w = synth.workload("small")
    x = synth.make_inputs(w, seed=22, device="cuda")
    parts = {n: split(x[n], 2) for n in ("q", "k", "v", "gate")}
    out = [torch.empty_like(p) for p in parts["q"]]
    plan = plan_for(vsa, w, heads=4)
    # head_offset + heads beyond heads_total
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_forward_parts(plan, parts["q"], parts["k"], parts["v"], parts["gate"], out, 5)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_SHAPE"
    # parts that do not add up to the sequence
    short = {n: [t[:, :-64].contiguous() for t in parts[n]] for n in parts}
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_forward_parts(plan, short["q"], short["k"], short["v"], short["gate"],
                              [t[:, :-64].contiguous() for t in out], 0)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_SHAPE"
    plan.destroy()
    seq_plan = plan_for(vsa, w, heads=4, seq_tiles=True)
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_forward_parts(seq_plan, parts["q"], parts["k"], parts["v"], parts["gate"], out, 0)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_UNSUPPORTED"
    seq_plan.destroy()
    with pytest.raises(ValueError):
        vsa.ulysses_partition(w.seq_len, w.heads, 3, 0)  # 3 does not divide the 8 heads
