"""The pages' prefix split (qk_fp8="prefix") on the GPU against the oracle's split fine branch.

The dense prefix query tiles take their logits from 8-bit Q/K (E4M3 codes, one binary32 scale per token
and head) with bf16 P.V; the video query tiles keep the bf16 logits ("FastH3 OmniRef inference", section
"Device profiles").  Bar: the code rows and row scales bit-exact with the oracle's quantiser; pooled
tiles, scores and the selection bit-exact; the output within max-abs 2e-2 and mean-abs 2e-3 of the
float64 oracle (fine_split), whose prefix rows use the dequantised 8-bit Q and K and whose video rows use
the bf16 ones.  The video rows are also bit-identical to the bf16 forward's (the same kernel on the same
items), which shows the split sends each query tile down the right path."""
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


def plan_for(vsa, w, qk):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, tile_size=w.tile,
                              cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep, qk_fp8=qk)


def forward(vsa, w, x, qk):
    plan = plan_for(vsa, w, qk)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return plan, ws, out


def tile_codes(codes, scales, geo):
    """Tile-order code rows [B, H, n_t, T, 128] and scales [B, H, n_t, T] of the oracle's quantisation."""
    B, L, H, D = codes.shape
    T = geo.tile
    c = np.zeros((B, H, geo.n_tiles, T, 128), np.uint8)
    s = np.zeros((B, H, geo.n_tiles, T), np.float32)
    tok = geo.tile_token
    valid = tok >= 0
    for b in range(B):
        c[b][:, valid, :D] = codes[b].transpose(1, 0, 2)[:, tok[valid]]
        s[b][:, valid] = scales[b].T[:, tok[valid]]
    return c, s


def prefix_tokens(geo, L):
    t = np.zeros(L, bool)
    for i in range(geo.n_prefix):
        t[geo.tile_token[i, :geo.tile_valid[i]]] = True
    return t


def full_parity(vsa, oracle_mod, w, seed=0):
    x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, qk8="prefix",
                             tile=w.tile, cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    plan, ws, out = forward(vsa, w, x, "prefix")
    views = vsa.workspace_views(plan, ws)
    P = ref.geo.n_prefix
    for n in ("q", "k"):
        codes, scales = oracle_mod.quant_e4m3(xb[n])
        ec, es = tile_codes(codes, scales, ref.geo)
        # queries: only the prefix tiles are quantised (the video query tiles keep bf16 logits)
        t = P if n == "q" else ref.geo.n_tiles
        assert np.array_equal(views[n + "_c"].cpu().numpy()[:, :, :t], ec[:, :, :t]), n
        assert np.array_equal(views[n + "_s"].cpu().numpy()[:, :, :t], es[:, :, :t]), n
    for n in ("pq", "pk", "pv"):
        assert np.array_equal(views[n].cpu().numpy(), getattr(ref, n)), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref.out)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    # video rows: the bf16 forward's bits
    _, _, bf = forward(vsa, w, x, False)
    vid = ~prefix_tokens(ref.geo, w.seq_len)
    assert torch.equal(out[:, torch.from_numpy(vid).cuda()], bf[:, torch.from_numpy(vid).cuda()])
    plan.destroy()
    return ref


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_prefix_split_full_parity(vsa, oracle_mod, name):
    full_parity(vsa, oracle_mod, synth.workload(name))


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((), (8, 8, 8), 0.5, 1, 2, 64),               # no prefix: the bf16 forward
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128),       # prefix only: every query tile on the 8-bit kernel
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128),      # ragged everywhere, batch 2
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 96),       # head_dim 96
    ((33,), (4, 4, 12), 0.5, 1, 2, 128),          # odd key-tile count
])
def test_prefix_split_edge_cases(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    w = synth.Workload("split", B, H, D, tuple(segments), tuple(grid), sparsity)
    full_parity(vsa, oracle_mod, w, seed=3)


def test_prefix_split_128_token_tiles(vsa, oracle_mod):
    w = dataclasses.replace(synth.workload("small"), tile=128, name="small_t128")
    full_parity(vsa, oracle_mod, w, seed=5)


def test_prefix_split_reference_keep(vsa, oracle_mod):
    w = synth.Workload("split_ref", 1, 4, 128, (40, 200, 24), (8, 8, 16), 0.5, ref_segments=(False, True, False),
                       ref_keep=0.1)
    full_parity(vsa, oracle_mod, w, seed=6)


def test_prefix_split_480p_sampled(vsa, oracle_mod):
    """480p-shaped workload: the whole selection, and sampled query tiles (every prefix tile of three heads,
    some video tiles) against the split oracle."""
    w = synth.workload("480p")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan, ws, out = forward(vsa, w, x, "prefix")
    views = vsa.workspace_views(plan, ws)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity)
    geo = sel["geo"]
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    q8 = (*oracle_mod.quant_e4m3(xb["q"]), *oracle_mod.quant_e4m3(xb["k"]))
    heads = [0, 27, 55]
    pre = [h * geo.n_tiles + i for h in heads for i in range(geo.n_prefix)]
    vid = [h * geo.n_tiles + i for h in heads for i in range(geo.n_prefix, geo.n_tiles, 41)]
    args = (xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"])
    for items, qk in ((pre, q8), (vid, None)):
        items = np.array(items, np.int64)
        of = oracle_mod.fine_tiles(*args, items, qk8=qk)
        ref = oracle_mod.output_tiles(of, sel["o_c"], xb["gate"], geo, items, w.heads)
        got = np.zeros_like(ref)
        for n, hi in enumerate(items):
            i, h = int(hi % geo.n_tiles), int(hi // geo.n_tiles)
            nv = int(geo.tile_valid[i])
            rows = torch.from_numpy(geo.tile_token[i, :nv].astype(np.int64)).cuda()
            got[n, :nv] = out[0][rows, h].double().cpu().numpy()
        err = np.abs(got - ref)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    plan.destroy()


def test_prefix_split_step_entry_points_reject(vsa):
    w = synth.workload("tiny")
    plan = plan_for(vsa, w, "prefix")
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_gather_tiles(plan, t, t, t, t, t, t)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_UNSUPPORTED"
    plan.destroy()
