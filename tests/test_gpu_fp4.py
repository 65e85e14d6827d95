"""FP4 video query tiles (qk_fp8="fp4") on the GPU against the oracle's FP4 variant.

The video query tiles take their logits from FP4 Q and K (E2M1 values with one E4M3 scale per 16
values, global scale 1), K smoothed first by its per-head mean; the dense prefix query tiles keep
the 8-bit split; P.V stays bf16 ("FastH3 OmniRef inference", sections "Device profiles",
"Environment" and "Fallbacks").  Bar: the key means, the FP4 roundings in the tile copies, the 8-bit
codes, pooled tiles, scores and the selection bit-exact with the oracle; the output within max-abs
2e-2 and mean-abs 2e-3 of the float64 oracle (forward with fp4=True, qk8="prefix"); the prefix rows
bit-identical to the prefix split's (the same 8-bit launch)."""
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


def forward(vsa, w, x, qk):
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, tile_size=w.tile,
                              cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep, qk_fp8=qk)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return plan, ws, out


def tile_values(bits, geo):
    """Tile-order float32 rows [B, H, n_t, T, D] of bf16-bit arrays [B, L, H, D] (pad rows 0)."""
    B, L, H, D = bits.shape
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    out = np.zeros((B, H, geo.n_tiles, geo.tile, D), np.float32)
    tok, valid = geo.tile_token, geo.tile_token >= 0
    for b in range(B):
        out[b][:, valid] = f[b].transpose(1, 0, 2)[:, tok[valid]]
    return out


def prefix_tokens(geo, L):
    t = np.zeros(L, bool)
    for i in range(geo.n_prefix):
        t[geo.tile_token[i, :geo.tile_valid[i]]] = True
    return t


def full_parity(vsa, oracle_mod, w, seed=0):
    x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, qk8="prefix",
                             fp4=True, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    geo, P = ref.geo, ref.geo.n_prefix
    plan, ws, out = forward(vsa, w, x, "fp4")
    views = vsa.workspace_views(plan, ws)
    for n in ("pq", "pk", "pv"):
        assert np.array_equal(views[n].cpu().numpy(), getattr(ref, n)), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    mu, _ = oracle_mod.smooth_keys(xb["k"])
    assert np.array_equal(views["k_mu"].cpu().numpy(), mu)
    q4, k4 = oracle_mod.fp4_operands(xb["q"], xb["k"])
    # the FP4 roundings in the tile copies (compared as values: a zero may carry either sign)
    gq, gk = views["q_t"].float().cpu().numpy(), views["k_t"].float().cpu().numpy()
    assert np.array_equal(gk, tile_values(k4, geo))
    assert np.array_equal(gq[:, :, P:], tile_values(q4, geo)[:, :, P:])
    assert np.array_equal(gq[:, :, :P], tile_values(xb["q"], geo)[:, :, :P])  # prefix query tiles: bf16
    # the prefix split's 8-bit codes (prefix query tiles and every key tile)
    for n in ("q", "k"):
        codes, scales = oracle_mod.quant_e4m3(xb[n])
        c = np.zeros((w.batch, w.heads, geo.n_tiles, geo.tile, 128), np.uint8)
        tok, valid = geo.tile_token, geo.tile_token >= 0
        for b in range(w.batch):
            c[b][:, valid, :w.head_dim] = codes[b].transpose(1, 0, 2)[:, tok[valid]]
        t = P if n == "q" else geo.n_tiles
        assert np.array_equal(views[n + "_c"].cpu().numpy()[:, :, :t], c[:, :, :t]), n
    got = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref.out)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    # the prefix rows: the prefix split's bits
    _, _, sp = forward(vsa, w, x, "prefix")
    pre = torch.from_numpy(prefix_tokens(geo, w.seq_len)).cuda()
    assert torch.equal(out[:, pre], sp[:, pre])
    plan.destroy()
    return ref


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_fp4_full_parity(vsa, oracle_mod, name):
    full_parity(vsa, oracle_mod, synth.workload(name))


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((), (8, 8, 8), 0.5, 1, 2, 64),               # no prefix: every query tile FP4
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128),       # prefix only: the split's 8-bit launch alone
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128),      # ragged everywhere, batch 2
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 96),       # head_dim 96 (six 16-value blocks per row)
    ((33,), (4, 4, 12), 0.5, 1, 2, 128),          # odd key-tile count
])
def test_fp4_edge_cases(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    w = synth.Workload("fp4", B, H, D, tuple(segments), tuple(grid), sparsity)
    full_parity(vsa, oracle_mod, w, seed=3)


def test_fp4_128_token_tiles(vsa, oracle_mod):
    w = dataclasses.replace(synth.workload("small"), tile=128, name="small_t128")
    full_parity(vsa, oracle_mod, w, seed=5)


def test_fp4_reference_keep(vsa, oracle_mod):
    w = synth.Workload("fp4_ref", 1, 4, 128, (40, 200, 24), (8, 8, 16), 0.5, ref_segments=(False, True, False),
                       ref_keep=0.1)
    full_parity(vsa, oracle_mod, w, seed=6)


def test_fp4_480p_sampled(vsa, oracle_mod):
    """480p-shaped workload: the selection, the key means and the key copies' FP4 roundings in full,
    and sampled video query tiles of three heads against the oracle's FP4 fine branch."""
    w = synth.workload("480p")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan, ws, out = forward(vsa, w, x, "fp4")
    views = vsa.workspace_views(plan, ws)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity)
    geo = sel["geo"]
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    assert np.array_equal(views["k_mu"].cpu().numpy(), oracle_mod.smooth_keys(xb["k"])[0])
    q4, k4 = oracle_mod.fp4_operands(xb["q"], xb["k"])
    assert np.array_equal(views["k_t"].float().cpu().numpy(), tile_values(k4, geo))
    heads = [0, 27, 55]
    items = np.array([h * geo.n_tiles + i for h in heads for i in range(geo.n_prefix, geo.n_tiles, 41)], np.int64)
    of = oracle_mod.fine_tiles(q4, k4, xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items)
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


def test_fp4_step_entry_points_reject(vsa):
    w = synth.workload("tiny")
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, qk_fp8="fp4")
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_gather_tiles(plan, t, t, t, t, t, t)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_UNSUPPORTED"
    plan.destroy()
