"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded bytes.

Bar: tile-order gather, pooled Q/K/V and pooled scores bit-exact; tile
selection bit-exact; compression within 1e-5 relative; the BF16 output within
max-abs 2e-2 and mean-abs 2e-3 of the float64 oracle.  Small workloads are
compared in full; the 480p- and 1344x768-shaped workloads compare the whole
selection and a fixed sample of query tiles of the attention.
"""
import dataclasses

import numpy as np
import pytest
import torch

import synth
from conftest import prefix_on_pair_kernel

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


def bits(t):
    return synth.as_bits(t)


def plan_for(vsa, w, seq_tiles=False):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, seq_tiles=seq_tiles)


def run_forward(vsa, w, x, seq_tiles=False):
    plan = plan_for(vsa, w, seq_tiles)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return plan, ws, out


def run_stepwise(vsa, plan, x):
    """S2..S5 through the separate entry points, pooling from tile order."""
    d, g = plan.dims, plan.geometry
    B, H, D, n_t, V, k = g["batch"], g["heads"], g["head_dim"], d["n_tiles"], d["n_video_tiles"], d["topk"]
    dev = x["q"].device
    bf = dict(dtype=torch.bfloat16, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    t = {n: torch.empty(B, H, n_t, 64, D, **bf) for n in ("q_t", "k_t", "v_t")}
    vsa.vsa_gather_tiles(plan, x["q"], x["k"], x["v"], t["q_t"], t["k_t"], t["v_t"])
    pq, pk, pv = (torch.empty(B, H, n_t, D, **f32) for _ in range(3))
    S = torch.empty(B, H, n_t, n_t, **f32)
    vsa.vsa_pool_and_score(plan, t["q_t"], t["k_t"], t["v_t"], pq, pk, pv, S)
    idx = torch.empty(B, H, max(V, 1), max(k, 1), dtype=torch.int32, device=dev)
    o_c = torch.empty(B, H, n_t, D, **f32)
    vsa.vsa_topk_select(plan, S, pv, idx, o_c)
    out = torch.empty_like(x["q"])
    vsa.vsa_sparse_attn_fwd(plan, t["q_t"], t["k_t"], t["v_t"], idx, o_c, x["gate"], out)
    torch.cuda.synchronize()
    return dict(t, pq=pq, pk=pk, pv=pv, S=S, idx=idx[:, :, :V, :k], o_c=o_c, out=out)


def expected_tiles(xbits, geo):
    """Tile-order copy of a [B, L, H, D] array, built from the oracle's token table."""
    B, L, H, D = xbits.shape
    tok = geo.tile_token
    res = np.zeros((B, H, geo.n_tiles, 64, D), np.uint16)
    valid = tok >= 0
    for b in range(B):
        src = xbits[b].transpose(1, 0, 2)  # [H, L, D]
        res[b][:, valid] = src[:, tok[valid]]
    return res


def compare_out(gpu_out, ref_out, mask=None):
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    if mask is not None:
        g, ref_out = g[mask], ref_out[mask]
    err = np.abs(g - ref_out)
    assert np.isfinite(g).all()
    assert err.max() <= MAX_ABS, f"max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"mean-abs {err.mean():.3e}"
    return err.max(), err.mean()


def full_parity(vsa, oracle_mod, w, seed=0, seq_tiles=False):
    x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity)
    plan, ws, out = run_forward(vsa, w, x, seq_tiles)
    views = vsa.workspace_views(plan, ws)
    step = run_stepwise(vsa, plan, x)
    for n in ("q", "k", "v"):
        exp = expected_tiles(xb[n], ref.geo)
        assert np.array_equal(bits(step[n + "_t"]), exp), n
        if not seq_tiles:  # vsa_forward made tile-order copies (with seq_tiles it read sequence order)
            assert np.array_equal(bits(views[n + "_t"]), exp), n
    for n in ("pq", "pk", "pv"):
        r = getattr(ref, n)
        assert np.array_equal(views[n].cpu().numpy(), r), n
        assert np.array_equal(step[n].cpu().numpy(), r), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(step["S"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    assert np.array_equal(step["idx"].cpu().numpy(), ref.idx)
    for oc in (views["o_c"], step["o_c"]):
        g = oc.cpu().numpy().astype(np.float64)
        assert np.abs(g - ref.o_c).max() <= 1e-5 * max(1.0, np.abs(ref.o_c).max())
    compare_out(out, ref.out)
    compare_out(step["out"], ref.out)
    # With tile-order copies in both routes the same kernels run on the same rows: identical bits.  A
    # seq_tiles forward keeps the prefix query rows on vsa_attn_kernel while the stepwise route (tile-order
    # copies) runs them on the prefix pair kernel, so there only the video rows must agree bit for bit, and
    # only with full tiles (partial tiles read from sequence order hold their rows at cube positions, which
    # changes the MMA summation order); both routes are checked against the oracle above.
    if not seq_tiles:
        assert torch.equal(out, step["out"])
    elif bool((ref.geo.tile_valid == 64).all()):
        vid = torch.ones(w.seq_len, dtype=torch.bool)
        for i in range(ref.geo.n_prefix):
            vid[torch.from_numpy(ref.geo.tile_token[i, :ref.geo.tile_valid[i]].astype(np.int64))] = False
        vid = vid.cuda()
        assert torch.equal(out[:, vid], step["out"][:, vid])
    plan.destroy()
    return ref


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_full_parity(vsa, oracle_mod, name):
    full_parity(vsa, oracle_mod, synth.workload(name))


def test_tiny_sparsity0_is_dense_attention(vsa, oracle_mod):
    """At sparsity 0 the fine branch is dense softmax attention over the packed
    sequence; check the GPU against torch SDPA (float64) plus the gate term."""
    w = synth.workload("tiny", sparsity=0.0)
    ref = full_parity(vsa, oracle_mod, w)
    x = synth.make_inputs(w, device="cuda")
    plan, ws, out = run_forward(vsa, w, x)
    q, k, v = (x[n].double()[0].transpose(0, 1) for n in ("q", "k", "v"))  # [H, L, D]
    dense = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=ref.scale).transpose(0, 1)
    comp = ref.out - ref.o_f  # gate * o_c, per row
    expect = dense.cpu().numpy()[None] + comp
    compare_out(out, expect)


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((), (8, 8, 8), 0.5, 1, 2, 64),               # no prefix
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128),       # prefix only: every query tile dense
    ((10,), (3, 2, 5), 0.5, 1, 3, 128),           # grid sides below 4: one partial cube
    ((40, 0, 24), (8, 8, 8), 1.0, 1, 2, 64),      # topk = 1
    ((40, 0, 24), (8, 8, 8), 0.0, 2, 2, 128),     # topk = V, batch 2
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128),      # ragged everywhere
    ((1,), (4, 4, 4), 0.0, 1, 1, 64),             # one-token prefix tile, one cube
    ((64, 64, 64), (4, 8, 12), 0.75, 1, 4, 128),  # even count of key tiles
    ((33,), (4, 4, 12), 0.5, 1, 2, 128),          # odd count of key tiles: half-masked last block
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 96),       # head_dim 96, ragged everywhere
    ((40, 0, 24), (5, 9, 6), 0.5, 5, 2, 128),     # batch 5, partial cubes
])
def test_edge_cases(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    w = synth.Workload("edge", B, H, D, tuple(segments), tuple(grid), sparsity)
    full_parity(vsa, oracle_mod, w, seed=3)


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((128, 0, 64), (4, 8, 8), 0.5, 2, 40, 128),  # 3 prefix tiles: a full pair and a half pair; 160 pairs
    ((100, 30), (0, 0, 0), 0.9, 1, 148, 64),     # prefix only: one pair of ragged tiles per head
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 50, 96),     # ragged prefix and video tiles, head_dim 96
])
def test_prefix_pairs_full_parity(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    """64-token tiles with enough heads that the prefix query row blocks go to the pair kernel, in full
    against the oracle (the smaller workloads above leave them to the video kernel)."""
    w = synth.Workload("pairs", B, H, D, tuple(segments), tuple(grid), sparsity)
    assert prefix_on_pair_kernel(w)
    full_parity(vsa, oracle_mod, w, seed=9)


def sampled_parity(vsa, oracle_mod, w, heads, video_every, batches=(0,), seq_tiles=False):
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan, ws, out = run_forward(vsa, w, x, seq_tiles)
    views = vsa.workspace_views(plan, ws)
    xb = {n: bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity)
    geo = sel["geo"]
    assert np.array_equal(views["pq"].cpu().numpy(), sel["pq"])
    assert np.array_equal(views["pk"].cpu().numpy(), sel["pk"])
    assert np.array_equal(views["scores"].cpu().numpy(), sel["S"])
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    g = views["o_c"].cpu().numpy().astype(np.float64)
    assert np.abs(g - sel["o_c"]).max() <= 1e-5 * max(1.0, np.abs(sel["o_c"]).max())
    tiles = [0, geo.n_prefix - 1] + list(range(geo.n_prefix, geo.n_tiles, video_every)) + [geo.n_tiles - 1]
    items = np.array([(b * w.heads + h) * geo.n_tiles + i for b in batches for h in heads for i in sorted(set(tiles))],
                     np.int64)
    of = oracle_mod.fine_tiles(xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items)
    ref = oracle_mod.output_tiles(of, sel["o_c"], xb["gate"], geo, items, w.heads)
    got = np.zeros_like(ref)
    for n, bhi in enumerate(items):
        i, bh = int(bhi % geo.n_tiles), int(bhi // geo.n_tiles)
        b, h = bh // w.heads, bh % w.heads
        nv = int(geo.tile_valid[i])
        got[n, :nv] = out[b][torch.from_numpy(geo.tile_token[i, :nv].astype(np.int64)).cuda(), h].double().cpu().numpy()
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    plan.destroy()


def test_480p_selection_full_attention_sampled(vsa, oracle_mod):
    sampled_parity(vsa, oracle_mod, synth.workload("480p"), heads=[0, 27, 55], video_every=19)


def test_768p_s09_selection_full_attention_sampled(vsa, oracle_mod):
    """The 1344x768-shaped workload at sparsity 0.9, in the launch configuration the bench times."""
    sampled_parity(vsa, oracle_mod, synth.workload("768p_s0.9"), heads=[0, 31, 55], video_every=131)


def test_repeatable_and_status_clean(vsa):
    w = synth.workload("small")
    x = synth.make_inputs(w, device="cuda")
    plan, ws, out1 = run_forward(vsa, w, x)
    out2 = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    assert vsa.device_status(plan) == (0, 0)


def test_call_errors(vsa):
    w = synth.workload("tiny")
    x = synth.make_inputs(w, device="cuda")
    plan = plan_for(vsa, w)
    ws = vsa.alloc_workspace(plan)
    out = torch.empty_like(x["q"])
    lib = vsa.load_library()
    import ctypes

    def call(q_ptr, ws_ptr, ws_bytes):
        return lib.vsa_forward(plan.handle, q_ptr, ctypes.c_void_p(x["k"].data_ptr()),
                               ctypes.c_void_p(x["v"].data_ptr()), ctypes.c_void_p(x["gate"].data_ptr()),
                               ctypes.c_void_p(out.data_ptr()), ws_ptr, ws_bytes, None)

    qp = x["q"].data_ptr()
    wsp = ctypes.c_void_p(ws.data_ptr())
    assert call(ctypes.c_void_p(qp + 2), wsp, ws.numel()) == 1  # misaligned -> VSA_ERR_INVALID_ARG
    assert call(None, wsp, ws.numel()) == 1  # NULL -> VSA_ERR_INVALID_ARG
    assert call(ctypes.c_void_p(qp), wsp, plan.dims["workspace_bytes"] - 256) == 4  # VSA_ERR_WORKSPACE
    assert call(ctypes.c_void_p(qp), ctypes.c_void_p(ws.data_ptr() + 16), ws.numel() - 16) == 1  # unaligned ws
    assert call(ctypes.c_void_p(qp), wsp, ws.numel()) == 0
    torch.cuda.synchronize()


def test_768p_s08_selection_full_attention_sampled(vsa, oracle_mod):
    """The 1344x768-shaped workload at sparsity 0.8 (topk 231)."""
    sampled_parity(vsa, oracle_mod, synth.workload("768p_s0.8"), heads=[0, 55], video_every=157)


@pytest.mark.parametrize("sparsity", [0.0, 0.95])
def test_768p_sweep_endpoints_sampled(vsa, oracle_mod, sparsity):
    """Ends of the sparsity sweep at 1344x768: dense video keys (topk 1152) and topk 58."""
    w = dataclasses.replace(synth.workload("768p_s0.9"), sparsity=sparsity, name=f"768p_s{sparsity}")
    sampled_parity(vsa, oracle_mod, w, heads=[13], video_every=383)


def test_768p_batch4_offsets_past_2_31_sampled(vsa, oracle_mod):
    """Batch 4 of the 1344x768-shaped workload: q/k/v/gate/out hold
    4*75008*56*128 = 2,150,629,376 elements each, past 2^31, so the last
    batch's token offsets only come out right in 64-bit arithmetic."""
    w = dataclasses.replace(synth.workload("768p_s0.9"), batch=4, name="768p_s0.9_b4")
    sampled_parity(vsa, oracle_mod, w, heads=[0, 55], video_every=509, batches=(0, 3))


def test_wait_selftest_times_out_and_context_stays_usable(vsa):
    """A bounded wait on a barrier that nothing arrives on ends with
    VSA_ERR_TIMEOUT in the status word; the next forward runs normally."""
    w = synth.workload("tiny")
    plan = plan_for(vsa, w)
    code, where = vsa.wait_selftest(plan, timeout_ns=50_000_000)
    assert code == 6 and where in (100, 101)
    assert vsa.device_status(plan) == (0, 0)
    x = synth.make_inputs(w, device="cuda")
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    assert vsa.device_status(plan) == (0, 0)
    plan.destroy()


@pytest.mark.parametrize("name,seed", [("small", 4), ("tiny", 5)])
def test_head_dim_96_full_parity(vsa, oracle_mod, name, seed):
    """head_dim 96 (the model's 5376 / 56): tile copies, pooled tiles, scores and indices bit-exact,
    compression and output within tolerance.  The attention kernel reads the 96-wide tiles as two
    64-column TMA boxes whose columns 96..127 are zero-filled."""
    w = dataclasses.replace(synth.workload(name), head_dim=96, name=f"{name}_d96")
    full_parity(vsa, oracle_mod, w, seed=seed)


def test_head_dim_96_480p_sampled(vsa, oracle_mod):
    """The 480p-shaped workload at head_dim 96, selection in full and sampled output tiles."""
    w = dataclasses.replace(synth.workload("480p"), head_dim=96, name="480p_d96")
    sampled_parity(vsa, oracle_mod, w, heads=[0, 29, 55], video_every=23)


@pytest.mark.parametrize("name,D", [("tiny", 64), ("small", 128), ("small", 96)])
def test_gate_per_channel_full_parity(vsa, oracle_mod, name, D):
    """Per-channel gate [B, L, H*D]: the epilogue scales column d of head h by channel h*D + d."""
    w = dataclasses.replace(synth.workload(name), head_dim=D, gate_per_channel=True, name=f"{name}_pc")
    full_parity(vsa, oracle_mod, w, seed=7)


def test_gate_per_channel_480p_sampled(vsa, oracle_mod):
    w = dataclasses.replace(synth.workload("480p"), gate_per_channel=True, name="480p_pc")
    sampled_parity(vsa, oracle_mod, w, heads=[3, 54], video_every=29)


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D,pc", [
    ((40, 0, 24), (8, 8, 8), 0.5, 1, 2, 64, False),   # tiny shape
    ((256, 64, 192), (8, 16, 32), 0.8, 1, 8, 128, False),  # small shape
    ((40, 0, 24), (5, 9, 6), 0.5, 4, 2, 64, False),   # batch 4 (the limit), partial cubes
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128, False),   # ragged everywhere: prefix boxes read past their run
    ((33,), (4, 4, 12), 0.5, 1, 2, 96, True),         # head_dim 96, per-channel gate, odd key-tile count
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128, False),    # prefix only
])
def test_seq_tiles_full_parity(vsa, oracle_mod, segments, grid, sparsity, B, H, D, pc):
    """Plans with seq_tiles: the attention reads every tile straight from sequence order (a 4-D TMA box per
    64-token prefix run, a 5-D box per 4x4x4 cube, out-of-tile rows masked) and no tile-order copy is made."""
    w = synth.Workload("seq", B, H, D, tuple(segments), tuple(grid), sparsity, gate_per_channel=pc)
    full_parity(vsa, oracle_mod, w, seed=14, seq_tiles=True)


def test_seq_tiles_480p_sampled(vsa, oracle_mod):
    sampled_parity(vsa, oracle_mod, synth.workload("480p"), heads=[0, 28, 55], video_every=19, seq_tiles=True)
