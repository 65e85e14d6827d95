"""8-bit Q/K plans (qk_fp8) on the GPU against the oracle's 8-bit variant.

Bar: the E4M3 code rows and row scales the gather kernel writes are bit-exact
with the oracle's quantiser (including the zero bytes past D and the zero
pad rows); pooled tiles, scores and the selection stay bit-exact (they read
the bf16 inputs); the output is within the bf16 path's tolerance (max-abs
2e-2, mean-abs 2e-3) of the float64 oracle whose logits use the dequantised
8-bit Q and K.  The sequence-part, host-pipeline and 1344x768 routes are
checked the same way (bit-identical to the device forward, or sampled).  The
8-bit prefix query row blocks run on the pair kernel when their pairs fill the
SMs, else on the transposed kernel; both are checked in full."""
import ctypes
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


def plan_for(vsa, w, heads=None):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=heads or w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, qk_fp8=True)


def run(vsa, w, x):
    plan = plan_for(vsa, w)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return plan, ws, out


def tile_codes(codes, scales, geo, tiles=None):
    """Tile-order code rows [B, H, n, 64, 128] and scales [B, H, n, 64] of the oracle's quantisation
    ([B, L, H, D] codes, [B, L, H] scales), for the listed tiles (default all): pad rows and bytes past
    D are zero."""
    B, L, H, D = codes.shape
    tiles = np.arange(geo.n_tiles) if tiles is None else np.asarray(tiles)
    c = np.zeros((B, H, len(tiles), 64, 128), np.uint8)
    s = np.zeros((B, H, len(tiles), 64), np.float32)
    tok = geo.tile_token[tiles]
    valid = tok >= 0
    for b in range(B):
        c[b][:, valid, :D] = codes[b].transpose(1, 0, 2)[:, tok[valid]]
        s[b][:, valid] = scales[b].T[:, tok[valid]]
    return c, s


def compare_out(got, ref):
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    return err.max(), err.mean()


def full_parity(vsa, oracle_mod, w, seed=0, x=None):
    if x is None:
        x = synth.make_inputs(w, seed=seed, device="cuda")
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, qk8=True)
    plan, ws, out = run(vsa, w, x)
    views = vsa.workspace_views(plan, ws)
    for n in ("q", "k"):
        codes, scales = oracle_mod.quant_e4m3(xb[n])
        ec, es = tile_codes(codes, scales, ref.geo)
        assert np.array_equal(views[n + "_t"].cpu().numpy(), ec), n
        assert np.array_equal(views[n + "_s"].cpu().numpy(), es), n
    for n in ("pq", "pk", "pv"):
        assert np.array_equal(views[n].cpu().numpy(), getattr(ref, n)), n
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    assert np.array_equal(views["idx"].cpu().numpy(), ref.idx)
    got = out.float().cpu().numpy().astype(np.float64)
    compare_out(got, ref.out)
    plan.destroy()
    return ref, got


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_fp8_full_parity(vsa, oracle_mod, name):
    ref, got = full_parity(vsa, oracle_mod, synth.workload(name))
    # the 8-bit logits change the result: the output is not the bf16 forward's
    w = synth.workload(name)
    x = synth.make_inputs(w, seed=0)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    bf = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity)
    assert np.abs(ref.out - bf.out).max() > 0


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((), (8, 8, 8), 0.5, 1, 2, 64),               # no prefix, head_dim 64 (code bytes 64..127 zero)
    ((100, 30), (0, 0, 0), 0.9, 1, 2, 128),       # prefix only
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 128),      # ragged everywhere, batch 2
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 3, 96),       # head_dim 96: three 32-byte K-steps
    ((33,), (4, 4, 12), 0.5, 1, 2, 128),          # odd key-tile count: half-masked last block
    ((40, 0, 24), (5, 9, 6), 0.5, 5, 2, 128),     # batch 5, partial cubes
    ((1,), (4, 4, 4), 0.0, 1, 1, 64),             # one-token prefix tile, one cube
])
def test_fp8_edge_cases(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    w = synth.Workload("edge8", B, H, D, tuple(segments), tuple(grid), sparsity)
    full_parity(vsa, oracle_mod, w, seed=3)


@pytest.mark.parametrize("segments,grid,sparsity,B,H,D", [
    ((128, 0, 64), (4, 8, 8), 0.5, 2, 40, 128),  # 3 prefix tiles: a full pair and a half pair; 160 pairs
    ((100, 30), (0, 0, 0), 0.9, 1, 148, 64),     # prefix only: one pair of ragged tiles per head, D = 64
    ((70, 0, 5), (5, 6, 7), 0.6, 2, 50, 96),     # ragged prefix and video tiles, head_dim 96
])
def test_fp8_prefix_pairs_full_parity(vsa, oracle_mod, segments, grid, sparsity, B, H, D):
    """Enough heads that the 8-bit prefix query row blocks go to the pair kernel (its kind::f8f6f4 S with
    the key and query row scales in the softmax), in full against the oracle's 8-bit variant."""
    w = synth.Workload("pairs8", B, H, D, tuple(segments), tuple(grid), sparsity)
    assert prefix_on_pair_kernel(w)
    full_parity(vsa, oracle_mod, w, seed=9)


def test_fp8_zero_and_extreme_rows(vsa, oracle_mod):
    """Rows that are all zero (scale 0, codes 0: their logits are 0), rows with one nonzero element, and
    rows of very different magnitudes in one tile (each row keeps its own scale)."""
    w = dataclasses.replace(synth.workload("small"), name="small_rows8")
    x = synth.make_inputs(w, seed=9, device="cuda")
    x["q"][0, 5:70, 2] = 0
    x["k"][0, 100:140, 3] = 0
    x["k"][0, 200:260, 1, 1:] = 0
    x["q"][0, 300:330, 4] *= 1e-4
    x["k"][0, 330:360, 4] *= 300.0
    full_parity(vsa, oracle_mod, w, x=x)


def test_fp8_gate_per_channel_and_gate_zero(vsa, oracle_mod):
    w = dataclasses.replace(synth.workload("small"), gate_per_channel=True, head_dim=96, name="small_pc8")
    full_parity(vsa, oracle_mod, w, seed=4)
    w = dataclasses.replace(synth.workload("tiny"), name="tiny_zg8")
    x = synth.make_inputs(w, seed=4, device="cuda")
    x["gate"].zero_()
    full_parity(vsa, oracle_mod, w, x=x)


def test_fp8_768p_sampled(vsa, oracle_mod):
    """The 1344x768-shaped workload at sparsity 0.9 with 8-bit Q/K, in the bench's launch configuration:
    the selection in full, the code rows and scales of sampled tiles bit-exact, sampled output tiles."""
    w = synth.workload("768p_s0.9")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan, ws, out = run(vsa, w, x)
    views = vsa.workspace_views(plan, ws)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(xb["q"], xb["k"], xb["v"], w.segments, w.grid, w.sparsity)
    geo = sel["geo"]
    assert np.array_equal(views["idx"].cpu().numpy(), sel["idx"])
    q8 = (*oracle_mod.quant_e4m3(xb["q"]), *oracle_mod.quant_e4m3(xb["k"]))
    tiles = [0, geo.n_prefix - 1, geo.n_prefix, geo.n_tiles // 2, geo.n_tiles - 1]
    for n, (codes, scales) in (("q", q8[:2]), ("k", q8[2:])):
        ec, es = tile_codes(codes, scales, geo, tiles)
        assert np.array_equal(views[n + "_t"][:, :, tiles].cpu().numpy(), ec), n
        assert np.array_equal(views[n + "_s"][:, :, tiles].cpu().numpy(), es), n
    heads = [0, 31, 55]
    items = np.array([h * geo.n_tiles + i for h in heads for i in sorted(set(tiles + list(range(geo.n_prefix,
                                                                                               geo.n_tiles, 211))))],
                     np.int64)
    of = oracle_mod.fine_tiles(xb["q"], xb["k"], xb["v"], geo, sel["idx"], sel["topk"], sel["scale"], items, qk8=q8)
    ref = oracle_mod.output_tiles(of, sel["o_c"], xb["gate"], geo, items, w.heads)
    got = np.zeros_like(ref)
    for n, bhi in enumerate(items):
        i, h = int(bhi % geo.n_tiles), int(bhi // geo.n_tiles)
        nv = int(geo.tile_valid[i])
        rows = torch.from_numpy(geo.tile_token[i, :nv].astype(np.int64)).cuda()
        got[n, :nv] = out[0][rows, h].double().cpu().numpy()
    compare_out(got, ref)
    plan.destroy()


def test_fp8_parts_and_host_pipeline_match_device_forward(vsa):
    """Sequence parts (4 emulated ranks) and the host pipeline give the device forward's bits."""
    w = synth.workload("small")
    x = synth.make_inputs(w, seed=6, device="cuda")
    plan, ws, ref = run(vsa, w, x)
    hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "gate")}
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=3)
    assert torch.equal(out, ref.cpu())
    plan.destroy()
    world = 4
    parts = {n: [c.contiguous() for c in torch.chunk(x[n], world, dim=1)] for n in ("q", "k", "v", "gate")}
    outs = [torch.full_like(p, float("nan")) for p in parts["q"]]
    for rank in range(world):
        ls, hn, h0 = vsa.ulysses_partition(w.seq_len, w.heads, world, rank)
        p = plan_for(vsa, w, heads=hn)
        vsa.vsa_forward_parts(p, parts["q"], parts["k"], parts["v"], parts["gate"], outs, h0)
        torch.cuda.synchronize()
        assert vsa.device_status(p) == (0, 0)
        p.destroy()
    assert torch.equal(torch.cat(outs, dim=1), ref)


def test_fp8_step_entry_points_refuse(vsa):
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=1, device="cuda")
    plan = plan_for(vsa, w)
    B, H, D, n_t = w.batch, w.heads, w.head_dim, plan.dims["n_tiles"]
    t = [torch.empty(B, H, n_t, 64, D, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_gather_tiles(plan, x["q"], x["k"], x["v"], *t)
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_UNSUPPORTED"
    lib = vsa.load_library()
    p = [ctypes.c_void_p(a.data_ptr()) for a in t]
    assert lib.vsa_sparse_attn_fwd(plan.handle, *p, p[0], p[0], p[0], p[0], None, None, None) == 3
    plan.destroy()
