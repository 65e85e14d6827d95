"""The attention's overflow bound on the GPU.

With bf16 Q/K the attention bounds every logit of a (b, h) by |q| max|k| (Cauchy-Schwarz).  When, for
every column of a softmax group, that bound lies within 124 - ceil(log2 keys) - ceil(log2 max|v|)+
(log2 units) of the first block's exact maximum, no later block can overflow P, l or O^T, and the group
stops voting on rescales for the rest of the item.  The statistics come from the gather (forward) or
from a kernel over the tile-order inputs (step entry point).

What is checked here:
  * the statistics: query row norms and the (b, h) maxima against float64 norms of the tile-order
    copies (64- and 128-token tiles, D = 96), and the sequence-order route's equal to the tile route's;
    the step route's (passed from the gather to the attention) equal to the fused forward's;
    with 8-bit Q/K the norms of the dequantised rows;
  * a workload built so that every group skips (the premise is recomputed here in float64) while the
    logits of later blocks exceed the first block's maximum by about 2^95: parity with the oracle;
  * a workload whose bound is too loose to skip (logit jumps of about 2^290): parity with the oracle;
  * |v| near 2^80: the output scales exactly with v;
  * in sequence order a partial video cube holds its rows at cube positions: one query row there with
    a norm that forbids the skip must get its own norm (a wrong row would let the group skip and the
    row's P overflow to infinity)."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
LOG2E = 1.4426950408889634


@pytest.fixture(scope="module")
def vsa():
    from block_sparse_tiled_b200 import build

    build.build()
    import block_sparse_tiled_b200 as m

    m.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    return m


def plan_for(vsa, w, seq_tiles=False):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel,
                              tile_size=w.tile, cube=w.cube, seq_tiles=seq_tiles)


def f64(t):
    return t.detach().double().cpu().numpy()


def run(vsa, w, x, seq_tiles=False):
    plan = plan_for(vsa, w, seq_tiles)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return plan, ws, out


def compare_to_oracle(oracle_mod, w, x, out):
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, tile=w.tile,
                             cube=w.cube)
    got = f64(out)
    assert np.isfinite(got).all()
    err = np.abs(got - ref.out)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    return ref


def premise(oracle_mod, w, x):
    """Per query token and head: (limit, first-block maximum) in log2 units, as the kernel forms them
    (float64 here; the margins used below dwarf the difference)."""
    geo = oracle_mod.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube)
    q, k, v = (f64(x[n]) for n in ("q", "k", "v"))
    cl = LOG2E / math.sqrt(w.head_dim)
    lg = math.ceil(math.log2(geo.n_tiles * geo.tile))
    cap = 124 - lg
    first = np.concatenate([geo.tile_token[t, :geo.tile_valid[t]] for t in range(min(geo.n_tiles, 128 // geo.tile))])
    kmax = np.linalg.norm(k, axis=-1).max(axis=1)                      # [B, H]
    ev = np.maximum(0, np.frexp(np.abs(v).max(axis=(1, 3)))[1])       # [B, H]
    lim = cl * np.linalg.norm(q, axis=-1) * kmax[:, None, :] + ev[:, None, :] - cap  # [B, L, H]
    m1 = cl * np.einsum("blhd,bkhd->blhk", q, k[:, first]).max(axis=-1)
    return lim, m1


def aligned_inputs(w, seed, a, c, q_noise=0.05):
    """q = a u + noise; prefix keys orthogonal to u (small); 30% of video keys c u + noise (u one random
    unit vector per head [H, D]), v ~ N(0, 1), gate ~ N(0, 0.1).  Returns the bf16 inputs and u."""
    g = torch.Generator().manual_seed(seed)
    B, L, H, D = w.batch, w.seq_len, w.heads, w.head_dim
    npre = sum(w.segments)
    u = torch.randn(H, D, generator=g, dtype=torch.float64)
    u /= u.norm(dim=-1, keepdim=True)
    q = a * u + q_noise * torch.randn(B, L, H, D, generator=g, dtype=torch.float64)
    k = 0.5 * torch.randn(B, L, H, D, generator=g, dtype=torch.float64)
    k[:, :npre] -= (k[:, :npre] * u).sum(-1, keepdim=True) * u
    hit = (torch.rand(B, L - npre, H, 1, generator=g, dtype=torch.float64) < 0.3).double()
    k[:, npre:] += c * u * hit
    v = torch.randn(B, L, H, D, generator=g, dtype=torch.float64)
    gate = 0.1 * torch.randn(B, L, H, generator=g, dtype=torch.float64)
    return {n: t.to(torch.bfloat16).cuda() for n, t in (("q", q), ("k", k), ("v", v), ("gate", gate))}, u


@pytest.mark.parametrize("name,over", [
    ("small", {}),
    ("small", {"tile": 128}),
    ("tiny", {"head_dim": 96}),
    ("edge", {}),
])
def test_statistics(vsa, name, over):
    if name == "edge":
        w = synth.Workload("edge", 2, 3, 128, (70, 0, 5), (5, 6, 7), 0.6)
    else:
        w = dataclasses.replace(synth.workload(name), **over)
    x = synth.make_inputs(w, seed=2, device="cuda")
    plan, ws, _ = run(vsa, w, x)
    views = vsa.workspace_views(plan, ws)
    qt, kt, vt = (f64(views[n]) for n in ("q_t", "k_t", "v_t"))
    qn = np.linalg.norm(qt, axis=-1)
    assert np.allclose(f64(views["q_n"]), qn, rtol=1e-5, atol=0), "query row norms"
    kv = f64(views["kv_max"])
    assert np.allclose(kv[..., 0], np.linalg.norm(kt, axis=-1).max(axis=(2, 3)), rtol=1e-5, atol=0)
    assert np.array_equal(kv[..., 1], np.abs(vt).max(axis=(2, 3, 4)))  # a bf16 value, exact
    plan.destroy()
    if w.tile == 64 and w.batch <= 4:  # the sequence-order route's gather: the same statistics, bit for bit
        plan2, ws2, _ = run(vsa, w, x, seq_tiles=True)
        v2 = vsa.workspace_views(plan2, ws2)
        assert torch.equal(v2["q_n"], views["q_n"]) and torch.equal(v2["kv_max"], views["kv_max"])
        plan2.destroy()


@pytest.mark.parametrize("tile", [64, 128])
def test_step_route_with_statistics(vsa, tile):
    """The step entry points with the gather's statistics passed to the attention: the statistics equal
    the fused forward's, and the output is bit-identical to the fused forward and to the step route that
    lets the attention take its own statistics."""
    w = dataclasses.replace(synth.workload("small"), tile=tile)
    x = synth.make_inputs(w, seed=6, device="cuda")
    plan, ws, out = run(vsa, w, x)
    views = vsa.workspace_views(plan, ws)
    B, H, D, n_t, V = w.batch, w.heads, w.head_dim, plan.dims["n_tiles"], plan.dims["n_video_tiles"]
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    t = {n: torch.empty(B, H, n_t, tile, D, **bf) for n in ("q_t", "k_t", "v_t")}
    pq, pk, pv = (torch.empty(B, H, n_t, D, **f32) for _ in range(3))
    qn = torch.full((B, H, n_t, tile), float("nan"), **f32)
    kv = torch.full((B, H, 2), float("nan"), **f32)  # the call zeroes it before raising it
    vsa.vsa_gather_tiles(plan, x["q"], x["k"], x["v"], t["q_t"], t["k_t"], t["v_t"], pq, pk, pv, q_norm=qn, kv_max=kv)
    S = torch.empty(B, H, n_t, n_t, **f32)
    vsa.vsa_pool_and_score(plan, None, None, None, pq, pk, pv, S)
    idx = torch.empty(B, H, max(V, 1), max(plan.dims["topk"], 1), dtype=torch.int32, device="cuda")
    o_c = torch.empty(B, H, n_t, D, **f32)
    vsa.vsa_topk_select(plan, S, pv, idx, o_c)
    out_passed = torch.empty_like(out)
    vsa.vsa_sparse_attn_fwd(plan, t["q_t"], t["k_t"], t["v_t"], idx, o_c, x["gate"], out_passed, q_norm=qn,
                            kv_max=kv)
    out_own = torch.empty_like(out)
    vsa.vsa_sparse_attn_fwd(plan, t["q_t"], t["k_t"], t["v_t"], idx, o_c, x["gate"], out_own)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    assert torch.equal(qn, views["q_n"]) and torch.equal(kv, views["kv_max"])
    assert torch.equal(out_passed, out) and torch.equal(out_own, out)
    with pytest.raises(vsa.VsaError):  # both statistics or neither
        vsa.vsa_sparse_attn_fwd(plan, t["q_t"], t["k_t"], t["v_t"], idx, o_c, x["gate"], out_own, q_norm=qn)
    plan.destroy()


@pytest.mark.parametrize("tile,D", [(64, 128), (128, 96)])
def test_statistics_fp8(vsa, oracle_mod, tile, D):
    """8-bit Q/K: the norms are those of the dequantised rows (scale times the norm of the E4M3 codes),
    the |v| maximum that of the bf16 values."""
    w = dataclasses.replace(synth.workload("small"), tile=tile, head_dim=D)
    x = synth.make_inputs(w, seed=5, device="cuda")
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=D, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, tile_size=tile, qk_fp8=True)
    ws = vsa.alloc_workspace(plan)
    vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    deq = {n: oracle_mod.dequant_e4m3(views[n + "_t"].cpu().numpy(), views[n + "_s"].cpu().numpy())
           for n in ("q", "k")}
    assert np.allclose(f64(views["q_n"]), np.linalg.norm(deq["q"], axis=-1), rtol=1e-5, atol=0)
    kv = f64(views["kv_max"])
    assert np.allclose(kv[..., 0], np.linalg.norm(deq["k"], axis=-1).max(axis=(2, 3)), rtol=1e-5, atol=0)
    assert np.array_equal(kv[..., 1], np.abs(f64(views["v_t"])).max(axis=(2, 3, 4)))
    plan.destroy()


@pytest.mark.parametrize("tile,seq_tiles", [(64, False), (128, False), (64, True)])
def test_skip_regime_large_logit_jumps(vsa, oracle_mod, tile, seq_tiles):
    """Every group skips the votes (premise checked with a margin of 4), and the aligned keys of later
    blocks sit about 2^95 above the first block's maximum."""
    w = dataclasses.replace(synth.workload("tiny"), tile=tile)
    x, _ = aligned_inputs(w, seed=11, a=23.0, c=23.0)
    lim, m1 = premise(oracle_mod, w, x)
    assert (lim <= m1 - 4).all()
    assert (LOG2E / math.sqrt(w.head_dim) * 23 * 23 - m1).min() > 90  # the jump the skip has to absorb
    plan, ws, out = run(vsa, w, x, seq_tiles)
    compare_to_oracle(oracle_mod, w, x, out)
    plan.destroy()


@pytest.mark.parametrize("tile", [64, 128])
def test_vote_regime_huge_logit_jumps(vsa, oracle_mod, tile):
    """The bound is too loose to skip (logits of later blocks about 2^290 above the first block's): the
    groups vote and rescale as without the bound."""
    w = dataclasses.replace(synth.workload("tiny"), tile=tile)
    x, _ = aligned_inputs(w, seed=12, a=40.0, c=40.0)
    lim, m1 = premise(oracle_mod, w, x)
    assert (lim > m1 + 4).all()
    plan, ws, out = run(vsa, w, x)
    compare_to_oracle(oracle_mod, w, x, out)
    plan.destroy()


def test_large_values_scale_exactly(vsa, oracle_mod):
    """v times 2^80 (exact in bf16): the bound's log2 max|v| term grows by 80; the output is the
    unscaled workload's output times 2^80, within the usual tolerance."""
    w = synth.workload("small")
    x = synth.make_inputs(w, seed=4, device="cuda")
    big = dict(x, v=(x["v"].float() * 2.0 ** 80).to(torch.bfloat16))
    assert torch.equal(big["v"].float() / 2.0 ** 80, x["v"].float())
    plan, ws, out = run(vsa, w, big)
    got = f64(out) / 2.0 ** 80
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity)
    assert np.isfinite(got).all()
    err = np.abs(got - ref.out)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    plan.destroy()


@pytest.mark.parametrize("seq_tiles", [False, True])
def test_partial_cube_row_gets_its_own_norm(vsa, oracle_mod, seq_tiles):
    """Grid 5x6x7: the last video token lies in a partial 1x2x3 cube (cube position 6, tile-order row 5).
    That query row gets a norm whose bound forbids the skip (logits about 2^300 above its first
    block); every other query row is tiny, so its neighbours alone would skip.  The row must be exact."""
    w = synth.Workload("cube", 1, 2, 64, (64, 0, 64), (5, 6, 7), 0.5)
    x, u = aligned_inputs(w, seed=13, a=0.0, c=8.0, q_noise=0.1)
    L = w.seq_len
    q = x["q"].clone()
    q[0, L - 1] = (190.0 * u).to(torch.bfloat16).cuda()
    x = dict(x, q=q)
    lim, m1 = premise(oracle_mod, w, x)
    assert (lim[0, L - 1] > m1[0, L - 1] + 4).all()          # this row forbids the skip
    assert (lim[0, :L - 1] <= m1[0, :L - 1] - 4).all()       # every other row allows it
    plan, ws, out = run(vsa, w, x, seq_tiles)
    ref = compare_to_oracle(oracle_mod, w, x, out)
    assert np.abs(f64(out)[0, L - 1] - ref.out[0, L - 1]).max() <= MAX_ABS
    plan.destroy()
