"""Tie-breaking of the tile selection on the GPU.

The method keeps, for every video query tile, the top-k video key tiles by pooled score ("Mike0021/
FastH3-4step-Preview-VSA", section "Video Sparse Attention is not optional here").  The pages do not
say how equal scores are ordered; the library's rule, like the oracle's, is that the lower tile index
wins, and the kept tiles are listed in ascending order.  Random inputs never produce equal binary32
scores, so these tests build them on purpose and compare the GPU's idx with the oracle's bit for bit:

* scores handed straight to the top-k entry point: rows of all-equal scores, scores drawn from a
  five-value set (with -0.0 and +0.0, which rank equal, and -inf), a tie group straddling the k-th
  place, and a boundary made only of signed zeros;
* whole forwards whose inputs make pooled scores equal: key tiles that are copies of one tile (so
  their score columns are identical for every query tile) and a head whose video key tiles are all
  the same, with 64- and 128-token tiles and through the reference-keep candidate list.

Each case also checks that the tie it is meant to exercise is present in the oracle's scores."""
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


def boundary_ties(S, n_prefix, k, cols=None):
    """Rows of S [B, H, n_t, n_t] (video query rows, over the video key columns or `cols`) whose k-th and
    (k+1)-th largest scores are equal (-0.0 == +0.0)."""
    B, H, n_t, _ = S.shape
    sub = S[:, :, n_prefix:, n_prefix:] if cols is None else S[:, :, n_prefix:, cols]
    if k >= sub.shape[-1]:
        return 0
    srt = -np.sort(-sub.astype(np.float64), axis=-1)
    return int((srt[..., k - 1] == srt[..., k]).sum())


def plan_for(vsa, w):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, tile_size=w.tile, cube=w.cube, ref_segments=w.ref_segments,
                              ref_keep=w.ref_keep)


# ----------------------------------------------------------------------------- top-k entry point


def engineered_scores(n_t, P, k, heads, seed):
    """[1, heads, n_t, n_t] float32 score matrices, one pattern per head (cycled)."""
    rng = np.random.default_rng(seed)
    V = n_t - P
    S = rng.standard_normal((1, heads, n_t, n_t)).astype(np.float32)
    for h in range(heads):
        kind = h % 5
        vid = S[0, h, P:, P:]  # video query rows x video key columns (a view)
        if kind == 0:  # every video score of a row equal: the first k video tiles
            vid[:] = np.float32(0.25)
        elif kind == 1:  # a five-value set: ties everywhere, -0.0 and +0.0 mixed, some -inf
            vals = np.array([-1.0, -0.0, 0.0, 0.5, 1.0], np.float32)
            vid[:] = vals[rng.integers(0, 5, vid.shape)]
            vid[rng.random(vid.shape) < 0.05] = -np.inf
        elif kind == 2:  # a tie group straddling the k-th place in every row
            for r in range(V):
                perm = rng.permutation(V)
                top = max(0, k - 3)
                vid[r, perm[:top]] = np.float32(2.0)
                vid[r, perm[top:top + 7]] = np.float32(1.0)
                vid[r, perm[top + 7:]] = rng.uniform(-1, 0.5, V - top - 7).astype(np.float32)
        elif kind == 3:  # k - 2 distinct positives, every other video score a signed zero
            for r in range(V):
                perm = rng.permutation(V)
                vid[r, :] = np.where(rng.random(V) < 0.5, np.float32(-0.0), np.float32(0.0))
                vid[r, perm[:k - 2]] = np.arange(1, k - 1, dtype=np.float32)
        else:  # duplicated columns: a few score columns copied into others, for every row
            src = rng.integers(0, V, 4)
            for c in range(V):
                if rng.random() < 0.5:
                    vid[:, c] = vid[:, src[c % 4]]
    return S


@pytest.mark.parametrize("segments,grid,sparsity,tile", [
    ((40, 0, 24), (8, 16, 16), 0.8, 64),     # V = 32, topk 7
    ((100,), (8, 8, 12), 0.5, 64),            # V = 12, topk 6
    ((200, 0, 60), (8, 16, 16), 0.9, 128),   # 128-token tiles: V = 16, topk 2
])
def test_topk_entry_point_engineered_ties(vsa, oracle_mod, segments, grid, sparsity, tile):
    w = synth.Workload("ties", 1, 5, 128, tuple(segments), tuple(grid), sparsity, tile=tile)
    plan = plan_for(vsa, w)
    d = plan.dims
    n_t, P, k = d["n_tiles"], d["n_prefix_tiles"], d["topk"]
    V = n_t - P
    S = engineered_scores(n_t, P, k, 5, seed=11)
    assert boundary_ties(S, P, k) > 0
    pv = np.random.default_rng(12).standard_normal((1, 5, n_t, 128)).astype(np.float32)
    idx = torch.full((1, 5, V, k), -7, dtype=torch.int32, device="cuda")
    o_c = torch.empty(1, 5, n_t, 128, dtype=torch.float32, device="cuda")
    vsa.vsa_topk_select(plan, torch.from_numpy(S).cuda(), torch.from_numpy(pv).cuda(), idx, o_c)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    want = oracle_mod.select(S, P, k)
    got = idx.cpu().numpy()
    assert np.array_equal(got, want), np.argwhere(got != want)[:5]
    # the all-equal head keeps the first k video tiles
    assert np.array_equal(got[0, 0], np.broadcast_to(np.arange(P, P + k, dtype=np.int32), (V, k)))
    ref_oc = oracle_mod.compress(S, pv)
    g = o_c.cpu().numpy().astype(np.float64)
    assert np.abs(g - ref_oc).max() <= 1e-5 * max(1.0, np.abs(ref_oc).max())
    plan.destroy()


# ----------------------------------------------------------------------------- whole forward


def tie_inputs(w, seed):
    """Seeded inputs whose pooled key tiles repeat: in head 0 a fifth of the video key tiles (and, with
    reference segments, half the reference tiles) are copies of one tile whose rows carry a large
    offset, so for about half the query tiles that group ranks first and straddles the k-th place; in
    head 1 every video key tile is the same tile, so every row's video scores are equal."""
    import oracle

    x = synth.make_inputs(w, seed=seed, device="cuda")
    geo = oracle.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments)
    P, V = geo.n_prefix, geo.n_video
    full = [i for i in range(P, geo.n_tiles) if geo.tile_valid[i] == w.tile]
    assert len(full) >= 8
    k = x["k"]

    def rows(i):
        return torch.from_numpy(geo.tile_token[i, :geo.tile_valid[i]].astype(np.int64)).cuda()

    src = full[0]
    k[:, rows(src), 0] = (k[:, rows(src), 0].float() + 3.0).to(torch.bfloat16)
    for i in full[1:][::5]:
        k[:, rows(i), 0] = k[:, rows(src), 0]
    for i in full[1:]:
        k[:, rows(i), 1] = k[:, rows(full[0]), 1]
    if geo.is_ref is not None:
        ref = [i for i in range(P) if geo.is_ref[i] and geo.tile_valid[i] == w.tile]
        for i in ref[1::2]:
            k[:, rows(i), 0] = k[:, rows(ref[0]), 0]
    return x, geo


@pytest.mark.parametrize("over", [
    dict(),                                                        # 64-token tiles
    dict(tile=128, segments=(256, 0, 128), grid=(8, 16, 32)),      # 128-token tiles (4x4x8 cubes)
    dict(segments=(40, 640, 24), ref_segments=(False, True, False), ref_keep=0.4),  # reference keep
])
def test_forward_with_repeated_key_tiles(vsa, oracle_mod, over):
    base = dict(name="ties", batch=1, heads=3, head_dim=128, segments=(256, 64, 192), grid=(8, 16, 32),
                sparsity=0.8)
    base.update(over)
    w = synth.Workload(**base)
    x, geo = tie_inputs(w, seed=21)
    xb = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(xb["q"], xb["k"], xb["v"], xb["gate"], w.segments, w.grid, w.sparsity, tile=w.tile,
                             cube=w.cube, ref_segments=w.ref_segments, ref_keep=w.ref_keep)
    k = ref.topk
    assert boundary_ties(ref.S[:, :1], geo.n_prefix, k) > 0        # head 0: the copied group straddles k
    assert boundary_ties(ref.S[:, 1:2], geo.n_prefix, k) == geo.n_video  # head 1: every row
    if geo.is_ref is not None:
        refcols = np.flatnonzero(geo.is_ref)
        kr = oracle_mod.ref_count(w.ref_keep, len(refcols))
        assert boundary_ties(ref.S[:, :1], geo.n_prefix, kr, cols=refcols) > 0
    plan = plan_for(vsa, w)
    ws = vsa.alloc_workspace(plan)
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    views = vsa.workspace_views(plan, ws)
    assert np.array_equal(views["scores"].cpu().numpy(), ref.S)
    got = views["idx"].cpu().numpy()
    assert np.array_equal(got, ref.idx), np.argwhere(got != ref.idx)[:5]
    g = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref.out)
    assert np.isfinite(g).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    plan.destroy()
