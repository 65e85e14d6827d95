"""vsa_forward_parts: the forward over a sequence split by token into parts,
as a sequence-parallel (Ulysses) layout holds it.

On several GPUs each rank's parts are peer mappings and the gather kernel's
loads and the epilogue's stores carry the all-to-all exchanges.  Here every
part lives on one GPU: the ranks' forwards run one after another (no kernel
waits on another), each for its head group over all parts, and the assembled
output must equal vsa_forward on the whole tensors bit for bit (every head's
computation is the same; only where its rows are read from and written to
differs)."""
import dataclasses

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vsa():
    from block_sparse_tiled_b200 import build

    build.build()
    import block_sparse_tiled_b200 as m

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def plan_for(vsa, w, heads=None, **kw):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=heads or w.heads, head_dim=w.head_dim, segments=w.segments,
                              grid=w.grid, sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, **kw)


def split(t, n):
    return [c.contiguous() for c in torch.chunk(t, n, dim=1)]


def run_ranks(vsa, w, x, world):
    L, H = w.seq_len, w.heads
    parts = {n: split(x[n], world) for n in ("q", "k", "v", "gate")}
    out_parts = [torch.full_like(p, float("nan")) for p in parts["q"]]
    for rank in range(world):
        ls, hn, h0 = vsa.ulysses_partition(L, H, world, rank)
        assert ls * world == L and parts["q"][0].shape[1] == ls
        plan = plan_for(vsa, w, heads=hn)
        vsa.vsa_forward_parts(plan, parts["q"], parts["k"], parts["v"], parts["gate"], out_parts, h0)
        torch.cuda.synchronize()
        assert vsa.device_status(plan) == (0, 0)
        plan.destroy()
    return torch.cat(out_parts, dim=1)


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
def test_parts_match_whole_forward(vsa, name, world, over):
    w = dataclasses.replace(synth.workload(name), **over)
    x = synth.make_inputs(w, seed=21, device="cuda")
    ref = reference(vsa, w, x)
    got = run_ranks(vsa, w, x, world)
    assert torch.equal(got, ref)


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
