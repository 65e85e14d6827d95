"""The gate-all-zero fast path of vsa_forward.

When every gate is zero the compression term adds nothing: a device-side check
sets a flag, the compression kernel returns at once and the epilogue leaves the
o_c term out, so the output is the fine branch.  The checks: an all-zero gate
(and one of -0 values) gives the oracle's output and leaves the workspace's o_c
untouched (pre-filled with NaN); a gate whose only nonzero value is its last
element still takes the full path; the host pipeline, whose head slices scan
an unaligned part of the whole gate, agrees with the device forward."""
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

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def plan_for(vsa, w):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, gate_per_channel=w.gate_per_channel)


def oracle_out(oracle_mod, w, x):
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    return oracle_mod.forward(b["q"], b["k"], b["v"], b["gate"], w.segments, w.grid, w.sparsity)


def run(vsa, plan, x):
    ws = vsa.alloc_workspace(plan)
    views = vsa.workspace_views(plan, ws)
    views["o_c"].fill_(float("nan"))
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    return out, views


def close(out, ref):
    g = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(g - ref)
    assert np.isfinite(g).all()
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


@pytest.mark.parametrize("name,pc,negzero", [("small", False, False), ("small", True, False), ("tiny", False, True)])
def test_zero_gate_skips_compression(vsa, oracle_mod, name, pc, negzero):
    w = dataclasses.replace(synth.workload(name), gate_per_channel=pc, name=f"{name}_zg")
    x = synth.make_inputs(w, seed=11, device="cuda")
    x["gate"] = torch.full_like(x["gate"], -0.0 if negzero else 0.0)
    ref = oracle_out(oracle_mod, w, x)
    assert (ref.out == ref.o_f).all()
    plan = plan_for(vsa, w)
    out, views = run(vsa, plan, x)
    close(out, ref.out)
    assert torch.isnan(views["o_c"]).all()  # the compression kernel did not run
    plan.destroy()


@pytest.mark.parametrize("pc", [False, True])
def test_last_gate_element_nonzero_keeps_branch(vsa, oracle_mod, pc):
    w = dataclasses.replace(synth.workload("small"), gate_per_channel=pc, name="small_lastg")
    x = synth.make_inputs(w, seed=12, device="cuda")
    g = torch.zeros_like(x["gate"])
    g.view(-1)[-1] = 0.5
    x["gate"] = g
    ref = oracle_out(oracle_mod, w, x)
    plan = plan_for(vsa, w)
    out, views = run(vsa, plan, x)
    close(out, ref.out)
    oc = views["o_c"].cpu().numpy().astype(np.float64)
    assert np.abs(oc - ref.o_c).max() <= 1e-5 * max(1.0, np.abs(ref.o_c).max())
    plan.destroy()


@pytest.mark.parametrize("pc", [False, True])
def test_zero_gate_host_pipeline(vsa, oracle_mod, pc):
    w = dataclasses.replace(synth.workload("small"), gate_per_channel=pc, name="small_zg_host")
    x = synth.make_inputs(w, seed=13, device="cuda")
    x["gate"] = torch.zeros_like(x["gate"])
    # one nonzero gate value in head 5 only: chunks without it skip the branch, the one with it does not
    g = x["gate"].view(w.batch, w.seq_len, w.heads, -1)
    g[0, 100, 5, 0] = 0.25
    plan = plan_for(vsa, w)
    dev_out, _ = run(vsa, plan, x)
    hx = {n: x[n].cpu().pin_memory() for n in ("q", "k", "v", "gate")}
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=3)
    assert torch.equal(out, dev_out.cpu())
    close(dev_out, oracle_out(oracle_mod, w, x).out)
    plan.destroy()
