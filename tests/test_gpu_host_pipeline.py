"""The host-memory entry point (vsa_forward_host): heads in chunks, copies on
their own streams overlapping the forward of neighbouring chunks.

Every head's forward is independent of the other heads (pooling, scores,
top-k, compression and the attention items all work per (b, h)), so the
chunked result must be bit-identical to vsa_forward on the same inputs --
except on the prefix query rows of 64-token tiles where a chunk has too few
heads for the pair kernel and the whole forward enough: those rows run on the
video attention kernel in the chunks and must agree within the output
tolerance.
The cases cover a chunk that divides the heads, one that leaves a remainder
chunk (a second head-slice plan), one chunk holding every head, the default
(the smallest chunk with 512-byte copy rows), pageable host memory, a second call reusing the pipeline,
and the argument errors."""
import ctypes

import pytest
import torch

import synth
from conftest import assert_routes_agree

pytestmark = pytest.mark.gpu


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
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, gate_per_channel=w.gate_per_channel, seq_tiles=seq_tiles)


def device_reference(vsa, plan, x):
    out = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=vsa.alloc_workspace(plan))
    torch.cuda.synchronize()
    return out.cpu()


def host_copies(x, pinned=True):
    h = {}
    for n in ("q", "k", "v", "gate"):
        h[n] = torch.empty(x[n].shape, dtype=x[n].dtype, pin_memory=pinned)
        h[n].copy_(x[n])
    return h


@pytest.mark.parametrize("name,chunk", [("small", 3), ("small", 4), ("small", 8), ("small", None), ("tiny", 1),
                                        ("480p", None), ("480p", 13)])
def test_host_pipeline_matches_device_forward(vsa, name, chunk):
    w = synth.workload(name)
    x = synth.make_inputs(w, seed=5, device="cuda")
    plan = plan_for(vsa, w)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x)
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=chunk)
    assert not out.is_cuda
    hc = chunk or vsa.default_head_chunk(w.heads, w.head_dim)
    assert_routes_agree(w, out, ref, hc)
    assert vsa.device_status(plan) == (0, 0)
    # a second call reuses the plan's pipeline and staging workspace
    first = out.clone()
    out.zero_()
    vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], out=out, head_chunk=chunk)
    assert torch.equal(out, first)
    plan.destroy()


def test_host_pipeline_1344x768_default_chunks(vsa):
    """The bench workload in the e2e configuration (28 chunks of 2 heads)."""
    w = synth.workload("768p_s0.9")
    x = synth.make_inputs(w, seed=0, device="cuda")
    plan = plan_for(vsa, w)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x)
    del x
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"])
    assert_routes_agree(w, out, ref, vsa.default_head_chunk(w.heads, w.head_dim))
    assert vsa.device_status(plan) == (0, 0)
    plan.destroy()


def test_host_pipeline_pageable_memory(vsa):
    w = synth.workload("small")
    x = synth.make_inputs(w, seed=6, device="cuda")
    plan = plan_for(vsa, w)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x, pinned=False)
    out = vsa.vsa_forward(plan, hx["q"], hx["k"], hx["v"], hx["gate"])  # CPU inputs take the host pipeline
    assert torch.equal(out, ref)
    plan.destroy()


def test_host_pipeline_errors(vsa):
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=1, device="cuda")
    plan = plan_for(vsa, w)
    hx = host_copies(x)
    lib = vsa.load_library()
    n = ctypes.c_size_t()
    assert lib.vsa_forward_host_workspace(plan.handle, 0, ctypes.byref(n)) == 1  # VSA_ERR_INVALID_ARG
    assert lib.vsa_forward_host_workspace(plan.handle, w.heads + 1, ctypes.byref(n)) == 1
    need = vsa.host_workspace_bytes(plan, 1)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], workspace=small, head_chunk=1)
    assert e.value.status == 4  # VSA_ERR_WORKSPACE
    with pytest.raises(ValueError):
        vsa.vsa_forward_host(plan, x["q"], hx["k"], hx["v"], hx["gate"], head_chunk=1)  # a device tensor
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=1)
    assert torch.equal(out, device_reference(vsa, plan, x))
    plan.destroy()


def test_host_pipeline_head_dim_96(vsa):
    import dataclasses

    w = dataclasses.replace(synth.workload("small"), head_dim=96, name="small_d96")
    x = synth.make_inputs(w, seed=8, device="cuda")
    plan = plan_for(vsa, w)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x)
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=3)
    assert torch.equal(out, ref)
    plan.destroy()


def test_host_pipeline_gate_per_channel(vsa):
    import dataclasses

    w = dataclasses.replace(synth.workload("small"), gate_per_channel=True, name="small_pc")
    x = synth.make_inputs(w, seed=9, device="cuda")
    plan = plan_for(vsa, w)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x)
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=3)
    assert torch.equal(out, ref)
    plan.destroy()


def test_host_pipeline_seq_tiles(vsa):
    """A seq_tiles plan through the host pipeline: its head-slice plans read sequence order too."""
    w = synth.workload("480p")
    x = synth.make_inputs(w, seed=10, device="cuda")
    plan = plan_for(vsa, w, seq_tiles=True)
    ref = device_reference(vsa, plan, x)
    hx = host_copies(x)
    out = vsa.vsa_forward_host(plan, hx["q"], hx["k"], hx["v"], hx["gate"], head_chunk=13)
    assert torch.equal(out, ref)
    plan.destroy()
