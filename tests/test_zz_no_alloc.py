"""vsa_forward_noalloc: the whole forward for callers that cannot allocate
device memory (its scratch is a static array inside libvsa).  Checked through
the C ABI against vsa_forward with a caller workspace, on two calls in a row
with different inputs, so the second call runs over the first call's leftover
scratch contents."""
import pytest
import torch

import synth

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


def _plan(vsa, w):
    return vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity)


def test_noalloc_matches_forward_on_two_calls(vsa):
    w = synth.workload("small")
    plan = _plan(vsa, w)
    assert plan.dims["workspace_bytes"] <= vsa.NOALLOC_SCRATCH_BYTES
    ws = vsa.alloc_workspace(plan)
    for seed in (0, 1):
        x = synth.make_inputs(w, seed=seed, device="cuda")
        ref = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=ws)
        out = torch.full_like(x["q"], float("nan"))
        vsa.vsa_forward_noalloc(plan, x["q"], x["k"], x["v"], x["gate"], out)
        torch.cuda.synchronize()
        assert vsa.device_status(plan) == (0, 0)
        # the same kernels on the same plan: bit-identical, so leftover scratch from the first call would show
        assert torch.equal(out, ref), seed
    plan.destroy()


def test_noalloc_rejects_oversized_geometry(vsa):
    w = synth.workload("480p")
    plan = _plan(vsa, w)
    assert plan.dims["workspace_bytes"] > vsa.NOALLOC_SCRATCH_BYTES
    x = {n: torch.zeros(1, dtype=torch.bfloat16, device="cuda").expand(16).contiguous() for n in "qkv"}
    with pytest.raises(vsa.VsaError) as e:
        vsa.vsa_forward_noalloc(plan, x["q"], x["k"], x["v"], x["q"], x["q"])
    assert vsa.STATUS_NAMES[e.value.status] == "VSA_ERR_WORKSPACE"
    assert "static scratch" in str(e.value)
    plan.destroy()


def test_noalloc_480p_with_seq_tiles(vsa):
    """A seq_tiles plan needs no tile-order copies, so the 480p-shaped problem (0.69 GB of workspace
    with copies) fits the 64 MiB static scratch; the result is bit-identical to vsa_forward with the
    same plan."""
    w = synth.workload("480p")
    plan = vsa.vsa_plan_tiles(batch=w.batch, heads=w.heads, head_dim=w.head_dim, segments=w.segments, grid=w.grid,
                              sparsity=w.sparsity, seq_tiles=True)
    assert plan.dims["workspace_bytes"] <= vsa.NOALLOC_SCRATCH_BYTES
    x = synth.make_inputs(w, seed=3, device="cuda")
    ref = vsa.vsa_forward(plan, x["q"], x["k"], x["v"], x["gate"], workspace=vsa.alloc_workspace(plan))
    out = torch.full_like(x["q"], float("nan"))
    vsa.vsa_forward_noalloc(plan, x["q"], x["k"], x["v"], x["gate"], out)
    torch.cuda.synchronize()
    assert vsa.device_status(plan) == (0, 0)
    assert torch.equal(out, ref)
    plan.destroy()
