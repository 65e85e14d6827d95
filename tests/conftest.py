import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle


def prefix_on_pair_kernel(w, heads=None):
    """Whether a forward over `heads` heads of workload w (64-token tiles) runs its prefix query row blocks
    on the pair kernel: the library sends them there when their pairs, B * heads * ceil(P / 2), fill the
    GPU's SMs, and otherwise leaves them to the video attention kernel's item schedule.  With 128-token
    tiles every query tile runs on the pair kernel whatever the head count."""
    import oracle
    import torch

    if w.tile != 64:
        return True
    P = oracle.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments).n_prefix
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return P > 0 and w.batch * (heads or w.heads) * ((P + 1) // 2) >= sms


def prefix_token_mask(w):
    """[L] bool: the tokens of w's prefix query tiles."""
    import numpy as np
    import oracle

    geo = oracle.geometry(w.segments, w.grid, tile=w.tile, cube=w.cube, ref_segments=w.ref_segments)
    m = np.zeros(w.seq_len, bool)
    for i in range(geo.n_prefix):
        m[geo.tile_token[i, :geo.tile_valid[i]]] = True
    return m


def assert_routes_agree(w, got, ref, heads_got, heads_ref=None, max_abs=4e-2, mean_abs=4e-3):
    """Outputs [B, L, H, D] of two routes over the same inputs: bit-identical where both run the same
    kernels on the same items (always the video query rows; the prefix rows when both routes put them on
    the same attention kernel).  On prefix rows that one route runs on the pair kernel and the other on the
    video kernel, each is held to max-abs 2e-2 / mean-abs 2e-3 against the oracle elsewhere, so the two
    may differ by twice that (dense rows over every key of 1344x768 come within 0.012 of the oracle with
    either kernel)."""
    import torch

    if prefix_on_pair_kernel(w, heads_got) == prefix_on_pair_kernel(w, heads_ref):
        assert torch.equal(got, ref)
        return
    pre = torch.from_numpy(prefix_token_mask(w)).to(got.device)
    assert torch.equal(got[:, ~pre], ref[:, ~pre])
    d = (got[:, pre].float() - ref[:, pre].float()).abs()
    assert torch.isfinite(got[:, pre].float()).all()
    assert d.max().item() <= max_abs and d.mean().item() <= mean_abs, (d.max().item(), d.mean().item())
