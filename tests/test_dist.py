"""Multi-rank bench logic on CPU (gloo, world size 2): the max-over-ranks
timing reduction and barrier, and the reference arm under torchrun, where
rank 0 alone runs and prints one JSON line and the other rank exits 0."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        q.put((rank, bench.max_over_ranks(1.5 + rank, world)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 2.5), (1, 2.5)]


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny", "--ref-every", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT,
                       env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny"


MODES = {"bf16": {}, "prefix": {"qk8": "prefix"}, "fp4": {"qk8": "prefix", "fp4": True}}


def _ulysses_worker(rank, world, port, q, mode="bf16"):
    import numpy as np
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import oracle
    import synth
    from block_sparse_tiled_b200 import ulysses_partition

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.workload("tiny")
        x = synth.make_inputs(w, seed=31)
        full = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
        ls, hn, h0 = ulysses_partition(w.seq_len, w.heads, world, rank)
        mine = {n: full[n][:, rank * ls:(rank + 1) * ls] for n in full}  # this rank's token part
        # seq -> head: every rank gets every token part, keeps its head group
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        heads = {n: np.concatenate([p[n] for p in parts], axis=1)[:, :, h0:h0 + hn] for n in mine}
        kw = MODES[mode]
        r = oracle.forward(heads["q"], heads["k"], heads["v"], heads["gate"], w.segments, w.grid, w.sparsity, **kw)
        # head -> seq: every rank gets every head group's output, keeps its token part
        groups = [None] * world
        dist.all_gather_object(groups, (h0, r.out))
        out = np.zeros((w.batch, ls, w.heads, w.head_dim))
        for g0, o in groups:
            out[:, :, g0:g0 + o.shape[2]] = o[:, rank * ls:(rank + 1) * ls]
        whole = oracle.forward(full["q"], full["k"], full["v"], full["gate"], w.segments, w.grid, w.sparsity, **kw)
        q.put((rank, bool(np.array_equal(out, whole.out[:, rank * ls:(rank + 1) * ls]))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", list(MODES))
def test_ulysses_decomposition_gloo(mode):
    """The sequence-parallel decomposition the parts entry point implements (token parts in, head
    groups computed independently, token parts out) reproduces the whole forward: two gloo ranks
    exchange parts with collectives and run the oracle on their head groups.  The precision modes need
    no further exchange either: the 8-bit and FP4 scales are per (token, head) row or block, and the FP4
    key mean is per head over all tokens, which a rank holds once it has its heads."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_worker, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, True), (1, True)]
