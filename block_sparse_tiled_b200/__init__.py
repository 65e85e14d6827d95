"""Python binding of libvsa, the VSA-H3 block-sparse attention forward for B200.

Argument marshalling only: every step of the forward runs in the CUDA kernels
of ``libvsa.so`` (built from ``csrc/`` for sm_100a).  PyTorch supplies device
memory and streams.  There is no fallback: if the library is missing or the
device is not sm_100, the calls raise.

The functions mirror the C ABI in ``include/vsa.h``:

    vsa_plan_tiles      S1  tile plan (host) + upload of the tile tables
    vsa_gather_tiles    S2  sequence order -> tile order (optionally pooled)
    vsa_pool_and_score  S3  pooled tiles and fp32 pooled tile scores
    vsa_topk_select     S4  top-k key tiles per video query tile + compression
    vsa_sparse_attn_fwd S5  block-sparse attention + gated epilogue
    vsa_forward             S2..S5 in one call
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvsa.so")

VSA_OK = 0
STATUS_NAMES = {
    0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_SHAPE", 3: "VSA_ERR_UNSUPPORTED",
    4: "VSA_ERR_WORKSPACE", 5: "VSA_ERR_CUDA", 6: "VSA_ERR_TIMEOUT", 7: "VSA_ERR_DEVICE",
}

# every symbol include/vsa.h declares
EXPORTED = (
    "vsa_plan_tiles", "vsa_plan_info", "vsa_plan_tables", "vsa_plan_query", "vsa_plan_tables_host",
    "vsa_plan_destroy",
    "vsa_gather_tiles", "vsa_pool_and_score", "vsa_topk_select", "vsa_sparse_attn_fwd", "vsa_forward",
    "vsa_forward_noalloc", "vsa_forward_host", "vsa_forward_host_workspace", "vsa_forward_parts", "vsa_wait_selftest",
    "vsa_plan_workspace", "vsa_device_status", "vsa_last_error", "vsa_version",
)


class VsaError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")


class Geometry(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("n_segments", ctypes.c_int32), ("segment_len", ctypes.POINTER(ctypes.c_int32)),
        ("token_tags", ctypes.POINTER(ctypes.c_int32)), ("seq_len", ctypes.c_int64),
        ("video_tag", ctypes.c_int32),
        ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
        ("tile_size", ctypes.c_int32), ("sparsity", ctypes.c_double), ("softmax_scale", ctypes.c_float),
        ("gate_per_channel", ctypes.c_int32), ("seq_tiles", ctypes.c_int32), ("qk_fp8", ctypes.c_int32),
        ("cube_t", ctypes.c_int32), ("cube_h", ctypes.c_int32), ("cube_w", ctypes.c_int32),
        ("segment_reference", ctypes.POINTER(ctypes.c_int32)), ("reference_keep", ctypes.c_double),
    ]


class SeqParts(ctypes.Structure):
    _fields_ = [
        ("nparts", ctypes.c_int32), ("tokens_per_part", ctypes.c_int64), ("heads_total", ctypes.c_int32),
        ("head_offset", ctypes.c_int32),
        ("q", ctypes.POINTER(ctypes.c_void_p)), ("k", ctypes.POINTER(ctypes.c_void_p)),
        ("v", ctypes.POINTER(ctypes.c_void_p)), ("gate", ctypes.POINTER(ctypes.c_void_p)),
        ("out", ctypes.POINTER(ctypes.c_void_p)),
    ]


class PlanDims(ctypes.Structure):
    _fields_ = [
        ("n_tiles", ctypes.c_int32), ("n_prefix_tiles", ctypes.c_int32), ("n_video_tiles", ctypes.c_int32),
        ("topk", ctypes.c_int32), ("seq_len", ctypes.c_int64), ("softmax_scale", ctypes.c_float),
        ("workspace_bytes", ctypes.c_size_t), ("selected_pairs", ctypes.c_int64), ("tile_size", ctypes.c_int32),
        ("n_ref_tiles", ctypes.c_int32), ("ref_topk", ctypes.c_int32),
    ]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t)
                for n in ("q_t", "k_t", "v_t", "q_s", "k_s", "q_n", "kv_max", "pq", "pk", "pv", "scores", "idx", "o_c",
                          "q_c", "k_c", "q_n8", "kv_max8", "k_sum", "k_mu", "total")]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libvsa.so; raise if it is missing (no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libvsa.so not found at {path}; build it with `python -m block_sparse_tiled_b200.build`")
    lib = ctypes.CDLL(path)
    P, st = ctypes.c_void_p, ctypes.c_int
    lib.vsa_last_error.restype = ctypes.c_char_p
    lib.vsa_version.restype = ctypes.c_char_p
    lib.vsa_plan_query.argtypes = [ctypes.POINTER(Geometry), ctypes.POINTER(PlanDims)]
    lib.vsa_plan_tables_host.argtypes = [ctypes.POINTER(Geometry), P, P]
    lib.vsa_plan_tiles.argtypes = [ctypes.POINTER(Geometry), P, ctypes.POINTER(P)]
    lib.vsa_plan_info.argtypes = [P, ctypes.POINTER(PlanDims)]
    lib.vsa_plan_tables.argtypes = [P, P, P]
    lib.vsa_plan_workspace.argtypes = [P, ctypes.POINTER(WorkspaceLayout)]
    lib.vsa_plan_destroy.argtypes = [P]
    lib.vsa_gather_tiles.argtypes = [P] * 13
    lib.vsa_pool_and_score.argtypes = [P] * 9
    lib.vsa_topk_select.argtypes = [P] * 6
    lib.vsa_sparse_attn_fwd.argtypes = [P] * 11
    lib.vsa_forward.argtypes = [P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.vsa_forward_noalloc.argtypes = [P] * 7
    lib.vsa_forward_host_workspace.argtypes = [P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.vsa_forward_host.argtypes = [P, P, P, P, P, P, ctypes.c_int32, P, ctypes.c_size_t, P]
    lib.vsa_forward_parts.argtypes = [P, ctypes.POINTER(SeqParts), P, ctypes.c_size_t, P]
    lib.vsa_wait_selftest.argtypes = [P, ctypes.c_int64, P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
    lib.vsa_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
    for name in EXPORTED:
        if name not in ("vsa_last_error", "vsa_version"):
            getattr(lib, name).restype = st
    _lib = lib
    return lib


def _check(rc: int, where: str):
    if rc != VSA_OK:
        raise VsaError(rc, where, load_library().vsa_last_error().decode())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t, dtype=None, name="tensor"):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _qk_mode(qk_fp8) -> int:
    """qk_fp8: False / True (8-bit Q/K logits for every query tile) / "prefix" (for the dense prefix query
    tiles only, the pages' split) / "fp4" (the split, and FP4 Q and smoothed FP4 K for the video query
    tiles) -> the geometry's 0 / 1 / 2 / 3."""
    if isinstance(qk_fp8, str):
        modes = {"prefix": 2, "fp4": 3}
        if qk_fp8 not in modes:
            raise ValueError(f"qk_fp8 must be a bool, 'prefix' or 'fp4', got {qk_fp8!r}")
        return modes[qk_fp8]
    return int(bool(qk_fp8))


def make_geometry(batch, heads, head_dim, segments=(), grid=(0, 0, 0), sparsity=0.0, softmax_scale=0.0,
                  token_tags=None, video_tag=0, tile_size=64, gate_per_channel=False, seq_tiles=False, qk_fp8=False,
                  cube=None, ref_segments=None, ref_keep=0.0):
    """Build the ``vsa_geometry`` struct; returns (struct, keep-alive buffers).  cube: (t, h, w) of a
    video tile, None for the default (4x4x4 for 64-token tiles, 4x4x8 for 128).  ref_segments: one
    flag per prefix segment marking reference segments, with their keep ratio ref_keep."""
    g = Geometry()
    g.batch, g.heads, g.head_dim = int(batch), int(heads), int(head_dim)
    keep = []
    if token_tags is not None:
        tags = (ctypes.c_int32 * len(token_tags))(*[int(t) for t in token_tags])
        keep.append(tags)
        g.token_tags = ctypes.cast(tags, ctypes.POINTER(ctypes.c_int32))
        g.seq_len = len(token_tags)
        g.video_tag = int(video_tag)
        g.n_segments = 0
    else:
        seg = (ctypes.c_int32 * max(1, len(segments)))(*[int(s) for s in segments])
        keep.append(seg)
        g.segment_len = ctypes.cast(seg, ctypes.POINTER(ctypes.c_int32))
        g.n_segments = len(segments)
        g.seq_len = 0
    g.grid_t, g.grid_h, g.grid_w = (int(x) for x in grid)
    g.tile_size = int(tile_size)
    g.sparsity = float(sparsity)
    g.softmax_scale = float(softmax_scale)
    g.gate_per_channel = int(bool(gate_per_channel))
    g.seq_tiles = int(bool(seq_tiles))
    g.qk_fp8 = _qk_mode(qk_fp8)
    g.cube_t, g.cube_h, g.cube_w = (int(c) for c in (cube or (0, 0, 0)))
    if ref_segments is not None:
        flags = (ctypes.c_int32 * max(1, len(ref_segments)))(*[int(f) for f in ref_segments])
        keep.append(flags)
        g.segment_reference = ctypes.cast(flags, ctypes.POINTER(ctypes.c_int32))
        g.reference_keep = float(ref_keep)
    return g, keep


def vsa_plan_query(**kw) -> dict:
    """Resolve sizes without touching a device."""
    g, keep = make_geometry(**kw)
    d = PlanDims()
    _check(load_library().vsa_plan_query(ctypes.byref(g), ctypes.byref(d)), "vsa_plan_query")
    return d.as_dict()


def vsa_plan_tables_host(**kw):
    """Host-only token table of a geometry: (tile_token [n_tiles, tile_size], tile_valid [n_tiles])."""
    import numpy as np

    d = vsa_plan_query(**kw)
    g, keep = make_geometry(**kw)
    n = d["n_tiles"]
    tok = np.empty((max(n, 1), d["tile_size"]), np.int32)
    val = np.empty((max(n, 1),), np.int32)
    _check(load_library().vsa_plan_tables_host(ctypes.byref(g), tok.ctypes.data_as(ctypes.c_void_p),
                                               val.ctypes.data_as(ctypes.c_void_p)), "vsa_plan_tables_host")
    return tok[:n], val[:n]


class Plan:
    """Owns a ``vsa_plan`` handle (the device tile tables of one geometry)."""

    def __init__(self, handle, geometry_kwargs):
        self._h = handle
        self.geometry = dict(geometry_kwargs)
        d = PlanDims()
        _check(load_library().vsa_plan_info(self._h, ctypes.byref(d)), "vsa_plan_info")
        self.dims = d.as_dict()
        ws = WorkspaceLayout()
        _check(load_library().vsa_plan_workspace(self._h, ctypes.byref(ws)), "vsa_plan_workspace")
        self.workspace_layout = {f: getattr(ws, f) for f, _ in WorkspaceLayout._fields_}

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("plan destroyed")
        return self._h

    def tables(self):
        import numpy as np

        n = self.dims["n_tiles"]
        tok = np.empty((max(n, 1), self.dims["tile_size"]), np.int32)
        val = np.empty((max(n, 1),), np.int32)
        _check(load_library().vsa_plan_tables(self.handle, tok.ctypes.data_as(ctypes.c_void_p),
                                              val.ctypes.data_as(ctypes.c_void_p)), "vsa_plan_tables")
        return tok[:n], val[:n]

    def destroy(self):
        if self._h is not None:
            load_library().vsa_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def vsa_plan_tiles(batch, heads, head_dim, segments=(), grid=(0, 0, 0), sparsity=0.0, softmax_scale=0.0,
                   token_tags=None, video_tag=0, tile_size=64, gate_per_channel=False, seq_tiles=False,
                   qk_fp8=False, cube=None, ref_segments=None, ref_keep=0.0, stream=None) -> Plan:
    kw = dict(batch=batch, heads=heads, head_dim=head_dim, segments=tuple(segments), grid=tuple(grid),
              sparsity=sparsity, softmax_scale=softmax_scale, token_tags=token_tags, video_tag=video_tag,
              tile_size=tile_size, gate_per_channel=bool(gate_per_channel), seq_tiles=bool(seq_tiles),
              qk_fp8=qk_fp8 if isinstance(qk_fp8, str) else bool(qk_fp8), cube=None if cube is None else tuple(cube),
              ref_segments=None if ref_segments is None else tuple(ref_segments), ref_keep=float(ref_keep))
    g, keep = make_geometry(**kw)
    h = ctypes.c_void_p()
    _check(load_library().vsa_plan_tiles(ctypes.byref(g), _stream(stream), ctypes.byref(h)), "vsa_plan_tiles")
    return Plan(h, kw)


def vsa_gather_tiles(plan, q, k, v, q_t, k_t, v_t, pq=None, pk=None, pv=None, q_norm=None, kv_max=None,
                     stream=None):
    bf, f32 = torch.bfloat16, torch.float32
    _check(load_library().vsa_gather_tiles(
        plan.handle, _ptr(q, bf, "q"), _ptr(k, bf, "k"), _ptr(v, bf, "v"), _ptr(q_t, bf, "q_t"),
        _ptr(k_t, bf, "k_t"), _ptr(v_t, bf, "v_t"), _ptr(pq, f32, "pq"), _ptr(pk, f32, "pk"), _ptr(pv, f32, "pv"),
        _ptr(q_norm, f32, "q_norm"), _ptr(kv_max, f32, "kv_max"), _stream(stream)), "vsa_gather_tiles")


def vsa_pool_and_score(plan, q_t, k_t, v_t, pq, pk, pv, scores, stream=None):
    bf, f32 = torch.bfloat16, torch.float32
    _check(load_library().vsa_pool_and_score(
        plan.handle, _ptr(q_t, bf, "q_t"), _ptr(k_t, bf, "k_t"), _ptr(v_t, bf, "v_t"), _ptr(pq, f32, "pq"),
        _ptr(pk, f32, "pk"), _ptr(pv, f32, "pv"), _ptr(scores, f32, "scores"), _stream(stream)),
        "vsa_pool_and_score")


def vsa_topk_select(plan, scores, pv, idx, o_c, stream=None):
    f32 = torch.float32
    _check(load_library().vsa_topk_select(
        plan.handle, _ptr(scores, f32, "scores"), _ptr(pv, f32, "pv"), _ptr(idx, torch.int32, "idx"),
        _ptr(o_c, f32, "o_c"), _stream(stream)), "vsa_topk_select")


def vsa_sparse_attn_fwd(plan, q_t, k_t, v_t, idx, o_c, gate, out, q_norm=None, kv_max=None, stream=None):
    bf, f32 = torch.bfloat16, torch.float32
    _check(load_library().vsa_sparse_attn_fwd(
        plan.handle, _ptr(q_t, bf, "q_t"), _ptr(k_t, bf, "k_t"), _ptr(v_t, bf, "v_t"),
        _ptr(idx, torch.int32, "idx"), _ptr(o_c, f32, "o_c"), _ptr(gate, bf, "gate"),
        _ptr(out, bf, "out"), _ptr(q_norm, f32, "q_norm"), _ptr(kv_max, f32, "kv_max"), _stream(stream)),
        "vsa_sparse_attn_fwd")


def alloc_workspace(plan, device=None) -> torch.Tensor:
    """A uint8 device buffer of ``workspace_bytes`` (torch's allocator aligns to >= 256 bytes)."""
    n = max(256, plan.dims["workspace_bytes"])
    return torch.empty(n, dtype=torch.uint8, device=device or torch.device("cuda", torch.cuda.current_device()))


def default_head_chunk(heads: int, head_dim: int = 128) -> int:
    """Heads per chunk of the host pipeline.  Small chunks keep the forward and copy-back of the last
    chunk, which nothing overlaps, short; but each chunk's copies are strided rows of chunk*head_dim
    bf16 values, and rows under 512 bytes copy slowly (measured at 1344x768, 56 heads, D = 128:
    1 head per chunk 104.7 ms, 2: 62.7 ms, 4: 64.2 ms, 8: 67.5 ms, 14: 76.2 ms).  So: the smallest
    chunk with rows of at least 512 bytes, and at most 32 chunks."""
    rows = -(-512 // (2 * head_dim))
    return max(1, min(heads, max(rows, -(-heads // 32))))


def host_workspace_bytes(plan, head_chunk=None) -> int:
    g = plan.geometry
    hc = default_head_chunk(g["heads"], g["head_dim"]) if head_chunk is None else int(head_chunk)
    n = ctypes.c_size_t()
    _check(load_library().vsa_forward_host_workspace(plan.handle, hc, ctypes.byref(n)), "vsa_forward_host_workspace")
    return n.value


def _host_ptr(t, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a CPU tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def vsa_forward_host(plan, q, k, v, gate, out=None, workspace=None, head_chunk=None, stream=None):
    """The whole forward for CPU (ideally pinned) q, k, v, gate; returns the CPU
    output.  The heads run in chunks whose copies overlap the compute of the
    neighbouring chunks (vsa_forward_host).  Without a workspace, one is
    allocated on first use and kept on the plan.  Returns once the stream has
    drained."""
    g = plan.geometry
    hc = default_head_chunk(g["heads"], g["head_dim"]) if head_chunk is None else int(head_chunk)
    need = host_workspace_bytes(plan, hc)
    if workspace is None:
        cached = getattr(plan, "_host_ws", None)
        if cached is None or cached.numel() < need:
            cached = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", torch.cuda.current_device()))
            plan._host_ws = cached
        workspace = cached
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    _check(load_library().vsa_forward_host(
        plan.handle, _host_ptr(q, "q"), _host_ptr(k, "k"), _host_ptr(v, "v"), _host_ptr(gate, "gate"),
        _host_ptr(out, "out"), hc, _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "vsa_forward_host")
    if stream is None:
        torch.cuda.current_stream().synchronize()
    elif isinstance(stream, torch.cuda.Stream):
        stream.synchronize()
    else:
        torch.cuda.synchronize()
    return out


def vsa_forward(plan, q, k, v, gate, out=None, workspace=None, stream=None):
    """The whole forward.  CUDA inputs: runs in place on the stream.  CPU
    inputs (ideally pinned): the head-chunked host pipeline (vsa_forward_host),
    with `workspace` sized by host_workspace_bytes when given."""
    if not q.is_cuda:
        return vsa_forward_host(plan, q, k, v, gate, out=out, workspace=workspace, stream=stream)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(plan, q.device)
    bf = torch.bfloat16
    _check(load_library().vsa_forward(
        plan.handle, _ptr(q, bf, "q"), _ptr(k, bf, "k"), _ptr(v, bf, "v"), _ptr(gate, bf, "gate"),
        _ptr(out, bf, "out"), _ptr(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "vsa_forward")
    return out


MAX_PARTS = 64


def ulysses_partition(seq_len: int, heads: int, world: int, rank: int):
    """Sequence-parallel layout of one rank: (tokens per part, heads of this rank, first head).  Rank r
    holds tokens [r*Ls, (r+1)*Ls) of q/k/v/gate/out and runs the forward for heads [r*Hn, (r+1)*Hn)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if seq_len % world or heads % world:
        raise ValueError(f"the world size {world} must divide the sequence length {seq_len} and the heads {heads}")
    hn = heads // world
    return seq_len // world, hn, rank * hn


def vsa_forward_parts(plan, q_parts, k_parts, v_parts, gate_parts, out_parts, head_offset, workspace=None, stream=None):
    """The forward for this plan's heads over a sequence split into parts (lists of CUDA tensors
    [B, Ls, Htot, D], gate [B, Ls, Htot] or [B, Ls, Htot*D]); parts may be peer mappings of other
    GPUs' buffers.  Writes heads [head_offset, head_offset + H) of every out part."""
    n = len(q_parts)
    if not (len(k_parts) == len(v_parts) == len(gate_parts) == len(out_parts) == n) or not 1 <= n <= MAX_PARTS:
        raise ValueError("q, k, v, gate and out need the same number of parts, at most MAX_PARTS")
    B, Ls, Htot, D = q_parts[0].shape
    if workspace is None:
        workspace = alloc_workspace(plan, q_parts[0].device)
    bf = torch.bfloat16

    def arr(ts, name):
        return (ctypes.c_void_p * n)(*[_ptr(t, bf, f"{name}[{i}]") for i, t in enumerate(ts)])

    keep = [arr(q_parts, "q"), arr(k_parts, "k"), arr(v_parts, "v"), arr(gate_parts, "gate"), arr(out_parts, "out")]
    cast = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))  # noqa: E731
    sp = SeqParts(n, Ls, Htot, int(head_offset), *[cast(a) for a in keep])
    _check(load_library().vsa_forward_parts(plan.handle, ctypes.byref(sp), _ptr(workspace, torch.uint8, "workspace"),
                                            workspace.numel(), _stream(stream)), "vsa_forward_parts")
    return out_parts


NOALLOC_SCRATCH_BYTES = 64 << 20


def vsa_forward_noalloc(plan, q, k, v, gate, out, stream=None):
    """The whole forward with the library's static device scratch instead of a
    caller workspace (for callers that cannot allocate device memory).  Calls
    on one device share that scratch: do not let them overlap on the GPU."""
    bf = torch.bfloat16
    _check(load_library().vsa_forward_noalloc(
        plan.handle, _ptr(q, bf, "q"), _ptr(k, bf, "k"), _ptr(v, bf, "v"), _ptr(gate, bf, "gate"),
        _ptr(out, bf, "out"), _stream(stream)), "vsa_forward_noalloc")
    return out


def wait_selftest(plan, timeout_ns=50_000_000, stream=None):
    """Run the bounded-wait self-test; returns the (code, site) it recorded."""
    code, where = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().vsa_wait_selftest(plan.handle, int(timeout_ns), _stream(stream), ctypes.byref(code),
                                            ctypes.byref(where)), "vsa_wait_selftest")
    return code.value, where.value


def device_status(plan, stream=None):
    code, where = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().vsa_device_status(plan.handle, _stream(stream), ctypes.byref(code), ctypes.byref(where)),
           "vsa_device_status")
    return code.value, where.value


def workspace_views(plan, workspace):
    """Typed views of vsa_forward's intermediates inside ``workspace`` (no tile-order views for a plan
    with seq_tiles, whose workspace holds none).  With qk_fp8, q_t and k_t are the E4M3 codes
    [B, H, n_t, tile, 128] (uint8) and q_s, k_s their row scales [B, H, n_t, tile].  q_n holds the
    query row norms [B, H, n_t, tile] (with qk_fp8 of the dequantised rows) and kv_max the (b, h)
    maxima of key norm and |v| [B, H, 2] (the attention's overflow bound).  With qk_fp8="prefix" q_t and
    k_t are the bf16 copies, q_c and k_c the codes, q_s and k_s their scales, and q_n8, kv_max8 the
    statistics of the dequantised rows.  With qk_fp8="fp4" the same, except that q_t's video query tiles
    and k_t's valid rows hold their FP4 roundings (bf16 numbers; keys after smoothing), k_sum the binary64
    key column sums [B, H, D] and k_mu the key means [B, H, D]; q_n and kv_max describe the rounded copies."""
    d, g = plan.dims, plan.geometry
    B, H, D, n_t, V, k = g["batch"], g["heads"], g["head_dim"], d["n_tiles"], d["n_video_tiles"], d["topk"]
    lay = plan.workspace_layout
    seq = bool(g.get("seq_tiles", False))
    mode = _qk_mode(g.get("qk_fp8", False))
    f8, split = mode == 1, mode >= 2
    T = d["tile_size"]  # rows per tile

    def view(off, n, dtype, shape):
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return workspace[off:off + nbytes].view(dtype).view(*shape)

    def tiles(name):
        return None if seq else view(lay[name], B * H * n_t * T * D, torch.bfloat16, (B, H, n_t, T, D))

    def codes(name):
        return view(lay[name], B * H * n_t * T * 128, torch.uint8, (B, H, n_t, T, 128))

    def row_scales(name):
        return view(lay[name], B * H * n_t * T, torch.float32, (B, H, n_t, T)) if (f8 or split) else None

    extra = {} if not split else {
        "q_c": codes("q_c"), "k_c": codes("k_c"),
        "q_n8": view(lay["q_n8"], B * H * n_t * T, torch.float32, (B, H, n_t, T)),
        "kv_max8": view(lay["kv_max8"], B * H * 2, torch.float32, (B, H, 2)),
    }
    if mode == 3:
        extra["k_sum"] = view(lay["k_sum"], B * H * D, torch.float64, (B, H, D))
        extra["k_mu"] = view(lay["k_mu"], B * H * D, torch.float32, (B, H, D))
    return {
        **extra,
        "q_t": codes("q_t") if f8 else tiles("q_t"),
        "k_t": codes("k_t") if f8 else tiles("k_t"),
        "v_t": tiles("v_t"),
        "q_s": row_scales("q_s"),
        "k_s": row_scales("k_s"),
        "q_n": view(lay["q_n"], B * H * n_t * T, torch.float32, (B, H, n_t, T)),
        "kv_max": view(lay["kv_max"], B * H * 2, torch.float32, (B, H, 2)),
        "pq": view(lay["pq"], B * H * n_t * D, torch.float32, (B, H, n_t, D)),
        "pk": view(lay["pk"], B * H * n_t * D, torch.float32, (B, H, n_t, D)),
        "pv": view(lay["pv"], B * H * n_t * D, torch.float32, (B, H, n_t, D)),
        "scores": view(lay["scores"], B * H * n_t * n_t, torch.float32, (B, H, n_t, n_t)),
        "idx": view(lay["idx"], B * H * V * (k + d["ref_topk"]), torch.int32, (B, H, V, k + d["ref_topk"])),
        "o_c": view(lay["o_c"], B * H * n_t * D, torch.float32, (B, H, n_t, D)),
    }
