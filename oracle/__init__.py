"""VSA-H3 forward -- plain CPU oracle (ctypes wrapper around ``oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import this package.  The
CUDA library never links or calls it, and it shares no code with that library.

The C file states the method and every reading of the pages it takes.  This
wrapper only marshals numpy arrays and runs whole-forward compositions in the
order the method states them:

    geometry -> pool(q, k, v) -> scores -> top-k -> compression, fine -> output

Parity unpinned: the compression key scope (all tiles, reading R9) and the
compression on prefix query rows (reading R10) follow a reading, not a printed
value; nothing on the pages fixes them.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import time
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        lib.vsa_oracle_geometry.argtypes = [i32, P, i32, i32, i32, i32, i32, i32, i32, P, P, P]
        lib.vsa_oracle_tiles.argtypes = [i32, P, i32, i32, i32, i32, i32, i32, i32, P, P]
        lib.vsa_oracle_topk_count.argtypes = [f64, i32]
        lib.vsa_oracle_topk_count.restype = i32
        lib.vsa_oracle_pool.argtypes = [P, i32, i64, i32, i32, i32, i32, P, P, P]
        lib.vsa_oracle_scores.argtypes = [P, P, i32, i32, i32, f32, P]
        lib.vsa_oracle_select.argtypes = [P, i32, i32, i32, i32, P]
        lib.vsa_oracle_compress.argtypes = [P, P, i32, i32, i32, P]
        lib.vsa_oracle_fine.argtypes = [P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, i32, P, i32, i32, P, P, P,
                                        f64, P, P]
        lib.vsa_oracle_fine_tiles.argtypes = [P, P, P, P, P, P, P, i32, i64, i32, i32, i32, i32, i32, P, i32, i32, P,
                                              P, P, f64, i32, P, P]
        lib.vsa_oracle_select_ref.argtypes = [P, i32, i32, i32, P, i32, i32, P]
        lib.vsa_oracle_ref_count.argtypes = [f64, i32]
        lib.vsa_oracle_ref_count.restype = i32
        lib.vsa_oracle_e4m3_value.argtypes = [i32]
        lib.vsa_oracle_e4m3_value.restype = f64
        lib.vsa_oracle_e4m3_round.argtypes = [f32]
        lib.vsa_oracle_e4m3_round.restype = i32
        lib.vsa_oracle_e4m3_round_array.argtypes = [P, i64, P]
        lib.vsa_oracle_quant_e4m3.argtypes = [P, i64, i32, P, P]
        lib.vsa_oracle_e2m1_value.argtypes = [i32]
        lib.vsa_oracle_e2m1_value.restype = f64
        lib.vsa_oracle_e2m1_round.argtypes = [f32]
        lib.vsa_oracle_e2m1_round.restype = i32
        lib.vsa_oracle_e2m1_round_array.argtypes = [P, i64, P]
        lib.vsa_oracle_quant_fp4.argtypes = [P, i64, i32, P, P]
        lib.vsa_oracle_smooth_keys.argtypes = [P, i64, i64, i32, i32, P, P]
        lib.vsa_oracle_fine_masked.argtypes = [P, P, P, i32, i64, i32, i32, i32, i32, i32, P, i32, i32, P, P, P, f64,
                                               P]
        lib.vsa_oracle_output.argtypes = [P, P, P, i32, i32, i64, i32, i32, i32, i32, P, P, P, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


@dataclass
class Geometry:
    """The oracle's own tiling of one packed sequence."""

    segments: tuple
    grid: tuple
    n_tiles: int
    n_prefix: int
    n_video: int
    tile_token: np.ndarray  # [n_tiles, tile] int32, -1 = pad
    tile_valid: np.ndarray  # [n_tiles] int32
    tile: int = 64
    cube: tuple = (4, 4, 4)
    is_ref: np.ndarray = None  # [n_prefix] uint8: 1 for a tile of a reference segment (R18), or None

    @property
    def n_ref(self) -> int:
        return 0 if self.is_ref is None else int(self.is_ref.sum())

    @property
    def seq_len(self) -> int:
        return int(sum(self.segments)) + int(np.prod(self.grid))


def default_cube(tile: int) -> tuple:
    """(ct, ch, cw) of a video tile: 4x4x4 for 64 tokens, 4x4x8 for 128 (R17)."""
    return {64: (4, 4, 4), 128: (4, 4, 8)}[int(tile)]


def geometry(segments, grid, tile=64, cube=None, ref_segments=None) -> Geometry:
    """ref_segments: one flag per prefix segment, true for a reference segment (R18), or None."""
    lib = _load()
    seg = np.asarray(segments, dtype=np.int32)
    T, H, W = (int(x) for x in grid)
    ct, ch, cw = (int(c) for c in (cube or default_cube(tile)))
    nt, npf, nv = (ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32())
    rc = lib.vsa_oracle_geometry(len(seg), _p(seg), T, H, W, int(tile), ct, ch, cw, ctypes.byref(nt),
                                 ctypes.byref(npf), ctypes.byref(nv))
    if rc:
        raise ValueError("bad geometry")
    tok = np.empty((nt.value, int(tile)), np.int32)
    val = np.empty((nt.value,), np.int32)
    lib.vsa_oracle_tiles(len(seg), _p(seg), T, H, W, int(tile), ct, ch, cw, _p(tok), _p(val))
    is_ref = None
    if ref_segments is not None:
        assert len(ref_segments) == len(seg)
        is_ref = np.concatenate([np.full(-(-int(n) // int(tile)), int(bool(f)), np.uint8)
                                 for n, f in zip(seg, ref_segments)] + [np.zeros(0, np.uint8)])
        assert len(is_ref) == npf.value
    return Geometry(tuple(int(s) for s in segments), (T, H, W), nt.value, npf.value, nv.value, tok, val, int(tile),
                    (ct, ch, cw), is_ref)


def topk_count(sparsity: float, n_video: int) -> int:
    return int(_load().vsa_oracle_topk_count(float(sparsity), int(n_video)))


def ref_count(keep: float, n_ref: int) -> int:
    """Reference tiles kept per video query tile (R18)."""
    return int(_load().vsa_oracle_ref_count(float(keep), int(n_ref)))


def default_scale(head_dim: int) -> float:
    """1/sqrt(D) rounded once to binary32."""
    return float(np.float32(1.0 / math.sqrt(float(head_dim))))


def pool(x_bf16: np.ndarray, geo: Geometry) -> np.ndarray:
    """x_bf16: [B, L, H, D] uint16 (bf16 bits) -> pooled [B, H, n_t, D] float32."""
    x = _c(x_bf16, np.uint16)
    B, L, H, D = x.shape
    out = np.empty((B, H, geo.n_tiles, D), np.float32)
    _load().vsa_oracle_pool(_p(x), B, L, H, D, geo.n_tiles, geo.tile, _p(geo.tile_token), _p(geo.tile_valid),
                            _p(out))
    return out


def scores(pq: np.ndarray, pk: np.ndarray, scale: float) -> np.ndarray:
    """pq, pk: [B, H, n_t, D] float32 -> S [B, H, n_t, n_t] float32."""
    pq = _c(pq, np.float32)
    pk = _c(pk, np.float32)
    B, H, n_t, D = pq.shape
    S = np.empty((B, H, n_t, n_t), np.float32)
    _load().vsa_oracle_scores(_p(pq), _p(pk), B * H, n_t, D, ctypes.c_float(scale), _p(S))
    return S


def select(S: np.ndarray, n_prefix: int, k: int, is_ref=None, kr: int = 0) -> np.ndarray:
    """S: [B, H, n_t, n_t] -> idx [B, H, V, k] int32 (global tile indices, ascending); with reference
    tiles (is_ref, R18) [B, H, V, kr + k]: the kr kept reference tiles, then the k video tiles."""
    S = _c(S, np.float32)
    B, H, n_t, _ = S.shape
    V = n_t - n_prefix
    if is_ref is not None:
        is_ref = _c(np.asarray(is_ref, np.uint8), np.uint8)
        idx = np.empty((B, H, V, kr + k), np.int32)
        if _load().vsa_oracle_select_ref(_p(S), B * H, n_t, n_prefix, _p(is_ref), kr, k, _p(idx)):
            raise ValueError("NaN pooled score")
        return idx
    idx = np.empty((B, H, V, k), np.int32)
    if _load().vsa_oracle_select(_p(S), B * H, n_t, n_prefix, k, _p(idx)):
        raise ValueError("NaN pooled score")
    return idx


def compress(S: np.ndarray, pv: np.ndarray) -> np.ndarray:
    """-> o_c [B, H, n_t, D] float64."""
    S = _c(S, np.float32)
    pv = _c(pv, np.float32)
    B, H, n_t, D = pv.shape
    out = np.empty((B, H, n_t, D), np.float64)
    _load().vsa_oracle_compress(_p(S), _p(pv), B * H, n_t, D, _p(out))
    return out


def _qk8_args(qk8, shape):
    """(q codes, q scales, k codes, k scales) for the 8-bit variant (R16), or four NULLs."""
    if qk8 is None:
        return (None, None, None, None)
    qc, qs, kc, ks = qk8
    B, L, H, D = shape
    qc, kc = (_c(t, np.uint8) for t in (qc, kc))
    qs, ks = (_c(t, np.float32) for t in (qs, ks))
    assert qc.shape == kc.shape == (B, L, H, D) and qs.shape == ks.shape == (B, L, H)
    return (qc, qs, kc, ks)


def _ref_args(geo: Geometry, idx, topk: int):
    """(reference flags, kr) for the C fine branch: an idx row holds kr reference tiles, then topk (R18)."""
    if geo.is_ref is None:
        return None, 0
    return _c(geo.is_ref, np.uint8), int(np.shape(idx)[-1]) - int(topk)


def fine(q, k, v, geo: Geometry, idx, topk: int, scale: float, todo=None, qk8=None) -> np.ndarray:
    """List formulation of the fine branch -> o_f [B, L, H, D] float64 (NaN where not computed).
    qk8 = (q codes, q scales, k codes, k scales) from quant_e4m3: the logits use those instead of q, k."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    B, L, H, D = q.shape
    idx = _c(idx, np.int32)
    if todo is not None:
        todo = _c(todo.astype(np.uint8), np.uint8)
    q8 = _qk8_args(qk8, q.shape)
    out = np.full((B, L, H, D), np.nan, np.float64)
    ref, kr = _ref_args(geo, idx, topk)
    _load().vsa_oracle_fine(_p(q), _p(k), _p(v), *(_p(t) for t in q8), B, L, H, D, geo.n_tiles, geo.n_prefix, topk,
                            _p(ref), kr, geo.tile,
                            _p(geo.tile_token), _p(geo.tile_valid), _p(idx), float(scale), _p(todo), _p(out))
    return out


def fine_split(q, k, v, geo: Geometry, idx, topk: int, scale: float, todo=None, qk8=None,
               video_qk=None) -> np.ndarray:
    """The fine branch with the pages' prefix split (reading R19): the dense prefix query tiles take
    their logits from the 8-bit Q/K of ``qk8`` (as fine() with qk8), the video query tiles from the bf16
    q, k (as fine() without), or with ``video_qk`` = (q4, k4) from those bf16 arrays instead (the
    dequantised FP4 operands of fp4_operands, reading R20).  Both branches run in full over their own
    tiles and the rows are merged by the tile each token belongs to; bf16 P.V throughout.  ("FastH3
    OmniRef inference", section "Device profiles": Q and K of the dense prefix query tiles rounded to
    8 bits with P.V in bf16, the video query tiles on another kernel.)"""
    B, L, H, _ = np.shape(q)
    n_t, P = geo.n_tiles, geo.n_prefix
    sel = np.ones((B, H, n_t), bool) if todo is None else np.asarray(todo, bool)
    is_prefix = np.zeros((B, H, n_t), bool)
    is_prefix[:, :, :P] = True
    pre = fine(q, k, v, geo, idx, topk, scale, todo=sel & is_prefix, qk8=qk8)
    qv, kv = (q, k) if video_qk is None else video_qk
    vid = fine(qv, kv, v, geo, idx, topk, scale, todo=sel & ~is_prefix)
    tok_prefix = np.zeros(L, bool)  # tokens of prefix tiles
    for i in range(P):
        tok_prefix[geo.tile_token[i, :geo.tile_valid[i]]] = True
    return np.where(tok_prefix[None, :, None, None], pre, vid)


def fine_tiles(q, k, v, geo: Geometry, idx, topk: int, scale: float, items, qk8=None) -> np.ndarray:
    """Fine branch of the listed query tiles only.  items: int64 array of
    (b*H + h)*n_t + i.  Returns [n_items, tile, D] float64 in tile row order
    (pad rows 0).  qk8: as for fine()."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    B, L, H, D = q.shape
    idx = _c(idx, np.int32)
    items = _c(np.asarray(items, np.int64), np.int64)
    q8 = _qk8_args(qk8, q.shape)
    ref, kr = _ref_args(geo, idx, topk)
    out = np.zeros((len(items), geo.tile, D), np.float64)
    _load().vsa_oracle_fine_tiles(_p(q), _p(k), _p(v), *(_p(t) for t in q8), B, L, H, D, geo.n_tiles,
                                  geo.n_prefix, topk, _p(ref), kr, geo.tile,
                                  _p(geo.tile_token), _p(geo.tile_valid), _p(idx), float(scale), len(items),
                                  _p(items), _p(out))
    return out


def e4m3_value(codes) -> np.ndarray:
    """float64 values of E4M3 codes (uint8 array), from the format's definition (R16)."""
    lib = _load()
    table = np.array([lib.vsa_oracle_e4m3_value(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def e4m3_round(y) -> np.ndarray:
    """E4M3 codes of binary32 values: nearest, ties to the even code, saturating at +-448."""
    y = _c(np.asarray(y, np.float32), np.float32)
    out = np.empty(y.shape, np.uint8)
    _load().vsa_oracle_e4m3_round_array(_p(y), y.size, _p(out))
    return out


def quant_e4m3(x_bf16: np.ndarray):
    """The 8-bit Q/K quantiser (R16): x [..., D] bf16 bits -> (codes [..., D] uint8, scale [...] float32),
    one scale per row of D (per batch, token and head)."""
    x = _c(x_bf16, np.uint16)
    D = x.shape[-1]
    n = x.size // D
    code = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1], np.float32)
    _load().vsa_oracle_quant_e4m3(_p(x), n, D, _p(code), _p(scale))
    return code, scale


def dequant_e4m3(code, scale) -> np.ndarray:
    """code * scale in float64 (exact: a 4-bit significand times a binary32 scale)."""
    return e4m3_value(code) * np.asarray(scale, np.float64)[..., None]


def e2m1_value(codes) -> np.ndarray:
    """float64 values of E2M1 codes (low 4 bits of a uint8 array), from the format's definition (R20)."""
    lib = _load()
    table = np.array([lib.vsa_oracle_e2m1_value(c) for c in range(16)], np.float64)
    return table[np.asarray(codes, np.uint8) & 15]


def e2m1_round(y) -> np.ndarray:
    """E2M1 codes of binary32 values: nearest, ties to the even code, saturating at +-6."""
    y = _c(np.asarray(y, np.float32), np.float32)
    out = np.empty(y.shape, np.uint8)
    _load().vsa_oracle_e2m1_round_array(_p(y), y.size, _p(out))
    return out


def quant_fp4(x) -> tuple:
    """The FP4 block quantiser (R20): x [..., D] binary32 (D a multiple of 16) -> (codes [..., D] uint8,
    one E2M1 code per element; scales [..., D / 16] uint8, one E4M3 code per 16 elements)."""
    x = _c(np.asarray(x, np.float32), np.float32)
    D = x.shape[-1]
    assert D % 16 == 0
    code = np.empty(x.shape, np.uint8)
    scale = np.empty(x.shape[:-1] + (D // 16,), np.uint8)
    _load().vsa_oracle_quant_fp4(_p(x), x.size // D, D, _p(code), _p(scale))
    return code, scale


def dequant_fp4(code, scale) -> np.ndarray:
    """code * scale in float64 (exact): each block of 16 elements times its E4M3 scale."""
    v = e2m1_value(code)
    sv = np.repeat(e4m3_value(scale), 16, axis=-1)
    return v * sv


def smooth_keys(k_bf16) -> tuple:
    """Key smoothing (R20): k [B, L, H, D] bf16 bits -> (mu [B, H, D] float32, the per-head key mean,
    summed in binary64 in token order; k - mu [B, L, H, D] binary32)."""
    k = _c(k_bf16, np.uint16)
    B, L, H, D = k.shape
    mu = np.empty((B, H, D), np.float32)
    ks = np.empty((B, L, H, D), np.float32)
    _load().vsa_oracle_smooth_keys(_p(k), B, L, H, D, _p(mu), _p(ks))
    return mu, ks


def bf16_bits_exact(x) -> np.ndarray:
    """bf16 bits of float64 values that bf16 holds exactly (asserted)."""
    f = np.asarray(x, np.float64).astype(np.float32)
    assert (f.astype(np.float64) == np.asarray(x, np.float64)).all()
    u = f.view(np.uint32)
    assert not (u & 0xFFFF).any(), "value not representable in bf16"
    return (u >> 16).astype(np.uint16)


def fp4_operands(q_bf16, k_bf16, smooth: bool = True) -> tuple:
    """(q4, k4): the dequantised FP4 Q and K (R20) as bf16 bits [B, L, H, D]; K smoothed first
    when ``smooth``.  They replace q, k in the video query tiles' logits."""
    qf = (_c(q_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32)
    kf = smooth_keys(k_bf16)[1] if smooth else (_c(k_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32)
    return tuple(bf16_bits_exact(dequant_fp4(*quant_fp4(t))) for t in (qf, kf))


def output_tiles(o_f_tiles, o_c, gate, geo: Geometry, items, H: int) -> np.ndarray:
    """out rows of the listed tiles: o_f + gate * o_c[tile] (tile row order; pad rows 0); the gate
    is [B, L, H] (one per token and head) or [B, L, H*D] (one per channel, R12)."""
    D = o_f_tiles.shape[-1]
    B, L = np.shape(gate)[0], np.shape(gate)[1]
    per_channel = gate_is_per_channel(gate, B, L, H, D)
    gate = _c(gate, np.uint16)
    gf = (gate.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if per_channel:
        gf = gf.reshape(B, L, H, D)
    res = np.zeros_like(o_f_tiles)
    for n, bhi in enumerate(np.asarray(items, np.int64)):
        i = int(bhi % geo.n_tiles)
        bh = int(bhi // geo.n_tiles)
        h, b = bh % H, bh // H
        nv = int(geo.tile_valid[i])
        toks = geo.tile_token[i, :nv]
        g = gf[b, toks, h] if per_channel else gf[b, toks, h][:, None]
        res[n, :nv] = o_f_tiles[n, :nv] + g * o_c[b, h, i][None, :]
    return res


def selection(q, k, v, segments, grid, sparsity, scale=None, tile=64, cube=None, ref_segments=None, ref_keep=None):
    """Pool, scores, top-k and compression only (every tile, every head).  ref_segments / ref_keep:
    reference segments and their keep ratio (R18)."""
    geo = geometry(segments, grid, tile, cube, ref_segments)
    if scale is None:
        scale = default_scale(q.shape[-1])
    kc = topk_count(sparsity, geo.n_video)
    kr = ref_count(ref_keep, geo.n_ref) if geo.is_ref is not None and geo.n_video > 0 else 0
    pq, pk, pv = pool(q, geo), pool(k, geo), pool(v, geo)
    S = scores(pq, pk, scale)
    idx = select(S, geo.n_prefix, kc, geo.is_ref, kr)
    o_c = compress(S, pv)
    return dict(geo=geo, topk=kc, kr=kr, scale=scale, pq=pq, pk=pk, pv=pv, S=S, idx=idx, o_c=o_c)


def fine_masked(q, k, v, geo: Geometry, idx, topk: int, scale: float) -> np.ndarray:
    """Mask formulation (dense L x L masked softmax attention) -> [B, L, H, D] float64."""
    q, k, v = (_c(t, np.uint16) for t in (q, k, v))
    B, L, H, D = q.shape
    idx = _c(idx, np.int32)
    out = np.full((B, L, H, D), np.nan, np.float64)
    ref, kr = _ref_args(geo, idx, topk)
    _load().vsa_oracle_fine_masked(_p(q), _p(k), _p(v), B, L, H, D, geo.n_tiles, geo.n_prefix, topk, _p(ref), kr,
                                   geo.tile,
                                   _p(geo.tile_token), _p(geo.tile_valid), _p(idx), float(scale), _p(out))
    return out


def gate_is_per_channel(gate, B, L, H, D) -> bool:
    """[B, L, H]: one gate per token and head; [B, L, H*D] or [B, L, H, D]: one per channel (R12)."""
    shape = tuple(np.shape(gate))
    if shape == (B, L, H):
        return False
    if shape in ((B, L, H * D), (B, L, H, D)):
        return True
    raise ValueError(f"gate shape {shape} is neither [B, L, H] nor [B, L, H*D]")


def output(o_f, o_c, gate, geo: Geometry, todo=None) -> np.ndarray:
    o_f = _c(o_f, np.float64)
    o_c = _c(o_c, np.float64)
    B, L, H, D = o_f.shape
    per_channel = gate_is_per_channel(gate, B, L, H, D)
    gate = _c(gate, np.uint16)
    if todo is not None:
        todo = _c(todo.astype(np.uint8), np.uint8)
    out = np.full((B, L, H, D), np.nan, np.float64)
    _load().vsa_oracle_output(_p(o_f), _p(o_c), _p(gate), int(per_channel), B, L, H, D, geo.n_tiles, geo.tile,
                              _p(geo.tile_token), _p(geo.tile_valid), _p(todo), _p(out))
    return out


@dataclass
class ForwardResult:
    geo: Geometry
    topk: int
    scale: float
    pq: np.ndarray
    pk: np.ndarray
    pv: np.ndarray
    S: np.ndarray
    idx: np.ndarray
    o_c: np.ndarray
    o_f: np.ndarray
    out: np.ndarray
    seconds: float


def forward(q, k, v, gate, segments, grid, sparsity, scale=None, todo=None, qk8=False, tile=64,
            cube=None, ref_segments=None, ref_keep=None, fp4=False, k_smooth=True) -> ForwardResult:
    """The whole VSA-H3 forward on bf16-bit arrays q, k, v [B,L,H,D] and gate [B,L,H] (or
    [B,L,H*D], one per channel).

    Selection (pool, scores, top-k) always runs in full; the fine branch and
    the output run for the query tiles flagged in ``todo`` ([B, H, n_t] bool,
    None = all).  qk8: the fine branch's logits use 8-bit Q/K (R16); the
    selection still reads the bf16 inputs; qk8="prefix": only the dense prefix
    query tiles do (R19, fine_split).  tile, cube: the tile size and video
    cube shape (64 and 4x4x4 as the method states; 128 per R17).  ref_segments,
    ref_keep: reference segments and their keep ratio (R18).  fp4: the video
    query tiles' logits use the dequantised FP4 Q and K (R20; K smoothed when
    k_smooth), the prefix query tiles' follow qk8 (False: bf16, "prefix": 8-bit);
    fp4 with qk8=True (8-bit video tiles) is refused."""
    t0 = time.perf_counter()
    geo = geometry(segments, grid, tile, cube, ref_segments)
    D = q.shape[-1]
    if scale is None:
        scale = default_scale(D)
    kc = topk_count(sparsity, geo.n_video)
    kr = ref_count(ref_keep, geo.n_ref) if geo.is_ref is not None and geo.n_video > 0 else 0
    pq, pk, pv = pool(q, geo), pool(k, geo), pool(v, geo)
    S = scores(pq, pk, scale)
    idx = select(S, geo.n_prefix, kc, geo.is_ref, kr)
    o_c = compress(S, pv)
    q8 = (*quant_e4m3(q), *quant_e4m3(k)) if qk8 else None
    if fp4:
        if qk8 not in (False, None, "prefix"):
            raise ValueError("fp4 video tiles go with bf16 or 8-bit (qk8='prefix') prefix tiles")
        o_f = fine_split(q, k, v, geo, idx, kc, scale, todo, qk8=q8, video_qk=fp4_operands(q, k, k_smooth))
    elif qk8 == "prefix":
        o_f = fine_split(q, k, v, geo, idx, kc, scale, todo, qk8=q8)
    else:
        o_f = fine(q, k, v, geo, idx, kc, scale, todo, qk8=q8)
    out = output(o_f, o_c, gate, geo, todo)
    return ForwardResult(geo, kc, scale, pq, pk, pv, S, idx, o_c, o_f, out, time.perf_counter() - t0)
