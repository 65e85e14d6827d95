"""Seeded synthetic workloads for the VSA-H3 forward.

This module is the ONLY thing the oracle and the CUDA library share: it draws
the inputs.  It holds none of the method's arithmetic (no tiling of tokens
into attention tiles, no pooling, no scores, no selection).

Workloads stand in for the pages' two operating points -- 480p (~14-15k packed
tokens) and 1344x768 (~75k packed tokens), 56 heads -- plus two small shapes
the CPU oracle finishes in seconds.  There is no dataset: values are drawn
from a counter-based generator.

Generator: every value is a pure function of (seed, stream id, element index):
    h = splitmix64(index + splitmix64(seed * 1_000_003 + stream))
    u1 = (h >> 40 + 1) / 2^24 in (0, 1],  u2 = (h & 0xffffff) / 2^24
    z  = sqrt(-2 ln u1) * cos(2 pi u2)                    (Box-Muller)
computed in float64 and rounded once to bfloat16 (round to nearest even).
splitmix64 is Steele, Lea & Flood's finaliser (constants 0x9E3779B97F4A7C15,
0xBF58476D1CE4E5B9, 0x94D049BB133111EB).  The same code runs on CPU or CUDA
tensors; parity tests feed the oracle the exact bytes the GPU saw.

Structure (the "structured tile scores" workloads): the latent video is
divided into 4x4x4 (t, h, w) blocks and each prefix segment into runs of 64
tokens; for every (batch, head, block) one offset vector mu in {+-2}^D is
drawn, and each (token, head) row of Q -- and independently of K -- gets mu
added with probability 0.2.  This gives neighbouring latent voxels a shared
content direction, so tile-level scores carry signal.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

# ----------------------------------------------------------------------------
# workload shapes
# ----------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    head_dim: int
    segments: tuple  # prefix segment lengths in order: (text, cond, audio)
    grid: tuple  # post-patchify video grid (T, H, W)
    sparsity: float
    structured: bool = False
    gate_std: float = 0.1
    description: str = ""
    gate_per_channel: bool = False  # gate [B, L, H*D] (one per channel) instead of [B, L, H]
    tile: int = 64  # tokens per attention tile (64, or 128 for the OmniRef-style variant)
    cube: tuple = None  # video cube (t, h, w) of a tile; None = the plan's default for `tile`
    ref_segments: tuple = None  # per prefix segment: True for a reference segment (reference keep)
    ref_keep: float = 0.0  # keep ratio of reference tiles

    @property
    def seq_len(self) -> int:
        return int(sum(self.segments)) + self.grid[0] * self.grid[1] * self.grid[2]


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 2, 64, (40, 0, 24), (8, 8, 8), 0.5,
                 description="1x2 heads, D=64, text 40 + audio 24, video 8x8x8, sparsity 0.5"),
        Workload("small", 1, 8, 128, (256, 64, 192), (8, 16, 32), 0.8,
                 description="1x8 heads, D=128, text 256 + cond 64 + audio 192, video 8x16x32, sparsity 0.8"),
        Workload("480p", 1, 56, 128, (384, 0, 384), (8, 30, 56), 0.9, structured=True,
                 description="480p-shaped: 56 heads, D=128, text 384 + audio 384, video 8x30x56, sparsity 0.9"),
        Workload("768p_s0.8", 1, 56, 128, (512, 0, 768), (24, 48, 64), 0.8, structured=True,
                 description="1344x768-shaped: 56 heads, D=128, text 512 + audio 768, video 24x48x64, sparsity 0.8"),
        Workload("768p_s0.9", 1, 56, 128, (512, 0, 768), (24, 48, 64), 0.9, structured=True,
                 description="1344x768-shaped: 56 heads, D=128, text 512 + audio 768, video 24x48x64, sparsity 0.9"),
        Workload("768p_t128_s0.9", 1, 56, 128, (512, 0, 768), (24, 48, 64), 0.9, structured=True, tile=128,
                 description="1344x768-shaped with 128-token tiles (4x4x8 cubes): 56 heads, D=128, text 512 + "
                             "audio 768, video 24x48x64, sparsity 0.9"),
        Workload("omniref_768p", 1, 56, 128, (512, 6144, 768), (24, 48, 64), 0.9, structured=True, tile=128,
                 ref_segments=(False, True, False), ref_keep=0.1,
                 description="OmniRef-shaped: 1344x768 video with 128-token tiles, text 512 + 6144 reference "
                             "tokens (reference keep 0.1) + audio 768, 56 heads, D=128, sparsity 0.9"),
    ]
}

SPARSITY_SWEEP = (0.0, 0.5, 0.8, 0.9, 0.95)


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    if overrides:
        d = dict(w.__dict__)
        d.update(overrides)
        w = Workload(**d)
    return w


# ----------------------------------------------------------------------------
# counter-based generator
# ----------------------------------------------------------------------------

_M64 = (1 << 64) - 1


def _i64(c: int) -> int:
    """Reinterpret an unsigned 64-bit constant as a signed int64."""
    c &= _M64
    return c - (1 << 64) if c >= (1 << 63) else c


_GOLDEN = _i64(0x9E3779B97F4A7C15)
_C1 = _i64(0xBF58476D1CE4E5B9)
_C2 = _i64(0x94D049BB133111EB)


def _splitmix64_int(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _M64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & _M64
    return x ^ (x >> 31)


def _lsr(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _splitmix64(x: torch.Tensor) -> torch.Tensor:
    x = x + _GOLDEN
    x = (x ^ _lsr(x, 30)) * _C1
    x = (x ^ _lsr(x, 27)) * _C2
    return x ^ _lsr(x, 31)


def _stream_key(seed: int, stream: int) -> int:
    return _i64(_splitmix64_int(seed * 1_000_003 + stream))


def _hash(seed: int, stream: int, index: torch.Tensor) -> torch.Tensor:
    return _splitmix64(index + _stream_key(seed, stream))


def _normal(h: torch.Tensor) -> torch.Tensor:
    u1 = (_lsr(h, 40) + 1).double() * (1.0 / (1 << 24))
    u2 = (h & 0xFFFFFF).double() * (1.0 / (1 << 24))
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


def _uniform(h: torch.Tensor) -> torch.Tensor:
    return _lsr(h, 40).double() * (1.0 / (1 << 24))


# stream ids
_Q, _K, _V, _GATE, _MU, _MASK_Q, _MASK_K = 1, 2, 3, 4, 5, 6, 7
_CHUNK = 1 << 24


def _normal_tensor(seed, stream, numel, device, std=1.0):
    out = torch.empty(numel, dtype=torch.float64, device=device)
    for s in range(0, numel, _CHUNK):
        n = min(_CHUNK, numel - s)
        idx = torch.arange(s, s + n, dtype=torch.int64, device=device)
        out[s:s + n] = _normal(_hash(seed, stream, idx)) * std
    return out


def block_ids(w: Workload) -> torch.Tensor:
    """Structure groups of the workload: one id per token of the packed
    sequence -- 64-token runs inside each prefix segment, 4x4x4 latent blocks
    of the video.  Returns (ids [L] int64, number of groups)."""
    ids = []
    g = 0
    for n in w.segments:
        r = torch.arange(n, dtype=torch.int64)
        ids.append(g + r // 64)
        g += (n + 63) // 64
    T, H, W = w.grid
    t = torch.arange(T).view(T, 1, 1)
    h = torch.arange(H).view(1, H, 1)
    x = torch.arange(W).view(1, 1, W)
    nb_h, nb_w = (H + 3) // 4, (W + 3) // 4
    vid = (t // 4) * (nb_h * nb_w) + (h // 4) * nb_w + (x // 4)
    ids.append(g + vid.reshape(-1).to(torch.int64))
    g += ((T + 3) // 4) * nb_h * nb_w
    return torch.cat(ids), g


def make_inputs(w: Workload, seed: int = 0, device="cpu", keep_fp64: bool = False):
    """Q, K, V [B, L, H, D] bf16 and gate [B, L, H] (or [B, L, H*D] with gate_per_channel) bf16 on ``device``.

    With ``keep_fp64`` the unrounded float64 draws are returned as well (the
    tiny workload's "fp32 originals")."""
    B, L, H, D = w.batch, w.seq_len, w.heads, w.head_dim
    n = B * L * H * D
    out = {}
    raw = {}
    for name, stream in (("q", _Q), ("k", _K), ("v", _V)):
        x = _normal_tensor(seed, stream, n, device)
        if w.structured and name in ("q", "k"):
            x = x.view(B, L, H, D)
            ids, ngroups = block_ids(w)
            ids = ids.to(device)
            # mu[b, h, g, d] = +-2
            mu_idx = torch.arange(B * H * ngroups * D, dtype=torch.int64, device=device)
            mu = torch.where(_hash(seed, _MU, mu_idx) & 1 == 1, 2.0, -2.0).double()
            mu = mu.view(B, H, ngroups, D)
            row_idx = torch.arange(B * L * H, dtype=torch.int64, device=device)
            hit = _uniform(_hash(seed, _MASK_Q if name == "q" else _MASK_K, row_idx)) < 0.2
            hit = hit.view(B, L, H)
            for b in range(B):
                # offset for token l, head h: mu[b, h, ids[l], :]
                off = mu[b][:, ids, :].permute(1, 0, 2)  # [L, H, D]
                x[b] += torch.where(hit[b].unsqueeze(-1), off, torch.zeros((), dtype=off.dtype, device=device))
            x = x.reshape(-1)
        if keep_fp64:
            raw[name] = x.view(B, L, H, D).clone()
        out[name] = x.to(torch.bfloat16).view(B, L, H, D)
        del x
    gw = H * D if w.gate_per_channel else H
    g = _normal_tensor(seed, _GATE, B * L * gw, device, std=w.gate_std)
    out["gate"] = g.to(torch.bfloat16).view(B, L, gw)
    if keep_fp64:
        raw["gate"] = g.view(B, L, gw)
        out["fp64"] = raw
    return out


def as_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bits (host copy)."""
    import numpy as np

    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
