"""Pins for the oracle's FP4 video-tile variant (reading R20: E2M1 codes with one E4M3 scale per 16
values and a global scale of 1, each head's mean key removed from K before the rounding, the
dequantised Q and K in the video query tiles' logits; the prefix query tiles per the split).

What pins it, independently of the oracle's code:
  - the E2M1 value of every code against ml_dtypes.float4_e2m1fn (library) and the format's closed
    forms; the rounding against ml_dtypes' float32 -> float4_e2m1fn conversion over every bf16
    pattern and random binary32 values, and against a brute-force nearest search written here;
  - the block quantiser against numpy's binary32 division, torch's float8_e4m3fn conversion for the
    block scales and ml_dtypes' conversion for the codes, and on blocks that are exactly codes times
    a power of two (the quantiser is then the identity);
  - the premise that every dequantised value is a bf16 number (all 16 x 255 products);
  - the key mean against numpy's float64 mean, and the smoothed keys against numpy's binary32
    subtraction;
  - the fine branch with FP4 operands: invariant, bit for bit, under a per-channel offset added to
    every key (what the smoothing is for: without it the same offset changes the output, and the
    error against bf16 grows); within a derived bound of the bf16 fine branch; and the forward's
    rows follow their branch (prefix rows the split's, video rows the FP4 operands').
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import synth

F4 = ml_dtypes.float4_e2m1fn
E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]  # codes 0..7: 2-bit exponent (bias 1), 1-bit mantissa


def lib_e2m1_round(y) -> np.ndarray:
    return np.asarray(y, np.float32).astype(F4).view(np.uint8) & 15


def lib_e4m3_round(y) -> np.ndarray:
    return torch.from_numpy(np.asarray(y, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def lib_e4m3_value(c) -> np.ndarray:
    return torch.from_numpy(np.asarray(c, np.uint8)).view(torch.float8_e4m3fn).to(torch.float32).numpy()


def brute_e2m1(y: float) -> int:
    """Nearest E2M1 magnitude by exhaustive search; a tie picks the even code; saturates at 6."""
    a = abs(y)
    sign = 8 if np.signbit(np.float32(y)) else 0
    best = None
    for c, v in enumerate(E2M1_MAGS):
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return synth.as_bits(x.to(torch.bfloat16))


def as_f32(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# the E2M1 format
# ---------------------------------------------------------------------------


def test_e2m1_decode_all_codes(oracle_mod):
    ours = oracle_mod.e2m1_value(np.arange(16, dtype=np.uint8))
    ref = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    assert (ours == ref).all() and (np.signbit(ours) == np.signbit(ref)).all()
    assert list(ours[:8]) == E2M1_MAGS and list(-ours[8:]) == E2M1_MAGS
    assert np.signbit(ours[8])  # code 8 is -0


def test_e2m1_round_matches_library(oracle_mod):
    mags = np.array(E2M1_MAGS)
    mids = (mags[1:] + mags[:-1]) / 2
    y = [mags, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
         np.nextafter(mids.astype(np.float32), np.float32(np.inf)), [6.0001, 7.0, 100.0, 3.0e38]]
    bits = np.arange(65536, dtype=np.uint32)
    bf = (bits << 16).view(np.float32)
    y.append(bf[np.isfinite(bf)])
    rng = np.random.default_rng(0)
    y.append((rng.uniform(-1, 1, 200000) * 2.0 ** rng.uniform(-6, 4, 200000)).astype(np.float32))
    y = np.concatenate([np.concatenate([a, -a]) for a in (np.asarray(t, np.float32) for t in y)])
    assert (oracle_mod.e2m1_round(y) == lib_e2m1_round(y)).all()


def test_e2m1_round_brute_force(oracle_mod):
    rng = np.random.default_rng(1)
    vals = [0.0, -0.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 1e-30, -1e-30, 0.2500001, 4.999999]
    vals += list(rng.standard_normal(400) * 3.0)
    y = np.array(vals, np.float32)
    assert (oracle_mod.e2m1_round(y) == np.array([brute_e2m1(float(t)) for t in y], np.uint8)).all()


def test_dequantised_values_are_bf16_numbers(oracle_mod):
    """Every E2M1 value times every finite E4M3 scale has at most 6 significant bits and lies in
    [2^-10, 2688]: a bf16 number, so the dequantised FP4 operands can be handed over as bf16."""
    codes = np.repeat(np.arange(16, dtype=np.uint8), 256).reshape(16, 256)
    scales = np.tile(np.arange(256, dtype=np.uint8), (16, 1))
    finite = (scales & 0x7F) != 0x7F
    prod = oracle_mod.e2m1_value(codes) * oracle_mod.e4m3_value(scales)
    bits = oracle_mod.bf16_bits_exact(prod[finite])  # raises if any product is not a bf16 number
    assert np.array_equal(as_f32(bits).astype(np.float64), prod[finite])
    nz = np.abs(prod[finite]) > 0
    assert np.abs(prod[finite][nz]).min() == 2.0 ** -10 and np.abs(prod[finite]).max() == 2688.0


# ---------------------------------------------------------------------------
# the per-16 block quantiser
# ---------------------------------------------------------------------------


def lib_quant_fp4(x: np.ndarray):
    """The same quantiser from library conversions: scale = float8_e4m3fn(amax / 6), codes =
    float4_e2m1fn(x / scale), binary32 divisions by numpy; a zero scale gives +0 codes."""
    x = np.asarray(x, np.float32)
    blocks = x.reshape(x.shape[:-1] + (x.shape[-1] // 16, 16))
    amax = np.abs(blocks).max(-1)
    sc = lib_e4m3_round(amax / np.float32(6.0))
    sv = lib_e4m3_value(sc)
    with np.errstate(divide="ignore", invalid="ignore"):
        codes = lib_e2m1_round(blocks / sv[..., None])
    codes = np.where(sv[..., None] == 0, np.uint8(0), codes)
    return codes.reshape(x.shape), sc


@pytest.mark.parametrize("D,mag", [(128, 1.0), (128, 1e-3), (96, 30.0), (64, 1.0), (64, 2.0 ** -12)])
def test_quant_fp4_matches_library(oracle_mod, D, mag):
    g = torch.Generator().manual_seed(D)
    x = (torch.randn(2, 40, 3, D, generator=g, dtype=torch.float64) * mag).to(torch.float32).numpy()
    x[0, 0, 0, :16] = 0.0           # an all-zero block
    x[0, 1, 0, 16:32] = -0.0
    x[1, 2, 1, :16] = 2.0 ** -20    # a block whose scale rounds to zero
    code, scale = oracle_mod.quant_fp4(x)
    assert code.shape == x.shape and scale.shape == x.shape[:-1] + (D // 16,)
    ref_code, ref_scale = lib_quant_fp4(x)
    assert np.array_equal(scale, ref_scale)
    assert np.array_equal(code, ref_code)
    assert (scale[0, 0, 0, 0] == 0) and (code[0, 0, 0, :16] == 0).all() and (code[1, 2, 1, :16] == 0).all()


def test_quant_fp4_brute_force_codes(oracle_mod):
    """Each code is the nearest E2M1 value to x / scale (ties even, saturating), by exhaustive search."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((5, 64)) * 2.0 ** rng.uniform(-4, 4, (5, 1))).astype(np.float32)
    code, scale = oracle_mod.quant_fp4(x)
    sv = np.repeat(lib_e4m3_value(scale), 16, axis=-1)
    want = np.array([brute_e2m1(float(t)) for t in (x / sv).ravel()], np.uint8).reshape(x.shape)
    assert np.array_equal(code, want)


def test_quant_fp4_identity_on_representable_blocks(oracle_mod):
    """A block of E2M1 values times 2^e holding one +-6 * 2^e: its scale is 2^e (an E4M3 number for
    e in [-9, 8]) and the codes come back unchanged, so the dequantised block equals the input."""
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, (6, 8, 16)).astype(np.uint8)
    lead = rng.integers(0, 16, (6, 8))
    np.put_along_axis(codes, lead[..., None], (rng.integers(0, 2, (6, 8, 1)) * 8 + 7).astype(np.uint8), -1)
    e = rng.integers(-9, 9, (6, 8))
    x = (np.array(E2M1_MAGS * 2)[codes] * np.where(codes >= 8, -1.0, 1.0) * np.exp2(e)[..., None])
    x = x.reshape(6, 128).astype(np.float32)
    got_c, got_s = oracle_mod.quant_fp4(x)
    want = codes.reshape(6, 128)
    assert np.array_equal(got_c & 7, want & 7)  # magnitudes; a zero may come back as either +0 or -0
    assert np.array_equal(oracle_mod.dequant_fp4(got_c, got_s), x.astype(np.float64))
    assert np.array_equal(lib_e4m3_value(got_s), np.exp2(e).astype(np.float32))


# ---------------------------------------------------------------------------
# key smoothing
# ---------------------------------------------------------------------------


def test_smooth_keys_mean_and_difference(oracle_mod):
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=2)
    kb = synth.as_bits(x["k"])
    mu, ks = oracle_mod.smooth_keys(kb)
    kf = as_f32(kb)
    # numpy's float64 mean (pairwise order): every partial sum of these bf16 values is exact in float64
    want = kf.astype(np.float64).mean(axis=1).astype(np.float32)
    assert np.array_equal(mu, want)
    assert np.array_equal(ks, kf - mu[:, None])
    # the smoothed keys have (float64) mean zero up to the rounding of mu and of the differences
    assert np.abs(ks.astype(np.float64).mean(axis=1)).max() < 1e-6


def grid_case(seed, offsets=None):
    """A 512-token case (one 64-token prefix segment and a 7 x 8 x 8 video grid, so every mean is a
    division by 2^9) whose keys lie on a 1/16 grid inside (-4, 4): with per-(head, channel) offsets of
    +-8 the keys stay bf16 numbers and every mean and difference of the smoothing stays exact."""
    w = synth.Workload("fp4grid", 1, 2, 64, (64,), (7, 8, 8), 0.5)
    assert w.seq_len == 512
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(1, 512, 2, 64, generator=g)
    v = torch.randn(1, 512, 2, 64, generator=g)
    gate = torch.randn(1, 512, 2, generator=g) * 0.1
    k = torch.randint(-62, 63, (1, 512, 2, 64), generator=g).double() / 16
    if offsets is not None:
        k = k + torch.from_numpy(offsets)[None, None]
    kb = bf16_bits(k)
    assert np.array_equal(as_f32(kb).astype(np.float64), k.numpy())
    return w, {"q": bf16_bits(q), "k": kb, "v": bf16_bits(v), "gate": bf16_bits(gate)}


def test_fp4_video_rows_invariant_to_key_offsets(oracle_mod):
    """With smoothing, adding a constant to a channel of every key of a head leaves the FP4 video rows
    unchanged bit for bit (the mean takes the offset away before quantisation); without smoothing the
    same offset changes them, and moves them farther from the bf16 result."""
    off = np.where(np.random.default_rng(5).integers(0, 2, (2, 64)) == 1, 8.0, -8.0)
    w, a = grid_case(11)
    _, b = grid_case(11, off)
    run = lambda t, **kw: oracle_mod.forward(t["q"], t["k"], t["v"], t["gate"], w.segments, w.grid, w.sparsity,
                                             fp4=True, **kw)
    geo = oracle_mod.geometry(w.segments, w.grid)
    vid = np.ones(w.seq_len, bool)
    vid[geo.tile_token[0, :geo.tile_valid[0]]] = False
    ra, rb = run(a), run(b)
    assert np.array_equal(ra.o_f[:, vid], rb.o_f[:, vid])
    # the prefix rows (bf16 logits, unsmoothed): the offset shifts each row's logits by one constant
    assert np.abs(ra.o_f[:, ~vid] - rb.o_f[:, ~vid]).max() < 1e-9
    na, nb = run(a, k_smooth=False), run(b, k_smooth=False)
    assert np.abs(na.o_f[:, vid] - nb.o_f[:, vid]).max() > 1e-2
    bf = oracle_mod.forward(b["q"], b["k"], b["v"], b["gate"], w.segments, w.grid, w.sparsity)
    err_s = np.abs(rb.o_f[:, vid] - bf.o_f[:, vid]).mean()
    err_n = np.abs(nb.o_f[:, vid] - bf.o_f[:, vid]).mean()
    assert err_s < err_n / 2, (err_s, err_n)


# ---------------------------------------------------------------------------
# the fine branch with FP4 operands
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_fp4_fine_within_bound_of_bf16(oracle_mod, sparsity):
    """Video rows with FP4 Q and smoothed FP4 K against the bf16 fine branch: the logit of (i, j) moves
    by scale * (q4_i . k4_j - q_i . k_j) = -scale * (q4_i . mu) [one constant per row, which the softmax
    removes] + r_ij with |r_ij| <= scale * sum_d (|q - q4| |k| + |q4| |k4 - (k - mu)|) =: rho_ij, so every
    output moves by at most (exp(2 max_j rho_ij) - 1) * max |v| (over every key: an upper bound)."""
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=3)
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(b["q"], b["k"], b["v"], w.segments, w.grid, sparsity)
    geo = sel["geo"]
    args = (b["q"], b["k"], b["v"], geo, sel["idx"], sel["topk"], sel["scale"])
    ref = oracle_mod.fine(*args)
    q4, k4 = oracle_mod.fp4_operands(b["q"], b["k"])
    got = oracle_mod.fine_split(*args, video_qk=(q4, k4))
    qf, kf = x["q"].double().numpy(), x["k"].double().numpy()
    mu = kf.mean(axis=1).astype(np.float32).astype(np.float64)  # per (b, h, d), as in the pin above
    q4f, k4f = as_f32(q4).astype(np.float64), as_f32(k4).astype(np.float64)
    dq = np.abs(qf - q4f)
    ek = np.abs(k4f - (kf - mu[:, None]))
    vmax = np.abs(x["v"].double().numpy()).max()
    vid = np.ones(w.seq_len, bool)
    for i in range(geo.n_prefix):
        vid[geo.tile_token[i, :geo.tile_valid[i]]] = False
    for h in range(w.heads):
        rho = sel["scale"] * (dq[0, :, h] @ np.abs(kf[0, :, h]).T + np.abs(q4f[0, :, h]) @ ek[0, :, h].T)
        bound = (np.exp(2 * rho.max(axis=1)) - 1) * vmax
        err = np.abs(got[0, :, h] - ref[0, :, h]).max(axis=1)
        assert (err[vid] <= bound[vid] * (1 + 1e-9)).all()
        assert (err[~vid] == 0).all()  # prefix rows: bf16 logits, as the reference
    assert np.abs(got[0][vid] - ref[0][vid]).max() > 0


@pytest.mark.parametrize("qk8", [False, "prefix"])
def test_forward_fp4_rows_follow_their_branch(oracle_mod, qk8):
    """forward(fp4=True): selection as the bf16 forward; prefix rows exactly the rows of forward(qk8)
    (bf16, or the 8-bit split); video rows exactly the fine branch on the FP4 operands; the output the
    gated sum of those."""
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=8)
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    fwd = lambda **kw: oracle_mod.forward(b["q"], b["k"], b["v"], b["gate"], w.segments, w.grid, w.sparsity, **kw)
    got = fwd(qk8=qk8, fp4=True)
    base = fwd(qk8=qk8)
    assert np.array_equal(got.S, base.S) and np.array_equal(got.idx, base.idx) and np.array_equal(got.o_c, base.o_c)
    geo = got.geo
    pre = np.zeros(w.seq_len, bool)
    for i in range(geo.n_prefix):
        pre[geo.tile_token[i, :geo.tile_valid[i]]] = True
    assert np.array_equal(got.o_f[:, pre], base.o_f[:, pre])
    q4, k4 = oracle_mod.fp4_operands(b["q"], b["k"])
    vidf = oracle_mod.fine(q4, k4, b["v"], geo, got.idx, got.topk, got.scale)
    assert np.array_equal(got.o_f[:, ~pre], vidf[:, ~pre])
    assert np.abs(got.o_f[:, ~pre] - base.o_f[:, ~pre]).max() > 1e-3
    assert np.array_equal(got.out, oracle_mod.output(got.o_f, got.o_c, b["gate"], geo))
    with pytest.raises(ValueError):
        fwd(qk8=True, fp4=True)


def test_key_sums_order_free_on_the_480p_keys(oracle_mod):
    """The GPU adds each key column in 512-row binary64 partial sums over the tile-order copy (pads
    zero) and combines the partials atomically, in any order.  The structured 480p keys hold residues
    near 1e-16 (a sample near -2 plus its +2 tile offset), so exactness is not guaranteed a priori; this
    replays that summation structure on the CPU with three combination orders and finds every binary64
    column sum equal to the oracle's token-order sum, hence every binary32 mean equal too."""
    w = synth.workload("480p")
    kb = synth.as_bits(synth.make_inputs(w, seed=0)["k"])
    mu, _ = oracle_mod.smooth_keys(kb)
    geo = oracle_mod.geometry(w.segments, w.grid)
    tok = geo.tile_token.reshape(-1)
    f = as_f32(kb)[0]  # [L, H, D]
    assert (np.abs(f[f != 0]) < 1e-12).any()  # the residues are there
    rng = np.random.default_rng(0)
    for h in range(w.heads):
        rows = np.where(tok[:, None] >= 0, f[np.maximum(tok, 0), h, :], 0.0).astype(np.float64)
        nb = (rows.shape[0] + 511) // 512
        part = [np.add.accumulate(rows[i * 512:(i + 1) * 512], axis=0)[-1] for i in range(nb)]
        token_order = np.add.accumulate(f[:, h, :].astype(np.float64), axis=0)[-1]
        for order in (range(nb), range(nb - 1, -1, -1), rng.permutation(nb)):
            s = np.zeros(w.head_dim)
            for i in order:
                s = s + part[i]
            assert np.array_equal(s, token_order), h
        assert np.array_equal((token_order / w.seq_len).astype(np.float32), mu[0, h])
