"""Pins for the oracle's 8-bit Q/K variant (reading R16: E4M3 codes, one
binary32 scale s = amax / 448 per batch, token and head, round to nearest
even with saturation at 448; the dequantised Q and K replace the bf16 ones in
the fine branch's logits only).

What pins it, independently of the oracle's code:
  - the E4M3 value of every code against torch.float8_e4m3fn (library) and
    against hand-worked closed forms;
  - the rounding against torch's float -> float8_e4m3fn conversion (library)
    wherever that conversion is defined (|y| < 464), against the saturation
    rule above it, and against a brute-force nearest search written here;
  - the quantiser against its invariants (the amax element codes to +-448,
    the error bound of a 4-bit significand, zero rows) and against torch's
    binary32 division followed by torch's conversion;
  - the fine branch with 8-bit operands: exactly equal to the bf16 fine
    branch when every row is already representable as code * 2^e (the
    quantiser is then the identity), and within a derived bound of it
    otherwise.
"""
import math

import numpy as np
import pytest
import torch

import synth


def f8_torch_values():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def torch_round(y: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(y, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_magnitudes():
    """The 127 finite non-negative E4M3 magnitudes by code, from the bit layout (sign, 4-bit exponent
    with bias 7, 3-bit mantissa; exponent 0 is subnormal; 0x7F is NaN)."""
    out = []
    for c in range(127):
        e, m = c >> 3, c & 7
        out.append(m * 2.0 ** -9 if e == 0 else (8 + m) * 2.0 ** (e - 10))
    return out


def brute_round(y: float) -> int:
    """Nearest finite E4M3 magnitude by exhaustive search; a tie picks the even code; saturates at 448."""
    mags = e4m3_magnitudes()
    a = abs(y)
    sign = 0x80 if math.copysign(1.0, y) < 0 else 0
    best = None
    for c, v in enumerate(mags):
        d = abs(a - v)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


# ---------------------------------------------------------------------------
# the E4M3 format
# ---------------------------------------------------------------------------


def test_e4m3_decode_all_codes_match_torch(oracle_mod):
    ours = oracle_mod.e4m3_value(np.arange(256, dtype=np.uint8))
    ref = f8_torch_values()
    nan = np.isnan(ref)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()
    assert (np.signbit(ours[~nan]) == np.signbit(ref[~nan])).all()


def test_e4m3_decode_closed_forms(oracle_mod):
    v = lambda c: float(oracle_mod.e4m3_value(np.array([c], np.uint8))[0])
    assert v(0x00) == 0.0 and v(0x80) == 0.0 and math.copysign(1, v(0x80)) < 0
    assert v(0x01) == 2.0 ** -9          # smallest subnormal: mantissa 1/8 times 2^-6
    assert v(0x07) == 7 * 2.0 ** -9      # largest subnormal
    assert v(0x08) == 2.0 ** -6          # smallest normal
    assert v(0x38) == 1.0 and v(0x40) == 2.0 and v(0x39) == 1.125
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0  # 1.75 * 2^8, the largest finite value
    assert v(0x77) == 240.0              # exponent 14, mantissa 7: 1.875 * 2^7


def test_e4m3_round_matches_torch_where_defined(oracle_mod):
    mags = np.array(e4m3_magnitudes())
    mids = (mags[1:] + mags[:-1]) / 2  # exact in binary32 (at most 5 significant bits)
    y = [mags, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
         np.nextafter(mids.astype(np.float32), np.float32(np.inf))]
    # every bf16 pattern below 464 in magnitude, and random binary32 over the whole range
    bits = np.arange(65536, dtype=np.uint32)
    bf = (bits << 16).view(np.float32)
    y.append(bf[np.isfinite(bf) & (np.abs(bf) < 464)])
    rng = np.random.default_rng(0)
    y.append((rng.uniform(-1, 1, 200000) * 2.0 ** rng.uniform(-14, 8.8, 200000)).astype(np.float32))
    y = np.concatenate([np.concatenate([a, -a]) for a in (np.asarray(t, np.float32) for t in y)])
    assert np.abs(y).max() < 464
    assert (oracle_mod.e4m3_round(y) == torch_round(y)).all()


def test_e4m3_round_saturates(oracle_mod):
    y = np.array([448.0, 448.0001, 463.99, 464.0, 480.0, 1e6, 3.0e38, np.inf], np.float32)
    assert (oracle_mod.e4m3_round(y) == 0x7E).all()
    assert (oracle_mod.e4m3_round(-y) == 0xFE).all()


def test_e4m3_round_brute_force(oracle_mod):
    mags = e4m3_magnitudes()
    vals = [0.0, -0.0, 2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -10, -3 * 2.0 ** -10, 1.0625, 1.1875, 17.0, 19.0,
            232.0, 240.0, 248.0, 440.0, 447.9]
    vals += [(a + b) / 2 for a, b in zip(mags[:-1], mags[1:])][::3]
    rng = np.random.default_rng(1)
    vals += list(rng.standard_normal(300) * 40.0)
    y = np.array(vals, np.float32)
    ours = oracle_mod.e4m3_round(y)
    ref = np.array([brute_round(float(t)) for t in y], np.uint8)
    assert (ours == ref).all()


# ---------------------------------------------------------------------------
# the per-(token, head) quantiser
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("D,mag", [(128, 1.0), (128, 1e-3), (96, 30.0), (64, 1.0)])
def test_quant_e4m3_properties(oracle_mod, D, mag):
    g = torch.Generator().manual_seed(D)
    x = (torch.randn(3, 50, 4, D, generator=g, dtype=torch.float64) * mag).to(torch.bfloat16)
    xb = synth.as_bits(x)
    code, s = oracle_mod.quant_e4m3(xb)
    assert code.shape == xb.shape and s.shape == xb.shape[:-1] and s.dtype == np.float32
    xf = x.to(torch.float32)
    amax = xf.abs().amax(-1)
    # torch's binary32 division and float8 conversion give the same codes
    st = amax / torch.tensor(448.0, dtype=torch.float32)
    assert (torch.from_numpy(s) == st).all()
    ref = (xf / st[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (code == ref).all()
    # the amax element of every row codes to +-448
    arg = xf.abs().argmax(-1).numpy()
    top = np.take_along_axis(code, arg[..., None], -1)[..., 0]
    assert np.isin(top, [0x7E, 0xFE]).all()
    # error bound of a 4-bit significand (half an ulp: 2^-4 relative; 2^-10 s below the normal range)
    deq = oracle_mod.dequant_e4m3(code, s)
    xd = xf.double().numpy()
    bound = 2.0 ** -4 * np.abs(xd) * (1 + 2.0 ** -20) + 2.0 ** -10 * s[..., None].astype(np.float64)
    assert (np.abs(deq - xd) <= bound).all()


def test_quant_e4m3_zero_and_single_rows(oracle_mod):
    x = torch.zeros(1, 3, 2, 64, dtype=torch.bfloat16)
    x[0, 1, 0, 5] = -3.5
    x[0, 2, 1, :] = 2.0 ** -120  # tiny but nonzero: its own scale, every code 448
    code, s = oracle_mod.quant_e4m3(synth.as_bits(x))
    assert s[0, 0, 0] == 0 and (code[0, 0] == 0).all() and s[0, 0, 1] == 0
    assert s[0, 1, 0] == np.float32(3.5) / np.float32(448)
    assert code[0, 1, 0, 5] == 0xFE and (np.delete(code[0, 1, 0], 5) == 0).all()
    assert (code[0, 2, 1] == 0x7E).all()
    assert oracle_mod.dequant_e4m3(code, s)[0, 1, 0, 5] == -3.5


# ---------------------------------------------------------------------------
# the fine branch with 8-bit Q/K
# ---------------------------------------------------------------------------


def representable(shape, seed):
    """bf16 rows that are exactly E4M3 codes times 2^e (e per row), each row holding one +-448 * 2^e:
    the quantiser must return exactly those codes with scale 2^e."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 127, size=shape).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=shape) << 7).astype(np.uint8)
    lead = rng.integers(0, shape[-1], size=shape[:-1])
    np.put_along_axis(codes, lead[..., None], np.uint8(0x7E), -1)
    e = rng.integers(-9, -4, size=shape[:-1])
    mags = np.array(e4m3_magnitudes() + [np.nan])
    val = mags[codes & 0x7F] * np.where(codes & 0x80, -1.0, 1.0) * np.exp2(e)[..., None]
    bits = synth.as_bits(torch.from_numpy(val).to(torch.bfloat16))
    assert (torch.from_numpy(bits.astype(np.int32)).to(torch.int16).view(torch.bfloat16).double().numpy()
            == val).all()
    return bits, codes, np.exp2(e).astype(np.float32)


def test_fine_q8_equals_bf16_on_representable_inputs(oracle_mod):
    w = synth.workload("tiny")
    B, L, H, D = w.batch, w.seq_len, w.heads, w.head_dim
    q, qc, qs = representable((B, L, H, D), 5)
    k, kc, ks = representable((B, L, H, D), 6)
    v = synth.as_bits(torch.randn(B, L, H, D, generator=torch.Generator().manual_seed(7)).to(torch.bfloat16))
    gq, gk = oracle_mod.quant_e4m3(q), oracle_mod.quant_e4m3(k)
    assert (gq[0] == qc).all() and (gq[1] == qs).all() and (gk[0] == kc).all() and (gk[1] == ks).all()
    sel = oracle_mod.selection(q, k, v, w.segments, w.grid, 0.5)
    args = (q, k, v, sel["geo"], sel["idx"], sel["topk"], sel["scale"])
    ref = oracle_mod.fine(*args)
    got = oracle_mod.fine(*args, qk8=(qc, qs, kc, ks))
    assert np.array_equal(got, ref)
    # a scale taken from the wrong token (or the codes of the wrong operand) shows
    bad = oracle_mod.fine(*args, qk8=(qc, qs[:, ::-1].copy(), kc, ks))
    assert np.abs(bad - ref).max() > 1e-3
    bad = oracle_mod.fine(*args, qk8=(kc, ks, qc, qs))
    assert np.abs(bad - ref).max() > 1e-3


@pytest.mark.parametrize("sparsity", [0.0, 0.5])
def test_fine_q8_within_bound_of_bf16(oracle_mod, sparsity):
    """General inputs: each dequantised element is within 2^-4 |x| + 2^-10 s of x, so each logit moves by
    at most delta = scale * sum_d (|q||dk| + |dq||k| + |dq||dk|) and every output by at most
    (exp(2 delta_max) - 1) * max |v| over the row's keys; the change is also not zero."""
    w = synth.workload("tiny")
    x = synth.make_inputs(w, seed=3)
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(b["q"], b["k"], b["v"], w.segments, w.grid, sparsity)
    args = (b["q"], b["k"], b["v"], sel["geo"], sel["idx"], sel["topk"], sel["scale"])
    ref = oracle_mod.fine(*args)
    q8 = (*oracle_mod.quant_e4m3(b["q"]), *oracle_mod.quant_e4m3(b["k"]))
    got = oracle_mod.fine(*args, qk8=q8)
    qf = x["q"].double().numpy()
    kf = x["k"].double().numpy()
    dq = 2.0 ** -4 * np.abs(qf) + 2.0 ** -10 * q8[1][..., None]
    dk = 2.0 ** -4 * np.abs(kf) + 2.0 ** -10 * q8[3][..., None]
    vmax = np.abs(x["v"].double().numpy()).max()
    for h in range(w.heads):
        aq, ak = np.abs(qf[0, :, h]), np.abs(kf[0, :, h])
        delta = sel["scale"] * (aq @ dk[0, :, h].T + dq[0, :, h] @ ak.T + dq[0, :, h] @ dk[0, :, h].T)
        bound = (np.exp(2 * delta.max(axis=1)) - 1) * vmax  # per query token (over every key: an upper bound)
        err = np.abs(got[0, :, h] - ref[0, :, h]).max(axis=1)
        assert (err <= bound * (1 + 1e-9)).all()
    assert np.abs(got - ref).max() > 0


# ---------------------------------------------------------------------------
# the pages' prefix split: 8-bit Q/K for the dense prefix query tiles only (R19)
# ---------------------------------------------------------------------------


def _split_case(oracle_mod, name, seed, **over):
    w = synth.workload(name, **over)
    x = synth.make_inputs(w, seed=seed)
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    sel = oracle_mod.selection(b["q"], b["k"], b["v"], w.segments, w.grid, w.sparsity)
    args = (b["q"], b["k"], b["v"], sel["geo"], sel["idx"], sel["topk"], sel["scale"])
    q8 = (*oracle_mod.quant_e4m3(b["q"]), *oracle_mod.quant_e4m3(b["k"]))
    return w, sel, args, q8


def _prefix_tokens(geo, L):
    t = np.zeros(L, bool)
    for i in range(geo.n_prefix):
        t[geo.tile_token[i, :geo.tile_valid[i]]] = True
    return t


@pytest.mark.parametrize("name,over", [("tiny", {}), ("tiny", dict(sparsity=0.0)), ("small", dict(heads=2))])
def test_fine_split_rows_follow_their_branch(oracle_mod, name, over):
    """Prefix query rows take the 8-bit logits, video query rows the bf16 ones, each over the same key
    sets: the split equals the all-8-bit branch on every prefix token and the bf16 branch on every video
    token, and differs from each on the other side (so the rows are not swapped)."""
    w, sel, args, q8 = _split_case(oracle_mod, name, 4, **over)
    got = oracle_mod.fine_split(*args, qk8=q8)
    all8 = oracle_mod.fine(*args, qk8=q8)
    bf16 = oracle_mod.fine(*args)
    pre = _prefix_tokens(sel["geo"], w.seq_len)
    assert pre.any() and (~pre).any()
    assert np.array_equal(got[:, pre], all8[:, pre])
    assert np.array_equal(got[:, ~pre], bf16[:, ~pre])
    assert np.abs(got[:, pre] - bf16[:, pre]).max() > 0
    assert np.abs(got[:, ~pre] - all8[:, ~pre]).max() > 0


def test_fine_split_special_cases(oracle_mod):
    """No prefix: the split is the bf16 branch; no video: it is the all-8-bit branch."""
    for segs, grid, same_as_8bit in (((), (8, 8, 8), False), ((100, 30), (0, 0, 0), True)):
        w = synth.Workload("split", 1, 2, 64, segs, grid, 0.5)
        x = synth.make_inputs(w, seed=9)
        b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v")}
        sel = oracle_mod.selection(b["q"], b["k"], b["v"], w.segments, w.grid, w.sparsity)
        args = (b["q"], b["k"], b["v"], sel["geo"], sel["idx"], sel["topk"], sel["scale"])
        q8 = (*oracle_mod.quant_e4m3(b["q"]), *oracle_mod.quant_e4m3(b["k"]))
        want = oracle_mod.fine(*args, qk8=q8 if same_as_8bit else None)
        assert np.array_equal(oracle_mod.fine_split(*args, qk8=q8), want)


def test_forward_prefix_split_matches_composition(oracle_mod):
    """forward(qk8="prefix") is the selection, the split fine branch and the gated output."""
    w, sel, args, q8 = _split_case(oracle_mod, "tiny", 6)
    x = synth.make_inputs(w, seed=6)
    b = {n: synth.as_bits(x[n]) for n in ("q", "k", "v", "gate")}
    ref = oracle_mod.forward(b["q"], b["k"], b["v"], b["gate"], w.segments, w.grid, w.sparsity, qk8="prefix")
    o_f = oracle_mod.fine_split(*args, qk8=q8)
    assert np.array_equal(ref.o_f, o_f)
    assert np.array_equal(ref.idx, sel["idx"])
    assert np.array_equal(ref.out, oracle_mod.output(o_f, sel["o_c"], b["gate"], sel["geo"]))
