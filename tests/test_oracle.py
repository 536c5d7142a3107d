"""Pins for the CPU oracle (no GPU).

Each check ties the oracle to something other than itself: hand-derived
values from the format and layout definitions (tests/golden), independent
library routines (torch's bf16 / float8_e4m3fn casts, numpy's bincount and
stable argsort), brute-force searches, exact rational arithmetic, and the
invariants the method must satisfy (counts sum to the valid slots, padding
rows are zero, combine of identity outputs returns x, dispatch and
unweighted combine are adjoint, FP8 round trip).
"""

import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W


# ---------------------------------------------------------------- helpers

def bf16_bits_of(values) -> np.ndarray:
    """Exact bf16 values -> bits, through torch (library cast)."""
    t = torch.tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_of_bf16(bits) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float32).numpy()


def round_fraction(q: Fraction, sig_bits: int, emin: int = -126) -> Fraction:
    """Round an exact rational to the nearest value with `sig_bits`
    significand bits and minimum exponent `emin` (ties to even).  Used with
    24 bits for binary32 and 8 bits for bfloat16 (no overflow in these tests)."""
    if q == 0:
        return Fraction(0)
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    quantum = Fraction(2) ** (e - (sig_bits - 1))
    n = a / quantum
    m = n.numerator // n.denominator
    r = n - m
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and m % 2 == 1):
        m += 1
    v = m * quantum
    return -v if q < 0 else v


def e4m3_brute(v: np.ndarray) -> np.ndarray:
    """Nearest of the 127 non-negative finite e4m3 codes by exhaustive search
    (ties: even mantissa), saturating at 448, sign reapplied."""
    codes = np.arange(0x7F, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float64)
    # The values are rebuilt independently of the oracle's decoder too:
    ef, m = codes >> 3, codes & 7
    indep = np.where(ef == 0, m * 2.0 ** -9, (8 + m) * 2.0 ** (ef.astype(np.int64) - 10))
    assert np.array_equal(vals, indep)
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[:, None] - indep[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equal-distance codes prefer an even mantissa
    even = (codes & 1) == 0
    pick = np.where((cand & even[None, :]).any(axis=1),
                    np.argmax(cand & even[None, :], axis=1), np.argmax(cand, axis=1))
    out = codes[pick]
    out = np.where(a >= 448.0, 0x7E, out).astype(np.uint8)
    sign = np.signbit(v.astype(np.float32))
    return np.where(sign, out | 0x80, out).astype(np.uint8)


# --------------------------------------------------------------- formats

def test_bf16_widening_matches_torch():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f32(bits)
    ref = f32_of_bf16(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_rounding_matches_torch_on_all_boundaries():
    # every bf16 upper half, with the dropped half at each rounding boundary
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF], dtype=np.uint32)
    pats = (hi[:, None] | lows[None, :]).reshape(-1)
    rng = np.random.default_rng(123)
    pats = np.concatenate([pats, rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64)
                           .astype(np.uint32)])
    v = pats.view(np.float32)
    v = v[~np.isnan(v)]
    ours = oracle.f32_to_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_e4m3_hand_derived_codes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e4m3_codes.json")))
    vals = np.array([float(v) for v in g["values"]], dtype=np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), np.array(g["codes"], dtype=np.uint8))


def _e4m3_probe_values():
    codes = np.arange(0x7F, dtype=np.uint8)
    ef, m = codes >> 3, codes & 7
    vals = np.where(ef == 0, m * 2.0 ** -9, (8 + m) * 2.0 ** (ef.astype(np.int64) - 10))
    vals = np.sort(vals)
    mids = (vals[:-1] + vals[1:]) / 2
    pts = np.concatenate([vals, mids, [448.0 + 16.0, 470.0, 480.0, 1e6]]).astype(np.float32)
    # each point and its 3 binary32 neighbours on each side
    u = pts.view(np.uint32).astype(np.int64)
    near = (u[:, None] + np.arange(-3, 4)[None, :]).reshape(-1)
    near = near[(near >= 0) & (near < 0x7F800000)].astype(np.uint32).view(np.float32)
    rng = np.random.default_rng(7)
    rand = np.concatenate([rng.uniform(0, 500, 200_000), rng.uniform(0, 2 ** -5, 100_000),
                           np.exp(rng.uniform(-30, 7, 100_000))]).astype(np.float32)
    allv = np.concatenate([near, rand, [0.0]]).astype(np.float32)
    return np.concatenate([allv, -allv])


def test_e4m3_encoder_matches_brute_force_search():
    v = _e4m3_probe_values()
    for chunk in np.array_split(v, 16):
        assert np.array_equal(oracle.e4m3_encode(chunk), e4m3_brute(chunk))


def test_e4m3_encoder_matches_torch_cast_in_range():
    v = _e4m3_probe_values()
    v = v[np.abs(v) <= 464.0]          # torch's cast does not saturate beyond this
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_decoder_matches_torch():
    c = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(c)
    ref = torch.from_numpy(c).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])


def e2m1_brute(v: np.ndarray) -> np.ndarray:
    """Nearest of the 8 E2M1 magnitudes by exhaustive search (ties: even
    mantissa = even code), saturating at 6, sign reapplied."""
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = np.minimum(np.abs(v.astype(np.float64)), 6.0)
    d = np.abs(a[:, None] - mags[None, :])
    cand = d == d.min(axis=1, keepdims=True)
    even = (np.arange(8) & 1) == 0
    pick = np.where((cand & even).any(axis=1), np.argmax(cand & even, axis=1), np.argmax(cand, axis=1))
    return np.where(np.signbit(v.astype(np.float32)), pick | 8, pick).astype(np.uint8)


def test_e2m1_hand_derived_codes(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "e2m1_codes.json")))
    vals = np.array([float(v) for v in g["values"]], dtype=np.float32)
    assert np.array_equal(oracle.e2m1_encode(vals), np.array(g["codes"], dtype=np.uint8))


def test_e2m1_encoder_matches_brute_force_search():
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    pts = np.concatenate([mags, (mags[:-1] + mags[1:]) / 2, [6.5, 7.0, 100.0]]).astype(np.float32)
    u = pts.view(np.uint32).astype(np.int64)
    near = (u[:, None] + np.arange(-3, 4)[None, :]).reshape(-1)
    near = near[near >= 0].astype(np.uint32).view(np.float32)
    rng = np.random.default_rng(31)
    v = np.concatenate([near, rng.uniform(0, 8, 100_000).astype(np.float32), [0.0]])
    v = np.concatenate([v, -v])
    assert np.array_equal(oracle.e2m1_encode(v), e2m1_brute(v))
    assert np.array_equal(oracle.e2m1_decode(np.arange(16, dtype=np.uint8)),
                          np.concatenate([mags, -mags]).astype(np.float32))


def test_nvfp4_block_invariants():
    rng = np.random.default_rng(37)
    H = 512
    x = rng.standard_normal((40, H)) * (10.0 ** rng.uniform(-1.5, 2.5, size=(40, H // 16))).repeat(16, axis=1)
    x[3, 16:32] = 0.0                                        # zero block -> smallest scale, zero codes
    x[4, 0:16] = 0.0
    x[4, 0], x[4, 1] = 5.0, 0.5                              # nibble order: even element in the low nibble
    xb = bf16_bits_of(x)
    xf = f32_of_bf16(xb).reshape(40, H // 16, 16).astype(np.float64)
    q, s = oracle.nvfp4_rows(xb)
    codes = np.stack([q & 0xF, q >> 4], axis=-1).reshape(40, H // 16, 16)
    sdec = oracle.e4m3_decode(s).astype(np.float64)
    amax = np.maximum(np.abs(xf).max(axis=2), 6.0 / 512)
    # the scale is the e4m3 rounding of amax/6: within half an e4m3 spacing, codes 0x01..0x7E
    assert np.all((s >= 1) & (s <= 0x7E))
    assert np.all(np.abs(sdec - amax / 6) <= 2.0 ** (np.floor(np.log2(np.maximum(amax / 6, 2.0 ** -6))) - 4) + 1e-12)
    # the largest element of every non-zero block lands on +-6
    am = np.abs(xf).argmax(axis=2)
    top = np.take_along_axis(codes, am[..., None], axis=2)[..., 0]
    nz = np.abs(xf).max(axis=2) > 0
    assert np.all((top[nz] & 7) == 7)
    # every code is the nearest E2M1 value (brute force) to x * (1/scale) in
    # binary32, saturating at 6
    inv = (np.float32(1.0) / sdec.astype(np.float32))[..., None]
    t = (xf.astype(np.float32) * inv).astype(np.float32)
    assert np.array_equal(codes.reshape(-1), e2m1_brute(t.reshape(-1)))
    assert np.all(codes[3, 1] == 0) and s[3, 1] == 0x01
    assert q[4, 0] & 0xF == 7 and q[4, 0] >> 4 == codes[4, 0, 1]    # x[0] (5.0, the amax) in the low nibble


# ---------------------------------------------------------- quantisation

def test_quantize_hand_example():
    x = np.zeros((1, 128), np.float32)
    x[0, :4] = [1.0, -2.0, 0.5, 0.1]
    q, s = oracle.quantize_rows(bf16_bits_of(x))
    # amax 2 -> inv 224: 224 -> 0x76, -448 -> 0xFE, 112 -> 0x6E, bf16(0.1)*224 = 22.42 -> 0x5B
    assert list(q[0, :4]) == [0x76, 0xFE, 0x6E, 0x5B]
    assert np.all(q[0, 4:] == 0)
    assert s[0, 0] == np.float32(2.0) / np.float32(448.0)


def test_quantize_product_form_golden(golden_dir):
    # Two blocks whose scaled value is exactly the e4m3 midpoint 336, derived
    # by hand: q = e4m3(RN(x * RN(448/amax))) rounds block 0 up and lands
    # block 1 on the tie, while q = e4m3(RN(x / RN(amax/448))) does the
    # opposite, so the two readings give different codes in both blocks.
    g = json.load(open(os.path.join(golden_dir, "fp8_quant_product_form.json")))
    H = g["hidden"]
    x = np.zeros((1, H), np.float32)
    for b, vals in enumerate(g["x"]):
        x[0, b * 128:b * 128 + len(vals)] = vals
    xb = bf16_bits_of(x)
    assert np.array_equal(f32_of_bf16(xb), x)          # every input is bf16-exact
    q, s = oracle.quantize_rows(xb)
    for b, codes in enumerate(g["codes"]):
        blk = q[0, b * 128:(b + 1) * 128]
        assert list(blk[:len(codes)]) == codes
        assert np.all(blk[len(codes):] == 0)
        m, e = g["scales_exact"][b]
        assert Fraction(float(s[0, b])) == Fraction(m) * Fraction(2) ** e


def test_quantize_invariants():
    rng = np.random.default_rng(3)
    H = 1024
    x = rng.standard_normal((64, H)).astype(np.float32)
    # very different magnitudes per block, so a wrong block index shows up
    x *= (10.0 ** rng.uniform(-3, 4, size=(64, H // 128))).repeat(128, axis=1).astype(np.float32)
    x[5, 128:256] = 0.0                     # an all-zero block: floored scale
    x[6, 256:384] = -3.0                    # a constant block
    xb = bf16_bits_of(x)
    xf = f32_of_bf16(xb).reshape(64, H // 128, 128)
    q, s = oracle.quantize_rows(xb)
    qb = q.reshape(64, H // 128, 128)
    deq = oracle.e4m3_decode(qb).astype(np.float64)
    amax = np.abs(xf).max(axis=2)
    # scale is amax/448 rounded once (floored amax for the zero block)
    floor = np.float32(1e-4)
    assert np.array_equal(s, np.maximum(amax, floor).astype(np.float32) / np.float32(448.0))
    # the largest element of each block lands on +-448 exactly
    am = np.abs(xf).argmax(axis=2)
    top = np.take_along_axis(qb, am[..., None], axis=2)[..., 0]
    nz = amax > 0
    assert np.all((top[nz] & 0x7F) == 0x7E)
    # sign preserved, |q| <= 448, and each code is the nearest to x/scale:
    t = xf.astype(np.float64) / s[..., None].astype(np.float64)
    assert np.all(np.abs(deq) <= 448.0)
    assert np.all((deq == 0) | (np.sign(deq) == np.sign(xf)))
    a = np.abs(t)
    binade = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    half_spacing = 2.0 ** (binade - 4)
    assert np.all(np.abs(np.abs(deq) - a) <= half_spacing * (1 + 2 ** -18) + 1e-12)
    # all-zero block -> zero codes, constant block -> all -448
    assert np.all(qb[5, 1] == 0) and s[5, 1] == floor / np.float32(448.0)
    assert np.all(qb[6, 2] == 0xFE)


# ---------------------------------------------------------------- layout

def test_layout_hand_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "layout_hand_example.json")))
    idx = np.array(g["topk_idx"], np.int64)
    w = np.array(g["topk_weights"], np.float32)
    assert oracle.max_recv_rows(g["T"], g["k"], g["E"], g["align"]) == g["max_recv_rows"]
    lay = oracle.layout(idx, g["E"], g["S"], g["align"], w)
    R = g["R"]
    assert lay["R"] == R and lay["flags"] == 0
    for key in ("counts", "offsets", "seg_tokens", "slot_map"):
        assert lay[key].tolist() == g[key], key
    assert lay["recv_src"][:R].tolist() == g["recv_src"]
    assert lay["recv_topk_idx"][:R].tolist() == g["recv_topk_idx"]
    assert lay["recv_topk_weights"][:R].tolist() == g["recv_topk_weights"]
    # dispatch (bf16) and combine of the same example
    recv, _ = oracle.dispatch(lay, bf16_bits_of(g["x"]), oracle.X_BF16)
    assert np.array_equal(f32_of_bf16(recv[:R]), np.array(g["recv_x"], np.float32))
    y = bf16_bits_of(g["y"])
    y = np.concatenate([y, np.zeros((g["max_recv_rows"] - R, 2), np.uint16)])
    out, _ = oracle.combine(lay["slot_map"], g["T"], g["k"], y, w)
    assert np.array_equal(f32_of_bf16(out), np.array(g["combine_weighted"], np.float32))
    rw = np.concatenate([np.array(g["recv_weights_in"], np.float32),
                         np.zeros(g["max_recv_rows"] - R, np.float32)])
    out, ow = oracle.combine(lay["slot_map"], g["T"], g["k"], y, None, rw, True)
    assert np.array_equal(f32_of_bf16(out), np.array(g["combine_unweighted"], np.float32))
    assert np.array_equal(ow, np.array(g["out_weights"], np.float32))


def brute_force_layout(idx, E, align):
    """O(E*T*k): for each expert in turn, scan every slot in flat order."""
    flat = idx.reshape(-1)
    slot_map = [-1] * flat.size
    recv_src = []
    offsets = [0]
    for e in range(E):
        for s in range(flat.size):
            if flat[s] == e:
                slot_map[s] = len(recv_src)
                recv_src.append(s)
        while len(recv_src) % align:
            recv_src.append(-1)
        offsets.append(len(recv_src))
    return np.array(slot_map), np.array(recv_src), np.array(offsets)


@pytest.mark.parametrize("T,k,E,S,align,drop,seed", [
    (1, 1, 1, 1, 1, 0.0, 0), (7, 3, 5, 5, 3, 0.2, 1), (33, 4, 16, 4, 8, 0.1, 2),
    (64, 8, 32, 8, 1, 0.0, 3), (50, 2, 12, 3, 128, 0.5, 4), (40, 6, 8, 2, 5, 1.0, 5)])
def test_layout_matches_brute_force(T, k, E, S, align, drop, seed):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)     # duplicates allowed
    idx[rng.random((T, k)) < drop] = -1
    w = rng.standard_normal((T, k)).astype(np.float32)
    lay = oracle.layout(idx, E, S, align, w)
    sm, src, offs = brute_force_layout(idx, E, align)
    R = lay["R"]
    assert R == offs[-1] and lay["flags"] == 0
    assert np.array_equal(lay["slot_map"], sm)
    assert np.array_equal(lay["recv_src"][:R], src)
    assert np.array_equal(lay["offsets"], offs)
    # library cross-checks: bincount for counts, stable argsort for the order
    valid = idx.reshape(-1) >= 0
    assert np.array_equal(lay["counts"], np.bincount(idx.reshape(-1)[valid], minlength=E))
    order = np.argsort(np.where(valid, idx.reshape(-1), E), kind="stable")[: valid.sum()]
    assert np.array_equal(lay["recv_src"][:R][lay["recv_src"][:R] >= 0], order)
    # per-row expert id and weight
    real = lay["recv_src"][:R] >= 0
    assert np.array_equal(lay["recv_topk_idx"][:R][real], idx.reshape(-1)[order])
    assert np.array_equal(lay["recv_topk_weights"][:R][real], w.reshape(-1)[order])
    assert np.all(lay["recv_topk_idx"][:R][~real] == -1)
    assert np.all(lay["recv_topk_weights"][:R][~real] == 0)
    # aligned offsets: multiples of align, each block the least one holding its count
    d = np.diff(lay["offsets"])
    assert np.all(d % align == 0) and np.all(d >= lay["counts"]) and np.all(d - lay["counts"] < align)
    assert R <= oracle.max_recv_rows(T, k, E, align)
    # tokens per segment: sets per token
    per = E // S
    seg = np.zeros(S, int)
    for t in range(T):
        for g in {int(e) // per for e in idx[t] if e >= 0}:
            seg[g] += 1
    assert np.array_equal(lay["seg_tokens"], seg)


def test_layout_flags_bad_indices_and_treats_them_as_dropped():
    idx = np.array([[0, 5], [-2, 1], [3, -1]], np.int64)
    lay = oracle.layout(idx, 4, 2, 1)
    assert lay["flags"] & 1
    assert lay["slot_map"].tolist() == [0, -1, -1, 1, 2, -1]
    assert lay["counts"].tolist() == [1, 1, 0, 1]


def test_layout_capacity_overflow_is_flagged_and_not_written():
    idx = np.zeros((4, 2), np.int64)
    lay = oracle.layout(idx, 2, 1, 4, max_rows=5)
    assert lay["flags"] & 2
    assert lay["slot_map"].tolist() == [0, 1, 2, 3, 4, -1, -1, -1]


def test_layout_empty():
    lay = oracle.layout(np.zeros((0, 4), np.int64), 8, 2, 16)
    assert lay["R"] == 0 and np.all(lay["counts"] == 0) and np.all(lay["seg_tokens"] == 0)


# -------------------------------------------------------------- dispatch

@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_dispatch_rows_are_the_source_tokens(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=11, T=min(w.T, 512))
    T = inp["x"].shape[0]
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    R = lay["R"]
    sm = lay["slot_map"]
    valid = sm >= 0
    src_tok = np.arange(T * w.k)[valid] // w.k
    pad = np.where(lay["recv_src"][:R] < 0)[0]
    recv, _ = oracle.dispatch(lay, inp["x"], oracle.X_BF16)
    assert np.array_equal(recv[sm[valid]], inp["x"][src_tok])           # numpy gather
    assert np.all(recv[pad] == 0)
    if w.H % 16 == 0:
        q4, s4 = oracle.nvfp4_rows(inp["x"])
        rq, rs = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_NVFP4)
        assert np.array_equal(rq[sm[valid]], q4[src_tok]) and np.array_equal(rs[sm[valid]], s4[src_tok])
        assert np.all(rq[pad] == 0) and np.all(rs[pad] == 0)
        assert np.all(rq[R:] == oracle.UNWRITTEN) and np.all(rs[R:] == oracle.UNWRITTEN)
    if w.H % 128 == 0:
        q, s = oracle.quantize_rows(inp["x"])
        rq, rs = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8)
        assert np.array_equal(rq[sm[valid]], q[src_tok]) and np.array_equal(rs[sm[valid]], s[src_tok])
        assert np.all(rq[pad] == 0) and np.all(rs[pad] == 0)
        pq, ps = W.make_prequant(T, w.H, seed=2)
        rq, rs = oracle.dispatch(lay, pq, oracle.X_FP8_PREQUANT, ps)
        assert np.array_equal(rq[sm[valid]], pq[src_tok]) and np.array_equal(rs[sm[valid]], ps[src_tok])
        assert np.all(rq[pad] == 0) and np.all(rs[pad] == 0)


# --------------------------------------------------------------- combine

def test_combine_equals_exact_rational_fma_chain():
    rng = np.random.default_rng(5)
    T, k, H, E = 12, 5, 24, 6
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)
    idx[rng.random((T, k)) < 0.2] = -1
    lay = oracle.layout(idx, E, 2, 4)
    rows = lay["max_rows"]
    y = bf16_bits_of(rng.standard_normal((rows, H)) * 10.0 ** rng.uniform(-3, 3, (rows, 1)))
    wts = (rng.standard_normal((T, k)) * 3).astype(np.float32)
    yf = f32_of_bf16(y)
    for weights in (wts, None):
        out, _ = oracle.combine(lay["slot_map"], T, k, y, weights)
        exp = np.empty((T, H), np.float32)
        for t in range(T):
            for h in range(H):
                acc = Fraction(0)
                for j in range(k):
                    r = lay["slot_map"][t * k + j]
                    if r < 0:
                        continue
                    wj = Fraction(float(weights[t, j])) if weights is not None else Fraction(1)
                    acc = round_fraction(wj * Fraction(float(yf[r, h])) + acc, 24)
                exp[t, h] = float(round_fraction(acc, 8))
        assert np.array_equal(out, bf16_bits_of(exp))


def _e4m3_codes(rng, shape):
    """Random e4m3 codes, both signs, no NaN (0x7F / 0xFF)."""
    c = rng.integers(0, 0x7F, size=shape).astype(np.uint8)
    return c | (rng.integers(0, 2, size=shape).astype(np.uint8) << 7)


def test_combine_fp8_hand_derived_examples(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "combine_fp8_hand_example.json")))
    H = g["H"]
    for case in g["cases"]:
        k = len(case["codes"])
        q = np.zeros((k, H), np.uint8)
        q[:, 0] = [c[0] for c in case["codes"]]
        s = np.array(case["scales"], np.float32).reshape(k, 1)
        sm = np.arange(k, dtype=np.int32)
        if case.get("drop_second"):
            sm[1] = -1
        out = oracle.combine_fp8(sm, 1, k, q, s, np.array([case["weights"]], np.float32))
        assert int(out[0, 0]) == case["out_bf16"], case["note"]
        assert np.all(out[0, 1:] == 0)


def test_combine_fp8_with_power_of_two_scales_is_the_bf16_combine_of_the_decoded_values():
    # With a power-of-two scale, decode(q) * scale is exact and fits bf16
    # (3 mantissa bits in 7), so the FP8 combine must equal the bf16 combine
    # of those values.  The decode here is torch's, not the oracle's, and
    # every 128-column block gets its own scale.
    rng = np.random.default_rng(41)
    T, k, E, H = 40, 6, 16, 384
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)
    idx[rng.random((T, k)) < 0.15] = -1
    lay = oracle.layout(idx, E, 4, 8)
    rows = lay["max_rows"]
    q = _e4m3_codes(rng, (rows, H))
    s = np.exp2(rng.integers(-8, 9, size=(rows, H // 128))).astype(np.float32)
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    vals = dec * np.repeat(s, 128, axis=1)
    y = bf16_bits_of(vals)
    assert np.array_equal(f32_of_bf16(y), vals)          # exact in bf16
    wts = rng.standard_normal((T, k)).astype(np.float32)
    for weights in (wts, None):
        ref, _ = oracle.combine(lay["slot_map"], T, k, y, weights)
        got = oracle.combine_fp8(lay["slot_map"], T, k, q, s, weights)
        assert np.array_equal(got, ref)


def test_combine_fp8_equals_exact_rational_chain_with_general_scales():
    # Arbitrary binary32 scales: the product decode(q) * scale rounds once
    # to binary32, then each FMA rounds once; bf16 at the end.
    rng = np.random.default_rng(43)
    T, k, E, H = 8, 4, 6, 256
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)
    idx[rng.random((T, k)) < 0.2] = -1
    lay = oracle.layout(idx, E, 2, 2)
    rows = lay["max_rows"]
    q = _e4m3_codes(rng, (rows, H))
    s = (rng.uniform(0.5, 2.0, (rows, H // 128)) * 10.0 ** rng.integers(-3, 3, (rows, H // 128))).astype(np.float32)
    dec = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    wts = (rng.standard_normal((T, k)) * 2).astype(np.float32)
    got = oracle.combine_fp8(lay["slot_map"], T, k, q, s, wts)
    exp = np.empty((T, H), np.float32)
    for t in range(T):
        for h in range(H):
            acc = Fraction(0)
            for j in range(k):
                r = lay["slot_map"][t * k + j]
                if r < 0:
                    continue
                v = round_fraction(Fraction(float(dec[r, h])) * Fraction(float(s[r, h // 128])), 24)
                acc = round_fraction(Fraction(float(wts[t, j])) * v + acc, 24)
            exp[t, h] = float(round_fraction(acc, 8))
    assert np.array_equal(got, bf16_bits_of(exp))


def test_combine_fp8_of_the_fp8_dispatch_returns_the_dequantised_rows():
    # dispatch (bf16 -> FP8) followed by the unweighted FP8 combine with one
    # valid slot per token: each token gets back bf16(decode(q) * scale) of
    # its own row, which is within the FP8 quantisation error of x.
    rng = np.random.default_rng(47)
    T, E, H = 64, 8, 256
    idx = np.full((T, 2), -1, np.int64)
    idx[:, 0] = rng.integers(0, E, T)
    lay = oracle.layout(idx, E, 1, 1)
    x = bf16_bits_of(rng.standard_normal((T, H)) * 10.0 ** rng.uniform(-2, 2, (T, 1)))
    rq, rs = oracle.dispatch(lay, x, oracle.X_BF16_QUANT_FP8)
    out = oracle.combine_fp8(lay["slot_map"], T, 2, rq, rs)
    qt, st = oracle.quantize_rows(x)
    dec = torch.from_numpy(qt).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    deq = (dec * np.repeat(st, 128, axis=1)).astype(np.float32)
    assert np.array_equal(out, bf16_bits_of(deq))
    xf = f32_of_bf16(x)
    assert np.all(np.abs(f32_of_bf16(out) - xf) <= np.repeat(st, 128, axis=1) * 16 + np.abs(xf) * 2.0 ** -8)


def test_combine_near_cancellation_equals_exact_rational_fma_chain():
    # Sums that nearly cancel: the result is tiny next to its terms, so every
    # binary32 rounding step, and the order of the steps, reaches the bf16
    # output.  Each token's last weight is chosen to cancel the others.
    rng = np.random.default_rng(17)
    T, k, H, E = 64, 4, 8, 16
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)
    lay = oracle.layout(idx, E, 1, 1)
    y = bf16_bits_of(rng.uniform(0.5, 2.0, (lay["max_rows"], H)) * rng.choice([-1, 1], (lay["max_rows"], H)))
    yf = f32_of_bf16(y).astype(np.float64)
    sm = lay["slot_map"].reshape(T, k)
    w = rng.uniform(-2, 2, (T, k)).astype(np.float32)
    for t in range(T):           # w[t,k-1] * y[last, 0] ~ -(sum of the others at column 0)
        part = sum(float(w[t, j]) * yf[sm[t, j], 0] for j in range(k - 1))
        w[t, k - 1] = np.float32(-part / yf[sm[t, k - 1], 0] * (1 + rng.uniform(-1e-5, 1e-5)))
    out, _ = oracle.combine(lay["slot_map"], T, k, y, w)
    exp = np.empty((T, H), np.float32)
    for t in range(T):
        for h in range(H):
            acc = Fraction(0)
            for j in range(k):
                acc = round_fraction(Fraction(float(w[t, j])) * Fraction(float(yf[sm[t, j], h])) + acc, 24)
            exp[t, h] = float(round_fraction(acc, 8))
    assert np.array_equal(out, bf16_bits_of(exp))
    # the case is sensitive: two roundings per step, or the reverse order, changes the bf16 result
    twice = np.empty(T, np.float32)
    for t in range(T):
        acc = Fraction(0)
        for j in range(k):
            acc = round_fraction(round_fraction(Fraction(float(w[t, j])) * Fraction(float(yf[sm[t, j], 0])), 24) + acc, 24)
        twice[t] = float(round_fraction(acc, 8))
    assert not np.array_equal(bf16_bits_of(twice), out[:, 0])


def test_combine_of_identity_outputs_returns_x():
    w = W.WORKLOADS["mid"]
    inp = W.make_inputs(w, seed=3, T=256)
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    y, _ = oracle.dispatch(lay, inp["x"], oracle.X_BF16)      # every expert is the identity
    sm = lay["slot_map"].reshape(256, w.k)
    wts = np.where(sm >= 0, inp["topk_weights"], 0).astype(np.float64)
    wts = (wts / np.maximum(wts.sum(axis=1, keepdims=True), 1e-30)).astype(np.float32)
    out, _ = oracle.combine(lay["slot_map"], 256, w.k, y, wts)
    x = f32_of_bf16(inp["x"]).astype(np.float64)
    o = f32_of_bf16(out).astype(np.float64)
    has = (sm >= 0).any(axis=1)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126))) - 7)
    assert np.all(np.abs(o - x)[has] <= ulp[has])
    assert np.all(o[~has] == 0)


def test_dispatch_and_unweighted_combine_are_adjoint():
    # small integers: every sum is exact, so the two inner products must agree exactly
    rng = np.random.default_rng(9)
    T, k, E, H, a = 40, 4, 10, 16, 3
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)
    idx[rng.random((T, k)) < 0.15] = -1
    lay = oracle.layout(idx, E, 5, a)
    x = rng.integers(-8, 9, size=(T, H)).astype(np.float32)
    g = rng.integers(-8, 9, size=(lay["max_rows"], H)).astype(np.float32)
    dx, _ = oracle.dispatch(lay, bf16_bits_of(x), oracle.X_BF16)
    cg, _ = oracle.combine(lay["slot_map"], T, k, bf16_bits_of(g), None)
    R = lay["R"]
    lhs = int((f32_of_bf16(dx)[:R].astype(np.int64) * g[:R].astype(np.int64)).sum())
    rhs = int((x.astype(np.int64) * f32_of_bf16(cg).astype(np.int64)).sum())
    assert lhs == rhs


def test_fp8_dispatch_then_combine_matches_dequantised_x():
    w = W.WORKLOADS["mid"]
    inp = W.make_inputs(w, seed=4, T=128)
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    rq, rs = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8)
    deq = oracle.e4m3_decode(rq).reshape(rq.shape[0], -1, 128) * rs[..., None]
    y = bf16_bits_of(deq.reshape(rq.shape[0], -1))
    sm = lay["slot_map"].reshape(128, w.k)
    wts = np.where(sm >= 0, 1.0, 0.0)
    wts = (wts / np.maximum(wts.sum(axis=1, keepdims=True), 1)).astype(np.float32)
    out, _ = oracle.combine(lay["slot_map"], 128, w.k, y, wts)
    q, s = oracle.quantize_rows(inp["x"])
    ref = f32_of_bf16(bf16_bits_of((oracle.e4m3_decode(q).reshape(128, -1, 128) * s[..., None])
                                   .reshape(128, -1))).astype(np.float64)
    o = f32_of_bf16(out).astype(np.float64)
    has = (sm >= 0).any(axis=1)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    assert np.all(np.abs(o - ref)[has] <= ulp[has])


def test_combine_token_with_no_valid_slot_is_positive_zero():
    idx = np.full((2, 3), -1, np.int64)
    idx[1, 1] = 0
    lay = oracle.layout(idx, 2, 1, 1)
    y = bf16_bits_of(np.full((lay["max_rows"], 8), -2.5))
    out, ow = oracle.combine(lay["slot_map"], 2, 3, y, np.ones((2, 3), np.float32),
                             np.full(lay["max_rows"], 7.0, np.float32), True)
    assert np.all(out[0] == 0x0000)
    assert np.all(f32_of_bf16(out[1]) == -2.5)
    assert ow.tolist() == [[0, 0, 0], [0, 7.0, 0]]


# ------------------------------------------------------ combine backward

def test_combine_backward_matches_library_gather_and_dot():
    rng = np.random.default_rng(23)
    T, k, H, E, a = 48, 4, 64, 12, 3
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)
    idx[rng.random((T, k)) < 0.2] = -1
    w = rng.standard_normal((T, k)).astype(np.float32)
    lay = oracle.layout(idx, E, 4, a, w)
    g = bf16_bits_of(rng.standard_normal((T, H)))
    y = bf16_bits_of(rng.standard_normal((lay["max_rows"], H)))
    gy, gw = oracle.combine_backward(lay, g, y, w)
    R, sm = lay["R"], lay["slot_map"].reshape(T, k)
    gf, yf = f32_of_bf16(g), f32_of_bf16(y)
    for t in range(T):
        for j in range(k):
            r = sm[t, j]
            if r < 0:
                assert gw[t, j] == 0.0
                continue
            # numpy binary32 multiply, torch's bf16 cast
            assert np.array_equal(gy[r], bf16_bits_of(np.float32(w[t, j]) * gf[t]))
            assert np.isclose(gw[t, j], np.dot(gf[t].astype(np.float64), yf[r].astype(np.float64)),
                              rtol=1e-12, atol=1e-12)
    pad = lay["recv_src"][:R] < 0
    assert np.all(gy[:R][pad] == 0)
    assert np.all(gy[R:] == oracle.UNWRITTEN * 0x0101)


def test_combine_backward_is_the_derivative_of_the_weighted_combine():
    # small integers: every value and sum is exact, so finite differences are exact
    rng = np.random.default_rng(29)
    T, k, H, E, a = 20, 3, 16, 7, 2
    idx = rng.integers(0, E, size=(T, k)).astype(np.int64)
    idx[rng.random((T, k)) < 0.15] = -1
    w = rng.integers(-3, 4, size=(T, k)).astype(np.float32)
    lay = oracle.layout(idx, E, 1, a, w)
    y = bf16_bits_of(rng.integers(-4, 5, size=(lay["max_rows"], H)))
    g = bf16_bits_of(rng.integers(-4, 5, size=(T, H)))
    gf = f32_of_bf16(g).astype(np.int64)

    def loss(weights):      # <combine(y, weights), g>
        out, _ = oracle.combine(lay["slot_map"], T, k, y, weights)
        return int((f32_of_bf16(out).astype(np.int64) * gf).sum())

    gy, gw = oracle.combine_backward(lay, g, y, w)
    base = loss(w)
    for t in range(T):
        for j in range(k):
            w2 = w.copy()
            w2[t, j] += 1.0
            assert loss(w2) - base == gw[t, j]          # d loss / d w[t,j]
    # adjoint in y: <combine(y), g> = <y, grad_y> over the real rows
    R = lay["R"]
    real = lay["recv_src"][:R] >= 0
    lhs = int((f32_of_bf16(y)[:R][real].astype(np.int64) * f32_of_bf16(gy)[:R][real].astype(np.int64)).sum())
    assert lhs == base


# ------------------------------------------------------------- workloads

def test_workloads_are_seeded_and_shaped():
    for name, w in W.WORKLOADS.items():
        T = min(w.T, 256)
        a = W.make_inputs(w, seed=1, T=T)
        b = W.make_inputs(w, seed=1, T=T)
        for key in a:
            assert np.array_equal(a[key], b[key])
        assert a["x"].shape == (T, w.H) and a["topk_idx"].shape == (T, w.k)
        idx = a["topk_idx"]
        for t in range(T):
            v = idx[t][idx[t] >= 0]
            assert len(set(v.tolist())) == len(v)          # distinct experts per token
        assert np.all((idx >= -1) & (idx < w.E))
        assert np.allclose(a["topk_weights"].sum(axis=1), 1.0, atol=1e-6)
    mid = W.make_inputs("mid")
    assert int((mid["topk_idx"] == -1).sum()) == round(0.05 * 4096 * 6)


def test_skewed_workload_is_skewed_and_has_outliers():
    v3 = W.make_inputs("v3", T=2048)
    sk = W.make_inputs("skewed", T=2048)
    c_u = np.bincount(v3["topk_idx"].reshape(-1), minlength=256)
    c_s = np.bincount(sk["topk_idx"].reshape(-1), minlength=256)
    assert c_s.max() > 4 * c_u.max()
    amax = np.abs(f32_of_bf16(sk["x"])).max(axis=1)
    assert int((amax > 50).sum()) == round(0.01 * 2048)
