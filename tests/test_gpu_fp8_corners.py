"""FP8 1x128 quantising dispatch on the GPU at the format's corners, bit for
bit against the CPU oracle.

The workload tests draw x from N(0,1) (plus x100 rows), which never reach
the corners of the block quantiser (FP8 dispatch, DeepEP V2 README
"Performance"; per-block scale: amax floored at 1e-4, scale = amax/448,
q = e4m3_rn_satfinite(x * (448/amax))).  Here every block is built to hit
one: all +0, all -0, mixed signed zeros, amax below and around the floor,
constant blocks, values whose scaled value x*inv falls exactly on an e4m3
midpoint (ties both ways, and the two hand-derived blocks of
tests/golden/fp8_quant_product_form.json), e4m3 subnormal outputs, amax at
the bf16 maximum, one dominant element over tiny ones, and every finite
bf16 value in [-448, 448] with amax = 448 (inv = 1, so the hardware e4m3
conversion itself is compared with the oracle's encoder on every bf16
input).  Codes and scale bits must equal the oracle's for every written
row, through the two-call and the one-call path."""

import dataclasses
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import assert_parity, run_cuda, run_cuda_one_call, run_oracle

pytestmark = pytest.mark.gpu

H = 1024                       # 8 blocks of 128 per row
NB = H // 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_quant_product_form.json")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _bf16_values(lo: float, hi: float) -> np.ndarray:
    """Every finite non-negative bf16 value in [lo, hi], ascending, as float32."""
    u = np.arange(0, 0x7F80, dtype=np.uint32) << 16
    v = u.view(np.float32)
    return v[(v >= lo) & (v <= hi)]


def _e4m3_midpoints() -> set:
    """Exact midpoints between adjacent non-negative e4m3 values (as Fractions)."""
    vals = sorted({Fraction(float(oracle.e4m3_decode(np.array([c], np.uint8))[0])) for c in range(0x7F)})
    return {(a + b) / 2 for a, b in zip(vals, vals[1:])}


def _midpoint_blocks() -> list:
    """Blocks [amax, x1, x2, ...] whose x*448/amax is exactly an e4m3 midpoint."""
    mids = _e4m3_midpoints()
    xs = _bf16_values(2.0 ** -12, 64.0)
    blocks = []
    for amax in (3.25, 3.875, 0.8125, 1.9375, 6.5, 7.0, 1.5, 0.375, 12.0, 48.0):
        fa = Fraction(amax)
        hits = [float(x) for x in xs if x <= amax and Fraction(float(x)) * 448 / fa in mids]
        for i in range(0, len(hits), 63):
            part = hits[i:i + 63]
            blocks.append([amax] + part + [-v for v in part])
    return blocks


def _exhaustive_blocks() -> list:
    """Every finite bf16 value in [-448, 448], 127 to a block after amax = 448."""
    pos = _bf16_values(0.0, 448.0)
    allv = np.concatenate([pos, -pos[1:], np.array([-0.0], np.float32)])
    return [[448.0] + list(allv[i:i + 127]) for i in range(0, allv.size, 127)]


def corner_rows() -> np.ndarray:
    rng = np.random.default_rng(21)
    blocks = []
    blocks.append([0.0] * 128)                                            # all +0
    blocks.append([-0.0] * 128)                                           # all -0
    blocks.append([0.0, -0.0] * 64)                                       # mixed signed zeros
    blocks.append(list(1e-6 * rng.standard_normal(128)))                  # amax far below the floor
    blocks.append(list(np.full(128, 9.98e-5) * rng.choice([-1, 1], 128)))  # amax just below 1e-4
    blocks.append(list(np.full(128, 1.0014e-4) * rng.choice([-1, 1], 128)))  # just above
    blocks.append([3.0] * 128)                                            # constant
    blocks.append([-0.7] * 128)
    blocks.append([448.0] * 128)
    blocks.append([3.3895313892515355e38] + list(rng.standard_normal(127) * 1e37))  # amax = bf16 max
    blocks.append([-3.3895313892515355e38] * 128)
    blocks.append([100.0] + list(0.5 * rng.standard_normal(127)))         # dominant element: subnormal codes
    blocks.append([1e4] + list(1e-3 * rng.standard_normal(127)))          # ... and underflow to +-0
    blocks.append([1.0] + list(np.exp2(-rng.uniform(9, 16, 127)) * rng.choice([-1, 1], 127)))
    g = json.load(open(GOLDEN))
    blocks += [list(v) for v in g["x"]]                                   # hand-derived midpoint blocks
    blocks += _midpoint_blocks()
    blocks += _exhaustive_blocks()
    rows = -(-len(blocks) // NB)
    x = np.zeros((rows * NB, 128), np.float32)
    for i, b in enumerate(blocks):
        x[i, :len(b)] = np.asarray(b, np.float32)
    x = x.reshape(rows, H)
    return W._to_bf16_bits(x)


def _workload(T: int) -> W.Workload:
    return dataclasses.replace(W.WORKLOADS["tiny"], name="fp8_corners", T=T, H=H, align=4,
                               x_mode="fp8_quant")


def test_corner_rows_are_what_they_claim():
    # host-side check of the construction (no oracle arithmetic): the
    # golden blocks are present and bf16-exact, the exhaustive part covers
    # every finite bf16 value of magnitude <= 448
    x = corner_rows()
    f = (x.astype(np.uint32) << 16).view(np.float32).reshape(-1, 128)
    g = json.load(open(GOLDEN))
    for vals in g["x"]:
        assert any(np.array_equal(b[:len(vals)], np.float32(vals)) for b in f)
    mag = np.unique(np.abs(f[f[:, 0] == 448.0][:, 1:]))
    assert mag.size == _bf16_values(0.0, 448.0).size
    assert len(_midpoint_blocks()) >= 10


@pytest.mark.parametrize("one_call", [False, True])
def test_fp8_corner_blocks_match_oracle_bit_exactly(one_call):
    x = corner_rows()
    w = _workload(x.shape[0])
    inp = W.make_inputs(w, seed=22)
    inp["x"] = x
    if one_call:
        g = run_cuda_one_call(inp, w, ep.EP_X_BF16_TO_FP8)
    else:
        g = run_cuda(inp, w, None, ep.EP_X_BF16_TO_FP8)
    o = run_oracle(inp, w, None, oracle.X_BF16_QUANT_FP8)
    assert_parity(g, o, oracle.X_BF16_QUANT_FP8)


def test_fp8_golden_blocks_on_the_gpu():
    # the two hand-derived blocks, checked against the golden codes directly
    g = json.load(open(GOLDEN))
    x = np.zeros((1, H), np.float32)
    for b, vals in enumerate(g["x"]):
        x[0, b * 128:b * 128 + len(vals)] = vals
    w = _workload(1)
    w = dataclasses.replace(w, k=1)
    inp = W.make_inputs(w, seed=23)
    inp["x"] = W._to_bf16_bits(x)
    inp["topk_idx"][:] = 0
    res = run_cuda(inp, w, None, ep.EP_X_BF16_TO_FP8)
    row = int(res["slot_map"][0])
    assert row >= 0
    for b, codes in enumerate(g["codes"]):
        assert list(res["recv_x"][row, b * 128:b * 128 + len(codes)]) == codes
        m, e = g["scales_exact"][b]
        assert Fraction(float(res["recv_scales"][row, b])) == Fraction(m) * Fraction(2) ** e
