"""The FP8 combine on the GPU vs the CPU oracle, bit for bit.

Expert outputs arrive as e4m3 codes with one f32 scale per 1x128 block
(the FP8 dispatch's output layout).  The output must equal the oracle's
for every token at the full size of every workload, weighted and
unweighted, for top-k up to 32 (all four slot-group instances).  Padding
rows, and rows past the total, hold NaN codes: reading one would show up
as a NaN in the output."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def fp8_outputs(lay, H, seed):
    """Random FP8 expert outputs for every valid row; NaN codes elsewhere."""
    rows = lay["max_rows"]
    q, s = W.make_prequant(rows, H, seed=seed)
    unused = lay["recv_src"] < 0            # padding rows and rows >= R
    q[unused] = 0x7F
    return q, s


def run(w: W.Workload, inp, q, s, weighted=True):
    idx = torch.from_numpy(inp["topk_idx"]).cuda()
    wts = torch.from_numpy(inp["topk_weights"]).cuda() if weighted else None
    h, _, _ = ep.get_layout(idx, w.E, num_segments=w.S, expert_alignment=w.align)
    out = ep.combine_fp8(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda(), h, wts)
    torch.cuda.synchronize()
    assert h.check_error() == 0
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", ["v3", "skewed", "mid", "decode"])
def test_combine_fp8_matches_oracle_bit_exactly(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=31)
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align)
    q, s = fp8_outputs(lay, w.H, seed=32)
    for weighted in (True, False):
        got = run(w, inp, q, s, weighted)
        exp = oracle.combine_fp8(lay["slot_map"], w.T, w.k, q, s, inp["topk_weights"] if weighted else None)
        assert not np.any(np.isnan(oracle.bf16_to_f32(got)))
        np.testing.assert_array_equal(got, exp)


@pytest.mark.parametrize("k,E,H", [(12, 64, 256), (20, 40, 128), (32, 1024, 384), (1, 3, 128)])
def test_combine_fp8_topk_groups_and_shapes(k, E, H):
    w = W.Workload("fp8c", T=700, H=H, E=E, S=1, k=k, align=8, x_mode="fp8_quant")
    rng = np.random.default_rng(k * 7 + E)
    idx = np.stack([rng.permutation(E)[:k] if k <= E else rng.integers(0, E, k) for _ in range(w.T)])
    idx = idx.astype(np.int64)
    idx[rng.random(idx.shape) < 0.1] = -1
    inp = {"topk_idx": idx, "topk_weights": rng.standard_normal((w.T, k)).astype(np.float32)}
    lay = oracle.layout(idx, E, 1, 8)
    q, s = fp8_outputs(lay, H, seed=k)
    got = run(w, inp, q, s)
    np.testing.assert_array_equal(got, oracle.combine_fp8(lay["slot_map"], w.T, k, q, s, inp["topk_weights"]))


def test_fp8_dispatch_then_fp8_combine():
    # the FP8 dispatch's output fed straight to the FP8 combine: the token
    # gets back the weighted sum of its dequantised rows
    w = W.WORKLOADS["v3"]
    inp = W.make_inputs(w, seed=33, T=2048)
    idx = torch.from_numpy(inp["topk_idx"]).cuda()
    wts = torch.from_numpy(inp["topk_weights"]).cuda()
    (rq, rs), _, _, h = ep.dispatch(to_dev_bf16(inp["x"]), idx, wts, w.E, expert_alignment=w.align,
                                    num_segments=w.S, use_fp8=True)
    out = ep.combine_fp8(rq, rs, h, wts)
    torch.cuda.synchronize()
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    oq, os_ = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8)
    exp = oracle.combine_fp8(lay["slot_map"], 2048, w.k, oq, os_, inp["topk_weights"])
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), exp)


def test_combine_fp8_empty_and_bad_arguments():
    w = dataclasses.replace(W.WORKLOADS["mid"], T=0)
    h = ep.EPHandle(0, w.k, w.E, w.S, w.align, device="cuda")
    ep.get_layout(torch.zeros(0, w.k, dtype=torch.int64, device="cuda"), w.E, num_segments=w.S,
                  expert_alignment=w.align, handle=h)
    rows = h.max_recv_rows
    out = ep.combine_fp8(torch.zeros(rows, 256, dtype=torch.uint8, device="cuda"),
                         torch.ones(rows, 2, dtype=torch.float32, device="cuda"), h)
    assert out.shape == (0, 256)
    q = torch.zeros(rows, 200, dtype=torch.uint8, device="cuda")
    s = torch.ones(rows, 1, dtype=torch.float32, device="cuda")
    with pytest.raises(ep.EPError):          # the library refuses: hidden not a multiple of 128
        ep.combine_fp8(q, s, h)
    st = ep.lib().ep_combine_fp8(h.ref, q.data_ptr(), s.data_ptr(), 200, None, None, None)
    assert st == 1   # EP_ERR_INVALID_ARG, nothing launched
    with pytest.raises(ValueError):          # the binding refuses a scale array of the wrong shape
        ep.combine_fp8(torch.zeros(rows, 256, dtype=torch.uint8, device="cuda"), s, h)
