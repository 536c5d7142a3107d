"""GEMM-ready outputs: FP8 dispatch with MN-major block scales
(ep_dispatch_mn_scales) and the per-expert row counts on the host.  The
scales must equal the oracle's row-major scales transposed, bit for bit;
entries for rows >= R and the column tails are not written."""

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


@pytest.mark.parametrize("name,T,prequant", [("v3", None, False), ("mid", None, False), ("mid", 999, True),
                                             ("decode", None, False)])
def test_mn_major_scales_are_the_row_major_scales_transposed(name, T, prequant):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=8, T=T)
    T = inp["x"].shape[0]
    h, _, _ = ep.get_layout(torch.from_numpy(inp["topk_idx"]).cuda(), w.E, num_segments=w.S,
                            expert_alignment=w.align)
    rows, B = h.max_recv_rows, w.H // 128
    ld = (rows + 3) // 4 * 4 + 4                     # a column tail that must stay untouched
    sc = torch.full((B, ld), float("nan"), device="cuda")
    if prequant:
        pq = W.make_prequant(T, w.H, seed=8)
        xin = (torch.from_numpy(pq[0]).cuda(), torch.from_numpy(pq[1]).cuda())
    else:
        xin = to_dev_bf16(inp["x"])
    rx, _ = ep.dispatch_mn_scales(xin, h, recv_scales_mn=sc, scales_ld=ld)
    torch.cuda.synchronize()
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align)
    if prequant:
        q, s = oracle.dispatch(lay, pq[0], oracle.X_FP8_PREQUANT, pq[1])
    else:
        q, s = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8)
    R = lay["R"]
    got = sc.cpu().numpy()
    np.testing.assert_array_equal(rx.view(torch.uint8).cpu().numpy()[:R], q[:R])
    np.testing.assert_array_equal(got[:, :R].view(np.uint32), s[:R].T.copy().view(np.uint32))
    assert np.all(np.isnan(got[:, R:]))
    assert h.recv_counts_host() == np.diff(lay["offsets"]).tolist()
    assert h.check_error() == 0


def test_mn_major_scales_reject_bad_leading_dimension():
    w = W.WORKLOADS["tiny"]
    h = ep.EPHandle(64, 2, 16, 4, 8)
    x = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ep.EPError, match="scales_ld"):
        ep.dispatch_mn_scales(x, h, scales_ld=h.max_recv_rows + 2)
