"""Backward of the weighted combine on the GPU vs the oracle.

grad_y (binary32 product, one bf16 rounding) is compared bit for bit;
padding rows must be zero and rows >= R untouched.  grad_w is accumulated
in binary32 on the GPU in a fixed order and exactly (binary64) in the
oracle; their difference must stay within the standard error bound of
summing H products in binary32 in any order: |err| <= g_H * sum_h |g_h y_h|,
g_n = n u / (1 - n u), u = 2^-24 (each FMA rounds once)."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import SENTINEL, bits16, guarded, to_dev_bf16

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check(w: W.Workload, inp: dict, weighted: bool = True, seed: int = 0):
    T, k, H = inp["x"].shape[0], w.k, w.H
    rng = np.random.default_rng(seed)
    rows = oracle.max_recv_rows(T, k, w.E, w.align)
    g = W._to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    y = W.make_y(w, seed=seed, rows=rows)
    wts = inp["topk_weights"] if weighted else np.ones((T, k), np.float32)

    h, _, _ = ep.get_layout(torch.from_numpy(inp["topk_idx"]).cuda(), w.E, num_segments=w.S,
                            expert_alignment=w.align)
    gy_buf, gy = guarded(rows, H, torch.bfloat16)
    gw = torch.full((T, k), float("nan"), device="cuda")
    ep.combine_backward(to_dev_bf16(g), to_dev_bf16(y), h,
                        torch.from_numpy(inp["topk_weights"]).cuda() if weighted else None,
                        grad_y=gy, grad_weights=gw)
    torch.cuda.synchronize()
    assert h.check_error() == 0

    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align)
    ref_gy, ref_gw = oracle.combine_backward(lay, g, y, wts)
    R = lay["R"]
    got = bits16(gy)
    np.testing.assert_array_equal(got[:R], ref_gy[:R])
    assert np.all(got[R:] == (SENTINEL << 8 | SENTINEL))
    assert bool((gy_buf[rows * H * 2:] == SENTINEL).all())

    # grad_w within the binary32 summation bound
    sm = lay["slot_map"].reshape(T, k)
    gf = oracle.bf16_to_f32(g).astype(np.float64)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    absdot = np.zeros((T, k))
    for j in range(k):
        r = np.maximum(sm[:, j], 0)
        absdot[:, j] = np.abs(gf * yf[r]).sum(axis=1) * (sm[:, j] >= 0)
    gamma = H * U / (1 - H * U)
    err = np.abs(gw.cpu().numpy().astype(np.float64) - ref_gw)
    assert np.all(err <= gamma * absdot + 1e-30), float((err / np.maximum(absdot, 1e-30)).max())
    assert np.all(gw.cpu().numpy()[sm < 0] == 0)


@pytest.mark.parametrize("name", ["tiny", "mid", "v3"])
def test_combine_backward_on_workloads(name):
    w = W.WORKLOADS[name]
    _check(w, W.make_inputs(w, seed=5), seed=5)


def test_combine_backward_unweighted_is_a_plain_dispatch_of_the_gradient():
    w = W.WORKLOADS["mid"]
    _check(w, W.make_inputs(w, seed=6, T=700), weighted=False, seed=6)


@pytest.mark.parametrize("T,k,E,S,align,H,drop", [
    (1, 1, 1, 1, 1, 8, 0.0), (37, 3, 5, 5, 3, 136, 0.2), (300, 12, 40, 4, 16, 256, 0.1),
    (64, 32, 1024, 16, 2, 64, 0.0), (0, 4, 8, 2, 4, 128, 0.0), (257, 20, 48, 4, 7, 512, 0.3)])
def test_combine_backward_edge_shapes(T, k, E, S, align, H, drop):
    w = W.Workload("bwd", T=T, H=H, E=E, S=S, k=k, align=align, x_mode="bf16")
    rng = np.random.default_rng(T + k)
    idx = (np.stack([rng.permutation(E)[:k] for _ in range(T)]) if T else np.zeros((0, k))).astype(np.int64)
    idx[rng.random((T, k)) < drop] = -1
    inp = {"x": np.zeros((T, H), np.uint16), "topk_idx": idx,
           "topk_weights": rng.standard_normal((T, k)).astype(np.float32)}
    _check(w, inp, seed=T + k)
