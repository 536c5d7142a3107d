"""CUDA path vs the CPU oracle, element by element, on the same seeded inputs.

Layout, counts, slot maps, recv_topk_idx / weights, FP8 bytes and scales
are compared bit for bit; so is combine (its accumulation order is fixed:
fp32 FMA in ascending j, one bf16 rounding).  Every workload runs at its
full size in the launch configuration the benchmark times, and every
output buffer carries guard bytes that must stay untouched."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import (assert_parity, bits16, max_bf16_ulp_diff, run_cuda, run_oracle,
                         to_dev_bf16)

pytestmark = pytest.mark.gpu

MODE = {"bf16": ep.EP_X_BF16, "fp8_quant": ep.EP_X_BF16_TO_FP8}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("name", ["tiny", "mid", "v3", "skewed", "decode"])
def test_workload_matches_oracle_bit_exactly(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=0)
    y = W.make_y(w, seed=0)
    mode = MODE[w.x_mode]
    g = run_cuda(inp, w, y, mode)
    o = run_oracle(inp, w, y, mode)
    assert max_bf16_ulp_diff(g["combined"], o["combined"]) <= 1     # stated fallback bound
    assert_parity(g, o, mode)                                          # and in fact bit-exact


@pytest.mark.parametrize("name", ["mid", "v3"])
def test_int32_topk_idx_gives_the_same_layout(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=5, T=1000)
    g64 = run_cuda(inp, w, None, MODE[w.x_mode])
    g32 = run_cuda(inp, w, None, MODE[w.x_mode], idx_int32=True)
    for key in ("slot_map", "recv_src", "offsets", "counts", "seg_tokens", "recv_x"):
        np.testing.assert_array_equal(g64[key], g32[key])


def test_prequantised_fp8_tuple_is_copied():
    w = W.WORKLOADS["mid"]
    inp = W.make_inputs(w, seed=6)
    pq = W.make_prequant(w.T, w.H, seed=6)
    g = run_cuda(inp, w, None, ep.EP_X_FP8, prequant=pq)
    o = run_oracle(inp, w, None, oracle.X_FP8_PREQUANT, prequant=pq)
    assert_parity(g, o, oracle.X_FP8_PREQUANT)


def test_bf16_dispatch_at_v3_shape_and_unweighted_combine_with_weight_gradient():
    # combine_backward (bf16 dispatch) and dispatch_backward (unweighted combine
    # plus the recv_topk_weights gradient gathered back to [T, k])
    w = W.WORKLOADS["v3"]
    inp = W.make_inputs(w, seed=7, T=2048)
    y = W.make_y(w, seed=7, rows=oracle.max_recv_rows(2048, w.k, w.E, w.align))
    rwi = np.random.default_rng(7).standard_normal(y.shape[0]).astype(np.float32)
    g = run_cuda(inp, w, y, ep.EP_X_BF16, weighted=False, recv_weights_in=rwi)
    o = run_oracle(inp, w, y, oracle.X_BF16, weighted=False, recv_weights_in=rwi)
    assert_parity(g, o, oracle.X_BF16)


EDGE = [
    # T, k, E, S, align, H, mode, drop
    (1, 1, 1, 1, 1, 8, "bf16", 0.0),
    (37, 3, 5, 5, 3, 136, "bf16", 0.1),         # ragged row: 17 items
    (300, 2, 16, 4, 1, 384, "fp8_quant", 0.2),   # 24 items per row
    (513, 6, 64, 8, 128, 896, "fp8_quant", 0.05),
    (1000, 12, 96, 12, 16, 256, "fp8_quant", 0.3),   # k > 8: two slot groups
    (257, 20, 40, 4, 7, 128, "fp8_quant", 0.0),      # three slot groups
    (64, 32, 1024, 16, 2, 128, "bf16", 0.0),         # k = 32, E = 1024
    (5000, 4, 1024, 1024, 1, 64, "bf16", 0.0),       # many chunks, S = E
    (3000, 8, 8, 2, 512, 512, "fp8_quant", 0.0),     # alignment larger than most counts
    (2049, 1, 3, 1, 5, 1024, "fp8_quant", 1.0),      # every slot dropped
    (131072, 8, 256, 8, 128, 128, "fp8_quant", 0.01),  # 1M slots: 1024 layout chunks
    (65536, 8, 1024, 32, 16, 64, "bf16", 0.0),        # 512 chunks x 1024 experts
    # the dispatch's slices of 1024 elements: many slices, a short last slice,
    # each on the warp-unit path (T*k > 1024) and on the row path (T*k <= 1024)
    (300, 4, 32, 4, 8, 16512, "fp8_quant", 0.05),   # 17 slices, the last of 128 elements
    (60, 4, 32, 4, 8, 16512, "fp8_quant", 0.05),    # row path: a 16.5 KB row buffer
    (600, 3, 16, 2, 4, 9224, "bf16", 0.0),          # bf16: 10 slices, the last of 8 elements
    (90, 3, 16, 2, 4, 9224, "bf16", 0.0),           # row path
    (700, 2, 16, 4, 1, 24, "bf16", 0.1),            # a single slice of 24 elements (3 lanes)
    # the combine's unit sizes: two 448-thread units a row with k > 8 (two slot
    # groups), and 128-thread units for a one-wave batch
    (200, 12, 64, 4, 8, 7168, "bf16", 0.1),
    (24, 12, 64, 4, 8, 7168, "fp8_quant", 0.1),
]


@pytest.mark.parametrize("T,k,E,S,align,H,xm,drop", EDGE)
def test_edge_shapes(T, k, E, S, align, H, xm, drop):
    w = W.Workload("edge", T=T, H=H, E=E, S=S, k=k, align=align, x_mode=xm)
    rng = np.random.default_rng(T * 31 + k)
    idx = np.stack([rng.permutation(E)[:k] if k <= E else rng.integers(0, E, k) for _ in range(T)])
    idx = idx.astype(np.int64)
    idx[rng.random((T, k)) < drop] = -1
    inp = {"x": W._to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32)),
           "topk_idx": idx,
           "topk_weights": rng.standard_normal((T, k)).astype(np.float32)}
    y = W._to_bf16_bits(rng.standard_normal((oracle.max_recv_rows(T, k, E, align), H))
                        .astype(np.float32))
    mode = MODE[xm]
    g = run_cuda(inp, w, y, mode)
    o = run_oracle(inp, w, y, mode)
    assert_parity(g, o, mode)


def test_duplicate_experts_within_a_token_each_get_a_row():
    w = W.Workload("dup", T=100, H=256, E=4, S=2, k=6, align=4, x_mode="fp8_quant")
    rng = np.random.default_rng(1)
    inp = {"x": W._to_bf16_bits(rng.standard_normal((100, 256)).astype(np.float32)),
           "topk_idx": rng.integers(-1, 4, size=(100, 6)).astype(np.int64),
           "topk_weights": rng.random((100, 6)).astype(np.float32)}
    y = W._to_bf16_bits(rng.standard_normal((oracle.max_recv_rows(100, 6, 4, 4), 256))
                        .astype(np.float32))
    g = run_cuda(inp, w, y, ep.EP_X_BF16_TO_FP8)
    o = run_oracle(inp, w, y, oracle.X_BF16_QUANT_FP8)
    assert_parity(g, o, oracle.X_BF16_QUANT_FP8)


def test_bad_topk_idx_sets_the_error_word_and_is_dropped():
    w = W.Workload("bad", T=600, H=128, E=16, S=4, k=4, align=8, x_mode="fp8_quant")
    inp = W.make_inputs(W.WORKLOADS["tiny"], seed=3, T=600)
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 16, size=(600, 4)).astype(np.int64)
    idx[5, 1], idx[300, 0], idx[599, 3] = 16, -2, 1 << 40
    inp = {"x": W._to_bf16_bits(rng.standard_normal((600, 128)).astype(np.float32)),
           "topk_idx": idx, "topk_weights": inp["topk_weights"][:600, :1].repeat(4, axis=1)}
    g = run_cuda(inp, w, None, ep.EP_X_BF16_TO_FP8)
    o = run_oracle(inp, w, None, oracle.X_BF16_QUANT_FP8)
    assert o["lay"]["flags"] == 1
    assert_parity(g, o, oracle.X_BF16_QUANT_FP8)
    with pytest.raises(ep.EPError, match="topk_idx"):
        g["handle"].check_error()
    assert g["handle"].check_error() == 0            # read-and-clear


def test_empty_batch():
    h, ri, rw = ep.get_layout(torch.empty(0, 8, dtype=torch.int64, device="cuda"), 32,
                              num_segments=4, expert_alignment=16)
    recv = ep.dispatch_with_handle(torch.empty(0, 256, dtype=torch.bfloat16, device="cuda"), h,
                                   use_fp8=True)
    out, _ = ep.combine(torch.zeros(h.max_recv_rows, 256, dtype=torch.bfloat16, device="cuda"), h)
    torch.cuda.synchronize()
    assert h.total_rows() == 0 and out.shape == (0, 256)
    assert int(h.counts.sum()) == 0 and int(h.seg_tokens.sum()) == 0 and int(h.num_pad_rows) == 0


def test_cached_handle_reuse_and_relayout():
    w = W.WORKLOADS["mid"]
    a = W.make_inputs(w, seed=21, T=1500)
    b = W.make_inputs(w, seed=22, T=1500)
    h = ep.EPHandle(1500, w.k, w.E, w.S, w.align)
    for inp in (a, b, a):
        ep.get_layout(torch.from_numpy(inp["topk_idx"]).cuda(), w.E, num_segments=w.S,
                      expert_alignment=w.align, handle=h)
        x = to_dev_bf16(inp["x"])
        r1 = ep.dispatch_with_handle(x, h, use_fp8=True)
        r2 = ep.dispatch_with_handle(x, h, use_fp8=True)         # cached handle, no new layout
        lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align)
        rq, rs = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_FP8)
        R = lay["R"]
        for q, s in (r1, r2):
            np.testing.assert_array_equal(q.view(torch.uint8).cpu().numpy()[:R], rq[:R])
            np.testing.assert_array_equal(s.cpu().numpy()[:R], rs[:R])
        np.testing.assert_array_equal(h.slot_map.cpu().numpy(), lay["slot_map"])


def test_decode_pairs_in_a_cuda_graph():
    w = W.WORKLOADS["decode"]
    n_pairs = 4
    inps = [W.make_inputs(w, seed=100 + i) for i in range(n_pairs)]
    y_np = W.make_y(w, seed=100)
    rows = oracle.max_recv_rows(w.T, w.k, w.E, w.align)
    idx = [torch.from_numpy(i["topk_idx"]).cuda() for i in inps]
    wts = [torch.from_numpy(i["topk_weights"]).cuda() for i in inps]
    xs = [to_dev_bf16(i["x"]) for i in inps]
    y = to_dev_bf16(y_np)
    hs = [ep.EPHandle(w.T, w.k, w.E, w.S, w.align) for _ in range(n_pairs)]
    ri = [torch.empty(rows, dtype=torch.int32, device="cuda") for _ in range(n_pairs)]
    rw = [torch.empty(rows, dtype=torch.float32, device="cuda") for _ in range(n_pairs)]
    rq = [torch.empty(rows, w.H, dtype=torch.uint8, device="cuda") for _ in range(n_pairs)]
    rs = [torch.empty(rows, w.H // 128, dtype=torch.float32, device="cuda") for _ in range(n_pairs)]
    outs = [torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda") for _ in range(n_pairs)]

    def step():
        for i in range(n_pairs):
            ep.get_layout(idx[i], w.E, num_segments=w.S, expert_alignment=w.align,
                          topk_weights=wts[i], handle=hs[i], recv_topk_idx=ri[i], recv_topk_weights=rw[i])
            ep.dispatch_with_handle(xs[i], hs[i], use_fp8=True, recv_x=rq[i], recv_scales=rs[i])
            ep.combine(y, hs[i], wts[i], out=outs[i])

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                   # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(s)
    for o in outs:
        o.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    for i in range(n_pairs):
        lay = oracle.layout(inps[i]["topk_idx"], w.E, w.S, w.align, inps[i]["topk_weights"])
        q, sc = oracle.dispatch(lay, inps[i]["x"], oracle.X_BF16_QUANT_FP8)
        out, _ = oracle.combine(lay["slot_map"], w.T, w.k, y_np, inps[i]["topk_weights"])
        R = lay["R"]
        np.testing.assert_array_equal(rq[i].cpu().numpy()[:R], q[:R])
        np.testing.assert_array_equal(rs[i].cpu().numpy()[:R], sc[:R])
        np.testing.assert_array_equal(bits16(outs[i]), out)
