"""The one-call dispatch (layout + dispatch, ep_layout_dispatch) vs the
oracle.  Here the dispatch reads its x rows before waiting on the layout,
so these cases cover that ordering, small (one layout CTA) and large (two
layout kernels).  Bit-exact on every output, guard bytes untouched."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import assert_parity, run_cuda_one_call, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _random_case(T, k, E, S, align, H, drop, seed, duplicates=False):
    rng = np.random.default_rng(seed)
    if duplicates or k > E:
        idx = rng.integers(0, E, size=(T, k))
    else:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]) if T else np.zeros((0, k))
    idx = idx.astype(np.int64)
    idx[rng.random((T, k)) < drop] = -1
    return {"x": W._to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32)),
            "topk_idx": idx, "topk_weights": rng.standard_normal((T, k)).astype(np.float32)}


@pytest.mark.parametrize("name", ["decode", "tiny", "mid"])
def test_one_call_dispatch_on_workloads(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=3)
    mode = {"bf16": ep.EP_X_BF16, "fp8_quant": ep.EP_X_BF16_TO_FP8}[w.x_mode]
    assert_parity(run_cuda_one_call(inp, w, mode), run_oracle(inp, w, None, mode), mode)


FUSED = [
    # T, k, E, S, align, H, mode, drop, duplicates
    (128, 8, 256, 8, 128, 7168, "fp8_quant", 0.1, False),   # padding rows
    (170, 6, 64, 8, 16, 4096, "fp8_quant", 0.05, False),    # k does not divide 32
    (500, 2, 16, 4, 1, 256, "bf16", 0.0, False),            # more tokens than CTAs
    (1024, 1, 7, 7, 3, 128, "fp8_quant", 0.2, False),       # k = 1, 1024 slots
    (32, 32, 1024, 16, 4, 1024, "fp8_quant", 0.0, False),   # E = 1024, k = 32
    (100, 10, 12, 3, 5, 384, "fp8_quant", 0.3, True),       # duplicate experts, ragged scale rows
    (1, 1, 1, 1, 1, 8, "bf16", 0.0, False),
    (0, 4, 8, 2, 4, 128, "fp8_quant", 0.0, False),          # empty batch
    (300, 4, 32, 4, 8, 512, "bf16", 0.0, False),            # 1200 slots: two layout kernels
]


@pytest.mark.parametrize("T,k,E,S,align,H,xm,drop,dup", FUSED)
def test_one_call_dispatch_edge_shapes(T, k, E, S, align, H, xm, drop, dup):
    w = W.Workload("one_call", T=T, H=H, E=E, S=S, k=k, align=align, x_mode=xm)
    inp = _random_case(T, k, E, S, align, H, drop, seed=T + 7 * k, duplicates=dup)
    mode = {"bf16": ep.EP_X_BF16, "fp8_quant": ep.EP_X_BF16_TO_FP8}[xm]
    assert_parity(run_cuda_one_call(inp, w, mode), run_oracle(inp, w, None, mode), mode)


@pytest.mark.parametrize("dtype,shift", [(torch.int32, 0), (torch.int32, 1), (torch.int64, 1)])
@pytest.mark.parametrize("T", [128, 127, 300])
def test_one_call_index_types_and_alignment(T, dtype, shift):
    # the one-chunk path loads four indices a thread with 16-byte loads when
    # the pointer allows it, else one by one; T = 127 leaves a partial group.
    # T = 300 (2400 slots, three chunks) takes the layout grids, whose count
    # kernel prefetches only the 16-byte aligned interior of its chunk
    w = W.Workload("idx", T=T, H=1024, E=64, S=4, k=8, align=4, x_mode="fp8_quant")
    inp = _random_case(T, 8, 64, 4, 4, 1024, 0.1, seed=T + shift)
    g = run_cuda_one_call(inp, w, ep.EP_X_BF16_TO_FP8, idx_dtype=dtype, idx_shift=shift)
    assert_parity(g, run_oracle(inp, w, None, oracle.X_BF16_QUANT_FP8), oracle.X_BF16_QUANT_FP8)


def test_one_call_dispatch_prequantised_tuple():
    w = W.Workload("pq", T=96, H=1024, E=32, S=4, k=8, align=4, x_mode="fp8_quant")
    inp = _random_case(96, 8, 32, 4, 4, 1024, 0.1, seed=11)
    pq = W.make_prequant(96, 1024, seed=11)
    g = run_cuda_one_call(inp, w, ep.EP_X_FP8, prequant=pq)
    assert_parity(g, run_oracle(inp, w, None, oracle.X_FP8_PREQUANT, prequant=pq), oracle.X_FP8_PREQUANT)


def test_one_call_dispatch_flags_bad_indices():
    w = W.Workload("bad", T=64, H=256, E=16, S=4, k=4, align=2, x_mode="fp8_quant")
    inp = _random_case(64, 4, 16, 4, 2, 256, 0.0, seed=5)
    inp["topk_idx"][3, 2] = 99
    inp["topk_idx"][40, 0] = -5
    g = run_cuda_one_call(inp, w, ep.EP_X_BF16_TO_FP8)
    o = run_oracle(inp, w, None, oracle.X_BF16_QUANT_FP8)
    assert_parity(g, o, oracle.X_BF16_QUANT_FP8)
    with pytest.raises(ep.EPError, match="topk_idx"):
        g["handle"].check_error()
