"""NVFP4 dispatch on the GPU vs the CPU oracle, bit for bit.

The mode quantises bf16 x per 1x16 block to E2M1 codes with one E4M3 scale
per block (DeepEP V2 README, "Roadmap": NVFP4 data type in the Hybrid-EP
branch).  Packed codes and scale bytes must equal the oracle's for every
written row; rows at or past the receive total keep the sentinel and the
guard bytes after every buffer stay untouched.  Sizes: every workload at
full size in the benchmark's launch configuration, hidden sizes whose scale
rows are not a multiple of 16 bytes (scales stored byte by byte instead of
by bulk copy), hand-built blocks at the format's corners, and empty input."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import SENTINEL, guard_ok, guarded, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def run_nvfp4(inp: dict, w: W.Workload, *, one_call: bool = False):
    T = inp["x"].shape[0]
    H = inp["x"].shape[1]
    idx = torch.from_numpy(inp["topk_idx"]).cuda()
    wts = torch.from_numpy(inp["topk_weights"]).cuda()
    handle = ep.EPHandle(T, w.k, w.E, w.S, w.align, device="cuda")
    rows = handle.max_recv_rows
    rx_buf, recv_x = guarded(rows, H // 2, torch.uint8)
    rs_buf, recv_s = guarded(rows, H // 16, torch.uint8)
    x = to_dev_bf16(inp["x"])
    if one_call:
        ep.dispatch(x, idx, wts, w.E, expert_alignment=w.align, num_segments=w.S, handle=handle,
                    use_nvfp4=True, recv_x=recv_x, recv_scales=recv_s)
    else:
        ep.get_layout(idx, w.E, num_segments=w.S, expert_alignment=w.align, topk_weights=wts,
                      handle=handle)
        out = ep.dispatch_with_handle(x, handle, use_nvfp4=True, recv_x=recv_x, recv_scales=recv_s)
        assert out[0] is recv_x and out[1] is recv_s
    torch.cuda.synchronize()
    return {"recv_x": recv_x.cpu().numpy(), "recv_scales": recv_s.cpu().numpy(),
            "slot_map": handle.slot_map.cpu().numpy(), "R": handle.total_rows(),
            "guards": [(rx_buf, rows * (H // 2)), (rs_buf, rows * (H // 16))],
            "error_bits": handle.check_error()}


def check(inp: dict, w: W.Workload, g: dict):
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    q, s = oracle.dispatch(lay, inp["x"], oracle.X_BF16_QUANT_NVFP4)
    R = lay["R"]
    assert g["R"] == R
    np.testing.assert_array_equal(g["slot_map"], lay["slot_map"])
    np.testing.assert_array_equal(g["recv_x"][:R], q[:R])
    np.testing.assert_array_equal(g["recv_scales"][:R], s[:R])
    assert np.all(g["recv_x"][R:] == SENTINEL)
    assert np.all(g["recv_scales"][R:] == SENTINEL)
    for buf, start in g["guards"]:
        assert guard_ok(buf, start)
    assert g["error_bits"] == 0
    return lay, q, s


@pytest.mark.parametrize("name", ["v3", "skewed", "mid", "decode"])
def test_nvfp4_workload_matches_oracle_bit_exactly(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=11)
    check(inp, w, run_nvfp4(inp, w))


@pytest.mark.parametrize("name,T", [("v3", 2048), ("decode", 128)])
def test_nvfp4_one_call_matches_oracle(name, T):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=12, T=T)
    check(inp, w, run_nvfp4(inp, w, one_call=True))


@pytest.mark.parametrize("H", [32, 96, 1056, 4128])
def test_nvfp4_ragged_hidden_byte_scales(H):
    # H/16 scale bytes per row not a multiple of 16: scales go out byte by
    # byte; alignment 128 gives padding rows whose codes and scales are zero.
    w = dataclasses.replace(W.WORKLOADS["mid"], name=f"mid_h{H}", H=H, T=777)
    inp = W.make_inputs(w, seed=13)
    lay, q, s = check(inp, w, run_nvfp4(inp, w))
    pad = lay["recv_src"][: lay["R"]] < 0
    assert pad.any()
    assert np.all(q[: lay["R"]][pad] == 0) and np.all(s[: lay["R"]][pad] == 0)


def _corner_rows(H: int) -> np.ndarray:
    """bf16 rows exercising the format's corners, one kind of block per row."""
    rng = np.random.default_rng(14)
    r = np.zeros((16, H), np.float32)
    r[1] = 1e4                                              # scale saturates at 448
    r[2] = np.tile(np.array([6, .25, .75, 1.25, 1.75, 2.5, 3.5, 5] * 2, np.float32), H // 16)  # ties
    r[3] = 1e-6 * rng.standard_normal(H)                    # below the amax floor
    r[4] = -0.0
    r[5] = -rng.standard_normal(H).astype(np.float32) * 0.01
    r[6] = np.tile(np.array([6] + [-0.1] * 15, np.float32), H // 16)   # small negatives -> -0
    r[7] = 3.0e38                                           # near the bf16 maximum
    r[8] = rng.standard_normal(H) * np.exp2(rng.integers(-20, 20, H))  # wide dynamic range
    r[9] = np.tile(np.array([2688.0, 1.0] * 8, np.float32), H // 16)   # amax/6 just at 448
    r[10] = np.tile(np.array([0.01171875] * 16, np.float32), H // 16)  # amax exactly the floor
    r[11:] = rng.standard_normal((5, H))
    return W._to_bf16_bits(r)


def test_nvfp4_corner_blocks():
    w = dataclasses.replace(W.WORKLOADS["tiny"], name="corners", T=16, H=256, align=4)
    inp = W.make_inputs(w, seed=14)
    inp["x"] = _corner_rows(w.H)
    check(inp, w, run_nvfp4(inp, w))


def test_nvfp4_empty_input():
    w = dataclasses.replace(W.WORKLOADS["mid"], name="empty", T=0, H=256)
    inp = W.make_inputs(w, seed=15)
    g = run_nvfp4(inp, w)
    assert g["R"] == 0
    check(inp, w, g)


def test_nvfp4_codes_decode_within_half_a_quantum_at_full_size():
    # a property that holds at any size, independent of the oracle: every
    # code times its block's scale lies within half a grid step of x/scale
    # (or x saturates at 6 * scale), and each block's scale is e4m3(amax/6).
    w = W.WORKLOADS["v3"]
    inp = W.make_inputs(w, seed=16)
    g = run_nvfp4(inp, w)
    R = g["R"]
    sm = g["slot_map"].reshape(w.T, w.k)
    rng = np.random.default_rng(16)
    toks = rng.choice(w.T, 64, replace=False)
    x = inp["x"].view(np.uint16).astype(np.uint32) << 16
    x = x.view(np.float32)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    for t in toks:
        for j in range(w.k):
            row = sm[t, j]
            if row < 0:
                continue
            assert row < R
            codes = g["recv_x"][row]
            c = np.empty(w.H, np.uint8)
            c[0::2], c[1::2] = codes & 0xF, codes >> 4
            val = np.where(c & 8, -1.0, 1.0) * grid[c & 7]
            sc = oracle.e4m3_decode(g["recv_scales"][row]).astype(np.float64)
            xs = x[t].astype(np.float64).reshape(-1, 16) / sc[:, None]
            step = np.where(np.abs(xs) < 2, 0.5, np.where(np.abs(xs) < 4, 1.0, 2.0))
            err = np.abs(val.reshape(-1, 16) - np.clip(xs, -6, 6))
            assert np.all(err <= step / 2 * (1 + 1e-6))
            amax = np.maximum(np.abs(x[t]).reshape(-1, 16).max(1), 6 / 512)
            np.testing.assert_array_equal(g["recv_scales"][row], oracle.e4m3_encode(amax / 6))


def test_nvfp4_rejects_hidden_not_multiple_of_32():
    w = dataclasses.replace(W.WORKLOADS["tiny"], name="bad_h", H=48)
    inp = W.make_inputs(w, seed=17)
    handle = ep.EPHandle(w.T, w.k, w.E, w.S, w.align, device="cuda")
    ep.get_layout(torch.from_numpy(inp["topk_idx"]).cuda(), w.E, num_segments=w.S,
                  expert_alignment=w.align, handle=handle)
    with pytest.raises(ValueError):
        ep.dispatch_with_handle(to_dev_bf16(inp["x"]), handle, use_nvfp4=True)
    rx = torch.empty(handle.max_recv_rows, 24, dtype=torch.uint8, device="cuda")
    rs = torch.empty(handle.max_recv_rows, 3, dtype=torch.uint8, device="cuda")
    st = ep.lib().ep_dispatch(handle.ref, ep.EP_X_BF16_TO_NVFP4, to_dev_bf16(inp["x"]).data_ptr(), None,
                              48, rx.data_ptr(), rs.data_ptr(), None)
    assert st == 1  # EP_ERR_INVALID_ARG, nothing launched
    with pytest.raises(ValueError):
        ep.dispatch_with_handle(to_dev_bf16(inp["x"]), handle, use_fp8=True, use_nvfp4=True)
