"""Dispatch and combine on an SM budget, beside a compute kernel.

The pages run their dispatch / combine kernels on a bounded number of SMs
(DeepEP V2 README, "Interfaces and examples": num_sms and running the
communication beside the compute stream; "Performance": throughput at a
given #SMs) so that the expert GEMMs keep the rest of the GPU.  Here:
  - with a budget of 24 or 64 SMs the results stay bit-exact against the
    oracle (one-call dispatch, FP8, then the weighted combine);
  - the budget takes effect: at 24 SMs the kernels run markedly slower
    than with the whole GPU;
  - dispatch -> combine on a side stream with a budget of 24 SMs overlaps
    in time with a long matmul loop on another stream (events on both
    streams), and still matches the oracle."""

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from gpu_helpers import bits16, bytes8, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    yield
    ep.set_num_sms(0)


class Case:
    def __init__(self, name, seed=31):
        w = W.WORKLOADS[name]
        self.w = w
        self.inp = W.make_inputs(w, seed=seed)
        self.y_np = W.make_y(w, seed=seed)
        self.x = to_dev_bf16(self.inp["x"])
        self.y = to_dev_bf16(self.y_np)
        self.idx = torch.from_numpy(self.inp["topk_idx"]).cuda()
        self.wts = torch.from_numpy(self.inp["topk_weights"]).cuda()
        self.h = ep.EPHandle(w.T, w.k, w.E, w.S, w.align, device="cuda")
        rows = self.h.max_recv_rows
        self.rx = torch.empty(rows, w.H, dtype=torch.uint8, device="cuda")
        self.rs = torch.empty(rows, w.H // 128, dtype=torch.float32, device="cuda")
        self.out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")

    def step(self):
        w = self.w
        ep.dispatch(self.x, self.idx, self.wts, w.E, expert_alignment=w.align, num_segments=w.S,
                    handle=self.h, use_fp8=True, recv_x=self.rx, recv_scales=self.rs)
        ep.combine(self.y, self.h, self.wts, out=self.out)

    def check(self):
        torch.cuda.synchronize()
        w = self.w
        lay = oracle.layout(self.inp["topk_idx"], w.E, w.S, w.align, self.inp["topk_weights"])
        q, s = oracle.dispatch(lay, self.inp["x"], oracle.X_BF16_QUANT_FP8)
        o, _ = oracle.combine(lay["slot_map"], w.T, w.k, self.y_np, self.inp["topk_weights"])
        R = lay["R"]
        np.testing.assert_array_equal(self.h.slot_map.cpu().numpy(), lay["slot_map"])
        np.testing.assert_array_equal(bytes8(self.rx)[:R], q[:R])
        np.testing.assert_array_equal(self.rs.cpu().numpy()[:R].view(np.uint32), s[:R].view(np.uint32))
        np.testing.assert_array_equal(bits16(self.out), o)
        assert self.h.check_error() == 0


def _time(fn, n=10):
    fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        fn()
    b.record()
    b.synchronize()
    return a.elapsed_time(b) / n


@pytest.mark.parametrize("name,budget", [("mid", 24), ("mid", 64), ("decode", 16)])
def test_budget_results_match_oracle(name, budget):
    # decode-sized batches take the row path without a budget, warp units with one
    c = Case(name)
    with ep.sm_budget(budget):
        c.step()
    assert ep.get_num_sms() == 0
    c.check()


def test_budget_of_24_sms_takes_effect():
    c = Case("v3")
    full = _time(c.step)
    with ep.sm_budget(24):
        part = _time(c.step)
    # 24 of 148 SMs cannot sustain the full HBM rate: the step must be
    # clearly slower (a grid that ignored the budget would not be)
    assert part > 1.5 * full, (part, full)
    c.check()


def test_budget_dispatch_combine_overlaps_a_compute_stream():
    c = Case("mid")
    a = torch.randn(8192, 8192, dtype=torch.bfloat16, device="cuda")
    b = torch.randn(8192, 8192, dtype=torch.bfloat16, device="cuda")
    d = torch.empty_like(a)

    def gemms(n=12):
        for _ in range(n):
            torch.matmul(a, b, out=d)

    def ep_steps(n=12):
        for _ in range(n):
            c.step()

    gemms(2)
    with ep.sm_budget(24):
        ep_steps(2)
    torch.cuda.synchronize()
    t_gemm = _time(gemms, 1)
    with ep.sm_budget(24):
        t_ep = _time(ep_steps, 1)

    s_comp, s_ep = torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def concurrent():
        ev = {k: torch.cuda.Event(enable_timing=True) for k in ("t0", "g0", "g1", "e0", "e1")}
        ev["t0"].record(main)
        s_comp.wait_stream(main)
        s_ep.wait_stream(main)
        with torch.cuda.stream(s_comp):
            ev["g0"].record(s_comp)
            gemms()
            ev["g1"].record(s_comp)
        with torch.cuda.stream(s_ep), ep.sm_budget(24):
            ev["e0"].record(s_ep)
            ep_steps()
            ev["e1"].record(s_ep)
        main.wait_stream(s_comp)
        main.wait_stream(s_ep)
        torch.cuda.synchronize()
        return {k: ev["t0"].elapsed_time(e) for k, e in ev.items() if k != "t0"}

    concurrent()  # untimed: first use of the two streams (allocator and library set-up per stream)
    at = concurrent()
    overlap = min(at["g1"], at["e1"]) - max(at["g0"], at["e0"])
    ep_span = at["e1"] - at["e0"]
    # the EP work ran while the GEMMs ran for most of its span, and the two
    # streams together took less than the two alone back to back
    assert overlap > 0.5 * min(ep_span, t_ep), (at, t_gemm, t_ep)
    assert max(at["g1"], at["e1"]) - min(at["g0"], at["e0"]) < 0.95 * (t_gemm + t_ep), (at, t_gemm, t_ep)
    c.check()
