"""Shared plumbing for the GPU tests: move the seeded numpy inputs to the
device, run the CUDA path through the binding, run the oracle on the very
same arrays, and compare bit for bit."""

from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep

SENTINEL = 0xA5


def to_dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def bytes8(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def guarded(rows: int, cols: int, dtype, guard_rows: int = 3):
    """A [rows, cols] view at the front of a buffer whose every byte starts
    as SENTINEL, with guard rows after it: writes past the view show up."""
    elem = torch.empty(0, dtype=dtype).element_size()
    buf = torch.full(((rows + guard_rows) * cols * elem,), SENTINEL, dtype=torch.uint8, device="cuda")
    return buf, buf.view(dtype).view(rows + guard_rows, cols)[:rows]


def guard_ok(buf: torch.Tensor, start_byte: int) -> bool:
    return bool((buf[start_byte:] == SENTINEL).all())


def run_cuda(inp: dict, w: W.Workload, y: np.ndarray | None, mode: int, *, idx_int32=False,
             prequant=None, weighted=True, recv_weights_in=None):
    """layout -> dispatch -> combine on the GPU; returns host arrays."""
    T = inp["x"].shape[0]
    idx = torch.from_numpy(inp["topk_idx"]).cuda()
    if idx_int32:
        idx = idx.to(torch.int32)
    wts = torch.from_numpy(inp["topk_weights"]).cuda()
    handle = ep.EPHandle(T, w.k, w.E, w.S, w.align, device="cuda")
    rows = handle.max_recv_rows
    ri_buf, recv_idx = guarded(rows, 1, torch.int32)
    rw_buf, recv_w = guarded(rows, 1, torch.float32)
    ep.get_layout(idx, w.E, num_segments=w.S, expert_alignment=w.align, topk_weights=wts,
                  handle=handle, recv_topk_idx=recv_idx.view(-1), recv_topk_weights=recv_w.view(-1))
    out = {"handle": handle}
    H = w.H
    if mode == ep.EP_X_BF16:
        rx_buf, recv_x = guarded(rows, H, torch.bfloat16)
        ep.dispatch_with_handle(to_dev_bf16(inp["x"]), handle, recv_x=recv_x)
        out["recv_x"] = bits16(recv_x)
        out["guards"] = [(rx_buf, rows * H * 2)]
    else:
        rx_buf, recv_x = guarded(rows, H, torch.uint8)
        rs_buf, recv_s = guarded(rows, H // 128, torch.float32)
        if mode == ep.EP_X_FP8:
            q, s = prequant
            xin = (torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda())
        else:
            xin = to_dev_bf16(inp["x"])
        ep.dispatch_with_handle(xin, handle, use_fp8=True, recv_x=recv_x, recv_scales=recv_s)
        out["recv_x"] = bytes8(recv_x)
        out["recv_scales"] = recv_s.cpu().numpy()
        out["guards"] = [(rx_buf, rows * H), (rs_buf, rows * (H // 128) * 4)]
    out["guards"] += [(ri_buf, rows * 4), (rw_buf, rows * 4)]
    if y is not None:
        rwi = None if recv_weights_in is None else torch.from_numpy(recv_weights_in).cuda()
        o, ow = ep.combine(to_dev_bf16(y), handle, wts if weighted else None, recv_topk_weights=rwi)
        out["combined"] = bits16(o)
        out["out_weights"] = None if ow is None else ow.cpu().numpy()
    torch.cuda.synchronize()
    out["recv_topk_idx"] = recv_idx.view(-1).cpu().numpy()
    out["recv_topk_weights"] = recv_w.view(-1).cpu().numpy()
    for key in ("counts", "num_recv_tokens_per_expert", "offsets", "seg_tokens", "slot_map",
                "recv_src", "pad_rows", "num_pad_rows"):
        out[key] = getattr(handle, key).cpu().numpy()
    out["error_bits"] = handle.check_error() if not _has_bad_idx(inp, w) else None
    return out


def _has_bad_idx(inp, w):
    i = inp["topk_idx"]
    return bool(((i < -1) | (i >= w.E)).any())


def run_oracle(inp: dict, w: W.Workload, y: np.ndarray | None, mode: int, *, prequant=None,
               weighted=True, recv_weights_in=None):
    lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
    if mode == oracle.X_FP8_PREQUANT:
        recv, scales = oracle.dispatch(lay, prequant[0], mode, prequant[1])
    else:
        recv, scales = oracle.dispatch(lay, inp["x"], mode)
    res = {"lay": lay, "recv_x": recv, "recv_scales": scales}
    if y is not None:
        T = inp["x"].shape[0]
        o, ow = oracle.combine(lay["slot_map"], T, w.k, y, inp["topk_weights"] if weighted else None,
                               recv_weights_in, recv_weights_in is not None)
        res["combined"], res["out_weights"] = o, ow
    return res


def assert_parity(g: dict, o: dict, mode: int):
    lay = o["lay"]
    R = lay["R"]
    E = lay["E"]
    assert g["offsets"][E] == R
    np.testing.assert_array_equal(g["counts"], lay["counts"])
    np.testing.assert_array_equal(g["offsets"], lay["offsets"])
    np.testing.assert_array_equal(g["num_recv_tokens_per_expert"], np.diff(lay["offsets"]))
    np.testing.assert_array_equal(g["seg_tokens"], lay["seg_tokens"])
    np.testing.assert_array_equal(g["slot_map"], lay["slot_map"])
    np.testing.assert_array_equal(g["recv_src"][:R], lay["recv_src"][:R])
    np.testing.assert_array_equal(g["recv_topk_idx"][:R], lay["recv_topk_idx"][:R])
    np.testing.assert_array_equal(g["recv_topk_weights"][:R].view(np.uint32),
                                  lay["recv_topk_weights"][:R].view(np.uint32))
    pad = np.nonzero(lay["recv_src"][:R] < 0)[0]
    assert int(g["num_pad_rows"][0]) == pad.size
    np.testing.assert_array_equal(g["pad_rows"][: pad.size], pad)
    np.testing.assert_array_equal(g["recv_x"][:R], o["recv_x"][:R])
    if mode != oracle.X_BF16:
        np.testing.assert_array_equal(g["recv_scales"][:R].view(np.uint32),
                                      o["recv_scales"][:R].view(np.uint32))
    # rows >= R are never written; guard bytes after each buffer untouched
    tail = g["recv_x"][R:]
    if mode == oracle.X_BF16:
        assert np.all(tail == (SENTINEL << 8 | SENTINEL))
    else:
        assert np.all(tail == SENTINEL)
        assert np.all(g["recv_scales"][R:].view(np.uint32) == 0xA5A5A5A5)
    assert np.all(g["recv_topk_idx"][R:].view(np.uint32) == 0xA5A5A5A5)
    for buf, start in g["guards"]:
        assert guard_ok(buf, start)
    if "combined" in o:
        np.testing.assert_array_equal(g["combined"], o["combined"])
    if o.get("out_weights") is not None:
        np.testing.assert_array_equal(g["out_weights"], o["out_weights"])
    if g.get("error_bits") is not None:
        assert g["error_bits"] == 0


def max_bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> int:
    """Largest distance in bf16 units in the last place (ordered integer encoding)."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, 0x8000 - (b & 0x7FFF), 0x8000 + (b & 0x7FFF))
    return int(np.abs(ordered(a_bits) - ordered(b_bits)).max(initial=0))


def run_cuda_one_call(inp: dict, w: W.Workload, mode: int, *, prequant=None, idx_dtype=torch.int64,
                      idx_shift=0):
    """layout + dispatch through one ep.dispatch(x, topk_idx, ...) call;
    returns host arrays like run_cuda (no combine).  idx_dtype: int64 or
    int32 indices; idx_shift: elements by which topk_idx starts past a
    256-byte aligned allocation (1 gives a pointer that is not 16-byte
    aligned)."""
    T = inp["x"].shape[0]
    src = torch.from_numpy(inp["topk_idx"]).to(idx_dtype)
    base = torch.empty(src.numel() + idx_shift, dtype=idx_dtype, device="cuda")
    idx = base[idx_shift:].view(src.shape)
    idx.copy_(src.cuda())
    wts = torch.from_numpy(inp["topk_weights"]).cuda()
    handle = ep.EPHandle(T, w.k, w.E, w.S, w.align, device="cuda")
    rows = handle.max_recv_rows
    ri_buf, recv_idx = guarded(rows, 1, torch.int32)
    rw_buf, recv_w = guarded(rows, 1, torch.float32)
    H = w.H
    out = {"handle": handle}
    if mode == ep.EP_X_BF16:
        rx_buf, recv_x = guarded(rows, H, torch.bfloat16)
        ep.dispatch(to_dev_bf16(inp["x"]), idx, wts, w.E, expert_alignment=w.align, num_segments=w.S,
                    handle=handle, recv_x=recv_x, recv_topk_idx=recv_idx.view(-1),
                    recv_topk_weights=recv_w.view(-1))
        out["recv_x"] = bits16(recv_x)
        out["guards"] = [(rx_buf, rows * H * 2)]
    else:
        rx_buf, recv_x = guarded(rows, H, torch.uint8)
        rs_buf, recv_s = guarded(rows, H // 128, torch.float32)
        if mode == ep.EP_X_FP8:
            xin = (torch.from_numpy(prequant[0]).cuda(), torch.from_numpy(prequant[1]).cuda())
        else:
            xin = to_dev_bf16(inp["x"])
        ep.dispatch(xin, idx, wts, w.E, expert_alignment=w.align, num_segments=w.S, handle=handle,
                    use_fp8=True, recv_x=recv_x, recv_scales=recv_s, recv_topk_idx=recv_idx.view(-1),
                    recv_topk_weights=recv_w.view(-1))
        out["recv_x"] = bytes8(recv_x)
        out["recv_scales"] = recv_s.cpu().numpy()
        out["guards"] = [(rx_buf, rows * H), (rs_buf, rows * (H // 128) * 4)]
    out["guards"] += [(ri_buf, rows * 4), (rw_buf, rows * 4)]
    torch.cuda.synchronize()
    out["recv_topk_idx"] = recv_idx.view(-1).cpu().numpy()
    out["recv_topk_weights"] = recv_w.view(-1).cpu().numpy()
    for key in ("counts", "num_recv_tokens_per_expert", "offsets", "seg_tokens", "slot_map",
                "recv_src", "pad_rows", "num_pad_rows"):
        out[key] = getattr(handle, key).cpu().numpy()
    out["error_bits"] = handle.check_error() if not _has_bad_idx(inp, w) else None
    return out
