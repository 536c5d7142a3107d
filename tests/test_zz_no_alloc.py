"""ep_get_layout_static: the layout step for callers that cannot allocate
device memory themselves (code running inside a host program that owns
every device allocation, or plain C code with no device allocator), so
cannot pass ep_get_layout a workspace.  Its scratch lives in a fixed array
inside the library.  Through the C ABI, it must give exactly what
ep_get_layout gives with a caller-owned workspace, call after call, and
must refuse a layout too large for that array.  Its results are also
compared with the CPU oracle's layout directly, not only through the
workspace entry.

This file is named so that pytest collects it last."""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from combine_ep_get_06_b200 import ep as B

KEYS = ("counts", "num_recv_tokens_per_expert", "offsets", "seg_tokens", "slot_map", "pad_rows",
        "num_pad_rows")


def _snapshot(h, ri, rw):
    torch.cuda.synchronize()
    out = {key: getattr(h, key).cpu().numpy().copy() for key in KEYS}
    R = int(out["offsets"][-1])
    out["recv_src"] = h.recv_src.cpu().numpy()[:R].copy()
    out["recv_topk_idx"] = ri.cpu().numpy()[:R].copy()
    out["recv_topk_weights"] = rw.cpu().numpy()[:R].view(np.uint32).copy()
    return out


@pytest.mark.gpu
def test_static_scratch_layout_equals_workspace_layout_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    L = B.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # v3 and mid have many chunks, so the per-chunk histograms really pass
    # through the scratch; decode (T*k = 1024) is one chunk, which never
    # touches it but still goes through the size check and the address
    for name, idx_dtype in (("v3", torch.int64), ("mid", torch.int32), ("decode", torch.int64)):
        w = W.WORKLOADS[name]
        ref_h = B.EPHandle(w.T, w.k, w.E, w.S, w.align)
        new_h = B.EPHandle(w.T, w.k, w.E, w.S, w.align)
        rows = ref_h.max_recv_rows
        ri_ref, rw_ref = torch.empty(rows, dtype=torch.int32, device="cuda"), torch.empty(rows, device="cuda")
        ri_new, rw_new = torch.empty(rows, dtype=torch.int32, device="cuda"), torch.empty(rows, device="cuda")
        for seed in (11, 12):   # two calls in a row on the same handle, different routing
            inp = W.make_inputs(w, seed=seed)
            idx = torch.from_numpy(inp["topk_idx"]).cuda().to(idx_dtype)
            wts = torch.from_numpy(inp["topk_weights"]).cuda()
            is64 = int(idx_dtype == torch.int64)
            st = L.ep_get_layout(ref_h.ref, idx.data_ptr(), is64, wts.data_ptr(), ri_ref.data_ptr(),
                                 rw_ref.data_ptr(), ref_h.workspace_ptr, ref_h.workspace_bytes, stream)
            assert st == 0, L.ep_last_error()
            st = L.ep_get_layout_static(new_h.ref, idx.data_ptr(), is64, wts.data_ptr(), ri_new.data_ptr(),
                                        rw_new.data_ptr(), stream)
            assert st == 0, L.ep_last_error()
            ref = _snapshot(ref_h, ri_ref, rw_ref)
            new = _snapshot(new_h, ri_new, rw_new)
            for key in ref:
                np.testing.assert_array_equal(new[key], ref[key], err_msg=f"{name} seed {seed}: {key}")
            assert new_h.check_error() == 0
            lay = oracle.layout(inp["topk_idx"], w.E, w.S, w.align, inp["topk_weights"])
            R = int(lay["R"])
            np.testing.assert_array_equal(new["counts"], lay["counts"])
            np.testing.assert_array_equal(new["offsets"], lay["offsets"])
            np.testing.assert_array_equal(new["seg_tokens"], lay["seg_tokens"])
            np.testing.assert_array_equal(new["slot_map"], lay["slot_map"])
            np.testing.assert_array_equal(new["recv_src"], lay["recv_src"][:R])
            np.testing.assert_array_equal(new["recv_topk_idx"], lay["recv_topk_idx"][:R])
            np.testing.assert_array_equal(new["recv_topk_weights"], lay["recv_topk_weights"][:R].view(np.uint32))


def test_static_scratch_layout_refuses_layouts_larger_than_its_array():
    # host-side check: no GPU needed, nothing is launched
    L = B.lib()
    T, k, E, S, a = 1 << 20, 8, 1024, 8, 1
    rows = L.ep_max_recv_rows(T, k, E, a)
    h = B._HandleC()
    assert L.ep_handle_init(ctypes.byref(h), T, k, E, S, a, rows, 1 << 30,
                            L.ep_handle_bytes(T, k, E, S, a, rows)) == 0
    assert L.ep_layout_workspace_bytes(ctypes.byref(h)) > (1 << 20)
    st = L.ep_get_layout_static(ctypes.byref(h), 1 << 20, 1, None, None, None, None)
    assert st == B.EP_ERR_INVALID_ARG
    assert "scratch" in L.ep_last_error().decode()
