"""The C-ABI library without a GPU: it loads, exports every symbol that
include/ep.h declares, and rejects bad arguments on the host before
launching anything (these calls never reach CUDA)."""

import ctypes
import os
import re

import pytest

import oracle
from combine_ep_get_06_b200 import ep as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    L = ctypes.CDLL(B.library_path())
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B.SIGNATURES)        # the binding covers exactly the ABI


def test_library_exports_nothing_else():
    out = os.popen(f"nm -D --defined-only {B.library_path()}").read()
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {n for n in exported if n.startswith("ep_")} == set(declared_functions())


def test_version_and_status_strings():
    L = B.lib()
    assert L.ep_abi_version() == 1
    for code, name in [(0, b"EP_OK"), (1, b"EP_ERR_INVALID_ARG"), (2, b"EP_ERR_DEVICE"), (3, b"EP_ERR_CUDA")]:
        assert L.ep_status_string(code) == name


@pytest.mark.parametrize("T,k,E,a", [(0, 1, 1, 1), (128, 2, 16, 1), (4096, 6, 64, 128),
                                     (8192, 8, 256, 128), (3, 32, 1024, 7)])
def test_max_recv_rows_agrees_with_the_oracle(T, k, E, a):
    assert B.lib().ep_max_recv_rows(T, k, E, a) == oracle.max_recv_rows(T, k, E, a)


def test_max_recv_rows_rejects_bad_shapes():
    L = B.lib()
    assert L.ep_max_recv_rows(-1, 2, 4, 1) == -1
    assert L.ep_max_recv_rows(1 << 30, 8, 4, 1) == -1        # int32 overflow


def _init(T=16, k=2, E=8, S=2, a=4, rows=None, base=1 << 20, nbytes=None):
    L = B.lib()
    rows = L.ep_max_recv_rows(T, k, E, a) if rows is None else rows
    need = L.ep_handle_bytes(T, k, E, S, a, rows)
    h = B._HandleC()
    st = L.ep_handle_init(ctypes.byref(h), T, k, E, S, a, rows, base,
                          need if nbytes is None else nbytes)
    return st, h, need


@pytest.mark.parametrize("kw,msg", [
    (dict(k=0), "num_topk"), (dict(k=33), "num_topk"), (dict(E=0), "num_experts"),
    (dict(E=1025, S=1), "num_experts"), (dict(E=8, S=3), "num_segments"), (dict(a=0), "alignment"),
    (dict(T=-1), "num_tokens"), (dict(rows=10), "max_recv_rows"), (dict(base=1 << 20 | 16), "aligned"),
    (dict(nbytes=64), "bytes")])
def test_handle_init_rejects(kw, msg):
    st, _, _ = _init(**kw)
    assert st == B.EP_ERR_INVALID_ARG
    assert msg in B.lib().ep_last_error().decode()


def test_handle_init_carves_disjoint_aligned_arrays():
    T, k, E, S, a = 100, 3, 12, 4, 5
    st, h, need = _init(T, k, E, S, a)
    assert st == 0 and need > 0
    rows = B.lib().ep_max_recv_rows(T, k, E, a)
    sizes = [("counts", E), ("recv_counts", E), ("offsets", E + 1), ("seg_tokens", S),
             ("slot_map", T * k), ("recv_src", rows), ("pad_rows", E * (a - 1)),
             ("num_pad_rows", 1), ("error_word", 1)]
    spans = sorted((getattr(h, n), getattr(h, n) + 4 * m) for n, m in sizes)
    base = 1 << 20
    for (s0, e0), (s1, _) in zip(spans, spans[1:]):
        assert e0 <= s1
    assert spans[0][0] >= base and spans[-1][1] <= base + need
    assert all(s % 256 == 0 for s, _ in spans)
    assert (h.num_tokens, h.num_topk, h.num_experts, h.num_segments, h.expert_alignment,
            h.max_recv_rows) == (T, k, E, S, a, rows)


def test_layout_rejects_bad_arguments_before_launch():
    L = B.lib()
    st, h, _ = _init()
    ws = L.ep_layout_workspace_bytes(ctypes.byref(h))
    assert ws > 0
    cases = [
        (dict(idx=None), "topk_idx"), (dict(idx=(1 << 20) + 4), "topk_idx"),
        (dict(is64=2), "idx_is_int64"), (dict(ws_bytes=ws - 1), "workspace"),
        (dict(ws=(1 << 22) + 16), "workspace"), (dict(w=(1 << 21) + 2), "topk_weights")]
    for kw, msg in cases:
        args = dict(idx=1 << 20, is64=1, w=None, ws=1 << 22, ws_bytes=ws)
        args.update(kw)
        st = L.ep_get_layout(ctypes.byref(h), args["idx"], args["is64"], args["w"], None, None,
                             args["ws"], args["ws_bytes"], None)
        assert st == B.EP_ERR_INVALID_ARG, kw
        assert msg in L.ep_last_error().decode(), (kw, L.ep_last_error())
    bad = B._HandleC()
    assert L.ep_get_layout(ctypes.byref(bad), 1 << 20, 1, None, None, None, 1 << 22, ws, None) == 1


def test_dispatch_rejects_bad_arguments_before_launch():
    L = B.lib()
    st, h, _ = _init()
    X, R, S_ = 1 << 24, 1 << 26, 1 << 28
    cases = [
        (dict(mode=7), "mode"), (dict(mode=2, H=200), "multiple of 128"),
        (dict(mode=0, H=12), "multiple of 8"), (dict(x=X + 8), "x must"),
        (dict(recv=R + 4), "recv_x"), (dict(mode=2, scales=None), "recv_scales"),
        (dict(mode=1, xs=None), "x_scales")]
    for kw, msg in cases:
        a = dict(mode=2, x=X, xs=1 << 27, H=256, recv=R, scales=S_)
        a.update(kw)
        st = L.ep_dispatch(ctypes.byref(h), a["mode"], a["x"], a["xs"], a["H"], a["recv"],
                           a["scales"], None)
        assert st == B.EP_ERR_INVALID_ARG, kw
        assert msg in L.ep_last_error().decode(), (kw, L.ep_last_error())


def test_combine_rejects_bad_arguments_before_launch():
    L = B.lib()
    st, h, _ = _init()
    Y, O = 1 << 24, 1 << 26
    cases = [(dict(H=12), "multiple of 8"), (dict(y=Y + 4), "y must"), (dict(out=O + 8), "out must"),
             (dict(ow=1 << 27), "together"), (dict(w=(1 << 25) + 1), "topk_weights")]
    for kw, msg in cases:
        a = dict(y=Y, H=64, w=None, rw=None, ow=None, out=O)
        a.update(kw)
        st = L.ep_combine(ctypes.byref(h), a["y"], a["H"], a["w"], a["rw"], a["ow"], a["out"], None)
        assert st == B.EP_ERR_INVALID_ARG, kw
        assert msg in L.ep_last_error().decode(), (kw, L.ep_last_error())


def test_sm_budget_is_a_per_thread_setting():
    # host only: the budget is stored, read back, rejected when negative,
    # and belongs to the calling thread
    import threading
    L = B.lib()
    assert L.ep_get_num_sms() == 0
    assert L.ep_set_num_sms(24) == B.EP_OK and L.ep_get_num_sms() == 24
    seen = []
    th = threading.Thread(target=lambda: seen.append(L.ep_get_num_sms()))
    th.start(); th.join()
    assert seen == [0]
    assert L.ep_set_num_sms(-1) == B.EP_ERR_INVALID_ARG and L.ep_get_num_sms() == 24
    with B.sm_budget(64):
        assert B.get_num_sms() == 64
    assert B.get_num_sms() == 24
    assert L.ep_set_num_sms(0) == B.EP_OK and L.ep_get_num_sms() == 0


def test_checked_build_exports_the_same_abi():
    # EP_CHECKED: the debug build with device-side invariant checks compiles
    # (nvcc cross-compiles here) and exports exactly the production ABI
    import subprocess
    from combine_ep_get_06_b200 import build
    path = build.build(checked=True)
    def exported(p):
        out = subprocess.run(["nm", "-D", "--defined-only", p], capture_output=True, text=True).stdout
        return {line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("ep_")}
    assert exported(path) == exported(build.build()) == set(B.SIGNATURES)
