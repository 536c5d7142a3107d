"""Host side of the multi-GPU expert parallelism, on CPU.

* ep_mgpu_geometry_init: sizes and section offsets, and its limits.
* ep_mgpu_dispatch / ep_mgpu_combine / IPC calls: every bad argument is
  refused on the host before anything launches (no case here passes the
  checks, so no kernel ever sees the fake addresses).
* ExpertParallelGroup over two gloo ranks, with host fakes of the CUDA IPC
  and the kernels.  Checked: the order of the handle exchange and the peer
  table built from it, the all-gather of per-expert counts ahead of the
  dispatch, the barriers around dispatch and combine, the unmapping at
  close, and that ranks which disagree on the shape all refuse together.
"""

import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from combine_ep_get_06_b200 import mgpu
from combine_ep_get_06_b200.ep import EP_ERR_INVALID_ARG, EP_OK, _GeomC, _HandleC


def geom(rank=0, world=8, T=1024, k=8, E=256, a=128, H=7168, mode=ep.EP_X_BF16_TO_FP8):
    g = _GeomC()
    st = ep.lib().ep_mgpu_geometry_init(ctypes.byref(g), rank, world, T, k, E, a, H, mode)
    return st, g


def test_geometry_sizes_and_sections():
    for mode, row, scale in [(ep.EP_X_BF16, 2 * 7168, 0), (ep.EP_X_FP8, 7168, 56 * 4),
                             (ep.EP_X_BF16_TO_FP8, 7168, 56 * 4), (ep.EP_X_BF16_TO_NVFP4, 3584, 448)]:
        st, g = geom(rank=3, mode=mode)
        assert st == EP_OK
        assert g.max_recv_rows == 8 * 1024 * 8 + 32 * 127
        assert (g.row_bytes, g.scale_bytes, g.experts_per_rank) == (row, scale, 32)
        assert g.x_mode == (ep.EP_X_FP8 if mode == ep.EP_X_BF16_TO_FP8 else mode)
        R = g.max_recv_rows
        secs = [(g.off_recv_x, R * row), (g.off_recv_scales, R * scale), (g.off_recv_src, R * 4),
                (g.off_recv_topk_idx, R * 4), (g.off_recv_topk_weights, R * 4), (g.off_y, R * 7168 * 2),
                (g.off_all_counts, 8 * 256 * 4), (g.off_dest, 1024 * 8 * 8), (g.off_raw_counts, 32 * 4),
                (g.off_recv_counts, 32 * 4), (g.off_recv_offsets, 33 * 4), (g.off_num_pad_rows, 4),
                (g.off_error_word, 4)]
        end = 0
        for off, n in secs:
            assert off % 256 == 0 and off >= end      # aligned, in order, disjoint
            end = off + n
        assert g.block_bytes >= end


@pytest.mark.parametrize("kw,msg", [
    (dict(rank=8), "rank"), (dict(rank=-1), "rank"), (dict(world=3), "divisible"),
    (dict(world=0), "world"), (dict(world=256, E=256), "world"), (dict(k=0), "num_topk"),
    (dict(k=33), "num_topk"), (dict(a=0), "alignment"), (dict(T=-1), "max_tokens"),
    (dict(H=7168 + 8), "hidden"), (dict(mode=ep.EP_X_BF16_TO_NVFP4, H=48), "hidden"),
    (dict(mode=7), "mode"), (dict(T=1 << 26), "int32"), (dict(E=2048, world=2), "num_experts"),
])
def test_geometry_rejects(kw, msg):
    st, _ = geom(**kw)
    assert st == EP_ERR_INVALID_ARG
    assert msg in ep.lib().ep_last_error().decode()


FAKE = 0x7F0000000000   # never dereferenced: every call below fails its host checks


def local_handle(T=64, k=8, E=256, S=8, a=1):
    h = _HandleC()
    h.num_tokens, h.num_topk, h.num_experts, h.num_segments, h.expert_alignment = T, k, E, S, a
    h.max_recv_rows = T * k
    for name in ("counts", "recv_counts", "offsets", "seg_tokens", "slot_map", "recv_src", "pad_rows",
                 "num_pad_rows", "error_word"):
        setattr(h, name, FAKE)
    return h


@pytest.mark.parametrize("case,msg", [
    ("segments", "num_segments"), ("alignment", "expert_alignment"), ("topk", "num_topk"),
    ("tokens", "max_tokens"), ("block_null", "local_block"), ("block_misaligned", "local_block"),
    ("peers_null", "peer_blocks"), ("mode", "receive format"), ("geometry", "modified"),
    ("x_null", "x must"),
])
def test_mgpu_dispatch_rejects_before_launch(case, msg):
    st, g = geom(T=64)
    assert st == EP_OK
    h = local_handle()
    block, peers, mode, x = FAKE, FAKE, ep.EP_X_BF16_TO_FP8, FAKE
    if case == "segments":
        h.num_segments = 4
    elif case == "alignment":
        h.expert_alignment = 2
    elif case == "topk":
        h.num_topk = 4
    elif case == "tokens":
        h.num_tokens = 65
    elif case == "block_null":
        block = None
    elif case == "block_misaligned":
        block = FAKE + 16
    elif case == "peers_null":
        peers = None
    elif case == "mode":
        mode = ep.EP_X_BF16_TO_NVFP4
    elif case == "geometry":
        g.off_y += 256
    elif case == "x_null":
        x = None
    st = ep.lib().ep_mgpu_dispatch(ctypes.byref(g), ctypes.byref(h), FAKE, 1, None, mode, x, None, block,
                                   peers, None)
    assert st == EP_ERR_INVALID_ARG
    assert msg in ep.lib().ep_last_error().decode()


def test_mgpu_combine_and_ipc_reject_before_any_cuda_call():
    st, g = geom(T=64)
    h = local_handle()
    L = ep.lib()
    assert L.ep_mgpu_combine(ctypes.byref(g), ctypes.byref(h), None, FAKE, FAKE, None, None) == EP_ERR_INVALID_ARG
    assert "out" in L.ep_last_error().decode()
    assert L.ep_mgpu_combine(ctypes.byref(g), ctypes.byref(h), None, FAKE, FAKE, FAKE + 8, None) == EP_ERR_INVALID_ARG
    h.num_segments = 2
    assert L.ep_mgpu_combine(ctypes.byref(g), ctypes.byref(h), None, FAKE, FAKE, FAKE, None) == EP_ERR_INVALID_ARG
    p = ctypes.c_void_p(0)
    assert L.ep_mgpu_block_alloc(0, ctypes.byref(p)) == EP_ERR_INVALID_ARG
    assert L.ep_ipc_export(None, None) == EP_ERR_INVALID_ARG
    assert L.ep_ipc_import(None, ctypes.byref(p)) == EP_ERR_INVALID_ARG
    assert L.ep_ipc_close(None) == EP_ERR_INVALID_ARG
    assert L.ep_mgpu_block_free(None) == EP_OK
    assert L.ep_mgpu_read_total_rows(ctypes.byref(g), None, None, None) == EP_ERR_INVALID_ARG
    assert L.ep_mgpu_check_error(ctypes.byref(g), None, None, None) == EP_ERR_INVALID_ARG


# ------------------------------------------------- two gloo ranks, host fakes

class FakeBlock:
    def __init__(self, g, rank):
        self.geom, self.ptr = g, 0x10000 * (rank + 1)
        self.all_counts = torch.full((g.world, g.num_experts), -1, dtype=torch.int32)
        self.closed = False

    def close(self):
        self.closed = True


class FakeIpc:
    """Handles are the block address; a mapped peer is that address + 1 GiB."""

    def __init__(self, log):
        self.log = log

    def alloc(self, g, device):
        self.block = FakeBlock(g, g.rank)
        return self.block

    def export(self, block):
        return block.ptr.to_bytes(8, "little") + bytes(56)

    def open(self, handle):
        p = int.from_bytes(handle[:8], "little") + (1 << 30)
        self.log.append(("open", p))
        return p

    def close(self, ptr):
        self.log.append(("close", ptr))


class FakeHandle:
    def __init__(self, counts):
        self.counts = counts


class FakeKernels:
    """Counts by the oracle; records what the dispatch saw."""

    def __init__(self, group_ref, log, E, world):
        self.group_ref, self.log, self.E, self.world = group_ref, log, E, world

    def layout(self, topk_idx):
        lay = oracle.layout(topk_idx.numpy(), self.E, self.world, 1)
        self.log.append("layout")
        return FakeHandle(torch.from_numpy(lay["counts"].astype(np.int32)))

    def dispatch(self, h, x, topk_idx, topk_weights, use_fp8=False, use_nvfp4=False):
        self.log.append(("dispatch", self.group_ref[0].block.all_counts.clone()))

    def combine(self, h, topk_weights, out):
        self.log.append("combine")
        return "out"


class LoggingComm(mgpu._TorchComm):
    def __init__(self, log):
        super().__init__(None)
        self.log = log

    def barrier(self, device):
        self.log.append("barrier")
        super().barrier(device)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out, mismatch):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        log, ref = [], [None]
        E, k = 16, 2
        T = 64 + (8 if (mismatch and rank == 1) else 0)
        try:
            grp = mgpu.ExpertParallelGroup(T, k, E, 256, mode=ep.EP_X_BF16, device="cpu", comm=LoggingComm(log),
                                           ipc=FakeIpc(log), kernels=FakeKernels(ref, log, E, world))
        except ValueError as exc:
            out[rank] = ("refused", str(exc))
            return
        ref[0] = grp
        inp = W.make_inputs("tiny", seed=40 + rank, T=64)
        h = grp.dispatch(torch.zeros(64, 256), torch.from_numpy(inp["topk_idx"]))
        res = grp.combine(h)
        grp.close()
        seen = [e for e in log if isinstance(e, tuple) and e[0] == "dispatch"][0][1]
        out[rank] = ("ok", grp.peers.tolist(), seen.numpy().tolist(),
                     [e if isinstance(e, str) else e[0] for e in log], res, grp.block.closed)
    finally:
        dist.destroy_process_group()


def _run(mismatch=False):
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out, mismatch), nprocs=world, join=True,
                       start_method="spawn")
    return dict(out)


def test_group_exchanges_handles_and_counts_in_order():
    out = _run()
    E, k = 16, 2
    expect = [oracle.layout(W.make_inputs("tiny", seed=40 + r, T=64)["topk_idx"], E, 2, 1)["counts"].tolist()
              for r in range(2)]
    for rank in range(2):
        status, peers, seen, events, res, closed = out[rank]
        assert status == "ok"
        other = 1 - rank
        assert peers[rank] == 0x10000 * (rank + 1)                   # own block by its own address
        assert peers[other] == 0x10000 * (other + 1) + (1 << 30)     # the peer's, as mapped here
        assert seen == expect                                        # counts gathered before dispatch
        # order: open peer; layout, (all-gather), dispatch, barrier; barrier, combine; close
        assert events == ["open", "layout", "dispatch", "barrier", "barrier", "combine",
                          "barrier", "close", "barrier"]
        assert res == "out" and closed


def test_ranks_that_disagree_on_the_shape_all_refuse():
    out = _run(mismatch=True)
    assert out[0][0] == "refused" and out[1][0] == "refused"
    assert "disagree" in out[0][1]
