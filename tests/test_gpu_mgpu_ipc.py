"""The multi-process expert-parallel path on one GPU, through real CUDA IPC.

Two or four processes share GPU 0, one per rank.  Each allocates its rank block
with the library (cudaMalloc) and exports it.  Every other process maps it
(cudaIpcOpenMemHandle), and the dispatch and combine kernels store into
and load from the peers' blocks.  The ranks' kernels never wait on one
another: each step's ordering comes from the host, where every collective
first synchronises the rank's stream and then meets the other ranks over
gloo.  Each rank checks its own block and its combine output bit for bit
against the oracle's one-GPU layout of the concatenated batch, then the
group unmaps and frees."""

import datetime
import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu


class HostComm:
    """The group's collectives over gloo, for ranks that share one GPU: the
    device side is synchronised before every exchange."""

    def __init__(self):
        self.rank, self.world = dist.get_rank(), dist.get_world_size()

    def all_gather_objects(self, obj):
        out = [None] * self.world
        dist.all_gather_object(out, obj)
        return out

    def all_gather_counts(self, out, inp):
        torch.cuda.synchronize()
        parts = [torch.empty_like(inp, device="cpu") for _ in range(self.world)]
        dist.all_gather(parts, inp.cpu())
        out.copy_(torch.stack(parts))

    def barrier(self, device):
        torch.cuda.synchronize()
        dist.barrier()


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    # a short timeout: a rank that fails ends the other's next collective
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        import workloads as W
        import combine_ep_get_06_b200 as ep
        from combine_ep_get_06_b200 import mgpu

        w = W.WORKLOADS["mid"]
        Ts = [700, 512, 300, 640][:world]
        Tmax, E, k, a, H = 1024, w.E, w.k, w.align, w.H
        epr = E // world
        inps = [W.make_inputs(w, seed=80 + r, T=Ts[r]) for r in range(world)]
        grp = mgpu.ExpertParallelGroup(Tmax, k, E, H, expert_alignment=a, mode=ep.EP_X_BF16_TO_FP8,
                                       device="cuda:0", comm=HostComm())
        blk = grp.block
        blk.mem.fill_(0xA5)
        blk.error_word.zero_()
        grp.comm.barrier(grp.device)   # no peer stores before both blocks are filled

        mine = inps[rank]
        bf = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
        x = bf(mine["x"])
        idx = torch.from_numpy(mine["topk_idx"]).cuda()
        wts = torch.from_numpy(mine["topk_weights"]).cuda()
        h = grp.dispatch(x, idx, wts, use_fp8=True)

        cum = np.concatenate([[0], np.cumsum(Ts)])
        idx_all = np.concatenate([i["topk_idx"] for i in inps])
        w_all = np.concatenate([i["topk_weights"] for i in inps])
        lay = oracle.layout(idx_all, E, world, a, w_all)
        q_all, s_all = oracle.dispatch(lay, np.concatenate([i["x"] for i in inps]), oracle.X_BF16_QUANT_FP8)
        off = lay["offsets"]
        base, end = off[rank * epr], off[(rank + 1) * epr]
        R = end - base
        assert grp.kernels.total_rows() == R
        np.testing.assert_array_equal(blk.recv_offsets.cpu().numpy(), off[rank * epr:(rank + 1) * epr + 1] - base)
        rx = blk.recv_x.view(torch.uint8).cpu().numpy()
        np.testing.assert_array_equal(rx[:R], q_all[base:end])
        assert np.all(rx[R:] == 0xA5)
        np.testing.assert_array_equal(blk.recv_scales.cpu().numpy()[:R].view(np.uint32),
                                      s_all[base:end].view(np.uint32))
        np.testing.assert_array_equal(blk.recv_topk_idx.cpu().numpy()[:R], lay["recv_topk_idx"][base:end])
        gs = lay["recv_src"][base:end].astype(np.int64)
        tg, j = gs // k, gs % k
        src_rank = np.searchsorted(cum, tg, side="right") - 1
        expect_src = np.where(gs >= 0, src_rank * Tmax * k + (tg - cum[src_rank]) * k + j, -1)
        np.testing.assert_array_equal(blk.recv_src.cpu().numpy()[:R], expect_src.astype(np.int32))

        y_all = W.make_y(w, seed=81, rows=lay["max_rows"])
        if R:
            blk.y[:R].copy_(bf(y_all[base:end]))
        o = grp.combine(h, wts)
        torch.cuda.synchronize()
        o_all, _ = oracle.combine(lay["slot_map"], int(cum[-1]), k, y_all, w_all)
        got = o.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, o_all[cum[rank]:cum[rank + 1]])
        assert grp.kernels.check_error() == 0
        assert h.check_error() == 0
        grp.close()
        out[rank] = "ok"
    except Exception:
        out[rank] = traceback.format_exc()
        raise
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 4])
def test_processes_share_blocks_through_cuda_ipc(world):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    try:
        mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
    finally:
        res = dict(out)
    for r in range(world):
        assert res.get(r) == "ok", res.get(r)
