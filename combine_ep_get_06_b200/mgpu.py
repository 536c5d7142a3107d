"""Expert parallelism across GPUs: the binding of include/ep_multi.h.

Segments are ranks (DeepEP V2 README, "Performance": EP over the GPUs of an
NVLink domain).  Each rank owns a rank block with the same section offsets
on every rank; the dispatch kernel stores rows into the owners' blocks and
the combine kernel loads expert outputs from them, through a device table
of the W blocks' addresses.

Layers:
  * ``Geometry`` / ``RankBlock``: one rank's block and tensor views of its
    sections (receive rows, scales, metadata, y, totals).
  * ``RankEP``: the per-rank calls -- layout, dispatch, combine -- given a
    block and a peer table.  No collective.
  * ``ExpertParallelGroup``: one process per GPU over torch.distributed.
    It exchanges the blocks by CUDA IPC, all-gathers the per-expert counts
    before each dispatch, and runs the barriers the ordering needs.
  * ``LocalRanks``: all W ranks' blocks on one GPU, with the all-gather
    done as device copies.  This is the form the one-GPU tests and the
    benchmark run.
"""

from __future__ import annotations

import ctypes
from typing import List, Optional, Sequence

import torch

from .ep import (EP_X_BF16, EP_X_BF16_TO_FP8, EP_X_BF16_TO_NVFP4, EP_X_FP8, EPHandle, _GeomC,
                 _check, _need, _ptr, _stream, lib)

IPC_HANDLE_BYTES = 64


def _mode_of(x, use_fp8: bool, use_nvfp4: bool) -> int:
    if use_fp8 and use_nvfp4:
        raise ValueError("use_fp8 and use_nvfp4 are exclusive")
    if isinstance(x, (tuple, list)):
        return EP_X_FP8
    return EP_X_BF16_TO_NVFP4 if use_nvfp4 else EP_X_BF16_TO_FP8 if use_fp8 else EP_X_BF16


class Geometry:
    """ep_mgpu_geometry of one rank."""

    def __init__(self, rank: int, world: int, max_tokens: int, num_topk: int, num_experts: int,
                 hidden: int, *, expert_alignment: int = 1, mode: int = EP_X_BF16_TO_FP8):
        self.c = _GeomC()
        _check(lib().ep_mgpu_geometry_init(ctypes.byref(self.c), rank, world, max_tokens, num_topk,
                                           num_experts, expert_alignment, hidden, mode), "geometry")

    def __getattr__(self, name):
        c = self.__dict__.get("c")
        if c is not None and hasattr(c, name):
            return getattr(c, name)
        raise AttributeError(name)

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def key(self) -> tuple:
        """What every rank must agree on (all but the rank)."""
        c = self.c
        return (c.world, c.max_tokens, c.num_topk, c.num_experts, c.expert_alignment, c.hidden, c.x_mode,
                c.block_bytes)


class _CudaArray:
    """__cuda_array_interface__ over raw device memory (for torch.as_tensor)."""

    def __init__(self, ptr: int, nbytes: int):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3, "strides": None}


class RankBlock:
    """One rank's block.  ``memory`` (a uint8 device tensor of at least
    block_bytes, 256-byte aligned) backs it; without it the block is
    allocated by the library (cudaMalloc), as CUDA IPC needs."""

    def __init__(self, geom: Geometry, device, memory: Optional[torch.Tensor] = None):
        self.geom = geom
        self.device = torch.device(device)
        self._owned = None
        if memory is None:
            p = ctypes.c_void_p(0)
            _check(lib().ep_mgpu_block_alloc(geom.block_bytes, ctypes.byref(p)), "block_alloc")
            self._owned = p.value
            memory = torch.as_tensor(_CudaArray(p.value, geom.block_bytes), device=self.device)
        if memory.dtype != torch.uint8 or memory.numel() < geom.block_bytes or memory.data_ptr() % 256:
            raise ValueError("block memory must be uint8, >= block_bytes and 256-byte aligned")
        self.mem = memory
        self.ptr = memory.data_ptr()
        g, R, H = geom, geom.max_recv_rows, geom.hidden

        def sec(off, nbytes, dtype=torch.uint8):
            return memory[off: off + nbytes].view(dtype)

        fmt = g.x_mode
        if fmt == EP_X_BF16:
            self.recv_x = sec(g.off_recv_x, R * g.row_bytes).view(torch.bfloat16).view(R, H)
            self.recv_scales = None
        elif fmt == EP_X_FP8:
            self.recv_x = sec(g.off_recv_x, R * g.row_bytes).view(torch.float8_e4m3fn).view(R, H)
            self.recv_scales = sec(g.off_recv_scales, R * g.scale_bytes, torch.float32).view(R, H // 128)
        else:
            self.recv_x = sec(g.off_recv_x, R * g.row_bytes).view(R, H // 2)
            self.recv_scales = sec(g.off_recv_scales, R * g.scale_bytes).view(R, H // 16)
        self.recv_src = sec(g.off_recv_src, R * 4, torch.int32)
        self.recv_topk_idx = sec(g.off_recv_topk_idx, R * 4, torch.int32)
        self.recv_topk_weights = sec(g.off_recv_topk_weights, R * 4, torch.float32)
        self.y = sec(g.off_y, R * H * 2).view(torch.bfloat16).view(R, H)
        epr = g.experts_per_rank
        self.all_counts = sec(g.off_all_counts, g.world * g.num_experts * 4, torch.int32).view(
            g.world, g.num_experts)
        self.dest = sec(g.off_dest, g.max_tokens * g.num_topk * 8, torch.int32).view(-1, 2)
        self.raw_counts = sec(g.off_raw_counts, epr * 4, torch.int32)
        self.recv_counts = sec(g.off_recv_counts, epr * 4, torch.int32)
        self.recv_offsets = sec(g.off_recv_offsets, (epr + 1) * 4, torch.int32)
        self.num_pad_rows = sec(g.off_num_pad_rows, 4, torch.int32)
        self.error_word = sec(g.off_error_word, 4, torch.int32)
        self.error_word.zero_()

    def close(self):
        if self._owned is not None:
            torch.cuda.synchronize(self.device)
            self.mem = None
            _check(lib().ep_mgpu_block_free(self._owned), "block_free")
            self._owned = None


class RankEP:
    """The per-rank steps of one multi-GPU dispatch / combine: no collective.

    ``peers`` is the device table [W] int64 of the blocks' addresses in this
    process (peers[rank] == block.ptr)."""

    def __init__(self, geom: Geometry, block: RankBlock, peers: torch.Tensor):
        _need(peers, "peers", (torch.int64,), block.device, 1)
        if peers.numel() != geom.world:
            raise ValueError("peer table must have world entries")
        self.geom, self.block, self.peers = geom, block, peers
        self.device = block.device
        self._handles = {}

    def handle(self, num_tokens: int) -> EPHandle:
        """The local layout handle for num_tokens (cached per size)."""
        h = self._handles.get(num_tokens)
        if h is None:
            g = self.geom
            if num_tokens > g.max_tokens:
                raise ValueError(f"{num_tokens} tokens > max_tokens {g.max_tokens}")
            h = EPHandle(num_tokens, g.num_topk, g.num_experts, g.world, 1, device=self.device)
            self._handles[num_tokens] = h
        return h

    def layout(self, topk_idx: torch.Tensor) -> EPHandle:
        """Step 1: this rank's counts (handle.counts, the all-gather's input)."""
        _need(topk_idx, "topk_idx", (torch.int64, torch.int32), self.device, 2)
        T, k = topk_idx.shape
        if k != self.geom.num_topk:
            raise ValueError("topk_idx has the wrong number of columns")
        h = self.handle(T)
        _check(lib().ep_get_layout(h.ref, topk_idx.data_ptr(), int(topk_idx.dtype == torch.int64), None,
                                   None, None, h.workspace_ptr, h.workspace_bytes, _stream(self.device)),
               "mgpu layout")
        return h

    def dispatch(self, handle: EPHandle, x, topk_idx: torch.Tensor, topk_weights=None, *,
                 use_fp8: bool = False, use_nvfp4: bool = False):
        """Step 3, after all_counts holds every rank's handle.counts."""
        mode = _mode_of(x, use_fp8, use_nvfp4)
        x_scales = None
        if isinstance(x, (tuple, list)):
            x, x_scales = x
            _need(x, "x[0]", (torch.float8_e4m3fn, torch.uint8), self.device, 2)
            _need(x_scales, "x[1]", (torch.float32,), self.device, 2)
        else:
            _need(x, "x", (torch.bfloat16,), self.device, 2)
        if x.shape != (handle.num_tokens, self.geom.hidden):
            raise ValueError("x must be [num_tokens, hidden]")
        if topk_weights is not None:
            _need(topk_weights, "topk_weights", (torch.float32,), self.device, 2)
        _check(lib().ep_mgpu_dispatch(self.geom.ref, handle.ref, topk_idx.data_ptr(),
                                      int(topk_idx.dtype == torch.int64), _ptr(topk_weights), mode,
                                      x.data_ptr(), _ptr(x_scales), self.block.ptr, self.peers.data_ptr(),
                                      _stream(self.device)), "mgpu dispatch")

    def combine(self, handle: EPHandle, topk_weights=None, out: Optional[torch.Tensor] = None):
        """Step 7, after every rank's y is complete."""
        T, H = handle.num_tokens, self.geom.hidden
        if out is None:
            out = torch.empty(T, H, dtype=torch.bfloat16, device=self.device)
        _need(out, "out", (torch.bfloat16,), self.device, 2)
        if topk_weights is not None:
            _need(topk_weights, "topk_weights", (torch.float32,), self.device, 2)
        _check(lib().ep_mgpu_combine(self.geom.ref, handle.ref, _ptr(topk_weights), self.block.ptr,
                                     self.peers.data_ptr(), out.data_ptr(), _stream(self.device)),
               "mgpu combine")
        return out

    def total_rows(self) -> int:
        r = ctypes.c_int32(0)
        _check(lib().ep_mgpu_read_total_rows(self.geom.ref, self.block.ptr, ctypes.byref(r),
                                             _stream(self.device)), "total_rows")
        return r.value

    def check_error(self) -> int:
        bits = ctypes.c_uint32(0)
        _check(lib().ep_mgpu_check_error(self.geom.ref, self.block.ptr, ctypes.byref(bits),
                                         _stream(self.device)), "check_error")
        return bits.value


class LocalRanks:
    """W ranks with all blocks on one GPU.  The peer table holds plain
    device addresses and the all-gather is a device copy.  The ranks'
    launches run one after another on the current stream, or, with
    ``concurrent``, each rank's on a stream of its own, joined by events
    around the exchange and at the end.  No kernel waits on another."""

    def __init__(self, world: int, max_tokens: int, num_topk: int, num_experts: int, hidden: int, *,
                 expert_alignment: int = 1, mode: int = EP_X_BF16_TO_FP8, device=None,
                 concurrent: bool = False):
        device = torch.device("cuda") if device is None else torch.device(device)
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.world, self.device = world, device
        self.geoms = [Geometry(r, world, max_tokens, num_topk, num_experts, hidden,
                               expert_alignment=expert_alignment, mode=mode) for r in range(world)]
        nbytes = self.geoms[0].block_bytes
        self.blocks = [RankBlock(g, device, torch.empty(nbytes, dtype=torch.uint8, device=device))
                       for g in self.geoms]
        self.peers = torch.tensor([b.ptr for b in self.blocks], dtype=torch.int64, device=device)
        self.ranks = [RankEP(g, b, self.peers) for g, b in zip(self.geoms, self.blocks)]
        self.streams = [torch.cuda.Stream(device) for _ in range(world)] if concurrent else None

    def _per_rank(self, fn):
        """fn(r) for every rank: in order on the current stream, or each on
        its own stream after the current stream's work, joined back."""
        if self.streams is None:
            return [fn(r) for r in range(self.world)]
        main = torch.cuda.current_stream(self.device)
        out = []
        for r, s in enumerate(self.streams):
            s.wait_stream(main)
            with torch.cuda.stream(s):
                out.append(fn(r))
        for s in self.streams:
            main.wait_stream(s)
        return out

    def exchange_counts(self, handles: Sequence[EPHandle]):
        """The all-gather of step 2, as device copies: one stack, then one
        multi-tensor copy into every block (a launch each instead of one per
        block)."""
        stacked = torch.stack([h.counts for h in handles])
        dsts = [b.all_counts for b in self.blocks]
        if hasattr(torch, "_foreach_copy_"):
            torch._foreach_copy_(dsts, [stacked] * len(dsts))
        else:
            for d in dsts:
                d.copy_(stacked)

    def dispatch(self, xs, topk_idxs, topk_weights=None, *, use_fp8=False, use_nvfp4=False) -> List[EPHandle]:
        handles = self._per_rank(lambda r: self.ranks[r].layout(topk_idxs[r]))
        self.exchange_counts(handles)
        ws = topk_weights if topk_weights is not None else [None] * self.world
        self._per_rank(lambda r: self.ranks[r].dispatch(handles[r], xs[r], topk_idxs[r], ws[r], use_fp8=use_fp8,
                                                        use_nvfp4=use_nvfp4))
        return handles

    def combine(self, handles, topk_weights=None, outs=None):
        ws = topk_weights if topk_weights is not None else [None] * self.world
        os_ = outs if outs is not None else [None] * self.world
        return self._per_rank(lambda r: self.ranks[r].combine(handles[r], ws[r], os_[r]))


class _TorchComm:
    """The collectives of the multi-GPU step, over torch.distributed."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self._nccl = dist.get_backend(group) == "nccl"
        self._word = None

    def all_gather_objects(self, obj) -> list:
        out = [None] * self.world
        self.dist.all_gather_object(out, obj, group=self.group)
        return out

    def all_gather_counts(self, out: torch.Tensor, inp: torch.Tensor):
        if self._nccl:
            self.dist.all_gather_into_tensor(out.view(-1), inp, group=self.group)
        else:
            self.dist.all_gather(list(out.unbind(0)), inp, group=self.group)

    def barrier(self, device):
        if self._word is None or self._word.device != torch.device(device):
            self._word = torch.zeros(1, dtype=torch.int32, device=device)
        self.dist.all_reduce(self._word, group=self.group)


class _SingleRank:
    """The collectives of a group of one rank (no process group)."""

    rank, world = 0, 1

    def all_gather_objects(self, obj) -> list:
        return [obj]

    def all_gather_counts(self, out: torch.Tensor, inp: torch.Tensor):
        out[0].copy_(inp)

    def barrier(self, device):
        pass


def _default_comm(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return _TorchComm(group)
    return _SingleRank()


class _CudaIpc:
    """Block allocation and CUDA IPC through the library."""

    def alloc(self, geom: Geometry, device) -> RankBlock:
        return RankBlock(geom, device)

    def export(self, block: RankBlock) -> bytes:
        buf = (ctypes.c_char * IPC_HANDLE_BYTES)()
        _check(lib().ep_ipc_export(block.ptr, buf), "ipc_export")
        return bytes(buf)

    def open(self, handle: bytes) -> int:
        p = ctypes.c_void_p(0)
        buf = (ctypes.c_char * IPC_HANDLE_BYTES).from_buffer_copy(handle)
        _check(lib().ep_ipc_import(buf, ctypes.byref(p)), "ipc_import")
        return p.value

    def close(self, ptr: int):
        _check(lib().ep_ipc_close(ptr), "ipc_close")


class ExpertParallelGroup:
    """One process per GPU: rank r of the group owns experts
    [r*E/W, (r+1)*E/W).  ``dispatch`` runs layout, the all-gather of counts,
    the dispatch kernel and a barrier; ``combine`` a barrier and the combine
    kernel.  Received rows, their metadata and y are views of ``block``.

    Every rank must make the same calls in the same order (each one holds
    collectives).  ``comm``, ``ipc`` and ``kernels`` default to
    torch.distributed (a group of one rank when no process group is
    initialised), CUDA IPC and this library; tests pass host fakes."""

    def __init__(self, max_tokens: int, num_topk: int, num_experts: int, hidden: int, *,
                 expert_alignment: int = 1, mode: int = EP_X_BF16_TO_FP8, group=None, device=None,
                 comm=None, ipc=None, kernels=None):
        self.comm = comm if comm is not None else _default_comm(group)
        self.ipc = ipc if ipc is not None else _CudaIpc()
        self.rank, self.world = self.comm.rank, self.comm.world
        self.device = torch.device(device) if device is not None else torch.device(
            "cuda", torch.cuda.current_device())
        self.geom = Geometry(self.rank, self.world, max_tokens, num_topk, num_experts, hidden,
                             expert_alignment=expert_alignment, mode=mode)
        keys = self.comm.all_gather_objects(self.geom.key())
        if any(k != keys[0] for k in keys):
            raise ValueError(f"ranks disagree on the expert-parallel shape: {keys}")
        self.block = self.ipc.alloc(self.geom, self.device)
        handles = self.comm.all_gather_objects(self.ipc.export(self.block))
        self._opened = {}
        ptrs = []
        for r, hb in enumerate(handles):
            if r == self.rank:
                ptrs.append(self.block.ptr)
            else:
                self._opened[r] = self.ipc.open(hb)
                ptrs.append(self._opened[r])
        self.peers = torch.tensor(ptrs, dtype=torch.int64, device=self.device)
        self.kernels = kernels if kernels is not None else RankEP(self.geom, self.block, self.peers)

    def dispatch(self, x, topk_idx: torch.Tensor, topk_weights=None, *, use_fp8=False, use_nvfp4=False):
        """-> the local layout handle; received rows are in self.block."""
        h = self.kernels.layout(topk_idx)
        self.comm.all_gather_counts(self.block.all_counts, h.counts)
        self.kernels.dispatch(h, x, topk_idx, topk_weights, use_fp8=use_fp8, use_nvfp4=use_nvfp4)
        self.comm.barrier(self.device)
        return h

    def combine(self, handle, topk_weights=None, out=None):
        """After this rank's expert outputs are in self.block.y."""
        self.comm.barrier(self.device)
        return self.kernels.combine(handle, topk_weights, out)

    def close(self):
        """Collective: every rank unmaps its peers, then frees its block."""
        self.comm.barrier(self.device)
        for ptr in self._opened.values():
            self.ipc.close(ptr)
        self._opened = {}
        self.comm.barrier(self.device)
        self.block.close()
