"""Multi-GPU expert parallelism, its kernels checked with all ranks on one GPU.

W ranks' blocks live on one device (LocalRanks): every dispatch stores
into the owners' blocks through the peer table, just as over NVLink.  The
reference is the oracle's one-GPU layout of the W batches concatenated in
rank order, with num_segments = W: rank d's block must hold exactly that
layout's rows of d's experts, renumbered from 0.  Everything is compared
bit for bit: codes, scales, recv_src (as rank, slot), recv_topk_idx and
weights, totals, each slot's (rank, row), and the combine output.  Rows
past each rank's total keep their sentinel."""

import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads as W
import combine_ep_get_06_b200 as ep
from combine_ep_get_06_b200 import mgpu
from gpu_helpers import SENTINEL, to_dev_bf16

pytestmark = pytest.mark.gpu

MODES = {"bf16": (ep.EP_X_BF16, oracle.X_BF16), "fp8": (ep.EP_X_BF16_TO_FP8, oracle.X_BF16_QUANT_FP8),
         "prequant": (ep.EP_X_FP8, oracle.X_FP8_PREQUANT), "nvfp4": (ep.EP_X_BF16_TO_NVFP4, oracle.X_BF16_QUANT_NVFP4)}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def run_case(w: W.Workload, world: int, Ts, mode_name: str, *, seed=0, idx_int32=False, weighted=True):
    gpu_mode, o_mode = MODES[mode_name]
    E, k, a, H = w.E, w.k, w.align, w.H
    epr = E // world
    Tmax = max(max(Ts), 1)
    inps = [W.make_inputs(w, seed=seed * 101 + r, T=Ts[r]) for r in range(world)]
    pqs = [W.make_prequant(Ts[r], H, seed=seed * 101 + r) for r in range(world)] if mode_name == "prequant" else None

    lr = mgpu.LocalRanks(world, Tmax, k, E, H, expert_alignment=a, mode=gpu_mode)
    for b in lr.blocks:
        b.mem.fill_(SENTINEL)
        b.error_word.zero_()
    if pqs is not None:
        xs = [(torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda()) for q, s in pqs]
    else:
        xs = [to_dev_bf16(i["x"]) for i in inps]
    idxs = [torch.from_numpy(i["topk_idx"]).cuda() for i in inps]
    if idx_int32:
        idxs = [i.to(torch.int32) for i in idxs]
    wts = [torch.from_numpy(i["topk_weights"]).cuda() for i in inps] if weighted else None
    handles = lr.dispatch(xs, idxs, wts, use_fp8=mode_name == "fp8", use_nvfp4=mode_name == "nvfp4")
    torch.cuda.synchronize()

    # the oracle over the concatenated batch
    cum = np.concatenate([[0], np.cumsum(Ts)]).astype(np.int64)
    idx_all = np.concatenate([i["topk_idx"] for i in inps])
    w_all = np.concatenate([i["topk_weights"] for i in inps])
    lay = oracle.layout(idx_all, E, world, a, w_all if weighted else None)
    if pqs is not None:
        q_all, s_all = oracle.dispatch(lay, np.concatenate([p[0] for p in pqs]), o_mode,
                                       np.concatenate([p[1] for p in pqs]))
    else:
        q_all, s_all = oracle.dispatch(lay, np.concatenate([i["x"] for i in inps]), o_mode)
    off = lay["offsets"]

    def local_src(gs):
        gs = np.asarray(gs, np.int64)
        out = np.full(gs.shape, -1, np.int64)
        ok = gs >= 0
        tg, j = gs[ok] // k, gs[ok] % k
        r = np.searchsorted(cum, tg, side="right") - 1
        out[ok] = r * Tmax * k + (tg - cum[r]) * k + j
        return out.astype(np.int32)

    for d, b in enumerate(lr.blocks):
        base, end = off[d * epr], off[(d + 1) * epr]
        R = end - base
        assert lr.ranks[d].total_rows() == R
        np.testing.assert_array_equal(b.recv_offsets.cpu().numpy(), off[d * epr:(d + 1) * epr + 1] - base)
        np.testing.assert_array_equal(b.raw_counts.cpu().numpy(), lay["counts"][d * epr:(d + 1) * epr])
        np.testing.assert_array_equal(b.recv_counts.cpu().numpy(), np.diff(off[d * epr:(d + 1) * epr + 1]))
        assert int(b.num_pad_rows.item()) == R - int(lay["counts"][d * epr:(d + 1) * epr].sum())
        rx = b.recv_x.view(torch.uint8).cpu().numpy()
        qv = q_all.view(np.uint8).reshape(q_all.shape[0], -1)
        np.testing.assert_array_equal(rx[:R], qv[base:end])
        assert np.all(rx[R:] == SENTINEL)
        if b.recv_scales is not None:
            rs = b.recv_scales.view(torch.uint8).cpu().numpy()
            sv = s_all.view(np.uint8).reshape(s_all.shape[0], -1)
            np.testing.assert_array_equal(rs[:R], sv[base:end])
            assert np.all(rs[R:] == SENTINEL)
        np.testing.assert_array_equal(b.recv_src.cpu().numpy()[:R], local_src(lay["recv_src"][base:end]))
        np.testing.assert_array_equal(b.recv_topk_idx.cpu().numpy()[:R], lay["recv_topk_idx"][base:end])
        np.testing.assert_array_equal(b.recv_topk_weights.cpu().numpy()[:R].view(np.uint32),
                                      lay["recv_topk_weights"][base:end].view(np.uint32))
        assert np.all(b.recv_src.view(torch.uint8).cpu().numpy()[4 * R:] == SENTINEL)
        assert lr.ranks[d].check_error() == 0

    # each slot's (rank, row)
    sm = lay["slot_map"]
    for r, b in enumerate(lr.blocks):
        T = Ts[r]
        got = b.dest.cpu().numpy()[: T * k]
        g_rows = sm[cum[r] * k:(cum[r] + T) * k]
        e = inps[r]["topk_idx"].reshape(-1)
        dd = np.where(g_rows >= 0, np.clip(e, 0, E - 1) // epr, -1)
        rr = np.where(g_rows >= 0, g_rows - off[np.clip(dd, 0, world - 1) * epr], -1)
        np.testing.assert_array_equal(got[:, 0], dd)
        np.testing.assert_array_equal(got[:, 1], rr)

    # combine: expert outputs y placed in each owner's block
    y_all = W.make_y(w, seed=seed + 7, rows=lay["max_rows"])
    for d, b in enumerate(lr.blocks):
        base, end = off[d * epr], off[(d + 1) * epr]
        if end > base:
            b.y[: end - base].copy_(to_dev_bf16(y_all[base:end]))
    outs = lr.combine(handles, wts)
    torch.cuda.synchronize()
    o_all, _ = oracle.combine(sm, int(cum[-1]), k, y_all, w_all if weighted else None)
    for r in range(world):
        got = outs[r].view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(got, o_all[cum[r]:cum[r + 1]])
        assert lr.ranks[r].check_error() == 0
    return lr, lay


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_v3_ranks_fp8_match_oracle(world):
    w = W.WORKLOADS["v3"]
    run_case(w, world, [8192 // world] * world, "fp8", seed=world)


@pytest.mark.parametrize("mode", ["bf16", "prequant", "nvfp4"])
def test_modes_match_oracle(mode):
    w = W.WORKLOADS["mid"]
    run_case(w, 4, [700, 512, 333, 640], mode, seed=3)


def test_skewed_ragged_ranks_with_an_empty_rank():
    w = W.WORKLOADS["skewed"]
    run_case(w, 8, [1024, 0, 900, 1024, 17, 600, 1, 1000], "fp8", seed=4)


def test_int32_idx_and_unweighted_combine():
    w = W.WORKLOADS["mid"]
    run_case(w, 2, [1500, 1200], "fp8", seed=5, idx_int32=True, weighted=False)


@pytest.mark.parametrize("align", [1, 16])
def test_decode_shape_and_alignments(align):
    w = dataclasses.replace(W.WORKLOADS["decode"], align=align)
    run_case(w, 8, [16] * 8, "fp8", seed=6)


def test_bad_indices_are_dropped_and_flagged_by_the_layout():
    w = W.WORKLOADS["tiny"]
    inps_T = [128, 100]
    lr, lay = run_case(w, 2, inps_T, "bf16", seed=8)
    # run again with planted bad indices on rank 1
    inp0 = W.make_inputs(w, seed=9, T=64)
    inp1 = W.make_inputs(w, seed=10, T=64)
    inp1["topk_idx"][3, 0] = w.E + 5
    inp1["topk_idx"][7, 1] = -9
    idxs = [torch.from_numpy(inp0["topk_idx"]).cuda(), torch.from_numpy(inp1["topk_idx"]).cuda()]
    xs = [to_dev_bf16(inp0["x"]), to_dev_bf16(inp1["x"])]
    handles = lr.dispatch(xs, idxs)
    torch.cuda.synchronize()
    assert handles[0].check_error() == 0
    with pytest.raises(ep.EPError):
        handles[1].check_error()
    d1 = lr.blocks[1].dest.cpu().numpy()[: 64 * w.k]
    assert tuple(d1[3 * w.k + 0]) == (-1, -1) and tuple(d1[7 * w.k + 1]) == (-1, -1)
    for r in lr.ranks:
        assert r.check_error() == 0


def test_capacity_error_when_counts_are_not_from_this_step():
    # all_counts that understate the traffic: rows past max_recv_rows are
    # skipped and flagged, nothing is written out of bounds
    w = dataclasses.replace(W.WORKLOADS["tiny"], align=1)
    lr = mgpu.LocalRanks(2, 64, w.k, w.E, w.H, mode=ep.EP_X_BF16)
    inps = [W.make_inputs(w, seed=20 + r, T=64) for r in range(2)]
    idxs = [torch.from_numpy(i["topk_idx"]).cuda() for i in inps]
    xs = [to_dev_bf16(i["x"]) for i in inps]
    for b in lr.blocks:
        b.mem.fill_(SENTINEL)
        b.error_word.zero_()
    handles = [r.layout(i) for r, i in zip(lr.ranks, idxs)]
    lr.exchange_counts(handles)
    for b in lr.blocks:   # pretend rank 0 sent far more to every expert
        b.all_counts[0].add_(10_000)
    for r, h, x, i in zip(lr.ranks, handles, xs, idxs):
        r.dispatch(h, x, i)
    torch.cuda.synchronize()
    bits = [int(b.error_word.item()) for b in lr.blocks]
    assert all(v & ep.EP_DEVERR_CAPACITY for v in bits)
    # sections a bf16 dispatch never writes keep their sentinel
    g = lr.geoms[0]
    for b in lr.blocks:
        assert bool((b.mem[g.off_recv_scales: g.off_recv_src] == SENTINEL).all())
        assert bool((b.y.view(torch.uint8) == SENTINEL).all())


def test_concurrent_ranks_give_the_same_bytes():
    # each rank's launches on a stream of its own (joined by events around
    # the exchange): identical blocks and outputs to the sequential form
    w = W.WORKLOADS["mid"]
    world, Ts = 4, [800, 640, 1024, 512]
    inps = [W.make_inputs(w, seed=60 + r, T=Ts[r]) for r in range(world)]
    xs = [to_dev_bf16(i["x"]) for i in inps]
    idxs = [torch.from_numpy(i["topk_idx"]).cuda() for i in inps]
    wts = [torch.from_numpy(i["topk_weights"]).cuda() for i in inps]
    ys = None
    res = []
    for concurrent in (False, True):
        lr = mgpu.LocalRanks(world, 1024, w.k, w.E, w.H, expert_alignment=w.align, concurrent=concurrent)
        for b in lr.blocks:
            b.mem.fill_(SENTINEL)
            b.error_word.zero_()
        hs = lr.dispatch(xs, idxs, wts, use_fp8=True)
        if ys is None:
            ys = [torch.randn(b.y.shape, device="cuda").to(torch.bfloat16) for b in lr.blocks]
        for b, y in zip(lr.blocks, ys):
            b.y.copy_(y)
        outs = lr.combine(hs, wts)
        torch.cuda.synchronize()
        g = lr.geoms[0]
        res.append(([b.mem[: g.off_y].clone() for b in lr.blocks],
                    [b.mem[g.off_all_counts: g.block_bytes].clone() for b in lr.blocks], outs))
    for a, b in zip(res[0][0] + res[0][1], res[1][0] + res[1][1]):
        assert torch.equal(a, b)
    for a, b in zip(res[0][2], res[1][2]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))



@pytest.mark.parametrize("world,E,k", [(16, 64, 12), (64, 64, 32), (3, 48, 20), (2, 64, 9)])
def test_many_ranks_large_topk(world, E, k):
    # k > 8 takes the combine's 2-4 groups of 8 slots; E/W down to one expert per rank
    w = dataclasses.replace(W.WORKLOADS["tiny"], name=f"w{world}_e{E}_k{k}", E=E, S=world, k=k, align=4)
    # blocks hold world * max_tokens * k rows each: few tokens per rank when many ranks
    Ts = [8 + r % 5 for r in range(world)] if world >= 16 else [40 + 3 * r for r in range(world)]
    run_case(w, world, Ts, "bf16", seed=world + k)


@pytest.mark.parametrize("mode,H", [("fp8", 1152), ("fp8", 384), ("prequant", 1152), ("nvfp4", 1056),
                                    ("bf16", 1032)])
def test_ragged_hidden_sizes(mode, H):
    # a last slice shorter than 1024 elements, and scale rows that are not a
    # multiple of 16 bytes (FP8 at H=1152: 36 B; NVFP4 at H=1056: 66 B), so
    # the peer stores fall back to 4- and 1-byte units
    w = dataclasses.replace(W.WORKLOADS["mid"], name=f"mid_h{H}", H=H, align=8)
    run_case(w, 4, [200, 77, 150, 33], mode, seed=H)
