"""The expert-parallel protocol's bookkeeping on the host (no GPU): the
partition of experts and tokens over R ranks, the windows' geometry, the
Sentinel and Fence steps in their stated order, checked end to end over
ranks that are threads of one process and over torch.distributed gloo
processes, against the single-process oracle layer.

Each rank routes its own tokens, pushes its rows into the owners' windows
(the host model of moe_ep_dispatch), every owner applies its experts to
whole windows once all sources have closed and every tile it takes carries
its sentinel, and each source reads its pairs' outputs where they lie. The
ranks' outputs, concatenated, must equal the oracle's layer on all tokens bit
for bit (the same arithmetic per token, applied wherever the token's rows
went). The window geometry of the model must be the library's
(moe_ep_sizes, a host call).
"""
import os
import socket
import threading

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from combine_softmax_top_b200 import ep as EP
from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W

H, I, K = 128, 128, 3


def _problem(R, T_per, seed=0):
    E = 4 * R
    rng = np.random.default_rng(seed)
    T = T_per * R
    x = rng.standard_normal((T, H)).astype(np.float32) * 0.5
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wg, wu = (rng.standard_normal((E, I, H)).astype(np.float32) * 0.05 for _ in range(2))
    wd = rng.standard_normal((E, H, I)).astype(np.float32) * 0.05
    F = oracle.F32
    p = oracle.Problem(T, H, E, K, I, x_dtype=F, xq_dtype=F, w_dtype=F, h_dtype=F, y_dtype=F, out_dtype=F,
                       renorm=1, w_gate=wg, w_up=wu, w_down=wd)
    return p, x, logits


def _rank_layer(rank, R, protocol, p, x, logits, T_per, exchange, epoch=1):
    sl = slice(rank * T_per, (rank + 1) * T_per)
    idx, w = oracle.route(logits[sl], K, 1)

    def expert_fn(e, rows):
        return oracle.expert_rows(p, np.full(len(rows), e, np.int32), rows.astype(np.float32))[2]

    y, rec = EP.model_layer(rank, R, protocol, p.E, T_per, idx, x[sl], expert_fn, epoch=epoch, exchange=exchange)
    out = oracle.combine(y.reshape(T_per * K, H).astype(np.float32), w, oracle.F32, oracle.F32)
    return out, rec, idx


class _ThreadExchange:
    """All-to-all among R threads: exchange(list of R objects) returns the
    objects the other threads addressed to the caller. `drop(src, dst, f)`
    lets a test alter what src sends dst (a lost or damaged message)."""

    def __init__(self, R, drop=None):
        self.R, self.drop = R, drop
        self.box = [[None] * R for _ in range(R)]
        self.bar = threading.Barrier(R)

    def for_rank(self, r):
        def exchange(objs):
            for d in range(self.R):
                self.box[r][d] = self.drop(r, d, objs[d]) if self.drop else objs[d]
            self.bar.wait()
            got = [self.box[s][r] for s in range(self.R)]
            self.bar.wait()
            return got
        return exchange


def _run_threads(R, protocol, T_per=40, drop=None):
    p, x, logits = _problem(R, T_per)
    ex = _ThreadExchange(R, drop)
    res, errs = [None] * R, [None] * R

    def body(r):
        try:
            res[r] = _rank_layer(r, R, protocol, p, x, logits, T_per, ex.for_rank(r))
        except Exception as e:   # reported to the test
            errs[r] = e
            ex.bar.abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(R)]
    for t in th:
        t.start()
    for t in th:
        t.join(60)
    return p, x, logits, res, errs


PROTOS = [("sentinel", moe.MOE_EP_SENTINEL), ("fence", moe.MOE_EP_FENCE)]


@pytest.mark.parametrize("pname,protocol", PROTOS, ids=[q[0] for q in PROTOS])
@pytest.mark.parametrize("R", [1, 2, 3, 4])
def test_protocol_over_thread_ranks_matches_oracle(R, pname, protocol):
    p, x, logits, res, errs = _run_threads(R, protocol)
    assert errs == [None] * R, errs
    out = np.concatenate([r[0] for r in res])
    ref = oracle.moe_layer(p, x, logits)["out"]
    assert np.array_equal(out, ref)
    T_per = p.T // R
    for rank, (_, rec, idx) in enumerate(res):
        pos = rec["pos"]
        rows = rec["rows"]
        assert np.array_equal(pos // rows, idx // (p.E // R))                 # the expert's owner
        if protocol == moe.MOE_EP_SENTINEL:                                    # the source's own region
            cap = -(-T_per // 128) * 128
            v = (idx % (p.E // R)) * R + rank
            assert ((pos % rows) // cap == v).all()
    for rank, (_, rec, _) in enumerate(res):                                   # every window row filled once
        assert len(rec["window_rows"]) == int(rec["counts"].sum())


def test_fence_windows_are_packed():
    """Fence: each owner's windows lie back to back in whole tiles, the
    bound of moe_ep_sizes respected."""
    R = 3
    p, x, logits, res, errs = _run_threads(R, moe.MOE_EP_FENCE, T_per=200)
    assert errs == [None] * R
    for rank, (_, rec, _) in enumerate(res):
        rows = np.array(rec["window_rows"])
        tiles = np.unique(rows // 128)
        assert len(tiles) == int(np.sum(-(-rec["counts"] // 128)))
        assert tiles.max() < rec["rows"] // 128


@pytest.mark.parametrize("R", [2, 4])
def test_a_lost_tile_flag_is_caught_before_the_ffn_takes_the_tile(R):
    def drop(src, dst, obj):
        if src == 1 and dst == 0 and isinstance(obj, tuple) and len(obj) == 3 and obj[1]:
            return (obj[0], obj[1][1:], obj[2])   # the first tile flag source 1 sends owner 0 is lost
        return obj
    _, _, _, _, errs = _run_threads(R, moe.MOE_EP_SENTINEL, drop=drop)
    assert isinstance(errs[0], AssertionError) and "sentinel" in str(errs[0])


@pytest.mark.parametrize("protocol", [moe.MOE_EP_SENTINEL, moe.MOE_EP_FENCE])
@pytest.mark.parametrize("R,E,k,t_max", [(1, 8, 2, 16), (2, 16, 4, 100), (4, 256, 8, 128), (8, 256, 8, 8192),
                                          (3, 12, 5, 7)])
def test_model_geometry_is_the_library_geometry(protocol, R, E, k, t_max):
    s = W.spec("decode", T=t_max, E=E, k=k)
    ep = moe.moe_ep()
    ep.ranks, ep.rank, ep.protocol, ep.t_max = R, R - 1, protocol, t_max
    rows, ws = moe.moe_ep_sizes(moe.make_shape(s), ep)
    assert rows == EP.window_rows(protocol, R, E, k, t_max)
    assert ws % 256 == 0


def test_ep_arguments_checked_on_the_host():
    s = W.spec("decode", T=64, E=16)
    sh = moe.make_shape(s)
    n, b = __import__("ctypes").c_int64(0), __import__("ctypes").c_size_t(0)
    L = moe.lib()
    import ctypes
    for bad in (dict(ranks=3), dict(ranks=0), dict(rank=2), dict(rank=-1), dict(protocol=2), dict(reserved=1),
                dict(t_max=32)):
        ep = moe.moe_ep()
        ep.ranks, ep.rank, ep.protocol, ep.t_max = 2, 0, 0, 64
        for f, v in bad.items():
            setattr(ep, f, v)
        assert L.moe_ep_sizes(ctypes.byref(sh), ctypes.byref(ep), ctypes.byref(n), ctypes.byref(b)) == 1, bad
    ep = moe.moe_ep()
    ep.ranks, ep.rank, ep.protocol, ep.t_max = 2, 0, 0, 64
    shared = moe.make_shape(s.with_(shared=1))
    assert L.moe_ep_sizes(ctypes.byref(shared), ctypes.byref(ep), ctypes.byref(n), ctypes.byref(b)) == 2
    assert L.moe_ep_dispatch(ctypes.byref(sh), ctypes.byref(ep), None, None, None, None, None) == 1


# ------------------------------------------------ gloo processes --

def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, protocol, T_per, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        def exchange(objs):
            gathered = [None] * world
            dist.all_gather_object(gathered, objs)
            return [gathered[s][rank] for s in range(world)]
        p, x, logits = _problem(world, T_per)
        o, rec, idx = _rank_layer(rank, world, protocol, p, x, logits, T_per, exchange)
        got = [None] * world
        dist.all_gather_object(got, o)
        if rank == 0:
            ref = oracle.moe_layer(p, x, logits)["out"]
            out["equal"] = bool(np.array_equal(np.concatenate(got), ref))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("protocol", [moe.MOE_EP_SENTINEL, moe.MOE_EP_FENCE])
def test_protocol_over_gloo_ranks_matches_oracle(world, protocol):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_gloo_rank, args=(world, _free_port(), protocol, 24, out), nprocs=world,
                           join=True, start_method="spawn")
        assert out.get("equal") is True
