"""Running the GPU path stage by stage and preparing matching oracle inputs.
Test infrastructure; no layer arithmetic here."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W
from tests.helpers import raw

ODT = {W.F32: oracle.F32, W.BF16: oracle.BF16, W.E4M3: oracle.E4M3, W.E2M1: oracle.E2M1}


def run_stages(s: W.Spec, inp: dict, layer: bool = False) -> moe.Buffers:
    """Route, dispatch, grouped FFN and combine on the GPU (each stage through
    its own C-ABI entry point, or all through moe_layer)."""
    b = moe.alloc_buffers(s)
    if layer:
        moe.run_layer(b, inp)
    else:
        moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
        bufs = b.dispatch_bufs()
        moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, bufs)
        if not s.identity:
            moe.moe_grouped_ffn(b.shape, bufs, moe.weights_struct(inp), b.ws, b.y)
        moe.moe_combine(b.shape, bufs, b.y, b.topk_w, b.ws, b.out)
    torch.cuda.synchronize()
    return b


def poll(b: moe.Buffers) -> int:
    return moe.moe_poll_status(b.ws)


def oracle_problem(s: W.Spec, inp: dict, experts=None) -> oracle.Problem:
    """Oracle problem for `s`; weights of only `experts` (all if None) are
    copied to the host."""
    kw = dict(x_dtype=ODT[s.act], xq_dtype=ODT[s.xq], w_dtype=ODT[s.weight], h_dtype=ODT[s.h],
              y_dtype=ODT[s.y], out_dtype=ODT[s.out], renorm=s.renorm, identity=s.identity,
              shared=s.shared)
    if not s.identity:
        es = range(s.ne) if experts is None else sorted(set(int(e) for e in experts) | ({s.E} if s.shared else set()))
        for name in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
            # 4-bit weights: the oracle reads the per-row scales, the library the atoms
            t = inp.get(name + "_rows" if (s.weight == W.E2M1 and name[0] == "s") else name)
            if t is not None:
                kw[name] = {e: raw(t[e]) for e in es}
    return oracle.Problem(s.T, s.H, s.E, s.k, s.I, **kw)


def window_offsets(s: W.Spec, counts: np.ndarray) -> np.ndarray:
    """First row of each expert window: e * cap, or with compact windows the
    running sum of the windows before it, each rounded up to 128 rows (the
    layout moe.h states for MOE_FLAG_COMPACT)."""
    if not s.compact:
        return np.arange(len(counts), dtype=np.int64) * s.cap
    tiles = -(-counts.astype(np.int64) // 128)
    return 128 * np.concatenate([[0], np.cumsum(tiles)[:-1]])


def placed_rows(b: moe.Buffers):
    """(row ids, pair ids, expert ids) of every filled row, from counts,
    offsets and row_src."""
    counts = b.counts.cpu().numpy()
    offsets = b.offsets.cpu().numpy().astype(np.int64)
    rows = np.concatenate([o + np.arange(c) for o, c in zip(offsets, counts)]) if counts.sum() \
        else np.zeros(0, np.int64)
    experts = np.repeat(np.arange(b.spec.ne), counts)
    pairs = b.row_src.cpu().numpy()[rows]
    return rows.astype(np.int64), pairs.astype(np.int64), experts.astype(np.int32)


def gather(t: torch.Tensor | None, rows: np.ndarray):
    if t is None:
        return None
    return raw(t[torch.from_numpy(rows).to(t.device)])
