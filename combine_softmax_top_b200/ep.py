"""Expert parallelism over R ranks: the moe_ep_* calls put together.

Rank d owns experts [d E/R, (d + 1) E/R) and dispatches its own tokens. Every
rank receives into V = E virtual experts v = el * R + src (one region per
local expert el and source rank src), reached through rank-major address
ranges (rank d's part at d * rows rows, d * ws_bytes bytes); the layout and
the two protocols are described in include/moe.h ("expert parallelism").

EmulatedRanks runs R ranks on one device: each rank-major range is one
allocation, and every protocol step is enqueued for all ranks before the next
step of any rank, so that stream order satisfies every cross-rank wait before
it begins (the ranks' kernels never wait on one another while running).

window_rows and the host protocol model below restate the window geometry and
the order of protocol steps in plain Python; the multi-process tests run the
model over torch.distributed ranks to check the partitioning and the
bookkeeping (regions, tiles and their flags, counts, closes, the Fence
layout) end to end, and check its geometry against moe_ep_sizes.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np
import torch

from . import moe
from .workloads import E4M3, Spec

TILE = 128


# ------------------------------------------------------------ geometry --

def owner(e: int, E: int, R: int) -> int:
    return e // (E // R)


def virtual_expert(e: int, src: int, E: int, R: int) -> int:
    """Window of global expert e's rows from source rank src at its owner."""
    return (e % (E // R)) * R + src


def window_rows(protocol: int, R: int, E: int, k: int, t_max: int) -> int:
    """Rows of one rank's windows: Sentinel, E regions of round_up(t_max, 128)
    rows; Fence, whole tiles for the most pairs R sources can send one rank
    (R t_max min(k, E/R)) plus one partial tile per window."""
    if protocol == moe.MOE_EP_SENTINEL:
        return E * (-(-max(t_max, 1) // TILE) * TILE)
    pairs = R * t_max * min(k, E // R)
    return (-(-pairs // TILE) + E) * TILE


# ------------------------------------------------ one device, R ranks --

@dataclass
class _Rank:
    ep: moe.moe_ep
    idx: torch.Tensor
    w: torch.Tensor
    pos: torch.Tensor
    out: torch.Tensor


class EmulatedRanks:
    """R ranks of one expert-parallel layer on one device. `spec` is the
    global layer with T = tokens per rank."""

    def __init__(self, spec: Spec, R: int, protocol: int, device="cuda"):
        self.spec, self.R, self.protocol = spec, R, protocol
        self.shape = moe.make_shape(spec)
        self.ranks = []
        for r in range(R):
            ep = moe.moe_ep()
            ep.ranks, ep.rank, ep.protocol, ep.reserved, ep.t_max = R, r, protocol, 0, spec.T
            z = dict(device=device)
            self.ranks.append(_Rank(ep, torch.empty((spec.T, spec.k), dtype=torch.int32, **z),
                                    torch.empty((spec.T, spec.k), dtype=torch.float32, **z),
                                    torch.empty(spec.T * spec.k, dtype=torch.int32, **z),
                                    torch.empty((spec.T, spec.H), dtype=moe._TORCH[spec.out], **z)))
        self.rows, self.ws_bytes = moe.moe_ep_sizes(self.shape, self.ranks[0].ep)
        n = R * self.rows
        z = dict(device=device)
        self.xq = torch.empty((n, spec.H), dtype=moe._TORCH[spec.xq], **z)
        self.xs = torch.empty((n, spec.H // 128), dtype=torch.float32, **z) if spec.xq == E4M3 else None
        self.row_src = torch.full((n,), -1, dtype=torch.int32, **z)
        ffn = not spec.identity
        self.hq = torch.empty((n, spec.I), dtype=moe._TORCH[spec.h], **z) if ffn else None
        self.hs = torch.empty((n, spec.I // 128), dtype=torch.float32, **z) if ffn and spec.h == E4M3 else None
        self.y = torch.empty((n, spec.H), dtype=moe._TORCH[spec.y], **z) if ffn else None
        self.ws = torch.empty(R * self.ws_bytes, dtype=torch.uint8, **z)
        self.win = moe.moe_ep_windows()
        for f in ("xq", "xs", "row_src", "hq", "hs", "y", "ws"):
            t = getattr(self, f)
            setattr(self.win, f, t.data_ptr() if t is not None else 0)
        for rk in self.ranks:
            moe.moe_ep_workspace_init(self.shape, rk.ep, self.win)

    def ws_of(self, r: int) -> torch.Tensor:
        return self.ws[r * self.ws_bytes:(r + 1) * self.ws_bytes]

    def local_weights(self, inp: dict, r: int) -> moe.moe_weights:
        el = self.spec.E // self.R
        part = {k: (v[r * el:(r + 1) * el] if v is not None else None) for k, v in inp.items()
                if k in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")}
        return moe.weights_struct(part)

    def run(self, xs: list, logits: list, inp: dict | None = None) -> list:
        """One layer on every rank: xs[r] [T, H] and logits[r] [T, E] are rank
        r's tokens; `inp` holds the global weights. Returns each rank's out."""
        sh, win = self.shape, self.win
        for r, rk in enumerate(self.ranks):
            moe.moe_route(sh, logits[r], rk.idx, rk.w, self.ws_of(r))
        if self.protocol == moe.MOE_EP_FENCE:
            for rk in self.ranks:
                moe.moe_ep_count(sh, rk.ep, rk.idx, win)
            for rk in self.ranks:
                moe.moe_ep_layout(sh, rk.ep, win)
        for r, rk in enumerate(self.ranks):
            moe.moe_ep_dispatch(sh, rk.ep, xs[r], rk.idx, win, rk.pos)
        if not self.spec.identity:
            for r, rk in enumerate(self.ranks):
                moe.moe_ep_grouped_ffn(sh, rk.ep, self.local_weights(inp, r), win)
        for rk in self.ranks:
            moe.moe_ep_combine(sh, rk.ep, rk.pos, rk.w, win, rk.out)
        return [rk.out for rk in self.ranks]

    def poll(self) -> list:
        return [moe.moe_poll_status(self.ws_of(r)) for r in range(self.R)]


# ------------------------------------------- host model of the protocol --

def model_layer(rank: int, R: int, protocol: int, E: int, t_max: int, idx: np.ndarray, rows_in: np.ndarray,
                expert_fn, epoch: int = 1, exchange=None) -> tuple[np.ndarray, dict]:
    """The protocol's bookkeeping for one source/owner rank, in plain Python,
    with `exchange(list_of_R_objects) -> list_of_R_objects` delivering object
    i to rank i (an all-to-all). rows_in [T, H] are this rank's token rows,
    idx [T, k] their global experts. expert_fn(global_expert, rows) returns
    the expert's output rows. Returns, for every (t, j), the expert output
    row that combine reads in place, and the owner-side records (windows,
    sentinels, counts) for the checks. Steps, in the order of include/moe.h:
    [Fence: counts to owners, layout, bases back], claims and pushes, tile
    flags, close (partial tiles, counts), grouped FFN per window once all R
    sources closed, then the pull of every pair's output row."""
    T, k = idx.shape
    el = E // R
    rows = window_rows(protocol, R, E, k, t_max)
    cap = -(-max(t_max, 1) // TILE) * TILE
    # Fence: pair counts to the owners, each owner lays its windows out, bases back
    base = None
    if protocol == moe.MOE_EP_FENCE:
        cnt = np.bincount(idx.ravel(), minlength=E)
        got = exchange([cnt[d * el:(d + 1) * el].copy() for d in range(R)])   # got[src][el]
        pre = np.zeros(E, np.int64)
        for src in range(R):
            for e_l in range(el):
                pre[e_l * R + src] = got[src][e_l]
        tiles = -(-pre // TILE)
        mine = np.concatenate([[0], np.cumsum(tiles)])                          # base[v], base[V]
        assert mine[-1] * TILE <= rows, "Fence windows exceed their bound"
        back = exchange([mine.copy() for _ in range(R)])                        # every owner's layout
        base = back

    def region(d, v):
        if protocol == moe.MOE_EP_FENCE:
            return base[d][v] * TILE, (base[d][v + 1] - base[d][v]) * TILE
        return v * cap, cap

    # claims in this source's regions, pushes, and tile fill counts
    claims = np.zeros(E, np.int64)
    pos = np.full((T, k), -1, np.int64)
    msgs = [[] for _ in range(R)]            # (row, src pair id, data) per owner
    fill = [dict() for _ in range(R)]
    flags = [[] for _ in range(R)]           # (tile, (epoch << 8) | rows) per owner
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            d, v = owner(e, E, R), virtual_expert(e, rank, E, R)
            first, room = region(d, v)
            p = claims[e]
            claims[e] += 1
            assert p < room, "a region overflowed"
            row = first + p
            pos[t, j] = d * rows + row
            msgs[d].append((row, rank * t_max * k + t * k + j, rows_in[t]))
            g = row // TILE
            fill[d][g] = fill[d].get(g, 0) + 1
            if fill[d][g] == TILE:
                flags[d].append((g, (epoch << 8) | TILE))
    # close: partial tiles and the region counts
    counts = [dict() for _ in range(R)]
    for e in range(E):
        d, v = owner(e, E, R), virtual_expert(e, rank, E, R)
        first, _ = region(d, v)
        c = int(claims[e])
        counts[d][v] = c
        if c % TILE:
            flags[d].append((first // TILE + c // TILE, (epoch << 8) | (c % TILE)))
    inbox = exchange([(msgs[d], flags[d], counts[d]) for d in range(R)])
    # the owner: windows, sentinels and counts from all R sources
    assert len(inbox) == R, "an owner must hear from every source before its FFN"
    window = {}
    row_src = {}
    sentinel = {}
    vcount = np.zeros(E, np.int64)
    for src, (m, fl, cn) in enumerate(inbox):
        for row, pid, data in m:
            assert row not in window, "two pairs placed in one row"
            window[row], row_src[row] = data, pid
        for g, word in fl:
            assert g not in sentinel, "a tile published twice"
            sentinel[g] = word
        for v, c in cn.items():
            vcount[v] = c
    out_rows = {}
    for v in range(E):
        c = int(vcount[v])
        if c == 0:
            continue
        first, _ = (base[rank][v] * TILE, None) if base is not None else (v * cap, None)
        for g in range(first // TILE, first // TILE + -(-c // TILE)):   # every tile the FFN takes
            want = TILE if (g - first // TILE + 1) * TILE <= c else c % TILE
            assert sentinel.get(g) == (epoch << 8) | want, "a tile taken before its sentinel"
        e = rank * el + v // R                                              # the weights of v
        block = np.stack([window[first + i] for i in range(c)])
        ys = expert_fn(e, block)
        for i in range(c):
            out_rows[first + i] = ys[i]
    # combine: every pair's output row, read where it lies (an all-to-all of requests)
    want = [[] for _ in range(R)]
    for t in range(T):
        for j in range(k):
            want[int(pos[t, j] // rows)].append(int(pos[t, j] % rows))
    asked = exchange(want)
    replies = exchange([[out_rows[r] for r in asked[src]] for src in range(R)])
    got = [iter(replies[d]) for d in range(R)]
    y = np.empty((T, k) + np.shape(rows_in[0]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            y[t, j] = next(got[int(pos[t, j] // rows)])
    return y, {"pos": pos, "rows": rows, "window_rows": sorted(window), "row_src": row_src, "counts": vcount}
