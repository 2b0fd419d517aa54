"""Compact expert windows (moe_shape.flags |= MOE_FLAG_COMPACT) through the C
ABI, against the oracle.

A counting pass settles every expert's pair count before any row moves (the
NVLinkOneSided abstract's Fence protocol); the windows are then packed back
to back, each rounded up to whole 128-row tiles, so the expert buffers hold
T * k + 127 * E rows instead of E * round_up(T, 128). Routing, counts and
the rows' bytes must be those of the window layout; offsets follow the packed
layout; the FFN and the layer output must match the oracle, and since a row's
arithmetic does not depend on where its window sits, the layer output must
equal the window layout's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W
from tests import gpu_harness as G
from tests.helpers import as_f64, bf16_bits_to_f32, max_abs_rel, raw

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2, "e4m3": 2e-2}

CASES = [
    ("tiny_f32", "tiny", {}),                                            # SIMT FFN (ring of tiles)
    ("decode", "decode", {}),                                            # e4m3, 64-row tiles
    ("prefill", "prefill", {}),                                          # e4m3, 128-row tiles, full size
    ("skew_bf16", "skew", dict(T=1024)),                                 # Zipf counts, bf16
    ("big_tiles_shared", "decode", dict(T=300, H=512, E=4, k=2, I=384, shared=1)),
    ("sweep_identity", "sweep", dict(T=512)),
]
SAMPLE = 96   # rows / tokens the oracle recomputes for large cases


def _run(base, over, layer=False, seed=0):
    s = W.spec(base, compact=1, **over)
    inp = W.make_inputs(s, seed=seed, device="cuda")
    b = G.run_stages(s, inp, layer=layer)
    return s, inp, b


@pytest.mark.parametrize("name,base,over", CASES, ids=[c[0] for c in CASES])
def test_compact_dispatch_layout(name, base, over, cuda_device):
    s, inp, b = _run(base, over)
    assert G.poll(b) == 0
    assert b.xq.shape[0] == s.rows()
    idx = b.topk_idx.cpu().numpy()
    counts = b.counts.cpu().numpy()
    assert np.array_equal(counts[: s.E], oracle.counts(idx[:, : s.k], s.E))
    assert counts.sum() == s.T * s.ks
    offsets = b.offsets.cpu().numpy()
    assert np.array_equal(offsets, G.window_offsets(s, counts))
    assert offsets[-1] + counts[-1] <= s.rows()
    rows, pairs, experts = G.placed_rows(b)
    assert np.array_equal(np.sort(pairs), np.arange(s.T * s.ks))      # every pair once
    assert np.array_equal(idx.ravel()[pairs], experts)                 # in its expert's window
    assert np.array_equal(b.pos.cpu().numpy()[pairs], rows)
    sel = rows if len(rows) <= 4096 else rows[np.random.default_rng(0).choice(len(rows), 4096, replace=False)]
    src_tok = b.row_src.cpu().numpy()[sel] // s.ks
    xq = G.gather(b.xq, sel)
    x_src = raw(inp["x"])[src_tok]
    if s.xq == W.E4M3:
        x32 = bf16_bits_to_f32(x_src) if s.act == W.BF16 else x_src
        q, sc = oracle.quantize_rows(x32)
        same = (xq == q) | (((xq & 0x7F) == 0) & ((q & 0x7F) == 0))
        assert same.all()
        assert np.array_equal(G.gather(b.xs, sel), sc)
    else:
        assert np.array_equal(xq, x_src)


@pytest.mark.parametrize("name,base,over", [c for c in CASES if c[1] != "sweep"],
                         ids=[c[0] for c in CASES if c[1] != "sweep"])
def test_compact_grouped_ffn(name, base, over, cuda_device):
    s, inp, b = _run(base, over)
    assert G.poll(b) == 0
    rows, pairs, experts = G.placed_rows(b)
    if len(rows) > SAMPLE:
        pick = np.random.default_rng(1).choice(len(rows), SAMPLE, replace=False)
        rows, pairs, experts = rows[pick], pairs[pick], experts[pick]
    p = G.oracle_problem(s, inp, experts)
    h, hs, y = oracle.expert_rows(p, experts, G.gather(b.xq, rows), G.gather(b.xs, rows))
    vy = (lambda a, dt: as_f64(a, dt) if dt != "e4m3" else oracle.e4m3_decode(a))
    err = max_abs_rel(vy(G.gather(b.y, rows), s.y), vy(y, s.y))
    assert err < TOL[s.weight], err


@pytest.mark.parametrize("name,base,over", CASES, ids=[c[0] for c in CASES])
def test_compact_layer_matches_oracle_and_window_layout(name, base, over, cuda_device):
    s, inp, b = _run(base, over, layer=True)
    assert G.poll(b) == 0
    n = min(s.T, 128)
    idx = b.topk_idx.cpu().numpy()
    p = G.oracle_problem(s, inp, None if s.identity else idx[:n].ravel())
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), 0, n)
    assert np.array_equal(r["idx"], idx[:, : s.k])
    tol = TOL[s.weight] if not s.identity else 2e-2
    err = max_abs_rel(as_f64(raw(b.out)[:n], s.out), as_f64(r["out"], s.out))
    assert err < tol, err
    # the same layer with windows of cap rows gives the same bits
    sw = s.with_(compact=0)
    bw = G.run_stages(sw, inp, layer=True)
    assert G.poll(bw) == 0
    assert torch.equal(b.out, bw.out)


def test_compact_workspace_reuse_with_changing_routing(cuda_device):
    """Consecutive layers on one workspace alternate counter sets; each
    dispatch clears the set the next one counts into. Different routing in
    between must not leak counts or window bases from one call to the next."""
    s = W.spec("decode", T=256, H=1024, E=32, I=256, compact=1)
    ins = [W.make_inputs(s, seed=sd, device="cuda") for sd in (0, 1)]
    ins[1]["logits"][:, :4] += 50.0          # the second call piles onto experts 0-3
    b = moe.alloc_buffers(s)
    outs = []
    for i in (0, 1, 0, 1):
        moe.run_layer(b, ins[i])
        torch.cuda.synchronize()
        assert G.poll(b) == 0
        outs.append(b.out.clone())
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[1], outs[3])
    fresh = G.run_stages(s, ins[1], layer=True)
    assert torch.equal(fresh.out, outs[1])
    assert not torch.equal(outs[0], outs[1])
