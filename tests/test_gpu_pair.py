"""The grouped FFN on CTA pairs (layers with e4m3 weights and at least 128 rows
per expert): every MMA has M = 256 over the two CTAs of a cluster, a job
takes two 128-row tiles of one expert, and an expert's last tile joins the
job before it when it holds at most 64 rows.

Routing is set token by token (k = 1, one large logit) so that the experts'
row counts hit every chunk shape: one partial tile, one full tile, two
tiles, two tiles and a joined third (257..320 rows), three tiles that do not
join (321..384), four, and five with a joined fifth. h and y of every placed
row (or a sample) must match the oracle fed the same quantised rows, and the
layer output must match the oracle's layer.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W
from tests import gpu_harness as G
from tests.helpers import as_f64, max_abs_rel, raw

pytestmark = pytest.mark.gpu

COUNTS = {
    "one_two_tiles": [1, 100, 128, 129, 200, 256, 60, 150],
    "joined_tails": [257, 288, 300, 320, 256, 129, 200, 150],
    "several_chunks": [321, 384, 385, 448, 449, 576, 600, 130],
}


def _inputs(counts, H=512, I=256, seed=0, compact=0):
    E = len(counts)
    T = int(sum(counts))
    s = W.spec("decode", T=T, H=H, E=E, k=1, I=I, compact=compact)
    inp = W.make_inputs(s, seed=seed, device="cuda")
    assign = np.repeat(np.arange(E), counts)
    np.random.default_rng(seed).shuffle(assign)
    logits = torch.zeros((T, E), dtype=torch.float32)
    logits[torch.arange(T), torch.from_numpy(assign)] = 10.0
    inp["logits"] = logits.cuda()
    return s, inp


@pytest.mark.parametrize("compact", [0, 1])
@pytest.mark.parametrize("name", list(COUNTS))
def test_pair_ffn_rows_and_layer(name, compact, cuda_device):
    counts = COUNTS[name]
    s, inp = _inputs(counts, compact=compact)
    assert s.T * s.k // s.E >= 128          # the pair kernel's regime
    b = G.run_stages(s, inp)
    assert G.poll(b) == 0
    assert np.array_equal(b.counts.cpu().numpy(), np.array(counts))
    rows, pairs, experts = G.placed_rows(b)
    p = G.oracle_problem(s, inp, experts)
    h, hs, y = oracle.expert_rows(p, experts, G.gather(b.xq, rows), G.gather(b.xs, rows))
    gy, ry = as_f64(G.gather(b.y, rows), "bf16"), as_f64(y, "bf16")
    assert max_abs_rel(gy, ry) < 2e-2, max_abs_rel(gy, ry)
    gh = oracle.e4m3_decode(G.gather(b.hq, rows)) * np.repeat(G.gather(b.hs, rows).astype(np.float64), 128, axis=1)
    rh = oracle.e4m3_decode(h) * np.repeat(hs.astype(np.float64), 128, axis=1)
    assert max_abs_rel(gh, rh) < 2e-2, max_abs_rel(gh, rh)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), 0, 256)
    err = max_abs_rel(as_f64(raw(b.out)[:256], "bf16"), as_f64(r["out"], "bf16"))
    assert err < 2e-2, err


def test_pair_ffn_repeated_and_bitwise_stable(cuda_device):
    """Two layers give the same output bits (rows land in a different order
    inside each window, the arithmetic of a row does not depend on it), and
    a second FFN call on the last dispatch gives the same y bits."""
    s, inp = _inputs(COUNTS["joined_tails"], seed=3)
    b = moe.alloc_buffers(s)
    outs = []
    for _ in range(2):
        moe.run_layer(b, inp)
        torch.cuda.synchronize()
        assert G.poll(b) == 0
        outs.append(b.out.clone())
    assert torch.equal(outs[0], outs[1])
    rows, _, _ = G.placed_rows(b)
    idx = torch.from_numpy(rows).cuda()
    y1 = b.y[idx].clone()
    moe.moe_grouped_ffn(b.shape, b.dispatch_bufs(), moe.weights_struct(inp), b.ws, b.y)
    torch.cuda.synchronize()
    assert G.poll(b) == 0
    assert torch.equal(y1, b.y[idx])
