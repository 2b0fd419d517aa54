"""The whole layer through the C ABI on shapes off the five workloads: ragged
tails, a single token, no tokens, k = 1, a hidden size whose K loop crosses 64
scale blocks, routing skewed so one expert's window spans several tiles
(split into chunks by the tensor-core FFN), and layers with more than 32 rows
per expert, whose tensor-core FFN uses 128-row tiles (down jobs over pairs of
H slices when H/128 is even, single slices when it is odd), and layers with at
most 4 rows per expert, whose FFN uses 16-row tiles (an expert with more rows
is split into 16-row chunks)."""
import numpy as np
import pytest
import torch

import oracle
from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W
from tests import gpu_harness as G
from tests.helpers import as_f64, max_abs_rel, raw

pytestmark = pytest.mark.gpu

CASES = [
    # name, base workload, overrides, extra logit bias on expert 0
    ("ragged_fp8", "decode", dict(T=37, H=384, E=5, k=3, I=640), 0.0),
    ("ragged_bf16", "skew", dict(T=53, H=256, E=6, k=2, I=384, zipf_s=0.0), 0.0),
    ("one_token_fp8", "decode", dict(T=1, H=512, E=16, k=4, I=256), 0.0),
    ("k1_fp8", "decode", dict(T=64, H=256, E=8, k=1, I=256, renorm=1), 0.0),
    ("long_k_fp8", "decode", dict(T=16, H=8320, E=4, k=2, I=256), 0.0),
    ("hot_expert_fp8", "decode", dict(T=256, H=512, E=64, k=2, I=256), 30.0),
    ("hot_expert_bf16", "skew", dict(T=256, H=256, E=64, k=2, I=256, zipf_s=0.0), 30.0),
    # > 32 rows per expert: 128-row token tiles; ragged last tiles
    ("big_tiles_pairs_fp8", "decode", dict(T=300, H=512, E=4, k=2, I=384), 0.0),     # H/128 even: down pairs
    ("big_tiles_odd_h_fp8", "decode", dict(T=300, H=384, E=4, k=2, I=256), 0.0),     # H/128 odd: single slices
    ("big_tiles_pairs_bf16", "skew", dict(T=260, H=256, E=4, k=2, I=256, zipf_s=0.0), 0.0),
    # <= 4 rows per expert: 16-row token tiles, six pipeline stages, down pairs
    ("r16_fp8", "decode", dict(T=64, H=512, E=64, k=4, I=256), 0.0),
    ("r16_hot_expert_fp8", "decode", dict(T=64, H=512, E=64, k=4, I=256), 30.0),   # 64 rows: 4 chunks
    ("r16_odd_h_fp8", "decode", dict(T=64, H=384, E=64, k=4, I=256), 0.0),         # no pairs: one slab
    ("r16_hot_expert_fp4", "decode_fp4", dict(T=64, H=512, E=64, k=4, I=256), 30.0),
    ("r16_odd_h_fp4", "decode_fp4", dict(T=64, H=384, E=64, k=4, I=256), 0.0),      # one 4-bit slab per stage
    ("r16_bf16", "skew", dict(T=64, H=256, E=64, k=4, I=256, zipf_s=0.0), 0.0),
    # MX FP4 weights and compact windows off the standard shapes
    ("one_token_fp4", "decode_fp4", dict(T=1, H=512, E=16, k=4, I=256), 0.0),
    ("ragged_fp4", "decode_fp4", dict(T=37, H=384, E=5, k=3, I=640), 0.0),
    ("one_token_compact", "decode", dict(T=1, H=512, E=16, k=4, I=256, compact=1), 0.0),
    ("hot_expert_compact_fp4", "decode_fp4", dict(T=256, H=512, E=64, k=2, I=256, compact=1), 30.0),
    ("many_experts_compact_fp4", "decode_fp4", dict(T=64, H=256, E=1024, k=8, I=256, compact=1), 0.0),
    ("many_experts_fp8", "decode", dict(T=64, H=256, E=1000, k=32, I=256), 0.0),
    ("tiny_no_renorm", "tiny", dict(renorm=0), 0.0),
    ("fp32_ragged", "tiny", dict(T=45, H=384, E=7, k=3, I=256), 0.0),
]


@pytest.mark.parametrize("name,base,over,bias", CASES, ids=[c[0] for c in CASES])
def test_layer_shapes(name, base, over, bias, cuda_device):
    s = W.spec(base, **over)
    inp = W.make_inputs(s, seed=7, device="cuda")
    if bias:
        inp["logits"][:, 0] += bias
    b = G.run_stages(s, inp, layer=True)
    assert G.poll(b) == 0
    counts = b.counts.cpu().numpy()
    idx = b.topk_idx.cpu().numpy()
    assert np.array_equal(counts, oracle.counts(idx, s.E))
    p = G.oracle_problem(s, inp)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    assert np.array_equal(r["idx"], idx)
    tol = 1e-5 if s.weight == "f32" else 2e-2
    err = max_abs_rel(as_f64(raw(b.out), s.out), as_f64(r["out"], s.out))
    assert err < tol, err
    if bias:
        assert counts[0] == s.T            # one window spans several 128-row tiles


def test_zero_tokens(cuda_device):
    s = W.spec("decode", T=0, H=256, E=8, k=2, I=256)
    inp = W.make_inputs(s, device="cuda")
    b = moe.alloc_buffers(s)
    moe.run_layer(b, inp)
    torch.cuda.synchronize()
    assert moe.moe_poll_status(b.ws) == 0
    assert b.counts.cpu().numpy().sum() == 0


@pytest.mark.parametrize("over", [dict(), dict(compact=1), dict(weight=W.E2M1)],
                         ids=["windows", "compact", "fp4"])
def test_many_tokens(over, cuda_device):
    """65 536 tokens over 8 experts (16 384 rows each, 128 tiles per window):
    counts bit-exact, every pair placed once, and a sample of 256 tokens
    against the oracle."""
    s = W.spec("decode", T=65536, H=256, E=8, k=2, I=256, **over)
    inp = W.make_inputs(s, seed=12, device="cuda")
    b = G.run_stages(s, inp, layer=True)
    assert G.poll(b) == 0
    idx = b.topk_idx.cpu().numpy()
    counts = b.counts.cpu().numpy()
    assert np.array_equal(counts, oracle.counts(idx, s.E))
    rows, pairs, experts = G.placed_rows(b)
    assert np.array_equal(np.sort(pairs), np.arange(s.T * s.k))
    t0, t1 = 30000, 30256
    p = G.oracle_problem(s, inp)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), t0, t1)
    assert np.array_equal(r["idx"], idx)
    err = max_abs_rel(as_f64(raw(b.out)[t0:t1], s.out), as_f64(r["out"], s.out))
    assert err < 2e-2, err
