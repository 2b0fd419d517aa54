"""The layer with a shared expert (moe_shape.flags = MOE_FLAG_SHARED_EXPERT)
through the C ABI, against the oracle: every token's last slot is the shared
expert (index E, weight 1), its window takes all T tokens, and the output is
the routed mixture plus the shared expert's FFN (GC-MoE feed item: the compute
partition fuses optional shared experts)."""
import numpy as np
import pytest

import oracle
from combine_softmax_top_b200 import workloads as W
from tests import gpu_harness as G
from tests.helpers import as_f64, max_abs_rel, raw

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny_f32", "tiny", dict(shared=1)),
    ("decode_fp8_small", "decode", dict(T=32, H=512, E=16, k=4, I=256, shared=1)),        # 64-row tiles
    ("decode_fp8_big_tiles", "decode", dict(T=300, H=512, E=4, k=2, I=384, shared=1)),   # 128-row tiles
    ("bf16", "skew", dict(T=64, H=256, E=8, k=2, I=256, zipf_s=0.0, shared=1)),
]


@pytest.mark.parametrize("name,base,over", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("layer", [False, True], ids=["stages", "moe_layer"])
def test_shared_expert_layer(name, base, over, layer, cuda_device):
    s = W.spec(base, **over)
    inp = W.make_inputs(s, seed=11, device="cuda")
    b = G.run_stages(s, inp, layer=layer)
    assert G.poll(b) == 0
    idx = b.topk_idx.cpu().numpy()
    w = b.topk_w.cpu().numpy()
    assert idx.shape == (s.T, s.k + 1)
    assert np.all(idx[:, s.k] == s.E) and np.all(w[:, s.k] == 1.0)
    counts = b.counts.cpu().numpy()
    assert counts[s.E] == s.T                                     # every token, once
    assert np.array_equal(counts[: s.E], oracle.counts(idx[:, : s.k], s.E))
    p = G.oracle_problem(s, inp)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    assert np.array_equal(r["idx"], idx[:, : s.k])
    tol = 1e-5 if s.weight == "f32" else 2e-2
    err = max_abs_rel(as_f64(raw(b.out), s.out), as_f64(r["out"], s.out))
    assert err < tol, err
