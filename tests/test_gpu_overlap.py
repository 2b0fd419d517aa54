"""Dispatch beside the grouped FFN (moe_layer_overlap) through the C ABI.

The device is split in two: dispatch runs on a few SMs while the persistent
grouped FFN holds the rest, takes its unit table from the counting pass and
starts each tile once dispatch publishes its sentinel (GC-MoE explainer,
"GC-MoE's Core Idea" and "Three-Node CUDA Graph and token-ring Handshake").
A row's arithmetic does not depend on when its tile was taken, so the layer
output must equal moe_layer's bit for bit, and match the oracle at the usual
bars. A dispatch held back past the FFN's wait budget must end in
MOE_ERR_TIMEOUT with the context still usable.
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

TOL = {"bf16": 2e-2, "e4m3": 2e-2, "e2m1": 2e-2}

CASES = [
    # few rows per expert: 16- and 64-row tiles, every tile published when dispatch closes
    ("decode_small", "decode", dict(T=128, H=512, E=16, k=4, I=256)),
    ("decode_tiny_tiles", "decode", dict(T=16, H=512, E=32, k=4, I=256)),
    # 1024 rows per expert: full 128-row tiles published while dispatch still runs
    ("many_rows", "decode", dict(T=1024, H=512, E=8, k=2, I=256)),
    ("many_rows_compact", "decode", dict(T=1024, H=512, E=8, k=2, I=256, compact=1)),
    ("shared_compact", "decode", dict(T=300, H=512, E=4, k=2, I=384, shared=1, compact=1)),
    ("fp4_weights", "decode_fp4", dict(T=64, H=512, E=16, k=4, I=256)),
    ("skew_bf16", "skew", dict(T=512, H=1024, E=32, I=512)),
]


def _serial(s, inp):
    lw = moe.alloc_layer(s)
    moe.run_layer_ws(lw, inp)
    torch.cuda.synchronize()
    assert moe.moe_poll_status(lw.ws) == 0
    return lw.out.clone()


def _overlapped(s, inp, ov, calls=1):
    lw = moe.alloc_layer(s)
    outs = []
    for _ in range(calls):
        moe.run_layer_overlap(lw, inp, ov)
        torch.cuda.synchronize()
        assert moe.moe_poll_status(lw.ws) == 0
        outs.append(lw.out.clone())
    return outs


@pytest.mark.parametrize("dsms", [4, 20])
@pytest.mark.parametrize("name,base,over", CASES, ids=[c[0] for c in CASES])
def test_overlap_matches_serial_layer_and_oracle(name, base, over, dsms, cuda_device):
    s = W.spec(base, **over)
    inp = W.make_inputs(s, seed=2, device="cuda")
    ref = _serial(s, inp)
    ov = moe.Overlap(dsms)
    outs = _overlapped(s, inp, ov, calls=2)        # two calls: alternate counter sets
    for o in outs:
        assert torch.equal(o, ref)
    n = min(s.T, 128)
    idx, _ = oracle.route(raw(inp["logits"]), s.k, s.renorm)
    p = G.oracle_problem(s, inp, idx[:n].ravel())
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), 0, n)
    err = max_abs_rel(as_f64(raw(outs[0])[:n], s.out), as_f64(r["out"], s.out))
    assert err < TOL[s.weight], err


@pytest.mark.parametrize("green", [False, True], ids=["stream", "green"])
@pytest.mark.parametrize("name,over", [
    ("decode", {}),                       # the full decode layer (e4m3, 11 GB of weights)
    ("prefill", dict(compact=1)),         # the full prefill layer on compact windows
])
def test_overlap_full_size_bitwise(name, over, green, cuda_device):
    """Full layers, the split left to the FFN's grid size or enforced by two
    green contexts (a persistent FFN beside a dispatch-only green context
    could take dispatch's SMs; both sides confined, it cannot)."""
    if green:
        pytest.importorskip("cuda.bindings.driver")
    torch.cuda.empty_cache()
    s = W.spec(name, **over)
    inp = W.make_inputs(s, seed=0, device="cuda")
    ref = _serial(s, inp)
    ov = moe.Overlap(20, green=green)
    (out,) = _overlapped(s, inp, ov)
    ov.close()
    assert torch.equal(out, ref)
    # a token sample against the oracle
    idx, _ = oracle.route(raw(inp["logits"]), s.k, s.renorm)
    t = np.random.default_rng(5).choice(s.T, 24, replace=False)
    p = G.oracle_problem(s, inp, idx[t].ravel())
    for tok in t[:8]:
        r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), int(tok), int(tok) + 1)
        err = max_abs_rel(as_f64(raw(out)[tok:tok + 1], s.out), as_f64(r["out"], s.out))
        assert err < TOL[s.weight], (tok, err)
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dsms,ffn", [(1, 0), (8, 0), (32, 0), (74, 0), (147, 0), (16, 64)])
def test_overlap_partition_sizes(dsms, ffn, cuda_device):
    """Any split gives the same bits, down to one SM for dispatch and one
    persistent CTA for the FFN's share."""
    if dsms >= torch.cuda.get_device_properties(0).multi_processor_count:
        pytest.skip("fewer SMs")
    s = W.spec("decode", T=512, H=512, E=8, k=2, I=256)
    inp = W.make_inputs(s, seed=3, device="cuda")
    ref = _serial(s, inp)
    (out,) = _overlapped(s, inp, moe.Overlap(dsms, ffn))
    assert torch.equal(out, ref)


def test_overlap_on_green_contexts(cuda_device):
    """The partition enforced by the device: dispatch on a green context of
    20 SMs (rounded up to the driver's split granularity), the rest of the
    layer on a green context of all the other SMs."""
    pytest.importorskip("cuda.bindings.driver")
    s = W.spec("decode", T=1024, H=512, E=8, k=2, I=256)
    inp = W.make_inputs(s, seed=4, device="cuda")
    ref = _serial(s, inp)
    ov = moe.Overlap(20, green=True)
    n = torch.cuda.get_device_properties(0).multi_processor_count
    assert 20 <= ov.ov.dispatch_sms and ov.ov.dispatch_sms + ov.ov.ffn_sms <= n
    outs = _overlapped(s, inp, ov, calls=2)
    ov.close()
    for o in outs:
        assert torch.equal(o, ref)


def test_overlap_dispatch_held_back_times_out_cleanly(cuda_device):
    """The dispatch stream is kept busy (a bounded spin of ~0.4 s) past the
    grouped FFN's 200 ms wait budget: the FFN gives up and latches
    MOE_ERR_TIMEOUT, dispatch and combine still run, and the next layer on the
    same workspace and streams is exact again."""
    s = W.spec("decode", T=256, H=512, E=8, k=2, I=256)
    inp = W.make_inputs(s, seed=6, device="cuda")
    ref = _serial(s, inp)
    ov = moe.Overlap(8)
    lw = moe.alloc_layer(s)
    with torch.cuda.stream(ov.stream):
        torch.cuda._sleep(int(8e8))                 # 8e8 SM cycles: 0.4 s at 2 GHz, longer below
    moe.run_layer_overlap(lw, inp, ov)
    torch.cuda.synchronize()
    assert moe.moe_poll_status(lw.ws) == 5          # MOE_ERR_TIMEOUT
    moe.run_layer_overlap(lw, inp, ov)
    torch.cuda.synchronize()
    assert moe.moe_poll_status(lw.ws) == 0
    assert torch.equal(lw.out, ref)
