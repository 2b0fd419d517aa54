"""moe_dispatch_noalloc: dispatch for callers that cannot hand the library a
workspace (for example an engine whose device memory all belongs to its own
pool, with cudaMalloc forbidden while it serves).

The call must produce what moe_dispatch produces from the same inputs: equal
counts and offsets, the same set of pairs per expert, and for every pair the
same bytes (and scales) in its row. Rows inside an expert window may come in a
different order, so rows are matched through pos. Two calls in a row are
checked, since every call reuses the library's one fixed scratch array.

This file is named to be collected last: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from combine_softmax_top_b200 import moe
from combine_softmax_top_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _dispatch_outputs(b: moe.Buffers):
    torch.cuda.synchronize()
    return {
        "counts": b.counts.cpu().numpy(),
        "offsets": b.offsets.cpu().numpy(),
        "pos": b.pos.cpu().numpy().astype(np.int64),
        "row_src": b.row_src.cpu().numpy(),
        "xq": b.xq.cpu(),
        "xs": None if b.xs is None else b.xs.cpu(),
    }


def _assert_same_dispatch(got, ref, s):
    assert np.array_equal(got["counts"], ref["counts"])
    assert np.array_equal(got["offsets"], ref["offsets"])
    cap = s.cap
    gp, rp = got["pos"], ref["pos"]
    assert len(gp) == s.T * s.ks
    assert np.array_equal(gp >= 0, rp >= 0)
    placed = np.nonzero(rp >= 0)[0]
    # same expert window for every pair, and row_src pointing back at it
    assert np.array_equal(gp[placed] // cap, rp[placed] // cap)
    assert np.array_equal(got["row_src"][gp[placed]], placed)
    gi = torch.from_numpy(gp[placed])
    ri = torch.from_numpy(rp[placed])
    assert torch.equal(got["xq"][gi], ref["xq"][ri])
    if ref["xs"] is not None:
        assert torch.equal(got["xs"][gi], ref["xs"][ri])


@pytest.mark.parametrize("name,over", [
    ("decode", {}),                                     # e4m3 rows, 128 tokens
    ("skew", dict(T=256, H=1024, E=32)),                # bf16 rows, skewed counts
    ("tiny", {}),                                       # fp32 rows
    # a shared expert: every token's extra slot goes to expert E of E + 1
    ("decode", dict(T=32, H=512, E=16, k=4, I=256, shared=1)),
])
def test_noalloc_dispatch_matches_workspace_dispatch(name, over, cuda_device):
    s = W.spec(name, **over)
    outs = []
    for seed in (0, 1):                                 # two calls in a row
        inp = W.make_inputs(s, seed=seed, device="cuda", with_weights=False)
        ref = moe.alloc_buffers(s)
        moe.moe_route(ref.shape, inp["logits"], ref.topk_idx, ref.topk_w, ref.ws)
        moe.moe_dispatch(ref.shape, inp["x"], ref.topk_idx, ref.ws, ref.dispatch_bufs())
        assert moe.moe_poll_status(ref.ws) == 0
        got = moe.alloc_buffers(s)
        moe.moe_dispatch_noalloc(got.shape, inp["x"], ref.topk_idx, got.dispatch_bufs())
        outs.append((_dispatch_outputs(got), _dispatch_outputs(ref)))
    for g, r in outs:
        _assert_same_dispatch(g, r, s)


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    # 1024 experts x 512 tiles each: the counters alone need more than 4 MiB
    s = W.spec("decode", T=65536, E=1024)
    sh = moe.make_shape(s)
    b = moe.alloc_buffers(W.spec("decode", T=128, E=16, H=512, I=256))   # any valid pointers
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_dispatch_noalloc(sh, b.out, b.topk_idx, b.dispatch_bufs())
    assert ei.value.code == 1                           # MOE_ERR_INVALID_ARG


def _bound_T(E: int) -> int:
    """The smallest multiple of 128 tokens whose counters, sentinels and ring
    (the whole workspace of a bf16 layer with identity experts, which has no
    scale atoms) need more than the 4 MiB the no-workspace dispatch has."""
    T = 128
    while moe.moe_workspace_bytes(moe.make_shape(W.spec("skew", T=T, E=E, H=16, identity=1))) <= 4 << 20:
        T += 128
    return T


def test_noalloc_rejects_a_shape_just_over_its_scratch():
    """Refused on the host before any CUDA call (so this runs without a GPU;
    the pointers are never looked at)."""
    T = _bound_T(1024)
    sh = moe.make_shape(W.spec("skew", T=T, E=1024, H=16, identity=1))
    fake = ctypes.c_void_p(1 << 20)
    b = moe.moe_dispatch_bufs()
    for f, _ in b._fields_:
        setattr(b, f, 1 << 20)
    assert moe.lib().moe_dispatch_noalloc(ctypes.byref(sh), fake, fake, ctypes.byref(b), None) == 1


def test_noalloc_accepts_a_shape_just_under_its_scratch(cuda_device):
    T = _bound_T(1024) - 128
    s = W.spec("skew", T=T, E=1024, H=16, identity=1)   # 16 values per token keep the windows small
    inp = W.make_inputs(s, seed=3, device="cuda", with_weights=False)
    ref = moe.alloc_buffers(s)
    moe.moe_route(ref.shape, inp["logits"], ref.topk_idx, ref.topk_w, ref.ws)
    moe.moe_dispatch(ref.shape, inp["x"], ref.topk_idx, ref.ws, ref.dispatch_bufs())
    assert moe.moe_poll_status(ref.ws) == 0
    got = moe.alloc_buffers(s)
    moe.moe_dispatch_noalloc(got.shape, inp["x"], ref.topk_idx, got.dispatch_bufs())
    _assert_same_dispatch(_dispatch_outputs(got), _dispatch_outputs(ref), s)


def test_noalloc_accepts_prefill_token_and_expert_counts(cuda_device):
    """T = 8192 over 256 experts (the prefill layer's counts, with a small
    hidden size): 0.5 MB of counters, sentinels and ring."""
    s = W.spec("prefill", H=512, I=256)
    inp = W.make_inputs(s, seed=4, device="cuda", with_weights=False)
    ref = moe.alloc_buffers(s)
    moe.moe_route(ref.shape, inp["logits"], ref.topk_idx, ref.topk_w, ref.ws)
    moe.moe_dispatch(ref.shape, inp["x"], ref.topk_idx, ref.ws, ref.dispatch_bufs())
    assert moe.moe_poll_status(ref.ws) == 0
    got = moe.alloc_buffers(s)
    moe.moe_dispatch_noalloc(got.shape, inp["x"], ref.topk_idx, got.dispatch_bufs())
    _assert_same_dispatch(_dispatch_outputs(got), _dispatch_outputs(ref), s)


def test_noalloc_outputs_feed_identity_combine(cuda_device):
    """What the no-workspace dispatch writes is enough for moe_combine with
    identity experts: the output equals the oracle's identity layer (the
    dequantised token, weights summing to one) within one bf16 rounding."""
    import oracle
    from tests import gpu_harness as G
    from tests.helpers import as_f64, raw
    s = W.spec("sweep", T=512)
    inp = W.make_inputs(s, seed=6, device="cuda")
    b = moe.alloc_buffers(s)
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch_noalloc(b.shape, inp["x"], b.topk_idx, b.dispatch_bufs())
    moe.moe_combine(b.shape, b.dispatch_bufs(), None, b.topk_w, b.ws, b.out)
    assert moe.moe_poll_status(b.ws) == 0
    r = oracle.moe_layer(G.oracle_problem(s, inp), raw(inp["x"]), raw(inp["logits"]))
    out, ref = as_f64(raw(b.out), "bf16"), as_f64(r["out"], "bf16")
    assert np.all(np.abs(out - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-30)
