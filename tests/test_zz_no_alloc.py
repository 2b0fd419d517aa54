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
