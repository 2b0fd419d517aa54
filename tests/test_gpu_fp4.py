"""MX FP4 expert weights (weight_dtype = MOE_E2M1) through the C ABI, against
the oracle.

The GC-MoE explainer ("Two MMA Implementations in the Compute Partition")
names 4-bit microscaled weights, 32 elements to one shared exponent, for the
block-scaled tcgen05 MMA. Here the weights are E2M1 with a UE8M0 scale per 32
along K and the tokens stay e4m3 with their per-128 power-of-two scales: one
kind::mxf8f6f4 MMA of mixed operand types. Weight tiles arrive packed (half
the bytes of e4m3) and are spread to one code per byte in shared memory by
the copy itself. The cases cover 64-row token tiles (two K slabs per stage for
small down jobs), 128-row tiles with down pairs, an odd number of H slices,
joined tails, the shared expert and compact windows, and the full decode and
prefill shapes on sampled rows.
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

TOL = 2e-2
CASES = [
    ("small_tiles", "decode_fp4", dict(T=32, H=512, E=16, k=4, I=256)),     # 64-row tiles, 2-slab down
    ("big_tiles_pairs", "decode_fp4", dict(T=300, H=512, E=4, k=2, I=384)),  # 128-row tiles, down pairs
    ("big_tiles_odd_h", "decode_fp4", dict(T=300, H=640, E=4, k=2, I=256)),  # five H slices: no pairs
    ("joined_tails", "decode_fp4", dict(T=276, H=512, E=4, k=2, I=256)),     # ~138 rows each: 128 + a short tail
    ("decode", "decode_fp4", {}),
    ("prefill", "prefill_fp4", {}),
]
SAMPLE = 96


@pytest.mark.parametrize("name,base,over", CASES, ids=[c[0] for c in CASES])
def test_fp4_grouped_ffn(name, base, over, cuda_device):
    s = W.spec(base, **over)
    inp = W.make_inputs(s, seed=4, device="cuda")
    b = G.run_stages(s, inp)
    assert G.poll(b) == 0
    rows, pairs, experts = G.placed_rows(b)
    if len(rows) > SAMPLE:
        pick = np.random.default_rng(1).choice(len(rows), SAMPLE, replace=False)
        rows, pairs, experts = rows[pick], pairs[pick], experts[pick]
    p = G.oracle_problem(s, inp, experts)
    h, hs, y = oracle.expert_rows(p, experts, G.gather(b.xq, rows), G.gather(b.xs, rows))
    err = max_abs_rel(as_f64(G.gather(b.y, rows), s.y), as_f64(y, s.y))
    assert err < TOL, err
    gh = oracle.e4m3_decode(G.gather(b.hq, rows)) * np.repeat(G.gather(b.hs, rows).astype(np.float64), 128, axis=1)
    rh = oracle.e4m3_decode(h) * np.repeat(hs.astype(np.float64), 128, axis=1)
    assert max_abs_rel(gh, rh) < TOL, max_abs_rel(gh, rh)


LAYER_CASES = [
    ("small", "decode_fp4", dict(T=32, H=512, E=16, k=4, I=256)),
    ("shared_expert", "decode_fp4", dict(T=300, H=512, E=4, k=2, I=384, shared=1)),
    ("compact", "decode_fp4", dict(T=300, H=512, E=4, k=2, I=384, compact=1)),
    ("decode", "decode_fp4", {}),
    # <= 4 rows per expert with a shared expert: 16-row tiles, the shared
    # expert's 64 rows in four chunks (scale words gathered for rows 16..63)
    ("r16_shared", "decode_fp4", dict(T=64, H=512, E=64, k=4, I=256, shared=1)),
]


@pytest.mark.parametrize("name,base,over", LAYER_CASES, ids=[c[0] for c in LAYER_CASES])
def test_fp4_layer(name, base, over, cuda_device):
    s = W.spec(base, **over)
    inp = W.make_inputs(s, seed=5, device="cuda")
    b = G.run_stages(s, inp, layer=True)
    assert G.poll(b) == 0
    n = min(s.T, 128)
    idx = b.topk_idx.cpu().numpy()
    p = G.oracle_problem(s, inp, idx[:n].ravel())
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), 0, n)
    assert np.array_equal(r["idx"], idx[:, : s.k])
    err = max_abs_rel(as_f64(raw(b.out)[:n], s.out), as_f64(r["out"], s.out))
    assert err < TOL, err


def test_fp4_weights_equal_e4m3_weights_on_the_gpu(cuda_device):
    """4-bit weights whose scales are constant over each 128 x 128 block are
    also exact e4m3 weights with one fp32 scale per block; the layer must give
    the same bits through both tensor-core paths (different weight copies,
    scale atoms and MMA operand formats)."""
    s4 = W.spec("decode_fp4", T=64, H=512, E=8, k=2, I=256)
    inp = W.make_inputs(s4, seed=6, device="cuda")
    table = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0],
                         device="cuda")
    inp8 = {k: v for k, v in inp.items() if not k.startswith(("w_", "s_"))}
    for m in ("gate", "up", "down"):
        rows = inp[f"s_{m}_rows"]                                    # [E, R, C/32]
        ne, R, G32 = rows.shape
        blk = rows.view(ne, R // 128, 128, G32 // 4, 4)[:, :, 0, :, 0]   # one scale per block
        flat = blk.repeat_interleave(128, 1).repeat_interleave(4, 2).contiguous()
        inp[f"s_{m}_rows"] = flat
        inp[f"s_{m}"] = W.scale_atoms(flat)
        packed = inp[f"w_{m}"]
        codes = torch.stack([packed & 15, packed >> 4], dim=-1).view(ne, R, -1).long()
        inp8[f"w_{m}"] = table[codes].to(torch.float8_e4m3fn).view(torch.uint8)
        inp8[f"s_{m}"] = torch.exp2(blk.float() - 127.0).contiguous()
    b4 = G.run_stages(s4, inp, layer=True)
    b8 = G.run_stages(s4.with_(weight=W.E4M3), inp8, layer=True)
    assert G.poll(b4) == 0 and G.poll(b8) == 0
    assert torch.equal(b4.out, b8.out)
    assert b4.out.float().abs().max().item() > 0


def test_fp4_weight_alignment_is_checked(cuda_device):
    """Packed 4-bit matrices must start on 32 bytes (the copy unit's rule for
    them); an offset of 16 bytes is refused on the host."""
    s = W.spec("decode_fp4", T=32, H=512, E=16, k=4, I=256)
    inp = W.make_inputs(s, seed=7, device="cuda")
    b = moe.alloc_buffers(s)
    w = moe.weights_struct(inp)
    w.w_gate += 16
    w2 = moe.weights_struct(inp)
    w2.s_up += 8                                        # scale atoms move in 16-byte units
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, b.dispatch_bufs())
    for bad in (w, w2):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_grouped_ffn(b.shape, b.dispatch_bufs(), bad, b.ws, b.y)
        assert ei.value.code == 1


def test_fp4_compact_shared_workspace_reuse(cuda_device):
    """4-bit weights, compact windows and a shared expert on one workspace
    over calls with changing routing: each call gives the bits of a fresh run."""
    s = W.spec("decode_fp4", T=96, H=512, E=32, k=4, I=256, compact=1, shared=1)
    ins = [W.make_inputs(s, seed=sd, device="cuda") for sd in (0, 1)]
    ins[1]["logits"][:, :3] += 50.0
    b = moe.alloc_buffers(s)
    outs = []
    for i in (0, 1, 0):
        moe.run_layer(b, ins[i])
        torch.cuda.synchronize()
        assert G.poll(b) == 0
        outs.append(b.out.clone())
    assert torch.equal(outs[0], outs[2])
    fresh = G.run_stages(s, ins[1], layer=True)
    assert torch.equal(fresh.out, outs[1])
