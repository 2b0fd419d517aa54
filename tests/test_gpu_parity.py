"""GPU path vs the CPU oracle, stage by stage and end to end, through the C ABI.

Bars: bit-exact top-k indices, counts, offsets and the dispatch permutation
(as a set per expert) and e4m3 bytes; floating-point outputs within max-abs-rel
2e-2 of the oracle fed the same quantised operands, 1e-5 for the fp32 layer.
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
CONFIGS = ["tiny", "decode", "prefill", "skew"]
# rows / tokens the oracle recomputes at full size (tokens are independent)
SAMPLE = {"tiny": None, "decode": 256, "prefill": 96, "skew": 128}


def tol(s):
    return TOL[s.weight] if not s.identity else 2e-2


_cache = {}


def run(name, **over):
    key = (name, tuple(sorted(over.items())))
    if key not in _cache:
        _cache.clear()
        torch.cuda.empty_cache()
        s = W.spec(name, **over)
        inp = W.make_inputs(s, seed=0, device="cuda")
        b = G.run_stages(s, inp)
        assert G.poll(b) == 0
        _cache[key] = (s, inp, b)
    return _cache[key]


def values(a, dt):
    return as_f64(a, dt) if dt != "e4m3" else oracle.e4m3_decode(a)


# ------------------------------------------------------------------ route --

@pytest.mark.parametrize("name", CONFIGS)
def test_route_parity(name):
    s, inp, b = run(name)
    idx, w = oracle.route(raw(inp["logits"]), s.k, s.renorm)
    assert np.array_equal(b.topk_idx.cpu().numpy(), idx)
    assert np.allclose(b.topk_w.cpu().numpy(), w, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("renorm", [0, 1])
@pytest.mark.parametrize("E,k", [(256, 8), (8, 2), (100, 5), (1000, 32)])
def test_route_ties_and_shapes(E, k, renorm, cuda_device):
    g = torch.Generator(device="cuda").manual_seed(11)
    logits = torch.randint(-2, 2, (257, E), generator=g, device="cuda").float()
    logits[0] = 0.5                      # one token with all logits equal
    logits[1, ::3] = 7.0                 # many ties at the top
    s = W.spec("tiny", T=257, E=E, k=k, renorm=renorm)
    b = moe.alloc_buffers(s)
    moe.moe_route(b.shape, logits, b.topk_idx, b.topk_w, b.ws)
    assert G.poll(b) == 0
    idx, w = oracle.route(logits.cpu().numpy(), k, renorm)
    assert np.array_equal(b.topk_idx.cpu().numpy(), idx)
    assert np.allclose(b.topk_w.cpu().numpy(), w, rtol=1e-6, atol=1e-7)


def test_route_nonfinite_latches_error(cuda_device):
    s = W.spec("tiny")
    inp = W.make_inputs(s, device="cuda")
    inp["logits"][3, 5] = float("nan")
    b = moe.alloc_buffers(s)
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    assert G.poll(b) == 6        # MOE_ERR_NONFINITE
    assert G.poll(b) == 0        # cleared by the first poll


# --------------------------------------------------------------- dispatch --

@pytest.mark.parametrize("name", CONFIGS + ["sweep"])
def test_dispatch_parity(name):
    s, inp, b = run(name)
    idx = b.topk_idx.cpu().numpy()
    counts = b.counts.cpu().numpy()
    assert np.array_equal(counts, oracle.counts(idx, s.E))
    assert counts.sum() == s.T * s.k
    assert np.array_equal(b.offsets.cpu().numpy(), G.window_offsets(s, counts))
    rows, pairs, experts = G.placed_rows(b)
    # every pair placed exactly once, in its own expert's window
    assert np.array_equal(np.sort(pairs), np.arange(s.T * s.k))
    assert np.array_equal(idx.ravel()[pairs], experts)
    pos = b.pos.cpu().numpy()
    assert np.array_equal(pos[pairs], rows)
    # the rows hold the quantised (or copied) source tokens, bit-exactly
    sel = rows if s.T * s.k <= 8192 else rows[np.random.default_rng(0).choice(len(rows), 8192, replace=False)]
    src_tok = b.row_src.cpu().numpy()[sel] // s.k
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


def test_dispatch_capacity_overflow_is_reported(cuda_device):
    s = W.spec("tiny", T=300, E=8, k=2, cap_rows=128)
    inp = W.make_inputs(s, device="cuda", with_weights=False)
    inp["logits"][:, 0] += 100.0          # every token picks expert 0 first
    b = moe.alloc_buffers(s)
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, b.dispatch_bufs())
    assert G.poll(b) == 4                 # MOE_ERR_CAPACITY
    counts = b.counts.cpu().numpy()
    assert counts[0] == 128
    pos = b.pos.cpu().numpy().reshape(300, 2)
    assert (pos[:, 0] >= 0).sum() == 128 and (pos[:, 0] == -1).sum() == 172


def test_workspace_reuse_across_calls(cuda_device):
    """Consecutive layers on one workspace (alternating counter sets) agree."""
    s = W.spec("decode", T=64, H=1024, E=32, I=256)
    inp = W.make_inputs(s, seed=3, device="cuda")
    b = moe.alloc_buffers(s)
    outs = []
    for _ in range(3):
        moe.run_layer(b, inp)
        torch.cuda.synchronize()
        outs.append(b.out.clone())
        assert np.array_equal(b.counts.cpu().numpy(), oracle.counts(b.topk_idx.cpu().numpy(), s.E))
    assert G.poll(b) == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])


# -------------------------------------------------------------------- FFN --

@pytest.mark.parametrize("name", CONFIGS)
def test_grouped_ffn_parity(name):
    s, inp, b = run(name)
    rows, pairs, experts = G.placed_rows(b)
    n = SAMPLE[name]
    if n is not None and len(rows) > n:
        pick = np.random.default_rng(1).choice(len(rows), n, replace=False)
        rows, pairs, experts = rows[pick], pairs[pick], experts[pick]
    p = G.oracle_problem(s, inp, experts)
    h, hs, y = oracle.expert_rows(p, experts, G.gather(b.xq, rows), G.gather(b.xs, rows))
    gy = values(G.gather(b.y, rows), s.y)
    ry = values(y, s.y)
    assert max_abs_rel(gy, ry) < tol(s), max_abs_rel(gy, ry)
    gh = values(G.gather(b.hq, rows), s.h)
    rh = values(h, s.h)
    if s.h == W.E4M3:
        gh = gh * np.repeat(G.gather(b.hs, rows).astype(np.float64), 128, axis=1)
        rh = rh * np.repeat(hs.astype(np.float64), 128, axis=1)
    assert max_abs_rel(gh, rh) < tol(s), max_abs_rel(gh, rh)


# ---------------------------------------------------------------- combine --

@pytest.mark.parametrize("name", CONFIGS + ["sweep"])
def test_combine_parity(name):
    s, inp, b = run(name)
    pos = b.pos.cpu().numpy()
    w = b.topk_w.cpu().numpy()
    T = s.T if s.T <= 1024 else 1024
    pr = pos[: T * s.k].astype(np.int64)
    if s.identity:
        q = G.gather(b.xq, pr)
        ypairs = oracle.e4m3_decode(q) * np.repeat(G.gather(b.xs, pr).astype(np.float64), 128, axis=1)
        ypairs = ypairs.astype(np.float32)   # exact: e4m3 value times a power of two
        out = oracle.combine(ypairs, w[:T], oracle.F32, G.ODT[s.out])
    else:
        out = oracle.combine(G.gather(b.y, pr), w[:T], G.ODT[s.y], G.ODT[s.out])
    got = raw(b.out)[:T]
    # fp32 accumulation of k terms: error <= k 2^-24 sum_j |w_j y_j| (plus
    # one rounding of the result to the output dtype)
    if s.identity:
        mag = np.abs(ypairs.astype(np.float64))
    else:
        mag = np.abs(values(G.gather(b.y, pr), s.y))
    terms = (np.abs(w[:T].astype(np.float64)).reshape(-1, 1) * mag).reshape(T, s.k, -1).sum(1)
    acc_err = s.k * 2.0 ** -24 * terms
    if s.out == W.BF16:
        g, r = bf16_bits_to_f32(got).astype(np.float64), bf16_bits_to_f32(out).astype(np.float64)
        assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 2 * acc_err + 1e-30)
    else:
        g, r = got.astype(np.float64), out.astype(np.float64)
        assert np.all(np.abs(g - r) <= 2.0 ** -23 * np.abs(r) + 2 * acc_err + 1e-30)


# ------------------------------------------------------------ whole layer --

@pytest.mark.parametrize("name", CONFIGS)
def test_layer_parity(name):
    s, inp, _ = run(name)
    b = G.run_stages(s, inp, layer=True)        # moe_layer entry point
    assert G.poll(b) == 0
    n = SAMPLE[name] or s.T
    t0 = 0
    t1 = min(s.T, n if name != "decode" else s.T)
    idx = b.topk_idx.cpu().numpy()
    p = G.oracle_problem(s, inp, idx[t0:t1].ravel())
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), t0, t1)
    assert np.array_equal(r["idx"], idx)
    got = as_f64(raw(b.out)[t0:t1], s.out)
    ref = as_f64(r["out"], s.out)
    assert max_abs_rel(got, ref) < tol(s), max_abs_rel(got, ref)


def test_layer_bitwise_stable_across_runs(cuda_device):
    s, inp, b = run("decode")
    b2 = G.run_stages(s, inp, layer=True)
    assert torch.equal(b.out, b2.out)


@pytest.mark.parametrize("T", list(W.SWEEP_T))
def test_identity_experts_return_input(T, cuda_device):
    s = W.spec("sweep", T=T)
    inp = W.make_inputs(s, seed=2, device="cuda")
    b = G.run_stages(s, inp, layer=True)
    assert G.poll(b) == 0
    x = as_f64(raw(inp["x"]), "bf16")
    out = as_f64(raw(b.out), "bf16")
    # e4m3 relative bound 2^-4, plus one bf16 rounding, plus the subnormal step
    amax_blk = np.repeat(np.abs(x).reshape(T, -1, 128).max(2), 128, axis=1)
    assert np.all(np.abs(out - x) <= (2.0 ** -4 + 2.0 ** -7) * np.abs(x) + amax_blk * 2.0 ** -12)
    p = G.oracle_problem(s, inp)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    ref = as_f64(r["out"], "bf16")
    assert np.all(np.abs(out - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-30)


# ------------------------------------------------------- bounded waits --

def test_ffn_wait_runs_out_and_context_survives(cuda_device):
    """Withdraw one published tile's sentinel: the FFN's wait for that tile
    must give up (MOE_ERR_TIMEOUT) instead of hanging, and the device must
    stay usable."""
    s = W.spec("decode", T=32, H=512, E=16, k=4, I=256)
    inp = W.make_inputs(s, seed=5, device="cuda")
    b = moe.alloc_buffers(s)
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, b.dispatch_bufs())
    assert G.poll(b) == 0
    # workspace layout: 256-byte header (epoch_next, epoch_cur, ...), two
    # counter sets, then one 32-bit sentinel per (expert, 128-row tile)
    hdr = b.ws[:16].view(torch.int32)
    assert int(hdr[1]) == 1
    tpe = s.cap // 128
    set_words = 8 + s.E + 2 * s.E * tpe + 2 * s.E + 1
    sent_off = 256 + 2 * (((set_words * 4 + 255) // 256) * 256)
    sentinels = b.ws[sent_off:sent_off + 4 * s.E * tpe].view(torch.int32)
    e = int(np.nonzero(b.counts.cpu().numpy())[0][0])
    assert int(sentinels[e * tpe]) >> 8 == 1     # published in epoch 1
    sentinels[e * tpe] = 0                       # as if never published
    torch.cuda.synchronize()
    moe.moe_grouped_ffn(b.shape, b.dispatch_bufs(), moe.weights_struct(inp), b.ws, b.y)
    assert G.poll(b) == 5                        # MOE_ERR_TIMEOUT
    # the context is intact: a fresh layer runs and matches the oracle
    b2 = G.run_stages(s, inp, layer=True)
    assert G.poll(b2) == 0
    p = G.oracle_problem(s, inp)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    assert max_abs_rel(as_f64(raw(b2.out), "bf16"), as_f64(r["out"], "bf16")) < 2e-2


@pytest.mark.parametrize("xq", ["e4m3", "bf16"])
def test_staged_combine_with_dropped_rows(xq, cuda_device):
    """Layers with many tokens take the shared-memory-staged combine; slots
    whose row was dropped (capacity overflow, pos = -1) add nothing, and k = 3
    exercises a slot count that is not a power of two."""
    s = W.spec("sweep", T=1024, H=512, E=4, k=3, xq=xq, cap_rows=512)
    inp = W.make_inputs(s, seed=3, device="cuda")
    inp["logits"][:, 0] += 100.0              # every token picks expert 0 first: 512 of them kept
    b = G.run_stages(s, inp)
    assert G.poll(b) == 4                     # MOE_ERR_CAPACITY, reported; the layer still completes
    pos = b.pos.cpu().numpy().astype(np.int64)
    w = b.topk_w.cpu().numpy()
    assert (pos.reshape(s.T, s.k)[:, 0] == -1).sum() == 512   # (the other experts overflow too)
    keep = pos >= 0
    safe = np.where(keep, pos, 0)
    if xq == "e4m3":
        rows = oracle.e4m3_decode(G.gather(b.xq, safe)) * np.repeat(G.gather(b.xs, safe).astype(np.float64), 128, axis=1)
    else:
        rows = values(G.gather(b.xq, safe), "bf16")
    rows = np.where(keep[:, None], rows, 0.0).astype(np.float32)   # exact in fp32
    out = oracle.combine(rows, w, oracle.F32, G.ODT[s.out])
    got = raw(b.out)
    mag = (np.abs(w.astype(np.float64)).reshape(-1, 1) * np.abs(rows.astype(np.float64))).reshape(s.T, s.k, -1).sum(1)
    g, r = bf16_bits_to_f32(got).astype(np.float64), bf16_bits_to_f32(out).astype(np.float64)
    assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + 2 * s.k * 2.0 ** -24 * mag + 1e-30)


@pytest.mark.parametrize("over", [dict(T=64, H=512, E=8, k=2, I=256),        # 64-row tiles
                                  dict(T=300, H=512, E=4, k=2, I=384)],      # 128-row tiles, down pairs
                         ids=["small_tiles", "big_tiles"])
def test_ffn_repeated_on_one_dispatch(over, cuda_device):
    """The grouped FFN run three times on one dispatch: each call hands out its
    units from a counter that the call's last CTA resets, and counts its calls
    for the down units' dependency; every call must give the same bits."""
    s = W.spec("decode", **over)
    inp = W.make_inputs(s, seed=5, device="cuda")
    b = moe.alloc_buffers(s)
    bufs = b.dispatch_bufs()
    w = moe.weights_struct(inp)
    moe.moe_route(b.shape, inp["logits"], b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch(b.shape, inp["x"], b.topk_idx, b.ws, bufs)
    ys, hs = [], []
    for _ in range(3):
        b.y.zero_()
        b.hq.view(torch.uint8).zero_()
        moe.moe_grouped_ffn(b.shape, bufs, w, b.ws, b.y)
        torch.cuda.synchronize()
        assert G.poll(b) == 0
        ys.append(b.y.clone())
        hs.append(b.hq.view(torch.uint8).clone())
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    assert torch.equal(hs[0], hs[1]) and torch.equal(hs[1], hs[2])
    assert ys[0].abs().sum().item() > 0


def test_dispatch_e4m3_encoder_dense_sweep(cuda_device):
    """The dispatch kernel's e4m3 encoding against the oracle's encoder over a
    dense sample of fp32 values in [-448, 448]: every 137th bit pattern of
    each sign, from the subnormal range to 448 (ties, subnormals and the top
    binade included). Each 128-value block carries +-448, so its scale is
    exactly 1 and the stored byte is the encoding of the value itself."""
    stride = 137
    pos_bits = np.arange(0, 0x43E00001, stride, dtype=np.uint32)
    vals = np.concatenate([pos_bits.view(np.float32), -pos_bits.view(np.float32)])
    per_row = 127
    T = -(-len(vals) // per_row)
    x = np.zeros((T, 128), np.float32)
    x[:, 0] = np.where(np.arange(T) % 2 == 0, 448.0, -448.0)
    flat = np.zeros(T * per_row, np.float32)
    flat[: len(vals)] = vals
    x[:, 1:] = flat.reshape(T, per_row)
    s = W.spec("sweep", T=T, H=128, E=1, k=1, act=W.F32, xq=W.E4M3, out=W.F32)
    b = moe.alloc_buffers(s)
    xd = torch.from_numpy(x).cuda()
    logits = torch.zeros((T, 1), dtype=torch.float32, device="cuda")
    moe.moe_route(b.shape, logits, b.topk_idx, b.topk_w, b.ws)
    moe.moe_dispatch(b.shape, xd, b.topk_idx, b.ws, b.dispatch_bufs())
    assert G.poll(b) == 0
    pos = b.pos.cpu().numpy().astype(np.int64)
    assert (pos >= 0).all()
    got = b.xq[torch.from_numpy(pos).cuda()].cpu().numpy()
    assert np.array_equal(b.xs[torch.from_numpy(pos).cuda()].cpu().numpy(), np.ones((T, 1), np.float32))
    ref = oracle.e4m3_encode(x.astype(np.float64).ravel()).reshape(T, 128)
    same = (got == ref) | (((got & 0x7F) == 0) & ((ref & 0x7F) == 0))   # +-0
    assert same.all(), np.argwhere(~same)[:5]


# ------------------------------------------- the workspace-only layer call --

@pytest.mark.parametrize("name,over", [
    ("decode", dict(T=32, H=512, E=16, k=4, I=256)),
    ("decode", dict(T=300, H=512, E=4, k=2, I=384, compact=1)),
    ("tiny", {}),
])
def test_layer_with_intermediates_in_workspace(name, over, cuda_device):
    """moe_layer (every intermediate carved from its workspace) gives the same
    bytes as moe_layer_bufs (the caller's buffers) on the same inputs: the
    layer output is bitwise stable run to run."""
    s = W.spec(name, **over)
    inp = W.make_inputs(s, seed=7, device="cuda")
    b = G.run_stages(s, inp, layer=True)
    assert G.poll(b) == 0
    lw = moe.alloc_layer(s)
    for _ in range(2):                          # two calls on one workspace
        moe.run_layer_ws(lw, inp)
        torch.cuda.synchronize()
        assert moe.moe_poll_status(lw.ws) == 0
        assert torch.equal(lw.out, b.out)


# ------------------------------------------------ weight scale precondition --

@pytest.mark.parametrize("bad", [0.75, -1.0, 0.0, float("inf"), float("nan"), 2.0 ** -130])
@pytest.mark.parametrize("over", [dict(T=32, H=512, E=16, k=4, I=256), dict(T=16, H=512, E=32, k=4, I=256)])
def test_weight_scales_that_are_not_powers_of_two_are_refused(bad, over, cuda_device):
    """The block-scaled MMA applies a weight scale as an 8-bit exponent; a
    scale it cannot apply exactly (a mantissa, a sign, zero, inf, NaN, a
    subnormal) is refused on the device with MOE_ERR_INVALID_ARG instead of
    being truncated, whichever matrix holds it. A power of two passes."""
    s = W.spec("decode", **over)
    inp = W.make_inputs(s, seed=8, device="cuda")
    for name in ("s_gate", "s_up", "s_down"):
        case = dict(inp)
        sc = inp[name].clone()
        # a mantissa or a sign on a valid scale; zero, inf, NaN, a subnormal as is
        sc[:, 0, 1] = sc[:, 0, 1] * bad if bad in (0.75, -1.0) else torch.full_like(sc[:, 0, 1], bad)
        case[name] = sc
        b = G.run_stages(s, case)
        assert G.poll(b) == 1, (name, bad)      # MOE_ERR_INVALID_ARG
    ok = dict(inp)
    ok["s_up"] = inp["s_up"] * 2.0
    b = G.run_stages(s, ok)
    assert G.poll(b) == 0
