"""Pins of the CPU oracle against what the pages and the mathematics fix.

The pages print no worked numerical example for the MoE layer, so every pin
here is a closed form, an invariant, a special case that reduces to a library
routine (torch's float8/bfloat16 casts, float64 matmul, softmax, topk), or
brute force on tiny inputs. Each is chosen so that a plausible slip in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
rounding rule) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from combine_softmax_top_b200 import workloads as W
from tests.helpers import as_f64, bf16_bits_to_f32, max_abs_rel, raw

pytestmark = pytest.mark.filterwarnings("ignore")


# --------------------------------------------------------------- e4m3 codec --

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2  # S.1111.111 only
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_closed_form_landmarks():
    # OCP OFP8 E4M3: max normal 1.75*2^8, min normal 2^-6, subnormal step 2^-9
    v = oracle.e4m3_decode(np.array([0x7E, 0x08, 0x07, 0x01, 0x38, 0x40, 0x80, 0xFE], np.uint8))
    assert list(v[:6]) == [448.0, 2.0 ** -6, 7 * 2.0 ** -9, 2.0 ** -9, 1.0, 2.0]
    assert v[6] == 0.0 and math.copysign(1, v[6]) < 0
    assert v[7] == -448.0


def test_e4m3_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_e4m3_encode_matches_torch_rne():
    rng = np.random.default_rng(0)
    finite = oracle.e4m3_decode(np.array([c for c in range(128) if c != 0x7F], np.uint8))
    finite = np.unique(finite)
    mids = (finite[1:] + finite[:-1]) / 2                  # exact ties
    vals = np.concatenate([
        rng.uniform(-464, 464, 20000), rng.normal(0, 1, 20000), rng.normal(0, 1e-2, 5000),
        mids, -mids, mids * (1 + 1e-12), mids * (1 - 1e-12), [0.0, -0.0, 464.0, -464.0],
    ])
    vals32 = vals.astype(np.float32)  # torch casts from float32
    got = oracle.e4m3_encode(vals32.astype(np.float64))
    ref = torch.from_numpy(vals32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    zero = (got & 0x7F) == 0
    assert np.array_equal(got[~zero], ref[~zero])
    assert np.all((ref[zero] & 0x7F) == 0)


def test_e4m3_ties_to_even_examples():
    # 1.0625 lies halfway between 1.0 (mantissa 000) and 1.125 (001): even wins
    # 1.1875 lies halfway between 1.125 (001) and 1.25 (010): even wins
    got = oracle.e4m3_encode(np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10]))
    assert list(got) == [0x38, 0x3A, 0x00, 0x02]


def test_e4m3_satfinite_and_nan():
    got = oracle.e4m3_encode(np.array([448.0, 464.0, 465.0, 1e30, np.inf, -np.inf, np.nan]))
    assert list(got[:6]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    assert got[6] & 0x7F == 0x7F


# -------------------------------------------------------------- bf16 round --

def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.normal(0, 1, 50000), rng.normal(0, 1e-30, 1000), rng.normal(0, 1e30, 1000),
        np.ldexp(1.0, np.arange(-149, 127)).astype(np.float64),
    ]).astype(np.float32)
    # exact ties: bf16 value plus half a bf16 ulp
    base = torch.from_numpy(rng.normal(0, 1, 2000).astype(np.float32)).to(torch.bfloat16).float()
    ties = (base.view(torch.int32) + (1 << 15)).view(torch.float32).numpy()
    vals = np.concatenate([vals, ties])
    got = oracle.bf16_round(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------- power-of-two scale --

def test_pow2_scale_is_minimal_power_of_two():
    rng = np.random.default_rng(2)
    amax = np.concatenate([np.abs(rng.normal(0, 1, 5000)), np.abs(rng.normal(0, 1e-3, 500)),
                           448.0 * np.ldexp(1.0, np.arange(-20, 20)),
                           np.nextafter(448.0 * np.ldexp(1.0, np.arange(-20, 20)), np.inf)])
    s = oracle.pow2_scale(amax)
    m, e = np.frexp(s)
    assert np.all(m == 0.5)                       # powers of two
    assert np.all(amax <= 448.0 * s)              # never saturates
    assert np.all(amax > 224.0 * s)               # the smallest such power
    assert oracle.pow2_scale(np.array([0.0]))[0] == 1.0
    assert oracle.pow2_scale(np.array([448.0]))[0] == 1.0
    assert oracle.pow2_scale(np.array([np.nextafter(448.0, 1e9)]))[0] == 2.0
    assert oracle.pow2_scale(np.array([1e-45]))[0] == 2.0 ** -126   # clamped


def test_quantize_rows_matches_torch_cast():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (64, 512)).astype(np.float32)
    x[3, :128] = 0.0                 # an all-zero block
    x[4, 128:256] *= 1e-6            # a tiny block
    x[5, 256:384] *= 1e4             # a large block
    q, s = oracle.quantize_rows(x)
    blocks = x.reshape(64, 4, 128).astype(np.float64)
    amax = np.abs(blocks).max(axis=2)
    assert np.array_equal(s.astype(np.float64), oracle.pow2_scale(amax))
    scaled = (blocks / s[:, :, None]).astype(np.float32).reshape(64, 512)   # exact
    ref = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    zero = (q & 0x7F) == 0
    assert np.array_equal(q[~zero], ref[~zero])
    deq = oracle.e4m3_decode(q).reshape(64, 4, 128) * s[:, :, None]
    normal = np.abs(blocks) >= 2.0 ** -6 * s[:, :, None]
    assert np.all(np.abs(deq - blocks)[normal] <= 2.0 ** -4 * np.abs(blocks)[normal])
    assert np.all(np.abs(deq - blocks) <= 2.0 ** -10 * s[:, :, None] + 2.0 ** -4 * np.abs(blocks))


# ------------------------------------------------------------------- route --

def _brute_route(logits, k, renorm):
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        p = torch.softmax(torch.from_numpy(logits[t].astype(np.float64)), 0).numpy()
        idx[t] = order
        sel = p[order]
        w[t] = sel / sel.sum() if renorm else sel
    return idx, w


@pytest.mark.parametrize("renorm", [0, 1])
def test_route_brute_force_with_ties(renorm):
    rng = np.random.default_rng(4)
    logits = rng.integers(-3, 3, (40, 12)).astype(np.float32)   # many exact ties
    logits[0] = 1.0                                            # all equal
    logits[1, :] = np.float32(-0.0)
    logits[1, 5] = 0.0
    for k in (1, 3, 12):
        idx, w = oracle.route(logits, k, renorm)
        ridx, rw = _brute_route(logits, k, renorm)
        assert np.array_equal(idx, ridx)
        assert np.allclose(w, rw, rtol=1e-6, atol=0)
    idx, _ = oracle.route(logits, 3, renorm)
    assert list(idx[0]) == [0, 1, 2]


@pytest.mark.parametrize("renorm", [0, 1])
def test_route_matches_torch_topk_softmax(renorm):
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(300, 256, generator=g)
    idx, w = oracle.route(logits.numpy(), 8, renorm)
    tv, ti = torch.topk(logits, 8, dim=1)
    assert np.array_equal(idx, ti.numpy())
    p = torch.softmax(logits.double(), 1)
    sel = torch.gather(p, 1, ti)
    ref = sel / sel.sum(1, keepdim=True) if renorm else sel
    assert np.allclose(w, ref.numpy(), rtol=1e-6, atol=0)


def test_route_weight_invariants():
    g = torch.Generator().manual_seed(6)
    logits = (torch.randn(100, 64, generator=g) * 5).numpy()
    _, w = oracle.route(logits, 6, 1)
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0)                      # descending
    _, w1 = oracle.route(logits, 1, 1)
    assert np.all(w1 == 1.0)                                    # k = 1 renorm
    _, wall = oracle.route(logits, 64, 0)
    assert np.allclose(wall.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_route_rejects_nonfinite():
    logits = np.zeros((4, 8), np.float32)
    logits[2, 3] = np.nan
    with pytest.raises(oracle.OracleError) as ei:
        oracle.route(logits, 2)
    assert ei.value.code == oracle.NONFINITE


def test_counts_sum_and_bincount():
    g = torch.Generator().manual_seed(7)
    logits = torch.randn(513, 32, generator=g).numpy()
    idx, _ = oracle.route(logits, 4, 1)
    c = oracle.counts(idx, 32)
    assert c.sum() == 513 * 4
    assert np.array_equal(c, np.bincount(idx.ravel(), minlength=32))
    assert all(len(set(row)) == 4 for row in idx)               # distinct experts per token


# -------------------------------------------------- closed-form tiny layer --

def _silu(g):
    return g / (1.0 + math.exp(-g))


@pytest.mark.parametrize("renorm,k", [(1, 1), (0, 1), (1, 2), (0, 2)])
def test_layer_closed_form_two_experts(renorm, k):
    """T=2, E=2, H=2, I=1, fp32: every value below is a closed form."""
    wg = np.array([[[1, 1]], [[1, 0]]], np.float32)       # [E, I, H]
    wu = np.array([[[1, -1]], [[0, 1]]], np.float32)
    wd = np.array([[[1], [0.5]], [[3], [4]]], np.float32)  # [E, H, I]
    x = np.array([[1, 2], [1.5, -0.5]], np.float32)
    logits = np.array([[0.0, 1.0], [2.0, 2.0]], np.float32)
    p = oracle.Problem(2, 2, 2, k, 1, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                       w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                       out_dtype=oracle.F32, renorm=renorm, w_gate=wg, w_up=wu, w_down=wd)
    r = oracle.moe_layer(p, x, logits)

    def expert(e, xv):
        g = float(wg[e, 0] @ xv)
        u = float(wu[e, 0] @ xv)
        h = _silu(g) * u
        return np.array([wd[e, 0, 0] * h, wd[e, 1, 0] * h])

    # token 0: logits (0, 1) -> expert 1 first; token 1: tie -> expert 0 first
    e_ = math.e
    if k == 1:
        w0 = [1.0] if renorm else [e_ / (1 + e_)]
        w1 = [1.0] if renorm else [0.5]
        ref0 = w0[0] * expert(1, x[0].astype(np.float64))
        ref1 = w1[0] * expert(0, x[1].astype(np.float64))
        assert r["idx"].tolist() == [[1], [0]]
    else:
        w0 = [e_ / (1 + e_), 1 / (1 + e_)]
        w1 = [0.5, 0.5]
        ref0 = w0[0] * expert(1, x[0].astype(np.float64)) + w0[1] * expert(0, x[0].astype(np.float64))
        ref1 = w1[0] * expert(0, x[1].astype(np.float64)) + w1[1] * expert(1, x[1].astype(np.float64))
        assert r["idx"].tolist() == [[1, 0], [0, 1]]
    # hand values: expert 1 on x0 gives h = 2 silu(1), y = (3h, 4h)
    assert np.isclose(expert(1, np.array([1.0, 2.0]))[0], 6 / (1 + math.exp(-1)), rtol=1e-15)
    assert np.allclose(r["w"], [w0, w1], rtol=1e-7)
    assert np.allclose(r["out"], np.stack([ref0, ref1]), rtol=1e-6, atol=1e-7)


# --------------------------------------------- expert FFN vs float64 torch --

def _dense_ffn_torch(x, wg, wu, wd, h_round=None, y_round=None):
    g = x @ wg.T
    u = x @ wu.T
    h = torch.nn.functional.silu(g) * u
    if h_round is not None:
        h = h_round(h)
    y = h @ wd.T
    if y_round is not None:
        y = y_round(y)
    return h, y


def _torch_bf16(v):
    return v.float().to(torch.bfloat16).double()


def _torch_requant(h):
    """Per-128 power-of-two requantisation of float64 values, decided in fp32."""
    h32 = h.float()
    b = h32.view(h.shape[0], -1, 128).double()
    amax = b.abs().amax(2)
    s = torch.from_numpy(oracle.pow2_scale(amax.numpy()))
    q = (b / s[:, :, None]).float().to(torch.float8_e4m3fn).double()
    return (q * s[:, :, None]).view(h.shape)


def test_expert_rows_f32_matches_torch():
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=0)
    E = s.E
    p = oracle.Problem(s.T, s.H, E, s.k, s.I, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                       w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                       out_dtype=oracle.F32, w_gate=raw(inp["w_gate"]), w_up=raw(inp["w_up"]),
                       w_down=raw(inp["w_down"]))
    experts = np.arange(s.T, dtype=np.int32) % E
    h, _, y = oracle.expert_rows(p, experts, raw(inp["x"]))
    for r in range(s.T):
        e = experts[r]
        xr = inp["x"][r:r + 1].double()
        rh, ry = _dense_ffn_torch(xr, inp["w_gate"][e].double(), inp["w_up"][e].double(),
                                  inp["w_down"][e].double())
        assert max_abs_rel(h[r], rh[0].numpy()) < 1e-6
        assert max_abs_rel(y[r], ry[0].numpy()) < 1e-6


def test_expert_rows_bf16_matches_torch():
    s = W.spec("skew", T=8, H=256, E=4, I=384, zipf_s=0.0)
    inp = W.make_inputs(s, seed=1)
    p = oracle.Problem(s.T, s.H, s.E, s.k if s.k <= s.E else s.E, s.I, x_dtype=oracle.BF16,
                       xq_dtype=oracle.BF16, w_dtype=oracle.BF16, h_dtype=oracle.BF16,
                       y_dtype=oracle.BF16, out_dtype=oracle.BF16, w_gate=raw(inp["w_gate"]),
                       w_up=raw(inp["w_up"]), w_down=raw(inp["w_down"]))
    experts = (np.arange(s.T, dtype=np.int32) * 3) % s.E
    h, _, y = oracle.expert_rows(p, experts, raw(inp["x"]))
    for r in range(s.T):
        e = experts[r]
        rh, ry = _dense_ffn_torch(inp["x"][r:r + 1].double(), inp["w_gate"][e].double(),
                                  inp["w_up"][e].double(), inp["w_down"][e].double(),
                                  _torch_bf16, _torch_bf16)
        hv, yv = bf16_bits_to_f32(h[r]), bf16_bits_to_f32(y[r])
        # one rounding step may land on the neighbouring bf16 value
        assert np.allclose(hv, rh[0].numpy(), rtol=2 ** -7, atol=1e-30)
        assert max_abs_rel(yv, ry[0].numpy()) < 2 ** -7


def test_expert_rows_e4m3_matches_torch():
    s = W.spec("decode", T=6, H=512, E=3, I=384)
    inp = W.make_inputs(s, seed=2)
    p = oracle.Problem(s.T, s.H, s.E, 2, s.I, x_dtype=oracle.BF16, xq_dtype=oracle.E4M3,
                       w_dtype=oracle.E4M3, h_dtype=oracle.E4M3, y_dtype=oracle.BF16,
                       out_dtype=oracle.BF16, w_gate=raw(inp["w_gate"]), w_up=raw(inp["w_up"]),
                       w_down=raw(inp["w_down"]), s_gate=raw(inp["s_gate"]),
                       s_up=raw(inp["s_up"]), s_down=raw(inp["s_down"]))
    x32 = inp["x"].float().numpy()
    xq, xs = oracle.quantize_rows(x32)
    experts = np.array([0, 1, 2, 2, 1, 0], np.int32)
    h, hs, y = oracle.expert_rows(p, experts, xq, xs)

    def deq_w(q, sc):  # torch's own float8 decode, scales expanded per block
        v = q.view(torch.float8_e4m3fn).double()
        return v * sc.double().repeat_interleave(128, 0).repeat_interleave(128, 1)

    xh = torch.from_numpy(xq).view(torch.float8_e4m3fn).double() * \
        torch.from_numpy(xs).double().repeat_interleave(128, 1)
    for r in range(s.T):
        e = experts[r]
        wg = deq_w(inp["w_gate"][e], inp["s_gate"][e])
        wu = deq_w(inp["w_up"][e], inp["s_up"][e])
        wd = deq_w(inp["w_down"][e], inp["s_down"][e])
        rh, ry = _dense_ffn_torch(xh[r:r + 1], wg, wu, wd, _torch_requant, _torch_bf16)
        hv = oracle.e4m3_decode(h[r]) * np.repeat(hs[r].astype(np.float64), 128)
        assert np.array_equal(hv, rh[0].numpy())
        assert max_abs_rel(bf16_bits_to_f32(y[r]), ry[0].numpy()) < 2 ** -7


# -------------------------------------------------- layer-level invariants --

def test_identical_experts_reduce_to_dense_ffn():
    """All experts equal + renormalised weights: out = the dense FFN of x."""
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=3)
    wg = inp["w_gate"][:1].repeat(s.E, 1, 1).contiguous()
    wu = inp["w_up"][:1].repeat(s.E, 1, 1).contiguous()
    wd = inp["w_down"][:1].repeat(s.E, 1, 1).contiguous()
    p = oracle.Problem(s.T, s.H, s.E, s.k, s.I, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                       w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                       out_dtype=oracle.F32, renorm=1, w_gate=raw(wg), w_up=raw(wu),
                       w_down=raw(wd))
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    _, ref = _dense_ffn_torch(inp["x"].double(), wg[0].double(), wu[0].double(), wd[0].double())
    assert max_abs_rel(r["out"], ref.numpy()) < 1e-6


def test_identity_experts_return_input():
    """Identity experts + renormalised weights: combine returns the input."""
    s = W.spec("sweep", T=64, H=1024, E=32)
    inp = W.make_inputs(s, seed=4)
    p = oracle.Problem(s.T, s.H, s.E, s.k, s.I, x_dtype=oracle.BF16, xq_dtype=oracle.E4M3,
                       w_dtype=oracle.E4M3, h_dtype=oracle.E4M3, y_dtype=oracle.BF16,
                       out_dtype=oracle.BF16, renorm=1, identity=1)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), want_intermediates=True)
    x = inp["x"].double().numpy()
    xh = oracle.e4m3_decode(r["xq"]) * np.repeat(r["xs"].astype(np.float64), 128, axis=1)
    out = as_f64(r["out"], "bf16")
    ref = torch.from_numpy(xh).float().to(torch.bfloat16).double().numpy()
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-38
    assert np.all(np.abs(out - ref) <= ulp)                      # bf16(x_hat) within 1 ulp
    assert np.all(np.abs(out - x) <= 2.0 ** -4 * np.abs(x) + 2.0 ** -7 * np.abs(x)
                  + np.repeat(r["xs"].astype(np.float64), 128, axis=1) * 2.0 ** -10)


def test_layer_equals_composed_steps():
    """moe_layer == route, quantise, expert_rows, combine composed by hand."""
    s = W.spec("decode", T=12, H=256, E=16, k=4, I=256)
    inp = W.make_inputs(s, seed=5)
    kw = dict(x_dtype=oracle.BF16, xq_dtype=oracle.E4M3, w_dtype=oracle.E4M3,
              h_dtype=oracle.E4M3, y_dtype=oracle.BF16, out_dtype=oracle.BF16, renorm=1,
              w_gate=raw(inp["w_gate"]), w_up=raw(inp["w_up"]), w_down=raw(inp["w_down"]),
              s_gate=raw(inp["s_gate"]), s_up=raw(inp["s_up"]), s_down=raw(inp["s_down"]))
    p = oracle.Problem(s.T, s.H, s.E, s.k, s.I, **kw)
    r = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), want_intermediates=True)
    idx, w = oracle.route(raw(inp["logits"]), s.k, 1)
    assert np.array_equal(idx, r["idx"]) and np.array_equal(w, r["w"])
    xq, xs = oracle.quantize_rows(inp["x"].float().numpy())
    assert np.array_equal(xq, r["xq"]) and np.array_equal(xs, r["xs"])
    rows = np.repeat(np.arange(s.T), s.k)
    _, _, y = oracle.expert_rows(p, idx.ravel(), xq[rows], xs[rows])
    assert np.array_equal(y, r["y_pairs"])
    out = oracle.combine(y, w, oracle.BF16, oracle.BF16)
    assert np.array_equal(out, r["out"])


def test_token_subset_matches_full_run():
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=6)
    p = oracle.Problem(s.T, s.H, s.E, s.k, s.I, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                       w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                       out_dtype=oracle.F32, w_gate=raw(inp["w_gate"]), w_up=raw(inp["w_up"]),
                       w_down=raw(inp["w_down"]))
    full = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]))
    part = oracle.moe_layer(p, raw(inp["x"]), raw(inp["logits"]), 5, 11)
    assert np.array_equal(full["out"][5:11], part["out"])


def test_missing_expert_weights_is_an_error():
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=7)
    p = oracle.Problem(s.T, s.H, s.E, s.k, s.I, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                       w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                       out_dtype=oracle.F32, w_gate={0: raw(inp["w_gate"][0])},
                       w_up={0: raw(inp["w_up"][0])}, w_down={0: raw(inp["w_down"][0])})
    with pytest.raises(oracle.OracleError):
        oracle.expert_rows(p, np.array([1], np.int32), raw(inp["x"][:1]))


def _shared_problem(s, wg, wu, wd, shared):
    return oracle.Problem(s.T, s.H, s.E, s.k, s.I, x_dtype=oracle.F32, xq_dtype=oracle.F32,
                          w_dtype=oracle.F32, h_dtype=oracle.F32, y_dtype=oracle.F32,
                          out_dtype=oracle.F32, renorm=1, shared=shared, w_gate=raw(wg), w_up=raw(wu),
                          w_down=raw(wd))


def test_zero_shared_expert_changes_nothing():
    """A shared expert with all-zero weights adds exactly zero: the layer equals
    the one without it, bit for bit."""
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=6)
    z = torch.zeros_like(inp["w_gate"][:1])
    zd = torch.zeros_like(inp["w_down"][:1])
    wg = torch.cat([inp["w_gate"], z]).contiguous()
    wu = torch.cat([inp["w_up"], z]).contiguous()
    wd = torch.cat([inp["w_down"], zd]).contiguous()
    plain = oracle.moe_layer(_shared_problem(s, inp["w_gate"], inp["w_up"], inp["w_down"], 0),
                             raw(inp["x"]), raw(inp["logits"]))
    with_shared = oracle.moe_layer(_shared_problem(s, wg, wu, wd, 1), raw(inp["x"]), raw(inp["logits"]))
    assert np.array_equal(plain["idx"], with_shared["idx"])
    assert np.array_equal(plain["out"], with_shared["out"])


def test_shared_expert_alone_is_the_dense_ffn():
    """Routed experts with all-zero weights and a shared expert: the layer is
    the shared expert's dense SwiGLU FFN of every token, whatever the routing."""
    s = W.spec("tiny")
    inp = W.make_inputs(s, seed=7)
    E = s.E
    z = torch.zeros_like(inp["w_gate"])
    zd = torch.zeros_like(inp["w_down"])
    wg = torch.cat([z, inp["w_gate"][:1]]).contiguous()
    wu = torch.cat([z, inp["w_up"][:1]]).contiguous()
    wd = torch.cat([zd, inp["w_down"][:1]]).contiguous()
    r = oracle.moe_layer(_shared_problem(s, wg, wu, wd, 1), raw(inp["x"]), raw(inp["logits"]),
                         want_intermediates=True)
    _, ref = _dense_ffn_torch(inp["x"].double(), wg[E].double(), wu[E].double(), wd[E].double())
    assert max_abs_rel(r["out"], ref.numpy()) < 1e-6
    # the shared expert's row is the last of each token's k + 1 rows
    yp = r["y_pairs"].reshape(s.T, s.k + 1, s.H)
    assert max_abs_rel(yp[:, s.k], ref.numpy()) < 1e-6
    assert np.all(yp[:, : s.k] == 0)


# ---------------------------------------------------- MX FP4 (E2M1) weights --

# OCP Microscaling Formats (MX) v1.0, FP4 E2M1: the eight magnitudes the
# format represents (codes 0-7; codes 8-15 are their negatives).
_E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_all_codes():
    got = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    ref = np.array(_E2M1_TABLE + [-v for v in _E2M1_TABLE])
    assert np.array_equal(got, ref)
    assert np.signbit(got[8])   # code 8 is -0


def test_ue8m0_decode():
    """UE8M0 (MX v1.0): 2^(byte - 127), byte 255 is NaN."""
    got = oracle.ue8m0_decode(np.array([0, 1, 126, 127, 128, 254, 255], np.uint8))
    assert got[0] == 2.0 ** -127 and got[1] == 2.0 ** -126
    assert got[2] == 0.5 and got[3] == 1.0 and got[4] == 2.0 and got[5] == 2.0 ** 127
    assert np.isnan(got[6])


def _random_mxfp4(rng, rows, cols):
    """Random packed E2M1 codes (two per byte) and UE8M0 scales per 32."""
    packed = rng.integers(0, 256, size=(rows, cols // 2), dtype=np.uint8)
    scales = rng.integers(118, 124, size=(rows, cols // 32), dtype=np.uint8)
    return packed, scales


def _dequant_mxfp4(packed, scales):
    """Independent decode: element 2i is the low nibble of byte i, 2i + 1 the
    high one; every 32 consecutive elements of a row share one scale."""
    table = np.array(_E2M1_TABLE + [-v for v in _E2M1_TABLE])
    rows = packed.shape[0]
    codes = np.empty((rows, packed.shape[1] * 2), np.uint8)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    sc = np.repeat(np.exp2(scales.astype(np.float64) - 127.0), 32, axis=1)
    return torch.from_numpy(table[codes] * sc)


def _fp4_problem(T, H, E, I, wg, wu, wd, sg, su, sd):
    return oracle.Problem(T, H, E, 1, I, x_dtype=oracle.BF16, xq_dtype=oracle.E4M3,
                          w_dtype=oracle.E2M1, h_dtype=oracle.E4M3, y_dtype=oracle.BF16,
                          out_dtype=oracle.BF16, w_gate=wg, w_up=wu, w_down=wd,
                          s_gate=sg, s_up=su, s_down=sd)


def test_expert_rows_e2m1_matches_torch():
    """MX FP4 weights (GC-MoE explainer, "Two MMA Implementations": 4-bit
    weights, one shared exponent per 32 elements): the oracle's expert rows
    equal a float64 torch FFN over independently decoded weights."""
    rng = np.random.default_rng(7)
    T, H, E, I = 5, 256, 2, 384
    wg, sg = zip(*[_random_mxfp4(rng, I, H) for _ in range(E)])
    wu, su = zip(*[_random_mxfp4(rng, I, H) for _ in range(E)])
    wd, sd = zip(*[_random_mxfp4(rng, H, I) for _ in range(E)])
    st = lambda a: np.ascontiguousarray(np.stack(a))
    p = _fp4_problem(T, H, E, I, st(wg), st(wu), st(wd), st(sg), st(su), st(sd))
    x32 = rng.standard_normal((T, H)).astype(np.float32)
    xq, xs = oracle.quantize_rows(x32)
    experts = np.array([0, 1, 1, 0, 1], np.int32)
    h, hs, y = oracle.expert_rows(p, experts, xq, xs)
    xh = torch.from_numpy(xq).view(torch.float8_e4m3fn).double() * \
        torch.from_numpy(xs).double().repeat_interleave(128, 1)
    for r in range(T):
        e = experts[r]
        rh, ry = _dense_ffn_torch(xh[r:r + 1], _dequant_mxfp4(wg[e], sg[e]), _dequant_mxfp4(wu[e], su[e]),
                                  _dequant_mxfp4(wd[e], sd[e]), _torch_requant, _torch_bf16)
        hv = oracle.e4m3_decode(h[r]) * np.repeat(hs[r].astype(np.float64), 128)
        assert np.array_equal(hv, rh[0].numpy())
        assert max_abs_rel(bf16_bits_to_f32(y[r]), ry[0].numpy()) < 2 ** -7


def test_e2m1_weights_equal_e4m3_weights_with_one_scale_per_block():
    """Every E2M1 value is an E4M3 value. With one UE8M0 scale per 128 x 128
    block, the FP4 expert must give the same bytes as the E4M3 expert holding
    the same values with the equal fp32 block scales (two decode paths)."""
    rng = np.random.default_rng(9)
    T, H, I = 4, 256, 256
    mats = {}
    for name, (r, c) in (("g", (I, H)), ("u", (I, H)), ("d", (H, I))):
        packed, _ = _random_mxfp4(rng, r, c)
        blk = rng.integers(119, 123, size=(r // 128, c // 128), dtype=np.uint8)
        s32 = np.repeat(np.repeat(blk, 128, 0), 4, 1)             # [r, c/32], constant per block
        vals = _dequant_mxfp4(packed, np.full_like(s32, 127)).numpy()   # unscaled E2M1 values
        codes = torch.from_numpy(vals).float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy(), vals)
        mats[name] = (packed, s32, codes, np.exp2(blk.astype(np.float64) - 127).astype(np.float32))
    x32 = rng.standard_normal((T, H)).astype(np.float32)
    xq, xs = oracle.quantize_rows(x32)
    experts = np.zeros(T, np.int32)
    p4 = _fp4_problem(T, H, 1, I, *[mats[n][0][None] for n in "gud"], *[mats[n][1][None] for n in "gud"])
    p8 = oracle.Problem(T, H, 1, 1, I, x_dtype=oracle.BF16, xq_dtype=oracle.E4M3, w_dtype=oracle.E4M3,
                        h_dtype=oracle.E4M3, y_dtype=oracle.BF16, out_dtype=oracle.BF16,
                        w_gate=mats["g"][2][None], w_up=mats["u"][2][None], w_down=mats["d"][2][None],
                        s_gate=mats["g"][3][None], s_up=mats["u"][3][None], s_down=mats["d"][3][None])
    h4, hs4, y4 = oracle.expert_rows(p4, experts, xq, xs)
    h8, hs8, y8 = oracle.expert_rows(p8, experts, xq, xs)
    assert np.array_equal(h4, h8) and np.array_equal(hs4, hs8) and np.array_equal(y4, y8)
    assert np.abs(bf16_bits_to_f32(y4)).max() > 0


def test_e2m1_nibble_order_and_scale_index_matter():
    """Swapping the two nibbles of every byte, or transposing which 32-block a
    scale belongs to, must change the result (guards the layout reading)."""
    rng = np.random.default_rng(11)
    T, H, I = 2, 128, 128
    wg, sg = _random_mxfp4(rng, I, H)
    wu, su = _random_mxfp4(rng, I, H)
    wd, sd = _random_mxfp4(rng, H, I)
    x32 = rng.standard_normal((T, H)).astype(np.float32)
    xq, xs = oracle.quantize_rows(x32)
    ex = np.zeros(T, np.int32)
    base = oracle.expert_rows(_fp4_problem(T, H, 1, I, wg[None], wu[None], wd[None], sg[None], su[None], sd[None]),
                              ex, xq, xs)[2]
    swap = lambda b: ((b & 15) << 4) | (b >> 4)
    swapped = oracle.expert_rows(_fp4_problem(T, H, 1, I, swap(wg)[None], wu[None], wd[None], sg[None], su[None],
                                              sd[None]), ex, xq, xs)[2]
    rolled = oracle.expert_rows(_fp4_problem(T, H, 1, I, wg[None], wu[None], wd[None],
                                             np.ascontiguousarray(np.roll(sg, 1, axis=1))[None], su[None], sd[None]),
                                ex, xq, xs)[2]
    assert not np.array_equal(base, swapped)
    assert not np.array_equal(base, rolled)


def test_e2m1_needs_whole_scale_groups():
    """MX FP4 rows are made of whole 32-element scale groups: the oracle
    refuses an H that is not a multiple of 32 (fp32 tokens, so that no other
    block rule applies), and accepts H = 64."""
    rng = np.random.default_rng(3)

    def problem(H):
        wg, sg = _random_mxfp4(rng, 64, 64)
        wd, sd = _random_mxfp4(rng, 64, 64)
        gate = np.ascontiguousarray(wg[:, : H // 2])[None]
        gsc = np.ascontiguousarray(sg[:, : -(-H // 32)])[None]
        return oracle.Problem(1, H, 1, 1, 64, x_dtype=oracle.F32, xq_dtype=oracle.F32, w_dtype=oracle.E2M1,
                              h_dtype=oracle.F32, y_dtype=oracle.F32, out_dtype=oracle.F32,
                              w_gate=gate, w_up=gate.copy(), w_down=np.ascontiguousarray(wd[:H])[None],
                              s_gate=gsc, s_up=gsc.copy(), s_down=np.ascontiguousarray(sd[:H])[None])

    x = rng.standard_normal((1, 48)).astype(np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.expert_rows(problem(48), np.zeros(1, np.int32), x)
    x = rng.standard_normal((1, 64)).astype(np.float32)
    h, _, y = oracle.expert_rows(problem(64), np.zeros(1, np.int32), x)
    assert np.isfinite(y).all()
