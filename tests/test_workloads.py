"""Input preparation in workloads.py (CPU): the MX FP4 weight draw and the
scale-atom permutation the library reads. These hold no layer arithmetic;
the checks make sure the inputs are what the readings say they are."""
import numpy as np
import torch

import oracle
from combine_softmax_top_b200 import workloads as W


def _decode(packed, scales):
    codes = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    codes[..., 0::2] = packed & 15
    codes[..., 1::2] = packed >> 4
    return oracle.e2m1_decode(codes) * np.repeat(oracle.ue8m0_decode(scales), 32, axis=-1)


def test_mxfp4_draw_is_within_half_a_step():
    """Every 32-value group gets the smallest power-of-two scale that keeps it
    within +-6, and each value goes to a nearest E2M1 magnitude: the error is
    at most half the largest gap of the grid (1, between 4 and 6) times the
    scale, and the scale is minimal."""
    s = W.spec("decode_fp4", T=4, H=256, E=2, I=128)
    inp = W.make_inputs(s, seed=3)
    g = W._gen(3, 2, torch.device("cpu"))
    draw = (torch.randn((2, 128, 256), generator=g) * s.w_std).numpy().astype(np.float64)
    packed, sc = inp["w_gate"].numpy(), inp["s_gate_rows"].numpy()
    deq = _decode(packed, sc)
    scale = np.repeat(oracle.ue8m0_decode(sc), 32, axis=-1)
    assert np.all(np.abs(deq - draw) <= 1.0 * scale + 1e-30)
    amax = np.abs(draw).reshape(2, 128, 8, 32).max(-1)
    s32 = oracle.ue8m0_decode(sc)
    assert np.all(amax <= 6 * s32) and np.all(amax > 3 * s32)   # minimal power of two


def test_scale_atoms_are_the_stated_permutation():
    rng = np.random.default_rng(5)
    rows = rng.integers(0, 255, size=(2, 256, 12), dtype=np.uint8)   # 2 matrices, 256 x 384
    atoms = W.scale_atoms(torch.from_numpy(rows)).numpy()
    assert atoms.shape == (2, 2, 3, 512)
    for m in range(2):
        for r in range(256):
            for g in range(12):
                rr = r % 128
                assert atoms[m, r // 128, g // 4, (rr % 32) * 16 + (rr // 32) * 4 + g % 4] == rows[m, r, g]


def test_compact_rows_bound():
    """Compact windows hold the T * k pairs plus at most one partial tile per
    expert, for any routing."""
    for T, k, E in ((1, 1, 1), (37, 3, 5), (8192, 8, 256)):
        s = W.spec("decode", T=T, k=k, E=E, compact=1)
        counts = np.random.default_rng(T).multinomial(T * k, np.ones(E) / E)
        need = int((-(-counts // 128)).sum() * 128)
        assert need <= s.rows()
