"""Seeded synthetic workloads for the MoE layer.

This module only draws inputs. It holds none of the layer's arithmetic: the
GPU library and the CPU oracle both receive the tensors made here, and
neither is imported by it.

Recipe (one seed, several independent streams): stream ``seed * 16 + tag``
with tag 0 = router logits, 1 = activations, 2/3/4 = W_gate/W_up/W_down.
Each array is drawn as float32 normals and then cast to its stored dtype.

Weights stored as e4m3 are prepared the way a checkpoint would be: each
128 x 128 block of the float32 draw gets the smallest power-of-two scale that
keeps the block inside the e4m3 range, and the divided values are cast with
``torch``'s own float8 conversion (nearest-even). This is input preparation:
the layer takes quantised weights as given.

Weights stored as e2m1 (MX FP4) get one power-of-two scale per 32 values
along K, the smallest that keeps the 32 inside +-6, and each divided value goes
to the nearest E2M1 magnitude; two codes per byte, element 2i in the low
nibble. The scales come in two layouts of the same bytes: per row
([.., rows, cols/32], what the oracle reads) and in 512-byte tensor-memory
scale atoms ([.., rows/128, cols/128, 512], what the library reads).

Draws depend on the device the generator runs on (CPU and CUDA generators give
different streams for one seed); tests always feed both implementations the
same tensors.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

F32, BF16, E4M3, E2M1 = "f32", "bf16", "e4m3", "e2m1"


@dataclass(frozen=True)
class Spec:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    act: str          # dtype of x
    xq: str           # dtype tokens are stored in for the experts
    weight: str       # expert weight dtype
    h: str            # dtype of the SwiGLU output
    y: str            # dtype of expert outputs
    out: str          # dtype of the layer output
    renorm: int = 1
    identity: int = 0
    x_std: float = 1.0
    w_std: float = 0.02
    zipf_s: float = 0.0   # > 0: add log p_e, p_e proportional to (e+1)^-s, to the logits
    cap_rows: int = 0     # 0: default round_up(T, 128)
    shared: int = 0       # 1: one shared expert (index E) every token also goes through, weight 1
    compact: int = 0      # 1: expert windows packed back to back after a counting pass
    extra: dict = field(default_factory=dict)

    def with_(self, **kw) -> "Spec":
        return replace(self, **kw)

    @property
    def cap(self) -> int:
        return self.cap_rows if self.cap_rows else max(128, -(-self.T // 128) * 128)

    @property
    def ne(self) -> int:
        """Experts with weights and windows (the shared one included)."""
        return self.E + self.shared

    @property
    def ks(self) -> int:
        """Slots per token (the shared expert's included)."""
        return self.k + self.shared

    def rows(self, T: int | None = None) -> int:
        """Rows of the expert buffers: ne windows of cap rows, or with compact
        windows the T * ks pairs plus one partial 128-row tile per expert."""
        T = self.T if T is None else T
        if self.compact:
            return (-(-T * self.ks // 128) + self.ne) * 128
        cap = self.cap_rows if self.cap_rows else max(128, -(-T // 128) * 128)
        return self.ne * cap


# The five workloads of the layer (tiny fp32, decode, prefill, skewed routing,
# and the dispatch+combine sweep with identity experts).
CONFIGS = {
    "tiny": Spec("tiny", T=16, H=256, E=8, k=2, I=512, act=F32, xq=F32, weight=F32, h=F32,
                 y=F32, out=F32, x_std=0.02, w_std=0.02),
    "decode": Spec("decode", T=128, H=7168, E=256, k=8, I=2048, act=BF16, xq=E4M3, weight=E4M3,
                   h=E4M3, y=BF16, out=BF16),
    "prefill": Spec("prefill", T=8192, H=7168, E=256, k=8, I=2048, act=BF16, xq=E4M3,
                    weight=E4M3, h=E4M3, y=BF16, out=BF16),
    "decode_fp4": Spec("decode_fp4", T=128, H=7168, E=256, k=8, I=2048, act=BF16, xq=E4M3,
                       weight=E2M1, h=E4M3, y=BF16, out=BF16),
    "prefill_fp4": Spec("prefill_fp4", T=8192, H=7168, E=256, k=8, I=2048, act=BF16, xq=E4M3,
                        weight=E2M1, h=E4M3, y=BF16, out=BF16),
    "skew": Spec("skew", T=4096, H=4096, E=128, k=8, I=1536, act=BF16, xq=BF16, weight=BF16,
                 h=BF16, y=BF16, out=BF16, zipf_s=1.2),
    "sweep": Spec("sweep", T=128, H=7168, E=256, k=8, I=128, act=BF16, xq=E4M3, weight=E4M3,
                  h=E4M3, y=BF16, out=BF16, identity=1),
}
SWEEP_T = (1, 8, 32, 128, 512, 4096)


def spec(name: str, **overrides) -> Spec:
    return CONFIGS[name].with_(**overrides) if overrides else CONFIGS[name]


def _gen(seed: int, tag: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 16 + tag)
    return g


def _cast_act(x: torch.Tensor, dt: str) -> torch.Tensor:
    return x if dt == F32 else x.to(torch.bfloat16)


def _block_quantize_weights(w: torch.Tensor):
    """[n, R, C] float32 -> (e4m3 codes as uint8 [n, R, C], fp32 scales [n, R/128, C/128])."""
    n, R, C = w.shape
    b = w.view(n, R // 128, 128, C // 128, 128)
    amax = b.abs().amax(dim=(2, 4)).double()
    p = torch.where(amax > 0, torch.ceil(torch.log2(amax / 448.0)), torch.zeros_like(amax))
    p = p + (amax > 448.0 * torch.exp2(p)).double()          # guard the log2 rounding
    scale = torch.exp2(p).float()
    q = (b / scale[:, :, None, :, None]).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).view(n, R, C), scale


# E2M1 magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0-7) and the midpoints between them
_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _mxfp4_quantize_weights(w: torch.Tensor):
    """[n, R, C] float32 -> (packed E2M1 codes uint8 [n, R, C/2], UE8M0 scale
    bytes uint8 [n, R, C/32])."""
    n, R, C = w.shape
    b = w.view(n, R, C // 32, 32)
    amax = b.abs().amax(dim=3).double()
    p = torch.where(amax > 0, torch.ceil(torch.log2(amax / 6.0)), torch.zeros_like(amax))
    p = p + (amax > 6.0 * torch.exp2(p)).double()          # guard the log2 rounding
    p = p.clamp(-127, 127)
    v = b / torch.exp2(p).float()[..., None]
    mids = torch.tensor(_E2M1_MIDS, dtype=torch.float32, device=w.device)
    code = torch.bucketize(v.abs(), mids).to(torch.uint8) | ((v < 0).to(torch.uint8) << 3)
    code = code.view(n, R, C)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), (p + 127).to(torch.uint8)


def scale_atoms(s_rows: torch.Tensor) -> torch.Tensor:
    """Per-row UE8M0 scales [n, R, C/32] -> scale atoms [n, R/128, C/128, 512]:
    row r of a 128-row block, 32-value group b of a 128-value block at byte
    (r % 32) * 16 + (r // 32) * 4 + b (a byte permutation, no arithmetic)."""
    n, R, G = s_rows.shape
    a = s_rows.view(n, R // 128, 4, 32, G // 4, 4)          # [n, rb, r//32, r%32, kb, b]
    return a.permute(0, 1, 4, 3, 2, 5).reshape(n, R // 128, G // 4, 512).contiguous()


def _weights(s: Spec, seed: int, tag: int, rows: int, cols: int, device, chunk: int = 16):
    g = _gen(seed, tag, device)
    ne = s.ne
    if s.weight == E2M1:
        q = torch.empty((ne, rows, cols // 2), dtype=torch.uint8, device=device)
        sc = torch.empty((ne, rows, cols // 32), dtype=torch.uint8, device=device)
        for e0 in range(0, ne, chunk):
            n = min(chunk, ne - e0)
            w = torch.randn((n, rows, cols), generator=g, device=device) * s.w_std
            q[e0:e0 + n], sc[e0:e0 + n] = _mxfp4_quantize_weights(w)
            del w
        return q, sc
    if s.weight == E4M3:
        q = torch.empty((ne, rows, cols), dtype=torch.uint8, device=device)
        sc = torch.empty((ne, rows // 128, cols // 128), dtype=torch.float32, device=device)
        for e0 in range(0, ne, chunk):
            n = min(chunk, ne - e0)
            w = torch.randn((n, rows, cols), generator=g, device=device) * s.w_std
            q[e0:e0 + n], sc[e0:e0 + n] = _block_quantize_weights(w)
            del w
        return q, sc
    out = torch.empty((ne, rows, cols), dtype=torch.float32 if s.weight == F32 else torch.bfloat16,
                      device=device)
    for e0 in range(0, ne, chunk):
        n = min(chunk, ne - e0)
        w = torch.randn((n, rows, cols), generator=g, device=device) * s.w_std
        out[e0:e0 + n] = w.to(out.dtype)
    return out, None


def make_inputs(s: Spec, seed: int = 0, device="cpu", with_weights: bool = True) -> dict:
    """Router logits [T, E] fp32, activations x [T, H], and (unless identity
    experts) W_gate/W_up [E', I, H], W_down [E', H, I] with e4m3 block scales,
    E' = E + shared (the shared expert last)."""
    dev = torch.device(device)
    logits = torch.randn((s.T, s.E), generator=_gen(seed, 0, dev), device=dev)
    if s.zipf_s > 0:
        ranks = torch.arange(1, s.E + 1, dtype=torch.float64)
        p = ranks.pow(-s.zipf_s)
        p = p / p.sum()
        logits = logits + torch.log(p).float().to(dev)[None, :]
    x = torch.randn((s.T, s.H), generator=_gen(seed, 1, dev), device=dev) * s.x_std
    inp = {"logits": logits.contiguous(), "x": _cast_act(x, s.act).contiguous()}
    if with_weights and not s.identity:
        inp["w_gate"], inp["s_gate"] = _weights(s, seed, 2, s.I, s.H, dev)
        inp["w_up"], inp["s_up"] = _weights(s, seed, 3, s.I, s.H, dev)
        inp["w_down"], inp["s_down"] = _weights(s, seed, 4, s.H, s.I, dev)
        if s.weight == E2M1:   # per-row scales for the oracle, atoms for the library
            for k in ("s_gate", "s_up", "s_down"):
                inp[k + "_rows"] = inp[k]
                inp[k] = scale_atoms(inp[k])
    return inp


def bytes_per_expert(s: Spec) -> int:
    """Weight bytes one touched expert streams (matrices plus e4m3 scales)."""
    if s.weight == E2M1:   # half a byte per weight, one scale byte per 32
        return 3 * s.I * s.H // 2 + 3 * s.I * s.H // 32
    el = {F32: 4, BF16: 2, E4M3: 1}[s.weight]
    b = 3 * s.I * s.H * el
    if s.weight == E4M3:
        b += 3 * (s.I // 128) * (s.H // 128) * 4
    return b


def expected_touched_experts(s: Spec) -> float:
    """Expected number of experts with at least one token under uniform routing."""
    return s.E * (1.0 - (1.0 - s.k / s.E) ** s.T)


__all__ = ["Spec", "CONFIGS", "SWEEP_T", "spec", "make_inputs", "bytes_per_expert",
           "expected_touched_experts", "scale_atoms", "F32", "BF16", "E4M3", "E2M1"]
