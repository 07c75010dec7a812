"""Seeded synthetic MoE-layer inputs.

Shapes and distributions follow the five workloads of the MoE-layer study:
activations x ~ N(0, 1) in bf16, router weights ~ N(0, 0.02), expert weights
drawn from N(0, 0.02) and then encoded into one of four stored formats:

* ``bf16``  - plain bf16, [E, R, K].
* ``fp8``   - E4M3 codes [E, R, K] + one fp32 scale per (row, 128-wide K block).
* ``mxfp4`` - E2M1 codes, two per byte, low nibble = lower K index, [E, R, K/2]
              + one E8M0 scale byte per (row, 32-wide K block).
* ``nvfp4`` - E2M1 codes as above + one E4M3 scale byte per (row, 16-wide K
              block) + one fp32 tensor scale per (expert, tensor).

``w13`` is [E, 2I, H] (gate rows 0..I-1, then up rows I..2I-1) and ``w2`` is
[E, H, I]; in both the reduction dimension K is contiguous.

The encoders here are input preparation (what a checkpoint converter does
offline). Decoding, routing, the FFN and the combine live in the two
implementations under test, never here. Everything is a torch op so the same
code runs on the CPU (small cases) or on the GPU (full-size workloads, where
CPU generation would take minutes). Streams are seeded per (seed, role,
expert); CPU and CUDA generators are different streams, so a test that needs
both sides to see one input generates it once and copies it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, Optional

import torch

WFMT = {"bf16": 0, "fp8": 1, "mxfp4": 2, "nvfp4": 3}

# Workload table: the five MoE-layer configurations (sizes, formats, skew).
CONFIGS: Dict[str, dict] = {
    "tiny": dict(H=256, E=8, k=2, I=512, fmt="bf16", wr_fp32=True, zipf=None, T=(16,), y_fp32=False),
    "decode": dict(H=2048, E=128, k=8, I=768, fmt="mxfp4", wr_fp32=False, zipf=None, T=(1, 8, 64), y_fp32=False),
    "prefill": dict(H=2048, E=128, k=8, I=768, fmt="nvfp4", wr_fp32=False, zipf=1.1, T=(4096,), y_fp32=False),
    "large": dict(H=4096, E=256, k=6, I=2048, fmt="nvfp4", wr_fp32=False, zipf=1.0, T=(32, 8192), y_fp32=True),
    "stack": dict(H=2048, E=128, k=8, I=768, fmt="fp8", wr_fp32=False, zipf=1.2, T=(4,), y_fp32=False,
                  layers=43, steps=512, drift_every=128, cache_bytes=24 * 10**9),
}

_ROLE = {"wr": 1, "w13": 2, "w2": 3, "x": 4, "perm": 5, "bias": 6}


def _gen(seed: int, role: str, sub: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + _ROLE[role] * 100_003 + sub * 7) & 0x7FFF_FFFF_FFFF)
    return g


# --------------------------------------------------------------------------------------------
# encoders (input preparation only)
# --------------------------------------------------------------------------------------------

# E2M1 magnitudes in code order 0..7 and the midpoints between neighbours.
_E2M1_MAG = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _e2m1_encode(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code (ties to the even mantissa), saturating at 6. Returns uint8 codes 0..15."""
    a = v.abs()
    # code boundaries; at an exact tie the code with mantissa bit 0 wins
    code = torch.zeros_like(a, dtype=torch.uint8)
    code = torch.where(a > 0.25, torch.full_like(code, 1), code)
    code = torch.where(a >= 0.75, torch.full_like(code, 2), code)
    code = torch.where(a > 1.25, torch.full_like(code, 3), code)
    code = torch.where(a >= 1.75, torch.full_like(code, 4), code)
    code = torch.where(a > 2.5, torch.full_like(code, 5), code)
    code = torch.where(a >= 3.5, torch.full_like(code, 6), code)
    code = torch.where(a > 5.0, torch.full_like(code, 7), code)
    sign = (v < 0).to(torch.uint8) << 3
    return code | sign


def _pack_nibbles(codes: torch.Tensor) -> torch.Tensor:
    lo = codes[..., 0::2]
    hi = codes[..., 1::2]
    return (lo | (hi << 4)).to(torch.uint8)


def _e4m3_encode(v: torch.Tensor) -> torch.Tensor:
    return v.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)


def quantise(w: torch.Tensor, fmt: str, tscale: Optional[torch.Tensor] = None):
    """Encode fp32 weights [..., R, K] into ``fmt``. Returns (codes, scales, tscale)."""
    K = w.shape[-1]
    if fmt == "bf16":
        return w.to(torch.bfloat16), None, None
    if fmt == "fp8":
        assert K % 128 == 0
        blk = w.reshape(*w.shape[:-1], K // 128, 128)
        amax = blk.abs().amax(-1)
        scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).float()
        q = _e4m3_encode(blk / scale.unsqueeze(-1)).reshape(w.shape)
        return q, scale, None
    if fmt == "mxfp4":
        assert K % 32 == 0
        blk = w.reshape(*w.shape[:-1], K // 32, 32)
        amax = blk.abs().amax(-1)
        # shared exponent: floor(log2 amax) - 2 (the largest E2M1 exponent), E8M0 biased by 127
        e = torch.where(amax > 0, torch.floor(torch.log2(amax.clamp_min(1e-38))) - 2, torch.full_like(amax, -127))
        e = e.clamp(-127, 127)
        codes = _e2m1_encode(blk / torch.exp2(e).unsqueeze(-1)).reshape(w.shape)
        return _pack_nibbles(codes), (e + 127).to(torch.uint8), None
    if fmt == "nvfp4":
        assert K % 16 == 0
        if tscale is None:
            tscale = (w.abs().amax() / (448.0 * 6.0)).clamp_min(1e-30).float().reshape(1)
        blk = w.reshape(*w.shape[:-1], K // 16, 16)
        amax = blk.abs().amax(-1)
        sb = _e4m3_encode(amax / 6.0 / tscale)
        sbf = sb.view(torch.float8_e4m3fn).float()
        denom = torch.where(sbf > 0, sbf * tscale, torch.ones_like(sbf))
        codes = _e2m1_encode(blk / denom.unsqueeze(-1)).reshape(w.shape)
        return _pack_nibbles(codes), sb, tscale
    raise ValueError(fmt)


def expert_bytes(fmt: str, H: int, I: int) -> int:
    """Stored bytes of one expert (w13 + w2 with scales) in ``fmt``."""
    n = 3 * H * I
    if fmt == "bf16":
        return 2 * n
    if fmt == "fp8":
        return n + 4 * (n // 128)
    if fmt == "mxfp4":
        return n // 2 + n // 32
    if fmt == "nvfp4":
        return n // 2 + n // 16 + 8
    raise ValueError(fmt)


# --------------------------------------------------------------------------------------------
# layers
# --------------------------------------------------------------------------------------------


@dataclass
class LayerInputs:
    """One MoE layer's parameters in stored form (all tensors on one device)."""

    fmt: str
    H: int
    E: int
    I: int
    k: int
    wr: torch.Tensor                      # [H, E] fp32 or bf16
    w13: torch.Tensor                     # codes [E, 2I, H] or packed [E, 2I, H/2]
    w2: torch.Tensor                      # codes [E, H, I] or packed [E, H, I/2]
    w13_scale: Optional[torch.Tensor] = None
    w2_scale: Optional[torch.Tensor] = None
    w13_tscale: Optional[torch.Tensor] = None   # [E] fp32 (nvfp4)
    w2_tscale: Optional[torch.Tensor] = None
    bias: Optional[torch.Tensor] = None         # [E] fp32 routing skew
    extra: dict = field(default_factory=dict)

    def to(self, device) -> "LayerInputs":
        kw = {}
        for name in ("wr", "w13", "w2", "w13_scale", "w2_scale", "w13_tscale", "w2_tscale", "bias"):
            t = getattr(self, name)
            kw[name] = None if t is None else t.to(device)
        return LayerInputs(self.fmt, self.H, self.E, self.I, self.k, extra=dict(self.extra), **kw)


def zipf_bias(E: int, s: float, H: int, seed: int, device="cpu", perm: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Routing skew: b[e] = (sigma_l / (pi/sqrt 6)) * ln p_e with p_e ~ 1/(perm[e]+1)^s.

    sigma_l = 0.02*sqrt(H) is the spread of x.Wr for x ~ N(0,1), Wr ~ N(0,0.02);
    pi/sqrt(6) is the spread of a standard Gumbel variable, so adding b to the
    logits approximates drawing experts without replacement with probability p
    (Gumbel-top-k; Kool, van Hoof and Welling, 2019).
    """
    if perm is None:
        perm = torch.randperm(E, generator=_gen(seed, "perm", 0, "cpu"))
    rank = perm.double() + 1.0
    p = rank.pow(-s)
    p = p / p.sum()
    sigma_l = 0.02 * math.sqrt(H)
    b = (sigma_l / (math.pi / math.sqrt(6.0))) * torch.log(p)
    return b.float().to(device)


def make_tokens(T: int, H: int, seed: int, device="cpu", sub: int = 0) -> torch.Tensor:
    g = _gen(seed, "x", sub, device)
    return torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)


def make_router(cfg: str | dict, seed: int = 0, device="cpu", layer: int = 0):
    """(wr, bias) of one layer, identical to the ones make_layer draws for the same arguments."""
    c = dict(CONFIGS[cfg]) if isinstance(cfg, str) else dict(cfg)
    H, E_ = c["H"], c["E"]
    wr = torch.randn(H, E_, generator=_gen(seed, "wr", layer * 4096, device), device=device) * 0.02
    wr = wr.float() if c.get("wr_fp32") else wr.to(torch.bfloat16)
    bias = zipf_bias(E_, c["zipf"], H, seed + 7919 * layer, device) if c.get("zipf") else None
    return wr, bias


def make_layer(cfg: str | dict, seed: int = 0, device="cpu", E: Optional[int] = None,
               fmt: Optional[str] = None, layer: int = 0) -> LayerInputs:
    """All parameters of one layer of workload ``cfg`` (weights drawn N(0, 0.02), then encoded)."""
    c = dict(CONFIGS[cfg]) if isinstance(cfg, str) else dict(cfg)
    if E is not None:
        c["E"] = E
    if fmt is not None:
        c["fmt"] = fmt
    H, E_, I, k, f = c["H"], c["E"], c["I"], c["k"], c["fmt"]
    sub0 = layer * 4096
    wr = torch.randn(H, E_, generator=_gen(seed, "wr", sub0, device), device=device) * 0.02
    wr = wr.float() if c.get("wr_fp32") else wr.to(torch.bfloat16)
    w13s, w2s, s13, s2, t13, t2 = [], [], [], [], [], []
    for e in range(E_):
        a = torch.randn(2 * I, H, generator=_gen(seed, "w13", sub0 + e, device), device=device) * 0.02
        b = torch.randn(H, I, generator=_gen(seed, "w2", sub0 + e, device), device=device) * 0.02
        qa, sa, ta = quantise(a, f)
        qb, sb, tb = quantise(b, f)
        w13s.append(qa); w2s.append(qb)
        s13.append(sa); s2.append(sb); t13.append(ta); t2.append(tb)
        del a, b
    li = LayerInputs(
        f, H, E_, I, k, wr,
        torch.stack(w13s), torch.stack(w2s),
        torch.stack(s13) if s13[0] is not None else None,
        torch.stack(s2) if s2[0] is not None else None,
        torch.cat(t13) if t13[0] is not None else None,
        torch.cat(t2) if t2[0] is not None else None,
    )
    if c.get("zipf"):
        li.bias = zipf_bias(E_, c["zipf"], H, seed + 7919 * layer, device)
    return li
