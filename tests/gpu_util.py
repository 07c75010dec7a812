"""Helpers shared by the GPU parity tests (no arithmetic of the layer here)."""
import numpy as np
import torch

import synthetic

# Tolerance on floating-point outputs: max_i |gpu_i - oracle_i| / max_i |oracle_i|
# per output tensor (the layer's 2e-2 bound on bf16 outputs against the fp32 oracle).
TOL = 2e-2


def rel_err(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def deinterleave_cols(a: np.ndarray) -> np.ndarray:
    """Undo the operand column order 0,4,1,5,2,6,3,7 of every 8-column group."""
    n, c = a.shape
    g = a.reshape(n, c // 8, 8)
    out = np.empty_like(g)
    out[..., [0, 4, 1, 5, 2, 6, 3, 7]] = g
    return out.reshape(n, c)


def layer_to(layer, device):
    return layer.to(device)


def experts_of(layer):
    import expert_ffn_layer_top_b200 as moe

    return moe.Experts.from_layer(layer)


def make(cfg, seed=0, device="cpu", **kw):
    return synthetic.make_layer(cfg, seed, device=device, **kw)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()
