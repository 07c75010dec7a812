"""The prepacked (TILED) layouts, bit for bit: moe_prepack's output against the
byte arrangement that include/moe.h states, rebuilt here in NumPy from the
standard-layout inputs. Prepacking is a byte permutation, so every byte must
match."""
import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import expert_ffn_layer_top_b200 as m

    return m


def _tile_rows(which: int, H: int, I: int, m: int) -> np.ndarray:
    """Standard-layout rows of M tile m: gate/up (w13) 64 gate rows then the 64
    matching up rows; down (w2) 128 consecutive rows."""
    r = np.arange(128)
    if which == 0:
        return np.where(r < 64, m * 64 + r, I + m * 64 + (r - 64))
    return m * 128 + r


def _fp4_blobs(codes: np.ndarray, scales: np.ndarray, which: int, H: int, I: int, sblock: int) -> np.ndarray:
    """Expected prepacked bytes of one expert, FP4 formats: per (M tile, 256-wide
    K stage) 128 rows x 128 bytes of codes with chunk c of row r at
    r*128 + (c XOR r%8)*16, then 512-byte atoms, scale of row r and block j of
    the atom's K range at (r%32)*16 + (r/32)*4 + j."""
    K = H if which == 0 else I
    m_tiles = I // 64 if which == 0 else H // 128
    kst = K // 256
    natoms = 256 // (4 * sblock)            # atoms per stage: 4 scales per row each
    blob = 128 * 128 + 512 * natoms
    out = np.zeros(m_tiles * kst * blob, np.uint8)
    r = np.arange(128)
    for m in range(m_tiles):
        rows = _tile_rows(which, H, I, m)
        for st in range(kst):
            b = out[(m * kst + st) * blob:(m * kst + st + 1) * blob]
            src = codes[rows, st * 128:(st + 1) * 128]        # [128][128] packed bytes
            for c in range(8):
                pos = r * 128 + ((c ^ (r & 7)) << 4)
                for i in range(16):
                    b[pos + i] = src[:, c * 16 + i]
            for a in range(natoms):
                for j in range(4):
                    sidx = (st * 256 + a * 4 * sblock) // sblock + j
                    b[128 * 128 + a * 512 + (r % 32) * 16 + (r // 32) * 4 + j] = scales[rows, sidx]
    return out


@pytest.mark.parametrize("fmt,sblock", [("mxfp4", 32), ("nvfp4", 16)])
def test_prepacked_fp4_blobs_match_the_stated_layout(moe, fmt, sblock):
    cfg = dict(H=512, E=2, k=2, I=256, fmt=fmt, wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=3)
    ex = moe.moe_prepack(moe.Experts.from_layer(L.to("cuda")))
    torch.cuda.synchronize()
    got13 = ex.w13.cpu().numpy().reshape(L.E, -1)
    got2 = ex.w2.cpu().numpy().reshape(L.E, -1)
    w13 = L.w13.contiguous().view(torch.uint8).numpy().reshape(L.E, 2 * L.I, L.H // 2)
    w2 = L.w2.contiguous().view(torch.uint8).numpy().reshape(L.E, L.H, L.I // 2)
    s13 = L.w13_scale.contiguous().view(torch.uint8).numpy().reshape(L.E, 2 * L.I, L.H // sblock)
    s2 = L.w2_scale.contiguous().view(torch.uint8).numpy().reshape(L.E, L.H, L.I // sblock)
    for e in range(L.E):
        np.testing.assert_array_equal(got13[e], _fp4_blobs(w13[e], s13[e], 0, L.H, L.I, sblock))
        np.testing.assert_array_equal(got2[e], _fp4_blobs(w2[e], s2[e], 1, L.H, L.I, sblock))


def test_prepacked_fp8_chunk_major_layout(moe):
    """FP8: per (M tile, 128-wide K stage) the codes in 16-byte chunk-major order
    (chunk c of row r at (c*128 + r)*16), then each row's fp32 scale of the stage."""
    cfg = dict(H=256, E=2, k=2, I=256, fmt="fp8", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=4)
    ex = moe.moe_prepack(moe.Experts.from_layer(L.to("cuda")))
    torch.cuda.synchronize()
    got = ex.w2.cpu().numpy().reshape(L.E, -1)
    codes = L.w2.contiguous().view(torch.uint8).numpy().reshape(L.E, L.H, L.I)
    scales = L.w2_scale.contiguous().view(torch.uint8).numpy().reshape(L.E, L.H, (L.I // 128) * 4)
    blob = 128 * (128 + 4)
    for e in range(L.E):
        exp = np.zeros(got.shape[1], np.uint8)
        for m in range(L.H // 128):
            rows = np.arange(128) + m * 128
            for kb in range(L.I // 128):
                b = exp[(m * (L.I // 128) + kb) * blob:(m * (L.I // 128) + kb + 1) * blob]
                src = codes[e][rows, kb * 128:(kb + 1) * 128]
                for c in range(8):
                    for i in range(16):
                        b[(c * 128 + np.arange(128)) * 16 + i] = src[:, c * 16 + i]
                b[128 * 128 + np.arange(128)[:, None] * 4 + np.arange(4)] = scales[e][rows, kb * 4:(kb + 1) * 4]
        np.testing.assert_array_equal(got[e], exp)
