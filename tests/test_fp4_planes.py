"""The four-plane E2M1 form of activations used by the block-scaled FP4 path,
restated in NumPy and checked against the bounds the design relies on.

A bf16 value x of a block whose largest magnitude has binary exponent e is
carried as sum_p q_p 2^(s - 3p), p = 0..3, with s = e - 1: plane 0 rounds
x 2^-s to E2M1 (nearest, ties to even), each next plane rounds the residual at
a unit 8 times finer. The checks: no plane value leaves [-4, 4] (E2M1 reaches
6, so nothing saturates), and the planes are within 2^(e - 11) of x. For the
NVFP4 variant, the per-row offset C = 9 - E (E: exponent of the row maximum)
keeps every block scale 2^(e - 1 + C) inside E4M3's powers of two 2^-9..2^8
for blocks within 2^17 of the row maximum."""
import numpy as np
import pytest

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_rne(t: np.ndarray) -> np.ndarray:
    """Nearest E2M1 value, ties to the even code (code = index in E2M1)."""
    a = np.abs(t)
    d = np.abs(a[..., None] - E2M1)
    best = d.min(-1, keepdims=True)
    cand = np.isclose(d, best, rtol=0, atol=0)
    # among equally near codes take the even one
    codes = np.where(cand, np.arange(8), 99)
    even = np.where(codes % 2 == 0, codes, 99).min(-1)
    code = np.where(even < 99, even, codes.min(-1))
    return np.sign(t) * E2M1[code]


def bf16(x: np.ndarray) -> np.ndarray:
    u = x.astype(np.float32).view(np.uint32)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.view(np.float32).astype(np.float64)


def planes(block: np.ndarray):
    amax = np.abs(block).max()
    e = int(np.floor(np.log2(amax)))
    s = e - 1
    r = block.copy()
    qs = []
    for p in range(4):
        unit = 2.0 ** (s - 3 * p)
        t = r / unit
        q = e2m1_rne(t)
        qs.append(t)
        r = r - q * unit
    return e, qs, r


@pytest.mark.parametrize("seed", range(4))
def test_four_planes_never_saturate_and_are_within_2_to_the_e_minus_11(seed):
    rng = np.random.default_rng(seed)
    for _ in range(400):
        scale = 2.0 ** rng.integers(-20, 20)
        block = bf16(rng.standard_normal(32) * scale)
        if not np.any(block):
            continue
        e, ts, resid = planes(block)
        for t in ts:
            assert np.all(np.abs(t) <= 4.0)
        assert np.all(np.abs(resid) <= 2.0 ** (e - 11))


def test_worst_cases_at_the_block_maximum():
    # the largest bf16 value below 2^(e+1), and values on rounding ties of plane 0
    for e in (-3, 0, 5):
        top = bf16(np.array([2.0 ** (e + 1) * (1 - 2.0 ** -8)]))[0]
        block = np.array([top, 2.0 ** e * 1.25, 2.0 ** e * 0.75, -(2.0 ** e) * 1.75] + [0.0] * 28)
        block = bf16(block)
        ee, ts, resid = planes(block)
        assert ee == e
        assert all(np.all(np.abs(t) <= 4.0) for t in ts)
        assert np.all(np.abs(resid) <= 2.0 ** (e - 11))


def test_nvfp4_row_offset_keeps_block_scales_in_e4m3_range():
    rng = np.random.default_rng(7)
    for _ in range(200):
        row = bf16(rng.standard_normal(4096) * 2.0 ** rng.integers(-30, 30))
        E = int(np.floor(np.log2(np.abs(row).max())))
        C = 9 - E
        for b in range(0, 4096, 16):
            blk = row[b:b + 16]
            m = np.abs(blk).max()
            if m == 0:
                continue
            e = int(np.floor(np.log2(m)))
            k = e - 1 + C
            assert k <= 8
            if e >= E - 17:
                assert k >= -9
