"""Pins for the CPU oracle: each test ties one oracle function to something other
than itself (a hand-worked fixture, a library routine, a closed form, an
invariant or brute force). CPU only."""
import itertools
import math
import os
from collections import OrderedDict

import numpy as np
import pytest
import torch

import oracle
import synthetic
from oracle.lru import CacheFull, LruSim

from conftest import GOLDEN


def _bf16_round_np(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).float().numpy()


# ----------------------------------------------------------------------------- formats


def test_e2m1_matches_hand_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt")) if l.strip() and not l.startswith("#")]
    assert len(rows) == 16
    for code, val in rows:
        got = oracle.e2m1(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_matches_torch_float8_e4m3fn():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mine = np.array([oracle.e4m3(c) for c in range(256)])
    assert np.array_equal(np.isnan(lib), np.isnan(mine))
    ok = ~np.isnan(lib)
    assert np.array_equal(lib[ok], mine[ok])
    assert np.array_equal(np.signbit(lib[ok]), np.signbit(mine[ok]))
    assert oracle.e4m3(0x7E) == 448.0 and oracle.e4m3(0x01) == 2.0 ** -9


def test_e8m0_matches_torch_float8_e8m0fnu():
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    mine = np.array([oracle.e8m0(c) for c in range(256)])
    assert np.isnan(mine[255]) and np.isnan(lib[255])
    assert np.array_equal(lib[:255], mine[:255])


def test_mxfp4_row_hand_worked():
    f = {}
    for l in open(os.path.join(GOLDEN, "mxfp4_row.txt")):
        if l.startswith("#") or not l.strip():
            continue
        key, *vals = l.split()
        f[key] = vals
    w = np.array([int(b, 16) for b in f["bytes"]], np.uint8).reshape(1, 32)
    s = np.array([int(v) for v in f["scales"]], np.uint8).reshape(1, 2)
    want = np.array([float(v) for v in f["values"]], np.float32)
    got = oracle.dequant("mxfp4", w, s, rows=1, K=64)[0]
    assert np.array_equal(got, want)


def test_mxfp4_scale_step_doubles_block_only():
    g = np.random.default_rng(1)
    w = g.integers(0, 256, (4, 64), dtype=np.uint8)
    s = g.integers(100, 140, (4, 4), dtype=np.uint8)
    base = oracle.dequant("mxfp4", w, s, rows=4, K=128)
    s2 = s.copy()
    s2[2, 1] += 1
    bumped = oracle.dequant("mxfp4", w, s2, rows=4, K=128)
    diff = bumped != base
    # only row 2, elements 32..63 may change, and exactly by a factor of two
    assert not diff[:, :32].any() and not diff[:, 64:].any() and not diff[[0, 1, 3]].any()
    assert np.array_equal(bumped[2, 32:64], 2 * base[2, 32:64])


def test_nvfp4_is_code_times_block_scale_times_tensor_scale():
    g = np.random.default_rng(2)
    w = g.integers(0, 256, (3, 16), dtype=np.uint8)          # K = 32
    s = g.integers(0x20, 0x70, (3, 2), dtype=np.uint8)        # E4M3 block scales
    t = np.float32(0.37)
    got = oracle.dequant("nvfp4", w, s, tscale=float(t), rows=3, K=32)
    tab = {int(c): float(v) for c, v in (l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt"))
                                        if l.strip() and not l.startswith("#"))}
    sc = torch.from_numpy(s).view(torch.float8_e4m3fn).float().numpy()
    for r in range(3):
        for c in range(32):
            b = int(w[r, c // 2])
            code = (b >> 4) if c & 1 else (b & 15)
            want = np.float32(np.float32(tab[code]) * sc[r, c // 16]) * t
            assert got[r, c] == want


def test_fp8_is_code_times_row_block_scale():
    g = np.random.default_rng(3)
    w = g.integers(0, 0x7E, (2, 256), dtype=np.uint8)
    s = g.random((2, 2), dtype=np.float32) + 0.5
    got = oracle.dequant("fp8", w, s, rows=2, K=256)
    lib = torch.from_numpy(w).view(torch.float8_e4m3fn).float().numpy()
    want = lib * np.repeat(s, 128, axis=1)
    assert np.array_equal(got, want.astype(np.float32))


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is half-way between bf16 1.0 and 1+2^-7: ties to even -> 1.0
    assert oracle.bf16_round(1.0 + 2 ** -8) == 1.0
    assert oracle.bf16_round(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6
    x = np.random.default_rng(4).standard_normal(1000).astype(np.float32)
    assert np.array_equal(np.array([oracle.bf16_round(float(v)) for v in x], np.float32), _bf16_round_np(x))


# ----------------------------------------------------------------------------- router


def _tiny_inputs(seed=0, T=16):
    L = synthetic.make_layer("tiny", seed)
    x = synthetic.make_tokens(T, L.H, seed)
    return L, x


def test_router_logits_equal_fp64_matmul_rounded_once():
    L, x = _tiny_inputs()
    _, _, logits = oracle.route(x, L.wr, L.k)
    ref = (x.double().numpy() @ L.wr.double().numpy()).astype(np.float32)
    assert np.array_equal(logits, ref)
    # bf16 router weights
    wr = L.wr.to(torch.bfloat16)
    _, _, lg2 = oracle.route(x, wr, L.k)
    assert np.array_equal(lg2, (x.double().numpy() @ wr.double().numpy()).astype(np.float32))


def test_router_bias_is_one_fp32_add():
    L, x = _tiny_inputs()
    b = torch.linspace(-1, 1, L.E)
    _, _, lg = oracle.route(x, L.wr, L.k, bias=b)
    _, _, lg0 = oracle.route(x, L.wr, L.k)
    assert np.array_equal(lg, (lg0 + b.numpy()).astype(np.float32))


def test_topk_matches_lexsort_and_brute_force():
    L, x = _tiny_inputs(T=32)
    for k in (1, 2, 3, 8):
        idx, w, lg = oracle.route(x, L.wr, k)
        for t in range(lg.shape[0]):
            order = np.lexsort((np.arange(L.E), -lg[t]))   # logit desc, then index asc
            assert list(idx[t]) == list(order[:k])
        # brute force over all k-subsets (E=8): the chosen set maximises the
        # sorted logit vector lexicographically
        for t in range(4):
            best = max(itertools.combinations(range(L.E), k),
                       key=lambda s: (sorted((lg[t][e] for e in s), reverse=True), [-e for e in sorted(s)]))
            assert sorted(idx[t]) == sorted(best)


def test_topk_ties_go_to_lower_index():
    L, x = _tiny_inputs()
    wr = L.wr.clone()
    wr[:, 5] = wr[:, 2]          # experts 2 and 5 have equal logits for every token
    wr[:, 6] = wr[:, 2]
    idx, w, lg = oracle.route(x, wr, 8)
    for t in range(idx.shape[0]):
        pos = {int(e): j for j, e in enumerate(idx[t])}
        assert pos[2] < pos[5] < pos[6] and pos[6] == pos[5] + 1 and pos[5] == pos[2] + 1
    # all-equal logits: indices 0..k-1 with weight 1/k
    idx, w, _ = oracle.route(x, torch.zeros_like(L.wr), 3)
    assert (idx == np.arange(3)).all() and np.allclose(w, 1 / 3, atol=1e-7)


def test_gating_closed_form():
    L, x = _tiny_inputs(T=32)
    idx, w, lg = oracle.route(x, L.wr, 4)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    for t in range(idx.shape[0]):
        sel = lg[t][idx[t]].astype(np.float64)
        ratio = w[t][1:] / w[t][0]
        assert np.allclose(ratio, np.exp(sel[1:] - sel[0]), rtol=1e-5)
        assert (np.diff(w[t]) <= 0).all()
    _, w1, _ = oracle.route(x, L.wr, 1)
    assert (w1 == 1.0).all()


# ----------------------------------------------------------------------------- permutation


@pytest.mark.parametrize("T,k,E", [(16, 2, 8), (1, 8, 128), (64, 8, 128), (333, 6, 256)])
def test_permutation_is_stable_counting_sort(T, k, E):
    g = np.random.default_rng(T * 7 + k)
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    off, sp, pr = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    assert np.array_equal(sp, np.argsort(flat, kind="stable"))
    assert np.array_equal(np.sort(sp), np.arange(T * k))          # bijection
    assert np.array_equal(pr[sp], np.arange(T * k))               # inverse
    assert np.array_equal(np.diff(off), np.bincount(flat, minlength=E)) and off[0] == 0 and off[-1] == T * k


def test_permutation_empty_batch():
    off, sp, pr = oracle.permute(np.zeros((0, 4), np.int32), 16)
    assert (off == 0).all() and sp.size == 0 and pr.size == 0


# ----------------------------------------------------------------------------- FFN / combine


def test_ffn_single_expert_is_dense_swiglu_mlp():
    """k = E = 1: the layer is a dense SwiGLU MLP (numpy matmul + torch bf16 cast)."""
    cfg = dict(H=64, E=1, k=1, I=96, fmt="bf16", wr_fp32=True)
    L = synthetic.make_layer(cfg, 5)
    x = synthetic.make_tokens(7, 64, 5)
    r = oracle.layer_forward(x, L)
    xf = x.float().numpy().astype(np.float64)
    w13 = L.w13[0].float().numpy().astype(np.float64)
    w2 = L.w2[0].float().numpy().astype(np.float64)
    g, u = xf @ w13[:96].T, xf @ w13[96:].T
    h = _bf16_round_np(g / (1 + np.exp(-g)) * u).astype(np.float64)
    want = h @ w2.T
    assert (r["idx"] == 0).all() and (r["w"] == 1).all()
    assert np.abs(r["out"] - want).max() <= 1e-4 * np.abs(want).max()


def test_ffn_w2_power_of_two_scaling_is_exact():
    L = synthetic.make_layer(dict(H=64, E=4, k=2, I=64, fmt="mxfp4"), 6)
    x = synthetic.make_tokens(9, 64, 6)
    r1 = oracle.layer_forward(x, L)
    L.w2_scale = L.w2_scale + 1                       # every w2 weight doubles
    r2 = oracle.layer_forward(x, L)
    assert np.array_equal(r2["y_perm"], 2 * r1["y_perm"])


def test_ffn_zero_expert_contributes_nothing():
    L, x = _tiny_inputs()
    r = oracle.layer_forward(x, L)
    e0 = int(r["idx"][0, 0])
    L.w2[e0] = 0
    r2 = oracle.layer_forward(x, L)
    rows = r2["sorted_pair"][r2["offsets"][e0]:r2["offsets"][e0 + 1]]
    assert (r2["y_perm"][r2["offsets"][e0]:r2["offsets"][e0 + 1]] == 0).all() and len(rows) > 0


def test_combine_one_hot_and_linear():
    g = np.random.default_rng(8)
    T, k, H = 5, 3, 16
    y = g.standard_normal((T * k, H)).astype(np.float32)
    pr = g.permutation(T * k).astype(np.int32)
    w = np.zeros((T, k), np.float32)
    w[:, 1] = 1
    out = oracle.combine(y, pr, w, T, k)
    assert np.array_equal(out, y[pr.reshape(T, k)[:, 1]])
    w2 = g.random((T, k)).astype(np.float32)
    out2 = oracle.combine(y, pr, w2, T, k)
    want = np.einsum("tj,tjh->th", w2.astype(np.float64), y[pr.reshape(T, k)].astype(np.float64))
    assert np.allclose(out2, want, rtol=1e-6, atol=1e-6)


def test_layer_matches_per_token_brute_force_fp64():
    """Tiny layer: permute/FFN/combine plumbing against an fp64 per-token evaluation."""
    L, x = _tiny_inputs()
    r = oracle.layer_forward(x, L)
    xf = x.double().numpy()
    out = np.zeros_like(xf)
    w13 = L.w13.double().numpy()
    w2 = L.w2.double().numpy()
    for t in range(xf.shape[0]):
        for j in range(L.k):
            e = r["idx"][t, j]
            g = w13[e, :L.I] @ xf[t]
            u = w13[e, L.I:] @ xf[t]
            h = _bf16_round_np(g / (1 + np.exp(-g)) * u).astype(np.float64)
            out[t] += r["w"][t, j] * (w2[e] @ h)
    assert np.abs(r["out"] - out).max() <= 1e-3 * np.abs(out).max()


def _e2m1_table():
    return {int(c): float(v) for c, v in (l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt"))
                                          if l.strip() and not l.startswith("#"))}


def _decode_np(fmt, codes, scale, tscale):
    """Independent fp64 decode of one expert tensor [R, K] (codes as stored, NumPy and torch only)."""
    codes = codes.numpy()
    if fmt == "fp8":
        q = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
        return q * np.repeat(scale.double().numpy(), 128, axis=1)
    tab = _e2m1_table()
    lo, hi = codes & 15, codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)     # low nibble = lower K index
    q = np.vectorize(tab.get)(nib).astype(np.float64)
    if fmt == "mxfp4":
        return q * np.repeat(np.exp2(scale.numpy().astype(np.float64) - 127), 32, axis=1)
    sb = torch.from_numpy(scale.numpy()).view(torch.float8_e4m3fn).double().numpy()
    return q * np.repeat(sb, 16, axis=1) * float(tscale)


@pytest.mark.parametrize("fmt", ["fp8", "mxfp4", "nvfp4"])
def test_quantised_layer_matches_per_token_brute_force_fp64(fmt):
    """Per-expert scale planes, strides and tensor scales of the quantised formats, against an fp64
    per-token evaluation that decodes every expert independently of the oracle's decoder."""
    H, I, E, k = 128, 128, 4, 2
    L = synthetic.make_layer(dict(H=H, E=E, k=k, I=I, fmt=fmt), 11)
    x = synthetic.make_tokens(6, H, 11)
    r = oracle.layer_forward(x, L)
    xf = x.double().numpy()
    w13 = [_decode_np(fmt, L.w13[e], None if L.w13_scale is None else L.w13_scale[e],
                      None if L.w13_tscale is None else L.w13_tscale[e]) for e in range(E)]
    w2 = [_decode_np(fmt, L.w2[e], None if L.w2_scale is None else L.w2_scale[e],
                     None if L.w2_tscale is None else L.w2_tscale[e]) for e in range(E)]
    out = np.zeros_like(xf)
    for t in range(xf.shape[0]):
        for j in range(k):
            e = r["idx"][t, j]
            g = w13[e][:I] @ xf[t]
            u = w13[e][I:] @ xf[t]
            h = _bf16_round_np(g / (1 + np.exp(-g)) * u).astype(np.float64)
            out[t] += r["w"][t, j] * (w2[e] @ h)
    assert len(set(r["idx"].ravel().tolist())) > 1           # several experts, so strides matter
    assert np.abs(r["out"] - out).max() <= 1e-3 * np.abs(out).max()


def test_token_rows_agree_with_layer():
    L = synthetic.make_layer(dict(H=128, E=16, k=4, I=64, fmt="nvfp4"), 9)
    x = synthetic.make_tokens(20, 128, 9)
    r = oracle.layer_forward(x, L)
    rows = oracle.token_rows(x, L, r["idx"], r["w"], [0, 7, 19])
    assert np.array_equal(rows, r["out"][[0, 7, 19]])


# ----------------------------------------------------------------------------- LRU cache simulation


def test_lru_hand_worked_trace():
    s = LruSim(3, 2, 4, 100)
    for line in open(os.path.join(GOLDEN, "lru_trace.txt")):
        if line.startswith("#") or not line.strip():
            continue
        lhs, rhs = line.split("->")
        op, layer, ids = lhs.split()
        ids = [int(i) for i in ids.split(",")]
        if rhs.strip() == "FULL":
            before = s.table()
            with pytest.raises(CacheFull):
                getattr(s, op)(int(layer), ids)
            assert s.table() == before
            continue
        loads_s, counts = rhs.split("|")
        want = [tuple(int(v) for v in p.split(":")) for p in loads_s.split()]
        assert getattr(s, op)(int(layer), ids) == want
        assert (s.hits, s.misses) == tuple(int(v) for v in counts.split())


def test_lru_ids_resolved_once_in_ascending_order():
    """Hand-worked: 4 free slots, one call asking for 5, 2, 7, 2. The ids are
    taken once each in ascending order, so 2, 5, 7 land in slots 0, 1, 2 and
    the call counts three misses. A second call asking for 6, 5 with slot 3
    free: 5 hits, 6 takes slot 3."""
    s = LruSim(4, 1, 8, 1)
    assert s.resolve(0, [5, 2, 7, 2]) == [(2, 0), (5, 1), (7, 2)]
    assert (s.hits, s.misses, s.loads) == (0, 3, 3)
    assert s.resolve(0, [6, 5]) == [(6, 3)]
    assert (s.hits, s.misses, s.loads) == (1, 4, 4)


def test_lru_evict_hand_worked():
    """Hand-worked: 4 slots, 2 layers of 8 experts. Freed slots are taken
    again lowest first; evict(layer, ids) frees only those experts of that
    layer, evict(layer) all of the layer, evict() everything."""
    s = LruSim(4, 2, 8, 1)
    assert s.resolve(0, [1, 2]) == [(1, 0), (2, 1)]
    assert s.resolve(1, [3]) == [(3, 2)]
    s.evict(0, [2])
    assert s.table()[0 * 8 + 2] == -1 and s.table()[0 * 8 + 1] == 0 and s.table()[1 * 8 + 3] == 2
    assert s.resolve(1, [5, 6]) == [(5, 1), (6, 3)]
    s.evict(1)
    assert [v for v in s.table() if v >= 0] == [0]          # only layer 0 expert 1, in slot 0
    assert s.resolve(0, [7]) == [(7, 1)]
    s.evict()
    assert all(v == -1 for v in s.table())
    assert s.resolve(1, [0]) == [(0, 0)]


def test_lru_single_request_calls_equal_textbook_lru():
    """With one id per call the protection rule only shields the MRU slot,
    which textbook LRU never evicts: the two must agree exactly."""
    g = np.random.default_rng(11)
    S = 7
    sim = LruSim(S, 1, 20, 1)
    ref = OrderedDict()
    for _ in range(2000):
        e = int(g.zipf(1.3) % 20)
        loads = sim.resolve(0, [e])
        if e in ref:
            ref.move_to_end(e)
            assert loads == []
        else:
            if len(ref) == S:
                ref.popitem(last=False)
            ref[e] = True
            assert len(loads) == 1
        assert set(ref) == {k[1] for k in sim.slot_of}


def test_lru_large_cache_never_evicts():
    sim = LruSim(1000, 4, 16, 1)
    g = np.random.default_rng(12)
    seen = set()
    for step in range(50):
        for l in range(4):
            ids = g.choice(16, 5, replace=False)
            sim.resolve(l, ids)
            seen |= {(l, int(e)) for e in ids}
    assert sim.misses == len(seen) and sim.loads == len(seen)


# ----------------------------------------------------------------------------- activation format A4


def test_e2m1_encode_ties_saturation_and_identity():
    """The A4 rounding of activations: nearest E2M1 value, ties to the even code (the
    hand-worked cases 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4), magnitudes
    beyond 6 clamp to 6, and every representable value maps to its own code."""
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, -0.75: 10, -5.0: 14}
    for v, c in ties.items():
        assert oracle.e2m1_encode(v) == c, v
    for v in (6.5, 7.0, 100.0, 1e30):
        assert oracle.e2m1_encode(v) == 7 and oracle.e2m1_encode(-v) == 15
    tab = _e2m1_table()
    for c, v in tab.items():
        if v != 0.0:
            assert oracle.e2m1_encode(v) == c
    assert oracle.e2m1_encode(0.24) == 0 and oracle.e2m1_encode(0.26) == 1


def test_e4m3_encode_matches_torch_rounding():
    """E4M3 round-to-nearest-even of scale values against torch's float8_e4m3fn cast on
    random magnitudes and on every exact midpoint between neighbouring values; beyond 448
    the scale saturates."""
    g = np.random.default_rng(5)
    vals = np.concatenate([np.exp2(g.uniform(-12, 8.8, 3000)), g.uniform(0, 448, 1000)]).astype(np.float32)
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids[(mids.astype(np.float64) == (grid[1:] + grid[:-1]) / 2)]])
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals])
    assert np.array_equal(got, want)
    for v in (448.0, 449.0, 463.9, 1e6):
        assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_encode(0.0) == 0


def test_a4_tensor_scale_is_amax_over_6_times_448():
    x = synthetic.make_tokens(5, 64, 3)
    amax = float(x.float().abs().max())
    assert oracle.a4_tensor_scale(x) == float(np.float32(amax) / np.float32(2688.0))
    assert oracle.a4_tensor_scale(torch.zeros(3, 16, dtype=torch.bfloat16)) == 1.0


def test_a4_blocks_hand_worked():
    for line in open(os.path.join(GOLDEN, "a4_blocks.txt")):
        if line.startswith("#") or not line.strip():
            continue
        sg, v, sc, codes, vals = [p.split() for p in line.split("|")]
        out, c, s = oracle.a4_quant(np.array([[float(t) for t in v]], np.float32), float(sg[0]))
        assert s[0, 0] == int(sc[0]), line
        assert c[0].tolist() == [int(t) for t in codes], line
        assert out[0].tolist() == [float(t) for t in vals], line


def test_a4_round_trip_of_representable_values_is_the_identity():
    """Blocks built as q * s_b * s_g from E2M1 values q (largest 6) and power-of-two scales
    come back unchanged."""
    g = np.random.default_rng(6)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    for s_g in (1.0, 2.0 ** -10, 2.0 ** 3):
        q = mags[g.integers(0, 8, (8, 64))] * np.where(g.random((8, 64)) < 0.5, -1, 1).astype(np.float32)
        q[:, ::16] = 6.0
        sb = np.exp2(g.integers(-6, 8, (8, 4))).astype(np.float32)
        v = (q.reshape(8, 4, 16) * sb[..., None] * np.float32(s_g)).reshape(8, 64).astype(np.float32)
        out, _, _ = oracle.a4_quant(v, s_g)
        assert np.array_equal(out, v)


def _a4_np(v, s_g):
    """Independent A4 form of fp32 rows v[n, K]: torch's float8_e4m3fn cast for the scales
    and the input generator's E2M1 encoder for the codes."""
    v = np.asarray(v, np.float32)
    n, K = v.shape
    b = v.reshape(n, K // 16, 16)
    amax = np.abs(b).max(-1).astype(np.float32)
    t = ((amax / np.float32(6.0)) / np.float32(s_g)).astype(np.float32)
    sb = torch.from_numpy(np.minimum(t, np.float32(448.0))).to(torch.float8_e4m3fn).float().numpy()
    den = (sb * np.float32(s_g)).astype(np.float32)
    arg = np.where(den[..., None] > 0, b / np.where(den > 0, den, 1)[..., None], 0).astype(np.float32)
    codes = synthetic.gen._e2m1_encode(torch.from_numpy(arg)).numpy()
    tab = _e2m1_table()
    q = np.vectorize(tab.get)(codes).astype(np.float32)
    return ((q * sb[..., None]).astype(np.float32) * np.float32(s_g)).astype(np.float32).reshape(n, K)


def test_a4_layer_matches_per_token_brute_force():
    """NVFP4 layer in the A4 activation form against an fp64 per-token evaluation whose
    decoder and quantiser are written independently: x quantised with the batch's tensor
    scale, h (computed, then rounded to fp32) quantised with tensor scale 1."""
    H, I, E, k = 128, 64, 4, 2
    L = synthetic.make_layer(dict(H=H, E=E, k=k, I=I, fmt="nvfp4"), 13)
    x = synthetic.make_tokens(6, H, 13)
    r = oracle.layer_forward(x, L, act="a4")
    s_g = np.float32(float(x.float().abs().max())) / np.float32(2688.0)
    xq = _a4_np(x.float().numpy(), s_g).astype(np.float64)
    w13 = [_decode_np("nvfp4", L.w13[e], L.w13_scale[e], L.w13_tscale[e]) for e in range(E)]
    w2 = [_decode_np("nvfp4", L.w2[e], L.w2_scale[e], L.w2_tscale[e]) for e in range(E)]
    out = np.zeros((6, H))
    for t in range(6):
        for j in range(k):
            e = r["idx"][t, j]
            g = w13[e][:I] @ xq[t]
            u = w13[e][I:] @ xq[t]
            h = _a4_np((g / (1 + np.exp(-g)) * u).astype(np.float32)[None], 1.0)[0].astype(np.float64)
            out[t] += r["w"][t, j] * (w2[e] @ h)
    assert np.abs(r["out"] - out).max() <= 1e-3 * np.abs(out).max()
    # the token-row path agrees with the layer path (the tensor scale comes from the whole batch)
    rows = oracle.token_rows(x, L, r["idx"], r["w"], [1, 5], act="a4")
    assert np.array_equal(rows, r["out"][[1, 5]])


def test_a4_changes_the_layer_by_the_quantisation_error():
    """The A4 form is a different computation from A16: on an NVFP4 layer the two differ
    by a few percent (FP4 activations), not by rounding noise, and not by more than 25%."""
    L = synthetic.make_layer(dict(H=256, E=8, k=2, I=256, fmt="nvfp4"), 14)
    x = synthetic.make_tokens(16, 256, 14)
    a16 = oracle.layer_forward(x, L)["out"]
    a4 = oracle.layer_forward(x, L, act="a4")["out"]
    d = np.abs(a4 - a16).max() / np.abs(a16).max()
    assert 5e-3 < d < 0.25, d


def test_lru_resize_by_hand():
    """4 slots hold (0,0) (0,1) (0,2) (0,3), referenced in that order. Shrinking to 2 keeps
    the two most recent, (0,2) and (0,3), which sit in slots 2 and 3 and move, least recent
    first, to the free slots 0 and 1. Growing to 3 adds one free slot, which the next miss
    takes; shrinking to 1 keeps the most recent expert only."""
    sim = LruSim(4, 1, 8, 1)
    for e in range(4):
        sim.resolve(0, [e])
    assert sim.resize(2) == [(2, 0), (3, 1)]
    assert sim.table()[:4] == [-1, -1, 0, 1]
    assert sim.resize(3) == []
    assert sim.resolve(0, [5]) == [(5, 2)]
    assert sim.resize(1) == [(2, 0)]
    assert sim.table()[5] == 0 and sum(v >= 0 for v in sim.table()) == 1


def test_lru_prediction_ranks_by_pair_count_by_hand():
    """Experts 4 (three pairs), 1 (two), 6 and 2 (one each): depth 2 takes 4 and 1, depth 3
    adds 2 (ties to the lower id); the whole layer is every expert."""
    sim = LruSim(16, 2, 8, 1)
    sim.resolve(1, [4, 1, 6, 4, 2, 1, 4])
    assert sim.predict(1, 2) == [1, 4]
    assert sim.predict(1, 3) == [1, 2, 4]
    assert sim.predict(1, -1) == [1, 2, 4, 6]
    assert sim.predict(1, 0, full=True) == list(range(8))
