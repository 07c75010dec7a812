"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs. Integer outputs must match bit-exactly; floating-point
outputs within TOL = 2e-2 of max|oracle| per tensor (tighter where stated)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic
from gpu_util import TOL, bf16_np, deinterleave_cols, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import expert_ffn_layer_top_b200 as m

    return m


def _ulp_close(a, b, ulps=1):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    return np.all(np.abs(a - b) <= ulps * np.spacing(np.maximum(np.abs(a), np.abs(b))))


# ----------------------------------------------------------------------------- decode


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "mxfp4", "nvfp4"])
def test_dequantize_matches_oracle(moe, fmt):
    rows, K = 64, 256
    g = torch.Generator().manual_seed(3)
    t = 1.0
    s = None
    if fmt == "bf16":
        w = torch.randn(rows, K, generator=g).to(torch.bfloat16)
    elif fmt == "mxfp4":
        w = torch.randint(0, 256, (rows, K // 2), dtype=torch.uint8, generator=g)
        # scales spanning subnormal results (small), the common range, and > 2^1 (second multiply)
        s = torch.randint(0, 200, (rows, K // 32), dtype=torch.uint8, generator=g)
        s[0, :4] = torch.tensor([0, 1, 128, 129], dtype=torch.uint8)
    elif fmt == "nvfp4":
        w = torch.randint(0, 256, (rows, K // 2), dtype=torch.uint8, generator=g)
        s = torch.randint(0, 0x7F, (rows, K // 16), dtype=torch.uint8, generator=g)   # incl. 0 and subnormals
        t = 0.37
    else:
        w = torch.randint(0, 256, (rows, K), dtype=torch.uint8, generator=g)
        w[(w & 0x7F) == 0x7F] = 0x7E                                                   # no NaN codes
        s = (torch.rand(rows, K // 128, generator=g) + 0.5) * 1e-3
    got = moe.moe_dequantize(fmt, w.cuda(), None if s is None else s.cuda(), t, rows, K).float().cpu()
    ref = torch.from_numpy(oracle.dequant(fmt, w, s, tscale=t, rows=rows, K=K))
    if fmt == "fp8":
        assert rel_err(got, ref) < 2 ** -7
        assert torch.allclose(got, ref, rtol=2 ** -7, atol=0)
    else:
        # exact: the same binary32 value, rounded once to bf16
        assert torch.equal(got, ref.to(torch.bfloat16).float())


# ----------------------------------------------------------------------------- router


ROUTER_CASES = [("tiny", 16), ("decode", 1), ("decode", 2), ("decode", 8), ("decode", 64), ("decode", 130),
                ("decode", 256), ("decode", 257), ("prefill", 4096), ("large", 32), ("large", 200), ("large", 1000),
                # odd shapes: 40 fp32 experts (one warp holds 64 expert slots), 12 bf16 experts (24-byte
                # rows), H with an odd number of rows per eighth
                (dict(H=512, E=40, k=5, wr_fp32=True, zipf=None), 77),
                (dict(H=1024, E=12, k=3, wr_fp32=False, zipf=None), 50),
                (dict(H=520, E=40, k=4, wr_fp32=False, zipf=None), 9)]


@pytest.mark.parametrize("cfg,T", ROUTER_CASES)
def test_router_parity(moe, cfg, T):
    wr, bias = synthetic.make_router(cfg, seed=1)
    k = (synthetic.CONFIGS[cfg] if isinstance(cfg, str) else cfg)["k"]
    x = synthetic.make_tokens(T, wr.shape[0], seed=1)
    idx_o, w_o, lg_o = oracle.route(x, wr, k, bias=bias)
    idx, w, lg = moe.moe_route_topk(x.cuda(), wr.cuda(), k, bias=None if bias is None else bias.cuda(),
                                    want_logits=True)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert _ulp_close(lg.cpu().numpy(), lg_o, 1)
    assert np.allclose(w.cpu().numpy(), w_o, rtol=0, atol=2e-6)


def test_router_ties_and_equal_logits(moe):
    wr, _ = synthetic.make_router("tiny", seed=2)
    wr = wr.clone()
    wr[:, 5] = wr[:, 2]
    x = synthetic.make_tokens(33, wr.shape[0], seed=2)
    idx_o, w_o, _ = oracle.route(x, wr, 8)
    idx, w = moe.moe_route_topk(x.cuda(), wr.cuda(), 8)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    idx, w = moe.moe_route_topk(x.cuda(), torch.zeros_like(wr).cuda(), 3)
    assert (idx.cpu().numpy() == np.arange(3)).all()
    assert np.allclose(w.cpu().numpy(), 1 / 3, atol=1e-7)


# ----------------------------------------------------------------------------- permutation


def _rand_idx(T, k, E, seed):
    g = np.random.default_rng(seed)
    if T == 0:
        return np.zeros((0, k), np.int32)
    return np.argsort(g.random((T, E)), axis=1)[:, :k].astype(np.int32)


@pytest.mark.parametrize("T,k,E", [(16, 2, 8), (1, 8, 128), (64, 8, 128), (4096, 8, 128), (8192, 6, 256),
                                   (5, 3, 40), (0, 8, 128)])
def test_permute_parity(moe, T, k, E):
    idx = _rand_idx(T, k, E, T + k)
    H = 256
    x = synthetic.make_tokens(max(T, 1), H, seed=3)[:T]
    off_o, sp_o, pr_o = oracle.permute(idx, E)
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), E, x.cuda())
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(sp.cpu().numpy(), sp_o)
    assert np.array_equal(pr.cpu().numpy(), pr_o)
    if T:
        got = deinterleave_cols(xp.view(torch.int16).cpu().numpy())
        want = x.view(torch.int16).numpy()[sp_o // k]
        assert np.array_equal(got, want)


def test_permute_single_expert_takes_everything(moe):
    T, E = 300, 16
    idx = np.full((T, 1), 7, np.int32)
    off, sp, pr, _ = moe.moe_permute(torch.from_numpy(idx).cuda(), E)
    off = off.cpu().numpy()
    assert off[7] == 0 and off[8] == T and off[-1] == T
    assert np.array_equal(sp.cpu().numpy(), np.arange(T))


# ----------------------------------------------------------------------------- combine


@pytest.mark.parametrize("y_fp32", [False, True])
def test_combine_parity(moe, y_fp32):
    g = torch.Generator().manual_seed(5)
    T, k, H = 37, 4, 512
    y = torch.randn(T * k, H, generator=g)
    y = y if y_fp32 else y.to(torch.bfloat16)
    pr = torch.randperm(T * k, generator=g).to(torch.int32)
    w = torch.rand(T, k, generator=g)
    ref = oracle.combine(y.float().numpy(), pr.numpy(), w.numpy(), T, k)
    out = moe.moe_combine(y.cuda(), pr.cuda(), w.cuda())
    assert rel_err(bf16_np(out), ref) < 4e-3


# ----------------------------------------------------------------------------- grouped FFN


FFN_CASES = [(fmt, T, tiled) for fmt in ("bf16", "fp8", "mxfp4", "nvfp4") for T in (40, 100, 200, 600)
             for tiled in (False, True)] + [(f, T, True) for f in ("mxfp4", "nvfp4") for T in (24, 9, 3)]


@pytest.mark.parametrize("fmt,T,tiled", FFN_CASES)
def test_grouped_ffn_parity(moe, fmt, T, tiled):
    """T = 40/100/200/600 with E = 8, k = 2 exercises token tiles of 16/32/64/128,
    on row-major weights and on weights prepacked into the tiled layout.
    Prepacked MXFP4 runs the block-scaled FP4 path (token tiles of 8/16/32;
    T = 3, 9 and 24 give ragged tails), and so does prepacked NVFP4 while the
    mean rows per expert (2T / 8 here) is at most 16; larger NVFP4 batches take
    the decoding path, reading the same prepacked blobs. The block-scaled MXFP4
    h never exists in bf16, so there the down-projection output is compared;
    the block-scaled NVFP4 h is written in bf16, natural column order, at the
    start of the workspace."""
    mx = fmt == "mxfp4" and tiled
    nv_bs = fmt == "nvfp4" and tiled and -(-2 * T // 8) <= 16
    cfg = dict(H=256, E=8, k=2, I=256, fmt=fmt, wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=7)
    x = synthetic.make_tokens(T, 256, seed=7)
    idx = _rand_idx(T, 2, 8, T)
    off_o, sp_o, pr_o = oracle.permute(idx, 8)
    y_o, h_o = oracle.ffn(x, L, off_o, sp_o, 2, want_h=True)
    Ld = L.to("cuda")
    ex = moe.Experts.from_layer(Ld)
    if tiled:
        ex = moe.moe_prepack(ex)
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), 8, x.cuda())
    if mx:
        y = moe.moe_grouped_ffn(xp, off, ex)
        torch.cuda.synchronize()
    elif nv_bs:
        ws = torch.empty(moe.moe_workspace_size(T * 2, 256, 256, 8, 1, False), dtype=torch.uint8, device="cuda")
        y = moe.moe_grouped_ffn(xp, off, ex, ws=ws)
        torch.cuda.synchronize()
        h = ws[: T * 2 * 256 * 2].view(torch.bfloat16).view(T * 2, 256)
        assert rel_err(h.float().cpu().numpy(), h_o) < TOL, "gate/up + SwiGLU"
    else:
        ws = torch.empty(T * 2 * 256 * 2 + 256, dtype=torch.uint8, device="cuda")
        y = moe.moe_grouped_ffn(xp, off, ex, ws=ws)
        torch.cuda.synchronize()
        h = ws[: T * 2 * 256 * 2].view(torch.bfloat16).view(T * 2, 256)
        h_got = deinterleave_cols(h.float().cpu().numpy())
        assert rel_err(h_got, h_o) < TOL, "gate/up + SwiGLU"
    err = rel_err(bf16_np(y), y_o)
    assert err < TOL, f"down projection: error {err:.3e}, device error word {moe.moe_device_error()}"
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("fmt,T", [("mxfp4", 40), ("mxfp4", 9), ("nvfp4", 40)])
def test_grouped_ffn_item_parallel_down(moe, fmt, T):
    """I = 768 gives the down projection 3 stages of 256 per item on 3 pipelines;
    there the pipelines take whole items (item-parallel) and the epilogue reads
    one pipeline's accumulators per item."""
    cfg = dict(H=256, E=8, k=2, I=768, fmt=fmt, wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=11)
    x = synthetic.make_tokens(T, 256, seed=11)
    idx = _rand_idx(T, 2, 8, T)
    off_o, sp_o, pr_o = oracle.permute(idx, 8)
    y_o = oracle.ffn(x, L, off_o, sp_o, 2)
    ex = moe.moe_prepack(moe.Experts.from_layer(L.to("cuda")))
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), 8, x.cuda())
    y = moe.moe_grouped_ffn(xp, off, ex)
    torch.cuda.synchronize()
    err = rel_err(bf16_np(y), y_o)
    assert err < TOL, f"down projection: error {err:.3e}"
    assert moe.moe_device_error() == 0


def test_grouped_ffn_fp32_output(moe):
    cfg = dict(H=256, E=8, k=2, I=256, fmt="nvfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=8)
    x = synthetic.make_tokens(50, 256, seed=8)
    idx = _rand_idx(50, 2, 8, 50)
    off_o, sp_o, _ = oracle.permute(idx, 8)
    y_o = oracle.ffn(x, L, off_o, sp_o, 2)
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), 8, x.cuda())
    y = moe.moe_grouped_ffn(xp, off, moe.Experts.from_layer(L.to("cuda")), y_fp32=True)
    assert y.dtype == torch.float32
    assert rel_err(y.cpu().numpy(), y_o) < TOL


# ----------------------------------------------------------------------------- whole layer


def _layer_check(moe, L, x, y_fp32=False, sample=None, tiled=True, act="a16"):
    """Run the layer on the GPU; compare routing bit-exactly and outputs (all or sampled rows)."""
    Ld = L.to("cuda")
    T = x.shape[0]
    idx = torch.empty(T, L.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, L.k, dtype=torch.float32, device="cuda")
    ex = moe.Experts.from_layer(Ld)
    if tiled:
        ex = moe.moe_prepack(ex)
        del Ld.w13, Ld.w2          # keep device memory low for the large layer
    out = moe.moe_layer_forward(x.cuda(), Ld.wr, L.k, ex, bias=Ld.bias, y_fp32=y_fp32, idx_out=idx, w_out=w, act=act)
    torch.cuda.synchronize()
    idx_o, w_o, _ = oracle.route(x, L.wr, L.k, bias=L.bias, with_logits=False)
    assert np.array_equal(idx.cpu().numpy(), idx_o)
    assert np.allclose(w.cpu().numpy(), w_o, atol=2e-6, rtol=0)
    got = bf16_np(out)
    if sample is None:
        ref = oracle.layer_forward(x, L, act=act)["out"]
        err = rel_err(got, ref)
    else:
        ref = oracle.token_rows(x, L, idx_o, w_o, sample, act=act)
        err = rel_err(got[sample], ref)
    assert err < TOL, f"layer output error {err:.3e}"
    assert moe.moe_device_error() == 0
    return err


@pytest.mark.parametrize("tiled", [False, True])
def test_layer_tiny(moe, tiled):
    L = synthetic.make_layer("tiny", 0)
    x = synthetic.make_tokens(16, L.H, 0)
    _layer_check(moe, L, x, tiled=tiled)


@pytest.fixture(scope="module")
def decode_layer():
    return synthetic.make_layer("decode", 0)


@pytest.mark.parametrize("T", [1, 8, 64])
def test_layer_decode_mxfp4(moe, decode_layer, T):
    x = synthetic.make_tokens(T, 2048, seed=10 + T)
    _layer_check(moe, decode_layer, x)


@pytest.mark.parametrize("T,y_fp32", [(1, True), (37, False), (64, True), (256, False)])
def test_layer_decode_mxfp4_combine_in_down(moe, decode_layer, T, y_fp32):
    """Slot layout (the router claims the rows and writes the activation tiles; the combine
    maps slot rows to y rows through UP's count prefix): a ragged batch, the largest batch
    the layout takes, and y kept in fp32, against the oracle."""
    x = synthetic.make_tokens(T, 2048, seed=300 + T)
    _layer_check(moe, decode_layer, x, y_fp32=y_fp32)


def test_layer_top16_slot_layout(moe):
    """k = 16 through the slot layout (H a multiple of 2048): 16 claims per token in the
    router, 16 rows per token in the combine."""
    cfg = dict(H=2048, E=64, k=16, I=256, fmt="mxfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=27)
    _layer_check(moe, L, synthetic.make_tokens(40, 2048, seed=27))


def test_layer_fused_routing_and_permutation(moe, decode_layer):
    """A decode-sized MXFP4 batch takes the slot layout: the router claims each pair's
    row in its expert's slot and writes the activation rows itself, so a layer call is
    4 kernels: router, UP, DOWN, combine. CUDA-graph replays reuse one launch's
    arguments and the slot counts must be back at zero after every call; each replay
    (and a call on another stream, with its own counts) must give the eager result."""
    L = decode_layer.to("cuda")
    ex = moe.moe_prepack(moe.Experts.from_layer(L))
    T = 64
    x = synthetic.make_tokens(T, L.H, seed=77).cuda()
    ws = torch.empty(moe.moe_workspace_size(T, L.H, L.I, L.E, L.k), dtype=torch.uint8, device="cuda")
    out = torch.empty(T, L.H, dtype=torch.bfloat16, device="cuda")
    n0 = moe.moe_kernel_launch_count()
    ref = moe.moe_layer_forward(x, L.wr, L.k, ex, bias=L.bias, ws=ws, out=out).clone()
    assert moe.moe_kernel_launch_count() - n0 == 4
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        moe.moe_layer_forward(x, L.wr, L.k, ex, bias=L.bias, ws=ws, out=out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_forward(x, L.wr, L.k, ex, bias=L.bias, ws=ws, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert moe.moe_device_error() == 0


def test_layer_consecutive_calls_in_one_graph(moe, decode_layer):
    """Several layer calls captured in one CUDA graph, sharing one workspace (each layer's router
    starts its weight loads while the layer before finishes): every replay gives each call's eager
    output bit for bit: decode batches on the slot layout (T = 64 with head tiles, 37 and 1 without)
    and off it (T = 300: separate permutation, quantiser and combine launches)."""
    L = decode_layer.to("cuda")
    ex = [moe.moe_prepack(moe.Experts.from_layer(L)) for _ in range(2)]
    for T in (64, 37, 1, 300):
        xs = [synthetic.make_tokens(T, L.H, seed=700 + 10 * T + i).cuda() for i in range(4)]
        ws = torch.empty(moe.moe_workspace_size(T, L.H, L.I, L.E, L.k), dtype=torch.uint8, device="cuda")
        outs = [torch.empty(T, L.H, dtype=torch.bfloat16, device="cuda") for _ in xs]
        calls = [(xs[i], ex[i % 2], outs[i]) for i in range(len(xs))]
        refs = []
        for x, e, o in calls:
            moe.moe_layer_forward(x, L.wr, L.k, e, bias=L.bias, ws=ws, out=o)
            refs.append(o.clone())
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for x, e, o in calls:
                moe.moe_layer_forward(x, L.wr, L.k, e, bias=L.bias, ws=ws, out=o)
        for _ in range(3):
            for o in outs:
                o.zero_()
            g.replay()
            torch.cuda.synchronize()
            for o, r in zip(outs, refs):
                assert torch.equal(o, r)
    assert moe.moe_device_error() == 0


def test_layer_decode_mxfp4_standard_layout(moe, decode_layer):
    x = synthetic.make_tokens(64, 2048, seed=9)
    _layer_check(moe, decode_layer, x, tiled=False)


@pytest.fixture(scope="module")
def prefill_layer():
    return synthetic.make_layer("prefill", 0)


def test_layer_prefill_nvfp4_reduced_batch(moe, prefill_layer):
    x = synthetic.make_tokens(256, 2048, seed=11)
    _layer_check(moe, prefill_layer, x)


def test_layer_prefill_nvfp4_full_size_sampled(moe, prefill_layer):
    x = synthetic.make_tokens(4096, 2048, seed=12)
    _layer_check(moe, prefill_layer, x, sample=[0, 1, 777, 2048, 4095])


@pytest.fixture(scope="module")
def large_layer():
    # 3.6 GB of NVFP4 experts: generated on the GPU, copied to the host for the oracle
    return synthetic.make_layer("large", 0, device="cuda").to("cpu")


def test_layer_large_decode_sampled(moe, large_layer):
    x = synthetic.make_tokens(32, 4096, seed=13)
    _layer_check(moe, large_layer, x, y_fp32=True, sample=[0, 17, 31])


def test_layer_large_prefill_sampled(moe, large_layer):
    x = synthetic.make_tokens(8192, 4096, seed=14)
    _layer_check(moe, large_layer, x, y_fp32=True, sample=[0, 4096, 8191])


def test_layer_one_hot_expert_and_k1(moe):
    """k = 1 and a bias that sends every token to expert 3: one expert gets every row."""
    cfg = dict(H=256, E=16, k=1, I=256, fmt="mxfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=15)
    L.bias = torch.zeros(16)
    L.bias[3] = 100.0
    x = synthetic.make_tokens(300, 256, seed=15)
    _layer_check(moe, L, x)


def test_layer_empty_batch(moe):
    L = synthetic.make_layer("tiny", 0).to("cuda")
    x = torch.empty(0, L.H, dtype=torch.bfloat16, device="cuda")
    out = moe.moe_layer_forward(x, L.wr, L.k, moe.Experts.from_layer(L))
    assert out.shape == (0, L.H)


def test_layer_is_deterministic(moe):
    L = synthetic.make_layer("tiny", 0).to("cuda")
    x = synthetic.make_tokens(16, L.H, 0).cuda()
    a = moe.moe_layer_forward(x, L.wr, L.k, moe.Experts.from_layer(L))
    b = moe.moe_layer_forward(x, L.wr, L.k, moe.Experts.from_layer(L))
    assert torch.equal(a, b)


def test_bad_arguments_are_rejected(moe):
    L = synthetic.make_layer("tiny", 0).to("cuda")
    x = synthetic.make_tokens(4, L.H, 0).cuda()
    bad = moe.Experts("bf16", 8, 200, 512, L.w13, L.w2)       # H not a multiple of 128
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward(x, L.wr, L.k, bad)
    assert ei.value.name == "UNSUPPORTED"
    with pytest.raises(moe.MoeError):
        moe.moe_route_topk(x, L.wr, 17)                        # k > 16


# ----------------------------------------------------------------------------- wider full-size sampling


def _sample_rows(L, x, n_random, seed, BN=128):
    """Tokens whose outputs are checked at full size: rows at the start, end and every
    token-tile boundary (multiples of BN) of the three most-routed experts, the first and
    last row of every expert that has any, and random tokens; about 64-100 in all."""
    idx_o, _, _ = oracle.route(x, L.wr, L.k, bias=L.bias, with_logits=False)
    off, sp, _ = oracle.permute(idx_o, L.E)
    n = np.diff(off)
    rows = []
    for e in np.argsort(-n, kind="stable")[:3]:
        b, c = int(off[e]), int(n[e])
        for r in range(0, c, BN):
            rows += [b + r, b + r - 1] if r else [b]
        rows.append(b + c - 1)
    busy = [e for e in range(L.E) if n[e] > 0]
    g = np.random.default_rng(seed)
    for e in g.choice(busy, size=min(len(busy), 16), replace=False):
        rows += [int(off[e]), int(off[e + 1]) - 1]
    toks = set(int(sp[r]) // L.k for r in rows if 0 <= r < len(sp))
    toks |= set(int(t) for t in g.choice(x.shape[0], n_random, replace=False))
    return sorted(toks)


def test_layer_prefill_nvfp4_full_size_wide_sample(moe, prefill_layer):
    x = synthetic.make_tokens(4096, 2048, seed=12)
    sample = _sample_rows(prefill_layer, x, 16, 12)
    assert len(sample) >= 64
    _layer_check(moe, prefill_layer, x, sample=sample)


def test_layer_large_prefill_wide_sample(moe, large_layer):
    x = synthetic.make_tokens(8192, 4096, seed=14)
    sample = _sample_rows(large_layer, x, 16, 14)
    assert len(sample) >= 64
    _layer_check(moe, large_layer, x, y_fp32=True, sample=sample)


def test_layer_large_decode_every_row(moe, large_layer):
    x = synthetic.make_tokens(32, 4096, seed=13)
    _layer_check(moe, large_layer, x, y_fp32=True, sample=list(range(32)))


# ----------------------------------------------------------------------------- the boundary's limits


def test_router_top16(moe):
    cfg = dict(H=512, E=256, k=16, wr_fp32=False, zipf=None)
    wr, _ = synthetic.make_router(cfg, seed=31)
    for T in (5, 300):   # the cluster path and the fp64 tensor-core path
        x = synthetic.make_tokens(T, 512, seed=31 + T)
        idx_o, w_o, lg_o = oracle.route(x, wr, 16)
        idx, w, lg = moe.moe_route_topk(x.cuda(), wr.cuda(), 16, want_logits=True)
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        assert _ulp_close(lg.cpu().numpy(), lg_o, 1)
        assert np.allclose(w.cpu().numpy(), w_o, rtol=0, atol=2e-6)


def test_router_infinite_input(moe):
    """An infinite activation makes every logit of its token +-Inf: the experts tie and go
    in index order, as in the oracle; the other tokens are unaffected."""
    wr, _ = synthetic.make_router("decode", seed=32)
    for T in (6, 300):
        x = synthetic.make_tokens(T, 2048, seed=32)
        x[2, 100] = float("inf")
        idx_o, w_o, lg_o = oracle.route(x, wr, 8)
        idx, w, lg = moe.moe_route_topk(x.cuda(), wr.cuda(), 8, want_logits=True)
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        lg, w = lg.cpu().numpy(), w.cpu().numpy()
        assert np.array_equal(np.isinf(lg), np.isinf(lg_o)) and np.isinf(lg_o[2]).all()
        fin = np.isfinite(lg_o)
        assert _ulp_close(lg[fin], lg_o[fin], 1)
        assert np.array_equal(np.isnan(w), np.isnan(w_o))
        ok = ~np.isnan(w_o)
        assert np.allclose(w[ok], w_o[ok], rtol=0, atol=2e-6)


@pytest.mark.parametrize("T,k,E", [(512, 16, 1024), (3000, 16, 1024), (20000, 8, 1024)])
def test_permute_at_the_limits(moe, T, k, E):
    idx = _rand_idx(T, k, E, 17 + T)
    x = synthetic.make_tokens(T, 64, seed=17)
    off_o, sp_o, pr_o = oracle.permute(idx, E)
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), E, x.cuda())
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(sp.cpu().numpy(), sp_o)
    assert np.array_equal(pr.cpu().numpy(), pr_o)
    got = deinterleave_cols(xp.view(torch.int16).cpu().numpy())
    assert np.array_equal(got, x.view(torch.int16).numpy()[sp_o // k])


@pytest.mark.parametrize("fmt,tiled", [("mxfp4", True), ("bf16", False)])
def test_grouped_ffn_1024_experts(moe, fmt, tiled):
    """E = 1024 experts (the grouped FFN's limit), most with a row or two, some empty."""
    E, T, k = 1024, 700, 2
    cfg = dict(H=256, E=E, k=k, I=256, fmt=fmt, wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=19, device="cuda").to("cpu")
    x = synthetic.make_tokens(T, 256, seed=19)
    idx = _rand_idx(T, k, E, 19)
    off_o, sp_o, _ = oracle.permute(idx, E)
    y_o = oracle.ffn(x, L, off_o, sp_o, k)
    ex = moe.Experts.from_layer(L.to("cuda"))
    if tiled:
        ex = moe.moe_prepack(ex)
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), E, x.cuda())
    y = moe.moe_grouped_ffn(xp, off, ex)
    torch.cuda.synchronize()
    assert rel_err(bf16_np(y), y_o) < TOL
    assert moe.moe_device_error() == 0


def test_combine_top16(moe):
    g = torch.Generator().manual_seed(23)
    T, k, H = 29, 16, 256
    y = torch.randn(T * k, H, generator=g).to(torch.bfloat16)
    pr = torch.randperm(T * k, generator=g).to(torch.int32)
    w = torch.rand(T, k, generator=g)
    ref = oracle.combine(y.float().numpy(), pr.numpy(), w.numpy(), T, k)
    out = moe.moe_combine(y.cuda(), pr.cuda(), w.cuda())
    assert rel_err(bf16_np(out), ref) < 4e-3


def test_layer_top16(moe):
    cfg = dict(H=256, E=64, k=16, I=256, fmt="mxfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=24)
    x = synthetic.make_tokens(40, 256, seed=24)
    _layer_check(moe, L, x)
    _layer_check(moe, L, x, tiled=False)


def test_layer_block_scaled_unfused_routing(moe):
    """Prepacked MXFP4 with more than 8192 pairs: routing and permutation run in separate
    launches (the fused one-block sort stops at 8192 pairs), then the block-scaled path."""
    cfg = dict(H=512, E=16, k=8, I=256, fmt="mxfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=25)
    x = synthetic.make_tokens(1100, 512, seed=25)
    n0 = moe.moe_kernel_launch_count()
    _layer_check(moe, L, x)
    assert moe.moe_kernel_launch_count() - n0 > 5


def test_layer_on_more_streams_than_ticket_counters(moe, decode_layer):
    """Each stream gets one of 256 sets of slot counts (and ticket counters); calls on
    further streams permute and quantise in their own launches. Every stream's output must equal
    the default stream's, bit for bit, on both sides of that limit."""
    from cuda.bindings import runtime as rt

    L = decode_layer.to("cuda")
    ex = moe.moe_prepack(moe.Experts.from_layer(L))
    T = 16
    x = synthetic.make_tokens(T, L.H, seed=26).cuda()
    ws = torch.empty(moe.moe_workspace_size(T, L.H, L.I, L.E, L.k), dtype=torch.uint8, device="cuda")
    ref = moe.moe_layer_forward(x, L.wr, L.k, ex, ws=ws).clone()
    out = torch.empty_like(ref)      # nothing is allocated on the streams created below
    torch.cuda.synchronize()
    handles, launches = [], []
    try:
        for _ in range(300):
            err, h = rt.cudaStreamCreateWithFlags(1)
            assert int(err) == 0
            handles.append(h)
            s = torch.cuda.ExternalStream(int(h))
            s.wait_stream(torch.cuda.current_stream())
            n0 = moe.moe_kernel_launch_count()
            out.zero_()
            torch.cuda.synchronize()
            with torch.cuda.stream(s):
                moe.moe_layer_forward(x, L.wr, L.k, ex, ws=ws, out=out)
            launches.append(moe.moe_kernel_launch_count() - n0)
            s.synchronize()
            assert torch.equal(out, ref)
    finally:
        torch.cuda.synchronize()
        for h in handles:
            rt.cudaStreamDestroy(h)
    # slot layout (4 launches: router, UP, DOWN, combine) while the per-stream counts last,
    # then routing, permutation and quantiser apart (6)
    assert launches[-1] == 6 and set(launches) <= {4, 6}
    assert launches == sorted(launches)
    assert moe.moe_device_error() == 0


# ----------------------------------------------------------------------------- bounded waits


def test_bounded_wait_gives_up_and_reports(moe):
    """A kernel waits, through the FFN kernels' bounded wait, on a barrier that nothing
    completes (no copy or MMA in flight). With a 1 ms limit it returns, the device error
    word reads 1 (a wait timed out), and with the default limit back the next layer runs."""
    assert moe.moe_device_error() == 0
    moe.moe_set_wait_limit_ns(1_000_000)
    try:
        moe.moe_selftest_wait()
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit_ns(0)
    assert moe.moe_device_error() == 1
    assert moe.moe_device_error() == 0          # read and cleared
    L = synthetic.make_layer("tiny", 0)
    x = synthetic.make_tokens(16, L.H, 0)
    _layer_check(moe, L, x)


# ----------------------------------------------------------------------------- activation format A4


@pytest.mark.parametrize("E,T,H,I,y32", [(8, 40, 256, 512, False), (8, 100, 512, 256, False), (8, 300, 256, 256, False),
                                         (8, 3, 256, 256, False), (16, 700, 512, 512, True), (4, 129, 256, 768, False)])
def test_grouped_ffn_a4_parity(moe, E, T, H, I, y32):
    """Activations in NVFP4 form (A4) on prepacked NVFP4 experts: token tiles of 32, 64 and
    128 (mean rows per expert 2T/E), ragged tails, one and several stages per item, the
    down projection at 3 stages (I = 768), bf16 and fp32 outputs; against the oracle's A4
    FFN on the same permutation."""
    cfg = dict(H=H, E=E, k=2, I=I, fmt="nvfp4", wr_fp32=False)
    L = synthetic.make_layer(cfg, seed=40 + T)
    x = synthetic.make_tokens(T, H, seed=40 + T)
    idx = _rand_idx(T, 2, E, T + 1)
    off_o, sp_o, _ = oracle.permute(idx, E)
    y_o = oracle.ffn(x, L, off_o, sp_o, 2, act="a4")
    ex = moe.moe_prepack(moe.Experts.from_layer(L.to("cuda")))
    off, sp, pr, xp = moe.moe_permute(torch.from_numpy(idx).cuda(), E, x.cuda(), act="a4")
    # A4 rows are in natural column order
    assert torch.equal(xp.cpu(), x[torch.from_numpy(sp_o // 2).long()])
    y = moe.moe_grouped_ffn(xp, off, ex, y_fp32=y32, act="a4")
    torch.cuda.synchronize()
    err = rel_err(y.float().cpu().numpy(), y_o)
    assert err < TOL, f"A4 FFN error {err:.3e}"
    assert moe.moe_device_error() == 0


def test_a4_needs_prepacked_nvfp4(moe):
    L = synthetic.make_layer(dict(H=256, E=8, k=2, I=256, fmt="mxfp4", wr_fp32=False), 3).to("cuda")
    x = synthetic.make_tokens(8, 256, 3).cuda()
    for ex in (moe.moe_prepack(moe.Experts.from_layer(L)), moe.Experts.from_layer(L)):
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_layer_forward(x, L.wr, 2, ex, act="a4")
        assert ei.value.name == "UNSUPPORTED"


def test_layer_a4_prefill_reduced_batch(moe, prefill_layer):
    x = synthetic.make_tokens(256, 2048, seed=41)
    _layer_check(moe, prefill_layer, x, act="a4")


def test_layer_a4_prefill_full_size_sampled(moe, prefill_layer):
    x = synthetic.make_tokens(4096, 2048, seed=42)
    sample = _sample_rows(prefill_layer, x, 16, 42)
    _layer_check(moe, prefill_layer, x, sample=sample, act="a4")


def test_layer_a4_large_prefill_sampled(moe, large_layer):
    x = synthetic.make_tokens(8192, 4096, seed=43)
    sample = _sample_rows(large_layer, x, 16, 43)
    _layer_check(moe, large_layer, x, y_fp32=True, sample=sample, act="a4")


def test_layer_a4_large_decode_every_row(moe, large_layer):
    x = synthetic.make_tokens(32, 4096, seed=44)
    _layer_check(moe, large_layer, x, y_fp32=True, sample=list(range(32)), act="a4")


def test_layer_a4_through_the_cache_equals_resident(moe):
    cfg = dict(H=512, E=16, k=4, I=256, fmt="nvfp4", wr_fp32=False)
    dev = [synthetic.make_layer(cfg, seed=45, layer=l).to("cuda") for l in range(2)]
    packed = [moe.moe_prepack(moe.Experts.from_layer(L)) for L in dev]
    host = [moe.Experts(t.fmt, t.E, t.H, t.I, t.w13.cpu().pin_memory(), t.w2.cpu().pin_memory(),
                        w13_tscale=t.w13_tscale.cpu(), w2_tscale=t.w2_tscale.cpu(), layout=moe.LAYOUT_TILED)
            for t in packed]
    cache = moe.ExpertCache(1 << 30, host, device=0)
    for step in range(3):
        for l in range(2):
            x = synthetic.make_tokens(100, 512, seed=46 + 5 * step + l).cuda()
            out_c = moe.moe_layer_forward(x, dev[l].wr, 4, moe.Experts.from_layer(dev[l]), cache=cache, layer=l,
                                          act="a4")
            out_r = moe.moe_layer_forward(x, dev[l].wr, 4, packed[l], act="a4")
            torch.cuda.synchronize()
            assert torch.equal(out_c, out_r), (step, l)
    assert moe.moe_device_error() == 0
    cache.close()
