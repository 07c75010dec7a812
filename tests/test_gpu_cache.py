"""GPU tests of the device LRU expert cache and host->device streaming.

Cached forward must equal the all-resident forward bit for bit (same kernels,
same arithmetic, weights only relocated), and the hit/miss trace and final
table must equal the CPU simulation driven through the same calls."""
import os

import numpy as np
import pytest
import torch

import synthetic
from oracle.lru import CacheFull, LruSim

pytestmark = pytest.mark.gpu

L_, E_, H_, I_, K_, T_ = 4, 16, 256, 256, 4, 4
CFG = dict(H=H_, E=E_, k=K_, I=I_, fmt="fp8", wr_fp32=False)


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available()
    import expert_ffn_layer_top_b200 as m

    return m


@pytest.fixture(scope="module")
def stack():
    layers = [synthetic.make_layer(CFG, seed=21, layer=l) for l in range(L_)]
    host = []
    dev = []
    for L in layers:
        pinned = L.to("cpu")
        for name in ("w13", "w2", "w13_scale", "w2_scale"):
            setattr(pinned, name, getattr(pinned, name).contiguous().pin_memory())
        host.append(pinned)
        dev.append(L.to("cuda"))
    return layers, host, dev


def _slot_payload(moe, host_layer):
    return sum(t.numel() * t.element_size() // E_ for t in (host_layer.w13, host_layer.w13_scale, host_layer.w2,
                                                           host_layer.w2_scale))


def _bias(step, layer):
    # popularity drifts between two permutations every 3 steps
    g = torch.Generator().manual_seed(1000 + layer + 100 * ((step // 3) % 2))
    return synthetic.zipf_bias(E_, 1.2, H_, 0, perm=torch.randperm(E_, generator=g))


def test_cached_forward_equals_resident_and_matches_lru_sim(moe, stack):
    layers, host, dev = stack
    slot_payload = _slot_payload(moe, host[0])
    S = 40
    # capacity in slots: each slot is the 256-byte-aligned sum of the four parts
    slot_bytes = sum(((t.numel() * t.element_size() // E_) + 255) // 256 * 256
                     for t in (host[0].w13, host[0].w13_scale, host[0].w2, host[0].w2_scale))
    cache = moe.ExpertCache(S * slot_bytes, [moe.Experts.from_layer(h) for h in host], device=0)
    sim = LruSim(S, L_, E_, slot_payload)
    last = {}
    for step in range(12):
        for l in range(L_):
            x = synthetic.make_tokens(T_, H_, seed=step * 97 + l).cuda()
            b = _bias(step, l).cuda()
            shape = moe.Experts.from_layer(dev[l])
            idx = torch.empty(T_, K_, dtype=torch.int32, device="cuda")
            out_c = moe.moe_layer_forward(x, dev[l].wr, K_, shape, bias=b, cache=cache, layer=l, idx_out=idx)
            out_r = moe.moe_layer_forward(x, dev[l].wr, K_, shape, bias=b)
            torch.cuda.synchronize()
            assert torch.equal(out_c, out_r), (step, l)
            ids = sorted(set(idx.cpu().numpy().ravel().tolist()))
            sim.resolve(l, ids)
            last[l] = ids
            if l + 1 < L_:
                try:
                    sim.prefetch(l + 1, last.get(l + 1, []))
                except CacheFull:
                    pass
    st = cache.stats()
    assert (st["hits"], st["misses"]) == (sim.hits, sim.misses)
    assert st["bytes_h2d"] == sim.loads * slot_payload
    table = [cache.slot_of(l, e) for l in range(L_) for e in range(E_)]
    assert table == sim.table()
    assert sim.misses > 0 and sim.hits > 0
    # evict everything: the next forward misses again and still gives the same result
    cache.evict()
    x = synthetic.make_tokens(T_, H_, seed=5).cuda()
    shape = moe.Experts.from_layer(dev[0])
    a = moe.moe_layer_forward(x, dev[0].wr, K_, shape, cache=cache, layer=0)
    bref = moe.moe_layer_forward(x, dev[0].wr, K_, shape)
    assert torch.equal(a, bref)
    assert cache.stats()["misses"] > st["misses"]
    cache.close()
    assert moe.moe_device_error() == 0


def test_explicit_prefetch_turns_misses_into_hits(moe, stack):
    layers, host, dev = stack
    cache = moe.ExpertCache(1 << 30, [moe.Experts.from_layer(h) for h in host], device=0)
    x = synthetic.make_tokens(T_, H_, seed=9).cuda()
    idx = torch.empty(T_, K_, dtype=torch.int32, device="cuda")
    shape = moe.Experts.from_layer(dev[2])
    moe.moe_layer_forward(x, dev[2].wr, K_, shape, idx_out=idx)
    ids = sorted(set(idx.cpu().numpy().ravel().tolist()))
    cache.prefetch(2, ids)
    out = moe.moe_layer_forward(x, dev[2].wr, K_, shape, cache=cache, layer=2)
    st = cache.stats()
    assert st["misses"] == 0 and st["hits"] == len(ids)
    assert torch.equal(out, moe.moe_layer_forward(x, dev[2].wr, K_, shape))
    cache.close()


def test_tiled_host_pool_streams_and_matches(moe, stack):
    """Host pool in the prepacked (tiled) layout: two copies per miss, same results."""
    layers, host, dev = stack
    tiled_host = []
    for L in dev:
        t = moe.moe_prepack(moe.Experts.from_layer(L))
        tiled_host.append(moe.Experts(t.fmt, t.E, t.H, t.I, t.w13.cpu().pin_memory(), t.w2.cpu().pin_memory(),
                                      layout=moe.LAYOUT_TILED))
    cache = moe.ExpertCache(1 << 30, tiled_host, device=0)
    for l in range(L_):
        x = synthetic.make_tokens(T_, H_, seed=40 + l).cuda()
        shape = moe.Experts.from_layer(dev[l])
        out_c = moe.moe_layer_forward(x, dev[l].wr, K_, shape, cache=cache, layer=l)
        out_r = moe.moe_layer_forward(x, dev[l].wr, K_, shape)
        assert torch.equal(out_c, out_r)
    assert cache.stats()["misses"] > 0
    cache.close()


def test_mxfp4_prepacked_cache_matches_resident(moe):
    """Prepacked MXFP4 experts run the block-scaled path; through the cache they
    are addressed by slot, and the result must not change."""
    cfg = dict(H=H_, E=E_, k=K_, I=I_, fmt="mxfp4", wr_fp32=False)
    dev = [synthetic.make_layer(cfg, seed=31, layer=l).to("cuda") for l in range(2)]
    packed = [moe.moe_prepack(moe.Experts.from_layer(L)) for L in dev]
    host = [moe.Experts(t.fmt, t.E, t.H, t.I, t.w13.cpu().pin_memory(), t.w2.cpu().pin_memory(),
                        layout=moe.LAYOUT_TILED) for t in packed]
    cache = moe.ExpertCache(1 << 30, host, device=0)
    for step in range(3):
        for l in range(2):
            x = synthetic.make_tokens(T_, H_, seed=70 + 5 * step + l).cuda()
            out_c = moe.moe_layer_forward(x, dev[l].wr, K_, moe.Experts.from_layer(dev[l]), cache=cache, layer=l)
            out_r = moe.moe_layer_forward(x, dev[l].wr, K_, packed[l])
            torch.cuda.synchronize()
            assert torch.equal(out_c, out_r), (step, l)
    assert moe.moe_device_error() == 0
    cache.close()


def test_cache_full_is_reported(moe, stack):
    layers, host, dev = stack
    slot_bytes = sum(((t.numel() * t.element_size() // E_) + 255) // 256 * 256
                     for t in (host[0].w13, host[0].w13_scale, host[0].w2, host[0].w2_scale))
    cache = moe.ExpertCache(3 * slot_bytes, [moe.Experts.from_layer(h) for h in host], device=0)
    x = synthetic.make_tokens(T_, H_, seed=1).cuda()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward(x, dev[0].wr, K_, moe.Experts.from_layer(dev[0]), cache=cache, layer=0)
    assert ei.value.name == "CACHE_FULL"
    cache.close()


def test_injected_copy_failure_is_reported(moe, stack):
    layers, host, dev = stack
    os.environ["MOE_FAULT"] = "h2d_fail@3"
    try:
        cache = moe.ExpertCache(1 << 30, [moe.Experts.from_layer(h) for h in host], device=0)
    finally:
        del os.environ["MOE_FAULT"]
    x = synthetic.make_tokens(T_, H_, seed=2).cuda()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward(x, dev[0].wr, K_, moe.Experts.from_layer(dev[0]), cache=cache, layer=0)
    assert "injected" in str(ei.value)
    cache.close()


def test_injected_pinned_allocation_failure(moe, stack):
    layers, host, dev = stack
    os.environ["MOE_FAULT"] = "pin_alloc"
    try:
        with pytest.raises(moe.MoeError) as ei:
            moe.ExpertCache(1 << 30, [moe.Experts.from_layer(h) for h in host], device=0)
        assert ei.value.name == "OOM"
    finally:
        del os.environ["MOE_FAULT"]


def _slot_bytes(host0):
    return sum(((t.numel() * t.element_size() // E_) + 255) // 256 * 256
               for t in (host0.w13, host0.w13_scale, host0.w2, host0.w2_scale))


def _drive(moe, cache, sim, dev, steps, depth=-1, full=False, resize_at=None, seed0=0):
    """Cached layer calls over `steps` x L_ layers, mirrored in the simulation (each resolve
    followed by the next layer's prefetch of the given depth, or of the whole layer).
    Cached output must equal the resident output bit for bit."""
    for step in range(steps):
        if resize_at and step in resize_at:
            S_new = resize_at[step]
            cache.resize(S_new * _slot_bytes_cached[0])
            sim.resize(S_new)
        for l in range(L_):
            x = synthetic.make_tokens(T_, H_, seed=seed0 + step * 97 + l).cuda()
            b = _bias(step, l).cuda()
            shape = moe.Experts.from_layer(dev[l])
            idx = torch.empty(T_, K_, dtype=torch.int32, device="cuda")
            out_c = moe.moe_layer_forward(x, dev[l].wr, K_, shape, bias=b, cache=cache, layer=l, idx_out=idx)
            out_r = moe.moe_layer_forward(x, dev[l].wr, K_, shape, bias=b)
            torch.cuda.synchronize()
            assert torch.equal(out_c, out_r), (step, l)
            sim.resolve(l, idx.cpu().numpy().ravel().tolist())
            if l + 1 < L_:
                try:
                    sim.prefetch(l + 1, sim.predict(l + 1, depth, full))
                except CacheFull:
                    pass


_slot_bytes_cached = [0]


@pytest.mark.parametrize("depth", [0, 2, 5])
def test_prefetch_depth_follows_the_ranked_prediction(moe, stack, depth):
    """With a prefetch depth d, the next layer's d most-routed experts of its previous call
    (ties to the lower id) are loaded ahead: trace, counts and table equal the simulation."""
    layers, host, dev = stack
    sb = _slot_bytes(host[0])
    _slot_bytes_cached[0] = sb
    S = 40
    cache = moe.ExpertCache(S * sb, [moe.Experts.from_layer(h) for h in host], device=0)
    cache.set_prefetch("predicted", depth)
    sim = LruSim(S, L_, E_, _slot_payload(moe, host[0]))
    _drive(moe, cache, sim, dev, 8, depth=depth, seed0=300 + depth)
    st = cache.stats()
    assert (st["hits"], st["misses"]) == (sim.hits, sim.misses)
    assert st["bytes_h2d"] == sim.bytes_h2d
    assert [cache.slot_of(l, e) for l in range(L_) for e in range(E_)] == sim.table()
    rep = cache.report()
    assert rep["last_depth"] == depth and rep["calls"] == 8 * L_
    cache.close()
    assert moe.moe_device_error() == 0


def test_full_layer_streaming_loads_every_expert_once(moe, stack):
    """Whole-layer streaming (the prefill mode): while layer l computes, all E experts of
    layer l+1 stream in. With room for three layers, one pass over the stack misses only
    on layer 0, every other layer is all hits, the bytes streamed equal the whole pool,
    and the output equals the all-resident output bit for bit."""
    layers, host, dev = stack
    sb = _slot_bytes(host[0])
    cache = moe.ExpertCache(3 * E_ * sb, [moe.Experts.from_layer(h) for h in host], device=0)
    cache.set_prefetch("full_layer")
    T = 64   # 64 tokens x top-4 of 16 experts: every expert of every layer is routed to
    for l in range(L_):
        x = synthetic.make_tokens(T, H_, seed=500 + l).cuda()
        shape = moe.Experts.from_layer(dev[l])
        idx = torch.empty(T, K_, dtype=torch.int32, device="cuda")
        out_c = moe.moe_layer_forward(x, dev[l].wr, K_, shape, cache=cache, layer=l, idx_out=idx)
        out_r = moe.moe_layer_forward(x, dev[l].wr, K_, shape)
        torch.cuda.synchronize()
        assert torch.equal(out_c, out_r), l
        assert len(set(idx.cpu().numpy().ravel().tolist())) == E_
    st = cache.stats()
    pool = sum(t.numel() * t.element_size() for h in host for t in (h.w13, h.w13_scale, h.w2, h.w2_scale))
    assert st["misses"] == E_ and st["hits"] == (L_ - 1) * E_
    assert st["bytes_h2d"] == pool
    rep = cache.report()
    assert rep["prefetched"] == (L_ - 1) * E_ and rep["last_depth"] == E_
    assert 0.0 <= rep["overlap_s"] <= rep["copy_s"] + 1e-6
    cache.close()


def test_resize_keeps_resident_experts_without_reloading(moe, stack):
    """Shrink and grow the slot pool between calls: the kept experts move device to device
    (no host copy), the table follows the simulation's resize rule, and every cached
    output still equals the resident one bit for bit."""
    layers, host, dev = stack
    sb = _slot_bytes(host[0])
    _slot_bytes_cached[0] = sb
    S = 48
    cache = moe.ExpertCache(S * sb, [moe.Experts.from_layer(h) for h in host], device=0)
    sim = LruSim(S, L_, E_, _slot_payload(moe, host[0]))
    _drive(moe, cache, sim, dev, 3, seed0=700)
    before = cache.stats()["bytes_h2d"]
    cache.resize(20 * sb)
    moves = sim.resize(20)
    assert cache.stats()["bytes_h2d"] == before            # nothing came from the host
    assert cache.report()["moved"] == len(moves) and cache.report()["n_slots"] == 20
    assert [cache.slot_of(l, e) for l in range(L_) for e in range(E_)] == sim.table()
    _drive(moe, cache, sim, dev, 3, seed0=800, resize_at={1: 60, 2: 24})
    st = cache.stats()
    assert (st["hits"], st["misses"]) == (sim.hits, sim.misses)
    assert [cache.slot_of(l, e) for l in range(L_) for e in range(E_)] == sim.table()
    assert sim.moves > 0
    with pytest.raises(moe.MoeError) as ei:
        cache.resize(sb // 2)
    assert ei.value.name == "CACHE_FULL"
    cache.close()
    assert moe.moe_device_error() == 0


def test_adaptive_prefetch_streams_whole_layers_for_prefill_sized_calls(moe, stack):
    layers, host, dev = stack
    sb = _slot_bytes(host[0])
    cache = moe.ExpertCache(3 * E_ * sb, [moe.Experts.from_layer(h) for h in host], device=0)
    cache.set_prefetch("adaptive")
    # E (1 - (1 - k/E)^T) with k = 4, E = 16: T = 1 -> 4, T = 2 -> 7 experts (< E/2); T = 64 -> 16
    for T, want_full in ((1, False), (64, True), (2, False)):
        for l in range(L_):
            x = synthetic.make_tokens(T, H_, seed=900 + 10 * T + l).cuda()
            shape = moe.Experts.from_layer(dev[l])
            out_c = moe.moe_layer_forward(x, dev[l].wr, K_, shape, cache=cache, layer=l)
            out_r = moe.moe_layer_forward(x, dev[l].wr, K_, shape)
            torch.cuda.synchronize()
            assert torch.equal(out_c, out_r), (T, l)
        rep = cache.report()
        assert (rep["last_depth"] == E_) == want_full, (T, rep["last_depth"])
    rep = cache.report()
    assert rep["h2d_gbs"] > 0 and rep["compute_s"] > 0 and rep["table_s"] > 0
    cache.close()


def test_injected_copy_failure_rolls_the_table_back(moe, stack):
    """A copy that fails leaves no table entry pointing at a slot whose data never came:
    the same layer called again loads those experts and matches the resident output."""
    layers, host, dev = stack
    os.environ["MOE_FAULT"] = "h2d_fail@6"
    try:
        cache = moe.ExpertCache(1 << 30, [moe.Experts.from_layer(h) for h in host], device=0)
    finally:
        del os.environ["MOE_FAULT"]
    x = synthetic.make_tokens(T_, H_, seed=3).cuda()
    shape = moe.Experts.from_layer(dev[1])
    with pytest.raises(moe.MoeError):
        moe.moe_layer_forward(x, dev[1].wr, K_, shape, cache=cache, layer=1)
    out_c = moe.moe_layer_forward(x, dev[1].wr, K_, shape, cache=cache, layer=1)
    out_r = moe.moe_layer_forward(x, dev[1].wr, K_, shape)
    torch.cuda.synchronize()
    assert torch.equal(out_c, out_r)
    assert moe.moe_device_error() == 0
    cache.close()


# ----------------------------------------------------------------------------- the streaming-stack layer


def test_streaming_stack_layer_matches_the_oracle():
    """The streaming-stack layer at its own shape (FP8 experts with fp32 scales per 128-wide
    K block, H = 2048, I = 768, E = 128, top-8, T = 4, Zipf(1.2)-skewed routing) through
    moe_layer_forward with a cache of 40 slots, far fewer than the 3 x 128 experts, over
    several steps whose routing drifts between two popularity permutations: routing
    bit-exact and the output within the layer tolerance of the CPU oracle on every call,
    with misses and evictions along the way. The input of each layer is the previous
    layer's residual output, as in the stack."""
    import expert_ffn_layer_top_b200 as moe
    import oracle
    from gpu_util import TOL, rel_err

    cfg = dict(synthetic.CONFIGS["stack"])
    H, I, E, k, T, NL = cfg["H"], cfg["I"], cfg["E"], cfg["k"], 4, 3
    layers = [synthetic.make_layer("stack", 0, device="cuda", layer=l).to("cpu") for l in range(NL)]
    host = []
    for L in layers:
        for name in ("w13", "w2", "w13_scale", "w2_scale"):
            setattr(L, name, getattr(L, name).contiguous().pin_memory())
        host.append(moe.Experts.from_layer(L))
    slot = synthetic.expert_bytes("fp8", H, I) + 4 * 256
    cache = moe.ExpertCache(40 * slot, host, device=0)
    wr = [L.wr.cuda() for L in layers]
    misses = []
    for step in range(4):
        x = synthetic.make_tokens(T, H, seed=40 + step)
        for l in range(NL):
            g = torch.Generator().manual_seed(4000 + l + 100 * (step % 2))
            bias = synthetic.zipf_bias(E, cfg["zipf"], H, 0, perm=torch.randperm(E, generator=g))
            idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
            out = moe.moe_layer_forward(x.cuda(), wr[l], k, moe.Experts.from_layer(layers[l]), bias=bias.cuda(),
                                        cache=cache, layer=l, idx_out=idx)
            torch.cuda.synchronize()
            ref = oracle.layer_forward(x, layers[l], bias=bias)
            assert np.array_equal(idx.cpu().numpy(), ref["idx"]), (step, l)
            err = rel_err(out.float().cpu().numpy(), ref["out"])
            assert err < TOL, (step, l, err)
            misses.append(cache.stats()["misses"])
            x = (x.float() + out.float().cpu()).to(torch.bfloat16)
    assert misses[-1] > E // 2 and cache.stats()["hits"] > 0
    assert moe.moe_device_error() == 0
    cache.close()
