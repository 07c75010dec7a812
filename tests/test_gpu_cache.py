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
