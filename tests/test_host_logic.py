"""Host-side logic of the C ABI, on the CPU: argument checks that return the
status include/moe.h documents before any device work, workspace sizing, and
prepacked sizes.

The calls go through the raw ctypes entry points with NULL (or, in one case,
never-dereferenced) pointers. Every case here is rejected or finished by the
library's host-side checks, so no kernel is launched. The module runs only
where no CUDA device is visible, so that even a missing check could not reach
a device with those pointers; on a GPU the parity suite has its own
bad-argument test through real tensors."""
import ctypes

import pytest
import torch

import expert_ffn_layer_top_b200 as moe
from expert_ffn_layer_top_b200._lib import _Experts

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="host-only checks; run where no device is visible")

OK, INVALID_ARG, UNSUPPORTED, OOM = 0, 1, 2, 4
FMT = moe._lib.FMT


def _experts(fmt="bf16", E=8, H=256, I=512, w=None, scale=None, tscale=None, layout=0):
    return _Experts(FMT[fmt] if isinstance(fmt, str) else fmt, E, H, I, w, scale, tscale, w, scale, tscale,
                    0, 0, 0, 0, None, 0, layout)


def _err():
    return moe.lib().moe_last_error_string().decode()


def test_route_topk_checks():
    L = moe.lib()
    r = lambda T, H, E, k: L.moe_route_topk(None, T, H, None, 0, None, E, k, None, None, None, None, 0, None)
    assert r(4, 100, 8, 2) == INVALID_ARG          # H not a multiple of 8
    assert r(-1, 256, 8, 2) == INVALID_ARG
    assert r(4, 256, 8, 9) == UNSUPPORTED          # k > E
    assert r(4, 256, 8, 17) == UNSUPPORTED         # k > 16
    assert r(4, 256, 300, 2) == UNSUPPORTED        # the router takes E <= 256
    assert r(4, 256, 8, 0) == UNSUPPORTED
    assert r(0, 256, 8, 2) == OK                   # empty batch: nothing to do
    assert r(4, 256, 8, 2) == INVALID_ARG          # NULL pointers


def test_permute_checks():
    L = moe.lib()
    p = lambda T, k, E, af=0: L.moe_permute(None, T, k, E, None, 0, af, None, None, None, None, None, 0, None)
    assert p(-1, 2, 8) == INVALID_ARG
    assert p(4, 0, 8) == INVALID_ARG
    assert p(4, 17, 8) == INVALID_ARG
    assert p(4, 2, 2000) == INVALID_ARG            # E above the 1024 experts of the permutation
    assert p(4, 2, 8) == INVALID_ARG               # offsets is NULL
    assert p(4, 2, 8, af=2) == INVALID_ARG         # unknown activation format
    assert "activation format" in _err()
    # the fixed scratch of moe_permute_static covers ceil(T*k/1024)*E <= 131072 counters
    assert L.moe_permute_static(None, 1 << 20, 8, 1024, None, 0, None, None, None, None, None) == UNSUPPORTED
    assert "fixed scratch" in _err()


def test_grouped_ffn_and_prepack_check_the_experts_first():
    L = moe.lib()
    g = lambda ex, n=4, af=0: L.moe_grouped_ffn(None, n, None, ex, af, None, 0, None, 0, None)
    assert g(_experts(H=200)) == UNSUPPORTED        # H not a multiple of 256
    assert g(_experts(I=100)) == UNSUPPORTED
    assert g(_experts(fmt=7)) == UNSUPPORTED
    assert g(_experts(E=0)) == UNSUPPORTED
    assert g(_experts(E=1025)) == UNSUPPORTED
    assert g(_experts()) == INVALID_ARG             # NULL weights
    assert g(None) == INVALID_ARG
    assert g(_experts(), af=5) == INVALID_ARG
    # A4 activations: prepacked NVFP4 experts only
    assert g(_experts(fmt="mxfp4", w=1 << 24, scale=1 << 24), af=1) == UNSUPPORTED
    assert g(_experts(fmt="nvfp4", w=1 << 24, scale=1 << 24, tscale=1 << 24), af=1) == UNSUPPORTED
    assert "A4" in _err()
    assert L.moe_prepack(_experts(H=200), None, None, None) == UNSUPPORTED
    assert L.moe_prepack(_experts(), None, None, None) == INVALID_ARG


def test_combine_and_dequantize_checks():
    L = moe.lib()
    c = lambda T, k, H: L.moe_combine(None, 0, None, None, T, k, H, None, None)
    assert c(4, 0, 256) == INVALID_ARG
    assert c(4, 2, 12) == INVALID_ARG              # H not a multiple of 8
    assert c(0, 2, 256) == OK
    assert c(4, 2, 256) == INVALID_ARG             # NULL pointers
    d = lambda fmt, rows, K: L.moe_dequantize(fmt, None, None, 1.0, rows, K, None, None)
    assert d(9, 4, 256) == UNSUPPORTED
    assert d(FMT["mxfp4"], 4, 48) == INVALID_ARG   # K not a multiple of the 32-block
    assert d(FMT["nvfp4"], 4, 40) == INVALID_ARG   # ... of the 16-block
    assert d(FMT["fp8"], 4, 192) == INVALID_ARG    # ... of the 128-block
    assert d(FMT["nvfp4"], 0, 64) == OK
    assert d(FMT["bf16"], 4, 64) == INVALID_ARG    # NULL pointers


def test_layer_forward_checks():
    L = moe.lib()

    def f(ex, T=4, k=2, ptr=None, ws_bytes=0, af=0):
        return L.moe_layer_forward(ptr, T, ptr, 0, None, k, ex, af, None, 0, 0, ptr, None, None, ptr, ws_bytes, None)

    ex = _experts()
    assert f(None) == INVALID_ARG
    assert f(ex, T=-1) == INVALID_ARG
    assert f(ex, T=0) == OK
    assert f(ex, af=3) == INVALID_ARG
    for k in (0, 17, 9):                            # 9 > E = 8
        assert f(ex, k=k) == INVALID_ARG
        assert f"k={k}" in _err()
    assert f(_experts(H=200)) == UNSUPPORTED
    assert f(ex) == INVALID_ARG                     # NULL weights
    # weights, x, wr, out and ws set (never dereferenced): the workspace size is checked next
    fake = 1 << 24
    exw = _experts(w=fake)
    assert f(exw, ptr=fake, ws_bytes=256) == OOM
    need = moe.moe_workspace_size(4, 256, 512, 8, 2)
    assert f"< {need}" in _err()


def test_misaligned_arrays_are_rejected():
    """Non-NULL but misaligned pointers (never dereferenced: the checks return first)."""
    L = moe.lib()
    A = 1 << 24                 # 256-byte aligned
    odd2, odd8 = A + 2, A + 8   # 2 bytes off (breaks int32/fp32), 8 bytes off (breaks 16-byte vectors)
    route = lambda idx=A, w=A, logits=None, bias=None, ws=A: L.moe_route_topk(
        A, 4, 256, A, 0, bias, 8, 2, idx, w, logits, ws, 1 << 30, None)
    for kw in (dict(idx=odd2), dict(w=odd2), dict(logits=odd2), dict(bias=odd2), dict(ws=odd8)):
        assert route(**kw) == INVALID_ARG, kw
    perm = lambda idx=A, off=A, sp=A, pr=A, ws=A: L.moe_permute(idx, 4, 2, 8, None, 0, 0, off, sp, pr, None, ws,
                                                                1 << 30, None)
    for kw in (dict(idx=odd2), dict(off=odd2), dict(sp=odd2), dict(pr=odd2), dict(ws=odd8)):
        assert perm(**kw) == INVALID_ARG, kw
    comb = lambda pr=A, w=A, y=A, out=A: L.moe_combine(y, 0, pr, w, 4, 2, 256, out, None)
    for kw in (dict(pr=odd2), dict(w=odd2), dict(y=odd8), dict(out=odd8)):
        assert comb(**kw) == INVALID_ARG, kw
    ffn = lambda ex, off=A, y=A: L.moe_grouped_ffn(A, 4, off, ex, 0, y, 0, A, 1 << 40, None)
    ex = _experts(w=A)
    assert ffn(ex, off=odd2) == INVALID_ARG
    assert ffn(ex, y=odd8) == INVALID_ARG
    assert ffn(_experts(fmt="nvfp4", w=A, scale=A, tscale=odd2)) == INVALID_ARG
    assert L.moe_dequantize(FMT["fp8"], A, odd2, 1.0, 4, 128, A, None) == INVALID_ARG
    lay = lambda bias=None, idx=None, w=None, out=A: L.moe_layer_forward(A, 4, A, 0, bias, 2, ex, 0, None, 0, 0, out,
                                                                         idx, w, A, 1 << 40, None)
    for kw in (dict(bias=odd2), dict(idx=odd2), dict(w=odd2), dict(out=odd8)):
        assert lay(**kw) == INVALID_ARG, kw


def test_cache_init_checks_the_layers_first():
    L = moe.lib()
    h = ctypes.c_void_p()

    def init(layers, cap=1 << 30, out=True):
        arr = (_Experts * max(len(layers), 1))(*layers)
        return L.expert_cache_init(ctypes.byref(h) if out else None, cap, len(layers), arr, 0)

    assert init([_experts()], out=False) == INVALID_ARG
    assert init([]) == INVALID_ARG
    for bad in (_experts(H=0), _experts(I=0), _experts(H=-256), _experts(H=200), _experts(E=0), _experts(E=1025),
                _experts(fmt=7)):
        assert init([bad]) == UNSUPPORTED
    assert init([_experts(), _experts(I=256)]) == INVALID_ARG      # layers differ in shape
    assert init([_experts(), _experts(fmt="fp8")]) == INVALID_ARG  # ... in format
    assert not h.value                                              # nothing was created


def test_cache_calls_reject_a_null_cache():
    L = moe.lib()
    assert L.expert_cache_prefetch(None, 0, None, 0, None) == INVALID_ARG
    assert L.expert_cache_evict(None, -1, None, -1) == INVALID_ARG
    assert L.expert_cache_stats(None, None, None, None, None) == INVALID_ARG
    assert L.expert_cache_slot_of(None, 0, 0, None) == INVALID_ARG
    assert L.expert_cache_destroy(None) == OK


def test_workspace_size_is_monotone_and_rejects_bad_sizes():
    ws = moe.moe_workspace_size
    for cfg in ((2048, 768, 128, 8), (4096, 2048, 256, 6), (256, 512, 8, 2)):
        H, I, E, k = cfg
        sizes = [ws(T, H, I, E, k) for T in (1, 8, 64, 512, 4096)]
        assert all(0 < a < b for a, b in zip(sizes, sizes[1:]))
    # never smaller for a larger batch, across every step of the terms that depend on a tile
    # choice: the slot layout's tile height and its 256-token and 64 MiB limits, the activation
    # blobs' tile height (mean rows per expert past 8, 16, 32, 64), the router's H split per
    # 64-token tile
    for H, I, E, k in ((4096, 2048, 256, 6), (2048, 768, 128, 8), (2048, 1024, 32, 4), (6144, 1536, 160, 8)):
        prev = 0
        for T in list(range(1, 300)) + list(range(300, 2200, 7)):
            s = ws(T, H, I, E, k)
            assert s >= prev, (H, I, E, k, T, s, prev)
            prev = s
        assert ws(64, H, I, E, k, 1) > ws(64, H, I, E, k, 0)
        assert ws(64, H, I, E, k) < ws(64, H, I, E, k + 1)
        # at least the permuted activations and the expert outputs of every pair
        assert ws(64, H, I, E, k) >= 2 * 64 * k * H * 2
    for bad in ((-1, 2048, 768, 128, 8), (4, 0, 768, 128, 8), (4, 2048, 0, 128, 8), (4, 2048, 768, 0, 8),
                (4, 2048, 768, 128, 0)):
        assert ws(*bad) == 0
    assert ws(64, 2048, 768, 128, 8, 0, "a4") == ws(64, 2048, 768, 128, 8)   # one bound covers both formats
    assert moe.lib().moe_workspace_size(64, 2048, 768, 128, 8, 0, 7) == 0


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "mxfp4", "nvfp4"])
def test_prepacked_bytes_equal_the_standard_layout(fmt):
    code = {"bf16": 2.0, "fp8": 1.0, "mxfp4": 0.5, "nvfp4": 0.5}[fmt]
    scale = {"bf16": 0.0, "fp8": 4 / 128, "mxfp4": 1 / 32, "nvfp4": 1 / 16}[fmt]
    for H, I in ((2048, 768), (4096, 2048), (256, 512), (512, 256)):
        assert moe.moe_prepacked_expert_bytes(fmt, H, I, 0) == 2 * I * H * (code + scale)
        assert moe.moe_prepacked_expert_bytes(fmt, H, I, 1) == H * I * (code + scale)
    assert moe.moe_prepacked_expert_bytes(fmt, 200, 512, 0) == 0
    assert moe.moe_prepacked_expert_bytes(fmt, 256, 512, 2) == 0
