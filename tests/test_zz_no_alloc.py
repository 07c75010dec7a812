"""moe_permute_static: the permutation with the library's fixed device scratch
instead of a caller workspace, compared with moe_permute on the same inputs.

The file is named to be collected last; each test builds its own inputs, so it
passes alone or after the rest of the suite (the first call on the device
performs the scratch set-up in either order)."""
import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

LIMIT = 1 << 20   # MOE_PERMUTE_STATIC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def moe():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import expert_ffn_layer_top_b200 as m

    return m


def _idx(T, k, E, seed):
    g = np.random.default_rng(seed)
    return torch.from_numpy(np.argsort(g.random((T, E)), axis=1)[:, :k].astype(np.int32)).cuda()


def _same(a, b):
    for u, v in zip(a, b):
        if u is None or v is None:
            assert u is None and v is None
        else:
            assert torch.equal(u, v)


# (T, k, E, H): two shapes past the one-block path (they use the scratch), one on it
CASES = [(4096, 8, 128, 2048), (2048, 8, 64, 256), (64, 8, 128, 2048)]


def _matches_oracle(got, idx, E, x=None):
    import oracle
    from gpu_util import deinterleave_cols

    off_o, sp_o, pr_o = oracle.permute(idx.cpu().numpy(), E)
    off, sp, pr, xp = got
    assert np.array_equal(off.cpu().numpy(), off_o)
    assert np.array_equal(sp.cpu().numpy(), sp_o)
    assert np.array_equal(pr.cpu().numpy(), pr_o)
    if x is not None:
        k = idx.shape[1]
        want = x.cpu().view(torch.int16).numpy()[sp_o // k]
        assert np.array_equal(deinterleave_cols(xp.view(torch.int16).cpu().numpy()), want)


def test_static_permute_matches_the_oracle(moe):
    """Offsets, sorted pairs, pair rows and the gathered rows, bit for bit against the
    oracle's counting sort, for each case and for the largest accepted size."""
    for i, (T, k, E, H) in enumerate(CASES):
        idx = _idx(T, k, E, 30 + i)
        x = synthetic.make_tokens(T, H, seed=30 + i).cuda()
        _matches_oracle(moe.moe_permute_static(idx, E, x), idx, E, x)
    E, k = 1024, 8
    T2 = (LIMIT // 2 // (E * 4)) * 1024 // k
    idx2 = _idx(T2, k, E, 33)
    _matches_oracle(moe.moe_permute_static(idx2, E), idx2, E)


def test_static_permute_two_calls_in_a_row_match_workspace_permute(moe):
    ins = [(_idx(T, k, E, 10 + i), synthetic.make_tokens(T, H, seed=10 + i).cuda(), E)
           for i, (T, k, E, H) in enumerate(CASES)]
    # back-to-back calls on the shared scratch, then the workspace entry point
    got = [moe.moe_permute_static(idx, E, x) for idx, x, E in ins]
    again = moe.moe_permute_static(ins[0][0], ins[0][2], ins[0][1])
    torch.cuda.synchronize()
    want = [moe.moe_permute(idx, E, x) for idx, x, E in ins]
    torch.cuda.synchronize()
    for g_, w_ in zip(got, want):
        _same(g_, w_)
    _same(again, want[0])
    # the permutation is a bijection onto the expert-sorted rows
    off, sp, pr, _ = got[0]
    assert torch.equal(pr[sp.long()], torch.arange(sp.numel(), dtype=torch.int32, device=sp.device))
    assert int(off[-1]) == sp.numel()


def test_static_permute_without_x_and_empty(moe):
    idx = _idx(3000, 4, 96, 21)
    _same(moe.moe_permute_static(idx, 96), moe.moe_permute(idx, 96))
    empty = torch.zeros(0, 4, dtype=torch.int32, device="cuda")
    off, sp, pr, _ = moe.moe_permute_static(empty, 16)
    assert sp.numel() == 0 and int(off.abs().sum()) == 0


def test_static_permute_rejects_scratch_beyond_limit(moe):
    T, k, E = 20000, 8, 1024          # ceil(160000 / 1024) * 1024 * 4 bytes, twice: > 1 MiB
    need = 2 * ((-(-T * k // 1024) * E * 4 + 255) // 256 * 256)
    assert need > LIMIT
    idx = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    n0 = moe.moe_kernel_launch_count()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_static(idx, E)
    assert ei.value.name == "UNSUPPORTED"
    assert moe.moe_kernel_launch_count() == n0   # rejected before anything was enqueued
    # the largest accepted size on the same expert count still runs and matches
    T2 = (LIMIT // 2 // (E * 4)) * 1024 // k
    idx2 = _idx(T2, k, E, 22)
    _same(moe.moe_permute_static(idx2, E), moe.moe_permute(idx2, E))
