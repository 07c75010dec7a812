"""The byte accounting behind the bench's roofline figures, on the CPU.

achieved = algorithmic bytes / time, so the bytes must be what the format
stores: these tests tie bench.active_expert_bytes and synthetic.expert_bytes
to the tensors the generator actually builds, and to the closed forms of the
format definitions (codes plus scales per element)."""
import numpy as np
import pytest
import torch

import bench
import synthetic

# bytes per stored element: codes + scales (MXFP4: E8M0 per 32; NVFP4: E4M3 per 16; FP8: fp32 per 128)
PER_ELEMENT = {"bf16": 2.0, "fp8": 1 + 4 / 128, "mxfp4": 0.5 + 1 / 32, "nvfp4": 0.5 + 1 / 16}


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "mxfp4", "nvfp4"])
def test_expert_bytes_equal_the_generated_tensors(fmt):
    H, I, E = 256, 512, 4
    L = synthetic.make_layer(dict(H=H, E=E, k=2, I=I, fmt=fmt), 3)
    stored = 0
    for name in ("w13", "w2", "w13_scale", "w2_scale", "w13_tscale", "w2_tscale"):
        t = getattr(L, name, None)
        if t is not None:
            stored += t.numel() * t.element_size()
    assert stored % E == 0
    assert synthetic.expert_bytes(fmt, H, I) == stored // E


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "mxfp4", "nvfp4"])
def test_expert_bytes_closed_form(fmt):
    for H, I in ((2048, 768), (4096, 2048)):
        want = 3 * H * I * PER_ELEMENT[fmt] + (8 if fmt == "nvfp4" else 0)   # NVFP4: two fp32 tensor scales
        assert synthetic.expert_bytes(fmt, H, I) == want


def test_per_expert_bytes_of_the_workloads():
    # decode: w13 [1536][2048] and w2 [2048][768] at 0.53125 bytes per element
    assert synthetic.expert_bytes("mxfp4", 2048, 768) == 2_506_752
    # Large: [4096][4096] and [4096][2048] at 0.5625 bytes per element, plus two fp32 tensor scales
    assert synthetic.expert_bytes("nvfp4", 4096, 2048) == 14_155_784


def test_active_expert_bytes_count_each_used_expert_once():
    L = synthetic.make_layer(dict(H=256, E=8, k=2, I=256, fmt="mxfp4"), 1)
    per = synthetic.expert_bytes("mxfp4", 256, 256)
    idx = torch.tensor([[0, 1], [1, 3], [3, 0]], dtype=torch.int32)
    assert bench.active_expert_bytes(idx, L) == 3 * per
    assert bench.active_expert_bytes(torch.arange(8, dtype=torch.int32).reshape(4, 2), L) == 8 * per
    g = np.random.default_rng(0)
    idx = torch.from_numpy(np.stack([g.choice(8, 2, replace=False) for _ in range(50)]).astype(np.int32))
    assert bench.active_expert_bytes(idx, L) == len(set(idx.flatten().tolist())) * per


class _Replay:
    """Stands in for a CUDA graph: records the layer calls a replay would run."""

    def __init__(self, log, calls):
        self.log, self.calls = log, calls

    def replay(self):
        self.log.extend(self.calls)


@pytest.mark.parametrize("i0,n", [(0, 20), (20, 2000), (0, 3), (5, 16), (16, 32), (7, 41)])
def test_layer_bench_runs_exactly_the_steps_asked_for(i0, n):
    """bench.LayerBench.run(i0, n) replays the 16-call sequence graph only where a block of 16
    steps starts at a multiple of 16 and single-call graphs elsewhere: the layer calls it runs
    are exactly steps i0 .. i0 + n - 1, each on weight set step % 16, in order."""
    log = []
    lb = bench.LayerBench.__new__(bench.LayerBench)
    ns = bench.NSETS
    lb.graphs = [_Replay(log, [j]) for j in range(ns)]
    lb.seq = _Replay(log, list(range(ns)))
    lb.run(i0, n)
    assert log == [i % ns for i in range(i0, i0 + n)]
