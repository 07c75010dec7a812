"""The synthetic routing recipe against what the workloads ask for, on the CPU.

The prefill and Large workloads route with Zipf-skewed expert popularity "so
nearly every expert receives tokens"; the decode workload routes uniformly.
The generator draws a per-expert bias b[e] = (sigma_l / (pi/sqrt 6)) ln p_e
(synthetic.zipf_bias). These tests route seeded batches through the oracle's
router and check the outcome: with the Zipf bias, selection counts follow the
popularity order and nearly every expert is used; without it, the counts stay
close to uniform."""
import numpy as np

import oracle
import synthetic


def _counts(cfg, T, seed=0):
    c = synthetic.CONFIGS[cfg]
    wr, bias = synthetic.make_router(cfg, seed)
    x = synthetic.make_tokens(T, c["H"], seed=seed + 7)
    idx, w, _ = oracle.route(x, wr, c["k"], bias=bias, with_logits=False)
    return bias, np.bincount(idx.ravel(), minlength=c["E"])


def _ranks(v):
    return np.argsort(np.argsort(v, kind="stable"), kind="stable").astype(np.float64)


def _spearman(a, b):
    ra, rb = _ranks(a), _ranks(b)
    ra -= ra.mean()
    rb -= rb.mean()
    return float((ra * rb).sum() / np.sqrt((ra * ra).sum() * (rb * rb).sum()))


def test_zipf_routing_follows_popularity_and_reaches_nearly_every_expert():
    # the prefill-shaped workload: T = 4096, E = 128, top-8, Zipf(s = 1.1) popularity
    bias, counts = _counts("prefill", 4096)
    E = len(counts)
    # popularity of each expert, recovered from the bias: ln p_e is proportional to b[e]
    b = bias.double().numpy()
    assert _spearman(counts, b) > 0.9
    assert (counts > 0).sum() >= 0.95 * E
    # the most popular expert is chosen far more often than the least popular
    assert counts[np.argmax(b)] > 4 * max(counts[np.argmin(b)], 1)


def test_uniform_routing_stays_close_to_uniform():
    bias, counts = _counts("decode", 4096)
    assert bias is None or not np.any(bias.numpy())
    mean = counts.sum() / len(counts)   # 4096 * 8 / 128 = 256 pairs per expert
    assert counts.min() > 0.6 * mean and counts.max() < 1.5 * mean
