"""Planted mistakes in the oracle, caught by its pins. CPU only.

Each case edits one plausible error into a copy of the oracle (a wrong
exponent bias, a swapped nibble, a dropped term, a wrong sign or index, a
transposed operand, a broken cache rule), builds or loads that copy, and runs
every pin of test_oracle.py against it. At least one pin must fail. The copies
live under _build/planted; the oracle itself is never modified. Every planted
edit keeps all memory accesses inside the buffers the pins pass in.
"""
import os
import subprocess
import sys
import types

import pytest

import oracle
import test_oracle as pins
from conftest import ROOT

_DIR = os.path.join(ROOT, "_build", "planted")

# (name, exact text in oracle.c, replacement[, occurrences]). The text must occur exactly that many
# times (once unless stated); every occurrence is edited, so a mistake can sit in both the layer path
# and the per-token path at once.
C_PLANTS = [
    ("e2m1_exponent_bias", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)"),
    ("e2m1_subnormal_step", "(e == 0) ? 0.5 * m", "(e == 0) ? 1.0 * m"),
    ("e8m0_bias", "ldexp(1.0, code - 127)", "ldexp(1.0, code - 128)"),
    ("e4m3_exponent_bias", "ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    ("e4m3_subnormal_exponent", "ldexp(m / 8.0, -6)", "ldexp(m / 8.0, -7)"),
    ("e4m3_no_nan", "if (e == 15 && m == 7) return NAN;", ""),
    ("fp4_nibble_order", "(c & 1) ? (byte >> 4) : (byte & 15)", "(c & 1) ? (byte & 15) : (byte >> 4)"),
    ("mxfp4_scale_block_64", "(size_t)r * (K / 32) + c / 32]", "(size_t)r * (K / 32) + c / 64]"),
    ("mxfp4_scale_row_dropped", "(size_t)r * (K / 32) + c / 32]", "c / 32]"),
    ("nvfp4_tensor_scale_dropped", "v = (q * s) * tscale;", "v = q * s;"),
    ("nvfp4_scale_block_32", "(size_t)r * (K / 16) + c / 16]", "(size_t)r * (K / 16) + c / 32]"),
    ("fp8_scale_row_dropped", "(size_t)r * (K / 128) + c / 128]", "c / 128]"),
    ("bf16_round_half_up", "u += 0x7fffu + lsb;", "u += 0x7fffu;"),
    ("bf16_truncate", "u += 0x7fffu + lsb;", "u += 0;"),
    ("router_fp32_sum", "double acc = 0.0;\n            for (int h = 0; h < H; ++h) {",
     "float acc = 0.0f;\n            for (int h = 0; h < H; ++h) {"),
    ("router_bias_before_rounding", "float lf = (float)acc;\n            if (bias) lf = lf + bias[e];",
     "float lf = (float)(bias ? acc + bias[e] : acc);"),
    ("router_weight_transposed", "((const float *)wr)[(size_t)h * E + e]", "((const float *)wr)[(size_t)e * H + h]"),
    ("topk_ties_to_higher_index", "if (best < 0 || l[e] > l[best]) best = e;",
     "if (best < 0 || l[e] >= l[best]) best = e;"),
    ("topk_ascending", "if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] < l[best]) best = e;"),
    ("gating_sign", "w[(size_t)t * k + j] = expf(l[order[j]] - l0) / z;",
     "w[(size_t)t * k + j] = expf(l0 - l[order[j]]) / z;"),
    ("gating_not_normalised", "w[(size_t)t * k + j] = expf(l[order[j]] - l0) / z;",
     "w[(size_t)t * k + j] = expf(l[order[j]] - l0);"),
    ("permutation_descending_within_expert", "int r = offsets[e] + fill[e]++;",
     "int r = offsets[e + 1] - 1 - fill[e]++;"),
    ("silu_sign", "return z / (1.0f + expf(-z));", "return z / (1.0f + expf(z));"),
    ("silu_dropped", "float hv = bf16_to_f32(f32_to_bf16(silu(g) * u));",
     "float hv = bf16_to_f32(f32_to_bf16(g * u));"),
    ("gate_up_swapped", "*wg = w13f + (size_t)i * H, *wu = w13f + (size_t)(I + i) * H;",
     "*wu = w13f + (size_t)i * H, *wg = w13f + (size_t)(I + i) * H;"),
    ("h_not_rounded_to_bf16", "float hv = bf16_to_f32(f32_to_bf16(silu(g) * u));", "float hv = silu(g) * u;"),
    ("down_projection_transposed", "for (int i = 0; i < I; ++i) acc += hbuf[i] * w2r[i];",
     "for (int i = 0; i < I; ++i) acc += hbuf[i] * w2f[(size_t)i * H + j];"),
    ("token_of_row_modulo", "tok[r] = sorted_pair[offsets[e] + r] / k;", "tok[r] = sorted_pair[offsets[e] + r] % k;"),
    ("expert_stride_of_w2_used_for_w13",
     "\n        bad |= oracle_dequant(fmt, 2 * I, H, (const char *)w13 + e * b13,",
     "\n        bad |= oracle_dequant(fmt, 2 * I, H, (const char *)w13 + e * b2,"),
    ("combine_first_gate_only", "acc += w[(size_t)t * k + j] * y_perm[(size_t)r * H + c];",
     "acc += w[(size_t)t * k] * y_perm[(size_t)r * H + c];"),
    ("combine_skips_pair_row", "int r = pair_row[(size_t)t * k + j];", "int r = t * k + j;"),
    ("logits_written_before_bias",
     "            float lf = (float)acc;\n            if (bias) lf = lf + bias[e];\n            l[e] = lf;\n"
     "            if (logits) logits[(size_t)t * E + e] = lf;",
     "            float lf = (float)acc;\n            if (logits) logits[(size_t)t * E + e] = lf;\n"
     "            if (bias) lf = lf + bias[e];\n            l[e] = lf;"),
    ("router_bf16_weight_transposed", "bf16_to_f32(((const uint16_t *)wr)[(size_t)h * E + e])",
     "bf16_to_f32(((const uint16_t *)wr)[(size_t)e * H + h])"),
    ("gating_sum_skips_last", "for (int j = 0; j < k; ++j) z += expf(l[order[j]] - l0);",
     "for (int j = 0; j + 1 < k; ++j) z += expf(l[order[j]] - l0);"),
    ("offsets_scan_stops_early", "for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];",
     "for (int e = 0; e + 1 < E; ++e) offsets[e + 1] += offsets[e];"),
    ("nvfp4_multiplication_order", "v = (q * s) * tscale;", "v = q * (s * tscale);"),
    ("silu_of_up_instead_of_gate", "float hv = bf16_to_f32(f32_to_bf16(silu(g) * u));",
     "float hv = bf16_to_f32(f32_to_bf16(silu(u) * g));"),
    ("down_projection_drops_last_channel", "for (int i = 0; i < I; ++i) acc += hbuf[i] * w2r[i];",
     "for (int i = 0; i + 1 < I; ++i) acc += hbuf[i] * w2r[i];"),
    ("combine_pair_row_transposed", "int r = pair_row[(size_t)t * k + j];", "int r = pair_row[(size_t)j * T + t];"),
    ("w13_scale_stride_of_w2", "w13s ? (const char *)w13s + e * s13 : 0,", "w13s ? (const char *)w13s + e * s2 : 0,",
     2),
    ("w2_scale_of_expert_0", "w2s ? (const char *)w2s + e * s2 : 0,", "w2s ? (const char *)w2s : 0,", 2),
    ("w13_tensor_scale_of_expert_0", "w13t ? w13t[e] : 1.0f", "w13t ? w13t[0] : 1.0f", 2),
    ("w2_tensor_scale_of_expert_0", "w2t ? w2t[e] : 1.0f", "w2t ? w2t[0] : 1.0f", 2),
    # activation format A4
    ("a4_e2m1_ties_to_odd", "if (d < bd || (d == bd && (c & 1) == 0)) {\n            best = c;\n            bd = d;\n"
     "        }\n    }\n    return best | sgn;",
     "if (d < bd || (d == bd && (c & 1) == 1)) {\n            best = c;\n            bd = d;\n"
     "        }\n    }\n    return best | sgn;"),
    ("a4_e4m3_ties_to_odd", "if (d < bd || (d == bd && (c & 1) == 0)) {\n            best = c;\n            bd = d;\n"
     "        }\n    }\n    return best;",
     "if (d < bd || (d == bd && (c & 1) == 1)) {\n            best = c;\n            bd = d;\n"
     "        }\n    }\n    return best;"),
    ("a4_e2m1_saturates_at_4", "if (a >= 6.0) return 7 | sgn;", "if (a >= 4.0) return 6 | sgn;"),
    ("a4_tensor_scale_without_6", "amax / (6.0f * 448.0f)", "amax / 448.0f"),
    ("a4_block_scale_without_6", "int sc = e4m3_rn_sat((amax / 6.0f) / s_g);", "int sc = e4m3_rn_sat(amax / s_g);"),
    ("a4_block_amax_first_half", "for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[b + i]));",
     "for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[b + i]));"),
    ("a4_block_scale_not_rounded", "float sb = (float)oracle_e4m3(sc);",
     "float sb = (amax / 6.0f) / s_g; (void)sc;"),
    ("a4_x_not_quantised", "if (act == ACT_A4) oracle_a4_quant(xr, H, s_gx, xr, 0, 0);", ""),
    ("a4_h_with_the_tensor_scale_of_x", "oracle_a4_quant(hbuf, I, 1.0f, hbuf, 0, 0);",
     "oracle_a4_quant(hbuf, I, s_gx, hbuf, 0, 0);"),
    ("a4_h_not_quantised", "            oracle_a4_quant(hbuf, I, 1.0f, hbuf, 0, 0);\n", ""),
    ("a4_tensor_scale_of_first_token", "oracle_a4_tensor_scale(x, (size_t)T * H)", "oracle_a4_tensor_scale(x, (size_t)H)",
     2),
]

# (name, exact text in lru.py, replacement).
LRU_PLANTS = [
    ("evicts_most_recent", "s = min(cand, key=lambda i: (self.stamp[i], i))",
     "s = max(cand, key=lambda i: (self.stamp[i], i))"),
    ("previous_call_unprotected", "if self.ref_call[i] < c - 1]", "if self.ref_call[i] < c]"),
    ("highest_free_slot", "s = free[0]", "s = free[-1]"),
    ("ids_in_request_order", "ids = sorted(set(int(i) for i in ids))", "ids = list(dict.fromkeys(int(i) for i in ids))"),
    ("prefetch_counts_hits", "        if count:\n", "        if True:\n"),
    ("failed_call_not_rolled_back",
     "                        (self.owner, self.stamp, self.ref_call, self.slot_of, self.clock) = snapshot\n", ""),
    ("hit_not_refreshed", "                hits += 1\n", "                hits += 1\n                continue\n"),
    ("evict_ignores_layer", "            if layer >= 0 and o[0] != layer:\n                continue\n", ""),
    ("evict_ignores_ids", "            if ids is not None and o[1] not in set(ids):\n                continue\n", ""),
    ("prediction_least_routed_first", "ranked = sorted(counts, key=lambda e: (-min(counts[e], (1 << 20) - 1), e))",
     "ranked = sorted(counts, key=lambda e: (min(counts[e], (1 << 20) - 1), e))"),
    ("prediction_ties_to_higher_id", "ranked = sorted(counts, key=lambda e: (-min(counts[e], (1 << 20) - 1), e))",
     "ranked = sorted(counts, key=lambda e: (-min(counts[e], (1 << 20) - 1), -e))"),
    ("resize_keeps_least_recent", "keep = occ[len(occ) - min(len(occ), n_slots):]", "keep = occ[:min(len(occ), n_slots)]"),
    ("resize_moves_to_highest_free", "f = min(j for j in range(n_slots) if self.owner[j] is None)",
     "f = max(j for j in range(n_slots) if self.owner[j] is None)"),
]

PARAMS = {"test_permutation_is_stable_counting_sort": [(16, 2, 8), (64, 8, 128)],
          "test_quantised_layer_matches_per_token_brute_force_fp64": [("fp8",), ("mxfp4",), ("nvfp4",)]}


def _pins():
    out = []
    for name in sorted(dir(pins)):
        if name.startswith("test_"):
            fn = getattr(pins, name)
            for args in PARAMS.get(name, [()]):
                out.append((name, fn, args))
    return out


def _failing_pins():
    failed = []
    for name, fn, args in _pins():
        try:
            fn(*args)
        except (Exception, pytest.fail.Exception):
            failed.append(name)
    return failed


def _plant(text, old, new, n=1):
    assert text.count(old) == n, f"planting text occurs {text.count(old)} times, not {n}: {old!r}"
    return text.replace(old, new)


def test_unplanted_oracle_passes_every_pin():
    assert _failing_pins() == []


@pytest.mark.parametrize("plant", C_PLANTS, ids=[p[0] for p in C_PLANTS])
def test_planted_c_mistake_is_caught(plant, monkeypatch):
    name = plant[0]
    os.makedirs(_DIR, exist_ok=True)
    src = _plant(open(oracle._SRC).read(), *plant[1:])
    c = os.path.join(_DIR, f"{name}.c")
    so = os.path.join(_DIR, f"{name}.{os.getpid()}.so")
    with open(c, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", c, "-o", so, "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle._bind(so))
    assert _failing_pins(), f"no pin fails with '{name}' planted"


@pytest.mark.parametrize("name,old,new", LRU_PLANTS, ids=[p[0] for p in LRU_PLANTS])
def test_planted_lru_mistake_is_caught(name, old, new, monkeypatch):
    path = os.path.join(os.path.dirname(oracle.__file__), "lru.py")
    mod = types.ModuleType(f"planted_lru_{name}")
    exec(compile(_plant(open(path).read(), old, new), path, "exec"), mod.__dict__)
    sys.modules.pop(mod.__name__, None)
    monkeypatch.setattr(pins, "LruSim", mod.LruSim)
    monkeypatch.setattr(pins, "CacheFull", mod.CacheFull)
    assert _failing_pins(), f"no pin fails with '{name}' planted"
