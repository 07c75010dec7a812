"""CPU checks of the C ABI: the library builds for sm_100a, loads, and exports
every function include/moe.h declares; host-only calls behave. No GPU needed."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    with open(HEADER) as fh:
        src = fh.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\**\s*\**([a-z_][a-z_0-9]*)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n.startswith(("moe_", "expert_cache_"))))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("moe_route_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_layer_forward",
                 "moe_workspace_size", "expert_cache_init", "expert_cache_prefetch", "expert_cache_evict",
                 "expert_cache_stats", "expert_cache_destroy", "moe_last_error_string", "moe_dequantize"):
        assert want in names


def test_library_builds_and_exports_every_declared_symbol():
    from expert_ffn_layer_top_b200 import build

    path = build.build()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if " T " in l)
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing


def test_library_loads_and_host_only_calls_work():
    import expert_ffn_layer_top_b200 as moe

    L = moe.lib()
    assert moe.moe_version().startswith("libmoe")
    # workspace sizing is host arithmetic only
    a = moe.moe_workspace_size(1024, 2048, 768, 128, 8)
    b = moe.moe_workspace_size(2048, 2048, 768, 128, 8)
    assert 0 < a < b
    assert moe.moe_workspace_size(-1, 2048, 768, 128, 8) == 0
    assert L.moe_last_error_string() is not None


def test_binding_has_the_abi_names():
    import expert_ffn_layer_top_b200 as moe

    for n in ("moe_route_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_layer_forward",
              "moe_workspace_size", "moe_dequantize", "ExpertCache"):
        assert hasattr(moe, n)


def test_product_package_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "expert_ffn_layer_top_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    txt = fh.read()
                assert "oracle" not in txt.lower().replace("oracle.", "oracle"), f
