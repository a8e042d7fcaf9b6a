"""The bounds-checking debug build (ATTN_DEBUG_BOUNDS=1, libattn_b200_debug.so).

CPU: it builds, exports every call of include/attn.h, says it is the debug
build, and the header's site list matches the binding's. GPU (child
processes with ATTN_B200_DEBUG_BOUNDS=1): every call family runs through it
with a clear error word and oracle-exact results; and with each site planted
in turn, the word names exactly that site while the results stay the
oracle's (a planted check reports without changing the access)."""
import ctypes
import json
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")
SCRIPT = os.path.join(ROOT, "tests", "bounds_debug_cases.py")


def _declared_functions():
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def debug_lib():
    from attention_tiled_exact_b200 import build as _build
    path = _build.build(debug=True)
    return path, ctypes.CDLL(path)


def test_debug_library_exports_every_declared_symbol(debug_lib):
    path, _ = debug_lib
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing


def test_debug_and_release_report_their_build(debug_lib, lib):
    _, dl = debug_lib
    dl.attn_debug_plant_bounds.argtypes = [ctypes.c_int]
    assert dl.attn_debug_bounds_enabled() == 1
    assert dl.attn_debug_plant_bounds(300) == lib.ATTN_ERR_INVALID_ARG
    assert dl.attn_debug_plant_bounds(3) == lib.ATTN_OK
    assert dl.attn_debug_plant_bounds(0) == lib.ATTN_OK
    if not lib.DEBUG_BOUNDS:
        assert lib.LIB.attn_debug_bounds_enabled() == 0
        assert lib.LIB.attn_debug_plant_bounds(3) == lib.ATTN_ERR_UNSUPPORTED


def test_header_sites_match_the_binding(lib):
    src = open(HEADER).read()
    sites = {m.group(1): int(m.group(2)) for m in re.finditer(r"ATTN_SITE_(\w+)\s*=\s*(\d+)", src)}
    sites.pop("NONE")
    assert sites == lib.BOUNDS_SITES
    assert re.search(r"#define ATTN_FAULT_BOUNDS 0x10\b", src) and lib.ATTN_FAULT_BOUNDS == 0x10
    assert lib.fault_site((7 << 16) | 0x10 | 0x1) == 7


def _run_cases(*args):
    env = dict(os.environ, ATTN_B200_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, SCRIPT, *args], capture_output=True, text=True, timeout=900, env=env)
    assert r.returncode == 0, r.stdout + r.stderr
    return [json.loads(line) for line in r.stdout.splitlines() if line.startswith("{")]


def _close(res):
    tol_o = 1e-2 if res["case"] != "backward" else 1e-2  # backward: relative to max|ref| per gradient
    return res["err_o"] <= tol_o and res["err_lse"] <= 1e-3


@pytest.mark.gpu
def test_every_call_family_is_clean_under_the_checks():
    results = _run_cases()
    assert len(results) == 7
    for res in results:
        assert res["word"] == 0, res
        assert _close(res), res


@pytest.mark.gpu
def test_each_planted_site_is_reported_and_nothing_else_changes():
    from attention_tiled_exact_b200 import binding as attn
    results = _run_cases("--plant")
    assert [r["site"] for r in results] == list(attn.BOUNDS_SITES.values())
    for res in results:
        assert res["word"] == (res["site"] << 16) | attn.ATTN_FAULT_BOUNDS, res
        assert res["status"] == attn.ATTN_ERR_DEVICE_FAULT, res
        assert _close(res), res
