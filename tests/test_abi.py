"""The C-ABI library loads and exports every entry point its header declares (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ds4moe.h")


@pytest.fixture(scope="module")
def pkg():
    import __graft_entry__
    __graft_entry__.build_library()
    import bit_quantized_routed_sqrt_b200 as m
    return m


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"\b(ds4moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = declared()
    for n in ["ds4moe_create", "ds4moe_destroy", "ds4moe_load_q2k_experts", "ds4moe_route", "ds4moe_forward",
              "ds4moe_forward_host", "ds4moe_rms_renorm", "ds4moe_sync_status", "ds4moe_status_string",
              "ds4moe_last_error"]:
        assert n in names


def test_library_exports_every_declared_symbol(pkg):
    out = subprocess.check_output(["nm", "-D", "--defined-only", pkg.LIB_PATH]).decode()
    exported = set(re.findall(r"\bT (ds4moe_\w+)", out))
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(pkg.LIB_PATH)
    for n in declared():
        assert getattr(lib, n) is not None


def test_binding_has_the_same_names(pkg):
    methods = set(dir(pkg.Ds4Moe)) | set(dir(pkg))
    for n in declared():
        if n in ("ds4moe_create", "ds4moe_destroy", "ds4moe_last_error"):
            continue  # constructor, close() and error text of the handle class
        assert n in methods, n


def test_status_strings_without_gpu(pkg):
    assert pkg.ds4moe_status_string(0) == "ok"
    assert pkg.ds4moe_status_string(1) == "invalid argument"
    assert pkg.ds4moe_status_string(5).startswith("device-side wait")


@pytest.mark.parametrize("bad", [
    dict(hidden=300), dict(hidden=0), dict(inter=100), dict(n_experts=0), dict(n_experts=300),
    dict(top_k=0), dict(top_k=9, n_experts=8), dict(top_k=17), dict(shared_inter=128), dict(max_tokens=0),
])
def test_create_rejects_bad_config_before_touching_cuda(pkg, bad):
    cfg = dict(hidden=256, n_experts=8, top_k=2, inter=256, shared_inter=256, max_tokens=4, flags=0)
    cfg.update(bad)
    c = pkg.ds4moe_config(cfg["hidden"], cfg["n_experts"], cfg["top_k"], cfg["inter"], cfg["shared_inter"],
                          cfg["max_tokens"], cfg["flags"])
    h = ctypes.c_void_p()
    rc = pkg.lib.ds4moe_create(ctypes.byref(c), 0, ctypes.byref(h))
    assert rc == 1 and not h.value


def test_null_handle_calls_are_rejected(pkg):
    assert pkg.lib.ds4moe_forward(None, None, 1, None, None) == 1
    assert pkg.lib.ds4moe_sync_status(None) == 1
    pkg.lib.ds4moe_destroy(None)


def test_injected_allocation_failure_without_gpu(pkg, monkeypatch):
    """DS4MOE_FAULT=alloc: ds4moe_create reports ENOMEM (not a CUDA error) before it touches
    CUDA, so this runs on a machine without a GPU; without the variable the same call on
    such a machine fails with ECUDA instead."""
    c = pkg.ds4moe_config(256, 8, 2, 256, 256, 4, 0)
    h = ctypes.c_void_p()
    monkeypatch.setenv("DS4MOE_FAULT", "alloc")
    assert pkg.lib.ds4moe_create(ctypes.byref(c), 0, ctypes.byref(h)) == 2 and not h.value
    monkeypatch.delenv("DS4MOE_FAULT")
    import torch
    if not torch.cuda.is_available():
        assert pkg.lib.ds4moe_create(ctypes.byref(c), 0, ctypes.byref(h)) == 3 and not h.value
