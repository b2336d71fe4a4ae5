"""The C-ABI library loads, exports every declared entry point, and its host-only
logic (capacity, workspace sizing, argument validation) behaves -- no GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

from mixture_experts_sparse_b200 import native as nat
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert "moe_forward" in names and "moe_route" in names and len(names) >= 10
    handle = ctypes.CDLL(nat.LIB_PATH)
    for n in names:
        assert hasattr(handle, n), n
    assert set(nat._SIGS) >= set(names)


def declared_arity():
    """Number of parameters of every entry point declared in include/*.h."""
    out = {}
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", h)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(moe_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
            params = m.group(2).strip()
            out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header():
    # every ctypes signature has as many arguments as the C declaration
    arity = declared_arity()
    assert arity["moe_forward"] == 24 and arity["moe_ep_dispatch"] == 15
    for name, (args, _) in nat._SIGS.items():
        assert len(args) == arity[name], (name, len(args), arity[name])


def test_capacity_matches_oracle():
    rng = np.random.default_rng(0)
    cases = [(1024, 8, 2, 1.25), (65536, 64, 1, 1.25), (32768, 32, 2, 2.0), (16384, 8, 2, 1.25),
             (65536, 128, 1, 1.0), (512, 8, 1, 1.0), (10, 1, 1, 0.3), (10, 1, 1, 0.1), (0, 4, 1, 1.0),
             (7, 3, 2, 0.0), (-1, 2, 1, 1.0), (5, 0, 1, 1.0), (5, 2, 0, 1.0), (5, 2, 1, -0.5),
             (5, 2, 1, float("inf")), (5, 2, 1, float("nan")), ((1 << 27), 1, 2, 100.0)]
    for _ in range(500):
        cases.append((int(rng.integers(0, 1 << 24)), int(rng.integers(1, 129)), int(rng.integers(1, 3)),
                      float(rng.choice([0.5, 1.0, 1.25, 2.0, 0.3, 0.7, rng.random() * 5]))))
    for c in cases:
        assert nat.moe_capacity(*c) == oracle.capacity(*c), c


def test_workspace_bytes_and_validation():
    good = nat.config(4096, 768, 3072, 64, 1, 80)
    ws = nat.moe_workspace_bytes(good)
    rows = 4096
    assert ws >= rows * (768 * 2 * 2 + 3072 * 2)
    bad = [nat.config(-1, 768, 3072, 64, 1, 80), nat.config(16, 0, 3072, 64, 1, 80),
           nat.config(16, 768, 3072, 0, 1, 80), nat.config(16, 768, 3072, 4, 5, 80),
           nat.config(16, 768, 3072, 4, 1, -1), nat.config(16, 768, 3072, 129, 1, 8),
           nat.config(16, 760, 3072, 8, 1, 8), nat.config(16, 768, 3072, 2, 3, 8)]
    for cfg in bad:
        assert nat.moe_workspace_bytes(cfg) == 0
    assert nat.moe_workspace_bytes(nat.config(16, 760, 3072, 8, 1, 8, dtype="f32")) > 0
    # the batch-priority claim order needs its sort scratch on top; an unknown
    # claim order is rejected
    prio = nat.config(4096, 768, 3072, 64, 1, 80, priority=True)
    assert nat.moe_workspace_bytes(prio) >= ws + 4 * (2 * 65536 + 1 + 4 * 4096)
    odd = nat.config(4096, 768, 3072, 64, 1, 80)
    odd.priority = 3
    assert nat.moe_workspace_bytes(odd) == 0
    # re-routing keeps every token's probabilities and its stage state; top-1 only
    ntlb = nat.config(4096, 768, 3072, 64, 1, 80, priority=nat.MOE_ORDER_NTLB)
    assert nat.moe_workspace_bytes(ntlb) >= ws + 4 * 4096 * 64
    assert nat.moe_workspace_bytes(nat.config(4096, 768, 3072, 64, 2, 80, priority=nat.MOE_ORDER_NTLB)) == 0


def test_host_validation_rejects_before_launch():
    # every call below fails argument checks on the host, so no CUDA call is made
    P = ctypes.c_void_p
    lib = nat.lib()
    cfg = nat.config(64, 128, 256, 8, 1, 8)
    c = ctypes.byref(cfg)
    z = [None] * 30
    assert lib.moe_route(c, *z[:10], 0, None) == nat.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(c, *z[:21], 0, None) == nat.MOE_ERR_INVALID_ARG
    mis = P(0x1001)   # misaligned
    ok = P(0x1000)
    assert lib.moe_route(c, ok, mis, None, ok, ok, None, None, None, None, ok, 1 << 30, None) == \
        nat.MOE_ERR_INVALID_ARG
    # workspace too small / null
    assert lib.moe_route(c, ok, ok, None, ok, ok, None, None, None, None, ok, 16, None) == nat.MOE_ERR_WORKSPACE
    assert lib.moe_route(c, ok, ok, None, ok, ok, None, None, None, None, None, 1 << 30, None) == \
        nat.MOE_ERR_WORKSPACE
    unsup = nat.config(64, 128, 256, 200, 1, 8)
    assert lib.moe_route(ctypes.byref(unsup), *z[:10], 0, None) == nat.MOE_ERR_UNSUPPORTED
    assert lib.moe_combine(ctypes.byref(nat.config(64, 128, 256, 8, 3, 8)), *z[:8]) == nat.MOE_ERR_UNSUPPORTED
    assert lib.moe_read_device_status(None, None) == nat.MOE_ERR_WORKSPACE
    assert lib.moe_workspace_init(None, 1 << 20, None) == nat.MOE_ERR_WORKSPACE
    assert lib.moe_workspace_init(ok, 16, None) == nat.MOE_ERR_WORKSPACE
    assert lib.moe_test_lookback_timeout(ok, 1 << 20, 0, None) == nat.MOE_ERR_INVALID_ARG
    for s in range(6):
        assert nat.moe_status_string(s) != "unknown status"
    assert nat.moe_status_string(99) == "unknown status"


def test_native_raises_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(nat, "_lib", None)
    monkeypatch.setattr(nat, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(OSError):
        nat.lib()
