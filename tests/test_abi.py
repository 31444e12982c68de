"""The C-ABI library loads, exports every declared symbol, and rejects bad
configurations on the host before touching a device (CPU only)."""

import ctypes
import os
import re
import subprocess

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            names.update(re.findall(r"^ENGRAM_API\s+[\w\s\*]+?\b(engram_\w+)\s*\(", text, re.M))
    return names


@pytest.fixture(scope="module")
def eb():
    import hashed_gram_embedding_02_b200 as eb
    return eb


def test_header_declares_the_forward_path():
    names = _declared_symbols()
    for n in ("engram_remap", "engram_hash", "engram_gather", "engram_gate_conv", "engram_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(eb):
    lib = ctypes.CDLL(eb.LIB_PATH)
    declared = _declared_symbols()
    assert declared
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", eb.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(engram_\w+)$", out, re.M))
    assert declared == exported, (declared ^ exported)
    assert set(eb.EXPORTS) == declared


def test_library_is_built_for_sm100a(eb):
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", eb.LIB_PATH], capture_output=True,
                         text=True).stdout
    assert "sm_100a" in out


def _cfg(eb, wl=None, **over):
    wl = wl or synth.WORKLOADS["c2"]
    mult = synth.hash_multipliers(wl)
    kw = dict(orders=wl.orders, heads=wl.K, rows=[wl.M] * wl.J, mult=mult, row_dim=wl.D, hidden=wl.d,
              conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc,
              dtype=eb.ENGRAM_BF16 if wl.dtype == "bf16" else eb.ENGRAM_F32)
    kw.update(over)
    return eb.make_config(**kw)


@pytest.mark.parametrize("over,why", [
    (dict(rows=[1000001] * 16), "non-prime table size"),
    (dict(orders=(3, 2)), "orders not ascending"),
    (dict(orders=(2, 5)), "order above 4"),
    (dict(heads=17, rows=[1000003] * 32, mult=[[1, 1, 1, 0]] * 32), "more than 32 tables"),
    (dict(row_dim=60), "row not a multiple of 16 bytes"),
    (dict(hidden=2564), "hidden not a multiple of 8"),
    (dict(conv_width=9), "conv wider than 8"),
    (dict(canon_vocab=0), "empty canonical vocabulary"),
])
def test_create_rejects_bad_config_on_host(eb, over, why):
    cfg = _cfg(eb, **over)
    ctx = ctypes.c_void_p()
    from hashed_gram_embedding_02_b200 import binding
    st = binding._lib.engram_create(ctypes.byref(cfg), ctypes.byref(ctx))
    assert st == binding.ENGRAM_E_INVAL, why
    assert ctx.value is None
    assert eb.engram_last_error()


def test_null_context_is_rejected(eb):
    from hashed_gram_embedding_02_b200 import binding
    assert binding._lib.engram_forward(None, None, 1, 1, 1, 0, None, None, None, None, None, None, None, None,
                                       None, None, None, 0, None, 0, None) == binding.ENGRAM_E_INVAL
    assert eb.engram_workspace_bytes(None, 2, 10) == 0
    assert eb.engram_host_workspace_bytes(None, 2, 10, 0, 0) == 0
    assert binding._lib.engram_forward_host(None, None, 1, 1, 1, 0, None, None, None, None, None, None, None, None,
                                            None, None, 0, 0, None, 0, None) == binding.ENGRAM_E_INVAL
