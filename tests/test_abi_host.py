"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/gqa_attn.h declares, and rejects bad arguments on the
host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


@pytest.fixture(scope="module")
def binding():
    from gqa_attention_flash_b200 import build
    build.build()
    from gqa_attention_flash_b200 import binding as b
    return b


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(attn_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ["attn_fwd", "attn_fwd_varlen", "attn_decode", "attn_status_string",
                 "attn_last_device_status", "attn_check_bounded_wait"]:
        assert must in names


def test_library_exports_every_declared_symbol(binding):
    for name in declared_functions():
        assert hasattr(binding.lib, name), name
        assert isinstance(getattr(binding.lib, name), ctypes._CFuncPtr)


def test_status_strings(binding):
    for code, name in binding.STATUS.items():
        assert binding.status_string(code).startswith(name)
    assert "unknown" in binding.status_string(99)


P = ctypes.c_void_p(16)  # non-NULL, 16-byte aligned; never dereferenced on these paths


def fwd(binding, **kw):
    a = dict(O=P, Q=P, K=P, V=P, LSE=None, B=1, Hq=2, Hkv=1, Sq=4, Sk=4, D=128, scale=0.1,
             causal=1, window=0, input_pos=0, k_lengths=None)
    a.update(kw)
    return binding.lib.attn_fwd(a["O"], a["Q"], a["K"], a["V"], a["LSE"], a["B"], a["Hq"],
                                a["Hkv"], a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"],
                                a["window"], a["input_pos"], a["k_lengths"], None)


def test_fwd_host_validation(binding):
    assert fwd(binding, Hq=3, Hkv=2) == 2          # Hq % Hkv != 0
    assert fwd(binding, D=96) == 3                 # head size not built
    assert fwd(binding, D=256) == 3
    assert fwd(binding, O=None) == 1
    assert fwd(binding, K=None) == 1
    assert fwd(binding, causal=0, window=4) == 2   # window is causal only
    assert fwd(binding, B=-1) == 2
    assert fwd(binding, input_pos=-3) == 2
    assert fwd(binding, scale=0.0) == 2
    assert fwd(binding, scale=float("nan")) == 2
    assert fwd(binding, Q=ctypes.c_void_p(18)) == 2  # misaligned
    assert fwd(binding, causal=2) == 2
    assert fwd(binding, B=0) == 0                  # nothing to do
    assert fwd(binding, Sq=0) == 0


def test_decode_host_validation(binding):
    L = binding.lib

    def dec(**kw):
        a = dict(O=P, Q=P, K=P, V=P, lengths=P, n_splits=8, B=2, Hq=8, Hkv=2, S_cap=64, D=128)
        a.update(kw)
        return L.attn_decode(a["O"], a["Q"], a["K"], a["V"], a["lengths"], a["n_splits"], None,
                             a["B"], a["Hq"], a["Hkv"], a["S_cap"], a["D"])
    assert dec(n_splits=0) == 2
    assert dec(n_splits=65) == 2
    assert dec(Hq=6, Hkv=4) == 2
    assert dec(Hq=34, Hkv=2) == 2                  # more than 16 query heads per KV head
    assert dec(D=80) == 3
    assert dec(lengths=None) == 1
    assert dec(O=None) == 1
    assert dec(B=0) == 0


def test_bounded_wait_argument_range(binding):
    assert binding.lib.attn_check_bounded_wait(0, None) == 2
    assert binding.lib.attn_check_bounded_wait(3_000_000, None) == 2
