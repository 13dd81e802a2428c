"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/gqa_attn.h declares, and rejects bad arguments on the
host before touching CUDA."""
import ctypes
import os
import re

import numpy as np
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


def test_checked_library_exports_every_declared_symbol():
    """The range-checked build (GQA_ATTN_DEBUG) exports the same C ABI."""
    from gqa_attention_flash_b200 import build
    lib = ctypes.CDLL(build.build(debug=True))
    for name in declared_functions():
        assert hasattr(lib, name), name


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


def flex(binding, **kw):
    a = dict(O=P, Q=P, K=P, V=P, LSE=None, B=1, Hq=2, Hkv=1, Sq=4, Sk=4, D=128, scale=0.1,
             causal=1, window=0, input_pos=0, k_lengths=None, q_lengths=None, softcap=0.0,
             alibi=None, doc_q=None, doc_kv=None, block_mask=None)
    a.update(kw)
    return binding.lib.attn_fwd_flex(a["O"], a["Q"], a["K"], a["V"], a["LSE"], a["B"], a["Hq"],
                                     a["Hkv"], a["Sq"], a["Sk"], a["D"], a["scale"], a["causal"],
                                     a["window"], a["input_pos"], a["k_lengths"], a["q_lengths"],
                                     a["softcap"], a["alibi"], a["doc_q"], a["doc_kv"],
                                     a["block_mask"], a.get("per_head", 0), None)


def test_flex_host_validation(binding):
    assert flex(binding, Hq=3, Hkv=2) == 2
    assert flex(binding, D=96) == 3
    assert flex(binding, softcap=-1.0) == 2
    assert flex(binding, softcap=float("inf")) == 2
    assert flex(binding, softcap=float("nan")) == 2
    assert flex(binding, softcap=5.0, alibi=P) == 2      # one score mod per call
    assert flex(binding, doc_q=P) == 2                   # ids for both sides or neither
    assert flex(binding, doc_kv=P) == 2
    assert flex(binding, alibi=ctypes.c_void_p(18)) == 2  # misaligned slopes
    assert flex(binding, Sk=128 * 1024 + 1) == 3          # longer than the flex kernel takes
    assert flex(binding, per_head=2) == 2
    assert flex(binding, B=0) == 0
    assert flex(binding, Sq=0, softcap=3.0) == 0


def _brute_block_states(keep):
    Sq, Sk = keep.shape
    out = np.zeros(((Sq + 63) // 64, (Sk + 63) // 64), np.uint8)
    for qb in range(out.shape[0]):
        for kb in range(out.shape[1]):
            blk = keep[qb * 64:(qb + 1) * 64, kb * 64:(kb + 1) * 64]
            out[qb, kb] = 2 if blk.all() else (1 if blk.any() else 0)
    return out


@pytest.mark.parametrize("Sq,Sk,causal,window,input_pos", [
    (150, 200, 0, 0, 0), (150, 200, 1, 0, 0), (150, 200, 1, 16, 0), (130, 200, 1, 0, 50),
    (64, 64, 1, 0, 0), (1, 300, 1, 7, 299)])
def test_block_mask_document_matches_brute_force(binding, Sq, Sk, causal, window, input_pos):
    import torch
    from gqa_attention_flash_b200 import workloads as W
    doc = W.document_ids(Sk, seed=Sq + Sk, min_len=1, max_len=70)
    dq = doc[input_pos:input_pos + Sq].clone()
    i = np.arange(Sq)[:, None] + input_pos
    j = np.arange(Sk)[None, :]
    keep = dq.numpy()[:, None] == doc.numpy()[None, :]
    if causal:
        keep &= j <= i
    if window:
        keep &= j > i - window
    bm = binding.block_mask_document(Sq, Sk, dq, doc, causal, window, input_pos)
    assert bm.dtype == torch.uint8 and tuple(bm.shape) == ((Sq + 63) // 64, (Sk + 63) // 64)
    assert np.array_equal(bm.numpy(), _brute_block_states(keep))
    bm2 = binding.block_mask_build(Sq, Sk, lambda q, kv: bool(keep[q - input_pos, kv]), input_pos)
    assert np.array_equal(bm2.numpy(), _brute_block_states(keep))


def test_block_mask_builder_validation(binding):
    L = binding.lib
    assert L.attn_block_mask_document(None, 4, 4, 0, 1, 0, P, P) == 1
    assert L.attn_block_mask_document(P, 4, 4, 0, 0, 3, P, P) == 2   # window needs causal
    assert L.attn_block_mask_document(P, -1, 4, 0, 1, 0, P, P) == 2
    assert L.attn_block_mask_document(P, 0, 4, 0, 1, 0, None, None) == 0


def test_decode_paged_host_validation(binding):
    L = binding.lib

    def dec(**kw):
        a = dict(O=P, Q=P, K=P, V=P, bt=P, lens=P, n_splits=8, B=2, Hq=8, Hkv=2, num_blocks=10,
                 block_size=16, max_blocks=4, D=128)
        a.update(kw)
        return L.attn_decode_paged(a["O"], a["Q"], a["K"], a["V"], a["bt"], a["lens"],
                                   a["n_splits"], None, a["B"], a["Hq"], a["Hkv"],
                                   a["num_blocks"], a["block_size"], a["max_blocks"], a["D"])
    assert dec(block_size=12) == 2      # not a power of two
    assert dec(block_size=4) == 2       # below 8
    assert dec(num_blocks=0) == 2
    assert dec(n_splits=0) == 2
    assert dec(Hq=6, Hkv=4) == 2
    assert dec(D=96) == 3
    assert dec(bt=None) == 1
    assert dec(lens=None) == 1
    assert dec(K=ctypes.c_void_p(24)) == 2
    assert dec(B=0) == 0


def test_paged_layout_helper():
    from gqa_attention_flash_b200 import workloads as W
    lengths = [5, 17, 0, 32, 48]
    tables, n = W.paged_layout(lengths, 16, 3, 1)
    used = tables[tables >= 0]
    assert n == 1 + 2 + 0 + 2 + 3 + 3
    assert len(set(used.tolist())) == used.numel() and int(used.max()) < n
    for b, ln in enumerate(lengths):
        nb = (ln + 15) // 16
        assert bool((tables[b, :nb] >= 0).all()) and bool((tables[b, nb:] == -1).all())


def test_rbs_host_validation(binding):
    L = binding.lib

    def rbs(**kw):
        a = dict(mask=P, base=None, resc=None, Q=P, K=P, B=1, Hq=4, Hkv=2, Sq=128, Sk=128, D=128,
                 ab=0.22, ar=0.18, diag=1)
        a.update(kw)
        return L.attn_rbs_block_mask(a["mask"], a["base"], a["resc"], a["Q"], a["K"], a["B"],
                                     a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["D"], a["ab"], a["ar"],
                                     a["diag"], None)
    assert rbs(Hq=3) == 2
    assert rbs(ab=0.0) == 2
    assert rbs(ar=float("nan")) == 2
    assert rbs(diag=-1) == 2
    assert rbs(D=96) == 3
    assert rbs(Sk=131073) == 3
    assert rbs(mask=None) == 1
    assert rbs(Q=ctypes.c_void_p(20)) == 2
    assert rbs(B=0) == 0


def test_bwd_host_validation(binding):
    L = binding.lib

    def bwd(**kw):
        a = dict(dQ=P, dK=P, dV=P, dO=P, Q=P, K=P, V=P, O=P, LSE=P, B=1, Hq=2, Hkv=1, Sq=4, Sk=4,
                 D=128, scale=0.1, causal=1, window=0, input_pos=0)
        a.update(kw)
        return L.attn_bwd(a["dQ"], a["dK"], a["dV"], a["dO"], a["Q"], a["K"], a["V"], a["O"],
                          a["LSE"], a["B"], a["Hq"], a["Hkv"], a["Sq"], a["Sk"], a["D"], a["scale"],
                          a["causal"], a["window"], a["input_pos"], None, None, None)
    assert bwd(Hq=3, Hkv=2) == 2                   # Hq % Hkv != 0
    assert bwd(D=96) == 3                          # head size not built
    assert bwd(causal=0, window=4) == 2            # window is causal only
    assert bwd(scale=0.0) == 2
    assert bwd(input_pos=-1) == 2
    for name in ("dQ", "dK", "dV", "dO", "LSE", "O", "Q"):
        assert bwd(**{name: None}) == 1, name      # NULL buffer with work to do
    assert bwd(dQ=ctypes.c_void_p(24)) == 2        # gradients must be 16-byte aligned
    assert bwd(dK=ctypes.c_void_p(40)) == 2
    assert bwd(LSE=ctypes.c_void_p(18)) == 2       # LSE must be 4-byte aligned
    assert bwd(B=0) == 0                           # nothing to do
