"""attn_decode_noalloc, the decode entry point for callers that cannot allocate
device memory (a serving loop that reserved all of its memory up front, or a
program whose memory belongs to another allocator): called through the C ABI,
it must give the same output as attn_decode, on two calls in a row with
different inputs (the second call sees the first call's leftovers in the shared
fixed array), and must refuse a workspace larger than its 16 MiB array.

This file is named so that pytest collects it last."""
import ctypes

import pytest
import torch

from gpu_common import O_TOL

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Hq, Hkv, S_cap, D):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    lengths = torch.randint(1, S_cap + 1, (B,), generator=g).to(torch.int32)
    dev = torch.device("cuda")
    return Q.to(dev), K.to(dev), V.to(dev), lengths.to(dev)


def _call(fn, O, Q, K, V, lengths, n_splits):
    B, Hq, D = Q.shape
    _, Hkv, S_cap, _ = K.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(ctypes.c_void_p(O.data_ptr()), ctypes.c_void_p(Q.data_ptr()),
              ctypes.c_void_p(K.data_ptr()), ctypes.c_void_p(V.data_ptr()),
              ctypes.c_void_p(lengths.data_ptr()), n_splits, stream, B, Hq, Hkv, S_cap, D)


def test_noalloc_matches_allocating_decode_twice():
    from gqa_attention_flash_b200 import binding
    lib = binding.lib
    cases = [(1, 6, 32, 8, 3000, 128, 8), (2, 9, 16, 4, 1500, 64, 5)]
    for seed, B, Hq, Hkv, S_cap, D, n_splits in cases:
        Q, K, V, lengths = _inputs(seed, B, Hq, Hkv, S_cap, D)
        ref = torch.empty_like(Q)
        assert _call(lib.attn_decode, ref, Q, K, V, lengths, n_splits) == 0
        out = torch.full_like(Q, float("nan"))
        assert _call(lib.attn_decode_noalloc, out, Q, K, V, lengths, n_splits) == 0
        assert binding.last_device_status() == 0
        assert torch.all(torch.isfinite(out.float()))
        d = float((out.float() - ref.float()).abs().max())
        assert d <= O_TOL, (seed, d)


def test_noalloc_same_shape_shorter_lengths():
    """Two calls of one shape in a row: the first with long sequences fills every
    slice of the shared array; the second, with much shorter sequences, leaves
    most slices empty.  Those slices still hold the first call's partials, and
    they must not reach the second call's output."""
    from gqa_attention_flash_b200 import binding
    lib = binding.lib
    B, Hq, Hkv, S_cap, D, n_splits = 4, 16, 4, 4096, 128, 8
    Q, K, V, _ = _inputs(5, B, Hq, Hkv, S_cap, D)
    for lens in ([4096, 4000, 3900, 4096], [1, 65, 130, 0]):
        lengths = torch.tensor(lens, dtype=torch.int32, device=Q.device)
        ref = torch.empty_like(Q)
        assert _call(lib.attn_decode, ref, Q, K, V, lengths, n_splits) == 0
        out = torch.full_like(Q, float("nan"))
        assert _call(lib.attn_decode_noalloc, out, Q, K, V, lengths, n_splits) == 0
        assert binding.last_device_status() == 0
        assert torch.all(torch.isfinite(out.float()))
        d = float((out.float() - ref.float()).abs().max())
        assert d <= O_TOL, (lens, d)
    assert torch.all(out[3] == 0)  # length 0: no slice has a key


def test_noalloc_full_decode_shape_fits():
    """The benchmark's decode shape (B64 Hq32 n_splits 8 D128: 8.65 MB of
    workspace) fits in the fixed array; called through the Python wrapper."""
    from gqa_attention_flash_b200 import binding
    Q, K, V, lengths = _inputs(3, 64, 32, 8, 256, 128)
    ref = torch.empty_like(Q)
    out = torch.empty_like(Q)
    binding.attn_decode(ref, Q, K, V, lengths, 8)
    binding.attn_decode_noalloc(out, Q, K, V, lengths, 8)
    assert binding.last_device_status() == 0
    assert float((out.float() - ref.float()).abs().max()) <= O_TOL


def test_noalloc_refuses_workspace_above_limit():
    from gqa_attention_flash_b200 import binding
    lib = binding.lib
    # 64 * 32 * 64 splits * (128 + 4) * 4 bytes = 69 MB > 16 MiB: refused on the host.
    Q, K, V, lengths = _inputs(4, 64, 32, 8, 64, 128)
    out = torch.zeros_like(Q)
    rc = _call(lib.attn_decode_noalloc, out, Q, K, V, lengths, 64)
    assert rc == 7, binding.status_string(rc)
    assert "16 MiB" in binding.status_string(rc)
    assert torch.all(out == 0)
