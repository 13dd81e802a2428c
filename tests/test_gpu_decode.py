"""CUDA split-KV decode (attn_decode through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gpu_common import O_TOL, gpu_decode
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _oracle(orc, Q, K, V, lengths):
    O, _ = orc.decode(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                      lengths.numpy())
    return O


def _check(O_gpu, O_ref, what):
    Og = O_gpu.double().numpy()
    assert np.all(np.isfinite(Og)), what
    d = float(np.abs(Og - O_ref).max())
    assert d <= O_TOL, f"{what}: max |dO| = {d}"
    return d


@pytest.mark.parametrize("B,Hq,Hkv,S_cap,D,n_splits", [
    (3, 8, 2, 1000, 128, 8),
    (4, 4, 1, 513, 64, 3),
    (2, 16, 1, 300, 128, 1),
    (2, 32, 2, 700, 128, 64),
    (5, 2, 2, 130, 128, 8),
])
def test_small(orc, B, Hq, Hkv, S_cap, D, n_splits):
    g = torch.Generator().manual_seed(B * 1000 + S_cap)
    Q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    lengths = torch.randint(1, S_cap + 1, (B,), generator=g).to(torch.int32)
    lengths[0] = S_cap
    O = gpu_decode(Q, K, V, lengths, n_splits)
    _check(O, _oracle(orc, Q, K, V, lengths), "small")


def test_empty_and_poison(orc):
    """lengths = 0 gives O = 0; NaN / large values past the length never leak."""
    B, Hq, Hkv, S_cap, D = 4, 8, 2, 600, 128
    g = torch.Generator().manual_seed(5)
    Q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    lengths = torch.tensor([0, 1, 333, 600], dtype=torch.int32)
    ref = _oracle(orc, Q, K, V, lengths)
    Kp, Vp = K.clone(), V.clone()
    for b, n in enumerate(lengths.tolist()):
        Kp[b, :, n:] = float("nan")
        Vp[b, :, n:] = float("nan")
    O = gpu_decode(Q, Kp, Vp, lengths, 8)
    _check(O, ref, "poison")
    assert torch.all(O[0] == 0)


def test_full_size_sampled(orc):
    """The B64 / 32K-cache workload in the benchmark's launch configuration;
    all outputs are checked for finiteness and 8 sequences against the oracle."""
    w = W.DECODE
    Q, lengths = W.decode_query_and_lengths(w)
    dev = torch.device("cuda")
    K = torch.empty(w.B, w.Hkv, w.S_cap, w.D, dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    W.fill_decode_cache(w, lengths, K, V)
    from gqa_attention_flash_b200 import binding
    O = torch.empty(w.B, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
    binding.attn_decode(O, Q.to(dev), K, V, lengths.to(dev), w.n_splits)
    assert binding.last_device_status() == 0
    O = O.cpu()
    assert torch.all(torch.isfinite(O))
    del K, V
    torch.cuda.empty_cache()
    order = torch.argsort(lengths)
    picks = sorted({int(order[0]), int(order[-1]), int(order[w.B // 2]), 0, 1, 17, 40, 63})
    for b in picks:
        n = int(lengths[b])
        Kb, Vb = W.decode_sequence_kv(w, b, n)
        ref = _oracle(orc, Q[b:b + 1], Kb[None], Vb[None], lengths[b:b + 1].clone().fill_(n))
        _check(O[b:b + 1], ref, f"sequence {b} (len {n})")
