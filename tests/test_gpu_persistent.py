"""The persistent forward kernel in the settings a serving stack puts it in.

attn_fwd launches one CTA per work item, but a running CTA takes over the items
of CTAs of the same grid that have not started (cluster launch control).  These
tests check that this stays invisible to callers: two launches in flight at
the same time on different streams give bitwise the same outputs as the same
launches run one after the other, and a forward captured into a CUDA graph and
replayed gives bitwise the same outputs as a direct launch."""
import math

import pytest
import torch

from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _problem(seed, B, Hq, Hkv, S, D, ragged):
    dev = torch.device("cuda")
    Q, K, V = W.random_prefill(seed, B, Hq, Hkv, S, S, D)
    kl = ql = None
    if ragged:
        g = torch.Generator().manual_seed(seed)
        kl = torch.randint(S // 2, S + 1, (B,), generator=g).to(torch.int32).to(dev)
        ql = kl.clone()
    O = torch.empty(Q.shape, dtype=torch.bfloat16, device=dev)
    L = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    return dict(Q=Q.to(dev), K=K.to(dev), V=V.to(dev), kl=kl, ql=ql, O=O, L=L,
                scale=1.0 / math.sqrt(D))


def _run(binding, x, causal, window, stream=None):
    binding.attn_fwd(x["O"], x["Q"], x["K"], x["V"], x["L"], x["scale"], causal, window, 0,
                     x["kl"], x["ql"], stream=stream)


def _bits(x):
    return x["O"].view(torch.int16).clone(), x["L"].view(torch.int32).clone()


def test_concurrent_launches_on_two_streams():
    from gqa_attention_flash_b200 import binding
    a = _problem(1, 4, 16, 4, 2048, 128, False)
    b = _problem(2, 2, 8, 8, 3000, 64, True)
    _run(binding, a, True, 0)
    _run(binding, b, True, 700)
    torch.cuda.synchronize()
    ref_a, ref_b = _bits(a), _bits(b)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for _ in range(3):
        a["O"].zero_(), b["O"].zero_()
        torch.cuda.synchronize()
        _run(binding, a, True, 0, stream=s1)
        _run(binding, b, True, 700, stream=s2)
        torch.cuda.synchronize()
        assert binding.last_device_status() == 0
        got_a, got_b = _bits(a), _bits(b)
        assert torch.equal(got_a[0], ref_a[0]) and torch.equal(got_a[1], ref_a[1])
        assert torch.equal(got_b[0], ref_b[0]) and torch.equal(got_b[1], ref_b[1])


def test_forward_in_a_cuda_graph():
    from gqa_attention_flash_b200 import binding
    x = _problem(3, 2, 32, 8, 4096, 128, True)
    _run(binding, x, True, 1024)
    torch.cuda.synchronize()
    ref = _bits(x)
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        _run(binding, x, True, 1024, stream=s)  # first call outside capture (kernel set-up)
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            _run(binding, x, True, 1024, stream=s)
    for _ in range(3):
        x["O"].fill_(float("nan"))
        x["L"].fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert binding.last_device_status() == 0
        got = _bits(x)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
