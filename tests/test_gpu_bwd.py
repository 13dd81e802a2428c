"""Attention backward on the GPU (attn_bwd through the C ABI, after attn_fwd_varlen
on the GPU saved O and LSE) against the fp64 oracle's gradients from the
definition, on the same seeded bf16 Q, K, V, dO.

Tolerance (derived, the pages give none): the GPU rounds P and dS to bf16 before
their second products and reads the bf16 output O for rowsum(dO O); each rounding
is a relative 2^-9 on terms that add with mixed signs, so per tensor
max |g_gpu - g_ref| <= 1e-2 * max |g_ref| + 1e-3."""
import math

import numpy as np
import pytest
import torch

from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_fwd_bwd(Q, K, V, dO, scale, causal=False, window=0, input_pos=0, kl=None, ql=None):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    Qd, Kd, Vd, dOd = Q.to(dev), K.to(dev), V.to(dev), dO.to(dev)
    O = torch.empty_like(Qd)
    L = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    kld = kl.to(dev) if kl is not None else None
    qld = ql.to(dev) if ql is not None else None
    binding.attn_fwd(O, Qd, Kd, Vd, L, scale, causal, window, input_pos, kld, qld)
    dQ = torch.full_like(Qd, float("nan"))
    dK = torch.full_like(Kd, float("nan"))
    dV = torch.full_like(Vd, float("nan"))
    binding.attn_bwd(dQ, dK, dV, dOd, Qd, Kd, Vd, O, L, scale, causal, window, input_pos, kld, qld)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return dQ.cpu(), dK.cpu(), dV.cpu()


def check(gpu, ref, what):
    g = gpu.double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite"
    tol = 1e-2 * float(np.abs(ref).max()) + 1e-3
    err = float(np.abs(g - ref).max())
    assert err <= tol, f"{what}: max err {err} > {tol}"
    return err


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, ragged
    (1, 2, 2, 128, 128, 64, True, 0, 0, False),
    (1, 4, 1, 200, 200, 128, True, 0, 0, False),
    (2, 4, 2, 150, 333, 128, False, 0, 0, False),
    (2, 2, 1, 100, 300, 64, True, 0, 200, False),
    (1, 8, 2, 260, 260, 128, True, 70, 0, False),
    (3, 4, 2, 190, 190, 128, True, 0, 0, True),
    # long enough that the dQ kernel's 3-slot K ring and 2-slot V ring and the dK/dV
    # kernel's 2-slot Q/dO ring wrap several times
    (1, 4, 2, 640, 640, 64, True, 0, 0, False),
    (1, 2, 1, 300, 777, 128, False, 0, 0, False),
    (2, 4, 1, 520, 520, 128, True, 200, 0, True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_backward_matches_oracle(orc, case):
    B, Hq, Hkv, Sq, Sk, D, causal, window, ip, ragged = case
    Q, K, V = W.random_prefill(70 + CASES.index(case), B, Hq, Hkv, Sq, Sk, D)
    dO = torch.randn(B, Hq, Sq, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    kl = ql = None
    if ragged:
        g = torch.Generator().manual_seed(8)
        kl = torch.randint(0, Sk + 1, (B,), generator=g).to(torch.int32)
        ql = torch.randint(1, Sq + 1, (B,), generator=g).to(torch.int32)
    scale = 1.0 / math.sqrt(D)
    dQ, dK, dV = gpu_fwd_bwd(Q, K, V, dO, scale, causal, window, ip, kl, ql)
    rQ, rK, rV = orc.attn_bwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                              dO.double().numpy(), scale, causal=causal, window=window,
                              input_pos=ip, k_lengths=None if kl is None else kl.numpy(),
                              q_lengths=None if ql is None else ql.numpy())
    check(dQ, rQ, f"dQ {case}")
    check(dK, rK, f"dK {case}")
    check(dV, rV, f"dV {case}")


def test_backward_masked_rows_and_keys_are_zero():
    """Keys past k_len and rows past q_len get exactly zero gradients."""
    B, Hq, Hkv, S, D = 2, 2, 1, 200, 128
    Q, K, V = W.random_prefill(3, B, Hq, Hkv, S, S, D)
    dO = torch.randn(B, Hq, S, D, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    kl = torch.tensor([150, 0], dtype=torch.int32)
    ql = torch.tensor([90, 200], dtype=torch.int32)
    dQ, dK, dV = gpu_fwd_bwd(Q, K, V, dO, 0.1, True, 0, 0, kl, ql)
    assert torch.all(dK[0, :, 150:] == 0) and torch.all(dV[0, :, 150:] == 0)
    assert torch.all(dK[1] == 0) and torch.all(dV[1] == 0) and torch.all(dQ[1] == 0)
    assert torch.all(dQ[0, :, 90:] == 0)


def test_backward_finite_padding(orc):
    """Padding rows may hold any finite value (the documented limit: they enter the
    tensor-core products with weight zero, so they must not be NaN or Inf): Q and
    dO rows past q_lengths and K, V rows past k_lengths hold +-3e4, and the
    gradients still match the oracle's (computed from the clean tensors) with the
    padded rows of dQ, dK, dV exactly +0.0."""
    B, Hq, Hkv, S, D = 2, 4, 2, 333, 128
    Q, K, V = W.random_prefill(91, B, Hq, Hkv, S, S, D)
    dO = torch.randn(B, Hq, S, D, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    kl = torch.tensor([333, 190], dtype=torch.int32)
    ql = torch.tensor([250, 333], dtype=torch.int32)
    Qp, Kp, Vp, dOp = Q.clone(), K.clone(), V.clone(), dO.clone()
    Qp[0, :, 250:] = 3e4
    dOp[0, :, 250:] = -3e4
    Kp[1, :, 190:] = -3e4
    Vp[1, :, 190:] = 3e4
    scale = 1.0 / math.sqrt(D)
    dQ, dK, dV = gpu_fwd_bwd(Qp, Kp, Vp, dOp, scale, True, 0, 0, kl, ql)
    rQ, rK, rV = orc.attn_bwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                              dO.double().numpy(), scale, causal=True, k_lengths=kl.numpy(),
                              q_lengths=ql.numpy())
    check(dQ, rQ, "dQ finite padding")
    check(dK, rK, "dK finite padding")
    check(dV, rV, "dV finite padding")
    assert torch.all(dQ[0, :, 250:].view(torch.int16) == 0)
    assert torch.all(dK[1, :, 190:].view(torch.int16) == 0)
    assert torch.all(dV[1, :, 190:].view(torch.int16) == 0)


def test_backward_full_size_llm(orc):
    """The LLM causal shape (B4 Hq32 Hkv8 S4096 D128) as the benchmark runs it:
    dQ on sampled rows and dK / dV on sampled keys of one batch entry, against the
    oracle on a reduced problem that has exactly the same gradients there (the
    first 512 queries of batch 0 see only keys < 512 under the causal mask)."""
    w = W.LLM
    x = W.make_prefill(w)
    dO = torch.randn(x.Q.shape, generator=torch.Generator().manual_seed(11)).to(torch.bfloat16)
    dQ, dK, dV = gpu_fwd_bwd(x.Q, x.K, x.V, dO, w.scale, True, 0, 0, x.k_lengths, None)
    # rows < 512 of batch 0 depend only on keys < 512; keys < 512 collect gradients from every
    # row, so compare dQ rows < 512 and dK / dV only through the reduced problem's dQ
    n = 512
    Qs, Ks, Vs, dOs = (t[:1, :, :n] for t in (x.Q, x.K, x.V, dO))
    rQ, _, _ = orc.attn_bwd(Qs.double().numpy(), Ks.double().numpy(), Vs.double().numpy(),
                            dOs.double().numpy(), w.scale, causal=True)
    check(dQ[:1, :, :n], rQ, "full-size dQ rows < 512")
    # the last key tile of batch 3 is seen only by the last rows: a reduced problem of rows
    # [S - 128, S) against all keys gives the exact dK / dV of keys >= S - 128
    m = 128
    Qt, dOt = x.Q[3:4, :, -m:], dO[3:4, :, -m:]
    _, rK, rV = orc.attn_bwd(Qt.double().numpy(), x.K[3:4].double().numpy(),
                             x.V[3:4].double().numpy(), dOt.double().numpy(), w.scale,
                             causal=True, input_pos=w.Sq - m)
    check(dK[3:4, :, -m:], rK[:, :, -m:], "full-size dK keys >= S-128")
    check(dV[3:4, :, -m:], rV[:, :, -m:], "full-size dV keys >= S-128")


def test_backward_stream_order_graph_and_two_streams():
    """attn_bwd runs its dQ kernel on a library-owned stream joined back to the
    caller's stream: the gradients are bitwise the same when the call is replayed
    from a CUDA graph and when two calls are in flight on different streams."""
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")

    def problem(seed, B, Hq, Hkv, S, D):
        Q, K, V = W.random_prefill(seed, B, Hq, Hkv, S, S, D)
        Q, K, V = Q.to(dev), K.to(dev), V.to(dev)
        O = torch.empty_like(Q)
        L = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(D)
        binding.attn_fwd(O, Q, K, V, L, scale, True)
        dO = torch.randn(Q.shape, generator=torch.Generator().manual_seed(seed)).to(
            torch.bfloat16).to(dev)
        g = (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V))
        return dict(Q=Q, K=K, V=V, O=O, L=L, dO=dO, g=g, scale=scale)

    def run(x, stream=None):
        binding.attn_bwd(*x["g"], x["dO"], x["Q"], x["K"], x["V"], x["O"], x["L"], x["scale"],
                         True, stream=stream)

    def bits(x):
        return [t.view(torch.int16).clone() for t in x["g"]]

    a = problem(5, 2, 8, 2, 1000, 128)
    b = problem(6, 1, 4, 4, 700, 64)
    run(a)
    run(b)
    torch.cuda.synchronize()
    ref_a, ref_b = bits(a), bits(b)
    # two calls in flight on different streams
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for t in a["g"] + b["g"]:
        t.fill_(float("nan"))
    torch.cuda.synchronize()
    run(a, stream=s1)
    run(b, stream=s2)
    torch.cuda.synchronize()
    assert binding.last_device_status() == 0
    assert all(torch.equal(x, y) for x, y in zip(bits(a), ref_a))
    assert all(torch.equal(x, y) for x, y in zip(bits(b), ref_b))
    # captured in a CUDA graph and replayed
    s = torch.cuda.Stream()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        run(a, stream=s)  # first call outside capture (kernel and stream set-up)
        s.synchronize()
        with torch.cuda.graph(gr, stream=s):
            run(a, stream=s)
    for _ in range(2):
        for t in a["g"]:
            t.fill_(float("nan"))
        gr.replay()
        torch.cuda.synchronize()
        assert binding.last_device_status() == 0
        assert all(torch.equal(x, y) for x, y in zip(bits(a), ref_a))
