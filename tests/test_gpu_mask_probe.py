"""Which keys each query row attends to, checked bit-exactly on the hot-path
kernels: attn_fwd / attn_fwd_varlen (the plain prefill kernel) and the split-KV
decode, at the full workload sizes and on edge shapes.

The probe: K = 0 makes every visible score equal, so each visible key gets the
weight exactly 1 (exp2(0)) and the row sum is the number n of visible keys.
V is one-hot in key index over one D-wide chunk of keys: key j of chunk c
carries the unit vector e_(j - cD), every other key carries 0.  Then
O[i, j - cD] = 1/n != 0 exactly when key j is visible from row i, and 0 when it
is masked (a masked key has weight exactly 0; 1/n is a normal bf16 number for
n <= 2^20).  Each KV head carries a different chunk, so one launch checks
Hkv chunks; ceil(Sk / (D Hkv)) launches cover every key.  The expected key
sets come from the oracle (``attn_visible``, the same mask rows its scores
get), and LSE = ln n is checked against the oracle's counts.

Masks (mlx-arsenal "Attention" page: causal_mask, sliding_window_mask; Tylo.jl
"Primitives" page: CausalMask, attention! with input_pos, k_lengths,
q_lengths; decode_attention! with lengths).
"""
import math

import numpy as np
import pytest
import torch

from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-3


def _one_hot_v(V, run, D, Sk):
    """V (B, Hkv, Sk, D) on the device: KV head hk carries chunk run * Hkv + hk."""
    V.zero_()
    Hkv = V.shape[1]
    eye = torch.eye(D, dtype=V.dtype, device=V.device)
    for hk in range(Hkv):
        c = run * Hkv + hk
        j0 = c * D
        if j0 >= Sk:
            continue
        n = min(D, Sk - j0)
        V[:, hk, j0:j0 + n, :] = eye[:n]


def _expected_chunk(vis, c, D, Sk):
    """(B, Sq, D) bool: visibility of the keys of chunk c (False past Sk)."""
    B, Sq, _ = vis.shape
    out = torch.zeros(B, Sq, D, dtype=torch.bool, device=vis.device)
    j0 = c * D
    if j0 < Sk:
        n = min(D, Sk - j0)
        out[:, :, :n] = vis[:, :, j0:j0 + n]
    return out


def _first_mismatch(got, want):
    idx = torch.nonzero(got != want)
    return idx[0].tolist() if idx.numel() else None


def prefill_probe(orc, B, Hq, Hkv, Sq, Sk, D, causal, window=0, input_pos=0, k_lengths=None,
                  q_lengths=None, what=""):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    kl = None if k_lengths is None else torch.as_tensor(k_lengths, dtype=torch.int32)
    ql = None if q_lengths is None else torch.as_tensor(q_lengths, dtype=torch.int32)
    vis_np = orc.attn_visible(B, Sq, Sk, causal=causal, window=window, input_pos=input_pos,
                              k_lengths=None if kl is None else kl.numpy(),
                              q_lengths=None if ql is None else ql.numpy())
    vis = torch.from_numpy(vis_np).to(dev).bool()
    count = vis.sum(-1, dtype=torch.int64)                     # (B, Sq)
    del vis_np
    Q = torch.randn(B, Hq, Sq, D, generator=torch.Generator().manual_seed(Sq + Sk)).to(
        torch.bfloat16).to(dev)
    K = torch.zeros(B, Hkv, Sk, D, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    O = torch.empty_like(Q)
    LSE = torch.empty(B, Hq, Sq, dtype=torch.float32, device=dev)
    kld = None if kl is None else kl.to(dev)
    qld = None if ql is None else ql.to(dev)
    G = Hq // Hkv
    n_chunks = (Sk + D - 1) // D
    n_runs = max(1, (n_chunks + Hkv - 1) // Hkv)
    inv_n = torch.where(count > 0, 1.0 / count.clamp(min=1).double(), 0.0)  # (B, Sq)
    for run in range(n_runs):
        _one_hot_v(V, run, D, Sk)
        O.fill_(float("nan"))
        LSE.fill_(float("nan"))
        binding.attn_fwd(O, Q, K, V, LSE, 1.0 / math.sqrt(D), causal, window, input_pos, kld, qld)
        st = binding.last_device_status()
        assert st == 0, binding.status_string(st)
        for h in range(Hq):
            c = run * Hkv + h // G
            want = _expected_chunk(vis, c, D, Sk)
            got = O[:, h] != 0
            assert torch.equal(got, want), \
                f"{what}: head {h} chunk {c}: first mismatch (b, i, d) {_first_mismatch(got, want)}"
            # the visible entries hold 1/n to bf16 rounding
            vals = O[:, h].double()
            err = (vals - inv_n[:, :, None]).abs() * want
            assert float(err.max()) <= float((inv_n * 2.0 ** -8).max()) + 1e-12, what
        if run == 0:
            lse = LSE.double()
            empty = (count == 0)[:, None, :].expand_as(lse)
            assert torch.equal(torch.isneginf(lse), empty), f"{what}: -inf rows differ"
            ref = torch.log(count.clamp(min=1).double())[:, None, :].expand_as(lse)
            d = float(((lse - ref).abs() * (~empty)).nan_to_num(0.0).max())
            assert d <= LSE_TOL, f"{what}: max |LSE - ln n| = {d}"
            # rows past q_lengths / rows with no key: every bit of O is zero
            assert torch.all(O.view(torch.int16)[empty] == 0), f"{what}: empty rows not +0.0"
    return n_runs


@pytest.mark.parametrize("name", ["tiny", "llm", "window", "image"])
def test_workload_masks_bit_exact(orc, name):
    """Every query row, head and key of the four prefill workloads at full size,
    in the launch configuration the benchmark uses."""
    w = W.PREFILL_WORKLOADS[name]
    x = W.make_prefill(w)
    kl = None if x.k_lengths is None else x.k_lengths.numpy()
    ql = None if x.q_lengths is None else x.q_lengths.numpy()
    del x
    prefill_probe(orc, w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.D, w.causal, w.window, w.input_pos,
                  kl, ql, what=name)


EDGE = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, k_lengths, q_lengths
    (2, 4, 2, 700, 1100, 64, True, 0, 400, [1100, 517], [700, 333]),
    (1, 2, 1, 1000, 1000, 128, True, 1, 0, None, None),
    (1, 2, 1, 1000, 1000, 128, True, 100, 0, None, None),
    (1, 2, 1, 1000, 1000, 64, True, 128, 0, None, None),
    (1, 2, 1, 1000, 1000, 128, True, 129, 0, None, None),
    (2, 8, 2, 5000, 5000, 128, True, 4096, 0, [5000, 4321], [5000, 4321]),
    (2, 4, 1, 640, 2000, 128, True, 300, 1360, [2000, 1500], [640, 77]),
    (3, 2, 2, 300, 900, 64, False, 0, 0, [900, 0, 129], [300, 300, 1]),
    (1, 4, 1, 1, 1000, 128, True, 0, 999, None, None),
    (2, 4, 4, 257, 385, 128, False, 0, 0, [385, 127], [129, 257]),
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c[:9]) for c in EDGE])
def test_edge_masks_bit_exact(orc, case):
    """Windows of 1, 100, 128, 129 and 4096 keys, input_pos > 0 with Sq != Sk,
    lengths that cut tiles in the middle, empty sequences, one-row queries."""
    B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, kl, ql = case
    prefill_probe(orc, B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos,
                  None if kl is None else np.array(kl, dtype=np.int32),
                  None if ql is None else np.array(ql, dtype=np.int32), what=str(case))


def decode_probe(orc, B, Hq, Hkv, S_cap, D, lengths, n_splits, what=""):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    lengths = np.asarray(lengths, dtype=np.int32)
    vis = torch.from_numpy(orc.attn_visible(B, 1, S_cap, k_lengths=lengths)[:, 0]).to(dev).bool()
    count = vis.sum(-1, dtype=torch.int64)
    inv_n = torch.where(count > 0, 1.0 / count.clamp(min=1).double(), 0.0)
    Q = torch.randn(B, Hq, D, generator=torch.Generator().manual_seed(S_cap)).to(
        torch.bfloat16).to(dev)
    K = torch.zeros(B, Hkv, S_cap, D, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    O = torch.empty_like(Q)
    ld = torch.from_numpy(lengths).to(dev)
    G = Hq // Hkv
    n_chunks = (S_cap + D - 1) // D
    for run in range(max(1, (n_chunks + Hkv - 1) // Hkv)):
        _one_hot_v(V, run, D, S_cap)
        O.fill_(float("nan"))
        binding.attn_decode(O, Q, K, V, ld, n_splits)
        st = binding.last_device_status()
        assert st == 0, binding.status_string(st)
        for h in range(Hq):
            c = run * Hkv + h // G
            want = _expected_chunk(vis[:, None, :], c, D, S_cap)[:, 0]
            got = O[:, h] != 0
            assert torch.equal(got, want), \
                f"{what}: head {h} chunk {c}: first mismatch (b, d) {_first_mismatch(got, want)}"
            err = (O[:, h].double() - inv_n[:, None]).abs() * want
            assert float(err.max()) <= float((inv_n * 2.0 ** -8).max()) + 1e-12, what
    del K, V
    torch.cuda.empty_cache()


def test_decode_workload_keys_bit_exact(orc):
    """The B64 / 32K-cache decode workload: every sequence, head and cached key."""
    w = W.DECODE
    _, lengths = W.decode_query_and_lengths(w)
    decode_probe(orc, w.B, w.Hq, w.Hkv, w.S_cap, w.D, lengths.numpy(), w.n_splits, "decode")


@pytest.mark.parametrize("D,n_splits", [(128, 8), (64, 3), (128, 1), (128, 64)])
def test_decode_edge_lengths_bit_exact(orc, D, n_splits):
    """Lengths 0, 1, tile edges (63, 64, 65), split edges and the full capacity."""
    S_cap = 1300
    lengths = [0, 1, 63, 64, 65, 127, 128, 129, 640, 641, 1299, 1300]
    decode_probe(orc, len(lengths), 8, 2, S_cap, D, lengths, n_splits, f"D{D} splits{n_splits}")
