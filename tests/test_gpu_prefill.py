"""CUDA prefill path (attn_fwd / attn_fwd_varlen through the C ABI) against the
fp64 oracle, element by element on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

from gpu_common import compare, gpu_prefill, oracle_prefill, sample_rows
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_tiny_config_full(orc):
    """The tiny causal GQA workload, every output element."""
    w = W.TINY
    x = W.make_prefill(w)
    O, L = gpu_prefill(x.Q, x.K, x.V, w.scale, w.causal)
    Or, Lr = oracle_prefill(orc, x.Q, x.K, x.V, w.scale, w.causal)
    compare(O, L, Or, Lr, what="tiny")


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, ragged
    (1, 2, 1, 300, 300, 64, True, 0, 0, False),
    (2, 4, 2, 300, 333, 128, False, 0, 0, False),
    (2, 4, 2, 257, 700, 128, True, 0, 443, False),
    (1, 4, 1, 520, 520, 128, True, 100, 0, False),
    (2, 8, 2, 390, 390, 64, True, 130, 0, True),
    (2, 3, 3, 129, 600, 128, False, 0, 0, True),
    (1, 2, 2, 1, 257, 128, True, 0, 256, False),
    (3, 2, 1, 200, 200, 128, True, 1, 0, False),
    (1, 4, 4, 384, 384, 128, True, 0, 0, False),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_ragged_tiles(orc, case):
    B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, ragged = case
    Q, K, V = W.random_prefill(hash(case) % 1000, B, Hq, Hkv, Sq, Sk, D)
    kl = ql = None
    if ragged:
        g = torch.Generator().manual_seed(7)
        kl = torch.randint(1, Sk + 1, (B,), generator=g).to(torch.int32)
        ql = torch.randint(1, Sq + 1, (B,), generator=g).to(torch.int32)
    scale = 1.0 / np.sqrt(D)
    O, L = gpu_prefill(Q, K, V, scale, causal, window, input_pos, kl, ql)
    Or, Lr = oracle_prefill(orc, Q, K, V, scale, causal, window, input_pos, kl, ql)
    compare(O, L, Or, Lr, what=str(case))


def test_lse_optional(orc):
    Q, K, V = W.random_prefill(3, 1, 2, 1, 200, 200, 128)
    O, _ = gpu_prefill(Q, K, V, 0.1, True, want_lse=False)
    Or, Lr = oracle_prefill(orc, Q, K, V, 0.1, True)
    compare(O, None, Or, Lr, what="no LSE")


def test_edge_cases(orc):
    """Empty lengths, rows past q_len, keys cut entirely, Sk = 0."""
    B, Hq, Hkv, S, D = 4, 2, 1, 200, 128
    Q, K, V = W.random_prefill(11, B, Hq, Hkv, S, S, D)
    kl = torch.tensor([0, 200, 5, 130], dtype=torch.int32)
    ql = torch.tensor([200, 0, 200, 129], dtype=torch.int32)
    for causal, window, input_pos in [(False, 0, 0), (True, 0, 0), (True, 3, 0), (True, 0, 150)]:
        O, L = gpu_prefill(Q, K, V, 0.09, causal, window, input_pos, kl, ql)
        Or, Lr = oracle_prefill(orc, Q, K, V, 0.09, causal, window, input_pos, kl, ql)
        compare(O, L, Or, Lr, what=f"edge {causal} {window} {input_pos}")
    Qe = Q[:, :, :7].contiguous()
    Ke = torch.zeros(B, Hkv, 0, D, dtype=torch.bfloat16)
    O, L = gpu_prefill(Qe, Ke, Ke, 0.1, False)
    assert torch.all(O == 0) and torch.all(torch.isneginf(L))


def test_nan_beyond_k_lengths_ignored(orc):
    """Key/value rows past k_lengths may hold NaN; they must not leak."""
    B, Hq, Hkv, S, D = 2, 2, 1, 300, 128
    Q, K, V = W.random_prefill(12, B, Hq, Hkv, S, S, D)
    kl = torch.tensor([157, 300], dtype=torch.int32)
    Kp, Vp = K.clone(), V.clone()
    Kp[0, :, 157:] = float("nan")
    Vp[0, :, 157:] = float("nan")
    O, L = gpu_prefill(Q, Kp, Vp, 0.09, True, 0, 0, kl)
    Or, Lr = oracle_prefill(orc, Q, K, V, 0.09, True, 0, 0, kl)
    compare(O, L, Or, Lr, what="nan past k_len")


@pytest.mark.parametrize("name", ["llm", "window", "image"])
def test_full_size_sampled(orc, name):
    """Full-size workloads in the benchmark's launch configuration, compared on
    sampled query rows (all batches and heads): 512 random rows plus tile and mask
    edges."""
    w = W.PREFILL_WORKLOADS[name]
    x = W.make_prefill(w)
    O, L = gpu_prefill(x.Q, x.K, x.V, w.scale, w.causal, w.window, w.input_pos, x.k_lengths,
                       x.q_lengths)
    extra = []
    if x.k_lengths is not None:
        for v in x.k_lengths.tolist():
            extra += [v - 1, v, v - w.window, v - w.window + 1]
    rows = sample_rows(w.Sq, 5, n_random=512, extra=extra)
    Or, Lr = oracle_prefill(orc, x.Q, x.K, x.V, w.scale, w.causal, w.window, w.input_pos,
                            x.k_lengths, x.q_lengths, rows=rows)
    compare(O, L, Or, Lr, rows=rows, what=name)


@pytest.mark.parametrize("causal", [False, True])
def test_running_max_jumps(orc, causal):
    """Keys with scores far above the rest appear deep into the rows (different KV
    tiles for different rows), so the running row max jumps by more than 2^8 after
    a row's first tile: this exercises the redo of a tile's exponentials and the
    rescaling of the O accumulator."""
    B, Hq, Hkv, S, D = 1, 4, 2, 1100, 128
    Q, K, V = W.random_prefill(21, B, Hq, Hkv, S, S, D)
    K = K.float()
    for j, f in [(300, 8.0), (700, 14.0), (1030, 20.0)]:
        K[:, :, j] *= f
    K = K.to(torch.bfloat16)
    # such rows return nearly one V row; keep |V| < 2 so that bf16 rounding of O
    # (2^-7 there) stays well inside the tolerance
    V = (V.float() * 0.5).clamp(-1.9, 1.9).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(D)
    O, L = gpu_prefill(Q, K, V, scale, causal)
    Or, Lr = oracle_prefill(orc, Q, K, V, scale, causal)
    compare(O, L, Or, Lr, what=f"max jumps causal={causal}")


@pytest.mark.parametrize("D,poison", [(128, float("nan")), (64, float("inf"))])
def test_non_finite_q_rows_past_q_lengths(orc, D, poison):
    """Query rows past q_lengths may hold anything (uninitialised padding, NaN,
    Inf): their O rows are +0.0 in every bit and their LSE is -inf, and the valid
    rows still match the oracle (which gets the clean Q)."""
    B, Hq, Hkv, S = 3, 4, 2, 300
    Q, K, V = W.random_prefill(13, B, Hq, Hkv, S, S, D)
    ql = torch.tensor([300, 131, 7], dtype=torch.int32)
    kl = torch.tensor([300, 250, 300], dtype=torch.int32)
    Qp = Q.clone()
    for b, n in enumerate(ql.tolist()):
        Qp[b, :, n:] = poison
    for causal, window, input_pos in [(False, 0, 0), (True, 0, 0), (True, 50, 20)]:
        O, L = gpu_prefill(Qp, K, V, 0.09, causal, window, input_pos, kl, ql)
        Or, Lr = oracle_prefill(orc, Q, K, V, 0.09, causal, window, input_pos, kl, ql)
        compare(O, L, Or, Lr, what=f"poisoned Q {causal} {window} {input_pos}")
        for b, n in enumerate(ql.tolist()):
            assert torch.all(O[b, :, n:].view(torch.int16) == 0), (b, causal, window)
            assert torch.all(torch.isneginf(L[b, :, n:]))


def test_window_workload_finite_poison(orc):
    """Probe (ii) on the sliding-window workload at full size: every key and value
    row past k_lengths holds the finite value 1e4 and every query row past
    q_lengths holds NaN.  A masked key that leaked into a row would move it by far
    more than the tolerance; the padded rows must be +0.0 / -inf."""
    w = W.WINDOW
    x = W.make_prefill(w)
    Qp, Kp, Vp = x.Q.clone(), x.K.clone(), x.V.clone()
    for b, n in enumerate(x.k_lengths.tolist()):
        Kp[b, :, n:] = 1e4
        Vp[b, :, n:] = 1e4
    for b, n in enumerate(x.q_lengths.tolist()):
        Qp[b, :, n:] = float("nan")
    O, L = gpu_prefill(Qp, Kp, Vp, w.scale, w.causal, w.window, w.input_pos, x.k_lengths,
                       x.q_lengths)
    extra = []
    for v in x.k_lengths.tolist():
        extra += [v - 129, v - 128, v - 2, v - 1, v, v + 1, v - w.window, v - w.window + 1]
    rows = sample_rows(w.Sq, 9, n_random=24, extra=extra)
    Or, Lr = oracle_prefill(orc, x.Q, x.K, x.V, w.scale, w.causal, w.window, w.input_pos,
                            x.k_lengths, x.q_lengths, rows=rows)
    compare(O, L, Or, Lr, rows=rows, what="window poison")
    for b, n in enumerate(x.q_lengths.tolist()):
        assert torch.all(O[b, :, n:].view(torch.int16) == 0)
        assert torch.all(torch.isneginf(L[b, :, n:]))
