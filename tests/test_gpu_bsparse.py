"""Block-sparse prefill kernel: attn_fwd_flex with a BlockMask alone (no score mod,
no DocumentMask, not causal, no lengths), which runs 64-key steps over the kept
64x64 blocks, against the fp64 oracle (oracle.flex_fwd with block_keep).

Parity: random block masks at several densities, one per (batch, query head) and
one shared by all heads, with states 1 and 2 both meaning "kept" when no
document ids are given; ragged Sq and Sk; D 64 and 128; GQA; a query block whose
row of the mask is empty next to one that is not; a whole 128-row query tile with
nothing kept; every block kept (dense attention); and tiles with enough kept
blocks to wrap the K / V rings many times.

Mask: the one-hot probe (K = 0 makes every visible score equal; V is one-hot over
a D-wide key chunk per KV head) turns O != 0 into the set of visible keys, which
must equal the oracle's bit for bit, with LSE = ln(number of visible keys)."""
import math

import numpy as np
import pytest
import torch

from gpu_common import compare
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def random_block_mask(seed, B, Hq, Sq, Sk, density, per_head):
    """uint8 states: 0 (skip) with probability 1 - density, else 1 or 2 (kept)."""
    g = torch.Generator().manual_seed(seed)
    nqb, nkb = (Sq + 63) // 64, (Sk + 63) // 64
    shape = (B, Hq, nqb, nkb) if per_head else (nqb, nkb)
    kept = torch.rand(shape, generator=g) < density
    state = torch.randint(1, 3, shape, generator=g, dtype=torch.uint8)
    m = torch.where(kept, state, torch.zeros_like(state))
    if per_head and nqb >= 2:
        m[0, 0, 1, :] = 0          # query block 1 of tile 0 sees nothing, block 0 may
        if Hq > 1:
            m[0, 1, 0:2, :] = 0    # the whole first query tile of head 1 sees nothing
    return m.contiguous()


def keep_flags(mask, B, Hq):
    k = (mask.numpy() != 0).astype(np.uint8)
    if k.ndim == 2:
        k = np.broadcast_to(k, (B, Hq) + k.shape)
    return np.ascontiguousarray(k)


def gpu_block_sparse(Q, K, V, scale, mask):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    L = torch.full(Q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
    binding.attn_fwd_flex(O, Q.to(dev), K.to(dev), V.to(dev), L, scale, False,
                          block_mask=mask.to(dev))
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu(), L.cpu()


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, density, per_head
    (1, 4, 2, 300, 300, 128, 0.2, True),
    (2, 2, 1, 257, 700, 64, 0.3, True),
    (1, 4, 4, 640, 640, 128, 0.1, False),
    (1, 2, 2, 200, 1000, 128, 1.0, True),
    (1, 2, 1, 64, 129, 128, 0.5, True),
    (1, 2, 2, 384, 2048, 128, 0.6, True),
    (1, 2, 1, 1, 65, 64, 0.5, True),
    (2, 8, 2, 1000, 3000, 64, 0.15, True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_block_sparse_matches_oracle(orc, case):
    B, Hq, Hkv, Sq, Sk, D, density, per_head = case
    Q, K, V = W.random_prefill(70 + CASES.index(case), B, Hq, Hkv, Sq, Sk, D)
    mask = random_block_mask(80 + CASES.index(case), B, Hq, Sq, Sk, density, per_head)
    scale = 1.0 / math.sqrt(D)
    O, L = gpu_block_sparse(Q, K, V, scale, mask)
    Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                          block_keep=keep_flags(mask, B, Hq))
    compare(O, L, Or, Lr, what=str(case))
    # rows that see no key: every bit of O is +0.0
    empty = torch.from_numpy(np.isneginf(Lr))
    assert torch.all(O.view(torch.int16)[empty] == 0)


def test_all_kept_equals_dense(orc):
    """Every block kept: the same function as attn_fwd without a mask."""
    from gpu_common import gpu_prefill
    B, Hq, Hkv, S, D = 1, 4, 1, 1000, 128
    Q, K, V = W.random_prefill(91, B, Hq, Hkv, S, S, D)
    mask = torch.full(((S + 63) // 64, (S + 63) // 64), 2, dtype=torch.uint8)
    O, L = gpu_block_sparse(Q, K, V, 0.1, mask)
    Od, Ld = gpu_prefill(Q, K, V, 0.1)
    assert float((O.float() - Od.float()).abs().max()) <= 1.6e-2
    assert float((L - Ld).abs().max()) <= 1e-3


PROBES = [
    # B, Hq, Hkv, Sq, Sk, D, density
    (2, 4, 2, 300, 700, 64, 0.3),
    (1, 2, 1, 513, 1100, 128, 0.2),
]


@pytest.mark.parametrize("case", PROBES, ids=[str(c) for c in PROBES])
def test_one_hot_probe_bit_exact(orc, case):
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, Sq, Sk, D, density = case
    dev = torch.device("cuda")
    mask = random_block_mask(95 + PROBES.index(case), B, Hq, Sq, Sk, density, True)
    keep = keep_flags(mask, B, Hq)
    Q = torch.randn(B, Hq, Sq, D, generator=torch.Generator().manual_seed(Sq)).to(torch.bfloat16)
    K = torch.zeros(B, Hkv, Sk, D, dtype=torch.bfloat16)
    G = Hq // Hkv
    n_runs = max(1, ((Sk + D - 1) // D + Hkv - 1) // Hkv)
    O = torch.empty(Q.shape, dtype=torch.bfloat16, device=dev)
    L = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    Qd, Kd, md = Q.to(dev), K.to(dev), mask.to(dev)
    eye = torch.eye(D, dtype=torch.bfloat16)
    for run in range(n_runs):
        V = torch.zeros(B, Hkv, Sk, D, dtype=torch.bfloat16)
        for hk in range(Hkv):
            j0 = (run * Hkv + hk) * D
            if j0 < Sk:
                V[:, hk, j0:j0 + min(D, Sk - j0)] = eye[:min(D, Sk - j0)]
        O.fill_(float("nan"))
        L.fill_(float("nan"))
        binding.attn_fwd_flex(O, Qd, Kd, V.to(dev), L, 1.0 / math.sqrt(D), False, block_mask=md)
        st = binding.last_device_status()
        assert st == 0, binding.status_string(st)
        Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                              1.0 / math.sqrt(D), block_keep=keep)
        got = O.cpu().double().numpy() != 0.0
        want = Or != 0.0
        for h in range(Hq):
            assert np.array_equal(got[:, h], want[:, h]), \
                f"{case} run {run} head {h} (chunk {run * Hkv + h // G})"
        compare(O.cpu(), L.cpu(), Or, Lr, what=f"{case} run {run}")


@pytest.mark.parametrize("Sk", [65499, 65617])
def test_longest_key_sequences(orc, Sk):
    """1024 key blocks (the last one ragged), the most the block-sparse kernel's per-CTA
    list holds, and two blocks more (the call then runs on the flex kernel's list
    path): the same function."""
    B, Hq, Hkv, Sq, D = 1, 2, 1, 200, 128
    Q, K, V = W.random_prefill(99, B, Hq, Hkv, Sq, Sk, D)
    mask = random_block_mask(98, B, Hq, Sq, Sk, 0.05, True)
    # the last key block is kept by one query block, so the ragged end of the keys is visited
    mask[0, 0, 0, -1] = 2
    scale = 1.0 / math.sqrt(D)
    O, L = gpu_block_sparse(Q, K, V, scale, mask)
    Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                          block_keep=keep_flags(mask, B, Hq))
    compare(O, L, Or, Lr, what=f"Sk {Sk}")
