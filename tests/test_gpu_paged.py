"""Paged-KV split decode on the GPU (attn_decode_paged through the C ABI) against
the fp64 oracle (oracle.decode_paged): block sizes 8..128, GQA groups, lengths
0, 1, block and tile edges and full capacity, shuffled block pools, poisoned
unused blocks, and the measured workload at full size on sampled sequences."""
import math

import numpy as np
import pytest
import torch

from gpu_common import O_TOL
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_paged(Q, Kp, Vp, tables, lens, n_splits):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    binding.attn_decode_paged(O, Q.to(dev), Kp.to(dev), Vp.to(dev), tables.to(dev),
                              lens.to(dev), n_splits)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu()


def random_paged(seed, B, Hq, Hkv, D, block_size, lengths, spare=5, poison=None):
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    tables, nblk = W.paged_layout(lengths, block_size, spare, seed)
    shape = (nblk, block_size, Hkv, D)
    fillv = float("nan") if poison == "nan" else 0.0
    Kp = torch.full(shape, fillv, dtype=torch.bfloat16)
    Vp = torch.full(shape, fillv, dtype=torch.bfloat16)
    kv = {b: (torch.randn(Hkv, n, D, generator=g).to(torch.bfloat16),
              torch.randn(Hkv, n, D, generator=g).to(torch.bfloat16))
          for b, n in enumerate(lengths)}
    W.fill_paged_cache(Kp, Vp, tables, lambda b: kv[b])
    if poison == "nan":  # slots past each length inside used blocks too
        for b, n in enumerate(lengths):
            nb = (n + block_size - 1) // block_size
            if nb and n % block_size:
                Kp[tables[b, nb - 1], n % block_size:] = float("nan")
                Vp[tables[b, nb - 1], n % block_size:] = float("nan")
    return Q, Kp, Vp, tables, torch.tensor(lengths, dtype=torch.int32)


CASES = [
    # B, Hq, Hkv, D, block_size, lengths, n_splits
    (4, 8, 2, 128, 16, [1, 15, 16, 17], 4),
    (3, 32, 8, 128, 16, [0, 300, 1025], 8),
    (3, 4, 4, 64, 8, [63, 64, 65], 3),
    (2, 16, 1, 128, 32, [777, 96], 8),
    (3, 8, 8, 64, 64, [64, 640, 1], 5),
    (2, 12, 3, 128, 128, [129, 1000], 2),
    (2, 8, 2, 128, 256, [2048, 257], 8),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_paged_decode(orc, case):
    B, Hq, Hkv, D, bs, lengths, n_splits = case
    Q, Kp, Vp, tables, lens = random_paged(hash(str(case)) % 1000, B, Hq, Hkv, D, bs, lengths)
    O = gpu_paged(Q, Kp, Vp, tables, lens, n_splits)
    Or, _ = orc.decode_paged(Q.double().numpy(), Kp.double().numpy(), Vp.double().numpy(),
                             tables.numpy(), lens.numpy())
    d = float(np.abs(O.double().numpy() - Or).max())
    assert d <= O_TOL, (case, d)
    for b, n in enumerate(lengths):
        if n == 0:
            assert torch.all(O[b] == 0)


def test_paged_ignores_poisoned_slots(orc):
    """Unused blocks and slots past each length hold NaN: the output stays exact."""
    lengths = [5, 40, 33, 16]
    Q, Kp, Vp, tables, lens = random_paged(77, 4, 8, 2, 128, 16, lengths, spare=9, poison="nan")
    O = gpu_paged(Q, Kp, Vp, tables, lens, 4)
    assert torch.all(torch.isfinite(O.float()))
    clean = lambda t: torch.nan_to_num(t.double(), nan=0.0).numpy()
    Or, _ = orc.decode_paged(Q.double().numpy(), clean(Kp), clean(Vp), tables.numpy(), lens.numpy())
    assert float(np.abs(O.double().numpy() - Or).max()) <= O_TOL


def test_paged_equals_contiguous_decode():
    """The same sequences in a contiguous cache and in a shuffled paged pool give
    bit-identical outputs (same tile order, same arithmetic)."""
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    lengths = [100, 1, 2048, 513]
    B, Hq, Hkv, D, bs = 4, 16, 4, 128, 16
    Q, Kp, Vp, tables, lens = random_paged(5, B, Hq, Hkv, D, bs, lengths)
    S_cap = max(lengths)
    Kc = torch.zeros(B, Hkv, S_cap, D, dtype=torch.bfloat16)
    Vc = torch.zeros(B, Hkv, S_cap, D, dtype=torch.bfloat16)
    for b, n in enumerate(lengths):
        for j in range(0, n, bs):
            m = min(bs, n - j)
            Kc[b, :, j:j + m] = Kp[tables[b, j // bs], :m].permute(1, 0, 2)
            Vc[b, :, j:j + m] = Vp[tables[b, j // bs], :m].permute(1, 0, 2)
    O1 = gpu_paged(Q, Kp, Vp, tables, lens, 8)
    O2 = torch.empty(Q.shape, dtype=torch.bfloat16, device=dev)
    binding.attn_decode(O2, Q.to(dev), Kc.to(dev), Vc.to(dev), lens.to(dev), 8)
    assert torch.equal(O1, O2.cpu())


def test_paged_full_size_workload(orc):
    """The benchmark's paged workload at full size, in its launch configuration;
    sampled sequences (shortest, longest, random) against the oracle."""
    w = W.PAGED_DECODE
    dev = torch.device("cuda")
    Q, Kp, Vp, tables, lens = W.make_paged_decode(w, dev)
    O = gpu_paged(Q, Kp, Vp, tables, lens, w.base.n_splits)
    pick = sorted({int(torch.argmin(lens)), int(torch.argmax(lens)), 3, 17, 40})
    for b in pick:
        n = int(lens[b])
        nb = (n + w.block_size - 1) // w.block_size
        blocks = tables[b, :nb].to(torch.long)
        Kb = Kp[blocks.to(dev)].cpu()
        Vb = Vp[blocks.to(dev)].cpu()
        local = torch.arange(nb, dtype=torch.int32)[None]
        Or, _ = orc.decode_paged(Q[b:b + 1].double().numpy(), Kb.double().numpy(),
                                 Vb.double().numpy(), local.numpy(), np.array([n], np.int32))
        d = float(np.abs(O[b:b + 1].double().numpy() - Or).max())
        assert d <= O_TOL, (b, n, d)
