"""flex_attention! forward on the GPU (attn_fwd_flex through the C ABI) against the
fp64 oracle (oracle.flex_fwd), element by element on the same seeded bf16 inputs:
SoftCapScore, AliBiScore, DocumentMask with and without a BlockMask, a BlockMask
alone, and the one-hot probe that pins exactly which pairs are masked."""
import math

import numpy as np
import pytest
import torch

from gpu_common import compare
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def gpu_flex(Q, K, V, scale, causal=False, window=0, input_pos=0, k_lengths=None,
             q_lengths=None, softcap=0.0, alibi=None, doc_q=None, doc_kv=None, block_mask=None):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    LSE = torch.full(Q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
    to = lambda t: None if t is None else t.to(dev)
    binding.attn_fwd_flex(O, Q.to(dev), K.to(dev), V.to(dev), LSE, scale, causal, window,
                          input_pos, to(k_lengths), to(q_lengths), softcap, to(alibi),
                          to(doc_q), to(doc_kv), to(block_mask))
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu(), LSE.cpu()


def oracle_flex(orc, Q, K, V, scale, causal=False, window=0, input_pos=0, k_lengths=None,
                q_lengths=None, softcap=0.0, alibi=None, doc_q=None, doc_kv=None):
    npy = lambda t: None if t is None else t.numpy()
    return orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                        causal=causal, window=window, input_pos=input_pos,
                        k_lengths=npy(k_lengths), q_lengths=npy(q_lengths), softcap=softcap,
                        alibi_slopes=None if alibi is None else alibi.double().numpy(),
                        doc_q=npy(doc_q), doc_kv=npy(doc_kv))


SOFTCAP_CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, scale, cap
    (1, 4, 2, 300, 300, 128, True, 0, 0, 0.3, 5.0),
    (2, 2, 1, 257, 390, 64, False, 0, 0, 0.5, 2.0),
    (1, 4, 4, 200, 333, 128, True, 70, 133, 0.25, 30.0),
]


@pytest.mark.parametrize("case", SOFTCAP_CASES, ids=[str(c) for c in SOFTCAP_CASES])
def test_softcap(orc, case):
    B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, scale, cap = case
    Q, K, V = W.random_prefill(11 + hash(case) % 97, B, Hq, Hkv, Sq, Sk, D)
    O, L = gpu_flex(Q, K, V, scale, causal, window, input_pos, softcap=cap)
    Or, Lr = oracle_flex(orc, Q, K, V, scale, causal, window, input_pos, softcap=cap)
    compare(O, L, Or, Lr, what=f"softcap {case}")


ALIBI_CASES = [
    # B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, ragged
    (1, 8, 2, 300, 300, 128, True, 0, 0, False),
    (2, 4, 1, 130, 520, 64, True, 0, 390, True),
    (1, 4, 2, 384, 384, 128, False, 0, 0, False),
    (2, 4, 4, 260, 260, 128, True, 96, 0, True),
]


@pytest.mark.parametrize("case", ALIBI_CASES, ids=[str(c) for c in ALIBI_CASES])
def test_alibi(orc, case):
    B, Hq, Hkv, Sq, Sk, D, causal, window, input_pos, ragged = case
    Q, K, V = W.random_prefill(23 + hash(case) % 89, B, Hq, Hkv, Sq, Sk, D)
    slopes = W.alibi_slopes(Hq, seed=5)
    kl = ql = None
    if ragged:
        g = torch.Generator().manual_seed(3)
        kl = torch.randint(1, Sk + 1, (B,), generator=g).to(torch.int32)
        ql = torch.randint(1, Sq + 1, (B,), generator=g).to(torch.int32)
    scale = 1.0 / math.sqrt(D)
    O, L = gpu_flex(Q, K, V, scale, causal, window, input_pos, kl, ql, alibi=slopes)
    Or, Lr = oracle_flex(orc, Q, K, V, scale, causal, window, input_pos, kl, ql, alibi=slopes)
    compare(O, L, Or, Lr, what=f"alibi {case}")


DOC_CASES = [
    # B, Hq, Hkv, S, D, causal, window, min_len, max_len, use_block_mask
    (1, 4, 2, 700, 128, True, 0, 1, 200, True),
    (1, 4, 2, 700, 128, True, 0, 1, 200, False),
    (2, 2, 1, 513, 64, False, 0, 20, 300, True),
    (1, 4, 4, 640, 128, True, 100, 1, 400, True),
    (1, 2, 1, 1100, 128, True, 0, 100, 700, True),
]


@pytest.mark.parametrize("case", DOC_CASES, ids=[str(c) for c in DOC_CASES])
def test_document_mask(orc, case):
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, S, D, causal, window, lo, hi, use_bm = case
    Q, K, V = W.random_prefill(31 + hash(case) % 83, B, Hq, Hkv, S, S, D)
    doc = W.document_ids(S, seed=S + lo, min_len=lo, max_len=hi)
    bm = binding.block_mask_document(S, S, doc, doc, causal, window) if use_bm else None
    scale = 1.0 / math.sqrt(D)
    O, L = gpu_flex(Q, K, V, scale, causal, window, doc_q=doc, doc_kv=doc, block_mask=bm)
    Or, Lr = oracle_flex(orc, Q, K, V, scale, causal, window, doc_q=doc, doc_kv=doc)
    compare(O, L, Or, Lr, what=f"document {case}")


def test_document_mask_with_softcap_and_input_pos(orc):
    """Queries at absolute positions input_pos..: doc_q holds the ids of those
    positions, doc_kv the ids of every key."""
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, Sq, Sk, D, ip = 1, 4, 2, 300, 800, 128, 500
    Q, K, V = W.random_prefill(41, B, Hq, Hkv, Sq, Sk, D)
    doc = W.document_ids(Sk, seed=9, min_len=50, max_len=300)
    dq = doc[ip:ip + Sq].clone()
    bm = binding.block_mask_document(Sq, Sk, dq, doc, True, 0, ip)
    O, L = gpu_flex(Q, K, V, 0.2, True, 0, ip, softcap=4.0, doc_q=dq, doc_kv=doc, block_mask=bm)
    Or, Lr = oracle_flex(orc, Q, K, V, 0.2, True, 0, ip, softcap=4.0, doc_q=dq, doc_kv=doc)
    compare(O, L, Or, Lr, what="document + softcap + input_pos")


def test_block_mask_alone(orc):
    """Documents aligned to 64 positions: the BlockMask holds only 0 / 2 states and
    by itself is the document mask (no ids passed to the GPU)."""
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, S, D = 2, 4, 2, 640, 128
    Q, K, V = W.random_prefill(43, B, Hq, Hkv, S, S, D)
    doc = W.document_ids(S, seed=4, min_len=64, max_len=256, align=64)
    bm = binding.block_mask_document(S, S, doc, doc, False, 0)
    assert set(np.unique(bm.numpy()).tolist()) <= {0, 2}
    O, L = gpu_flex(Q, K, V, 0.09, False, block_mask=bm)
    Or, Lr = oracle_flex(orc, Q, K, V, 0.09, False, doc_q=doc, doc_kv=doc)
    compare(O, L, Or, Lr, what="block mask alone")


def test_one_hot_mask_probe(orc):
    """K = 0 and V = identity: O[i, j] = 1/n_i exactly where key j is visible from
    row i and 0 elsewhere, so the nonzero pattern is the mask, bit for bit
    (document + causal + window + block mask, row and key counts past a tile)."""
    from gqa_attention_flash_b200 import binding
    S, D = 128, 128
    for window in (0, 40):
        Q = torch.randn(1, 2, S, D, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
        K = torch.zeros(1, 1, S, D, dtype=torch.bfloat16)
        V = torch.eye(S, D, dtype=torch.bfloat16)[None, None]
        doc = W.document_ids(S, seed=12, min_len=1, max_len=40)
        bm = binding.block_mask_document(S, S, doc, doc, True, window)
        O, L = gpu_flex(Q, K, V, 0.1, True, window, doc_q=doc, doc_kv=doc, block_mask=bm)
        Or, Lr = oracle_flex(orc, Q, K, V, 0.1, True, window, doc_q=doc, doc_kv=doc)
        assert np.array_equal(O.double().numpy() != 0.0, Or != 0.0), f"window {window}"
        compare(O, L, Or, Lr, what=f"one-hot window {window}")


def test_all_blocks_empty():
    """A BlockMask of zeros: every row sees nothing, O = 0 and LSE = -inf."""
    B, Hq, Hkv, S, D = 1, 2, 1, 300, 64
    Q, K, V = W.random_prefill(47, B, Hq, Hkv, S, S, D)
    bm = torch.zeros((S + 63) // 64, (S + 63) // 64, dtype=torch.uint8)
    O, L = gpu_flex(Q, K, V, 0.125, False, block_mask=bm)
    assert torch.all(O == 0) and torch.all(torch.isneginf(L))


@pytest.mark.parametrize("key", sorted(W.FLEX_WORKLOADS))
def test_full_size_flex_workloads(orc, key):
    """The measured flex workloads at full size, in the launch configuration the
    benchmark times: sampled rows (tile edges, document boundaries, random)
    against the oracle."""
    from gpu_common import sample_rows
    from gqa_attention_flash_b200 import binding
    w = W.FLEX_WORKLOADS[key]
    Q, K, V, doc, slopes = W.make_flex(w)
    bm = binding.block_mask_document(w.S, w.S, doc, doc, w.causal) if doc is not None else None
    O, L = gpu_flex(Q, K, V, w.scale, w.causal, softcap=w.softcap, alibi=slopes, doc_q=doc,
                    doc_kv=doc, block_mask=bm)
    extra = ()
    if doc is not None:
        starts = np.flatnonzero(np.diff(doc.numpy())) + 1
        extra = tuple(starts) + tuple(starts - 1)
    rows = sample_rows(w.S, seed=w.seed, n_random=512, extra=extra)
    Or, Lr = orc.flex_fwd(Q[:, :, torch.as_tensor(rows, dtype=torch.long)].double().numpy(),
                          K.double().numpy(), V.double().numpy(), w.scale, causal=w.causal,
                          rows=rows, Sq=w.S, softcap=w.softcap,
                          alibi_slopes=None if slopes is None else slopes.double().numpy(),
                          doc_q=None if doc is None else doc.numpy(),
                          doc_kv=None if doc is None else doc.numpy())
    compare(O, L, Or, Lr, rows=rows, what=f"full-size {key}")


@pytest.mark.parametrize("mod", ["softcap", "alibi", "document"])
def test_nan_q_rows_past_q_lengths(orc, mod):
    """flex_attention! instantiations (soft cap, ALiBi, the document-mask list
    path): NaN query rows past q_lengths give O = +0.0 and LSE = -inf, and the
    valid rows match the oracle."""
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, S, D = 2, 4, 2, 390, 128
    Q, K, V = W.random_prefill(51, B, Hq, Hkv, S, S, D)
    ql = torch.tensor([390, 200], dtype=torch.int32)
    kl = torch.tensor([390, 390], dtype=torch.int32)
    Qp = Q.clone()
    Qp[1, :, 200:] = float("nan")
    kw = {}
    if mod == "softcap":
        kw = dict(softcap=5.0)
    elif mod == "alibi":
        kw = dict(alibi=W.alibi_slopes(Hq, seed=5))
    else:
        doc = W.document_ids(S, seed=6, min_len=20, max_len=150)
        kw = dict(doc_q=doc, doc_kv=doc)
    bm = binding.block_mask_document(S, S, kw["doc_q"], kw["doc_kv"], True, 0) \
        if mod == "document" else None
    O, L = gpu_flex(Qp, K, V, 0.09, True, 0, 0, kl, ql, block_mask=bm, **kw)
    Or, Lr = oracle_flex(orc, Q, K, V, 0.09, True, 0, 0, kl, ql, **kw)
    compare(O, L, Or, Lr, what=f"flex {mod} NaN past q_len")
    assert torch.all(O[1, :, 200:].view(torch.int16) == 0)
    assert torch.all(torch.isneginf(L[1, :, 200:]))
