"""Seeded random configurations of the whole hot path against the fp64 oracle.

The fixed parity cases elsewhere pick shapes and masks by hand.  Here a seeded
generator draws them: batch, query and KV heads (GQA groups 1-8), head size 64
or 128, Sq and Sk from 1 to several tiles with ragged ends, causal or not, a
sliding window (Tylo.jl "Primitives" page, `attention!` / mlx-arsenal
"Attention" page, `sliding_window_mask`), an input_pos offset, and per-batch
k_lengths / q_lengths that may be 0, cut a tile or cover the whole sequence.
Each draw runs through the C ABI and is compared with the oracle:

- forward O and LSE within the tolerances of every parity test (1.5e-2 / 1e-3),
  with rows that see no key exactly O = +0.0, LSE = -inf;
- which keys each row attends to, bit for bit (the one-hot probe of
  test_gpu_mask_probe: K = 0, V one-hot in key index);
- split-KV decode with random lengths and split counts;
- the backward's dQ, dK, dV (tolerance as in test_gpu_bwd);
- flex_attention! with a random score mod and mask mod, paged decode over random
  block sizes and pools, and BlockMask-only calls on the block-sparse kernel;
- larger forward draws (up to 8192 rows and keys) on sampled rows.

The seeds are fixed, so every run checks the same configurations."""
import math

import numpy as np
import pytest
import torch

from gpu_common import compare, gpu_decode, gpu_prefill, oracle_prefill
from gqa_attention_flash_b200 import workloads as W
from test_gpu_bwd import check, gpu_fwd_bwd
from test_gpu_mask_probe import prefill_probe

pytestmark = pytest.mark.gpu


def draw_prefill(rng, max_rows=400, max_keys=700, max_hq=8):
    """One random prefill configuration (all sizes small enough for the oracle)."""
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([g for g in (1, 2, 4, 8) if Hkv * g <= max_hq]))
    B = int(rng.integers(1, 4))
    D = int(rng.choice([64, 128]))
    Sq = int(rng.integers(1, max_rows + 1))
    Sk = int(rng.integers(1, max_keys + 1))
    causal = bool(rng.integers(0, 2))
    # the window is causal (sliding_window_mask); attn_fwd refuses it without causal
    window = int(rng.integers(1, Sk + 1)) if causal and rng.random() < 0.5 else 0
    input_pos = int(rng.integers(0, max(1, Sk - Sq + 1))) if rng.random() < 0.5 else 0
    kl = ql = None
    if rng.random() < 0.5:
        kl = rng.integers(0, Sk + 1, size=B).astype(np.int32)
        kl[rng.integers(0, B)] = Sk if rng.random() < 0.5 else kl[0]
    if rng.random() < 0.4:
        ql = rng.integers(0, Sq + 1, size=B).astype(np.int32)
    return dict(B=B, Hq=Hkv * G, Hkv=Hkv, Sq=Sq, Sk=Sk, D=D, causal=causal, window=window,
                input_pos=input_pos, k_lengths=kl, q_lengths=ql)


def describe(c):
    kl = None if c["k_lengths"] is None else c["k_lengths"].tolist()
    ql = None if c["q_lengths"] is None else c["q_lengths"].tolist()
    return (f"B{c['B']} Hq{c['Hq']} Hkv{c['Hkv']} Sq{c['Sq']} Sk{c['Sk']} D{c['D']} "
            f"causal {c['causal']} window {c['window']} input_pos {c['input_pos']} "
            f"k_lengths {kl} q_lengths {ql}")


FWD_SEEDS = list(range(1000, 1064))


@pytest.mark.parametrize("seed", FWD_SEEDS)
def test_forward_random_config(orc, seed):
    c = draw_prefill(np.random.default_rng(seed))
    Q, K, V = W.random_prefill(seed, c["B"], c["Hq"], c["Hkv"], c["Sq"], c["Sk"], c["D"])
    kl = None if c["k_lengths"] is None else torch.from_numpy(c["k_lengths"])
    ql = None if c["q_lengths"] is None else torch.from_numpy(c["q_lengths"])
    scale = 1.0 / math.sqrt(c["D"])
    O, L = gpu_prefill(Q, K, V, scale, c["causal"], c["window"], c["input_pos"], kl, ql)
    Or, Lr = oracle_prefill(orc, Q, K, V, scale, c["causal"], c["window"], c["input_pos"], kl, ql)
    compare(O, L, Or, Lr, what=describe(c))
    # rows that see no key (past q_lengths, or masked entirely): every bit is +0.0
    empty = torch.from_numpy(np.isneginf(Lr))
    assert torch.all(O.view(torch.int16)[empty] == 0), describe(c)


MASK_SEEDS = list(range(2000, 2024))


@pytest.mark.parametrize("seed", MASK_SEEDS)
def test_forward_random_config_masks_bit_exact(orc, seed):
    c = draw_prefill(np.random.default_rng(seed), max_rows=700, max_keys=1100)
    prefill_probe(orc, c["B"], c["Hq"], c["Hkv"], c["Sq"], c["Sk"], c["D"], c["causal"],
                  c["window"], c["input_pos"], c["k_lengths"], c["q_lengths"], what=describe(c))


DECODE_SEEDS = list(range(3000, 3024))


@pytest.mark.parametrize("seed", DECODE_SEEDS)
def test_decode_random_config(orc, seed):
    rng = np.random.default_rng(seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([g for g in (1, 2, 4, 8, 16) if Hkv * g <= 32]))
    B = int(rng.integers(1, 9))
    D = int(rng.choice([64, 128]))
    S_cap = int(rng.integers(1, 3000))
    n_splits = int(rng.choice([1, 2, 3, 8, 13, 64]))
    lengths = rng.integers(0, S_cap + 1, size=B).astype(np.int32)
    lengths[rng.integers(0, B)] = S_cap
    Hq = Hkv * G
    g = torch.Generator().manual_seed(seed)
    Q = torch.randn(B, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, S_cap, D, generator=g).to(torch.bfloat16)
    what = f"B{B} Hq{Hq} Hkv{Hkv} D{D} cap {S_cap} splits {n_splits} lengths {lengths.tolist()}"
    O = gpu_decode(Q, K, V, torch.from_numpy(lengths), n_splits)
    Or, _ = orc.decode(Q.double().numpy(), K.double().numpy(), V.double().numpy(), lengths)
    Og = O.double().numpy()
    assert np.all(np.isfinite(Og)), what
    err = float(np.abs(Og - Or).max())
    assert err <= 1.5e-2, f"{what}: max |dO| = {err}"
    # sequences of length 0 have no key: O is +0.0 in every bit
    zero = torch.from_numpy(lengths == 0)
    assert torch.all(O.view(torch.int16)[zero] == 0), what


BWD_SEEDS = list(range(4000, 4016))


@pytest.mark.parametrize("seed", BWD_SEEDS)
def test_backward_random_config(orc, seed):
    c = draw_prefill(np.random.default_rng(seed), max_rows=300, max_keys=400, max_hq=4)
    Q, K, V = W.random_prefill(seed, c["B"], c["Hq"], c["Hkv"], c["Sq"], c["Sk"], c["D"])
    dO = torch.randn(c["B"], c["Hq"], c["Sq"], c["D"],
                     generator=torch.Generator().manual_seed(seed + 1)).to(torch.bfloat16)
    kl = None if c["k_lengths"] is None else torch.from_numpy(c["k_lengths"])
    ql = None if c["q_lengths"] is None else torch.from_numpy(c["q_lengths"])
    scale = 1.0 / math.sqrt(c["D"])
    dQ, dK, dV = gpu_fwd_bwd(Q, K, V, dO, scale, c["causal"], c["window"], c["input_pos"], kl, ql)
    rQ, rK, rV = orc.attn_bwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(),
                              dO.double().numpy(), scale, causal=c["causal"], window=c["window"],
                              input_pos=c["input_pos"], k_lengths=c["k_lengths"],
                              q_lengths=c["q_lengths"])
    what = describe(c)
    check(dQ, rQ, f"dQ {what}")
    check(dK, rK, f"dK {what}")
    check(dV, rV, f"dV {what}")


def gpu_flex_any(Q, K, V, scale, c, softcap, alibi, doc_q, doc_kv, block_mask):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    to = lambda t: None if t is None else t.to(dev)
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    L = torch.full(Q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
    kl = None if c["k_lengths"] is None else torch.from_numpy(c["k_lengths"])
    ql = None if c["q_lengths"] is None else torch.from_numpy(c["q_lengths"])
    binding.attn_fwd_flex(O, Q.to(dev), K.to(dev), V.to(dev), L, scale, c["causal"], c["window"],
                          c["input_pos"], to(kl), to(ql), softcap, to(alibi), to(doc_q),
                          to(doc_kv), to(block_mask))
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return O.cpu(), L.cpu()


FLEX_SEEDS = list(range(5000, 5048))


@pytest.mark.parametrize("seed", FLEX_SEEDS)
def test_flex_random_config(orc, seed):
    """flex_attention! (Tylo.jl "Primitives" page): a random score mod (none,
    SoftCapScore or AliBiScore) with a random mask mod (none, DocumentMask with or
    without its BlockMask, or a random BlockMask alone, shared or per head) on top
    of the drawn causal / window / input_pos / lengths."""
    from gqa_attention_flash_b200 import binding
    rng = np.random.default_rng(seed)
    c = draw_prefill(rng, max_rows=500, max_keys=900)
    B, Hq, Sq, Sk, D = c["B"], c["Hq"], c["Sq"], c["Sk"], c["D"]
    Q, K, V = W.random_prefill(seed, B, Hq, c["Hkv"], Sq, Sk, D)
    scale = float(rng.uniform(0.05, 0.3))
    mod = int(rng.integers(0, 3))
    softcap = float(rng.uniform(2.0, 50.0)) if mod == 1 else 0.0
    alibi = None
    if mod == 2:
        alibi = torch.from_numpy((rng.choice([-1.0, 1.0], Hq) * 2.0 ** (-rng.uniform(0, 8, Hq)))
                                 .astype(np.float32))
    mask = int(rng.integers(0, 4))
    doc_q = doc_kv = bm = keep = None
    if mask in (1, 2):  # DocumentMask over absolute positions 0 .. max(Sk, input_pos + Sq)
        n = max(Sk, c["input_pos"] + Sq)
        lo = int(rng.integers(1, 200))
        doc = W.document_ids(n, seed=seed, min_len=lo, max_len=lo + int(rng.integers(0, 400)))
        doc_q = doc[c["input_pos"]:c["input_pos"] + Sq].clone()
        doc_kv = doc[:Sk].clone()
        if mask == 2:
            bm = binding.block_mask_document(Sq, Sk, doc_q, doc_kv, c["causal"], c["window"],
                                             c["input_pos"])
    elif mask == 3:  # a random BlockMask alone: states 1 and 2 both keep the block
        nqb, nkb = (Sq + 63) // 64, (Sk + 63) // 64
        per_head = bool(rng.integers(0, 2))
        shape = (B, Hq, nqb, nkb) if per_head else (nqb, nkb)
        density = float(rng.uniform(0.1, 1.0))
        kept = rng.random(shape) < density
        bm = torch.from_numpy(np.where(kept, rng.integers(1, 3, shape), 0).astype(np.uint8))
        keep = np.ascontiguousarray(np.broadcast_to((bm.numpy() != 0).astype(np.uint8),
                                                    (B, Hq, nqb, nkb)))
    what = (f"{describe(c)} scale {scale:.3f} softcap {softcap:.2f} alibi {alibi is not None} "
            f"mask {['none', 'document', 'document + BlockMask', 'BlockMask'][mask]}")
    O, L = gpu_flex_any(Q, K, V, scale, c, softcap, alibi, doc_q, doc_kv, bm)
    npy = lambda t: None if t is None else t.numpy()
    Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                          causal=c["causal"], window=c["window"], input_pos=c["input_pos"],
                          k_lengths=c["k_lengths"], q_lengths=c["q_lengths"], softcap=softcap,
                          alibi_slopes=None if alibi is None else alibi.double().numpy(),
                          doc_q=npy(doc_q), doc_kv=npy(doc_kv), block_keep=keep)
    compare(O, L, Or, Lr, what=what)
    empty = torch.from_numpy(np.isneginf(Lr))
    assert torch.all(O.view(torch.int16)[empty] == 0), what


PAGED_SEEDS = list(range(6000, 6024))


@pytest.mark.parametrize("seed", PAGED_SEEDS)
def test_paged_decode_random_config(orc, seed):
    """Paged split-KV decode: random block size (a power of two from 8 to 256),
    lengths, GQA group and split count over a shuffled pool with spare blocks."""
    from test_gpu_paged import gpu_paged, random_paged
    rng = np.random.default_rng(seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([g for g in (1, 2, 4, 8, 16) if Hkv * g <= 32]))
    B = int(rng.integers(1, 7))
    D = int(rng.choice([64, 128]))
    bs = int(rng.choice([8, 16, 32, 64, 128, 256]))
    lengths = [int(x) for x in rng.integers(0, 2500, size=B)]
    n_splits = int(rng.choice([1, 2, 5, 8, 16]))
    Q, Kp, Vp, tables, lens = random_paged(seed, B, Hkv * G, Hkv, D, bs, lengths,
                                           spare=int(rng.integers(0, 9)))
    what = f"B{B} Hq{Hkv * G} Hkv{Hkv} D{D} block {bs} splits {n_splits} lengths {lengths}"
    O = gpu_paged(Q, Kp, Vp, tables, lens, n_splits)
    Or, _ = orc.decode_paged(Q.double().numpy(), Kp.double().numpy(), Vp.double().numpy(),
                             tables.numpy(), lens.numpy())
    err = float(np.abs(O.double().numpy() - Or).max())
    assert err <= 1.5e-2, f"{what}: max |dO| = {err}"
    for b, n in enumerate(lengths):
        if n == 0:
            assert torch.all(O[b].view(torch.int16) == 0), what


BSPARSE_SEEDS = list(range(7000, 7024))


@pytest.mark.parametrize("seed", BSPARSE_SEEDS)
def test_block_sparse_random_config(orc, seed):
    """A BlockMask alone (no score mod, documents, causal mask or lengths), which
    runs the block-sparse kernel: random shapes, densities from empty to full,
    shared or per-head masks."""
    rng = np.random.default_rng(seed)
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4]))
    B = int(rng.integers(1, 3))
    D = int(rng.choice([64, 128]))
    Sq = int(rng.integers(1, 1200))
    Sk = int(rng.integers(1, 2500))
    Hq = Hkv * G
    nqb, nkb = (Sq + 63) // 64, (Sk + 63) // 64
    per_head = bool(rng.integers(0, 2))
    shape = (B, Hq, nqb, nkb) if per_head else (nqb, nkb)
    density = float(rng.choice([0.0, 0.05, 0.2, 0.5, 1.0]))
    kept = rng.random(shape) < density
    bm = torch.from_numpy(np.where(kept, rng.integers(1, 3, shape), 0).astype(np.uint8))
    keep = np.ascontiguousarray(np.broadcast_to((bm.numpy() != 0).astype(np.uint8),
                                                (B, Hq, nqb, nkb)))
    Q, K, V = W.random_prefill(seed, B, Hq, Hkv, Sq, Sk, D)
    scale = 1.0 / math.sqrt(D)
    c = dict(causal=False, window=0, input_pos=0, k_lengths=None, q_lengths=None)
    what = f"B{B} Hq{Hq} Hkv{Hkv} Sq{Sq} Sk{Sk} D{D} density {density} per_head {per_head}"
    O, L = gpu_flex_any(Q, K, V, scale, c, 0.0, None, None, None, bm)
    Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                          block_keep=keep)
    compare(O, L, Or, Lr, what=what)
    empty = torch.from_numpy(np.isneginf(Lr))
    assert torch.all(O.view(torch.int16)[empty] == 0), what


LARGE_SEEDS = list(range(8000, 8016))


@pytest.mark.parametrize("seed", LARGE_SEEDS)
def test_forward_random_large_config(orc, seed):
    """Larger draws (up to 8192 rows and keys, 32 query heads): enough work items that the
    persistent CTAs take over several in turn.  The oracle checks sampled rows: tile edges,
    the ends of the lengths and random rows, for every batch and head."""
    from gpu_common import sample_rows
    rng = np.random.default_rng(seed)
    c = draw_prefill(rng, max_rows=8192, max_keys=8192, max_hq=32)
    Q, K, V = W.random_prefill(seed, c["B"], c["Hq"], c["Hkv"], c["Sq"], c["Sk"], c["D"])
    kl = None if c["k_lengths"] is None else torch.from_numpy(c["k_lengths"])
    ql = None if c["q_lengths"] is None else torch.from_numpy(c["q_lengths"])
    scale = 1.0 / math.sqrt(c["D"])
    O, L = gpu_prefill(Q, K, V, scale, c["causal"], c["window"], c["input_pos"], kl, ql)
    extra = [] if ql is None else [int(x) + d for x in ql.tolist() for d in (-1, 0)]
    rows = sample_rows(c["Sq"], seed, n_random=24, extra=extra)
    Or, Lr = oracle_prefill(orc, Q, K, V, scale, c["causal"], c["window"], c["input_pos"], kl, ql,
                            rows=rows)
    compare(O, L, Or, Lr, rows=rows, what=describe(c))
