"""Seeded synthetic inputs for the attention forward and split-KV decode.

This module holds no attention arithmetic: it only draws random tensors, in a
fixed order from fixed seeds, so that the CUDA path and the fp64 oracle can be
fed identical inputs.  Every tensor is drawn on the CPU with
``torch.Generator('cpu')`` as float32 N(0, 1) and rounded to bf16 (round to
nearest even).

Workloads (shapes and value structure follow the attention pages' use cases:
LLM prefill and decode, and image-to-image attention on a 64x64 token grid):

  tiny     B1 Hq2 Hkv1 S128 D64, scale 1/8, causal                       seed 0
  llm      B4 Hq32 Hkv8 S4096 D128, scale 1/sqrt(128), causal,
           every k_length 4096                                         seed 1
  window   B2 Hq32 Hkv8 S16384 D128, causal window 4096,
           k_lengths = q_lengths ~ U{8192..16384}                      seed 2
  image    B1 Hq=Hkv=32 S4096 D128, no mask; K gets a per-(head, 64-token
           block, d) offset ~ N(0, 0.5^2) shared by the block's tokens   seed 3
  decode   B64 Hq32 Hkv8 D128, cache capacity 32768,
           lengths ~ U{1024..32768}, n_splits 8                        seed 4

Draw order for the prefill workloads: Q, K, V, then the K block offsets
(image), then the lengths (window), all from one generator.  For decode, one
generator draws Q then the lengths; the cached keys and values of sequence b
come from a generator seeded ``seed * 65536 + 1 + b`` (K then V, only the
first lengths[b] rows), so one sequence can be re-drawn on its own.  Cache
rows at or past lengths[b] are filled with ``fill`` (0 by default).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int
    scale: float
    causal: bool
    window: int = 0
    input_pos: int = 0
    seed: int = 0
    full_k_lengths: bool = False          # pass an explicit k_lengths array of Sk
    ragged: tuple | None = None           # (lo, hi) inclusive range for k_len = q_len
    block_offset_std: float = 0.0         # image workload: per-64-token-block K offset
    block: int = 64
    q_block_offset_std: float = 0.0       # per-64-token-block Q offset (block-structured)

    def flops(self, k_lengths=None, q_lengths=None) -> int:
        """Algorithmic FLOPs: 4 * D * (number of visible (query, key) pairs)."""
        return 4 * self.D * self.Hq * visible_pairs(self, k_lengths, q_lengths)


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    Hq: int
    Hkv: int
    S_cap: int
    D: int
    n_splits: int
    len_lo: int
    len_hi: int
    seed: int = 4


TINY = PrefillWorkload("tiny causal GQA fwd B1 Hq2 Hkv1 S128 D64", 1, 2, 1, 128, 128, 64,
                       1.0 / 8.0, True, seed=0)
LLM = PrefillWorkload("LLM causal prefill B4 Hq32 Hkv8 S4096 D128", 4, 32, 8, 4096, 4096, 128,
                      1.0 / math.sqrt(128.0), True, seed=1, full_k_lengths=True)
WINDOW = PrefillWorkload("sliding-window ragged prefill B2 Hq32 Hkv8 S16384 D128 w4096",
                         2, 32, 8, 16384, 16384, 128, 1.0 / math.sqrt(128.0), True, window=4096,
                         seed=2, ragged=(8192, 16384))
IMAGE = PrefillWorkload("image-image non-causal B1 H32 S4096 D128 (64x64 tokens)", 1, 32, 32,
                        4096, 4096, 128, 1.0 / math.sqrt(128.0), False, seed=3,
                        block_offset_std=0.5)
DECODE = DecodeWorkload("split-KV decode B64 Hq32 Hkv8 D128 cap32768 n_splits8", 64, 32, 8,
                        32768, 128, 8, 1024, 32768, seed=4)

BLOCK_SPARSE = PrefillWorkload("block-structured image attention B1 H32 S4096 D128: Q and K "
                               "offsets per 64-token block ~ N(0, 1.5^2)", 1, 32, 32, 4096, 4096,
                               128, 1.0 / math.sqrt(128.0), False, seed=8, block_offset_std=1.5,
                               q_block_offset_std=1.5)

PREFILL_WORKLOADS = {"tiny": TINY, "llm": LLM, "window": WINDOW, "image": IMAGE}


@dataclass(frozen=True)
class FlexWorkload:
    """flex_attention! forward workload: a prefill shape plus one score mod and,
    optionally, packed documents (DocumentMask with a BlockMask)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    causal: bool
    softcap: float = 0.0
    alibi: bool = False
    doc_len: tuple | None = None          # (min, max) document length, packed to S
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def flops(self, doc=None) -> int:
        """4 * D * visible (query, key) pairs, summed over heads and batch."""
        if doc is None:
            pairs = self.S * (self.S + 1) // 2 if self.causal else self.S * self.S
        else:
            n = torch.bincount(doc.to(torch.int64)).to(torch.int64)
            pairs = int((n * (n + 1) // 2).sum()) if self.causal else int((n * n).sum())
        return 4 * self.D * self.Hq * self.B * pairs


FLEX_DOC = FlexWorkload("document-masked causal prefill, soft-cap 50: B1 Hq32 Hkv8 S16384 D128, "
                        "documents 256..4096", 1, 32, 8, 16384, 128, True, softcap=50.0,
                        doc_len=(256, 4096), seed=5)
FLEX_ALIBI = FlexWorkload("ALiBi causal prefill B4 Hq32 Hkv8 S4096 D128", 4, 32, 8, 4096, 128,
                          True, alibi=True, seed=6)
FLEX_WORKLOADS = {"doc_softcap": FLEX_DOC, "alibi": FLEX_ALIBI}


def make_flex(w: FlexWorkload):
    """CPU inputs of a flex workload: (Q, K, V, doc ids or None, ALiBi slopes or None)."""
    Q, K, V = random_prefill(w.seed, w.B, w.Hq, w.Hkv, w.S, w.S, w.D)
    doc = document_ids(w.S, w.seed, *w.doc_len) if w.doc_len else None
    slopes = alibi_slopes(w.Hq, w.seed) if w.alibi else None
    return Q, K, V, doc, slopes


def visible_pairs(w: PrefillWorkload, k_lengths=None, q_lengths=None) -> int:
    """Number of (query row, key) pairs one query head sees, summed over batch.

    Interval counting per row: row i (absolute position p = input_pos + i) sees
    keys [lo, hi) with hi = min(k_len, p + 1) if causal else k_len, and lo =
    max(0, p - window + 1) for a window, 0 otherwise.
    """
    total = 0
    for b in range(w.B):
        kl = int(k_lengths[b]) if k_lengths is not None else w.Sk
        ql = int(q_lengths[b]) if q_lengths is not None else w.Sq
        kl, ql = min(kl, w.Sk), min(ql, w.Sq)
        if not w.causal:
            total += ql * kl
            continue
        # sum over rows of max(0, min(kl, p+1) - lo(p)), done in closed form by pieces
        for_rows = torch.arange(ql, dtype=torch.int64) + w.input_pos
        hi = torch.clamp(for_rows + 1, max=kl)
        lo = torch.clamp(for_rows - w.window + 1, min=0) if w.window > 0 else torch.zeros_like(hi)
        total += int(torch.clamp(hi - lo, min=0).sum())
    return total


@dataclass
class PrefillInputs:
    Q: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    k_lengths: torch.Tensor | None
    q_lengths: torch.Tensor | None
    extra: dict = field(default_factory=dict)


def make_prefill(w: PrefillWorkload) -> PrefillInputs:
    """bf16 CPU tensors Q (B,Hq,Sq,D), K/V (B,Hkv,Sk,D) and int32 lengths."""
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    Q = torch.randn(w.B, w.Hq, w.Sq, w.D, generator=g, dtype=torch.float32)
    K = torch.randn(w.B, w.Hkv, w.Sk, w.D, generator=g, dtype=torch.float32)
    V = torch.randn(w.B, w.Hkv, w.Sk, w.D, generator=g, dtype=torch.float32)
    if w.block_offset_std > 0:
        nblk = (w.Sk + w.block - 1) // w.block
        c = torch.randn(w.Hkv, nblk, w.D, generator=g, dtype=torch.float32) * w.block_offset_std
        K = K + c.repeat_interleave(w.block, dim=1)[:, :w.Sk].unsqueeze(0)
    if w.q_block_offset_std > 0:
        nqb = (w.Sq + w.block - 1) // w.block
        cq = torch.randn(w.Hq, nqb, w.D, generator=g, dtype=torch.float32) * w.q_block_offset_std
        Q = Q + cq.repeat_interleave(w.block, dim=1)[:, :w.Sq].unsqueeze(0)
    k_len = q_len = None
    if w.ragged is not None:
        lo, hi = w.ragged
        k_len = torch.randint(lo, hi + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
        q_len = k_len.clone()
    elif w.full_k_lengths:
        k_len = torch.full((w.B,), w.Sk, dtype=torch.int32)
    return PrefillInputs(Q.to(torch.bfloat16), K.to(torch.bfloat16), V.to(torch.bfloat16),
                         k_len, q_len)


def random_prefill(seed, B, Hq, Hkv, Sq, Sk, D):
    """Plain N(0,1) bf16 Q/K/V of arbitrary shape (parity and edge cases)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    Q = torch.randn(B, Hq, Sq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(B, Hkv, Sk, D, generator=g).to(torch.bfloat16)
    V = torch.randn(B, Hkv, Sk, D, generator=g).to(torch.bfloat16)
    return Q, K, V


def document_ids(total: int, seed: int, min_len: int = 1, max_len: int = 512, align: int = 1):
    """int32 (total,) document ids of packed documents: consecutive runs with
    lengths drawn uniformly from [min_len, max_len] (multiples of ``align``),
    the last one cut at ``total`` (the DocumentMask workloads)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    ids = torch.empty(total, dtype=torch.int32)
    pos, d = 0, 0
    lo, hi = max(1, min_len // align), max(1, max_len // align)
    while pos < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g)) * align
        ids[pos:pos + n] = d
        pos += n
        d += 1
    return ids


def alibi_slopes(Hq: int, seed: int):
    """fp32 (Hq,) ALiBi slopes: the geometric family -2^(-8 (h+1) / Hq) of the
    ALiBi paper with a random sign flip per head, so both signs are exercised."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    mag = torch.tensor([2.0 ** (-8.0 * (h + 1) / Hq) for h in range(Hq)], dtype=torch.float32)
    sign = torch.where(torch.rand(Hq, generator=g) < 0.5, -1.0, 1.0)
    return (mag * sign).to(torch.float32)


def decode_query_and_lengths(w: DecodeWorkload):
    g = torch.Generator(device="cpu").manual_seed(w.seed)
    Q = torch.randn(w.B, w.Hq, w.D, generator=g).to(torch.bfloat16)
    lengths = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=g,
                            dtype=torch.int64).to(torch.int32)
    return Q, lengths


def decode_sequence_kv(w: DecodeWorkload, b: int, length: int):
    """bf16 (Hkv, length, D) keys and values of sequence b."""
    g = torch.Generator(device="cpu").manual_seed(w.seed * 65536 + 1 + b)
    K = torch.randn(w.Hkv, length, w.D, generator=g).to(torch.bfloat16)
    V = torch.randn(w.Hkv, length, w.D, generator=g).to(torch.bfloat16)
    return K, V


def fill_decode_cache(w: DecodeWorkload, lengths, K_cache, V_cache, fill: float = 0.0):
    """Write every sequence's drawn K/V rows into caches of shape (B,Hkv,S_cap,D)
    (on any device); rows at or past lengths[b] get ``fill``."""
    K_cache.fill_(fill)
    V_cache.fill_(fill)
    for b in range(w.B):
        n = int(lengths[b])
        Kb, Vb = decode_sequence_kv(w, b, n)
        K_cache[b, :, :n].copy_(Kb, non_blocking=False)
        V_cache[b, :, :n].copy_(Vb, non_blocking=False)


@dataclass(frozen=True)
class PagedDecodeWorkload:
    """Decode from a paged KV cache (num_blocks, block_size, Hkv, D): the same
    queries, lengths and per-sequence K/V as ``base``, scattered into a pool of
    blocks in a seeded random order (plus ``spare`` unused blocks)."""
    name: str
    base: DecodeWorkload
    block_size: int
    spare: int = 64
    seed: int = 7


PAGED_DECODE = PagedDecodeWorkload("paged split-KV decode B64 Hq32 Hkv8 D128 block 16, "
                                   "lengths 1024..32768, n_splits 8", DECODE, 16)


def paged_layout(lengths, block_size: int, spare: int, seed: int):
    """(block_tables int32 (B, max_blocks), num_blocks): every sequence's logical
    blocks mapped to distinct physical blocks in a random order; table entries past
    a sequence's last block are -1."""
    n_blk = [(int(n) + block_size - 1) // block_size for n in lengths]
    max_blocks = max(1, max(n_blk) if n_blk else 1)
    num_blocks = sum(n_blk) + spare
    g = torch.Generator(device="cpu").manual_seed(seed)
    perm = torch.randperm(num_blocks, generator=g).to(torch.int32)
    tables = torch.full((len(n_blk), max_blocks), -1, dtype=torch.int32)
    pos = 0
    for b, n in enumerate(n_blk):
        tables[b, :n] = perm[pos:pos + n]
        pos += n
    return tables, num_blocks


def fill_paged_cache(K_pool, V_pool, tables, seq_kv):
    """Scatter per-sequence (Hkv, length, D) K/V (``seq_kv(b)`` returns them) into the
    block pools (num_blocks, block_size, Hkv, D) along the block tables."""
    bs = K_pool.shape[1]
    for b in range(tables.shape[0]):
        Kb, Vb = seq_kv(b)
        n = Kb.shape[1]
        nb = (n + bs - 1) // bs
        if nb == 0:
            continue
        idx = tables[b, :nb].to(torch.long).to(K_pool.device)
        for src, pool in ((Kb, K_pool), (Vb, V_pool)):
            pad = torch.zeros(src.shape[0], nb * bs, src.shape[2], dtype=src.dtype,
                              device=src.device)
            pad[:, :n] = src
            blocks = pad.reshape(src.shape[0], nb, bs, src.shape[2]).permute(1, 2, 0, 3)
            pool.index_copy_(0, idx, blocks.contiguous().to(pool.device))


def make_paged_decode(w: PagedDecodeWorkload, device="cpu"):
    """Q (B,Hq,D), K/V pools, block tables and seq_lens of a paged decode workload."""
    d = w.base
    Q, lengths = decode_query_and_lengths(d)
    tables, num_blocks = paged_layout(lengths.tolist(), w.block_size, w.spare, w.seed)
    shape = (num_blocks, w.block_size, d.Hkv, d.D)
    K_pool = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    V_pool = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    fill_paged_cache(K_pool, V_pool, tables,
                     lambda b: decode_sequence_kv(d, b, int(lengths[b])))
    return Q, K_pool, V_pool, tables, lengths


def decode_bytes(w: DecodeWorkload, lengths) -> int:
    """Algorithmic bytes of one decode: the valid K/V prefix plus Q and O."""
    kv = 2 * w.Hkv * w.D * 2 * int(sum(int(x) for x in lengths))
    return kv + 2 * (w.B * w.Hq * w.D * 2)
