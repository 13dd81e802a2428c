"""Block-sparse prefill on the GPU: RBS block scores and block mask
(attn_rbs_block_mask) and attention over the kept 64x64 blocks (attn_fwd_flex
with per-head block masks), against the fp64 oracle.

The keep/skip decision compares a float score with a threshold; blocks whose
oracle score lies within MARGIN of the threshold may go either way on the two
sides, so masks are compared away from the threshold, and attention rows are
compared where both masks agree on the whole row."""
import math

import numpy as np
import pytest
import torch

from gpu_common import compare
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu

SCORE_TOL = 2e-3
MARGIN = 1e-2


def gpu_rbs(Q, K, alpha_base=0.22, alpha_rescue=0.18, diagonal=1):
    from gqa_attention_flash_b200 import binding
    dev = torch.device("cuda")
    mask, base, resc = binding.rbs_block_mask(Q.to(dev), K.to(dev), alpha_base, alpha_rescue,
                                              diagonal, want_scores=True)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    return mask.cpu(), base.cpu().double().numpy(), resc.cpu().double().numpy()


def borderline(base, resc, alpha_base, alpha_rescue):
    """Blocks whose (oracle) score is within MARGIN of either branch's threshold."""
    tb = base.max(axis=-1, keepdims=True) + math.log(alpha_base)
    tr = resc.max(axis=-1, keepdims=True) + math.log(alpha_rescue)
    return (np.abs(base - tb) < MARGIN) | (np.abs(resc - tr) < MARGIN)


CASES = [
    # B, Hq, Hkv, Sq, Sk, D, block_offset_std
    (1, 4, 2, 300, 300, 128, 0.5),
    (2, 2, 1, 256, 700, 64, 1.0),
    (1, 4, 4, 640, 640, 128, 0.0),
    (1, 2, 2, 1000, 1000, 128, 0.8),
    (1, 2, 1, 200, 5000, 64, 0.8),    # 79 key blocks: two centroid groups, beta sorted apart
    (1, 1, 1, 64, 8192, 128, 1.2),    # 128 key blocks
]


def rbs_inputs(case, seed):
    B, Hq, Hkv, Sq, Sk, D, off = case
    Q, K, V = W.random_prefill(seed, B, Hq, Hkv, Sq, Sk, D)
    if off > 0:  # spread block centroids, like the image workload
        g = torch.Generator().manual_seed(seed + 1)
        nkb = (Sk + 63) // 64
        c = torch.randn(Hkv, nkb, D, generator=g) * off
        K = (K.float() + c.repeat_interleave(64, dim=1)[:, :Sk].unsqueeze(0)).to(torch.bfloat16)
    return Q, K, V


# Scores only: up to 64 key blocks, more query blocks than one wave of scores CTAs
# holds one each, so a CTA scores several in turn (with the next one's load in flight).
SCORE_CASES = CASES + [(1, 8, 2, 8192, 4096, 64, 0.8), (2, 16, 4, 4096, 4096, 128, 1.0)]


@pytest.mark.parametrize("case", SCORE_CASES, ids=[str(c) for c in SCORE_CASES])
def test_rbs_scores_and_mask(orc, case):
    Q, K, V = rbs_inputs(case, 50 + SCORE_CASES.index(case))
    mask, base, resc = gpu_rbs(Q, K)
    ob, orr = orc.rbs_block_scores(Q.double().numpy(), K.double().numpy())
    assert np.max(np.abs(base - ob)) <= SCORE_TOL, np.max(np.abs(base - ob))
    assert np.max(np.abs(resc - orr)) <= SCORE_TOL, np.max(np.abs(resc - orr))
    keep = orc.rbs_block_mask(ob, orr)
    assert set(np.unique(mask.numpy()).tolist()) <= {0, 2}
    gm = mask.numpy() == 2
    ok = ~borderline(ob, orr, 0.22, 0.18)
    assert np.array_equal(gm[ok], keep.astype(bool)[ok])
    assert ok.mean() > 0.9


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_block_sparse_attention(orc, case):
    from gqa_attention_flash_b200 import binding
    B, Hq, Hkv, Sq, Sk, D, off = case
    Q, K, V = rbs_inputs(case, 60 + CASES.index(case))
    dev = torch.device("cuda")
    mask = binding.rbs_block_mask(Q.to(dev), K.to(dev))
    O = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device=dev)
    L = torch.full(Q.shape[:3], float("nan"), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(D)
    binding.attn_fwd_flex(O, Q.to(dev), K.to(dev), V.to(dev), L, scale, False, block_mask=mask)
    st = binding.last_device_status()
    assert st == 0, binding.status_string(st)
    ob, orr = orc.rbs_block_scores(Q.double().numpy(), K.double().numpy())
    keep = orc.rbs_block_mask(ob, orr)
    Or, Lr = orc.flex_fwd(Q.double().numpy(), K.double().numpy(), V.double().numpy(), scale,
                          block_keep=keep)
    # rows of query blocks whose mask row agrees on both sides
    agree = np.all((mask.cpu().numpy() == 2) == keep.astype(bool), axis=-1)  # (B, Hq, nqb)
    assert agree.mean() > 0.9
    Og, Lg = O.cpu().double().numpy(), L.cpu().double().numpy()
    for b in range(B):
        for h in range(Hq):
            for qb in np.flatnonzero(agree[b, h]):
                sl = slice(64 * qb, min(64 * qb + 64, Sq))
                compare(torch.from_numpy(Og[b:b + 1, h:h + 1, sl]),
                        torch.from_numpy(Lg[b:b + 1, h:h + 1, sl]),
                        Or[b:b + 1, h:h + 1, sl], Lr[b:b + 1, h:h + 1, sl],
                        what=f"{case} b{b} h{h} qb{qb}")


@pytest.mark.parametrize("key", ["image", "block_sparse"])
def test_image_workloads_full_size(orc, key):
    """The image workload (B1 H32 S4096 D128, spread K block centroids) and the
    block-structured one the benchmark times (Q and K block offsets) at full size:
    scores and mask of every block, and sampled attention rows of agreeing blocks."""
    from gpu_common import sample_rows
    from gqa_attention_flash_b200 import binding
    w = W.IMAGE if key == "image" else W.BLOCK_SPARSE
    x = W.make_prefill(w)
    dev = torch.device("cuda")
    mask, base, resc = gpu_rbs(x.Q, x.K)
    ob, orr = orc.rbs_block_scores(x.Q.double().numpy(), x.K.double().numpy())
    assert np.max(np.abs(base - ob)) <= SCORE_TOL and np.max(np.abs(resc - orr)) <= SCORE_TOL
    keep = orc.rbs_block_mask(ob, orr)
    ok = ~borderline(ob, orr, 0.22, 0.18)
    assert np.array_equal((mask.numpy() == 2)[ok], keep.astype(bool)[ok])
    O = torch.empty(x.Q.shape, dtype=torch.bfloat16, device=dev)
    L = torch.empty(x.Q.shape[:3], dtype=torch.float32, device=dev)
    binding.attn_fwd_flex(O, x.Q.to(dev), x.K.to(dev), x.V.to(dev), L, w.scale, False,
                          block_mask=mask.to(dev))
    assert binding.last_device_status() == 0
    rows = sample_rows(w.Sq, seed=9, n_random=8)
    agree = np.all((mask.numpy() == 2) == keep.astype(bool), axis=-1)[0]  # (Hq, nqb)
    Or, Lr = orc.flex_fwd(x.Q[:, :, torch.as_tensor(rows, dtype=torch.long)].double().numpy(),
                          x.K.double().numpy(), x.V.double().numpy(), w.scale, rows=rows,
                          Sq=w.Sq, block_keep=keep)
    Og, Lg = O.cpu().double().numpy()[:, :, rows], L.cpu().double().numpy()[:, :, rows]
    for h in range(w.Hq):
        sel = agree[h][rows // 64]
        if sel.any():
            compare(torch.from_numpy(Og[:, h:h + 1][:, :, sel]), torch.from_numpy(Lg[:, h:h + 1][:, :, sel]),
                    Or[:, h:h + 1][:, :, sel], Lr[:, h:h + 1][:, :, sel], what=f"image h{h}")
