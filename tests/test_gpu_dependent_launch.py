"""Programmatic dependent launch: the forward, decode and block-sparse kernels may
start while the previous kernel on the stream still runs, and must read nothing
that kernel writes before it has finished.  Each chain below is launched with no
host synchronisation between its calls, where every call reads what the one
before it wrote, and must give bitwise the same results as the same calls with a
synchronisation after each."""
import pytest
import torch

from gqa_attention_flash_b200 import binding

pytestmark = pytest.mark.gpu


def _rand(shape, g):
    return torch.randn(shape, generator=g).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("B,Hq,Hkv,S,D", [(1, 2, 1, 128, 64), (2, 8, 2, 1000, 128)])
def test_forward_chain_reads_previous_output(B, Hq, Hkv, S, D):
    g = torch.Generator().manual_seed(11)
    Q, K, V = _rand((B, Hq, S, D), g), _rand((B, Hkv, S, D), g), _rand((B, Hkv, S, D), g)
    scale = D ** -0.5

    def chain(sync):
        outs, x = [], Q
        for _ in range(6):
            O = torch.empty_like(Q)
            L = torch.empty((B, Hq, S), dtype=torch.float32, device=Q.device)
            binding.attn_fwd(O, x, K, V, L, scale, True)
            if sync:
                torch.cuda.synchronize()
            outs.append((O, L))
            x = O  # the next launch's queries are this launch's output
        torch.cuda.synchronize()
        return outs

    want = chain(True)
    got = chain(False)
    assert binding.last_device_status() == 0
    for i, ((Og, Lg), (Ow, Lw)) in enumerate(zip(got, want)):
        assert torch.equal(Og, Ow), f"O of launch {i}"
        assert torch.equal(Lg, Lw), f"LSE of launch {i}"


def test_decode_after_in_place_cache_update():
    g = torch.Generator().manual_seed(12)
    B, Hq, Hkv, S_cap, D = 4, 32, 8, 2048, 128
    Q = _rand((B, Hq, D), g)
    K0, V0 = _rand((B, Hkv, S_cap, D), g), _rand((B, Hkv, S_cap, D), g)
    lengths = torch.tensor([1, 700, 2048, 1500], dtype=torch.int32).cuda()

    def chain(sync):
        K, V = K0.clone(), V0.clone()
        torch.cuda.synchronize()
        outs = []
        for step in range(5):
            K.mul_(-1.0)  # a kernel writes the cache right before the decode reads it
            V[:, :, step::7].mul_(2.0)
            if sync:
                torch.cuda.synchronize()
            O = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=Q.device)
            binding.attn_decode(O, Q, K, V, lengths, 8)
            if sync:
                torch.cuda.synchronize()
            outs.append(O)
        torch.cuda.synchronize()
        return outs

    want = chain(True)
    got = chain(False)
    assert binding.last_device_status() == 0
    for i, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a, b), f"decode step {i}"


def test_block_scores_then_sparse_attention():
    g = torch.Generator().manual_seed(13)
    B, H, S, D = 1, 4, 1024, 128
    Q, K, V = _rand((B, H, S, D), g), _rand((B, H, S, D), g), _rand((B, H, S, D), g)

    def chain(sync):
        outs = []
        for _ in range(4):
            m = binding.rbs_block_mask(Q, K)
            if sync:
                torch.cuda.synchronize()
            O = torch.empty_like(Q)
            L = torch.empty((B, H, S), dtype=torch.float32, device=Q.device)
            binding.attn_fwd_flex(O, Q, K, V, L, D ** -0.5, False, block_mask=m)
            if sync:
                torch.cuda.synchronize()
            outs.append((m, O, L))
        torch.cuda.synchronize()
        return outs

    want = chain(True)
    got = chain(False)
    assert binding.last_device_status() == 0
    for i, (a, b) in enumerate(zip(got, want)):
        assert torch.equal(a[0], b[0]), f"mask {i}"
        assert torch.equal(a[1], b[1]), f"O {i}"
        assert torch.equal(a[2], b[2]), f"LSE {i}"
