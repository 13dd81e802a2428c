"""The Python binding refuses tensors the C ABI cannot check (it sees only
pointers and sizes): a wrong dtype, a shape that does not fit the others, a
non-contiguous view, and tensors that are not on the current CUDA device.
Every refusal happens before any call into the library, so these run on CPU."""
import pytest
import torch


@pytest.fixture(scope="module")
def binding():
    from gqa_attention_flash_b200 import build
    build.build()
    from gqa_attention_flash_b200 import binding as b
    return b


def prefill(B=2, Hq=4, Hkv=2, Sq=8, Sk=12, D=64):
    bf = torch.bfloat16
    return dict(O=torch.zeros(B, Hq, Sq, D, dtype=bf), Q=torch.zeros(B, Hq, Sq, D, dtype=bf),
                K=torch.zeros(B, Hkv, Sk, D, dtype=bf), V=torch.zeros(B, Hkv, Sk, D, dtype=bf),
                LSE=torch.zeros(B, Hq, Sq, dtype=torch.float32))


def call_fwd(binding, t, **kw):
    binding.attn_fwd(t["O"], t["Q"], t["K"], t["V"], t["LSE"], 0.1, True, **kw)


def test_fwd_wrong_dtypes(binding):
    for name, dt in [("Q", torch.float16), ("K", torch.float32), ("V", torch.float16),
                     ("O", torch.float32), ("LSE", torch.bfloat16)]:
        t = prefill()
        t[name] = t[name].to(dt)
        with pytest.raises(TypeError, match=name):
            call_fwd(binding, t)
    t = prefill()
    with pytest.raises(TypeError, match="k_lengths"):
        call_fwd(binding, t, k_lengths=torch.zeros(2, dtype=torch.int64))
    with pytest.raises(TypeError, match="q_lengths"):
        call_fwd(binding, t, q_lengths=torch.zeros(2, dtype=torch.float32))


def test_fwd_shape_mismatches(binding):
    cases = {
        "K": torch.zeros(2, 3, 12, 64, dtype=torch.bfloat16),      # Hkv differs from V
        "V": torch.zeros(2, 2, 11, 64, dtype=torch.bfloat16),      # Sk differs from K
        "O": torch.zeros(2, 4, 8, 128, dtype=torch.bfloat16),      # D differs from Q
        "LSE": torch.zeros(2, 4, 9, dtype=torch.float32),          # Sq differs from Q
    }
    for name, bad in cases.items():
        t = prefill()
        t[name] = bad
        with pytest.raises(ValueError, match=r"(K|V|O|LSE) has shape"):
            call_fwd(binding, t)
    t = prefill()
    t["K"] = torch.zeros(3, 2, 12, 64, dtype=torch.bfloat16)       # batch differs from Q
    with pytest.raises(ValueError, match="K has shape"):
        call_fwd(binding, t)
    with pytest.raises(ValueError, match="k_lengths has shape"):
        call_fwd(binding, prefill(), k_lengths=torch.zeros(3, dtype=torch.int32))


def test_fwd_non_contiguous(binding):
    t = prefill(Sq=12, Sk=12)
    t["Q"] = torch.zeros(2, 4, 64, 12, dtype=torch.bfloat16).transpose(2, 3)
    with pytest.raises(ValueError, match="Q must be contiguous"):
        call_fwd(binding, t)
    t = prefill()
    t["V"] = torch.zeros(2, 12, 2, 64, dtype=torch.bfloat16).transpose(1, 2)
    with pytest.raises(ValueError, match="V must be contiguous"):
        call_fwd(binding, t)


def test_fwd_not_on_a_cuda_device(binding):
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        call_fwd(binding, prefill())


def test_flex_and_backward_checks(binding):
    t = prefill()
    with pytest.raises(ValueError, match="alibi_slopes has shape"):
        binding.attn_fwd_flex(t["O"], t["Q"], t["K"], t["V"], t["LSE"], 0.1, True,
                              alibi_slopes=torch.zeros(3, dtype=torch.float32))
    with pytest.raises(ValueError, match="doc_kv has shape"):
        binding.attn_fwd_flex(t["O"], t["Q"], t["K"], t["V"], t["LSE"], 0.1, True,
                              doc_q=torch.zeros(8, dtype=torch.int32),
                              doc_kv=torch.zeros(8, dtype=torch.int32))
    with pytest.raises(ValueError, match="block_mask has shape"):
        binding.attn_fwd_flex(t["O"], t["Q"], t["K"], t["V"], t["LSE"], 0.1, True,
                              block_mask=torch.zeros(2, 2, dtype=torch.uint8))
    g = {k: torch.zeros_like(v) for k, v in t.items()}
    with pytest.raises(ValueError, match="dK has shape"):
        binding.attn_bwd(g["Q"], g["Q"], g["V"], g["O"], t["Q"], t["K"], t["V"], t["O"],
                         t["LSE"], 0.1, True)
    with pytest.raises(TypeError, match="dO must be"):
        binding.attn_bwd(g["Q"], g["K"], g["V"], g["O"].float(), t["Q"], t["K"], t["V"], t["O"],
                         t["LSE"], 0.1, True)
    with pytest.raises(ValueError, match="LSE"):
        binding.attn_bwd(g["Q"], g["K"], g["V"], g["O"], t["Q"], t["K"], t["V"], t["O"],
                         None, 0.1, True)


def test_decode_checks(binding):
    bf = torch.bfloat16
    Q = torch.zeros(3, 8, 128, dtype=bf)
    K = torch.zeros(3, 2, 100, 128, dtype=bf)
    O = torch.zeros_like(Q)
    lengths = torch.zeros(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="V has shape"):
        binding.attn_decode(O, Q, K, torch.zeros(3, 2, 99, 128, dtype=bf), lengths)
    with pytest.raises(TypeError, match="lengths must be"):
        binding.attn_decode(O, Q, K, K.clone(), lengths.long())
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        binding.attn_decode(O, Q, K, K.clone(), lengths)
    with pytest.raises(ValueError, match="O has shape"):
        binding.attn_decode_noalloc(torch.zeros(3, 8, 64, dtype=bf), Q, K, K.clone(), lengths)
    pool = torch.zeros(10, 16, 2, 128, dtype=bf)
    tables = torch.zeros(3, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="V_cache has shape"):
        binding.attn_decode_paged(O, Q, pool, torch.zeros(10, 8, 2, 128, dtype=bf), tables,
                                  lengths)
    with pytest.raises(TypeError, match="block_tables must be"):
        binding.attn_decode_paged(O, Q, pool, pool.clone(), tables.long(), lengths)
