"""Device-side status reporting: bounded waits give up with ATTN_ERR_TIMEOUT
(without hanging or faulting the GPU), and out-of-range lengths are clamped and
flagged ATTN_ERR_DEVICE_BOUNDS."""
import pytest
import torch

from gpu_common import gpu_prefill
from gqa_attention_flash_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out():
    from gqa_attention_flash_b200 import binding
    assert binding.last_device_status() == 0
    binding.check_bounded_wait(2000)   # 2 ms limit on a barrier nobody completes
    st = binding.last_device_status()
    assert st == 5, binding.status_string(st)
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
    assert binding.last_device_status() == 0


def test_length_past_tensor_is_flagged(orc):
    from gqa_attention_flash_b200 import binding
    Q, K, V = W.random_prefill(2, 1, 2, 1, 64, 64, 64)
    dev = torch.device("cuda")
    O = torch.empty_like(Q, device=dev)
    kl = torch.tensor([1000], dtype=torch.int32, device=dev)
    binding.attn_fwd(O, Q.to(dev), K.to(dev), V.to(dev), None, 0.125, False, 0, 0, kl)
    assert binding.last_device_status() == 6
    # clamped to Sk: same result as without lengths
    O2, _ = gpu_prefill(Q, K, V, 0.125, False)
    assert torch.equal(O.cpu(), O2)
