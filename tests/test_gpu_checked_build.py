"""The range-checked build (libgqa_attn_debug.so, compiled with GQA_ATTN_DEBUG).

In it every TMA coordinate and global index a kernel is about to use is checked
first; a violation records ATTN_ERR_DEVICE_BOUNDS and the kernel gives up instead
of touching memory outside its buffers.  This stands in for a memory checker: the
small parity cases of every kernel family (prefill, flex, decode, paged decode,
backward, RBS block scores, the block-sparse kernel, the bit-exact mask
probes) run again in a child process that loads the checked library, and every
one of them must pass with the device status word at ATTN_OK."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

SELECTION = [
    "test_gpu_prefill.py::test_tiny_config_full",
    "test_gpu_prefill.py::test_ragged_tiles",
    "test_gpu_prefill.py::test_edge_cases",
    "test_gpu_prefill.py::test_nan_beyond_k_lengths_ignored",
    "test_gpu_prefill.py::test_non_finite_q_rows_past_q_lengths",
    "test_gpu_mask_probe.py::test_edge_masks_bit_exact",
    "test_gpu_mask_probe.py::test_decode_edge_lengths_bit_exact",
    "test_gpu_decode.py::test_small",
    "test_gpu_decode.py::test_empty_and_poison",
    "test_gpu_flex.py::test_softcap",
    "test_gpu_flex.py::test_alibi",
    "test_gpu_flex.py::test_document_mask",
    "test_gpu_flex.py::test_one_hot_mask_probe",
    "test_gpu_paged.py::test_paged_decode",
    "test_gpu_paged.py::test_paged_ignores_poisoned_slots",
    "test_gpu_bwd.py::test_backward_matches_oracle",
    "test_gpu_bwd.py::test_backward_masked_rows_and_keys_are_zero",
    "test_gpu_rbs.py::test_rbs_scores_and_mask",
    "test_gpu_rbs.py::test_block_sparse_attention",
    "test_gpu_bsparse.py::test_block_sparse_matches_oracle",
    "test_gpu_bsparse.py::test_one_hot_probe_bit_exact",
]


def test_small_cases_pass_in_the_checked_build():
    from gqa_attention_flash_b200 import build
    lib = build.build(debug=True)
    assert os.path.exists(lib)
    env = dict(os.environ, GQA_ATTN_DEBUG="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           *[os.path.join(HERE, t) for t in SELECTION]]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    tail = "\n".join((r.stdout + r.stderr).splitlines()[-30:])
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "failed" not in r.stdout, tail


def test_child_process_loads_the_checked_library():
    env = dict(os.environ, GQA_ATTN_DEBUG="1")
    code = ("from gqa_attention_flash_b200 import binding; "
            "print(binding.CHECKED, binding.LIBRARY)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split()[0] == "True" and r.stdout.strip().endswith("libgqa_attn_debug.so")
