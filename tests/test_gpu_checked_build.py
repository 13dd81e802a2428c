"""The range-checked build (libgqa_attn_debug.so, compiled with GQA_ATTN_DEBUG).

In it every TMA coordinate and global index a kernel is about to use is checked
first; a violation records ATTN_ERR_DEVICE_BOUNDS and the kernel gives up instead
of touching memory outside its buffers.  This stands in for a memory checker: the
whole GPU suite (every kernel family at small, edge and full sizes, the bit-exact
mask probes, the stream and CUDA-graph tests) runs again in a child process that
loads the checked library, and every test must pass with the device status word
at ATTN_OK (each test reads it after its calls)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_gpu_suite_passes_in_the_checked_build():
    if os.environ.get("GQA_ATTN_DEBUG") == "1":
        pytest.skip("already running in the checked build")
    from gqa_attention_flash_b200 import build
    lib = build.build(debug=True)
    assert os.path.exists(lib)
    env = dict(os.environ, GQA_ATTN_DEBUG="1")
    # node ids are relative to the root directory; this file is left out of the child run
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider", "tests",
           "--deselect", "tests/test_gpu_checked_build.py"]
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
