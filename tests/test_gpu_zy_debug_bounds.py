"""The bounds-checking debug build (compiled with -DVG_DEBUG_BOUNDS: every
checked index into memory records VG_ERR_DEVICE_BOUNDS with its site instead of
being used) runs a selection of the GPU parity tests: a stand-in for a memory
checker, which these GPUs do not offer. The selection covers the decode and
prefill MoE paths (entry kernel, grouping kernels, both expert kernels), the
fused verify, the single-launch step and the attention layer; each test checks
the device status word, so a failed bounds check fails it."""
import os
import subprocess
import sys

import pytest

from greedy_speculative_verify_b200 import build as vbuild

pytestmark = pytest.mark.gpu

SELECTION = [
    "tests/test_gpu_moe.py::test_layer_parity",
    "tests/test_gpu_moe.py::test_decode_skewed_routing",
    "tests/test_gpu_moe.py::test_layer_skewed_routing",
    "tests/test_gpu_verify.py::test_verify_parity",
    "tests/test_gpu_step_small.py::test_small_step_router_bias_and_small_vocabulary",
    "tests/test_gpu_attention.py::test_attention_matches_oracle",
]


def test_debug_bounds_build_passes_parity(root_dir):
    lib = vbuild.build(extra_flags=["-DVG_DEBUG_BOUNDS"], out=vbuild.DEBUG_LIB)
    env = dict(os.environ, VG_TEST_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider", *SELECTION],
                       cwd=root_dir, env=env, capture_output=True, text=True, timeout=1500)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
