"""The other decode kernels of affine layers: the fused single-kernel layer
(MOE_DECODE_KERNEL=fused) and the four-kernel chain (MOE_DECODE_KERNEL=chain).

The decode parity tests (certified router through the layer, near ties,
largest shapes, odd span counts), the grid-barrier failure path, the layer
tests at one token and the teacher-forced 24-layer stack run again in a child
process with the variable set, so that decode calls and stacks take that
kernel; each of those files also checks, through moe_layer_path, that the
path it ran is the one requested."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("kernel", ["fused", "chain"])
def test_decode_kernel_passes_the_decode_parity_tests(kernel):
    env = dict(os.environ, MOE_DECODE_KERNEL=kernel)
    args = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "tests/test_gpu_decode.py",
            "tests/test_gpu_failure.py", "tests/test_gpu_parity.py::test_layer_tiny_matches_oracle",
            "tests/test_gpu_parity.py::test_layer_q4_full_size_matches_oracle",
            "tests/test_gpu_parity.py::test_layer_q2_full_size_matches_oracle", "tests/test_gpu_stack.py"]
    r = subprocess.run(args, cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
