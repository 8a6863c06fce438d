"""The debug bounds-checking build (libwan_debug.so, WAN_DEBUG_BOUNDS): every
plain global store of the block's kernels is checked against its buffer's
extent before it is made, and a violation is reported by wan_device_status
as WAN_EBOUNDS. The fp32 and small bf16 parity cases, the attention and
CFG-Euler cases and the head-parallel phases run once under that build, in a
subprocess that loads it through WAN_LIBRARY; every one must pass with no
violation recorded (each parity test checks wan_device_status), on top of the
canary bytes around the outputs."""
import os
import subprocess
import sys

import pytest
import torch

from video_diffusion_transformer_fwd_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [
    "tests/test_gpu_parity.py::test_block_tiny_f32_full",
    "tests/test_gpu_parity.py::test_block_tiny_f32_ctx_lens_and_sharp",
    "tests/test_gpu_parity.py::test_block_f32_ragged_grid_head64",
    "tests/test_gpu_parity.py::test_block_bf16_small_ragged",
    "tests/test_gpu_parity.py::test_block_bf16_small_sharp",
    "tests/test_gpu_parity.py::test_attention_bf16",
    "tests/test_gpu_parity.py::test_attention_f32",
    "tests/test_gpu_parity.py::test_euler_cfg",
    "tests/test_gpu_ulysses.py::test_permute_chunks_matches_host",
    "tests/test_gpu_ulysses.py::test_sharded_step_equals_one_shard",
]


@pytest.mark.gpu
def test_parity_cases_under_the_debug_bounds_build():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = build_lib.build(debug=True, verbose=False)
    env = dict(os.environ, WAN_LIBRARY=lib)
    probe = subprocess.run(
        [sys.executable, "-c", "from video_diffusion_transformer_fwd_b200 import wan; print(wan.wan_debug_bounds())"],
        env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert probe.stdout.strip() == "1", probe.stdout + probe.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider", *CASES],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout
