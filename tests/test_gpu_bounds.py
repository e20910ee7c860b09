"""The ragged-shape parity tests again, against the bounds-checked build
(libq4_debug.so, -DQ4_DEBUG).

In that build every kernel checks the index range of each global load and
store before it is made; a failed check skips the access and sets a bit that
q4_bounds_flags() returns.  The tests run in a child process with
Q4_LIBRARY=debug, where conftest asserts after each GPU test that no check
failed, and every output is still compared with the oracle as usual.  This
covers the out-of-range reads and writes a memory checker would report,
without running one.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# every kernel family on ragged and edge shapes: M = 1 rings, M = 2..24,
# tensor cores (chunked, and every kind of persistent plan), two-bit, pack /
# dequant / embed, the allocation-free entry point and a recorded step
SELECTION = [
    "tests/test_gpu_parity.py::test_ragged_shapes",
    "tests/test_gpu_parity.py::test_gemv2_ragged",
    "tests/test_gpu_parity.py::test_gemv_rows_of_2kb",
    "tests/test_gpu_parity.py::test_pack_dequant_bit_exact",
    "tests/test_gpu_parity.py::test_pack2_dequant2_bit_exact",
    "tests/test_gpu_parity.py::test_embed_rows_bit_exact",
    "tests/test_gpu_parity.py::test_zero_scales_give_zero",
    "tests/test_gpu_parity.py::test_output_bounds_and_stream",
    "tests/test_gpu_parity.py::test_gemv2_output_bounds_and_stream",
    "tests/test_gpu_parity.py::test_integer_codebook_exact",
    "tests/test_gpu_parity.py::test_tensor_core_path_chunks_large_inputs",
    "tests/test_gpu_parity.py::test_tensor_core_plans",
    "tests/test_gpu_step.py::test_step_replays_every_path",
    "tests/test_zz_no_alloc.py",
]


def test_ragged_parity_on_the_bounds_checked_build():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, Q4_LIBRARY="debug")
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-p", "no:cacheprovider", *SELECTION]
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = "\n".join((res.stdout + res.stderr).splitlines()[-30:])
    assert res.returncode == 0, tail
    last = tail.splitlines()[-1] if tail else ""
    assert " passed" in last and "skipped" not in last, tail
