"""The checked build (libflux_checked.so: the same kernels with their bounds guards
compiled in, include/flux.h).  Its guard mechanism reports FLUX_DEVICE_BOUNDS without
touching memory outside the guarded buffer, and a set of parity cases -- decode at
every group size and head dim, ragged and ring caches, fused appends, KV appends,
prefill tails -- runs through it with no guard firing (each case asserts a clean status
word)."""

import os
import subprocess
import sys

import pytest

from sparse_attention_layer_b200 import build, flux

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PARITY_SUBSET = ("decode_tiny_config or decode_groups_and_head_dims or decode_ragged_edges or "
                 "decode_append_equals or ring_decode_identical or ring_compact or "
                 "kv_append_exact or prefill_ragged_tail")


@pytest.mark.gpu
def test_bounds_selftest():
    import torch
    torch.cuda.set_device(0)
    flux.flux_get_device_status()  # start from a clear word
    flux.flux_selftest_bounds()
    bits = flux.flux_get_device_status()
    if flux.flux_build_checked():
        assert bits == flux.FLUX_DEVICE_BOUNDS
    else:
        assert bits == 0  # the plain build compiles the guard away


@pytest.mark.gpu
def test_checked_build_runs_parity_cases_clean():
    if os.environ.get("FLUX_CHECKED") == "1":
        pytest.skip("this process already runs the checked build")
    build.build(checked=True)
    env = dict(os.environ, FLUX_CHECKED="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
           os.path.join("tests", "test_gpu_checked.py") + "::test_bounds_selftest",
           os.path.join("tests", "test_gpu_parity.py"), "-k", PARITY_SUBSET]
    r = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and "failed" not in r.stdout
