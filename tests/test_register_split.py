"""The decode kernel's warpgroup register split (setmaxnreg) must fit the registers a
block is launched with, or setmaxnreg.inc would wait forever on the GPU.  Checked on
the CPU from ptxas's report for every instantiation: each must launch with exactly
the 168 registers per thread that the split's arithmetic assumes (384 threads x 168 =
256 consumer threads x 232 + 128 producer threads x 40)."""

import os
import re
import subprocess

import pytest

from sparse_attention_layer_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sparse_attention_layer_b200", "csrc", "decode.cu")


def _split_constants():
    with open(SRC) as f:
        text = f.read()
    get = lambda name: int(re.search(rf"constexpr int {name} = (\d+);", text).group(1))  # noqa: E731
    return (get("kThreads"), get("kConsumerWarps") * 32, get("kLaunchRegs"),
            get("kProducerRegs"), get("kConsumerRegs"))


def test_split_arithmetic():
    threads, consumers, launch, prod, cons = _split_constants()
    assert consumers * cons + (threads - consumers) * prod <= threads * launch
    assert threads % 128 == 0 and consumers % 128 == 0   # whole warpgroups
    for r in (prod, cons):
        assert r % 8 == 0 and 24 <= r <= 256


def test_ptxas_launch_registers_match_the_split(tmp_path):
    try:
        nvcc = build.nvcc_path()
    except RuntimeError:
        pytest.skip("nvcc not available")
    threads, _, launch, _, _ = _split_constants()
    cmd = [nvcc] + build.NVCC_FLAGS + ["-Xptxas", "-v", "-c", SRC, "-o", str(tmp_path / "d.o")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    report = re.findall(r"Compiling entry function '(\w+)'.*?Used (\d+) registers", res.stderr,
                        flags=re.S)
    kernels = [(name, int(regs)) for name, regs in report if "decode_kernel" in name]
    assert len(kernels) == 16  # d 64/128 x group 1/2/4/8 x plain/appending
    for name, regs in kernels:
        assert regs == launch, f"{name} launches with {regs} registers, the split needs {launch}"
