"""Register-spill budgets of the CUDA kernels, read from ptxas's resource
report of the same compile the library uses (no GPU).  A kernel that starts
spilling more than its budget has lost registers somewhere (a role's
setmaxnreg split, an array the compiler no longer keeps in registers), which
costs time long before it costs correctness."""
import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MAIN = os.path.join(ROOT, "mixed_precision_quantized_act_b200", "csrc", "mixllm.cu")

# spill loads in bytes allowed per kernel (mangled-name prefix -> budget); the
# tiled GEMM and the few-token tensor-core kernel are the hot paths
BUDGETS = [
    ("_ZN6mixllm18gemm_w4w8a8_kernelILi128ELi128ELb0ELb0ELb0E", 0),  # 128-token tiles
    ("_ZN6mixllm18gemm_w4w8a8_kernelILi128ELi64ELb0ELb0ELb0E", 0),   # 64-token tiles
    ("_ZN6mixllm18gemm_w4w8a8_kernelILi128ELi128ELb0ELb0ELb1E", 0),  # quantizing X itself
    ("_ZN6mixllm18gemm_w4w8a8_kernelILi128ELi64ELb0ELb0ELb1E", 8),
    ("_ZN6mixllm19gemm_small_m_kernelILi16E", 0),
    ("_ZN6mixllm19gemm_small_m_kernelILi32E", 0),
    ("_ZN6mixllm19gemm_small_m_kernelILi64E", 32),
    ("_ZN6mixllm29gemv_w4w8a8_persistent_kernelILi1E", 0),
    ("_ZN6mixllm29gemv_w4w8a8_persistent_kernelILi2E", 0),
    ("_ZN6mixllm29gemv_w4w8a8_persistent_kernelILi4E", 64),
    ("_ZN6mixllm18gemv_w4w8a8_kernelILi1E", 0),
    ("_ZN6mixllm18gemv_w4w8a8_kernelILi2E", 0),
    ("_ZN6mixllm18gemv_w4w8a8_kernelILi4E", 32),
    ("_ZN6mixllm18gemv_w4w8a8_kernelILi8E", 192),
    ("_ZN6mixllm19quantize_act_kernel", 0),
    ("_ZN6mixllm23channel_salience_kernel", 0),
]


@pytest.fixture(scope="module")
def report():
    nvcc = os.environ.get("NVCC", "nvcc")
    if shutil.which(nvcc) is None:
        pytest.skip("nvcc not available")
    import mixed_precision_quantized_act_b200.build as b
    r = subprocess.run([nvcc, *b.NVCC_FLAGS, "-Xptxas", "-v", "-o", os.devnull, MAIN],
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    spills, cur = {}, None
    for line in r.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            cur = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and cur:
            spills[cur] = int(m.group(2))
            cur = None
    return spills


def test_every_budgeted_kernel_is_compiled(report):
    for prefix, _ in BUDGETS:
        assert any(k.startswith(prefix) for k in report), prefix


# The partials debug forms (their DBG / kDebugP template flag set) are for
# parity tests only: they store every int32 partial and get a looser budget.
DEBUG_FORMS = re.compile(r"gemv_w4w8a8_kernelILi\d+ELb[01]ELb1E|gemv_w4w8a8_persistent_kernelILi\d+ELb1E|"
                         r"gemm_small_m_kernelILi\d+ELb1E|gemm_w4w8a8_kernelILi128ELb1E")
DEBUG_BUDGET = 256


@pytest.mark.parametrize("prefix,budget", BUDGETS, ids=[p for p, _ in BUDGETS])
def test_spill_loads_within_budget(report, prefix, budget):
    for name, loads in report.items():
        if name.startswith(prefix):
            limit = DEBUG_BUDGET if DEBUG_FORMS.search(name) else budget
            assert loads <= limit, f"{name}: {loads} bytes of spill loads, budget {limit}"
