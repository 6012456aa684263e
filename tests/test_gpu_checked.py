"""The range-checked build on the GPU: its self-test makes the checks fire
(without any access) and the context stays usable; then the parity tests of
every GEMM kernel run on the checked build in a child process and must pass
with a clean status word (no range check failed).  GPU only."""
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

from mixed_precision_quantized_act_b200 import _lib  # noqa: E402
from mixed_precision_quantized_act_b200 import build as libbuild  # noqa: E402

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def checked_lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return libbuild.build(checked=True)


def test_checked_build_selftest_reports_bounds(checked_lib):
    code = (
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "from mixed_precision_quantized_act_b200 import _lib\n"
        "assert _lib.checked_build()\n"
        "_lib.sync_status()\n"
        "_lib.selftest_bounds()\n"
        "try:\n"
        "    _lib.sync_status()\n"
        "    raise SystemExit('no bounds status')\n"
        "except _lib.MixLLMError as e:\n"
        "    assert e.status == _lib.ERR_BOUNDS, e\n"
        "_lib.sync_status()  # cleared, and the context still works\n"
        "x = torch.ones(1024, device='cuda') * 2\n"
        "assert float(x.sum()) == 2048.0\n"
        "print('ok')\n")
    env = dict(os.environ, MIXLLM_LIBRARY=checked_lib)
    p = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0 and "ok" in p.stdout, p.stderr[-3000:]


def test_parity_suite_passes_on_the_checked_build(checked_lib):
    # the tiled kernel (both sets, ragged shapes, the partials debug path at
    # full q_proj size, bounds and overflow cases) and every few-token kernel
    sel = ("partials_bit_exact or y_matches_oracle or full_size_partials or reach_the_bounds "
           "or overflow or small_m_kernel_partials or test_small_m_matches_oracle")
    env = dict(os.environ, MIXLLM_LIBRARY=checked_lib)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-k", sel, "-p", "no:cacheprovider",
           os.path.join(ROOT, "tests", "test_gpu_parity.py"), os.path.join(ROOT, "tests", "test_gpu_small_m.py")]
    p = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=1800, cwd=ROOT)
    assert p.returncode == 0, p.stdout[-3000:] + p.stderr[-2000:]
    assert " passed" in p.stdout
