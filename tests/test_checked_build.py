"""The range-checked build of the library (MIXLLM_CHECKED=1): it builds,
exports the same C ABI as the release build, and says which build it is; the
release build refuses the range-check self-test on the host.  CPU only: no
compute calls (the GPU side is tests/test_gpu_checked.py)."""
import ctypes
import os
import re

from mixed_precision_quantized_act_b200 import _lib
from mixed_precision_quantized_act_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mixllm.h")


def _open(path):
    L = ctypes.CDLL(path)
    for name, (res, args) in _lib.SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    return L


def test_checked_build_exports_the_same_abi_and_says_so():
    rel = _open(libbuild.build())
    chk = _open(libbuild.build(checked=True))
    names = sorted(set(re.findall(r"MIXLLM_API\s+[\w\s\*]*?\b(mixllm_\w+)\s*\(", open(HEADER).read())))
    for n in names:
        assert hasattr(chk, n), n
    assert rel.mixllm_checked_build() == 0
    assert chk.mixllm_checked_build() == 1
    assert rel.mixllm_version() == chk.mixllm_version()


def test_release_build_refuses_the_range_check_selftest_on_the_host():
    rel = _open(libbuild.build())
    assert rel.mixllm_selftest_bounds(None) == _lib.ERR_UNSUPPORTED
    assert b"range checks" in rel.mixllm_last_error()
