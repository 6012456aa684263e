"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching a device (CPU only, no compute calls).
"""
import ctypes
import os
import re

import pytest

from mixed_precision_quantized_act_b200 import _lib
from mixed_precision_quantized_act_b200 import build as libbuild
from mixed_precision_quantized_act_b200 import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mixllm.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.load()


def declared_entry_points():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"MIXLLM_API\s+[\w\s\*]*?\b(mixllm_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_entry_points()
    for required in ("mixllm_quantize_act", "mixllm_pack_weights", "mixllm_gemm_w4w8a8",
                     "mixllm_gemm_debug_partials", "mixllm_packed_sizes", "mixllm_last_error",
                     "mixllm_sync_status"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    names = declared_entry_points()
    assert names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_library_has_no_runtime_dependency_on_a_gpu_driver():
    # static CUDA runtime; the driver is looked up lazily
    import subprocess
    out = subprocess.run(["ldd", _lib.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_packed_sizes_footprint(L):
    N, K, N8 = 4096, 4096, 410
    s = _lib.packed_sizes(N, K, N8)
    N4, G = N - N8, K // 128
    N4p, N8p = 3840, 512
    T4 = (N4 + 127) // 128  # W4 is stored as whole 128-channel tiles (rows past N4 are zero)
    assert s == [T4 * 128 * K // 2, G * N4p // 2, G * N4p * 2, N4 * 4, N8 * K, G * N8p * 2, N8 * 4]
    # without padding the per-weight footprints are the pages' 0.5 + 2.5/G and 1 + 2/G
    s2 = _lib.packed_sizes(512, 1024, 256)
    assert (s2[0] + s2[1] + s2[2]) / (256 * 1024) == 0.5 + 2.5 / 128
    assert (s2[4] + s2[5]) / (256 * 1024) == 1 + 2 / 128


@pytest.mark.parametrize("layer", [wl.TINY, wl.Q_PROJ_P10, wl.LLAMA70B[2]])
def test_packed_sizes_cover_the_binding_layout(L, layer):
    s = _lib.packed_sizes(layer.N, layer.K, layer.N8)
    N4p, N8p = _lib.padded(layer.N4), _lib.padded(layer.N8)
    assert s[1] == layer.G * N4p // 2 and s[5] == layer.G * N8p * 2


def _status(L, fn, *args):
    return getattr(L, fn)(*args)


def test_host_validation_rejects_before_any_device_call(L):
    null = None
    # unsupported group size / K
    assert L.mixllm_quantize_act(null, 4, 256, 64, null, null, null) == _lib.ERR_UNSUPPORTED
    assert L.mixllm_quantize_act(null, 4, 200, 128, null, null, null) == _lib.ERR_UNSUPPORTED
    assert b"group" in L.mixllm_last_error() or b"K" in L.mixllm_last_error()
    # null pointers
    assert L.mixllm_quantize_act(null, 4, 256, 128, null, null, null) == _lib.ERR_INVALID_ARG
    # misaligned pointer (never dereferenced: rejected on the host)
    assert L.mixllm_quantize_act(ctypes.c_void_p(0x1001), 4, 256, 128, ctypes.c_void_p(0x2000),
                                 ctypes.c_void_p(0x3000), null) == _lib.ERR_INVALID_ARG
    # M = 0 is a no-op that succeeds without a device
    assert L.mixllm_quantize_act(null, 0, 256, 128, null, null, null) == _lib.OK
    # GEMM: bad K, negative sizes, null outputs, misaligned A
    args = [null, null, 4, 256, null, null, null, null, 8, null, null, null, 0, null, null]
    a = list(args); a[3] = 100; a[13] = ctypes.c_void_p(0x3000)
    assert L.mixllm_gemm_w4w8a8(*a) == _lib.ERR_UNSUPPORTED
    a = list(args); a[8] = -1
    assert L.mixllm_gemm_w4w8a8(*a) == _lib.ERR_INVALID_ARG
    assert L.mixllm_gemm_w4w8a8(*args) == _lib.ERR_INVALID_ARG  # null Y
    a = list(args)
    a[0], a[1], a[13] = ctypes.c_void_p(0x1008), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000)
    assert L.mixllm_gemm_w4w8a8(*a) == _lib.ERR_INVALID_ARG
    assert b"16-byte" in L.mixllm_last_error()
    # empty problems succeed without a device
    a = list(args); a[2] = 0
    assert L.mixllm_gemm_w4w8a8(*a) == _lib.OK
    # pack: N8 > N
    assert L.mixllm_pack_weights(null, 4, 256, null, 5, 128, *([null] * 8)) == _lib.ERR_INVALID_ARG
    # self-test limit range
    assert L.mixllm_selftest_wait_timeout(0, null) == _lib.ERR_INVALID_ARG
    # packed sizes argument checks
    out = (ctypes.c_size_t * 7)()
    assert L.mixllm_packed_sizes(10, 256, 11, 128, out) == _lib.ERR_INVALID_ARG
    assert L.mixllm_packed_sizes(10, 256, 1, 32, out) == _lib.ERR_UNSUPPORTED


def test_binding_raises_without_cuda_tensors(L):
    import torch
    with pytest.raises(ValueError):
        _lib.quantize_act_into(torch.zeros(2, 128, dtype=torch.float16), torch.zeros(2, 128, dtype=torch.int8),
                               torch.zeros(2, 1), None)


def test_small_m_kernel_choice(L):
    """mixllm_small_m_kernel: tensor cores from M = 9, the GEMV below; the
    persistent GEMV only for M <= 4, M*K <= 32 KiB and >= 8 x 296 units."""
    def kind(M, K, N4, N8):
        out = ctypes.c_int32(-1)
        st = L.mixllm_small_m_kernel(M, K, N4, N8, ctypes.byref(out))
        return st, out.value

    assert kind(9, 4096, 3686, 410) == (_lib.OK, 0)
    assert kind(64, 4096, 3686, 410) == (_lib.OK, 0)
    assert kind(1, 4096, 3686, 410) == (_lib.OK, 1)       # q_proj: 296 units
    assert kind(8, 4096, 27238, 1434) == (_lib.OK, 1)     # 8B gate_up: 1896 units
    assert kind(1, 8192, 51610, 5734) == (_lib.OK, 2)     # 70B gate_up: 7904 units
    assert kind(4, 8192, 51610, 5734) == (_lib.OK, 2)
    assert kind(5, 8192, 51610, 5734) == (_lib.OK, 1)     # token bound 8
    assert kind(1, 28672, 7373, 819) == (_lib.OK, 2)      # 70B down: 4032 units, 1 x 28672 bytes of codes
    assert kind(2, 28672, 7373, 819) == (_lib.OK, 1)      # 2 x 28672 > 32 KiB
    assert kind(0, 4096, 100, 10)[0] == _lib.ERR_INVALID_ARG
    assert kind(65, 4096, 100, 10)[0] == _lib.ERR_INVALID_ARG
    assert kind(8, 100, 100, 10)[0] == _lib.ERR_UNSUPPORTED
    assert L.mixllm_small_m_kernel(1, 4096, 100, 10, None) == _lib.ERR_INVALID_ARG
    assert _lib.small_m_kernel(1, 8192, 51610, 5734) == "GEMV persistent"


def test_small_m_workspace_plan(L):
    """Workspace of the few-token path.  Tensor-core kernel (M > 8) and the
    split GEMV: S splits x tiles x (token tile x 128) fp32 partials + one int32
    counter per 128-channel tile, none without a split, at most 32 groups per
    CTA; the tensor-core kernel's S fills one wave of 148 CTAs (token tiles
    16 / 32 / 64), the split GEMV's S4 = 296 // (nt4 + 2 nt8) per 4-bit tile
    and twice that per 8-bit tile.  Persistent GEMV (M <= 4, bound*K <= 32 KiB
    and U >= 8 * 296 units, U = nt4*ceil(G/4) + nt8*ceil(G/2)): P = 296 CTAs,
    [P][2][bound][128] fp32 partials + one counter per tile."""
    def ws(M, K, N4, N8):
        out = ctypes.c_size_t(0)
        st = L.mixllm_small_m_workspace_bytes(M, K, N4, N8, ctypes.byref(out))
        return st, out.value

    # q_proj p10, 29 + 4 tiles (U = 296, too few units for the persistent GEMV):
    # split, S4 = 296 // 37 = 8, S8 = 16
    for M, bound in ((1, 1), (2, 2), (3, 4), (8, 8)):
        assert ws(M, 4096, 3686, 410) == (_lib.OK, 16 * 33 * bound * 128 * 4 + 33 * 4)
    # tensor-core kernel: M=9 -> S = 148 // 33 = 4, token tile 16
    assert ws(9, 4096, 3686, 410) == (_lib.OK, 4 * 33 * 16 * 128 * 4 + 33 * 4)
    # split, 213 + 12 tiles: S4 = 296 // 237 = 1, S8 = 2
    assert ws(1, 4096, 27238, 1434) == (_lib.OK, 2 * 225 * 1 * 128 * 4 + 225 * 4)
    # persistent, 70B gate_up (404 + 45 tiles, G = 64): U = 404*16 + 45*32 = 7904
    assert ws(1, 8192, 51610, 5734) == (_lib.OK, 296 * 2 * 1 * 128 * 4 + 449 * 4)
    assert ws(4, 8192, 51610, 5734) == (_lib.OK, 296 * 2 * 4 * 128 * 4 + 449 * 4)
    # ... but not at M = 5 (token bound 8): split, S4 = max(296 // 494, 1) = 1, S8 = 2
    assert ws(5, 8192, 51610, 5734) == (_lib.OK, 2 * 449 * 8 * 128 * 4 + 449 * 4)
    # split GEMV (8 x 28672 > 32 KiB), 58 + 7 tiles: S4 = max(296 // 72, 224 / 32) = 7, S8 = 8
    assert ws(8, 28672, 7373, 819) == (_lib.OK, 8 * 65 * 8 * 128 * 4 + 65 * 4)
    # split, one 4-bit tile only: S4 = 296 (capped at G = 32); one 8-bit tile only: S8 = 592 -> 32
    assert ws(1, 4096, 100, 0) == (_lib.OK, 32 * 1 * 1 * 128 * 4 + 1 * 4)
    assert ws(1, 4096, 0, 100) == (_lib.OK, 32 * 1 * 1 * 128 * 4 + 1 * 4)
    # token tiles 32 and 64
    assert ws(17, 4096, 3686, 410) == (_lib.OK, 4 * 33 * 32 * 128 * 4 + 33 * 4)
    assert ws(64, 4096, 3686, 410) == (_lib.OK, 4 * 33 * 64 * 128 * 4 + 33 * 4)
    # 225 tiles: more than one wave, no split, no workspace
    assert ws(16, 4096, 27238, 1434) == (_lib.OK, 0)
    # K = 28672 (224 groups), 58 + 7 tiles: S = max(148 // 65, 224 / 32) = 7
    assert ws(16, 28672, 7373, 819) == (_lib.OK, 7 * 65 * 16 * 128 * 4 + 65 * 4)
    # one group: nothing to split
    assert ws(3, 128, 300, 84) == (_lib.OK, 0)
    assert ws(9, 128, 300, 84) == (_lib.OK, 0)
    assert ws(65, 4096, 100, 10)[0] == _lib.ERR_INVALID_ARG
    assert ws(0, 4096, 100, 10)[0] == _lib.ERR_INVALID_ARG
    assert ws(8, 100, 100, 10)[0] == _lib.ERR_UNSUPPORTED
    null = L.mixllm_small_m_workspace_bytes(8, 4096, 100, 10, None)
    assert null == _lib.ERR_INVALID_ARG


def test_header_is_plain_c_and_links_from_c(tmp_path):
    """The boundary is a C ABI: a strict C99 program includes the header,
    links against the library and calls its host-only entry points."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "mixllm.h"
int main(void) {
  size_t sizes[7];
  if (mixllm_version() <= 0) return 1;
  if (mixllm_packed_sizes(4096, 4096, 410, 128, sizes) != MIXLLM_OK) return 2;
  if (mixllm_packed_sizes(4096, 4096, 410, 64, sizes) != MIXLLM_ERR_UNSUPPORTED) return 3;
  if (mixllm_last_error()[0] == '\0') return 4;
  printf("%zu\n", sizes[0]);
  return 0;
}
''')
    exe = tmp_path / "use_abi"
    libdir = os.path.dirname(_lib.LIB_PATH)
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, str(src), "-o", str(exe),
                        _lib.LIB_PATH, "-Wl,-rpath," + libdir], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert int(r.stdout) == _lib.packed_sizes(4096, 4096, 410)[0]


def test_linear_workspace_plan_and_host_checks(L):
    """Workspace of mixllm_linear / mixllm_linear_one_launch: for M > 64, A_q
    [M, K] int8, s_a [M, K/128] fp32 and two uint32 counters, each part
    rounded up to 256 bytes; for M <= 64 the few-token layer's own workspace.
    The host rejects the one-launch form for 1 <= M <= 64 and null buffers
    before touching a device; empty problems succeed without one."""
    def ws(fn, M, K, N4, N8):
        out = ctypes.c_size_t(0)
        st = getattr(L, fn)(M, K, N4, N8, ctypes.byref(out))
        return st, out.value

    r256 = lambda b: (b + 255) // 256 * 256  # noqa: E731
    for M in (65, 200, 512, 1024):
        for K in (384, 512, 4096, 14336):
            assert ws("mixllm_linear_workspace_bytes", M, K, 3686, 410) == (
                _lib.OK, r256(M * K) + r256(M * (K // 128) * 4) + 256)
    for M in (1, 2, 9, 64):
        assert ws("mixllm_linear_workspace_bytes", M, 4096, 3686, 410) == \
            ws("mixllm_linear_small_m_workspace_bytes", M, 4096, 3686, 410)
    assert ws("mixllm_linear_workspace_bytes", 0, 4096, 3686, 410) == (_lib.OK, 0)
    assert ws("mixllm_linear_workspace_bytes", 512, 100, 3686, 410)[0] == _lib.ERR_UNSUPPORTED
    assert ws("mixllm_linear_workspace_bytes", -1, 4096, 3686, 410)[0] == _lib.ERR_INVALID_ARG

    null = None
    # (X, M, K, W4, z4, s_w4, idx4, N4, W8, s_w8, idx8, N8, Y, workspace, bytes, stream)
    args = [null, 16, 4096, null, null, null, null, 100, null, null, null, 10, null, null, 0, null]
    assert L.mixllm_linear_one_launch(*args) == _lib.ERR_INVALID_ARG
    assert b"M > 64" in L.mixllm_last_error()
    a = list(args); a[1] = 512
    assert L.mixllm_linear(*a) == _lib.ERR_INVALID_ARG           # null X and Y
    assert L.mixllm_linear_one_launch(*a) == _lib.ERR_INVALID_ARG
    a = list(args); a[1] = 512; a[0] = ctypes.c_void_p(0x1008); a[12] = ctypes.c_void_p(0x3000)
    assert L.mixllm_linear(*a) == _lib.ERR_INVALID_ARG           # X not 16-byte aligned
    assert b"16-byte" in L.mixllm_last_error()
    a = list(args); a[1] = 0
    assert L.mixllm_linear(*a) == _lib.OK                        # empty: no device needed
    assert L.mixllm_linear_one_launch(*a) == _lib.OK
