"""CPU oracle for the MixLLM W4.4A8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It wraps ``mixllm_oracle.c`` (plain C,
compiled with gcc, no FMA contraction) with numpy-facing functions.  It shares
no code with the CUDA library and never imports it.

Functions take and return numpy arrays; fp16 values travel as ``np.float16``
arrays (their bit patterns are what the C code sees).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mixllm_oracle.c")
_LIB = os.path.join(_HERE, "libmixllm_oracle.so")
GROUP = 128

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmixllm_oracle.so`` (gcc, -O2,
    -ffp-contract=off so that no multiply-add is fused)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-Wall", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def configure(L):
    """Declare the C signatures on a loaded oracle library and return it."""
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    L.oracle_f16_to_f32.restype = ctypes.c_float
    L.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.oracle_f32_to_f16.restype = ctypes.c_uint16
    L.oracle_f32_to_f16.argtypes = [ctypes.c_float]
    L.oracle_f32_to_f16_array.argtypes = [vp, i64, vp]
    L.oracle_f16_to_f32_array.argtypes = [vp, i64, vp]
    L.oracle_i2f_bias.restype = ctypes.c_float
    L.oracle_i2f_bias.argtypes = [ctypes.c_int32]
    L.oracle_i2f_mismatches.restype = i64
    L.oracle_i2f_mismatches.argtypes = [i64, i64]
    L.oracle_quantize_act.argtypes = [vp, i64, i64, vp, vp]
    L.oracle_quantize_w4.argtypes = [vp, i64, i64, vp, vp, vp]
    L.oracle_quantize_w8.argtypes = [vp, i64, i64, vp, vp]
    L.oracle_split_channels.restype = i64
    L.oracle_split_channels.argtypes = [vp, i64, vp, vp]
    L.oracle_gemm_w4w8a8.argtypes = [vp, vp, i64, i64, vp, vp, vp, vp, i64,
                                     vp, vp, vp, i64, vp]
    L.oracle_group_partials.argtypes = [vp, i64, i64, vp, vp, vp, i64, vp, vp, i64, vp]
    L.oracle_pack_w4.argtypes = [vp, i64, i64, vp]
    L.oracle_pack_zeros.argtypes = [vp, i64, i64, i64, vp]
    L.oracle_pack_scales.argtypes = [vp, i64, i64, i64, vp]
    L.oracle_channel_salience.argtypes = [vp, i64, i64, vp, i64, vp]
    L.oracle_select_top_t.argtypes = [vp, i64, i64, vp]
    return L


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = configure(ctypes.CDLL(build()))
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- fp16 / I2F

def f32_to_f16(x) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_f32_to_f16_array(_p(x), x.size, _p(out))
    return out.view(np.float16)


def f16_to_f32(h) -> np.ndarray:
    h = _c(np.asarray(h).view(np.uint16) if np.asarray(h).dtype == np.float16 else h, np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_f16_to_f32_array(_p(h), h.size, _p(out))
    return out


def i2f_bias(p: int) -> float:
    return lib().oracle_i2f_bias(int(p))


def i2f_mismatches(lo: int, hi: int) -> int:
    return int(lib().oracle_i2f_mismatches(int(lo), int(hi)))


# ---------------------------------------------------------------- quantizers

def quantize_act(X: np.ndarray):
    """X fp16 [M, K] -> (A_q int8 [M, K], s_a fp32 [M, K/128])."""
    X = _c(X, np.float16)
    M, K = X.shape
    assert K % GROUP == 0
    A = np.empty((M, K), np.int8)
    s = np.empty((M, K // GROUP), np.float32)
    lib().oracle_quantize_act(_p(X), M, K, _p(A), _p(s))
    return A, s


def quantize_w4(W: np.ndarray):
    """W fp32 [N, K] -> (q uint8 [N, K] in 0..15, z uint8 [N, G], s fp16 [N, G])."""
    W = _c(W, np.float32)
    N, K = W.shape
    G = K // GROUP
    q = np.empty((N, K), np.uint8)
    z = np.empty((N, G), np.uint8)
    s = np.empty((N, G), np.uint16)
    lib().oracle_quantize_w4(_p(W), N, K, _p(q), _p(z), _p(s))
    return q, z, s.view(np.float16)


def quantize_w8(W: np.ndarray):
    """W fp32 [N, K] -> (q int8 [N, K], s fp16 [N, G])."""
    W = _c(W, np.float32)
    N, K = W.shape
    G = K // GROUP
    q = np.empty((N, K), np.int8)
    s = np.empty((N, G), np.uint16)
    lib().oracle_quantize_w8(_p(W), N, K, _p(q), _p(s))
    return q, s.view(np.float16)


def split_channels(is8: np.ndarray):
    """Channel bit map [N] -> (idx4 int32 ascending, idx8 int32 ascending)."""
    is8 = _c(np.asarray(is8) != 0, np.uint8)
    N = is8.size
    idx4 = np.empty(N, np.int32)
    idx8 = np.empty(N, np.int32)
    n8 = int(lib().oracle_split_channels(_p(is8), N, _p(idx4), _p(idx8)))
    return idx4[: N - n8].copy(), idx8[:n8].copy()


# ---------------------------------------------------------------- GEMM

class Quantized:
    """The logical (unpacked) quantized weights of one linear layer."""

    def __init__(self, W: np.ndarray, is8: np.ndarray):
        W = _c(W, np.float32)
        self.N, self.K = W.shape
        self.idx4, self.idx8 = split_channels(is8)
        self.q4, self.z4, self.s4 = quantize_w4(W[self.idx4]) if self.idx4.size else (
            np.zeros((0, self.K), np.uint8), np.zeros((0, self.K // GROUP), np.uint8),
            np.zeros((0, self.K // GROUP), np.float16))
        self.q8, self.s8 = quantize_w8(W[self.idx8]) if self.idx8.size else (
            np.zeros((0, self.K), np.int8), np.zeros((0, self.K // GROUP), np.float16))


def gemm_w4w8a8(A_q, s_a, Wq: Quantized) -> np.ndarray:
    """Two-step dequantization GEMM -> Y fp16 [M, N]."""
    A_q = _c(A_q, np.int8)
    s_a = _c(s_a, np.float32)
    M, K = A_q.shape
    assert K == Wq.K
    Y = np.zeros((M, Wq.N), np.uint16)
    q4, z4, s4 = _c(Wq.q4, np.uint8), _c(Wq.z4, np.uint8), _c(Wq.s4.view(np.uint16), np.uint16)
    q8, s8 = _c(Wq.q8, np.int8), _c(Wq.s8.view(np.uint16), np.uint16)
    i4, i8 = _c(Wq.idx4, np.int32), _c(Wq.idx8, np.int32)
    lib().oracle_gemm_w4w8a8(_p(A_q), _p(s_a), M, K, _p(q4), _p(z4), _p(s4), _p(i4), i4.size,
                             _p(q8), _p(s8), _p(i8), i8.size, _p(Y))
    return Y.view(np.float16)


def group_partials(A_q, Wq: Quantized) -> np.ndarray:
    """Per-group int32 partials P [M, N, G] (output-channel order)."""
    A_q = _c(A_q, np.int8)
    M, K = A_q.shape
    G = K // GROUP
    P = np.zeros((M, Wq.N, G), np.int32)
    q4, z4 = _c(Wq.q4, np.uint8), _c(Wq.z4, np.uint8)
    q8 = _c(Wq.q8, np.int8)
    i4, i8 = _c(Wq.idx4, np.int32), _c(Wq.idx8, np.int32)
    lib().oracle_group_partials(_p(A_q), M, K, _p(q4), _p(z4), _p(i4), i4.size,
                                _p(q8), _p(i8), i8.size, _p(P))
    return P


# ---------------------------------------------------------------- packed layout

def padded(n: int) -> int:
    """Channel count rounded up to the packed layout's multiple of 256."""
    return (n + 255) // 256 * 256


def pack_w4(q4: np.ndarray) -> np.ndarray:
    """Packed 4-bit codes, [tiles of 128 channels, G, 128, 64] bytes."""
    q4 = _c(q4, np.uint8)
    N4, K = q4.shape
    out = np.empty(((N4 + 127) // 128, K // 128, 128, 64), np.uint8)
    lib().oracle_pack_w4(_p(q4), N4, K, _p(out))
    return out


def pack_zeros(z: np.ndarray) -> np.ndarray:
    z = _c(z, np.uint8)
    N, G = z.shape
    Np = padded(N)
    out = np.empty((G, Np // 2), np.uint8)
    lib().oracle_pack_zeros(_p(z), N, G, Np, _p(out))
    return out


def pack_scales(s: np.ndarray) -> np.ndarray:
    s = _c(np.asarray(s).view(np.uint16), np.uint16)
    N, G = s.shape
    Np = padded(N)
    out = np.empty((G, Np), np.uint16)
    lib().oracle_pack_scales(_p(s), N, G, Np, _p(out))
    return out.view(np.float16)


def packed(Wq: Quantized) -> dict:
    """Every packed array of the library's layout, computed from the oracle's
    quantized values (for byte-exact comparison with the device packer)."""
    return {
        "W4": pack_w4(Wq.q4),
        "z4": pack_zeros(Wq.z4),
        "s_w4": pack_scales(Wq.s4),
        "idx4": Wq.idx4.copy(),
        "W8": Wq.q8.copy(),
        "s_w8": pack_scales(Wq.s8),
        "idx8": Wq.idx8.copy(),
    }


# ---------------------------------------------------------------- global search

def channel_salience(W: np.ndarray, G: np.ndarray) -> np.ndarray:
    """Salience S [N] (fp64) of every output channel of one layer:
    W fp32 [N, K], G fp32 [D, N, K] per-sample gradients."""
    W = _c(W, np.float32)
    G = _c(G, np.float32)
    N, K = W.shape
    D = G.shape[0]
    assert G.shape == (D, N, K)
    S = np.zeros(N, np.float64)
    lib().oracle_channel_salience(_p(W), N, K, _p(G), D, _p(S))
    return S


def select_top_t(S: np.ndarray, T: int) -> np.ndarray:
    """Bit map [Ntot] (uint8) of the T channels of largest fp32 salience,
    equal saliences in index order."""
    S = _c(S, np.float32)
    is8 = np.zeros(S.size, np.uint8)
    lib().oracle_select_top_t(_p(S), S.size, int(T), _p(is8))
    return is8
