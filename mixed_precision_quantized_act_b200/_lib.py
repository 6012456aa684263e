"""Python binding of the C ABI in ``include/mixllm.h`` (ctypes).

Argument marshalling only: torch provides device memory and streams; every
step of the layer runs in the CUDA library ``libmixllm_b200.so``.  There is no
fallback: if the library or a CUDA device is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmixllm_b200.so")
GROUP = 128

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = 0, 1, 2, 3, 4, 5
_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT", 5: "BOUNDS"}

# Every entry point declared in include/mixllm.h, with (restype, argtypes).
_i64, _i32, _u32, _vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_void_p
SIGNATURES = {
    "mixllm_version": (ctypes.c_int, []),
    "mixllm_last_error": (ctypes.c_char_p, []),
    "mixllm_packed_sizes": (ctypes.c_int, [_i64, _i64, _i64, _i32, ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_quantize_act": (ctypes.c_int, [_vp, _i64, _i64, _i32, _vp, _vp, _vp]),
    "mixllm_pack_weights_host": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32,
                                                _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mixllm_pack_weights": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _i32,
                                           _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mixllm_gemm_w4w8a8": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                          _vp, _vp, _vp, _i64, _vp, _vp]),
    "mixllm_gemm_debug_partials": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                                  _vp, _vp, _vp, _i64, _vp, _vp]),
    "mixllm_gemm_w4w8a8_plain_i2f": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                                    _vp, _vp, _vp, _i64, _vp, _vp]),
    "mixllm_small_m_workspace_bytes": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_small_m_kernel": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.POINTER(ctypes.c_int32)]),
    "mixllm_channel_salience": (ctypes.c_int, [_vp, _i64, _i64, _vp, _i64, _vp, _vp]),
    "mixllm_linear_small_m_workspace_bytes": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_linear_small_m": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64,
                                             _vp, _vp, ctypes.c_size_t, _vp]),
    "mixllm_linear_workspace_bytes": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_linear": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64,
                                     _vp, _vp, ctypes.c_size_t, _vp]),
    "mixllm_linear_one_launch": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64,
                                                _vp, _vp, ctypes.c_size_t, _vp]),
    "mixllm_select_top_t_workspace_bytes": (ctypes.c_int, [_i64, ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_select_top_t": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, ctypes.c_size_t, _vp]),
    "mixllm_gemm_w4w8a8_small_m": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                                  _vp, _vp, _vp, _i64, _vp, _vp, ctypes.c_size_t, _vp]),
    "mixllm_gemm_w4w8a8_small_m_noalloc": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                                          _vp, _vp, _vp, _i64, _vp, _vp]),
    "mixllm_small_m_debug_workspace_bytes": (ctypes.c_int, [_i64, _i64, _i64, _i64, ctypes.c_int32,
                                                            ctypes.POINTER(ctypes.c_size_t)]),
    "mixllm_small_m_debug_partials": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64,
                                                     _vp, _vp, _vp, _i64, ctypes.c_int32, _vp, _vp, _vp,
                                                     ctypes.c_size_t, _vp]),
    "mixllm_sync_status": (ctypes.c_int, [_vp]),
    "mixllm_selftest_wait_timeout": (ctypes.c_int, [_u32, _vp]),
    "mixllm_checked_build": (ctypes.c_int, []),
    "mixllm_selftest_bounds": (ctypes.c_int, [_vp]),
}


class MixLLMError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {_NAMES.get(status, status)}: {msg}")
        self.status = status


_lock = threading.Lock()
_lib = None


def load(path: str = None):
    """Load the CUDA library (raises if it was not built).  The path defaults
    to the in-tree release build; the environment variable MIXLLM_LIBRARY
    names another build of the same library (e.g. the checked one)."""
    global _lib
    with _lock:
        if _lib is None:
            path = path or os.environ.get("MIXLLM_LIBRARY") or LIB_PATH
            if not os.path.exists(path):
                raise RuntimeError(
                    f"{path} is missing: build it with `python -m mixed_precision_quantized_act_b200.build`")
            L = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _check(status: int, where: str):
    if status != OK:
        msg = load().mixllm_last_error().decode(errors="replace")
        raise MixLLMError(status, where, msg)


def _ptr(t):
    if t is None:
        return None
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _require(ok: bool, what: str):
    """Argument check that stays on under ``python -O`` (unlike assert)."""
    if not ok:
        raise ValueError(what)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and t.numel() > 0 and not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")


# ---------------------------------------------------------------- entry points

def version() -> int:
    return load().mixllm_version()


def packed_sizes(N: int, K: int, N8: int, group: int = GROUP):
    out = (ctypes.c_size_t * 7)()
    _check(load().mixllm_packed_sizes(N, K, N8, group, out), "mixllm_packed_sizes")
    return list(out)


def quantize_act_into(X: torch.Tensor, A_q: torch.Tensor, s_a: torch.Tensor, stream=None):
    _need_cuda(X, A_q, s_a)
    _require(X.dtype == torch.float16 and A_q.dtype == torch.int8 and s_a.dtype == torch.float32,
             "X must be fp16, A_q int8 and s_a fp32")
    _require(X.is_contiguous() and A_q.is_contiguous() and s_a.is_contiguous(), "X, A_q and s_a must be contiguous")
    M, K = X.shape
    _check(load().mixllm_quantize_act(_ptr(X), M, K, GROUP, _ptr(A_q), _ptr(s_a), _stream(stream)),
           "mixllm_quantize_act")


def quantize_act(X: torch.Tensor, stream=None):
    """X fp16 [M, K] (CUDA) -> (A_q int8 [M, K], s_a fp32 [M, K/128])."""
    M, K = X.shape
    A_q = torch.empty((M, K), dtype=torch.int8, device=X.device)
    s_a = torch.empty((M, K // GROUP), dtype=torch.float32, device=X.device)
    quantize_act_into(X, A_q, s_a, stream)
    return A_q, s_a


@dataclass
class PackedLinear:
    """Packed weights of one W4.4A8 linear layer (device tensors)."""
    N: int
    K: int
    N4: int
    N8: int
    W4: torch.Tensor    # uint8 [ceil(N4/128), K/128, 128, 64]: one block per (128-channel tile, group)
    z4: torch.Tensor    # uint8 [G, N4p/2]
    s_w4: torch.Tensor  # fp16 [G, N4p]
    idx4: torch.Tensor  # int32 [N4]
    W8: torch.Tensor    # int8 [N8, K]
    s_w8: torch.Tensor  # fp16 [G, N8p]
    idx8: torch.Tensor  # int32 [N8]

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.W4, self.z4, self.s_w4, self.idx4, self.W8, self.s_w8, self.idx8))

    def to(self, device) -> "PackedLinear":
        """The same packed layer with every buffer on `device` (a copy)."""
        return PackedLinear(self.N, self.K, self.N4, self.N8,
                            *(t.to(device).contiguous() for t in
                              (self.W4, self.z4, self.s_w4, self.idx4, self.W8, self.s_w8, self.idx8)))


def padded(n: int) -> int:
    return (n + 255) // 256 * 256


def empty_packed(N: int, K: int, N8: int, device) -> PackedLinear:
    N4, G = N - N8, K // GROUP
    u8, i8, f16, i32 = torch.uint8, torch.int8, torch.float16, torch.int32
    return PackedLinear(
        N, K, N4, N8,
        torch.empty(((N4 + 127) // 128, G, 128, 64), dtype=u8, device=device),
        torch.empty((G, padded(N4) // 2), dtype=u8, device=device),
        torch.empty((G, padded(N4)), dtype=f16, device=device),
        torch.empty((N4,), dtype=i32, device=device),
        torch.empty((N8, K), dtype=i8, device=device),
        torch.empty((G, padded(N8)), dtype=f16, device=device),
        torch.empty((N8,), dtype=i32, device=device),
    )


def pack_weights(W: torch.Tensor, is8: torch.Tensor, stream=None) -> PackedLinear:
    """W fp32 [N, K] and the channel bit map uint8 [N] (CUDA) -> PackedLinear.
    Synchronous (offline step)."""
    _need_cuda(W, is8)
    _require(W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2, "W must be a contiguous fp32 [N, K]")
    _require(is8.dtype == torch.uint8 and is8.is_contiguous() and is8.numel() == W.shape[0],
             "is8 must be a contiguous uint8 [N]")
    N, K = W.shape
    N8 = int((is8 != 0).sum().item())
    p = empty_packed(N, K, N8, W.device)
    sizes = packed_sizes(N, K, N8)
    got = [t.numel() * t.element_size() for t in (p.W4, p.z4, p.s_w4, p.idx4, p.W8, p.s_w8, p.idx8)]
    _require(got == sizes, f"packed buffer sizes {got} differ from the library's {sizes}")
    _check(load().mixllm_pack_weights(_ptr(W), N, K, _ptr(is8), N8, GROUP, _ptr(p.W4), _ptr(p.z4),
                                      _ptr(p.s_w4), _ptr(p.idx4), _ptr(p.W8), _ptr(p.s_w8),
                                      _ptr(p.idx8), _stream(stream)), "mixllm_pack_weights")
    return p


def pack_weights_host(W: torch.Tensor, is8: torch.Tensor) -> PackedLinear:
    """The same pack on the host CPU (mixllm_pack_weights_host): W fp32 [N, K]
    and is8 uint8 [N] in host memory -> a PackedLinear of CPU tensors with the
    same bytes as pack_weights (move it to a device with PackedLinear.to)."""
    _require(not W.is_cuda and not is8.is_cuda, "W and is8 must be host (CPU) tensors")
    _require(W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2, "W must be a contiguous fp32 [N, K]")
    _require(is8.dtype == torch.uint8 and is8.is_contiguous() and is8.numel() == W.shape[0],
             "is8 must be a contiguous uint8 [N]")
    N, K = W.shape
    N8 = int((is8 != 0).sum().item())
    p = empty_packed(N, K, N8, "cpu")
    _check(load().mixllm_pack_weights_host(_ptr(W), N, K, _ptr(is8), N8, GROUP, _ptr(p.W4), _ptr(p.z4),
                                           _ptr(p.s_w4), _ptr(p.idx4), _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8)),
           "mixllm_pack_weights_host")
    return p


def gemm_w4w8a8_into(A_q, s_a, p: PackedLinear, Y, stream=None):
    _need_cuda(A_q, s_a, Y)
    M, K = A_q.shape
    _require(K == p.K and tuple(Y.shape) == (M, p.N) and Y.dtype == torch.float16 and Y.is_contiguous(),
             "Y must be a contiguous fp16 [M, N] and A_q must have the layer's K")
    _check(load().mixllm_gemm_w4w8a8(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4),
                                     _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8,
                                     _ptr(Y), _stream(stream)), "mixllm_gemm_w4w8a8")


def gemm_w4w8a8_plain_i2f_into(A_q, s_a, p: PackedLinear, Y, stream=None):
    """The fused GEMM with a plain int -> float convert instead of the bias
    trick (the ablation the talk notes' fast-I2F section measures); same Y."""
    _need_cuda(A_q, s_a, Y)
    M, K = A_q.shape
    _require(K == p.K and tuple(Y.shape) == (M, p.N) and Y.dtype == torch.float16 and Y.is_contiguous(),
             "Y must be a contiguous fp16 [M, N] and A_q must have the layer's K")
    _check(load().mixllm_gemm_w4w8a8_plain_i2f(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4),
                                               _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8,
                                               _ptr(Y), _stream(stream)), "mixllm_gemm_w4w8a8_plain_i2f")


def gemm_w4w8a8(A_q, s_a, p: PackedLinear, stream=None) -> torch.Tensor:
    Y = torch.empty((A_q.shape[0], p.N), dtype=torch.float16, device=A_q.device)
    gemm_w4w8a8_into(A_q, s_a, p, Y, stream)
    return Y


def gemm_debug_partials(A_q, s_a, p: PackedLinear, stream=None) -> torch.Tensor:
    """Per-group int32 partials P [M, N, K/128] (debug path of the fused kernel)."""
    _need_cuda(A_q, s_a)
    M, K = A_q.shape
    P = torch.zeros((M, p.N, K // GROUP), dtype=torch.int32, device=A_q.device)
    _check(load().mixllm_gemm_debug_partials(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4),
                                             _ptr(p.s_w4), _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8),
                                             _ptr(p.idx8), p.N8, _ptr(P), _stream(stream)),
           "mixllm_gemm_debug_partials")
    return P


SMALL_M_MAX = 64


def small_m_workspace_bytes(M: int, K: int, N4: int, N8: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load().mixllm_small_m_workspace_bytes(M, K, N4, N8, ctypes.byref(out)), "mixllm_small_m_workspace_bytes")
    return out.value


def linear_small_m_workspace(M: int, p: PackedLinear, device) -> torch.Tensor:
    """A zero-filled workspace for mixllm_linear_small_m (every call leaves
    its counters at zero, so it can be reused)."""
    out = ctypes.c_size_t(0)
    _check(load().mixllm_linear_small_m_workspace_bytes(M, p.K, p.N4, p.N8, ctypes.byref(out)),
           "mixllm_linear_small_m_workspace_bytes")
    return torch.zeros(max(256, out.value), dtype=torch.uint8, device=device)


def linear_small_m_into(X, p: PackedLinear, Y, workspace: torch.Tensor, stream=None):
    """The few-token layer from fp16 X, quantization included (mixllm_linear_small_m)."""
    _need_cuda(X, Y, workspace)
    M, K = X.shape
    _check(load().mixllm_linear_small_m(_ptr(X), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4), _ptr(p.idx4), p.N4,
                                        _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8, _ptr(Y), _ptr(workspace),
                                        workspace.numel(), _stream(stream)), "mixllm_linear_small_m")


def linear_workspace(M: int, p: PackedLinear, device) -> torch.Tensor:
    """A zero-filled workspace for mixllm_linear (every call leaves its
    counters at zero, so it can be reused by calls that do not overlap)."""
    out = ctypes.c_size_t(0)
    _check(load().mixllm_linear_workspace_bytes(M, p.K, p.N4, p.N8, ctypes.byref(out)),
           "mixllm_linear_workspace_bytes")
    return torch.zeros(max(256, out.value), dtype=torch.uint8, device=device)


def linear_into(X, p: PackedLinear, Y, workspace: torch.Tensor, stream=None, one_launch: bool = False):
    """The layer from fp16 X for any M, quantization included (mixllm_linear);
    one_launch (M > 64): the tiled GEMM quantizes X itself
    (mixllm_linear_one_launch), same result."""
    _need_cuda(X, Y, workspace)
    M, K = X.shape
    _require(K == p.K and tuple(Y.shape) == (M, p.N) and Y.dtype == torch.float16 and Y.is_contiguous(),
             "Y must be a contiguous fp16 [M, N] and X must have the layer's K")
    _require(X.dtype == torch.float16 and X.is_contiguous() and workspace.is_contiguous(),
             "X must be a contiguous fp16 [M, K] and the workspace contiguous")
    fn = "mixllm_linear_one_launch" if one_launch else "mixllm_linear"
    _check(getattr(load(), fn)(_ptr(X), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4), _ptr(p.idx4), p.N4,
                               _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8, _ptr(Y), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)), fn)


SMALL_M_KERNELS = ("tensor-core split-K", "GEMV split-K", "GEMV persistent")


def small_m_kernel(M: int, K: int, N4: int, N8: int) -> str:
    """The few-token kernel the library runs for this shape (mixllm_small_m_kernel)."""
    out = ctypes.c_int32(-1)
    _check(load().mixllm_small_m_kernel(M, K, N4, N8, ctypes.byref(out)), "mixllm_small_m_kernel")
    return SMALL_M_KERNELS[out.value]


def small_m_workspace(M: int, p: PackedLinear, device) -> torch.Tensor:
    """A zero-filled workspace for mixllm_gemm_w4w8a8_small_m (every call
    returns its tile counters, the last 4 bytes per 128-channel tile, to zero)."""
    n = small_m_workspace_bytes(M, p.K, p.N4, p.N8)
    return torch.zeros(max(n, 16), dtype=torch.uint8, device=device)


def gemm_w4w8a8_small_m_into(A_q, s_a, p: PackedLinear, Y, workspace: torch.Tensor, stream=None):
    _need_cuda(A_q, s_a, Y, workspace)
    M, K = A_q.shape
    _require(K == p.K and tuple(Y.shape) == (M, p.N) and Y.dtype == torch.float16 and Y.is_contiguous(),
             "Y must be a contiguous fp16 [M, N] and A_q must have the layer's K")
    _require(workspace.is_contiguous(), "the workspace must be contiguous")
    _check(load().mixllm_gemm_w4w8a8_small_m(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4),
                                             _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8,
                                             _ptr(Y), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "mixllm_gemm_w4w8a8_small_m")


def gemm_w4w8a8_small_m(A_q, s_a, p: PackedLinear, workspace: torch.Tensor = None, stream=None) -> torch.Tensor:
    M = A_q.shape[0]
    if workspace is None:
        workspace = small_m_workspace(M, p, A_q.device)
    Y = torch.empty((M, p.N), dtype=torch.float16, device=A_q.device)
    gemm_w4w8a8_small_m_into(A_q, s_a, p, Y, workspace, stream)
    return Y


def gemm_w4w8a8_small_m_noalloc_into(A_q, s_a, p: PackedLinear, Y, stream=None):
    """The few-token GEMM on the library's static device scratch (no workspace,
    no allocation); calls must not overlap in time on one device."""
    _need_cuda(A_q, s_a, Y)
    M, K = A_q.shape
    _require(K == p.K and tuple(Y.shape) == (M, p.N) and Y.dtype == torch.float16 and Y.is_contiguous(),
             "Y must be a contiguous fp16 [M, N] and A_q must have the layer's K")
    _check(load().mixllm_gemm_w4w8a8_small_m_noalloc(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4),
                                                     _ptr(p.s_w4), _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8),
                                                     _ptr(p.idx8), p.N8, _ptr(Y), _stream(stream)),
           "mixllm_gemm_w4w8a8_small_m_noalloc")


def small_m_debug_partials(A_q, s_a, p: PackedLinear, kind: str, stream=None):
    """Debug form of one named few-token kernel (one of SMALL_M_KERNELS, run
    whatever the plan would pick): returns (Y fp16 [M, N], P int32 [M, N, K/128])."""
    _need_cuda(A_q, s_a)
    M, K = A_q.shape
    k = SMALL_M_KERNELS.index(kind)
    n = ctypes.c_size_t(0)
    _check(load().mixllm_small_m_debug_workspace_bytes(M, K, p.N4, p.N8, k, ctypes.byref(n)),
           "mixllm_small_m_debug_workspace_bytes")
    ws = torch.zeros(max(n.value, 16), dtype=torch.uint8, device=A_q.device)
    Y = torch.empty((M, p.N), dtype=torch.float16, device=A_q.device)
    P = torch.zeros((M, p.N, K // GROUP), dtype=torch.int32, device=A_q.device)
    _check(load().mixllm_small_m_debug_partials(_ptr(A_q), _ptr(s_a), M, K, _ptr(p.W4), _ptr(p.z4), _ptr(p.s_w4),
                                                _ptr(p.idx4), p.N4, _ptr(p.W8), _ptr(p.s_w8), _ptr(p.idx8), p.N8,
                                                k, _ptr(P), _ptr(Y), _ptr(ws), ws.numel(), _stream(stream)),
           "mixllm_small_m_debug_partials")
    return Y, P


def linear(X: torch.Tensor, p: PackedLinear, stream=None, workspace: torch.Tensor = None) -> torch.Tensor:
    """The whole layer from fp16 X (mixllm_linear), with `workspace` or a
    fresh zero-filled one."""
    M = X.shape[0]
    Y = torch.empty((M, p.N), dtype=torch.float16, device=X.device)
    if M == 0:
        return Y
    if workspace is None:
        workspace = linear_workspace(M, p, X.device)
    linear_into(X, p, Y, workspace, stream)
    return Y


def sync_status(stream=None):
    _check(load().mixllm_sync_status(_stream(stream)), "mixllm_sync_status")


def checked_build() -> bool:
    """True when the loaded library is the range-checked build."""
    return bool(load().mixllm_checked_build())


def selftest_bounds(stream=None):
    """Checked build: makes the range checks fire without an access (read the
    result with sync_status); the release build raises UNSUPPORTED."""
    _check(load().mixllm_selftest_bounds(_stream(stream)), "mixllm_selftest_bounds")


def selftest_wait_timeout(limit_us: int, stream=None):
    _check(load().mixllm_selftest_wait_timeout(limit_us, _stream(stream)), "mixllm_selftest_wait_timeout")


# ---------------------------------------------------------------- global search

def channel_salience(W: torch.Tensor, G: torch.Tensor, stream=None) -> torch.Tensor:
    """Salience of every output channel of one layer (mixllm_channel_salience):
    W fp32 [N, K], G fp32 [D, N, K] per-sample gradients, both on the device."""
    _need_cuda(W, G)
    W = W.contiguous()
    G = G.contiguous()
    N, K = W.shape
    D = G.shape[0]
    if G.dtype != torch.float32 or W.dtype != torch.float32 or tuple(G.shape) != (D, N, K):
        raise ValueError("W must be fp32 [N, K] and G fp32 [D, N, K]")
    S = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(load().mixllm_channel_salience(_ptr(W), N, K, _ptr(G), D, _ptr(S), _stream(stream)),
           "mixllm_channel_salience")
    return S


def channel_salience_into(W: torch.Tensor, G: torch.Tensor, S: torch.Tensor, stream=None):
    """mixllm_channel_salience into a caller's fp32 [N] tensor (e.g. a slice
    of one list of all layers' scores)."""
    N, K = W.shape
    D = G.shape[0]
    if not (W.is_contiguous() and G.is_contiguous() and S.is_contiguous()) or S.numel() != N:
        raise ValueError("contiguous W [N, K], G [D, N, K] and S [N] expected")
    _check(load().mixllm_channel_salience(_ptr(W), N, K, _ptr(G), D, _ptr(S), _stream(stream)),
           "mixllm_channel_salience")


def select_top_t_workspace(n: int, device) -> torch.Tensor:
    out = ctypes.c_size_t(0)
    _check(load().mixllm_select_top_t_workspace_bytes(n, ctypes.byref(out)), "mixllm_select_top_t_workspace_bytes")
    return torch.empty(max(16, out.value), dtype=torch.uint8, device=device)


def select_top_t_into(S: torch.Tensor, T: int, is8: torch.Tensor, workspace: torch.Tensor, stream=None):
    """mixllm_select_top_t with the caller's bit map and workspace."""
    _check(load().mixllm_select_top_t(_ptr(S), S.numel(), int(T), _ptr(is8), _ptr(workspace), workspace.numel(),
                                      _stream(stream)), "mixllm_select_top_t")


def select_top_t(S: torch.Tensor, T: int, stream=None) -> torch.Tensor:
    """Bit map of the T largest scores, equal scores in index order
    (mixllm_select_top_t): S fp32 [n] on the device."""
    _need_cuda(S)
    S = S.contiguous()
    n = S.numel()
    out = ctypes.c_size_t(0)
    _check(load().mixllm_select_top_t_workspace_bytes(n, ctypes.byref(out)), "mixllm_select_top_t_workspace_bytes")
    ws = torch.empty(max(1, out.value), dtype=torch.uint8, device=S.device)
    is8 = torch.empty(n, dtype=torch.uint8, device=S.device)
    _check(load().mixllm_select_top_t(_ptr(S), n, int(T), _ptr(is8), _ptr(ws), out.value, _stream(stream)),
           "mixllm_select_top_t")
    return is8
