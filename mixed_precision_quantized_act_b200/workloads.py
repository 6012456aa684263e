"""Seeded synthetic workloads for the W4.4A8 linear layer.

This module only draws inputs; it holds none of the method's arithmetic, so
both the CPU oracle (in the tests) and the CUDA path consume the very same
arrays.  The shapes and distributions stand in for the paper's workloads,
which are real Llama activations and weights (not available here):

* X fp16 [M, K] ~ N(0, 1), with ceil(1% of K) randomly chosen input columns
  scaled by 20 (exactly 4 columns for the tiny case) -- activation outliers;
* W fp32 [N, K] ~ N(0, 0.02);
* a random set of output channels flagged 8-bit (the global bit map); its
  size per slice is given per layer, otherwise round-half-up(frac * N);
* group size 128 along K.

Random numbers come from numpy's PCG64 generator seeded per (workload, seed).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

GROUP = 128


@dataclass(frozen=True)
class Linear:
    """One linear layer: Y[M, N] = X[M, K] . W[N, K]^T with a bit map.

    ``slices`` lists (start, stop, n8) ranges of output channels and how many
    of each range are 8-bit; channels outside every range are 4-bit.
    """

    name: str
    M: int
    N: int
    K: int
    slices: tuple = field(default_factory=tuple)
    outlier_cols: int | None = None  # None -> ceil(1% of K)

    @property
    def N8(self) -> int:
        return sum(s[2] for s in self.slices)

    @property
    def N4(self) -> int:
        return self.N - self.N8

    @property
    def G(self) -> int:
        return self.K // GROUP

    def ops(self) -> int:
        """Algorithmic integer operations, 2*M*N*K."""
        return 2 * self.M * self.N * self.K

    def algorithmic_bytes(self) -> int:
        """Bytes the layer must move at least once: packed weights with their
        scales and zero points, A_q with fp32 s_a, and the fp16 output."""
        return (self.N4 * self.K // 2 + self.N4 * self.G * 2 + self.N4 * self.G // 2
                + self.N8 * self.K + self.N8 * self.G * 2
                + self.M * self.K + self.M * self.G * 4
                + 2 * self.M * self.N)

    def with_m(self, M: int) -> "Linear":
        return Linear(f"{self.name}@M{M}", M, self.N, self.K, self.slices, self.outlier_cols)


def round_half_up(x: float) -> int:
    return int(math.floor(x + 0.5))


def _mix(name, M, N, K, frac):
    return Linear(name, M, N, K, ((0, N, round_half_up(frac * N)),))


# The tiny case: 52 of 512 channels 8-bit, 4 outlier columns.
TINY = Linear("tiny_w4.4a8_M16_N512_K512", 16, 512, 512, ((0, 512, 52),), outlier_cols=4)

# Llama-3.1-8B q_proj shape, p10: 410 of 4096 channels 8-bit.
Q_PROJ_P10 = Linear("llama3.1-8b_q_proj_p10_M512_N4096_K4096", 512, 4096, 4096, ((0, 4096, 410),))
M_SWEEP = (1, 16, 64, 256, 1024)

# Llama-3.1-8B decoder-layer linears at M=512.  qkv = q[0,4096) k[4096,5120)
# v[5120,6144); 71% of v's channels and 5% of q/k's are 8-bit.
LLAMA8B_LAYER = (
    Linear("llama3.1-8b_qkv_M512_N6144_K4096", 512, 6144, 4096,
           ((0, 5120, round_half_up(0.05 * 5120)), (5120, 6144, round_half_up(0.71 * 1024)))),
    _mix("llama3.1-8b_o_proj_M512_N4096_K4096", 512, 4096, 4096, 0.05),
    _mix("llama3.1-8b_gate_up_M512_N28672_K4096", 512, 28672, 4096, 0.05),
    _mix("llama3.1-8b_down_M512_N4096_K14336", 512, 4096, 14336, 0.54),
)

# Bit-mix sweep at M=512, N=K=4096: p0 (pure W4A8) ... p100 (pure W8A8).
BIT_MIX = tuple(_mix(f"mix_p{p}_M512_N4096_K4096", 512, 4096, 4096, p / 100.0)
                for p in (0, 10, 20, 50, 100))

# Llama-3.1-70B linear shapes at M=1024, p10.
LLAMA70B = (
    _mix("llama3.1-70b_qkv_M1024_N10240_K8192", 1024, 10240, 8192, 0.10),
    _mix("llama3.1-70b_o_proj_M1024_N8192_K8192", 1024, 8192, 8192, 0.10),
    _mix("llama3.1-70b_gate_up_M1024_N57344_K8192", 1024, 57344, 8192, 0.10),
    _mix("llama3.1-70b_down_M1024_N8192_K28672", 1024, 8192, 28672, 0.10),
)

ALL = (TINY, Q_PROJ_P10) + tuple(Q_PROJ_P10.with_m(m) for m in M_SWEEP) + LLAMA8B_LAYER + BIT_MIX + LLAMA70B


def _rng(layer: Linear, seed: int, stream: int) -> np.random.Generator:
    key = sum(ord(c) * 131 ** i for i, c in enumerate(layer.name)) % (2 ** 63)
    return np.random.default_rng([seed, stream, key])


def make_x(layer: Linear, seed: int = 0, M: int | None = None) -> np.ndarray:
    """Activations X fp16 [M, K] ~ N(0,1) with outlier columns x20."""
    M = layer.M if M is None else M
    rng = _rng(layer, seed, 1)
    X = rng.standard_normal((M, layer.K), dtype=np.float32)
    n_out = layer.outlier_cols if layer.outlier_cols is not None else math.ceil(0.01 * layer.K)
    cols = rng.choice(layer.K, size=n_out, replace=False)
    X[:, cols] *= 20.0
    return X.astype(np.float16)


def make_w(layer: Linear, seed: int = 0) -> np.ndarray:
    """Weights W fp32 [N, K] ~ N(0, 0.02)."""
    rng = _rng(layer, seed, 2)
    W = rng.standard_normal((layer.N, layer.K), dtype=np.float32)
    W *= np.float32(0.02)
    return W


def make_bitmap(layer: Linear, seed: int = 0) -> np.ndarray:
    """Global channel bit map uint8 [N]: 1 = 8-bit symmetric channel."""
    rng = _rng(layer, seed, 3)
    is8 = np.zeros(layer.N, np.uint8)
    for start, stop, n8 in layer.slices:
        if n8:
            is8[start + rng.choice(stop - start, size=n8, replace=False)] = 1
    return is8


def by_name(name: str) -> Linear:
    """A workload of ALL by name, or any of them with another token count as
    `<name>@M<m>`."""
    for layer in ALL:
        if layer.name == name:
            return layer
    base, sep, m = name.rpartition("@M")
    if sep and m.isdigit() and int(m) > 0:
        for layer in ALL:
            if layer.name == base:
                return layer.with_m(int(m))
    raise KeyError(name)
