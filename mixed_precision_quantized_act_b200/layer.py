"""The linears of one decoder layer as a single CUDA graph.

A Llama decoder layer runs four W4.4A8 linears -- fused qkv, o_proj, fused
gate_up and down -- each as activation quantization followed by the fused
GEMM (MLSys 2026 talk notes on MixLLM, notes.yuuk.io, §探索の特性: the
per-layer view of the method's kernels).  The attention core, the norms and
the SwiGLU between them are not part of the method and are not run here: each
linear reads its own input buffer.

`LinearChain` holds the packed weights and every intermediate buffer of such
a chain, runs it eagerly, and captures it once into a CUDA graph so that a
replay issues all eight kernels with one launch from the host (the few-token
path is used for M <= 64).  Buffers are allocated once, at construction; a
replay allocates nothing.
"""
from dataclasses import dataclass
from typing import List, Optional

import torch

from . import _lib


@dataclass
class _Stage:
    p: _lib.PackedLinear
    X: torch.Tensor      # fp16 [M, K] input (filled by the caller)
    A_q: torch.Tensor    # int8 [M, K]
    s_a: torch.Tensor    # fp32 [M, K/128]
    Y: torch.Tensor      # fp16 [M, N] output
    ws: Optional[torch.Tensor]  # few-token workspace, or None


class LinearChain:
    """A fixed sequence of W4.4A8 linears over one batch of M tokens."""

    def __init__(self, packed: List[_lib.PackedLinear], M: int, device):
        self.M = M
        self.device = torch.device(device)
        self.stages: List[_Stage] = []
        for p in packed:
            X = torch.zeros((M, p.K), dtype=torch.float16, device=self.device)
            A_q = torch.empty((M, p.K), dtype=torch.int8, device=self.device)
            s_a = torch.empty((M, p.K // _lib.GROUP), dtype=torch.float32, device=self.device)
            Y = torch.empty((M, p.N), dtype=torch.float16, device=self.device)
            ws = _lib.small_m_workspace(M, p, self.device) if 0 < M <= _lib.SMALL_M_MAX else None
            self.stages.append(_Stage(p, X, A_q, s_a, Y, ws))
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    @property
    def inputs(self) -> List[torch.Tensor]:
        return [s.X for s in self.stages]

    @property
    def outputs(self) -> List[torch.Tensor]:
        return [s.Y for s in self.stages]

    def ops(self) -> int:
        return sum(2 * self.M * s.p.N * s.p.K for s in self.stages)

    def run(self, stream=None):
        """Every stage, eagerly, on `stream` (default: the current stream)."""
        for s in self.stages:
            _lib.quantize_act_into(s.X, s.A_q, s.s_a, stream)
            if s.ws is not None:
                _lib.gemm_w4w8a8_small_m_into(s.A_q, s.s_a, s.p, s.Y, s.ws, stream)
            else:
                _lib.gemm_w4w8a8_into(s.A_q, s.s_a, s.p, s.Y, stream)

    def capture(self):
        """Record the chain into a CUDA graph (after one eager warm-up run on a
        side stream, which also builds the library's cached descriptors)."""
        side = torch.cuda.Stream(device=self.device)
        side.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(side):
            self.run()
        torch.cuda.current_stream(self.device).wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.run()
        self.graph = g
        return g

    def replay(self):
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def release(self):
        self.graph = None
