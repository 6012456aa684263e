"""The linears of one decoder layer as a single CUDA graph.

A Llama decoder layer runs four W4.4A8 linears -- fused qkv, o_proj, fused
gate_up and down -- each as activation quantization followed by the fused
GEMM (MLSys 2026 talk notes on MixLLM, notes.yuuk.io, §探索の特性: the
per-layer view of the method's kernels).  The attention core, the norms and
the SwiGLU between them are not part of the method and are not run here: each
linear reads its own input buffer.

`LinearChain` holds the packed weights and every intermediate buffer of such
a chain, runs it eagerly, and captures it once into a CUDA graph so that a
replay issues all of its kernels with one launch from the host.  For M <= 64
each linear is one mixllm_linear_small_m call (by default; fused=False keeps
quantize_act and the few-token GEMM as two calls): where the plan allows, the
GEMV quantizes its own slice of X and the layer is a single kernel.  Buffers
are allocated once, at construction; a replay allocates nothing.
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
    lws: Optional[torch.Tensor]  # workspace of the fused few-token layer, or None


class LinearChain:
    """A fixed sequence of W4.4A8 linears over one batch of M tokens."""

    def __init__(self, packed: List[_lib.PackedLinear], M: int, device, fused: bool = True):
        self.M = M
        self.fused = fused
        self.device = torch.device(device)
        self.stages: List[_Stage] = []
        for p in packed:
            X = torch.zeros((M, p.K), dtype=torch.float16, device=self.device)
            A_q = torch.empty((M, p.K), dtype=torch.int8, device=self.device)
            s_a = torch.empty((M, p.K // _lib.GROUP), dtype=torch.float32, device=self.device)
            Y = torch.empty((M, p.N), dtype=torch.float16, device=self.device)
            small = 0 < M <= _lib.SMALL_M_MAX
            ws = _lib.small_m_workspace(M, p, self.device) if small else None
            lws = _lib.linear_small_m_workspace(M, p, self.device) if small and fused else None
            self.stages.append(_Stage(p, X, A_q, s_a, Y, ws, lws))
        self.graph: Optional[torch.cuda.CUDAGraph] = None

    @property
    def inputs(self) -> List[torch.Tensor]:
        return [s.X for s in self.stages]

    @property
    def outputs(self) -> List[torch.Tensor]:
        return [s.Y for s in self.stages]

    def launches(self) -> int:
        """Kernels one run issues: one per linear whose GEMV quantizes its own
        activations (the fused workspace is no larger than the GEMM's alone),
        two otherwise."""
        n = 0
        for s in self.stages:
            fused = s.lws is not None and s.lws.numel() == max(
                256, _lib.small_m_workspace_bytes(self.M, s.p.K, s.p.N4, s.p.N8))
            n += 1 if fused else 2
        return n

    def ops(self) -> int:
        return sum(2 * self.M * s.p.N * s.p.K for s in self.stages)

    def run(self, stream=None):
        """Every stage, eagerly, on `stream` (default: the current stream)."""
        for s in self.stages:
            if s.lws is not None:
                _lib.linear_small_m_into(s.X, s.p, s.Y, s.lws, stream)
                continue
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
