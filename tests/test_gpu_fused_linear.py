"""The few-token layer from fp16 activations (mixllm_linear_small_m): the
activation quantization fused into the split GEMV's prologue where a CTA's
slice of X fits a ring slot, the quantizer then the planned kernel
elsewhere.  Either way Y must be bit-identical to quantize_act followed by
mixllm_gemm_w4w8a8_small_m (the same codes, scales and arithmetic), and within
the layer's tolerance of the CPU oracle.  GPU only.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mixed_precision_quantized_act_b200 as mx  # noqa: E402
from mixed_precision_quantized_act_b200 import _lib  # noqa: E402
from mixed_precision_quantized_act_b200 import workloads as wl  # noqa: E402

pytestmark = pytest.mark.gpu

REL, ABS_RMS = 2.0 ** -9, 1e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mx.load()
    return torch.device("cuda:0")


def _layer(name, M, N, K, n8):
    return wl.Linear(name, M, N, K, ((0, N, n8),), 4)


# (layer, fused?): the fused form runs for one token on the split GEMV (a CTA's
# slice of X, ceil(G / S4) x 256 bytes, fitting one 32 KiB slot)
CASES = [
    (wl.Q_PROJ_P10.with_m(1), True),
    (_layer("fl_m1_ragged", 1, 300, 384, 37), True),
    (_layer("fl_m1_one8", 1, 260, 256, 1), True),
    (_layer("fl_m1_p100", 1, 512, 1024, 512), True),
    (wl.LLAMA8B_LAYER[2].with_m(1), True),     # gate_up: 1 split, 32 groups per CTA
    (wl.LLAMA8B_LAYER[3].with_m(1), True),     # down: K = 14336
    (wl.Q_PROJ_P10.with_m(3), False),          # more than one token: quantizer, then the GEMV
    (_layer("fl_m5_ragged", 5, 300, 384, 37), False),
    (wl.LLAMA8B_LAYER[2].with_m(8), False),
    (wl.LLAMA70B[2].with_m(1), False),         # the persistent GEMV
    (wl.Q_PROJ_P10.with_m(16), False),         # the tensor-core kernel
]


def _sample(layer, seed):
    X, W, is8 = wl.make_x(layer, seed), wl.make_w(layer, seed), wl.make_bitmap(layer, seed)
    return X, W, is8


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_fused_linear_matches_two_calls_and_oracle(dev, case):
    layer, fused = case
    X, W, is8 = _sample(layer, 31)
    Xd = torch.from_numpy(X).to(dev)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.linear_small_m_workspace(layer.M, p, dev)
    plain = mx.small_m_workspace_bytes(layer.M, layer.K, p.N4, p.N8)
    assert (ws.numel() == max(256, plain)) == fused, "workspace size tells whether the fused form runs"
    Y = torch.full((layer.M, layer.N), float("nan"), dtype=torch.float16, device=dev)
    mx.linear_small_m_into(Xd, p, Y, ws)
    Y2 = torch.full_like(Y, float("nan"))
    mx.linear_small_m_into(Xd, p, Y2, ws)  # again, on the same workspace
    A_q, s_a = mx.quantize_act(Xd)
    Y_ref = mx.gemm_w4w8a8_small_m(A_q, s_a, p)
    mx.sync_status()
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    assert torch.equal(Y2.view(torch.int16), Y_ref.view(torch.int16))
    cols = np.arange(layer.N) if layer.N <= 8192 else np.sort(np.random.default_rng(5).choice(layer.N, 2048, replace=False))
    A_o, s_o = oracle.quantize_act(X)
    Y_o = oracle.gemm_w4w8a8(A_o, s_o, oracle.Quantized(W[cols], is8[cols])).astype(np.float64)
    rms = float(np.sqrt(np.mean(Y_o ** 2)))
    err = np.abs(Y.cpu().numpy()[:, cols].astype(np.float64) - Y_o)
    assert (err <= REL * np.abs(Y_o) + ABS_RMS * rms).all()


def test_fused_linear_validation(dev):
    layer = _layer("fl_val", 2, 256, 256, 20)
    X, W, is8 = _sample(layer, 1)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.linear_small_m_workspace(2, p, dev)
    Y = torch.empty((2, 256), dtype=torch.float16, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.linear_small_m_into(torch.zeros((65, 256), dtype=torch.float16, device=dev), p,
                               torch.empty((65, 256), dtype=torch.float16, device=dev), ws)
    assert ei.value.status == _lib.ERR_INVALID_ARG
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.linear_small_m_into(torch.from_numpy(X).to(dev), p, Y, ws[:16])
    assert ei.value.status == _lib.ERR_INVALID_ARG
    mx.sync_status()
