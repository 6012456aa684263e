"""The decoder-layer driver (LinearChain): a chain of W4.4A8 linears replayed
as one CUDA graph gives the same bytes as running the kernels eagerly, and the
eager chain matches the single-layer entry points.  GPU only."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mixed_precision_quantized_act_b200 as mx  # noqa: E402
from mixed_precision_quantized_act_b200 import workloads as wl  # noqa: E402
from mixed_precision_quantized_act_b200.layer import LinearChain  # noqa: E402

pytestmark = pytest.mark.gpu

REL, ABS_RMS = 2.0 ** -9, 1e-3


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mx.load()
    return torch.device("cuda:0")


def _chain_layers(M):
    # a small stand-in for qkv / o / gate_up / down: different N, K, 8-bit mixes
    return [wl.Linear(f"chain_a_M{M}", M, 640, 512, ((0, 512, 26), (512, 640, 91)), 4),
            wl.Linear(f"chain_b_M{M}", M, 512, 512, ((0, 512, 26),), 4),
            wl.Linear(f"chain_c_M{M}", M, 1536, 512, ((0, 1536, 77),), 4),
            wl.Linear(f"chain_d_M{M}", M, 512, 768, ((0, 512, 276),), 4)]


@pytest.mark.parametrize("M", [9, 200])
def test_graph_replay_equals_eager_and_single_calls(dev, M):
    layers = _chain_layers(M)
    packed = [mx.pack_weights(torch.from_numpy(wl.make_w(l, 31)).to(dev), torch.from_numpy(wl.make_bitmap(l, 31)).to(dev))
              for l in layers]
    chain = LinearChain(packed, M, dev)
    for l, x in zip(layers, chain.inputs):
        x.copy_(torch.from_numpy(wl.make_x(l, 32)))
    chain.run()
    torch.cuda.synchronize()
    eager = [y.clone() for y in chain.outputs]
    # the single-layer path on the same inputs
    for l, p, x, y in zip(layers, packed, chain.inputs, eager):
        ref = mx.linear(x, p)
        assert torch.equal(ref.view(torch.int16), y.view(torch.int16)), l.name
    for y in chain.outputs:
        y.fill_(float("nan"))
    chain.capture()
    for _ in range(3):
        chain.replay()
    torch.cuda.synchronize()
    mx.sync_status()
    for l, y, e in zip(layers, chain.outputs, eager):
        assert torch.equal(y.view(torch.int16), e.view(torch.int16)), l.name
    # new inputs flow through the same graph
    for l, x in zip(layers, chain.inputs):
        x.copy_(torch.from_numpy(wl.make_x(l, 33)))
    chain.replay()
    torch.cuda.synchronize()
    for l, p, x, y in zip(layers, packed, chain.inputs, chain.outputs):
        ref = mx.linear(x, p)
        assert torch.equal(ref.view(torch.int16), y.view(torch.int16)), l.name
    # and every linear of the replayed chain against the oracle on its inputs
    for l, x, y in zip(layers, chain.inputs, chain.outputs):
        X = x.cpu().numpy()
        A_o, s_o = oracle.quantize_act(X)
        Y_o = oracle.gemm_w4w8a8(A_o, s_o, oracle.Quantized(wl.make_w(l, 31), wl.make_bitmap(l, 31))).astype(np.float64)
        rms = float(np.sqrt(np.mean(Y_o ** 2)))
        err = np.abs(y.cpu().numpy().astype(np.float64) - Y_o)
        assert (err <= REL * np.abs(Y_o) + ABS_RMS * rms).all(), l.name
    chain.release()
    assert chain.ops() == sum(2 * M * l.N * l.K for l in layers)
