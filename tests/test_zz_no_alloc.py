"""The no-allocation few-token entry point (mixllm_gemm_w4w8a8_small_m_noalloc,
static device scratch) against the workspace entry point it mirrors.  GPU only;
collected last so that it runs after the other GPU tests in one process.
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


def _case(dev, layer, seed):
    X, W, is8 = wl.make_x(layer, seed), wl.make_w(layer, seed), wl.make_bitmap(layer, seed)
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    return X, W, is8, A_q, s_a, p


@pytest.mark.parametrize("layer", [wl.Q_PROJ_P10.with_m(1), wl.Q_PROJ_P10.with_m(64),
                                   wl.Linear("na_m9_ragged", 9, 300, 384, ((0, 300, 37),), 3),
                                   wl.Linear("na_m2_one_group", 2, 260, 128, ((0, 260, 5),), 2)],
                         ids=lambda l: l.name)
def test_no_alloc_matches_the_workspace_entry_point_twice_in_a_row(dev, layer):
    X, W, is8, A_q, s_a, p = _case(dev, layer, 21)
    ws = mx.small_m_workspace(layer.M, p, dev)
    Y_ref = mx.gemm_w4w8a8_small_m(A_q, s_a, p, ws)
    Y1 = torch.full_like(Y_ref, float("nan"))
    Y2 = torch.full_like(Y_ref, float("nan"))
    mx.gemm_w4w8a8_small_m_noalloc_into(A_q, s_a, p, Y1)
    mx.gemm_w4w8a8_small_m_noalloc_into(A_q, s_a, p, Y2)
    mx.sync_status()
    assert torch.equal(Y1.view(torch.int16), Y_ref.view(torch.int16))
    assert torch.equal(Y2.view(torch.int16), Y_ref.view(torch.int16))
    # and the layer itself, against the oracle
    A_o, s_o = oracle.quantize_act(X)
    Y_o = oracle.gemm_w4w8a8(A_o, s_o, oracle.Quantized(W, is8)).astype(np.float64)
    rms = float(np.sqrt(np.mean(Y_o ** 2)))
    err = np.abs(Y1.cpu().numpy().astype(np.float64) - Y_o)
    assert (err <= REL * np.abs(Y_o) + ABS_RMS * rms).all()


def test_no_alloc_runs_the_persistent_gemv_on_a_large_layer(dev):
    # 70B gate_up at one token: the plan picks the persistent GEMV, whose
    # scratch (unit partials + counters) must also come from the static array
    layer = wl.LLAMA70B[2].with_m(1)
    assert mx.small_m_kernel(1, layer.K, layer.N - layer.N8, layer.N8) == "GEMV persistent"
    g = torch.Generator(device="cpu").manual_seed(5)
    X = (torch.randn((1, layer.K), generator=g) * 0.5).to(torch.float16).to(dev)
    W = (torch.randn((layer.N, layer.K), generator=g) * 0.02).to(dev)
    is8 = torch.from_numpy(wl.make_bitmap(layer, 5)).to(dev)
    A_q, s_a = mx.quantize_act(X)
    p = mx.pack_weights(W, is8)
    del W
    ws = mx.small_m_workspace(1, p, dev)
    Y_ref = mx.gemm_w4w8a8_small_m(A_q, s_a, p, ws)
    for _ in range(2):
        Y = torch.full_like(Y_ref, float("nan"))
        mx.gemm_w4w8a8_small_m_noalloc_into(A_q, s_a, p, Y)
        mx.sync_status()
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))


def test_no_alloc_rejects_a_shape_larger_than_its_scratch(dev):
    # 70B down at M=64: 7 splits x 65 tiles x 64 x 128 fp32 partials = 14.9 MB > 8 MiB
    layer = wl.LLAMA70B[3]
    p = mx.empty_packed(layer.N, layer.K, layer.N8, dev)
    need = mx.small_m_workspace_bytes(64, layer.K, p.N4, p.N8)
    assert need > 8 << 20
    A_q = torch.zeros((64, layer.K), dtype=torch.int8, device=dev)
    s_a = torch.zeros((64, layer.K // 128), dtype=torch.float32, device=dev)
    Y = torch.empty((64, layer.N), dtype=torch.float16, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.gemm_w4w8a8_small_m_noalloc_into(A_q, s_a, p, Y)
    assert ei.value.status == _lib.ERR_UNSUPPORTED
    mx.sync_status()
