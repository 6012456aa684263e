"""Parity of the few-token GEMM (mixllm_gemm_w4w8a8_small_m, M <= 64) with the
CPU oracle.  GPU only.

Y within |dY| <= 2^-9 * |y_oracle| + 1e-3 * rms(y_oracle), per element; the
split-K reduction adds the splits in a fixed order, so repeated calls are
bit-identical, and every call returns the workspace's tile counters to zero.
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


def assert_y_close(Y, Y_ref, what=""):
    Y = np.asarray(Y, np.float64)
    Y_ref = np.asarray(Y_ref, np.float64)
    assert Y.shape == Y_ref.shape
    rms = float(np.sqrt(np.mean(Y_ref ** 2))) if Y_ref.size else 0.0
    err = np.abs(Y - Y_ref)
    bad = err > REL * np.abs(Y_ref) + ABS_RMS * rms
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {Y.size} outside tolerance, "
                           f"max excess {float(np.max(err - REL * np.abs(Y_ref) - ABS_RMS * rms)):.3g}")


def _layer(name, M, N, K, n8, outliers=4):
    return wl.Linear(name, M, N, K, ((0, N, n8),), outliers)


# GEMV (M <= 8: token bounds 1 / 2 / 4 / 8) and tensor-core kernel (token
# tiles 16 / 32 / 64) on either side of M = 8, ragged N, one set empty (on
# both kernels), one 8-bit channel, split counts from 1 (wide N) to the
# group cap (long K)
CASES = [
    wl.Q_PROJ_P10.with_m(1),
    wl.Q_PROJ_P10.with_m(2),
    wl.Q_PROJ_P10.with_m(8),
    wl.Q_PROJ_P10.with_m(9),
    wl.Q_PROJ_P10.with_m(16),
    wl.Q_PROJ_P10.with_m(64),
    _layer("sm_m5_ragged", 5, 300, 384, 37),
    _layer("sm_m17", 17, 1000, 1024, 101),
    _layer("sm_m33", 33, 640, 1024, 64),
    _layer("sm_m7_p0", 7, 512, 512, 0),
    _layer("sm_m7_p100", 7, 512, 512, 512),
    _layer("sm_m16_p0", 16, 384, 640, 0),
    _layer("sm_m40_p100", 40, 384, 512, 384),
    _layer("sm_m2_one_8bit", 2, 260, 256, 1),
    _layer("sm_m3_k128", 3, 384, 128, 40),
    _layer("sm_m1_k8960", 1, 200, 8960, 30),
    _layer("sm_m4_g33", 4, 640, 33 * 128, 70),
]


def counters_zero(ws, p, M, K):
    need = mx.small_m_workspace_bytes(M, K, p.N4, p.N8)
    tiles = -(-p.N4 // 128) + -(-p.N8 // 128)
    return need == 0 or not ws[need - 4 * tiles: need].any()


def _run(dev, layer, seed):
    X, W, is8 = wl.make_x(layer, seed), wl.make_w(layer, seed), wl.make_bitmap(layer, seed)
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.small_m_workspace(layer.M, p, dev)
    Y = mx.gemm_w4w8a8_small_m(A_q, s_a, p, ws)
    mx.sync_status()
    return X, W, is8, A_q, s_a, p, ws, Y


@pytest.mark.parametrize("layer", CASES, ids=lambda l: l.name)
def test_small_m_matches_oracle(dev, layer):
    X, W, is8, A_q, s_a, p, ws, Y = _run(dev, layer, 11)
    A_ref, s_ref = oracle.quantize_act(X)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W, is8))
    assert_y_close(Y.cpu().numpy(), Y_ref, layer.name)
    assert counters_zero(ws, p, layer.M, layer.K), "the tile counters must be back at zero"


@pytest.mark.parametrize("layer", [wl.Q_PROJ_P10.with_m(16), _layer("sm_m33", 33, 640, 1024, 64),
                                   wl.Q_PROJ_P10.with_m(1), _layer("sm_m6", 6, 1000, 2048, 100)],
                         ids=lambda l: l.name)
def test_small_m_deterministic_and_close_to_tiled(dev, layer):
    X, W, is8, A_q, s_a, p, ws, Y1 = _run(dev, layer, 12)
    Y2 = torch.empty_like(Y1)
    for _ in range(5):
        mx.gemm_w4w8a8_small_m_into(A_q, s_a, p, Y2, ws)
    Yt = mx.gemm_w4w8a8(A_q, s_a, p)
    mx.sync_status()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert counters_zero(ws, p, layer.M, layer.K)
    # the tiled kernel computes the same layer with another fp32 order
    A_ref, s_ref = oracle.quantize_act(X)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W, is8))
    assert_y_close(Yt.cpu().numpy(), Y_ref, layer.name + " tiled")
    assert_y_close(Y1.cpu().numpy(), Y_ref, layer.name + " small-M")


@pytest.mark.parametrize("layer", [wl.LLAMA8B_LAYER[2].with_m(8), wl.LLAMA70B[3].with_m(4),
                                   wl.LLAMA70B[3].with_m(1), wl.LLAMA70B[2].with_m(3), wl.LLAMA8B_LAYER[3].with_m(2),
                                   wl.LLAMA8B_LAYER[2].with_m(16), wl.LLAMA70B[3].with_m(12)],
                         ids=lambda l: l.name)
def test_small_m_wide_and_long_layers(dev, layer):
    """8B / 70B gate_up (N = 28672 / 57344) and 70B / 8B down (K = 28672 /
    14336): the persistent GEMV, whose CTAs take units of several tiles and
    share tiles with their neighbours (70B down M=1, 70B gate_up M=3), the
    split GEMV (8B gate_up M=8, 70B down M=4, 8B down M=2) and the
    tensor-core kernel (M=16, 12); a random subset of the columns against the
    oracle."""
    X, W, is8, A_q, s_a, p, ws, Y = _run(dev, layer, 13)
    cols = np.sort(np.random.default_rng(3).choice(layer.N, 2048, replace=False))
    A_ref, s_ref = oracle.quantize_act(X)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W[cols], is8[cols]))
    assert_y_close(Y.cpu().numpy()[:, cols], Y_ref, layer.name)
    assert torch.isfinite(Y).all()
    assert counters_zero(ws, p, layer.M, layer.K)


def test_small_m_linear_dispatch_and_validation(dev):
    layer = _layer("sm_m5_ragged", 5, 300, 384, 37)
    X, W, is8, A_q, s_a, p, ws, Y = _run(dev, layer, 14)
    Y_lin = mx.linear(torch.from_numpy(X).to(dev), p, workspace=mx.linear_workspace(layer.M, p, dev))
    mx.sync_status()
    assert torch.equal(Y.view(torch.int16), Y_lin.view(torch.int16))
    need = mx.small_m_workspace_bytes(layer.M, layer.K, p.N4, p.N8)
    assert need > 0
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.gemm_w4w8a8_small_m_into(A_q, s_a, p, torch.empty_like(Y), ws[: need - 4])
    assert ei.value.status == _lib.ERR_INVALID_ARG
    X65 = torch.from_numpy(wl.make_x(layer.with_m(65), 1)).to(dev)
    A65, s65 = mx.quantize_act(X65)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.gemm_w4w8a8_small_m(A65, s65, p, ws)
    assert ei.value.status == _lib.ERR_INVALID_ARG
    mx.sync_status()


# Every few-token kernel on shapes of its own range and on shapes the plan
# would give to another kernel: exact int32 group partials and Y of the
# kernel that ran.  (kind, layer): token bounds 1 / 2 / 4 / 8 of the GEMVs,
# 16 / 32 / 64 of the tensor-core kernel, ragged N, multiple splits, both sets.
DEBUG_CASES = [
    ("GEMV split-K", _layer("dbg_gs_m1", 1, 300, 384, 37)),
    ("GEMV split-K", _layer("dbg_gs_m3", 3, 1000, 2048, 101)),
    ("GEMV split-K", _layer("dbg_gs_m8", 8, 640, 4096, 64)),
    ("GEMV split-K", wl.Q_PROJ_P10.with_m(2)),
    ("GEMV persistent", _layer("dbg_gp_m1", 1, 1000, 2048, 101)),
    ("GEMV persistent", _layer("dbg_gp_m2", 2, 300, 1024, 37)),
    ("GEMV persistent", _layer("dbg_gp_m4", 4, 640, 8192, 64)),
    ("tensor-core split-K", _layer("dbg_tc_m1", 1, 300, 384, 37)),
    ("tensor-core split-K", _layer("dbg_tc_m9", 9, 1000, 1024, 101)),
    ("tensor-core split-K", _layer("dbg_tc_m32", 32, 640, 2048, 64)),
    ("tensor-core split-K", _layer("dbg_tc_m64_p0", 64, 512, 512, 0)),
    ("tensor-core split-K", wl.Q_PROJ_P10.with_m(40)),
    # 224 tiles of 16 tokens: the two-CTAs-per-SM form
    ("tensor-core split-K", _layer("dbg_tc_m16_wide", 16, 28672, 256, 2800)),
    ("tensor-core split-K", _layer("dbg_tc_m11_wide", 11, 28672, 384, 2800)),
]


@pytest.mark.parametrize("kind,layer", DEBUG_CASES, ids=lambda v: v if isinstance(v, str) else v.name)
def test_small_m_kernel_partials_bit_exact(dev, kind, layer):
    X, W, is8 = wl.make_x(layer, 13), wl.make_w(layer, 13), wl.make_bitmap(layer, 13)
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    Y, P = mx.small_m_debug_partials(A_q, s_a, p, kind)
    mx.sync_status()
    A_ref, s_ref = oracle.quantize_act(X)
    q = oracle.Quantized(W, is8)
    assert np.array_equal(P.cpu().numpy(), oracle.group_partials(A_ref, q))
    assert_y_close(Y.cpu().numpy(), oracle.gemm_w4w8a8(A_ref, s_ref, q), f"{kind} {layer.name}")


def test_small_m_debug_rejects_kernels_outside_their_range(dev):
    layer = _layer("dbg_reject", 9, 256, 512, 16)
    p = mx.empty_packed(layer.N, layer.K, layer.N8, dev)
    A_q = torch.zeros((9, layer.K), dtype=torch.int8, device=dev)
    s_a = torch.zeros((9, layer.K // 128), dtype=torch.float32, device=dev)
    for kind in ("GEMV split-K", "GEMV persistent"):
        with pytest.raises(_lib.MixLLMError) as ei:
            mx.small_m_debug_partials(A_q, s_a, p, kind)
        assert ei.value.status == _lib.ERR_UNSUPPORTED
    # the persistent GEMV keeps every token's codes resident: M*K <= 32768
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.small_m_debug_partials(A_q[:4].repeat(1, 32)[:, :16384].contiguous(),
                                  torch.zeros((4, 128), dtype=torch.float32, device=dev),
                                  mx.empty_packed(256, 16384, 16, dev), "GEMV persistent")
    assert ei.value.status == _lib.ERR_UNSUPPORTED
    mx.sync_status()
