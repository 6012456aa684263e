"""The layer from fp16 activations for more than 64 tokens: mixllm_linear
(the quantizer into the workspace, then the tiled GEMM) and
mixllm_linear_one_launch (the tiled GEMM quantizes X itself: every CTA an
even share of the (token, group) pairs into the workspace, published through
a counter there, then the two-step GEMM in the same launch).  Either way the
codes, scales and Y must be bit-identical to quantize_act followed by
mixllm_gemm_w4w8a8 (the same quantizer arithmetic, the same kernel
arithmetic), Y within the layer's tolerance of the CPU oracle, and the
workspace counters back at zero after every call.  GPU only.
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


def _r256(b):
    return (b + 255) // 256 * 256


def _parts(ws, M, K):
    """The workspace's A_q [M, K], s_a [M, G] (as uint32) and two counters."""
    G = K // 128
    aq, sa = _r256(M * K), _r256(M * G * 4)
    A = ws[: M * K].view(M, K).view(torch.int8)
    S = ws[aq: aq + M * G * 4].view(torch.int32).view(M, G)
    C = ws[aq + sa: aq + sa + 8].view(torch.int32)
    return A, S, C


# (layer, one launch possible?): the one-launch form takes K / 128 a multiple of 4
CASES = [
    (wl.Q_PROJ_P10, True),
    (_layer("lt_m65", 65, 640, 512, 70), True),              # the fewest tokens the tiled path takes
    (_layer("lt_m200_ragged", 200, 1000, 1024, 101), True),  # ragged token and channel tiles
    (_layer("lt_p0", 256, 512, 512, 0), True),               # 4-bit set only
    (_layer("lt_p100", 256, 512, 512, 512), True),           # 8-bit set only
    (_layer("lt_one8", 130, 260, 512, 1), True),
    (_layer("lt_multiwave", 1024, 8192, 1024, 819), True),   # 512 tiles on a persistent grid
    (wl.LLAMA8B_LAYER[3], True),                             # down projection, K = 14336
    (_layer("lt_k384", 130, 260, 384, 13), False),           # G = 3: two launches only
]


@pytest.mark.parametrize("one_launch", [False, True], ids=["two_launches", "one_launch"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0].name)
def test_linear_matches_two_calls_and_oracle(dev, case, one_launch):
    layer, one_ok = case
    X, W, is8 = wl.make_x(layer, 41), wl.make_w(layer, 41), wl.make_bitmap(layer, 41)
    Xd = torch.from_numpy(X).to(dev)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.linear_workspace(layer.M, p, dev)
    G = layer.K // 128
    assert ws.numel() >= _r256(layer.M * layer.K) + _r256(layer.M * G * 4) + 8
    Y = torch.full((layer.M, layer.N), float("nan"), dtype=torch.float16, device=dev)
    if one_launch and not one_ok:
        with pytest.raises(_lib.MixLLMError) as ei:
            mx.linear_into(Xd, p, Y, ws, one_launch=True)
        assert ei.value.status == _lib.ERR_UNSUPPORTED
        return
    mx.linear_into(Xd, p, Y, ws, one_launch=one_launch)
    Y2 = torch.full_like(Y, float("nan"))
    mx.linear_into(Xd, p, Y2, ws, one_launch=one_launch)  # again, on the same workspace
    A_q, s_a = mx.quantize_act(Xd)
    Y_ref = mx.gemm_w4w8a8(A_q, s_a, p)
    mx.sync_status()
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
    assert torch.equal(Y2.view(torch.int16), Y_ref.view(torch.int16))
    A_w, S_w, C_w = _parts(ws, layer.M, layer.K)
    assert torch.equal(A_w, A_q), "the codes the GEMM wrote differ from the quantizer's"
    assert torch.equal(S_w, s_a.view(torch.int32)), "the scales the GEMM wrote differ from the quantizer's"
    assert C_w.tolist() == [0, 0], "the counters must be back at zero"

    # the oracle on sampled rows (first, middle, last token tiles and a tile
    # boundary) x all columns, or 3072 random columns of the widest layers
    rows = np.array(sorted({r for r in [0, 1, 63, 64, 127, 128, 129, layer.M // 2, layer.M - 1] if r < layer.M}))
    cols = np.arange(layer.N) if layer.N <= 8192 else np.sort(np.random.default_rng(7).choice(layer.N, 3072, replace=False))
    A_o, s_o = oracle.quantize_act(X[rows])
    assert np.array_equal(A_w.cpu().numpy()[rows], A_o)
    assert np.array_equal(S_w.cpu().numpy()[rows].view(np.uint32), s_o.view(np.uint32))
    Y_o = oracle.gemm_w4w8a8(A_o, s_o, oracle.Quantized(W[cols], is8[cols])).astype(np.float64)
    rms = float(np.sqrt(np.mean(Y_o ** 2)))
    err = np.abs(Y.cpu().numpy()[rows][:, cols].astype(np.float64) - Y_o)
    assert (err <= REL * np.abs(Y_o) + ABS_RMS * rms).all()
    assert torch.isfinite(Y).all()


def test_linear_new_inputs_on_a_used_workspace(dev):
    """A second call with other activations on the same workspace sees only
    its own codes: the counters the first call left at zero gate the loads."""
    layer = _layer("lt_reuse", 384, 1536, 1024, 150)
    W, is8 = wl.make_w(layer, 3), wl.make_bitmap(layer, 3)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.linear_workspace(layer.M, p, dev)
    for seed in (5, 6, 7):
        Xd = torch.from_numpy(wl.make_x(layer, seed)).to(dev)
        Y = torch.empty((layer.M, layer.N), dtype=torch.float16, device=dev)
        mx.linear_into(Xd, p, Y, ws, one_launch=True)
        A_q, s_a = mx.quantize_act(Xd)
        Y_ref = mx.gemm_w4w8a8(A_q, s_a, p)
        mx.sync_status()
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), seed
    assert _parts(ws, layer.M, layer.K)[2].tolist() == [0, 0]


def test_linear_in_a_cuda_graph(dev):
    """Three layer calls on one workspace (one launch, two launches, one
    launch) captured in a CUDA graph and replayed twice: every one-launch call
    finds the counters at zero, as the previous left them."""
    layer = _layer("lt_graph", 512, 2048, 1024, 200)
    W, is8 = wl.make_w(layer, 8), wl.make_bitmap(layer, 8)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    Xs = [torch.from_numpy(wl.make_x(layer, s)).to(dev) for s in (11, 12, 13)]
    ws = mx.linear_workspace(layer.M, p, dev)
    Ys = [torch.empty((layer.M, layer.N), dtype=torch.float16, device=dev) for _ in Xs]
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        mx.linear_into(Xs[0], p, Ys[0], ws, st, one_launch=True)  # warm-up outside the capture
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            for X, Y in zip(Xs, Ys):
                mx.linear_into(X, p, Y, ws, st, one_launch=(X is not Xs[1]))
    refs = []
    for X in Xs:
        A_q, s_a = mx.quantize_act(X)
        refs.append(mx.gemm_w4w8a8(A_q, s_a, p))
    for _ in range(2):
        for Y in Ys:
            Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        mx.sync_status()
        for Y, R in zip(Ys, refs):
            assert torch.equal(Y.view(torch.int16), R.view(torch.int16))
    assert _parts(ws, layer.M, layer.K)[2].tolist() == [0, 0]
    del g


def test_linear_workspace_validation(dev):
    layer = _layer("lt_val", 130, 260, 512, 13)
    X, W, is8 = wl.make_x(layer, 1), wl.make_w(layer, 1), wl.make_bitmap(layer, 1)
    Xd = torch.from_numpy(X).to(dev)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ws = mx.linear_workspace(layer.M, p, dev)
    Y = torch.empty((layer.M, layer.N), dtype=torch.float16, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.linear_into(Xd, p, Y, ws[: ws.numel() - 256])
    assert ei.value.status == _lib.ERR_INVALID_ARG
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.linear_into(Xd[:64].contiguous(), p, Y[:64], ws, one_launch=True)  # few tokens: not this form
    assert ei.value.status == _lib.ERR_INVALID_ARG
    big = torch.zeros(ws.numel() + 256, dtype=torch.uint8, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.linear_into(Xd, p, Y, big[16: 16 + ws.numel()])  # large enough, not 256-byte aligned
    assert ei.value.status == _lib.ERR_INVALID_ARG
    mx.linear_into(Xd, p, Y, ws)
    mx.sync_status()
