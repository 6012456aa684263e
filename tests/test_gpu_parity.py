"""Parity of the CUDA path (through the C ABI) with the CPU oracle.  GPU only.

Bit-exact: A_q, s_a, every packed weight buffer, and the per-group int32
partials (debug path of the fused kernel).  Y within
|dY| <= 2^-9 * |y_oracle| + 1e-3 * rms(y_oracle), per element.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mixed_precision_quantized_act_b200 as mx  # noqa: E402
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


def gpu_layer(dev, X, W, is8):
    Xd = torch.from_numpy(X).to(dev)
    A_q, s_a = mx.quantize_act(Xd)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    Y = mx.gemm_w4w8a8(A_q, s_a, p)
    mx.sync_status()
    return A_q, s_a, p, Y


def layer_inputs(layer, seed=0):
    return wl.make_x(layer, seed), wl.make_w(layer, seed), wl.make_bitmap(layer, seed)


SMALL = [
    wl.TINY,
    wl.Linear("tiny_p0", 16, 512, 512, ((0, 512, 0),), 4),
    wl.Linear("tiny_p100", 16, 512, 512, ((0, 512, 512),), 4),
    wl.Linear("ragged_m1", 1, 300, 384, ((0, 300, 37),), 3),
    wl.Linear("ragged_m3", 3, 77, 128, ((0, 77, 9),), 2),
    wl.Linear("ragged_m200", 200, 1000, 768, ((0, 1000, 101),), 8),
    wl.Linear("tiles_m257", 257, 1280, 1024, ((0, 1280, 130),), 10),
    wl.Linear("one_8bit_channel", 130, 260, 256, ((0, 260, 1),), 3),
    wl.Linear("tiny_n", 5, 8, 256, ((0, 8, 3),), 2),
]


# ---------------------------------------------------------------- activations

@pytest.mark.parametrize("layer", SMALL + [wl.Q_PROJ_P10], ids=lambda l: l.name)
def test_quantize_act_bit_exact(dev, layer):
    X = wl.make_x(layer, 3)
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    A_ref, s_ref = oracle.quantize_act(X)
    assert np.array_equal(A_q.cpu().numpy(), A_ref)
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantize_act_special_values(dev):
    X = np.zeros((6, 384), np.float16)
    X[0, 0] = 127.0
    X[0, 1:9] = [2.5, 3.5, -2.5, 0.5, 1.5, -1.5, 126.5, -0.5]          # ties
    X[1, :128] = np.float16(65504.0)                                   # fp16 max
    X[1, 5] = np.float16(-65504.0)
    X[2, :128] = np.float16(6e-8)                                      # subnormal group
    X[2, 128:256] = np.linspace(-1e-4, 1e-4, 128).astype(np.float16)
    X[3] = np.linspace(-7, 7, 384).astype(np.float16)
    # row 4 all zero, row 5 one nonzero
    X[5, 300] = -3.0
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    A_ref, s_ref = oracle.quantize_act(X)
    assert np.array_equal(A_q.cpu().numpy(), A_ref)
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def _tie_groups():
    """Groups whose scale is known exactly (amax = 127 * s0 with 127 * s0
    fp16-valued, so s_a = s0), filled with the exact half-integer multiples
    (k + 1/2) * s0 that fp16 holds and with their fp16 neighbours on both sides:
    rounding ties and the values that must not be taken for ties."""
    rows = []
    for s0 in (2.0 ** -4, 3.0 / 256, 5.0 * 2 ** -10, 0.75, 1.5, 192.0, 2.0 ** -20):
        top = np.float16(127 * s0)
        assert float(top) == 127 * s0
        ties = []
        for k in range(-127, 127):
            v = np.float16((k + 0.5) * s0)
            if float(v) == (k + 0.5) * s0 and abs(float(v)) < 127 * s0:
                ties.append(v)
        ties = np.array(ties, np.float16)
        up = np.nextafter(ties, np.float16(np.inf))
        dn = np.nextafter(ties, np.float16(-np.inf))
        pool = np.concatenate([ties, up, dn])
        pool = pool[np.abs(pool.astype(np.float64)) < 127 * s0]
        for start in range(0, len(pool), 127):
            g = np.zeros(128, np.float16)
            g[0] = top if start % 2 == 0 else -top
            chunk = pool[start:start + 127]
            g[1:1 + len(chunk)] = chunk
            rows.append(g)
    G = 4
    rows += [np.zeros(128, np.float16)] * ((-len(rows)) % G)
    return np.stack(rows).reshape(-1, 128 * G)


def test_quantize_act_ties_and_near_ties(dev):
    X = _tie_groups()
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    A_ref, s_ref = oracle.quantize_act(X)
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(A_q.cpu().numpy(), A_ref)


def test_quantize_act_wide_magnitudes(dev):
    # every group at its own scale, from fp16 subnormals to near the fp16 maximum
    rng = np.random.default_rng(17)
    M, K = 256, 2048
    scale = np.exp2(rng.uniform(-24, 15, size=(M, K // 128, 1)))
    X = (rng.standard_normal((M, K // 128, 128)) * scale).clip(-65504, 65504).astype(np.float16).reshape(M, K)
    A_q, s_a = mx.quantize_act(torch.from_numpy(X).to(dev))
    A_ref, s_ref = oracle.quantize_act(X)
    assert np.array_equal(s_a.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(A_q.cpu().numpy(), A_ref)


def test_quantize_act_empty(dev):
    A_q, s_a = mx.quantize_act(torch.zeros((0, 256), dtype=torch.float16, device=dev))
    mx.sync_status()
    assert A_q.shape == (0, 256) and s_a.shape == (0, 2)


# ---------------------------------------------------------------- weight pack

@pytest.mark.parametrize("layer", SMALL + [wl.Q_PROJ_P10], ids=lambda l: l.name)
def test_pack_bit_exact(dev, layer):
    W, is8 = wl.make_w(layer, 4), wl.make_bitmap(layer, 4)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ref = oracle.packed(oracle.Quantized(W, is8))
    got = {"W4": p.W4, "z4": p.z4, "s_w4": p.s_w4, "idx4": p.idx4, "W8": p.W8, "s_w8": p.s_w8, "idx8": p.idx8}
    for k, v in got.items():
        a = v.cpu().numpy()
        b = ref[k]
        assert a.shape == b.shape, k
        assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)), k


def test_pack_special_groups(dev):
    K = 384
    W = np.random.default_rng(9).standard_normal((6, K)).astype(np.float32) * 0.02
    W[0, :128] = 0.0                      # all-zero group
    W[1, :128] = np.abs(W[1, :128])       # all-positive group -> z = 0
    W[2, 128:256] = -np.abs(W[2, 128:256])
    W[3, :] = 1e-3                        # constant
    W[4, 256:] = 3e4                      # large
    is8 = np.array([0, 0, 0, 1, 0, 1], np.uint8)
    p = mx.pack_weights(torch.from_numpy(W).to(dev), torch.from_numpy(is8).to(dev))
    ref = oracle.packed(oracle.Quantized(W, is8))
    for k in ("W4", "z4", "s_w4", "W8", "s_w8"):
        a = getattr(p, k).cpu().numpy()
        assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(ref[k]).view(np.uint8)), k


def test_pack_rejects_a_bit_map_that_disagrees_with_n8(dev):
    import ctypes
    from mixed_precision_quantized_act_b200 import _lib
    W = torch.zeros((64, 256), dtype=torch.float32, device=dev)
    is8 = torch.zeros(64, dtype=torch.uint8, device=dev)
    is8[:5] = 1
    p = _lib.empty_packed(64, 256, 4, dev)  # claims 4, the map holds 5
    L = _lib.load()
    st = L.mixllm_pack_weights(W.data_ptr(), 64, 256, is8.data_ptr(), 4, 128, p.W4.data_ptr(),
                               p.z4.data_ptr(), p.s_w4.data_ptr(), p.idx4.data_ptr(), p.W8.data_ptr(),
                               p.s_w8.data_ptr(), p.idx8.data_ptr(), ctypes.c_void_p(0))
    assert st == _lib.ERR_INVALID_ARG
    mx.sync_status()  # the status word was cleared; the context is fine


# ---------------------------------------------------------------- the GEMM

@pytest.mark.parametrize("layer", SMALL, ids=lambda l: l.name)
def test_partials_bit_exact(dev, layer):
    X, W, is8 = layer_inputs(layer, 5)
    A_q, s_a, p, _ = gpu_layer(dev, X, W, is8)
    P = mx.gemm_debug_partials(A_q, s_a, p)
    mx.sync_status()
    A_ref, _ = oracle.quantize_act(X)
    P_ref = oracle.group_partials(A_ref, oracle.Quantized(W, is8))
    assert np.array_equal(P.cpu().numpy(), P_ref)


@pytest.mark.parametrize("layer", SMALL, ids=lambda l: l.name)
def test_y_matches_oracle(dev, layer):
    X, W, is8 = layer_inputs(layer, 6)
    A_q, s_a, p, Y = gpu_layer(dev, X, W, is8)
    A_ref, s_ref = oracle.quantize_act(X)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W, is8))
    assert_y_close(Y.cpu().numpy(), Y_ref, layer.name)


def test_y_deterministic(dev):
    X, W, is8 = layer_inputs(wl.Q_PROJ_P10, 0)
    A_q, s_a, p, Y1 = gpu_layer(dev, X, W, is8)
    Y2 = mx.gemm_w4w8a8(A_q, s_a, p)
    Y3 = mx.linear(torch.from_numpy(X).to(dev), p)
    mx.sync_status()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(Y1.view(torch.int16), Y3.view(torch.int16))


def _sample_rows(M):
    rows = sorted(set([0, 1, M // 2, M - 1] + list(range(120, min(M, 136)))))
    return np.array([r for r in rows if r < M])


# the workloads whose sizes the benchmark and the sweeps use
FULL = ([wl.Q_PROJ_P10] + [wl.Q_PROJ_P10.with_m(m) for m in wl.M_SWEEP] + list(wl.BIT_MIX)
        + list(wl.LLAMA8B_LAYER) + list(wl.LLAMA70B))


@pytest.mark.parametrize("layer", FULL, ids=lambda l: l.name)
def test_full_size_sampled_rows(dev, layer):
    """Full-size launch; the oracle checks sampled rows (spanning the first,
    middle, last and two neighbouring M tiles) against every output column,
    or a random subset of 3072 columns for the widest layers."""
    X, W, is8 = layer_inputs(layer, 0)
    A_q, s_a, p, Y = gpu_layer(dev, X, W, is8)
    rows = _sample_rows(layer.M)
    A_ref, s_ref = oracle.quantize_act(X[rows])
    # activations: sampled rows bit-exact
    assert np.array_equal(A_q[torch.from_numpy(rows).to(dev)].cpu().numpy(), A_ref)
    assert np.array_equal(s_a[torch.from_numpy(rows).to(dev)].cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    if layer.N > 8192:
        cols = np.sort(np.random.default_rng(1).choice(layer.N, 3072, replace=False))
    else:
        cols = np.arange(layer.N)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W[cols], is8[cols]))
    Yg = Y[torch.from_numpy(rows).to(dev)].cpu().numpy()[:, cols]
    assert_y_close(Yg, Y_ref, layer.name)
    # property at every position: finite and within the bound of the inputs
    assert torch.isfinite(Y).all()


# full-size launches of the partials debug path: the headline shape (G = 32)
# and one shape of each larger workload family (long K, a bit mix, multi-wave)
FULL_P = [wl.Q_PROJ_P10, wl.LLAMA8B_LAYER[3], [l for l in wl.BIT_MIX if "p50" in l.name][0], wl.LLAMA70B[1]]


@pytest.mark.parametrize("layer", FULL_P, ids=lambda l: l.name)
def test_full_size_partials_sampled(dev, layer):
    """The int32 group partials of a full-size launch, bit-exact on sampled
    token rows (first, middle and last M tiles and an M-tile boundary) x
    sampled output columns from both channel sets."""
    X, W, is8 = layer_inputs(layer, 4)
    A_q, s_a, p, _ = gpu_layer(dev, X, W, is8)
    P = mx.gemm_debug_partials(A_q, s_a, p)
    mx.sync_status()
    assert P.shape == (layer.M, layer.N, layer.K // 128)
    rows = np.array(sorted(set([0, 127, 128, layer.M // 2, layer.M - 1])))
    rng = np.random.default_rng(7)
    c8 = np.flatnonzero(is8)
    c4 = np.flatnonzero(is8 == 0)
    cols = np.sort(np.concatenate([rng.choice(c4, min(384, c4.size), replace=False),
                                   rng.choice(c8, min(128, c8.size), replace=False),
                                   [0, layer.N - 1]])).astype(np.int64)
    cols = np.unique(cols)
    A_ref, _ = oracle.quantize_act(X[rows])
    P_ref = oracle.group_partials(A_ref, oracle.Quantized(W[cols], is8[cols]))
    Pg = P[torch.from_numpy(rows).to(dev)][:, torch.from_numpy(cols).to(dev)].cpu().numpy()
    assert np.array_equal(Pg, P_ref)
    del P


def _extreme_layer(dev, M, K, n4, n8, w_mag, seed):
    """Weights whose every group is constant (+w_mag or -w_mag per channel and
    group) and activations of +-1 per (token, group): every 4-bit product is
    (q - z) * a = +-15 * 127 and every 8-bit one +-127 * 127, so each group
    partial reaches the bound of its set, +-243840 or +-2064512."""
    rng = np.random.default_rng(seed)
    G = K // 128
    N = n4 + n8
    sw = rng.choice([-1.0, 1.0], size=(N, G)).astype(np.float32)
    W = np.repeat(sw, 128, axis=1) * np.float32(w_mag)
    sx = rng.choice([-1.0, 1.0], size=(M, G)).astype(np.float16)
    X = np.repeat(sx, 128, axis=1)
    is8 = np.zeros(N, np.uint8)
    is8[rng.choice(N, n8, replace=False)] = 1
    return X, W, is8


def test_partials_reach_the_bounds_of_both_sets(dev):
    M, K, n4, n8 = 130, 512, 200, 60
    X, W, is8 = _extreme_layer(dev, M, K, n4, n8, 0.5, 11)
    A_q, s_a, p, Y = gpu_layer(dev, X, W, is8)
    P = mx.gemm_debug_partials(A_q, s_a, p).cpu().numpy()
    mx.sync_status()
    A_ref, s_ref = oracle.quantize_act(X)
    P_ref = oracle.group_partials(A_ref, oracle.Quantized(W, is8))
    assert np.array_equal(P, P_ref)
    mag = np.abs(P)
    assert (mag[:, is8 == 0] == 15 * 127 * 128).all()
    assert (mag[:, is8 == 1] == 127 * 127 * 128).all()
    assert (P == 243840).any() and (P == -243840).any()
    assert (P == 2064512).any() and (P == -2064512).any()
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W, is8))
    assert_y_close(Y.cpu().numpy(), Y_ref, "extreme partials")


def test_y_overflow_to_inf_matches_oracle(dev):
    """Large weights drive some outputs past the fp16 range: those are +-inf
    on both sides (same sign), and the rest stay within the tolerance."""
    M, K, n4, n8 = 64, 1024, 160, 40
    X, W, is8 = _extreme_layer(dev, M, K, n4, n8, 100.0, 12)
    # one channel in each set with small weights: finite, mixed with the inf ones
    W[np.flatnonzero(is8 == 0)[0]] *= np.float32(1e-3)
    W[np.flatnonzero(is8 == 1)[0]] *= np.float32(1e-3)
    A_q, s_a, p, Y = gpu_layer(dev, X, W, is8)
    A_ref, s_ref = oracle.quantize_act(X)
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W, is8)).astype(np.float64)
    Yg = Y.cpu().numpy().astype(np.float64)
    inf_ref = np.isinf(Y_ref)
    assert inf_ref.any() and (~inf_ref).any()
    assert np.array_equal(np.isinf(Yg), inf_ref)
    assert np.array_equal(np.sign(Yg[inf_ref]), np.sign(Y_ref[inf_ref]))
    assert not np.isnan(Yg).any()
    fin = ~inf_ref
    rms = float(np.sqrt(np.mean(Y_ref[fin] ** 2)))
    err = np.abs(Yg[fin] - Y_ref[fin])
    assert (err <= REL * np.abs(Y_ref[fin]) + ABS_RMS * rms).all()


@pytest.mark.parametrize("layer", [wl.TINY, SMALL[6], wl.Q_PROJ_P10], ids=lambda l: l.name)
def test_plain_i2f_ablation_gives_the_same_bytes(dev, layer):
    """The plain int->float convert and the bias trick both round P*s_w once,
    so the two forms of the tiled kernel write bit-identical Y."""
    X, W, is8 = layer_inputs(layer, 8)
    A_q, s_a, p, Y = gpu_layer(dev, X, W, is8)
    Y2 = torch.full_like(Y, float("nan"))
    mx.gemm_w4w8a8_plain_i2f_into(A_q, s_a, p, Y2)
    mx.sync_status()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_hang_guard_reports_timeout_and_context_survives(dev):
    from mixed_precision_quantized_act_b200 import _lib
    mx.sync_status()
    mx.selftest_wait_timeout(2000)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.sync_status()
    assert ei.value.status == _lib.ERR_TIMEOUT
    # the context is usable and the status word was cleared
    X, W, is8 = layer_inputs(wl.TINY, 0)
    _, _, _, Y = gpu_layer(dev, X, W, is8)
    assert torch.isfinite(Y).all()


def test_back_to_back_multiwave_launches_are_identical(dev):
    """Many launches of a multi-wave grid (464 tiles, 64 groups each) in a row:
    every output must be bit-identical to the first and match the oracle on
    sampled rows.  Guards the inter-warp barrier protocol against rare races."""
    layer = wl.LLAMA70B[1]  # o_proj: M=1024, N=8192, K=8192
    X, W, is8 = layer_inputs(layer, 3)
    A_q, s_a, p, Y0 = gpu_layer(dev, X, W, is8)
    ref = Y0.view(torch.int16).clone()
    Y = torch.empty_like(Y0)
    for i in range(60):
        mx.gemm_w4w8a8_into(A_q, s_a, p, Y)
        if i % 20 == 19:
            torch.cuda.synchronize()
            assert torch.equal(Y.view(torch.int16), ref), f"launch {i} differs"
    mx.sync_status()
    rows = np.array([0, 511, 1023])
    A_ref, s_ref = oracle.quantize_act(X[rows])
    cols = np.sort(np.random.default_rng(2).choice(layer.N, 1024, replace=False))
    Y_ref = oracle.gemm_w4w8a8(A_ref, s_ref, oracle.Quantized(W[cols], is8[cols]))
    assert_y_close(Y0[torch.from_numpy(rows).to(dev)].cpu().numpy()[:, cols], Y_ref, layer.name)
