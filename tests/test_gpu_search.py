"""Parity of the global mixed-precision search on the GPU (mixllm_channel_salience,
mixllm_select_top_t) with the CPU oracle.  GPU only.

Salience: fp32 on the GPU, fp64 in the oracle, so per channel
|S_gpu - S| <= mean_d (e_d (1 + |t_d|) + e_d^2) + S (D + 4) 2^-24, with
e_d = 4 (K/256 + 16) 2^-24 sum_k |G[d,n,k] (c_q - c_0)[k]| the rounding bound of
an fp32 dot product in the kernel's order (slices of K/256 products per thread,
then a 256-way tree) plus one rounding of each c_q - c_0.  Selection: an
integer decision from fp32 keys, the same keys on both sides: bit-exact.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import mixed_precision_quantized_act_b200 as mx  # noqa: E402
from mixed_precision_quantized_act_b200 import _lib  # noqa: E402

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    mx.load()
    return torch.device("cuda:0")


def _inputs(N, K, D, seed, gscale=1.0):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.02, (N, K)).astype(np.float32)
    G = (rng.normal(0, gscale, (D, N, K))).astype(np.float32)
    return W, G


def _bound(W, G, S_ref):
    q, z, s = oracle.quantize_w4(W)
    N, K = W.shape
    sf = s.astype(np.float64).repeat(128, axis=1)
    delta = sf * (q.astype(np.float64) - z.astype(np.float64).repeat(128, axis=1)) - W.astype(np.float64)
    B = np.einsum("dnk,nk->dn", np.abs(G.astype(np.float64)), np.abs(delta))
    t = np.einsum("dnk,nk->dn", G.astype(np.float64), delta)
    e = 4 * (K / 256 + 16) * U32 * B
    D = G.shape[0]
    return np.mean(e * (1 + np.abs(t)) + e * e, axis=0) + S_ref * (D + 4) * U32


@pytest.mark.parametrize("N,K,D", [(300, 384, 5), (64, 128, 1), (512, 4096, 4), (8, 28672, 3), (97, 1024, 7)])
def test_salience_matches_oracle(dev, N, K, D):
    W, G = _inputs(N, K, D, seed=N + K + D)
    S_ref = oracle.channel_salience(W, G)
    S = mx.channel_salience(torch.from_numpy(W).to(dev), torch.from_numpy(G).to(dev))
    mx.sync_status()
    S = S.cpu().numpy().astype(np.float64)
    err = np.abs(S - S_ref)
    bound = _bound(W, G, S_ref)
    assert (err <= bound).all(), f"{int((err > bound).sum())} channels outside the bound; worst {float((err - bound).max()):.3g}"
    assert (S >= 0).all()


def test_salience_closed_form_and_zero_cases(dev):
    """A channel on the 4-bit grid has S = 0 exactly; one weight moved by eps
    with gradient lam * e_j gives S = mean |t + t^2/2|, t = -lam * eps."""
    s = 2.0 ** -6
    rng = np.random.default_rng(7)
    q = rng.integers(0, 16, (2, 256))
    q[:, 0], q[:, 1] = 0, 15
    q[:, 128], q[:, 129] = 0, 15
    W = ((q - 8) * s).astype(np.float32)
    j = next(i for i in range(2, 128) if q[1, i] not in (0, 15))
    eps = np.float32(0.25 * s)
    W[1, j] += eps
    lams = np.array([3.0, -500.0, 1.0], np.float32)
    G = np.zeros((3, 2, 256), np.float32)
    G[:, :, j] = lams[:, None]
    G[:, 0, :] += rng.normal(0, 1, (3, 256)).astype(np.float32)  # channel 0 is on the grid: S = 0 whatever g
    S = mx.channel_salience(torch.from_numpy(W).to(dev), torch.from_numpy(G).to(dev)).cpu().numpy()
    t = -lams.astype(np.float64) * float(eps)
    assert S[0] == 0.0
    assert S[1] == pytest.approx(np.mean(np.abs(t + 0.5 * t * t)), rel=1e-6)


def test_salience_is_deterministic(dev):
    W, G = _inputs(200, 2048, 6, seed=3)
    Wd, Gd = torch.from_numpy(W).to(dev), torch.from_numpy(G).to(dev)
    S1 = mx.channel_salience(Wd, Gd)
    S2 = mx.channel_salience(Wd, Gd)
    assert torch.equal(S1, S2)


def _sel_cases():
    rng = np.random.default_rng(11)
    yield "ties", np.array([3, 1, 3, 2, 3, 0, 3], np.float32), [0, 1, 2, 3, 4, 5, 6, 7]
    yield "signed_zeros", np.where(rng.random(3000) < 0.5, -0.0, 0.0).astype(np.float32), [0, 1, 1500, 2999, 3000]
    yield "few_values", rng.integers(0, 6, 5000).astype(np.float32), [1, 2500, 4999]
    yield "exponential", rng.exponential(1.0, 100_000).astype(np.float32), [1, 10_000, 99_999]
    yield "signed", rng.normal(0, 1, 4097).astype(np.float32), [0, 7, 2048, 4097]


@pytest.mark.parametrize("case", list(_sel_cases()), ids=lambda c: c[0])
def test_select_top_t_matches_oracle(dev, case):
    _, S, Ts = case
    Sd = torch.from_numpy(S).to(dev)
    for T in Ts:
        got = mx.select_top_t(Sd, T).cpu().numpy()
        assert np.array_equal(got, oracle.select_top_t(S, T)), f"T={T}"


def test_global_search_over_layers_feeds_the_packer(dev):
    """Algorithm 1 end to end on three small layers: per-layer salience,
    one global list, the top 10 % by the GPU; the same selection as the
    oracle's on the GPU's scores; the layers' bit maps pack and run."""
    shapes = [(256, 512), (384, 256), (128, 1024)]
    Ws, Ss = [], []
    for i, (N, K) in enumerate(shapes):
        W, G = _inputs(N, K, 4, seed=40 + i, gscale=1.0 + i)
        Ws.append(W)
        Ss.append(mx.channel_salience(torch.from_numpy(W).to(dev), torch.from_numpy(G).to(dev)))
    S = torch.cat(Ss)
    T = S.numel() // 10
    is8 = mx.select_top_t(S, T)
    assert int(is8.sum()) == T
    assert np.array_equal(is8.cpu().numpy(), oracle.select_top_t(S.cpu().numpy(), T))
    off = 0
    for (N, K), W in zip(shapes, Ws):
        m = is8[off:off + N]
        off += N
        p = mx.pack_weights(torch.from_numpy(W).to(dev), m)
        assert p.N8 == int(m.sum())
        X = torch.randn(3, K, device=dev).half()
        Y = mx.linear(X, p)
        mx.sync_status()
        assert torch.isfinite(Y).all()


def test_search_validation(dev):
    W = torch.zeros(4, 100, device=dev)
    G = torch.zeros(1, 4, 100, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.channel_salience(W, G)
    assert ei.value.status == _lib.ERR_UNSUPPORTED
    S = torch.zeros(10, device=dev)
    with pytest.raises(_lib.MixLLMError) as ei:
        mx.select_top_t(S, 11)
    assert ei.value.status == _lib.ERR_INVALID_ARG
    assert int(mx.select_top_t(S, 10).sum()) == 10
    assert int(mx.select_top_t(S, 0).sum()) == 0
    mx.sync_status()
