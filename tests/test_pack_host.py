"""The host-side pack (mixllm_pack_weights_host) against the oracle's
quantizers and packed layout, byte for byte, on CPU (no device touched).
Its bytes equal the device pack's too: tests/test_gpu_parity.py compares
both packs with the same oracle buffers."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from mixed_precision_quantized_act_b200 import _lib  # noqa: E402
from mixed_precision_quantized_act_b200 import workloads as wl  # noqa: E402

CASES = [
    wl.TINY,
    wl.Linear("hp_p0", 4, 256, 384, ((0, 256, 0),), 2),
    wl.Linear("hp_p100", 4, 256, 256, ((0, 256, 256),), 2),
    wl.Linear("hp_ragged", 4, 300, 512, ((0, 300, 37),), 3),
    wl.Linear("hp_one8", 4, 130, 128, ((0, 130, 1),), 2),
]


def _special_weights(N, K, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0, :128] = 0.0                                  # an all-zero group
    W[1, :128] = 0.5                                  # a constant positive group
    W[2, :128] = -0.25                                # a constant negative group
    W[3, :128] = np.linspace(-1, 1, 128, dtype=np.float32)
    W[4, 128:256] = 1e-30                             # scales that round to zero in fp16
    W[5, :128] = 7e4                                  # a scale past the fp16 range (clamped)
    return W


@pytest.mark.parametrize("layer", CASES, ids=lambda l: l.name)
def test_host_pack_matches_the_oracle_bytes(layer):
    W, is8 = wl.make_w(layer, 9), wl.make_bitmap(layer, 9)
    p = _lib.pack_weights_host(torch.from_numpy(W), torch.from_numpy(is8))
    ref = oracle.packed(oracle.Quantized(W, is8))
    for name in ("W4", "z4", "s_w4", "idx4", "W8", "s_w8", "idx8"):
        got = getattr(p, name).numpy()
        exp = np.ascontiguousarray(ref[name])
        assert got.view(np.uint8).tobytes() == exp.view(np.uint8).tobytes(), name


def test_host_pack_special_groups():
    N, K = 264, 256
    W = _special_weights(N, K, 3)
    is8 = np.zeros(N, np.uint8)
    is8[[1, 3, 5, 100, 263]] = 1
    p = _lib.pack_weights_host(torch.from_numpy(W), torch.from_numpy(is8))
    ref = oracle.packed(oracle.Quantized(W, is8))
    for name in ("W4", "z4", "s_w4", "idx4", "W8", "s_w8", "idx8"):
        assert getattr(p, name).numpy().view(np.uint8).tobytes() == np.ascontiguousarray(ref[name]).view(np.uint8).tobytes(), name


def test_host_pack_rejects_a_bit_map_that_disagrees_with_n8():
    W = torch.zeros((256, 128), dtype=torch.float32)
    is8 = torch.zeros(256, dtype=torch.uint8)
    is8[:3] = 1
    L = _lib.load()
    p = _lib.empty_packed(256, 128, 4, "cpu")
    st = L.mixllm_pack_weights_host(W.data_ptr(), 256, 128, is8.data_ptr(), 4, 128, p.W4.data_ptr(), p.z4.data_ptr(),
                                    p.s_w4.data_ptr(), p.idx4.data_ptr(), p.W8.data_ptr(), p.s_w8.data_ptr(),
                                    p.idx8.data_ptr())
    assert st == _lib.ERR_INVALID_ARG
