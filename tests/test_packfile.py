"""The packed-weight file (mixed_precision_quantized_act_b200.packfile) on the
CPU: buffers in the device layout, made here by the oracle, survive a round
trip byte for byte, and damaged files are refused rather than misread."""
import os
import struct

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from mixed_precision_quantized_act_b200 import _lib, packfile  # noqa: E402
from mixed_precision_quantized_act_b200 import workloads as wl  # noqa: E402

FIELDS = packfile.FIELDS


def _packed_on_host(oracle_mod, N, K, n8, seed):
    layer = wl.Linear("pf", 1, N, K, ((0, N, n8),), 2)
    W, is8 = wl.make_w(layer, seed), wl.make_bitmap(layer, seed)
    ref = oracle_mod.packed(oracle_mod.Quantized(W, is8))
    p = _lib.empty_packed(N, K, int(is8.sum()), "cpu")
    for name in FIELDS:
        t = getattr(p, name)
        a = np.ascontiguousarray(ref[name])
        assert a.nbytes == t.numel() * t.element_size(), name
        t.reshape(-1).view(torch.uint8).copy_(torch.from_numpy(a.reshape(-1).view(np.uint8).copy()))
    return p


@pytest.mark.parametrize("N,K,n8", [(300, 384, 37), (256, 256, 0), (130, 128, 130), (5, 512, 2)])
def test_round_trip_is_byte_exact(oracle_mod, tmp_path, N, K, n8):
    p = _packed_on_host(oracle_mod, N, K, n8, seed=N + K)
    path = os.path.join(tmp_path, "w.bin")
    packfile.save_packed(p, path)
    sizes = _lib.packed_sizes(N, K, p.N8)
    assert os.path.getsize(path) == 8 + 40 + 7 * 8 + sum(sizes)
    q = packfile.load_packed(path, "cpu")
    assert (q.N, q.K, q.N4, q.N8) == (p.N, p.K, p.N4, p.N8)
    for name in FIELDS:
        a, b = getattr(p, name), getattr(q, name)
        assert a.shape == b.shape and a.dtype == b.dtype, name
        assert torch.equal(a.reshape(-1).view(torch.uint8), b.reshape(-1).view(torch.uint8)), name


def test_damaged_files_are_refused(oracle_mod, tmp_path):
    p = _packed_on_host(oracle_mod, 300, 384, 37, seed=1)
    good = os.path.join(tmp_path, "good.bin")
    packfile.save_packed(p, good)
    data = open(good, "rb").read()

    def refused(blob, what):
        path = os.path.join(tmp_path, "bad.bin")
        with open(path, "wb") as f:
            f.write(blob)
        with pytest.raises(ValueError, match=what):
            packfile.load_packed(path, "cpu")

    refused(b"NOTMIXLL" + data[8:], "not a packed")
    refused(data[:30], "truncated header")
    refused(data[:8] + struct.pack("<5q", 300, 384, 263, 37, 64) + data[48:], "bad shape")
    refused(data[:8] + struct.pack("<5q", 300, 384, 260, 37, 128) + data[48:], "bad shape")
    refused(data[:8] + struct.pack("<5q", 300, 384, 262, 38, 128) + data[48:], "holds")
    refused(data[:-5], "truncated in idx8")
    refused(data + b"\0", "trailing")
