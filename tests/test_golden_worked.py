"""Hand-worked examples under tests/golden/, one quantisation group per
format, checked against the oracle, the host packer and (on a GPU) the device
packer, the dequantisation routine and both GEMM paths.

Each fixture gives a group of weights, and, derived by hand in its header, the
fp16 scale (and bias), the codes, the packed bytes and the dequantised values.
The inputs are chosen so that every step is exact or a stated rounding tie,
so the expected values can be checked by eye against the format's definition:
a swapped nibble, a wrong code offset, a mean taken as a max, a tie rounded
away from even or a -0.0 coded as negative fails here.
"""
import glob
import os
import pathlib

import numpy as np
import pytest
import torch

import oracle as O
import weight_quantised_gemm_b200 as wq

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FIXTURES = sorted(glob.glob(os.path.join(GOLDEN, "*.txt")))


def _load(path):
    d = {}
    for line in pathlib.Path(path).read_text().splitlines():
        if line.startswith("#") or not line.strip():
            continue
        key, *vals = line.split()
        d[key] = vals
    bits, group = int(d["bits"][0]), int(d["group"][0])
    fx = {
        "bits": bits,
        "group": group,
        "w": np.array([float(v) for v in d["w"]], dtype=np.float32),
        "scale": int(d["scale_f16"][0], 16),
        "bias": int(d["bias_f16"][0], 16) if "bias_f16" in d else None,
        "codes": np.array([int(v) for v in d["codes"]], dtype=np.int64),
        "packed": np.array([int(v, 16) for v in d["packed"]], dtype=np.uint8),
        "dequant": np.array([float(v) for v in d["dequant"]], dtype=np.float64),
    }
    assert fx["w"].size == group and fx["codes"].size == group and fx["dequant"].size == group
    assert fx["packed"].size == group * bits // 8
    assert (fx["bias"] is None) == (bits <= 2)
    return fx


def _ids():
    return [os.path.basename(f)[:-4] for f in FIXTURES]


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _tiled(fx, N, K):
    """W [N, K] with the fixture's group in every group position."""
    return np.tile(fx["w"], (N, K // fx["group"]))


def test_every_format_has_a_worked_example():
    assert sorted(_load(f)["bits"] for f in FIXTURES) == [1, 2, 4, 4, 8]


@pytest.mark.parametrize("path", FIXTURES, ids=_ids())
def test_oracle_reproduces_worked_example(path):
    fx = _load(path)
    bits, group = fx["bits"], fx["group"]
    packed, s16, b16 = O.pack_ref(fx["w"][None, :], bits, group)
    assert packed[0].tolist() == fx["packed"].tolist()
    assert int(s16.view(np.uint16)[0, 0]) == fx["scale"]
    if fx["bias"] is not None:
        assert int(b16.view(np.uint16)[0, 0]) == fx["bias"]
    assert O.unpack_codes(packed, bits, group)[0].tolist() == fx["codes"].tolist()
    wd = O.dequant_ref(packed, s16, b16, bits, group, group)[0]
    assert np.array_equal(wd, fx["dequant"])
    # the dequantised values are exact in bf16, so their bits are the bf16 bits of the fixture's values
    assert np.array_equal(O.dequant_ref_bits(packed, s16, b16, bits, group, group)[0], _bf16_bits(fx["dequant"]))


@pytest.mark.parametrize("path", FIXTURES, ids=_ids())
def test_host_packer_reproduces_worked_example(path):
    fx = _load(path)
    N, K = 16, 256
    pw = wq.qgemm_pack(_tiled(fx, N, K), fx["bits"])
    reps = K // fx["group"]
    assert np.array_equal(pw.packed, np.tile(fx["packed"], (N, reps)))
    assert np.all(pw.scales.view(np.uint16) == fx["scale"])
    if fx["bias"] is not None:
        assert np.all(pw.biases.view(np.uint16) == fx["bias"])


@pytest.mark.gpu
@pytest.mark.parametrize("path", FIXTURES, ids=_ids())
def test_device_reproduces_worked_example(path):
    fx = _load(path)
    bits, group = fx["bits"], fx["group"]
    N, K = 256, 256
    reps = K // group
    W = _tiled(fx, N, K)
    # the device packer
    dev = wq.qgemm_pack_device(torch.from_numpy(W).cuda(), bits)
    wq.check_device_status()
    assert np.array_equal(dev.packed.cpu().numpy(), np.tile(fx["packed"], (N, reps)))
    assert np.all(dev.scales.cpu().numpy().view(np.uint16) == fx["scale"])
    if fx["bias"] is not None:
        assert np.all(dev.biases.cpu().numpy().view(np.uint16) == fx["bias"])
    # the tile dequantisation routine
    want = np.tile(_bf16_bits(fx["dequant"]), (N, reps))
    wd = wq.qgemm_dequant_tile(dev)
    wq.check_device_status()
    assert np.array_equal(wd.contiguous().view(torch.int16).cpu().numpy().view(np.uint16), want)
    # both GEMM paths: a one-hot token row m picks k_m, so out[m, n] = Wdeq[n, k_m] exactly
    for M, kpath in ((16, wq.QGEMM_PATH_SMALL_M), (200, wq.QGEMM_PATH_LARGE_M)):
        ks = (np.arange(M) * 7) % K
        X = np.zeros((M, K), dtype=np.float32)
        X[np.arange(M), ks] = 1.0
        Xd = torch.from_numpy(X).cuda().to(torch.bfloat16)
        y = wq.qgemm(Xd, dev, path=kpath)
        wq.check_device_status()
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, want[:, ks].T), f"path {kpath}"
