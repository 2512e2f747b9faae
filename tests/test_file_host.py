"""The at-rest file (qgemm_save / qgemm_load_header / qgemm_load) on the host:
round trips of every format, and the documented rejections."""
import ctypes
import os
import pathlib
import struct

import numpy as np
import pytest

import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_round_trip_every_format(tmp_path, bits):
    W = WL.random_case(7, 1, 48, 512, bits, with_bias=False)[1]
    pw = wq.qgemm_pack(W, bits)
    path = str(tmp_path / f"w{bits}.qgw")
    pw.save(path)
    back = wq.qgemm_load(path)
    assert (back.N, back.K, back.bits, back.group) == (48, 512, bits, wq.GROUP_OF_BITS[bits])
    assert np.array_equal(back.packed, pw.packed)
    assert np.array_equal(back.scales.view(np.uint16), pw.scales.view(np.uint16))
    if bits > 2:
        assert np.array_equal(back.biases.view(np.uint16), pw.biases.view(np.uint16))
    else:
        assert back.biases is None
    # the file is exactly header + arrays, and the arrays are the oracle's
    p, s, b = O.pack_ref(W, bits, wq.GROUP_OF_BITS[bits])
    size = 48 + p.nbytes + s.nbytes + (0 if b is None else b.nbytes)
    assert os.path.getsize(path) == size
    with open(path, "rb") as f:
        head = f.read(48)
    assert head[:8] == b"QGEMMW01"
    assert struct.unpack("<4i3Q", head[8:]) == (48, 512, bits, wq.GROUP_OF_BITS[bits], p.nbytes, s.nbytes,
                                                 0 if b is None else b.nbytes)


def _expect(path, status):
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_load(path)
    assert e.value.status == status


def test_rejects_corrupt_files(tmp_path):
    pw = wq.qgemm_pack(WL.random_case(8, 1, 32, 256, 4, with_bias=False)[1], 4)
    good = str(tmp_path / "good.qgw")
    pw.save(good)
    data = pathlib.Path(good).read_bytes()
    bad = str(tmp_path / "bad.qgw")
    for blob, status in [(b"XGEMMW01" + data[8:], wq.QGEMM_ERR_INVALID_ARG),        # magic
                         (data[:40], wq.QGEMM_ERR_INVALID_ARG),                     # short header
                         (data[:-1], wq.QGEMM_ERR_INVALID_ARG),                     # truncated arrays
                         (data + b"\0", wq.QGEMM_ERR_INVALID_ARG),                  # trailing bytes
                         (data[:8] + struct.pack("<4i", 32, 256, 3, 64) + data[24:], wq.QGEMM_ERR_UNSUPPORTED),
                         (data[:24] + struct.pack("<Q", 1) + data[32:], wq.QGEMM_ERR_INVALID_ARG)]:  # sizes
        pathlib.Path(bad).write_bytes(blob)
        _expect(bad, status)
    _expect(str(tmp_path / "missing.qgw"), wq.QGEMM_ERR_INVALID_ARG)


def test_truncation_at_every_offset_and_a_lying_header(tmp_path):
    """Every proper prefix of a valid file, and the file with one byte more,
    is refused by both readers; a header whose shape claims far more data
    than the file holds is refused by qgemm_load_header before any buffer is
    sized from it."""
    pw = wq.qgemm_pack(WL.random_case(9, 1, 16, 128, 4, with_bias=False)[1], 4)
    good = str(tmp_path / "good.qgw")
    pw.save(good)
    data = pathlib.Path(good).read_bytes()
    bad = str(tmp_path / "bad.qgw")
    N, K, bits, group = (ctypes.c_int32() for _ in range(4))
    for cut in list(range(len(data))) + [len(data) + 1]:
        pathlib.Path(bad).write_bytes(data[:cut] if cut < len(data) else data + b"\0")
        st = wq._lib.qgemm_load_header(bad.encode(), ctypes.byref(N), ctypes.byref(K), ctypes.byref(bits),
                                       ctypes.byref(group))
        assert st == wq.QGEMM_ERR_INVALID_ARG, cut
        _expect(bad, wq.QGEMM_ERR_INVALID_ARG)
    # a consistent header for [2^20, 2^20] 8-bit weights (1 TiB of codes) over the small file's bytes
    n = k = 1 << 20
    lying = data[:8] + struct.pack("<4i3Q", n, k, 8, 64, n * k, n * (k // 64) * 2, n * (k // 64) * 2) + data[48:]
    pathlib.Path(bad).write_bytes(lying)
    st = wq._lib.qgemm_load_header(bad.encode(), ctypes.byref(N), ctypes.byref(K), ctypes.byref(bits),
                                   ctypes.byref(group))
    assert st == wq.QGEMM_ERR_INVALID_ARG
    _expect(bad, wq.QGEMM_ERR_INVALID_ARG)
    # and the untouched file still loads
    back = wq.qgemm_load(good)
    assert np.array_equal(back.packed, pw.packed)


def test_round_trip_property_over_shapes_and_formats(tmp_path):
    """Any supported shape and format: save then load gives back the same
    bytes, and the file is exactly the header plus the three arrays."""
    pytest.importorskip("hypothesis")
    from hypothesis import HealthCheck, given, settings, strategies as st

    @settings(max_examples=25, deadline=None, derandomize=True, database=None,
              suppress_health_check=list(HealthCheck))
    @given(bits=st.sampled_from([1, 2, 4, 8]), n16=st.integers(1, 6), k128=st.integers(1, 8),
           seed=st.integers(0, 2 ** 16))
    def check(bits, n16, k128, seed):
        N, K = 16 * n16, 128 * k128
        W = (np.random.default_rng(seed).standard_normal((N, K)) * 0.02).astype(np.float32)
        pw = wq.qgemm_pack(W, bits)
        path = str(tmp_path / f"p{bits}_{N}_{K}.qgw")
        pw.save(path)
        back = wq.qgemm_load(path)
        assert (back.N, back.K, back.bits, back.group) == (N, K, bits, wq.GROUP_OF_BITS[bits])
        assert np.array_equal(back.packed, pw.packed)
        assert np.array_equal(back.scales.view(np.uint16), pw.scales.view(np.uint16))
        assert (back.biases is None) == (pw.biases is None)
        if pw.biases is not None:
            assert np.array_equal(back.biases.view(np.uint16), pw.biases.view(np.uint16))
        assert os.path.getsize(path) == 48 + pw.nbytes

    check()
