"""The library's host packer (C++) against the oracle's packer (numpy): byte for
byte identical codes, scales and biases, on the workloads' weights and on
edge-case groups. Both take every rounding decision in fp64, ties to even."""
import numpy as np
import pytest

import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL


def _same(W, bits):
    group = wq.GROUP_OF_BITS[bits]
    got = wq.qgemm_pack(W, bits)
    p, s, b = O.pack_ref(W, bits, group)
    assert np.array_equal(got.packed, p)
    assert np.array_equal(got.scales.view(np.uint16), s.view(np.uint16))
    if bits <= 2:
        assert got.biases is None and b is None
    else:
        assert np.array_equal(got.biases.view(np.uint16), b.view(np.uint16))


@pytest.mark.parametrize("cid,lin_idx,rows", [(0, 0, None), (1, 0, 512), (2, 1, 256), (4, 0, 256)])
def test_workload_weights(cid, lin_idx, rows):
    lin = WL.workload(cid).linears[lin_idx]
    N = lin.N if rows is None else rows
    W = WL.make_w(cid, lin_idx, N, lin.K, lin.w_dist, lin.group)
    _same(W, lin.bits)


def test_ternary_workload_weights():
    lin = WL.workload(3).linears[0]
    W = WL.make_w(3, 0, 512, lin.K, "ternary", 128)
    _same(W, 2)


def test_binary_workload_weights():
    lin = WL.workload(5).linears[1]
    W = WL.make_w(5, 1, 512, lin.K, "binary", 128)
    _same(W, 1)
    _same((np.random.default_rng(4).standard_normal((64, 1024)) * 0.02).astype(np.float32), 1)


def _edge_matrix(g, K, group):
    rows = []
    rows.append(np.zeros(K))                                    # all zero
    rows.append(np.full(K, -0.0))                               # negative zeros
    rows.append(np.full(K, 0.125))                              # constant group
    rows.append(g.standard_normal(K) * 1e-7)                    # fp16-subnormal scales
    rows.append(g.standard_normal(K) * 1e-9)                    # scales underflow
    rows.append(g.standard_normal(K) * 1000.0)                  # large range
    rows.append(np.resize([-1.0, 1.0], K))                      # two-level groups
    r = np.resize(np.arange(group) * 0.5 - 3.75, K)             # exact ties at half steps
    rows.append(r)
    rows.append(np.resize([0.0, 1e-30, -1e-30, 3.0], K))        # tiny fp32 next to large
    rows.append(g.uniform(-1, 1, K).astype(np.float16).astype(np.float64))  # fp16-exact values
    W = np.stack(rows)
    W = np.concatenate([W, (g.standard_normal((6, K)) * 0.02)])
    return W.astype(np.float32)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_edge_groups(bits):
    g = np.random.default_rng(100 + bits)
    group = wq.GROUP_OF_BITS[bits]
    _same(_edge_matrix(g, 512, group), bits)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_random_scales_wide_dynamic_range(bits):
    g = np.random.default_rng(7 * bits)
    K = 256
    mags = 10.0 ** g.uniform(-6, 3, size=(64, 1))
    W = (g.standard_normal((64, K)) * mags).astype(np.float32)
    _same(W, bits)


def test_multithreaded_pack_matches_single_rows():
    """Large matrices are packed by several threads: rows are independent."""
    lin = WL.workload(2).linears[0]
    W = WL.make_w(2, 0, 2048, lin.K, "normal")
    whole = wq.qgemm_pack(W, 4)
    part = wq.qgemm_pack(W[1000:1016], 4)
    assert np.array_equal(whole.packed[1000:1016], part.packed)
    assert np.array_equal(whole.scales[:, 1000:1016].view(np.uint16), part.scales.view(np.uint16))
    assert whole.scales.shape == (lin.K // 64, 2048)


def test_1bit_scale_is_exact_in_any_order():
    """Groups whose 1-bit scale an fp64 running sum would get wrong (see the
    oracle pin): the host packer rounds the exact mean like the oracle, so
    the large weight first or last gives the same 8200."""
    w = np.full((16, 128), 2.0 ** -38, dtype=np.float32)
    w[::2, 0] = 1049088.0                # even rows: the large weight first
    w[1::2, 127] = 1049088.0             # odd rows: the large weight last
    pw = wq.qgemm_pack(w, 1)
    p, s16, _ = O.pack_ref(w, 1, 128)
    assert np.array_equal(pw.scales.view(np.uint16), s16.view(np.uint16))
    assert np.array_equal(pw.packed, p)
    assert np.all(pw.scales.astype(np.float64) == 8200.0)


def test_1bit_scale_near_fp16_ties_over_many_binades():
    """Groups built to sit on or next to an fp16 rounding tie, with the
    remainder spread over many binades and the weights in random order:
    host packer and oracle agree bit for bit."""
    g = np.random.default_rng(77)
    rows = []
    for i in range(256):
        big = np.float32(1049088.0 * 2.0 ** int(g.integers(-30, 3)))   # 128 x an fp16 tie value
        tail = (2.0 ** g.integers(-149, -20, size=127)).astype(np.float32) * g.choice([0, 1, 1], size=127)
        sign = np.where(g.integers(0, 2, size=128) == 1, 1.0, -1.0)
        row = np.concatenate([[big], tail]) * sign
        if i % 3 == 0:
            row[0] = np.nextafter(np.float32(row[0]), np.float32(0))       # just below the tie
        rows.append(g.permutation(row))
    _same(np.stack(rows).astype(np.float32), 1)


@pytest.mark.parametrize("limit", [3e4, 3.3999999521443642e+38], ids=["fp16-range", "fp32-range"])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_host_packer_matches_oracle_on_arbitrary_fp32(bits, limit):
    """Property test: any finite fp32 weights (subnormals, signed zeros,
    repeated values, rounding ties, values near and past the fp16 range) pack
    to the oracle's bytes, scales and biases exactly, and a group whose scale
    or bias overflows fp16 is refused by both."""
    pytest.importorskip("hypothesis")
    from hypothesis import HealthCheck, given, settings, strategies as st
    from hypothesis.extra.numpy import arrays

    group = wq.GROUP_OF_BITS[bits]
    elems = st.one_of(st.floats(-limit, limit, width=32, allow_nan=False, allow_infinity=False),
                      st.sampled_from([0.0, -0.0, 0.5, -0.5, 1.5, 2.5, 2.0 ** -149, -(2.0 ** -130),
                                       65504.0, -65504.0, 65520.0]))

    @settings(max_examples=40, deadline=None, derandomize=True, database=None,
              suppress_health_check=list(HealthCheck))
    @given(W=arrays(np.float32, (16, 2 * group), elements=elems))
    def check(W):
        try:
            pw, refused = wq.qgemm_pack(W, bits), None
        except wq.QGemmError as e:
            pw, refused = None, e.status
        try:
            p, s16, b16 = O.pack_ref(W, bits, group)
            expect = None
        except OverflowError:
            expect = wq.QGEMM_ERR_UNSUPPORTED
        assert refused == expect
        if expect is None:
            assert np.array_equal(pw.packed, p)
            assert np.array_equal(pw.scales.view(np.uint16), s16.view(np.uint16))
            if bits > 2:
                assert np.array_equal(pw.biases.view(np.uint16), b16.view(np.uint16))

    check()
