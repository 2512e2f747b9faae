"""qgemm_grouped: several small-M GEMVs of one format, as consecutive
overlapped launches (the default) and in one persistent launch
(QGEMM_FLAG_GROUPED_ONE_LAUNCH), each checked against the oracle on its own."""
import numpy as np
import pytest
import torch

import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL
from gpu_util import from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu


def _check(X, W, bias, bits, y, what):
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    ref = O.qgemm_ref(X, p, s, b, bits, group, W.shape[1], bias)
    yv = O.bf16_bits_to_f64(from_dev_bf16(y))
    assert np.all(np.isfinite(yv)), what
    rf, ma = O.rel_frobenius(yv, ref), O.max_abs_rel(yv, ref)
    assert rf <= O.REL_FROB_TOL and ma <= O.MAX_ABS_TOL, f"{what}: rel_frob={rf:.3e} max_abs={ma:.3e}"


def _run(shapes, bits, seed, overlap=False, one_launch=False):
    host, probs = [], []
    for i, (M, N, K, with_bias) in enumerate(shapes):
        X, W, bias = WL.random_case(seed + 17 * i, M, N, K, bits, with_bias=with_bias)
        dw = wq.qgemm_pack(W, bits).to_device()
        probs.append((to_dev_bf16(X), dw, None if bias is None else to_dev_bf16(bias)))
        host.append((X, W, bias))
    ys = wq.qgemm_grouped(probs, overlap_previous=overlap, one_launch=one_launch)
    wq.check_device_status()
    return host, ys, probs


# the FLUX double-stream block's linears at decode M, split by format as the
# mixed policy stores them: 4-bit QKV and MLP up, 8-bit modulation, output
# projection and MLP down
FLUX4 = [(9216, 3072), (12288, 3072)]
FLUX8 = [(18432, 3072), (3072, 3072), (3072, 12288)]


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("bits,shapes", [(4, FLUX4), (8, FLUX8)])
def test_grouped_flux_block_linears(bits, shapes, M, one_launch):
    host, ys, _ = _run([(M, N, K, True) for N, K in shapes], bits, 1000 + M + bits, one_launch=one_launch)
    for (X, W, bias), y in zip(host, ys):
        _check(X, W, bias, bits, y, f"bits={bits} M={M} N={W.shape[0]} K={W.shape[1]}")


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_grouped_ragged_mix(bits, one_launch):
    """Different M (including 0, a skipped problem), N not a multiple of the
    32-row item, K not a multiple of a stage, with and without bias."""
    K2 = 1280 if bits == 1 else 1152
    shapes = [(3, 400, K2, True), (0, 256, 512, False), (16, 1040, 512, False), (1, 48, 2048, True),
              (9, 4096, 3072, True)]
    host, ys, _ = _run(shapes, bits, 2000 + bits, one_launch=one_launch)
    for (X, W, bias), y, (M, N, K, _) in zip(host, ys, shapes):
        assert y.shape == (M, N)
        if M:
            _check(X, W, bias, bits, y, f"bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("bits", [2, 4])
def test_grouped_one_hot_rows_are_bit_exact(bits, one_launch):
    """One non-zero activation per token: each output is one weight's exact
    fp32 value s*q + b, rounded once to bf16, in every problem of the call."""
    g = np.random.default_rng(5 + bits)
    probs, expect = [], []
    for i, (N, K) in enumerate([(512, 1024), (1056, 3072), (96, 512)]):
        _, W, _ = WL.random_case(60 + i + bits, 1, N, K, bits, with_bias=False)
        M = 5 + i
        ks = g.choice(K, size=M, replace=False)
        X = np.zeros((M, K), dtype=np.uint16)
        X[np.arange(M), ks] = 0x3F80
        dw = wq.qgemm_pack(W, bits).to_device()
        probs.append((to_dev_bf16(X), dw, None))
        group = wq.GROUP_OF_BITS[bits]
        p, s, b = O.pack_ref(W, bits, group)
        w32 = O.wq_exact(p, s, b, bits, group, K).astype(np.float32)
        expect.append(WL.f32_to_bf16_bits(np.ascontiguousarray(w32[:, ks].T)))
    ys = wq.qgemm_grouped(probs, one_launch=one_launch)
    wq.check_device_status()
    for y, e in zip(ys, expect):
        assert np.array_equal(from_dev_bf16(y), e)


@pytest.mark.parametrize("one_launch", [False, True])
def test_grouped_overlap_reads_the_previous_kernels_output(one_launch):
    """A torch kernel writes the inputs right before an overlapped grouped
    call; the call must see them. Repeated, and replayed from a CUDA graph."""
    bits = 8
    shapes = [(4, 3072, 3072, True), (4, 6144, 3072, False)]
    host, ys, probs = _run(shapes, bits, 3000, one_launch=one_launch)
    src = [p[0].clone() for p in probs]
    outs = [torch.empty_like(y) for y in ys]
    for _ in range(2):
        for p in probs:
            p[0].zero_()
        for p, s in zip(probs, src):
            p[0].copy_(s)
        wq.qgemm_grouped(probs, outs=outs, overlap_previous=True, one_launch=one_launch)
        wq.check_device_status()
        for (X, W, bias), y in zip(host, outs):
            _check(X, W, bias, bits, y, "overlapped")
    eager = [o.clone() for o in outs]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for p, x in zip(probs, src):
            p[0].copy_(x)
        wq.qgemm_grouped(probs, outs=outs, overlap_previous=True, one_launch=one_launch)
    for p, o in zip(probs, outs):
        p[0].zero_()
        o.zero_()
    g.replay()
    torch.cuda.synchronize()
    wq.check_device_status()
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    del g


def test_grouped_equals_the_oracle_where_one_call_each_does():
    """The grouped call and one qgemm per problem both meet the gate on the
    same inputs (their summation orders differ, so bits may too)."""
    bits = 4
    shapes = [(2, 9216, 3072, True), (2, 3072, 3072, True)]
    host, ys, probs = _run(shapes, bits, 4000)
    for (X, W, bias), y, (Xd, dw, bd) in zip(host, ys, probs):
        single = wq.qgemm(Xd, dw, bias=bd)
        wq.check_device_status()
        _check(X, W, bias, bits, y, "grouped")
        _check(X, W, bias, bits, single, "single")
        assert O.rel_frobenius(O.bf16_bits_to_f64(from_dev_bf16(y)), O.bf16_bits_to_f64(from_dev_bf16(single))) < 2e-3


def test_grouped_default_equals_one_plain_call_per_problem():
    """The default form is one small-M launch per problem: the same bits as a
    qgemm call on each problem's own."""
    bits = 8
    shapes = [(3, 3072, 3072, True), (5, 6144, 3072, False), (1, 3072, 12288, True)]
    host, ys, probs = _run(shapes, bits, 5000)
    for y, (Xd, dw, bd) in zip(ys, probs):
        single = wq.qgemm(Xd, dw, bias=bd, path=wq.QGEMM_PATH_SMALL_M)
        wq.check_device_status()
        assert torch.equal(y, single)
