"""Parity of the CUDA path with the CPU oracle, through the C ABI.

* the dequantised weights (debug entry point) are bit-exact;
* GEMM outputs meet rel-Frobenius <= 5e-3 and max-abs <= 3e-2 * max|ref|
  against the oracle's fp64 X . Wq^T (+ bias), on both kernel paths, every
  format, ragged shapes and every workload at full size (sampled rows there);
* one-hot activations make the GEMM output bit-exact to the dequantised
  weights on both paths (one non-zero product: fp32 accumulation is exact).

The oracle packs its own copy of the weights; nothing it compares against
comes from the GPU.
"""
import numpy as np
import pytest
import torch

import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL
from gpu_util import from_dev_bf16, gpu_qgemm, gpu_qgemm_packed, to_dev_bf16

pytestmark = pytest.mark.gpu

SMALL, LARGE = wq.QGEMM_PATH_SMALL_M, wq.QGEMM_PATH_LARGE_M


def _ref(X, W, bias, bits):
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    return O.qgemm_ref(X, p, s, b, bits, group, W.shape[1], bias)


def _assert_close(y_bits, ref, what=""):
    y = O.bf16_bits_to_f64(y_bits)
    assert np.all(np.isfinite(y)), what
    rf, ma = O.rel_frobenius(y, ref), O.max_abs_rel(y, ref)
    assert rf <= O.REL_FROB_TOL and ma <= O.MAX_ABS_TOL, f"{what}: rel_frob={rf:.3e} max_abs={ma:.3e}"
    return rf, ma


# ----------------------------------------------------------------------------
# dequantisation: bit-exact
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_dequant_whole_matrix_bit_exact(bits):
    group = wq.GROUP_OF_BITS[bits]
    if bits == 1:
        W = WL.make_w(5, 1, 512, 3072, "binary", 128)
    elif bits == 2:
        W = WL.make_w(3, 0, 512, 3072, "ternary", 128)
    else:
        W = WL.make_w(0, 0, 512, 1024, "normal")
    dw = wq.qgemm_pack(W, bits).to_device()
    got = from_dev_bf16(wq.qgemm_dequant_tile(dw))
    wq.check_device_status()
    p, s, b = O.pack_ref(W, bits, group)
    ref = O.dequant_ref_bits(p, s, b, bits, group, W.shape[1])
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_dequant_edge_groups_and_windows_bit_exact(bits):
    group = wq.GROUP_OF_BITS[bits]
    g = np.random.default_rng(55 + bits)
    K = 1024
    rows = [np.zeros(K), np.full(K, 0.25), g.standard_normal(K) * 1e-6, g.standard_normal(K) * 300.0,
            np.resize([-1.0, 1.0], K)]
    W = np.concatenate([np.stack(rows), g.standard_normal((27, K)) * 0.02]).astype(np.float32)
    dw = wq.qgemm_pack(W, bits).to_device()
    p, s, b = O.pack_ref(W, bits, group)
    ref = O.dequant_ref_bits(p, s, b, bits, group, K)
    for (n0, k0, r, c) in [(0, 0, 32, K), (3, 8, 5, 40), (31, 1016, 1, 8), (10, 128, 16, 256)]:
        got = from_dev_bf16(wq.qgemm_dequant_tile(dw, n0, k0, r, c))
        assert np.array_equal(got, ref[n0:n0 + r, k0:k0 + c]), (n0, k0, r, c)
    wq.check_device_status()


# ----------------------------------------------------------------------------
# one-hot activations: the GEMM data path bit-exact to the dequantised weights
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("path,M", [(SMALL, 16), (SMALL, 5), (LARGE, 16), (LARGE, 300)])
def test_one_hot_rows_reproduce_dequantised_weights(bits, path, M):
    group = wq.GROUP_OF_BITS[bits]
    N, K = 272, 768
    g = np.random.default_rng(9)
    if bits == 1:
        c = 2.0 * g.integers(0, 2, size=(N, K)).astype(np.float32) - 1.0
        s = g.uniform(0.01, 0.05, size=(N, K // 128)).astype(np.float16).astype(np.float32)
        W = (c * np.repeat(s, 128, axis=1)).astype(np.float32)
    elif bits == 2:
        t = g.integers(-1, 2, size=(N, K)).astype(np.float32)
        s = g.uniform(0.01, 0.05, size=(N, K // 128)).astype(np.float16).astype(np.float32)
        W = (t * np.repeat(s, 128, axis=1)).astype(np.float32)
    else:
        W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    ks = g.choice(K, size=M, replace=M > K)
    X = np.zeros((M, K), dtype=np.uint16)
    X[np.arange(M), ks] = 0x3F80  # 1.0
    y, dw = gpu_qgemm(X, W, None, bits, path=path)
    p, s, b = O.pack_ref(W, bits, group)
    wd = O.dequant_ref_bits(p, s, b, bits, group, K)
    assert np.array_equal(y, wd[:, ks].T)


# ----------------------------------------------------------------------------
# GEMM parity on small and ragged shapes, both paths
# ----------------------------------------------------------------------------

def test_tiny_workload_default_path():
    lin = WL.workload(0).linears[0]
    X, W, bias = WL.make_inputs(lin, 0, 0)
    y, _ = gpu_qgemm(X, W, bias, lin.bits)
    _assert_close(y, _ref(X, W, bias, lin.bits), "tiny")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [1, 2, 3, 8, 9, 16, 17, 24, 31, 32])
def test_small_path_ragged(bits, M):
    K = 1280 if bits == 1 else 1152  # 1-bit rows on the small path: K % 256 == 0
    X, W, bias = WL.random_case(M * 10 + bits, M, 400, K, bits, with_bias=True)
    y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
    _assert_close(y, _ref(X, W, bias, bits), f"small bits={bits} M={M}")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M,N", [(5, 8176), (3, 12272), (5, 16368), (16, 8176), (16, 12272), (11, 16368),
                                 (20, 4080), (32, 8176), (32, 12272), (24, 16368)])
def test_small_path_every_row_count(bits, M, N):
    """Every rows-per-CTA choice beyond the smallest at every token width: on
    148 SMs N = 8176, 12272 and 16368 take 4, 6 and 8 16-row pairs per CTA,
    each one pair short of whole CTAs, so the last CTA is ragged. With more
    than 8 tokens, 6 or 8 pairs split the rows into halves, each warp taking
    two groups per stage, and the activations come through the ring. With
    more than 16 tokens CTAs take 2 (N = 4080), 4 (N = 8176, rows split into
    halves) or 8 pairs (N = 12272 and 16368, rows split into quarters, each
    warp taking four groups per stage), the activations always through the
    ring."""
    K = 512
    X, W, bias = WL.random_case(M + N + bits, M, N, K, bits, with_bias=True)
    y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
    _assert_close(y, _ref(X, W, bias, bits), f"small bits={bits} M={M} N={N}")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (17, 144, 256), (255, 272, 384), (256, 256, 512),
                                   (257, 400, 640), (600, 528, 1024)])
def test_large_path_ragged(bits, M, N, K):
    X, W, bias = WL.random_case(M + N + bits, M, N, K, bits, with_bias=(M % 2 == 1))
    y, _ = gpu_qgemm(X, W, bias, bits, path=LARGE)
    _assert_close(y, _ref(X, W, bias, bits), f"large bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("path,M", [(SMALL, 7), (LARGE, 100)])
def test_zero_weights_give_the_bias(path, M):
    X, _, bias = WL.random_case(3, M, 256, 256, 4, with_bias=True)
    W = np.zeros((256, 256), dtype=np.float32)
    y, _ = gpu_qgemm(X, W, bias, 4, path=path)
    assert np.array_equal(y, np.broadcast_to(bias, (M, 256)))


def test_both_paths_agree_at_m16():
    """The paths differ by the large path's bf16 rounding of the dequantised
    weight (~1.1e-3 rms relative) plus each one's bf16 output rounding."""
    X, W, bias = WL.random_case(77, 16, 512, 1024, 4, with_bias=True)
    ys, dw = gpu_qgemm(X, W, bias, 4, path=SMALL)
    yl = gpu_qgemm_packed(X, dw, bias, path=LARGE)
    a, b = O.bf16_bits_to_f64(ys), O.bf16_bits_to_f64(yl)
    assert O.rel_frobenius(a, b) < O.REL_FROB_TOL
    ref = _ref(X, W, bias, 4)
    # the small path keeps s*q + b exact, so it sits closer to the oracle
    assert O.rel_frobenius(a, ref) < O.rel_frobenius(b, ref)


def test_runs_on_a_side_stream_and_repeats_identically():
    X, W, bias = WL.random_case(5, 300, 256, 512, 8, with_bias=True)
    dw = wq.qgemm_pack(W, 8).to_device()
    Xd, bd = to_dev_bf16(X), to_dev_bf16(bias)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y1 = wq.qgemm(Xd, dw, bias=bd, stream=s)
        y2 = wq.qgemm(Xd, dw, bias=bd, stream=s)
    s.synchronize()
    wq.check_device_status(s)
    assert torch.equal(y1, y2)
    _assert_close(from_dev_bf16(y1), _ref(X, W, bias, 8), "side stream")


def test_m_zero_is_a_no_op():
    dw = wq.qgemm_pack(np.zeros((16, 128), np.float32), 4).to_device()
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = wq.qgemm(X, dw)
    assert y.shape == (0, 16)


# ----------------------------------------------------------------------------
# every workload at full size, in the launch configuration the bench times
# ----------------------------------------------------------------------------

FULL = [(cid, li) for cid in (1, 2, 3, 4, 5) for li in range(len(WL.workload(cid).linears))]


@pytest.mark.parametrize("cid,li", FULL)
def test_workload_full_size_sampled_rows(cid, li):
    lin = WL.workload(cid).linears[li]
    X, W, bias = WL.make_inputs(lin, cid, li)
    y, _ = gpu_qgemm(X, W, bias, lin.bits)
    group = lin.group
    p, s, b = O.pack_ref(W, lin.bits, group)
    g = np.random.default_rng(cid * 10 + li)
    rows = np.unique(np.concatenate([[0, lin.M - 1], g.choice(lin.M, size=min(lin.M, 48), replace=False)]))
    ref_rows = O.qgemm_ref_rows(rows, X, p, s, b, lin.bits, group, lin.K, bias)
    _assert_close(y[rows], ref_rows, f"{lin.name} sampled rows")
    # a property of every row at once: column sums equal (sum_m x_m) . Wq^T + M * bias
    yall = O.bf16_bits_to_f64(y)
    assert np.all(np.isfinite(yall))
    xsum = O.bf16_bits_to_f64(X).sum(axis=0)
    colsum_ref = O.wq_exact(p, s, b, lin.bits, group, lin.K) @ xsum
    if bias is not None:
        colsum_ref += lin.M * O.bf16_bits_to_f64(bias)
    assert O.rel_frobenius(yall.sum(axis=0), colsum_ref) < 1e-2


# ----------------------------------------------------------------------------
# failure reporting without a fault
# ----------------------------------------------------------------------------

def test_bounded_wait_reports_timeout_and_context_survives():
    assert wq.qgemm_get_device_status() == wq.QGEMM_OK
    wq.qgemm_debug_wait_timeout(2_000_000)  # 2 ms on a barrier nothing completes
    assert wq.qgemm_get_device_status() == wq.QGEMM_ERR_DEVICE_TIMEOUT
    assert wq.qgemm_get_device_status() == wq.QGEMM_OK  # read clears it
    # the context is still usable
    X, W, bias = WL.random_case(1, 4, 128, 128, 4, with_bias=False)
    y, _ = gpu_qgemm(X, W, bias, 4)
    _assert_close(y, _ref(X, W, bias, 4), "after timeout")


# ----------------------------------------------------------------------------
# launch overlap (QGEMM_FLAG_OVERLAP_PREVIOUS): the activations are read only
# after the previous kernel in the stream has finished
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 4, 8])
def test_overlap_reads_the_previous_kernels_output(bits):
    """A chain y1 = X W1^T, y2 = y1 W2^T with the second call overlapping the
    first: y2 must be the GEMM of the y1 that the first call produced."""
    M, K1, N1, N2 = 4, 1024, 1024, 2048
    X, W1, _ = WL.random_case(91 + bits, M, N1, K1, bits, with_bias=False)
    _, W2, bias2 = WL.random_case(92 + bits, M, N2, N1, bits, with_bias=True)
    d1, d2 = wq.qgemm_pack(W1, bits).to_device(), wq.qgemm_pack(W2, bits).to_device()
    Xd, b2 = to_dev_bf16(X), to_dev_bf16(bias2)
    for _ in range(3):  # repeat: each round re-writes y1 and y2 in place
        y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        y1 = wq.qgemm(Xd, d1, out=y1, path=SMALL)
        y2 = wq.qgemm(y1, d2, bias=b2, path=SMALL, overlap_previous=True)
        wq.check_device_status()
        y1_bits = from_dev_bf16(y1)
        _assert_close(y1_bits, _ref(X, W1, None, bits), "first")
        _assert_close(from_dev_bf16(y2), _ref(y1_bits, W2, bias2, bits), "second, overlapped")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_overlap_with_split_rows_reads_the_previous_kernels_output(bits):
    """The same chain with 16 tokens and N2 = 9728 in the overlapped call: 6
    16-row pairs per CTA, so the rows split into halves and the producer, not
    the consumers, waits for the previous grid before it copies the
    activations into the ring."""
    M, K1, N1, N2 = 16, 1024, 1024, 9728
    X, W1, _ = WL.random_case(191 + bits, M, N1, K1, bits, with_bias=False)
    _, W2, bias2 = WL.random_case(192 + bits, M, N2, N1, bits, with_bias=True)
    d1, d2 = wq.qgemm_pack(W1, bits).to_device(), wq.qgemm_pack(W2, bits).to_device()
    Xd, b2 = to_dev_bf16(X), to_dev_bf16(bias2)
    ref1 = _ref(X, W1, None, bits)
    for _ in range(2):
        y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        y1 = wq.qgemm(Xd, d1, out=y1, path=SMALL)
        y2 = wq.qgemm(y1, d2, bias=b2, path=SMALL, overlap_previous=True)
        wq.check_device_status()
        y1_bits = from_dev_bf16(y1)
        _assert_close(y1_bits, ref1, "first")
        _assert_close(from_dev_bf16(y2), _ref(y1_bits, W2, bias2, bits), "second, overlapped, split rows")


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_large_path_overlap_reads_and_writes_after_the_previous_kernel(bits):
    """The tile path with launch overlap. A chain y1 = X W1^T, y2 = y1 W2^T
    (the second reads what the first wrote); a gated residual update of y1 in
    place (it reads y1 as its residual); and a call whose output buffer the
    previous call also wrote (its stores must land last)."""
    M, K1, N1, N2 = 300, 1024, 2048, 1536
    X, W1, _ = WL.random_case(391 + bits, M, N1, K1, bits, with_bias=False)
    _, W2, bias2 = WL.random_case(392 + bits, M, N2, N1, bits, with_bias=True)
    _, W3, _ = WL.random_case(393 + bits, M, N1, K1, bits, with_bias=False)
    d1, d2, d3 = (wq.qgemm_pack(w, bits).to_device() for w in (W1, W2, W3))
    Xd, b2 = to_dev_bf16(X), to_dev_bf16(bias2)
    g_bits = _bf16_normal(394 + bits, (N1,))
    gd = to_dev_bf16(g_bits)
    group = wq.GROUP_OF_BITS[bits]
    for _ in range(2):
        y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        y1 = wq.qgemm(Xd, d1, out=y1, path=LARGE)
        y2 = wq.qgemm(y1, d2, bias=b2, path=LARGE, overlap_previous=True)
        wq.check_device_status()
        y1_bits = from_dev_bf16(y1)
        _assert_close(y1_bits, _ref(X, W1, None, bits), "first")
        _assert_close(from_dev_bf16(y2), _ref(y1_bits, W2, bias2, bits), "second, overlapped")
        # y1 <- y1 + gate * (X W3^T), in place, overlapping the kernel that wrote y1
        y1 = wq.qgemm(Xd, d1, out=y1, path=LARGE)
        wq.qgemm_fused(Xd, d3, wq.QGEMM_EPI_RESIDUAL_GATE, residual=y1, gate=gd, out=y1, path=LARGE,
                       overlap_previous=True)
        wq.check_device_status()
        p3, s3, b3 = O.pack_ref(W3, bits, group)
        ref = O.qgemm_ref_epilogue(X, p3, s3, b3, bits, group, K1, None, wq.QGEMM_EPI_RESIDUAL_GATE, y1_bits, g_bits)
        _assert_close(from_dev_bf16(y1), ref, "residual update in place, overlapped")
        # two calls into one buffer: the overlapped second one's output stands
        buf = torch.empty((M, N1), dtype=torch.bfloat16, device="cuda")
        wq.qgemm(Xd, d1, out=buf, path=LARGE)
        wq.qgemm(Xd, d3, out=buf, path=LARGE, overlap_previous=True)
        wq.check_device_status()
        _assert_close(from_dev_bf16(buf), _ref(X, W3, None, bits), "same output buffer, overlapped")


def test_overlap_after_a_torch_kernel_and_in_a_graph():
    """The previous kernel is a plain torch one (no trigger of its own), and the
    same overlapped call captured in a CUDA graph gives the same result."""
    M, N, K, bits = 3, 1536, 2048, 4
    X, W, bias = WL.random_case(95, M, N, K, bits, with_bias=True)
    dw = wq.qgemm_pack(W, bits).to_device()
    src, bd = to_dev_bf16(X), to_dev_bf16(bias)
    Xd = torch.zeros_like(src)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    Xd.copy_(src)  # a device kernel writes X right before the call
    wq.qgemm(Xd, dw, bias=bd, out=out, path=SMALL, overlap_previous=True)
    wq.check_device_status()
    y_eager = from_dev_bf16(out)
    _assert_close(y_eager, _ref(X, W, bias, bits), "eager")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        Xd.copy_(src)
        wq.qgemm(Xd, dw, bias=bd, out=out, path=SMALL, overlap_previous=True)
    out.zero_()
    Xd.zero_()
    g.replay()
    torch.cuda.synchronize()
    wq.check_device_status()
    assert np.array_equal(from_dev_bf16(out), y_eager)
    del g


# ----------------------------------------------------------------------------
# fused epilogues (qgemm_fused): tanh GELU and the gated residual update
# ----------------------------------------------------------------------------

def _bf16_normal(seed, shape, scale=1.0):
    g = np.random.default_rng(np.random.SeedSequence([7, seed] + list(shape)))
    return WL.f32_to_bf16_bits((scale * g.standard_normal(shape)).astype(np.float32))


def _fused_case(bits, M, N, K, op, seed, path, in_place=False):
    X, W, bias = WL.random_case(seed, M, N, K, bits, with_bias=True)
    r_bits, g_bits = _bf16_normal(seed, (M, N)), _bf16_normal(seed + 1, (N,))
    dw = wq.qgemm_pack(W, bits).to_device()
    Xd, bd = to_dev_bf16(X), to_dev_bf16(bias)
    rd, gd = to_dev_bf16(r_bits), to_dev_bf16(g_bits)
    out = rd if in_place else None
    y = wq.qgemm_fused(Xd, dw, op, bias=bd, residual=rd, gate=gd, out=out, path=path)
    wq.check_device_status()
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    ref = O.qgemm_ref_epilogue(X, p, s, b, bits, group, K, bias, op, r_bits, g_bits)
    return from_dev_bf16(y), ref


@pytest.mark.parametrize("op", [wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("path,M", [(SMALL, 1), (SMALL, 13), (SMALL, 29), (SMALL, 45), (LARGE, 300)])
def test_fused_epilogue_parity(op, bits, path, M):
    y, ref = _fused_case(bits, M, 400, 768, op, 100 + 10 * op + bits + M, path)
    _assert_close(y, ref, f"op={op} bits={bits} path={path} M={M}")


@pytest.mark.parametrize("op", [wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE])
@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_fused_epilogue_with_split_rows(op, bits):
    """The fused epilogues on the small-M path with 16 tokens and 6 16-row
    pairs per CTA (N = 12272): rows split into halves, activations in the ring."""
    y, ref = _fused_case(bits, 16, 12272, 512, op, 300 + 10 * op + bits, SMALL)
    _assert_close(y, ref, f"split rows op={op} bits={bits}")


@pytest.mark.parametrize("path,M", [(SMALL, 5), (SMALL, 27), (SMALL, 50), (LARGE, 257)])
def test_fused_residual_update_in_place(path, M):
    """out may be the residual itself: the same bits as the out-of-place call."""
    y_out, ref = _fused_case(4, M, 528, 512, wq.QGEMM_EPI_RESIDUAL_GATE, 77, path)
    y_in, _ = _fused_case(4, M, 528, 512, wq.QGEMM_EPI_RESIDUAL_GATE, 77, path, in_place=True)
    assert np.array_equal(y_in, y_out)
    _assert_close(y_in, ref, "in place")


def test_fused_none_equals_plain_qgemm():
    X, W, bias = WL.random_case(5, 300, 256, 512, 8, with_bias=True)
    dw = wq.qgemm_pack(W, 8).to_device()
    Xd, bd = to_dev_bf16(X), to_dev_bf16(bias)
    for path in (SMALL, LARGE):
        Xp = Xd[:16] if path == SMALL else Xd
        a = wq.qgemm(Xp, dw, bias=bd, path=path)
        b = wq.qgemm_fused(Xp, dw, wq.QGEMM_EPI_NONE, bias=bd, path=path)
        wq.check_device_status()
        assert torch.equal(a, b)


def test_fused_gelu_mlp_up_full_size_sampled_rows():
    """The MLP up projection of the FLUX workload with its GELU fused, checked
    on sampled rows against the oracle."""
    lin = WL.workload(2).linears[0]
    X, W, bias = WL.make_inputs(lin, 2, 0)
    dw = wq.qgemm_pack(W, lin.bits).to_device()
    y = from_dev_bf16(wq.qgemm_fused(to_dev_bf16(X), dw, wq.QGEMM_EPI_GELU_TANH))
    wq.check_device_status()
    p, s, b = O.pack_ref(W, lin.bits, lin.group)
    rows = np.arange(0, lin.M, 257)
    ref = O.gelu_tanh_ref(O.qgemm_ref_rows(rows, X, p, s, b, lin.bits, lin.group, lin.K, None))
    _assert_close(y[rows], ref, "mlp_up + gelu sampled rows")


# ----------------------------------------------------------------------------
# packing on the device: the host packer's bytes, bit for bit
# ----------------------------------------------------------------------------

def _edge_rows(g, K):
    rows = [np.zeros(K), np.full(K, -0.0), np.resize([0.0, -0.0], K), np.full(K, 0.125),
            g.standard_normal(K) * 1e-7, g.standard_normal(K) * 1e-9, g.standard_normal(K) * 1000.0,
            np.resize([-1.0, 1.0], K), np.resize(np.arange(64) * 0.5 - 3.75, K),
            np.resize([0.0, 1e-30, -1e-30, 3.0], K)]
    return np.concatenate([np.stack(rows), g.standard_normal((22, K)) * 0.02]).astype(np.float32)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_pack_device_matches_host_packer(bits):
    g = np.random.default_rng(300 + bits)
    K = 1024
    if bits == 1:
        W = np.concatenate([WL.make_w(5, 1, 96, K, "binary", 128), _edge_rows(g, K)])
    elif bits == 2:
        W = np.concatenate([WL.make_w(3, 0, 96, K, "ternary", 128), _edge_rows(g, K)])
    else:
        W = np.concatenate([WL.make_w(1, 0, 96, K, "normal"), _edge_rows(g, K)])
    if bits == 1:
        # groups at and next to fp16 ties of the exact mean, tails over many binades
        tie = np.full((16, K), 2.0 ** -38)       # 16 rows: N stays a multiple of 16 for the GEMM below
        for i in range(12):
            tie[i, (37 * i) % K] = 1049088.0
        tie[12:, :128] = 0.0
        tie[12:, 5] = 1049088.0
        W = np.concatenate([W, tie.astype(np.float32)])
    host = wq.qgemm_pack(W, bits)
    dev = wq.qgemm_pack_device(torch.from_numpy(W).cuda(), bits)
    wq.check_device_status()
    p, s, b = O.pack_ref(W, bits, wq.GROUP_OF_BITS[bits])
    dev_s = dev.scales.cpu().numpy().view(np.uint16).reshape(host.scales.shape)
    # the device packer against the oracle directly, and against the host packer
    assert np.array_equal(dev.packed.cpu().numpy(), p)
    assert np.array_equal(dev_s, s.view(np.uint16))
    assert np.array_equal(dev.packed.cpu().numpy(), host.packed)
    assert np.array_equal(dev_s, host.scales.view(np.uint16))
    if bits > 2:
        dev_b = dev.biases.cpu().numpy().view(np.uint16).reshape(host.biases.shape)
        assert np.array_equal(dev_b, b.view(np.uint16))
        assert np.array_equal(dev_b, host.biases.view(np.uint16))
    # and the device-packed weights run the GEMM like the host-packed ones
    X, _, bias = WL.random_case(bits, 5, W.shape[0], K, bits, with_bias=True)
    Xd, bd = to_dev_bf16(X), to_dev_bf16(bias)
    y1 = wq.qgemm(Xd, dev, bias=bd)
    y2 = wq.qgemm(Xd, host.to_device(), bias=bd)
    wq.check_device_status()
    assert torch.equal(y1, y2)


def test_pack_device_reports_bad_data_through_the_status_word():
    W = torch.zeros((16, 128), dtype=torch.float32, device="cuda")
    W[3, 7] = float("nan")
    wq.qgemm_pack_device(W, 4)
    assert wq.qgemm_get_device_status() == wq.QGEMM_ERR_NONFINITE
    W[3, 7] = 0.0
    W[0, 0], W[0, 1] = -7e5, 7e5          # range / 15 overflows fp16
    wq.qgemm_pack_device(W, 4)
    assert wq.qgemm_get_device_status() == wq.QGEMM_ERR_UNSUPPORTED
    W[0, 0], W[0, 1] = 0.0, 0.0
    wq.qgemm_pack_device(W, 4)
    assert wq.qgemm_get_device_status() == wq.QGEMM_OK


def test_binding_refuses_buffers_off_the_device():
    """The library takes raw pointers and launches on X's device, so the
    binding refuses a host buffer before any launch; the normal call works."""
    dw = wq.qgemm_pack(np.zeros((256, 256), dtype=np.float32), 4).to_device("cuda")
    X = torch.zeros((2, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="out is on cpu"):
        wq.qgemm(X, dw, out=torch.empty((2, 256), dtype=torch.bfloat16))
    host_packed = wq.DeviceWeights(dw.N, dw.K, dw.bits, dw.group, dw.packed.cpu(), dw.scales, dw.biases)
    with pytest.raises(ValueError, match="W.packed is on cpu"):
        wq.qgemm(X, host_packed)
    with pytest.raises(ValueError, match="out is on cpu"):
        wq.qgemm_dequant_tile(dw, out=torch.empty((256, 256), dtype=torch.bfloat16))
    y = wq.qgemm(X, dw)
    wq.check_device_status()
    assert y.shape == (2, 256) and bool(torch.all(y == 0))
