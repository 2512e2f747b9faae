"""The small-M kernel's K-split launches (a thread-block cluster per row
block, each CTA streaming a slice of K, partial sums met over distributed
shared memory) and its streaming-floor mode, through the C ABI, against the
oracle.

On 148 SMs the narrow FLUX shapes take the split: 3072 x 12288 and
3072 x 3072 run as 48 row blocks of 64 rows x 3 K slices (144 CTAs) in every
format; the smaller ragged shapes of the other parity tests take 2- to 4-slice
clusters as well.
"""
import numpy as np
import pytest
import torch

import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL
from gpu_util import from_dev_bf16, gpu_qgemm, to_dev_bf16

pytestmark = pytest.mark.gpu

SMALL = wq.QGEMM_PATH_SMALL_M


def _ref(X, W, bias, bits):
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    return O.qgemm_ref(X, p, s, b, bits, group, W.shape[1], bias)


def _assert_close(y_bits, ref, what=""):
    y = O.bf16_bits_to_f64(y_bits)
    assert np.all(np.isfinite(y)), what
    rf, ma = O.rel_frobenius(y, ref), O.max_abs_rel(y, ref)
    assert rf <= O.REL_FROB_TOL and ma <= O.MAX_ABS_TOL, f"{what}: rel_frob={rf:.3e} max_abs={ma:.3e}"


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("N,K", [(3072, 12288), (3072, 3072)])
def test_k_split_narrow_shapes(bits, M, N, K):
    X, W, bias = WL.random_case(N // 64 + K // 512 + M + bits, M, N, K, bits, with_bias=True)
    y, _ = gpu_qgemm(X, W, bias, bits)          # the default path: small for M <= 16
    _assert_close(y, _ref(X, W, bias, bits), f"bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [17, 32])
@pytest.mark.parametrize("N,K", [(3072, 12288), (3072, 3072)])
def test_k_split_narrow_shapes_32_tokens(bits, M, N, K):
    """32-token CTAs (4 MMA column tiles, activations through the ring) on
    the K-split shapes."""
    X, W, bias = WL.random_case(N // 64 + K // 512 + M + bits, M, N, K, bits, with_bias=True)
    y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
    _assert_close(y, _ref(X, W, bias, bits), f"bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [9, 25])
def test_k_split_one_hot_rows_are_bit_exact(bits, M):
    """One non-zero activation per token: every K slice but one contributes
    exact zeros, so the cluster's sum is the dequantised weight itself (16-
    and 32-token CTAs)."""
    N, K = 3072, 3072
    g = np.random.default_rng(31 + bits)
    _, W, _ = WL.random_case(41 + bits, 1, N, K, bits, with_bias=False)
    ks = g.choice(K, size=M, replace=False)
    X = np.zeros((M, K), dtype=np.uint16)
    X[np.arange(M), ks] = 0x3F80
    y, _ = gpu_qgemm(X, W, None, bits, path=SMALL)
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    # the small path multiplies s*q + b exactly in fp32: one product, one rounding to bf16
    wq_f32 = O.wq_exact(p, s, b, bits, group, K).astype(np.float32)
    expect = WL.f32_to_bf16_bits(np.ascontiguousarray(wq_f32[:, ks].T))
    assert np.array_equal(y, expect)


@pytest.mark.parametrize("op", [wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE])
@pytest.mark.parametrize("bits", [4, 8])
def test_k_split_fused_epilogues(op, bits):
    M, N, K = 5, 3072, 12288
    X, W, bias = WL.random_case(500 + op + bits, M, N, K, bits, with_bias=True)
    g = np.random.default_rng(600 + op + bits)
    r_bits = WL.f32_to_bf16_bits(g.standard_normal((M, N)).astype(np.float32))
    g_bits = WL.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
    dw = wq.qgemm_pack(W, bits).to_device()
    y = wq.qgemm_fused(to_dev_bf16(X), dw, op, bias=to_dev_bf16(bias), residual=to_dev_bf16(r_bits),
                       gate=to_dev_bf16(g_bits))
    wq.check_device_status()
    group = wq.GROUP_OF_BITS[bits]
    p, s, b = O.pack_ref(W, bits, group)
    ref = O.qgemm_ref_epilogue(X, p, s, b, bits, group, K, bias, op, r_bits, g_bits)
    _assert_close(from_dev_bf16(y), ref, f"fused op={op} bits={bits}")


@pytest.mark.parametrize("bits", [2, 8])
def test_k_split_overlap_reads_the_previous_kernels_output(bits):
    """y1 = X W1^T (12288 rows), then y2 = y1 W2^T with W2 [3072, 12288], a
    K-split launch overlapping the first call: y2 is the GEMM of y1 as the
    first call wrote it."""
    M, K1, N1, N2 = 4, 3072, 12288, 3072
    X, W1, _ = WL.random_case(71 + bits, M, N1, K1, bits, with_bias=False)
    _, W2, bias2 = WL.random_case(72 + bits, M, N2, N1, bits, with_bias=True)
    d1, d2 = wq.qgemm_pack(W1, bits).to_device(), wq.qgemm_pack(W2, bits).to_device()
    Xd, b2 = to_dev_bf16(X), to_dev_bf16(bias2)
    for _ in range(2):
        y1 = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        y1 = wq.qgemm(Xd, d1, out=y1, path=SMALL)
        y2 = wq.qgemm(y1, d2, bias=b2, path=SMALL, overlap_previous=True)
        wq.check_device_status()
        y1_bits = from_dev_bf16(y1)
        _assert_close(y1_bits, _ref(X, W1, None, bits), "first")
        _assert_close(from_dev_bf16(y2), _ref(y1_bits, W2, bias2, bits), "second, overlapped, K-split")


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M", [33, 47, 64])
@pytest.mark.parametrize("N,K", [(3072, 12288), (1008, 1024)])
def test_small_path_past_32_tokens(bits, M, N, K):
    """M = 33..64 on the small path: launches of 32 token rows back to back
    (the later ones overlapping the one before), the last one ragged."""
    X, W, bias = WL.random_case(900 + M + bits + N // 8, M, N, K, bits, with_bias=True)
    y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
    _assert_close(y, _ref(X, W, bias, bits), f"bits={bits} M={M} N={N} K={K}")


@pytest.mark.parametrize("bits", [2, 8])
@pytest.mark.parametrize("M", [47, 64])
def test_small_path_past_32_tokens_equals_calls_on_the_pieces(bits, M):
    """Past 32 tokens each launch is the one a call on its 32 (or fewer) rows
    makes: the same bits as separate calls on the pieces, fused residual
    update in place included."""
    N, K = 3072, 3072
    X, W, bias = WL.random_case(950 + M + bits, M, N, K, bits, with_bias=True)
    dw = wq.qgemm_pack(W, bits).to_device()
    Xd, bd = to_dev_bf16(X), to_dev_bf16(bias)
    y = wq.qgemm(Xd, dw, bias=bd, path=SMALL)
    parts = [wq.qgemm(Xd[m0:m0 + 32].contiguous(), dw, bias=bd, path=SMALL) for m0 in range(0, M, 32)]
    wq.check_device_status()
    assert torch.equal(y, torch.cat(parts))
    g = np.random.default_rng(960 + M + bits)
    r = to_dev_bf16(WL.f32_to_bf16_bits(g.standard_normal((M, N)).astype(np.float32)))
    gate = to_dev_bf16(WL.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32)))
    whole = r.clone()
    wq.qgemm_fused(Xd, dw, wq.QGEMM_EPI_RESIDUAL_GATE, bias=bd, residual=whole, gate=gate, out=whole, path=SMALL)
    pieces = []
    for m0 in range(0, M, 32):
        rp = r[m0:m0 + 32].clone()
        wq.qgemm_fused(Xd[m0:m0 + 32].contiguous(), dw, wq.QGEMM_EPI_RESIDUAL_GATE, bias=bd, residual=rp, gate=gate,
                       out=rp, path=SMALL)
        pieces.append(rp)
    wq.check_device_status()
    assert torch.equal(whole, torch.cat(pieces))


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
@pytest.mark.parametrize("M,N,K", [(1, 12288, 3072), (16, 12288, 3072), (1, 3072, 12288), (16, 12272, 512),
                                   (48, 3072, 3072)])
def test_stream_floor_runs_clean_and_leaves_the_output_alone(bits, M, N, K):
    """The streaming-floor launch (same grid, clusters and ring as the GEMV,
    no arithmetic) completes with a clean status, in both launch modes, and a
    GEMV after it is still correct."""
    X, W, bias = WL.random_case(800 + M + bits, M, N, K, bits, with_bias=True)
    dw = wq.qgemm_pack(W, bits).to_device()
    Xd = to_dev_bf16(X)
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    wq.qgemm_debug_stream(Xd, dw)
    wq.qgemm_debug_stream(Xd, dw, overlap_previous=True)
    wq.check_device_status()
    assert torch.all(out == 7.0)
    y = wq.qgemm(Xd, dw, bias=to_dev_bf16(bias), out=out)
    wq.check_device_status()
    _assert_close(from_dev_bf16(y), _ref(X, W, bias, bits), "after the floor launches")
