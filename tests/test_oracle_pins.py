"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against an independent fact: CPython's IEEE half
packing, torch's bf16 conversion, hand-derived bit layouts, closed forms of
the RTN quantiser, exact round trips of constructed weights, and a
pure-Python triple loop. A plausible slip anywhere in the oracle (a dropped
bias term, a wrong sign, a swapped nibble, a transposed operand, a wrong
rounding mode) fails at least one of them.
"""
import math
import struct

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL


# ----------------------------------------------------------------------------
# rounding helpers
# ----------------------------------------------------------------------------

def _struct_half_bits(x: float) -> int:
    return struct.unpack("<H", struct.pack("<e", x))[0]


def test_fp16_rn_every_half_and_midpoint():
    """Every finite fp16 value maps to itself; every midpoint ties to even.

    Reference: CPython's ``struct.pack('e')`` (IEEE 754 binary16, round half to even).
    """
    bits = np.arange(0, 0x7C00, dtype=np.uint16)          # +0 .. max finite
    vals = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(O.fp16_rn(vals).view(np.uint16), bits)
    assert np.array_equal(O.fp16_rn(-vals).view(np.uint16), bits | 0x8000)
    mids = (vals[:-1] + vals[1:]) / 2.0                    # exact in fp64
    got = O.fp16_rn(mids).view(np.uint16)
    ref = np.array([_struct_half_bits(float(m)) for m in mids], dtype=np.uint16)
    assert np.array_equal(got, ref)
    # ties go to the even neighbour
    assert np.all(got % 2 == 0)


def test_fp16_rn_random_doubles_match_struct():
    g = np.random.default_rng(11)
    x = np.concatenate([g.standard_normal(20000) * 10.0 ** g.integers(-9, 5, 20000),
                        g.uniform(-65504, 65504, 2000)])
    got = O.fp16_rn(x).view(np.uint16)
    ref = np.array([_struct_half_bits(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rn_matches_torch_on_stratified_fp32_patterns():
    """All 65536 upper halves x low halves {0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, random}."""
    hi = np.arange(65536, dtype=np.uint32) << 16
    lows = [0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF]
    g = np.random.default_rng(3)
    pats = np.concatenate([hi | np.uint32(lo) for lo in lows]
                          + [hi | g.integers(0, 65536, 65536).astype(np.uint32)])
    f = pats.view(np.float32)
    finite = np.isfinite(f)
    got = O.bf16_rn_bits(f[finite])
    ref = torch.from_numpy(f[finite].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    # NaN stays NaN
    nan_out = O.bf16_rn_bits(f[np.isnan(f)])
    assert np.all((nan_out & 0x7F80) == 0x7F80) and np.all((nan_out & 0x7F) != 0)


def test_bf16_rn_ties_to_even_examples():
    # 1 + 2^-8 is halfway between bf16 1.0 (0x3F80) and 1 + 2^-7 (0x3F81): ties to 0x3F80
    assert O.bf16_rn_bits(np.float32(1.0 + 2.0 ** -8))[()] == 0x3F80
    # 1 + 3*2^-8 is halfway between 0x3F81 and 0x3F82: ties to the even 0x3F82
    assert O.bf16_rn_bits(np.float32(1.0 + 3 * 2.0 ** -8))[()] == 0x3F82
    # just above the tie rounds up
    assert O.bf16_rn_bits(np.float32(1.0 + 2.0 ** -8 + 2.0 ** -20))[()] == 0x3F81


# ----------------------------------------------------------------------------
# bit layout
# ----------------------------------------------------------------------------

def test_layout_hand_derived_4bit():
    # codes 1..8 for k = 0..7. Even k in the low half-word, odd k in the high one:
    # bits 0-3 k0=1, 4-7 k2=3, 8-11 k4=5, 12-15 k6=7, 16-19 k1=2, 20-23 k3=4,
    # 24-27 k5=6, 28-31 k7=8  ->  word 0x86427531, little-endian bytes 31 75 42 86
    packed = O.pack_codes(np.array([[1, 2, 3, 4, 5, 6, 7, 8]]), 4)
    assert packed.tolist() == [[0x31, 0x75, 0x42, 0x86]]


def test_layout_hand_derived_8bit():
    packed = O.pack_codes(np.array([[0, 1, 127, 128, 255, 7, 9, 200]]), 8)
    assert packed.tolist() == [[0, 1, 127, 128, 255, 7, 9, 200]]


def test_layout_hand_derived_ternary():
    # t = +1 at k=0 (code 01 at bits 0-1), -1 at k=1 (code 11 at bits 16-17),
    # -1 at k=2 (11 at bits 2-3), +1 at k=15 (01 at bits 30-31), rest 0:
    # word = 0x1 | 0xC | 0x30000 | 0x40000000 = 0x4003000D -> bytes 0D 00 03 40
    t = np.zeros((1, 16), dtype=np.int64)
    t[0, 0], t[0, 1], t[0, 2], t[0, 15] = 1, -1, -1, 1
    assert O.pack_codes(t, 2).tolist() == [[0x0D, 0x00, 0x03, 0x40]]


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_unpack_bijection_every_code_every_position(bits):
    values = [-1, 0, 1] if bits == 2 else list(range(1 << bits))
    per = O.codes_per_word(bits)
    K = per * len(values)
    rows = []
    for r in range(len(values)):
        rows.append([values[(r + k) % len(values)] for k in range(K)])
    codes = np.array(rows)
    # each value appears at each in-word position in some row
    for j in range(per):
        assert set(codes[:, j].tolist()) == set(values)
    packed = O.pack_codes(codes, bits)
    assert packed.shape == (len(values), K * bits // 8)
    assert np.array_equal(O.unpack_codes(packed, bits, K), codes)
    # and the map on bytes is onto the valid patterns: repacking an unpacked
    # random byte stream (affine formats) reproduces it exactly
    if bits != 2:
        g = np.random.default_rng(bits)
        raw = g.integers(0, 256, size=(5, 64), dtype=np.uint8)
        Kr = 64 * 8 // bits
        assert np.array_equal(O.pack_codes(O.unpack_codes(raw, bits, Kr), bits), raw)


def test_ternary_invalid_code_rejected():
    bad = np.array([[0x02, 0, 0, 0]], dtype=np.uint8)   # code 10 at k = 0
    with pytest.raises(ValueError):
        O.unpack_codes(bad, 2, 16)


def test_single_code_positions_match_layout_definition():
    """A lone code at each k lands at the bit the layout definition names."""
    for bits in (2, 4, 8):
        per = O.codes_per_word(bits)
        K = 2 * per
        for k in range(K):
            c = np.zeros((1, K), dtype=np.int64)
            c[0, k] = 1
            words = O.pack_codes(c, bits).view("<u4")[0]
            w, j = divmod(k, per)
            if bits == 8:
                expect_bit = 8 * j
            else:
                expect_bit = (16 if j % 2 else 0) + bits * (j // 2)
            assert int(words[w]) == 1 << expect_bit
            assert all(int(words[x]) == 0 for x in range(len(words)) if x != w)


# ----------------------------------------------------------------------------
# RTN quantiser: closed forms and exact round trips
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_affine_error_bound(bits):
    g = np.random.default_rng(5 + bits)
    W = (g.standard_normal((64, 512)) * 0.02).astype(np.float32)
    packed, s16, b16 = O.pack_ref(W, bits, 64)
    assert s16.shape == (8, 64) and b16.shape == (8, 64)     # at rest: [K/group, N]
    s16, b16 = s16.T, b16.T
    q = O.unpack_codes(packed, bits, 512)
    qmax = (1 << bits) - 1
    assert q.min() >= 0 and q.max() <= qmax
    s = np.repeat(s16.astype(np.float64), 64, axis=1)
    b = np.repeat(b16.astype(np.float64), 64, axis=1)
    Wg = W.astype(np.float64).reshape(64, 8, 64)
    lo = np.repeat(Wg.min(axis=2), 64, axis=1)
    hi = np.repeat(Wg.max(axis=2), 64, axis=1)
    err = np.abs(W.astype(np.float64) - (s * q + b))
    bound = s / 2 + np.abs(lo - b) + np.abs(hi - (b + qmax * s)) + 1e-12
    assert np.all(err <= bound)
    # unclamped entries are within half a step
    inner = (q > 0) & (q < qmax)
    assert np.all(err[inner] <= s[inner] / 2 * (1 + 1e-9))
    # the scale is the fp16 rounding of the range over 2^b - 1
    rng = Wg.max(axis=2) - Wg.min(axis=2)
    assert np.all(np.abs(s16.astype(np.float64) - rng / qmax) <= np.abs(rng / qmax) * 2.0 ** -11)


@pytest.mark.parametrize("bits", [4, 8])
def test_affine_exact_grid_is_recovered(bits):
    """A group laid exactly on lo + s*{0..2^b-1} (fp16 s and lo) packs back exactly."""
    qmax = (1 << bits) - 1
    g = np.random.default_rng(bits)
    N = 16
    s = np.array([2.0 ** -e for e in g.integers(4, 12, N)])
    lo = -np.array([float(np.float16(v)) for v in g.uniform(0.0, 0.5, N)])
    q_true = np.stack([g.permutation(np.concatenate([[0, qmax], g.integers(0, qmax + 1, 62)]))
                       for _ in range(N)])
    W = (lo[:, None] + s[:, None] * q_true).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), lo[:, None] + s[:, None] * q_true)  # exact in fp32
    packed, s16, b16 = O.pack_ref(W, bits, 64)
    assert np.array_equal(s16[0, :].astype(np.float64), s)
    assert np.array_equal(b16[0, :].astype(np.float64), lo)
    assert np.array_equal(O.unpack_codes(packed, bits, 64), q_true)


def test_affine_degenerate_groups():
    W = np.zeros((3, 64), dtype=np.float32)
    W[1, :] = 0.25                 # constant group
    W[2, :] = -0.0                 # negative zeros
    packed, s16, b16 = O.pack_ref(W, 4, 64)
    assert np.all(s16 == 0)
    assert b16[0, 1] == np.float16(0.25)
    assert np.all(O.unpack_codes(packed, 4, 64) == 0)
    wd = O.dequant_ref(packed, s16, b16, 4, 64, 64)
    assert np.all(wd[1] == 0.25) and np.all(wd[0] == 0) and np.all(wd[2] == 0)
    # a group of negative zeros stores a +0 bias, so it dequantises to +0 bits
    assert b16.view(np.uint16)[0, 2] == 0
    assert np.all(O.dequant_ref_bits(packed, s16, b16, 4, 64, 64)[2] == 0)


def test_ternary_constructed_weights_round_trip_exactly():
    """W = s16 * t (the ternary workload's construction) packs back to t and s16."""
    lin = WL.workload(3).linears[0]
    W = WL.make_w(3, 0, 256, lin.K, "ternary", 128)
    g = np.random.default_rng(np.random.SeedSequence([0, 3, 0, 5, 0]))
    t = g.integers(-1, 2, size=(lin.N, lin.K))[:256].astype(np.int64)
    packed, s16, b = O.pack_ref(W, 2, 128)
    assert b is None
    codes = O.unpack_codes(packed, 2, lin.K)
    assert set(np.unique(codes).tolist()) <= {-1, 0, 1}
    assert np.array_equal(codes, t)
    recon = np.repeat(s16.T.astype(np.float32), 128, axis=1) * codes
    assert np.array_equal(recon.astype(np.float32), W)


def test_ternary_rtn_threshold_and_clamp():
    w = np.zeros((1, 128), dtype=np.float32)
    w[0, 0] = 1.0                  # the absmax: scale 1.0
    w[0, 1] = 0.5                  # exactly half: rint(0.5) = 0 (ties to even)
    w[0, 2] = 0.5000001            # just above half -> +1
    w[0, 3] = -0.75                # -> -1
    w[0, 4] = -0.25                # -> 0
    packed, s16, _ = O.pack_ref(w, 2, 128)
    t = O.unpack_codes(packed, 2, 128)
    assert s16[0, 0] == 1.0
    assert t[0, :5].tolist() == [1, 0, 1, -1, 0]


def test_pack_rejects_bad_inputs():
    W = np.zeros((2, 128), dtype=np.float32)
    with pytest.raises(ValueError):
        O.pack_ref(W, 3, 64)
    with pytest.raises(ValueError):
        O.pack_ref(W, 4, 128)
    with pytest.raises(ValueError):
        O.pack_ref(np.zeros((2, 96), np.float32), 4, 64)
    W[0, 0] = np.nan
    with pytest.raises(ValueError):
        O.pack_ref(W, 4, 64)
    big = np.zeros((1, 64), dtype=np.float32)
    big[0, 0] = -1e6
    big[0, 1] = 1e6
    with pytest.raises(OverflowError):
        O.pack_ref(big, 4, 64)


# ----------------------------------------------------------------------------
# dequantisation
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [4, 8])
def test_dequant_exact_when_representable(bits):
    """s16 = 1/2, b16 = -4: every s*q + b is a bf16 value, so dequant is exact."""
    qmax = (1 << bits) - 1
    q = np.resize(np.arange(qmax + 1), (4, 256))
    packed = O.pack_codes(q, bits)
    s16 = np.full((4, 4), 0.5, dtype=np.float16)
    b16 = np.full((4, 4), -4.0, dtype=np.float16)
    wd = O.dequant_ref(packed, s16, b16, bits, 64, 256)
    assert np.array_equal(wd, 0.5 * q - 4.0)


@pytest.mark.parametrize("bits", [4, 8])
def test_dequant_monotone_and_within_bf16_rounding(bits):
    g = np.random.default_rng(20 + bits)
    W = (g.standard_normal((32, 256)) * 0.02).astype(np.float32)
    packed, s16, b16 = O.pack_ref(W, bits, 64)
    q = O.unpack_codes(packed, bits, 256)
    wd = O.dequant_ref(packed, s16, b16, bits, 64, 256)
    exact = O.wq_exact(packed, s16, b16, bits, 64, 256)
    # bf16 keeps 8 significant bits: RNE error <= half an ulp <= 2^-8 relative (+ the fp32 step)
    assert np.all(np.abs(wd - exact) <= np.abs(exact) * (2.0 ** -8 + 2.0 ** -23) + 1e-45)
    # within a group, larger codes never give smaller weights (s16 >= 0)
    for n in range(32):
        for gi in range(4):
            sl = slice(64 * gi, 64 * gi + 64)
            order = np.argsort(q[n, sl], kind="stable")
            assert np.all(np.diff(wd[n, sl][order]) >= 0)
    # q = 0 gives the bias rounded to bf16
    zero = q == 0
    b = np.repeat(b16.T, 64, axis=1)
    tb = torch.from_numpy(b.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(wd[zero], tb[zero].astype(np.float64))


def test_dequant_final_rounding_matches_torch_bf16():
    """The bf16 step of the dequant agrees with torch's own fp32->bf16 conversion."""
    g = np.random.default_rng(31)
    W = (g.standard_normal((16, 256)) * 0.05).astype(np.float32)
    packed, s16, b16 = O.pack_ref(W, 4, 64)
    exact32 = O.wq_exact(packed, s16, b16, 4, 64, 256).astype(np.float32)
    tb = torch.from_numpy(exact32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.dequant_ref_bits(packed, s16, b16, 4, 64, 256), tb)


def test_ternary_dequant_is_signed_scale():
    g = np.random.default_rng(8)
    t = g.integers(-1, 2, size=(8, 256))
    s16 = g.uniform(0.01, 0.05, size=(8, 2)).astype(np.float16)      # [N, K/128]
    packed = O.pack_codes(t, 2)
    bits = O.dequant_ref_bits(packed, np.ascontiguousarray(s16.T), None, 2, 128, 256)
    sb = torch.from_numpy(np.repeat(s16.astype(np.float32), 128, axis=1)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(O.bf16_bits_to_f64(bits), t * sb.astype(np.float64))
    assert np.all(bits[t == 0] == 0)                      # +0, not -0
    assert np.all((bits[t < 0] & 0x8000) == 0x8000)


# ----------------------------------------------------------------------------
# the matmul
# ----------------------------------------------------------------------------

def _naive(X, Wq, bias):
    M, K = X.shape
    N = Wq.shape[0]
    out = [[0.0] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc = math.fsum([acc, float(X[m, k]) * float(Wq[n, k])])
            out[m][n] = acc + (float(bias[n]) if bias is not None else 0.0)
    return np.array(out)


@pytest.mark.parametrize("bits,K", [(4, 128), (8, 64), (2, 128)])
def test_qgemm_ref_equals_naive_triple_loop(bits, K):
    X, W, bias = WL.random_case(1, 5, 7, K, bits, with_bias=True)
    group = 128 if bits == 2 else 64
    packed, s, b = O.pack_ref(W, bits, group)
    ref = O.qgemm_ref(X, packed, s, b, bits, group, K, bias)
    Wq = O.wq_exact(packed, s, b, bits, group, K)
    brute = _naive(O.bf16_bits_to_f64(X), Wq, O.bf16_bits_to_f64(bias))
    assert np.allclose(ref, brute, rtol=1e-12, atol=1e-14)


def test_qgemm_ref_orientation():
    """out[m, n] pairs activation row m with weight row n (not its transpose)."""
    K = 64
    W = np.zeros((3, K), dtype=np.float32)
    for n in range(3):
        W[n, :] = np.linspace(-1, 1, K) * (n + 1)
    X = np.zeros((2, K), dtype=np.uint16)
    X[0, 5] = 0x3F80                 # 1.0 at k = 5
    X[1, 40] = 0x4000                # 2.0 at k = 40
    packed, s, b = O.pack_ref(W, 8, 64)
    ref = O.qgemm_ref(X, packed, s, b, 8, 64, K)
    Wq = O.wq_exact(packed, s, b, 8, 64, K)
    assert np.array_equal(ref[0], Wq[:, 5])
    assert np.array_equal(ref[1], 2 * Wq[:, 40])


def test_metrics():
    ref = np.array([[1.0, -2.0], [3.0, 4.0]])
    assert O.rel_frobenius(ref, ref) == 0.0
    assert abs(O.rel_frobenius(ref * 1.01, ref) - 0.01) < 1e-12
    assert abs(O.max_abs_rel(ref + 0.04, ref) - 0.01) < 1e-12
    assert abs(O.cosine(ref, 3 * ref) - 1.0) < 1e-15
    assert abs(O.cosine([1, 0], [0, 1])) < 1e-15


@pytest.mark.parametrize("bits,expect", [(4, 0.996), (8, 0.99998)])
def test_cosine_against_dense_matches_rtn_noise_model(bits, expect):
    """E cos(X Wq^T, X W^T) ~ cos(vec Wq, vec W); for Gaussian groups of 64 the
    RTN step is about range/(2^b - 1) with error variance step^2 / 12."""
    g = np.random.default_rng(42)
    W = (g.standard_normal((256, 1024)) * 0.02).astype(np.float32)
    packed, s, b = O.pack_ref(W, bits, 64)
    Wq = O.wq_exact(packed, s, b, bits, 64, 1024)
    c = O.cosine(Wq, W)
    tol = 2e-3 if bits == 4 else 2e-5
    assert abs(c - expect) < tol
    X = WL.f32_to_bf16_bits(g.standard_normal((64, 1024)).astype(np.float32))
    cy = O.cosine(O.qgemm_ref(X, packed, s, b, bits, 64, 1024), O.bf16_bits_to_f64(X) @ W.astype(np.float64).T)
    assert abs(cy - c) < 5 * (1 - c) + 1e-6


# ----------------------------------------------------------------------------
# fused epilogues
# ----------------------------------------------------------------------------

def test_gelu_tanh_matches_torch_and_its_identities():
    """Against torch's tanh-approximate GELU in fp64 (a library routine), at 0,
    far in both tails, and through the identity gelu(y) - gelu(-y) = y that
    the tanh form satisfies exactly."""
    y = np.concatenate([np.linspace(-12, 12, 4001), np.array([-1e3, -40.0, 0.0, 40.0, 1e3])])
    ref = torch.nn.functional.gelu(torch.from_numpy(y), approximate="tanh").numpy()
    got = O.gelu_tanh_ref(y)
    # fp64 rounding order differs only where 1 + tanh cancels (|difference| < 1e-15)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
    assert O.gelu_tanh_ref(0.0) == 0.0
    assert abs(O.gelu_tanh_ref(20.0) - 20.0) < 1e-12 and abs(O.gelu_tanh_ref(-20.0)) < 1e-12
    assert np.allclose(O.gelu_tanh_ref(y) - O.gelu_tanh_ref(-y), y, rtol=1e-12, atol=1e-12)
    # the constant inside the tanh: the slope at 0 is 1/2, the curvature sqrt(2/pi)
    h = 1e-5
    assert abs((O.gelu_tanh_ref(h) - O.gelu_tanh_ref(-h)) / (2 * h) - 0.5) < 1e-9
    second = (O.gelu_tanh_ref(h) - 2 * O.gelu_tanh_ref(0.0) + O.gelu_tanh_ref(-h)) / h ** 2
    assert abs(second - math.sqrt(2 / math.pi)) < 1e-4


def test_residual_gate_epilogue_special_cases():
    """gate = 0 gives the residual exactly; residual 0 and gate 1 give y; the
    update is linear in the gate; and one hand-computed element."""
    rng = np.random.default_rng(3)
    y = rng.standard_normal((5, 8))
    r_bits = WL.f32_to_bf16_bits(rng.standard_normal((5, 8)).astype(np.float32))
    zeros, ones = (WL.f32_to_bf16_bits(np.full(8, v, np.float32)) for v in (0.0, 1.0))
    r = O.bf16_bits_to_f64(r_bits)
    assert np.array_equal(O.epilogue_ref(y, O.EPI_RESIDUAL_GATE, r_bits, zeros), r)
    assert np.array_equal(O.epilogue_ref(y, O.EPI_RESIDUAL_GATE, WL.f32_to_bf16_bits(np.zeros((5, 8), np.float32)),
                                         ones), y)
    g1 = WL.f32_to_bf16_bits(rng.standard_normal(8).astype(np.float32))
    g2 = WL.f32_to_bf16_bits(rng.standard_normal(8).astype(np.float32))
    g12 = WL.f32_to_bf16_bits((O.bf16_bits_to_f64(g1) + O.bf16_bits_to_f64(g2)).astype(np.float32))
    if np.array_equal(O.bf16_bits_to_f64(g12), O.bf16_bits_to_f64(g1) + O.bf16_bits_to_f64(g2)):
        lhs = O.epilogue_ref(y, O.EPI_RESIDUAL_GATE, r_bits, g12) - r
        rhs = (O.epilogue_ref(y, O.EPI_RESIDUAL_GATE, r_bits, g1) - r) + \
              (O.epilogue_ref(y, O.EPI_RESIDUAL_GATE, r_bits, g2) - r)
        assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    # out[0, 0] = r + g * y with r = 1.5, g = -0.25, y = 2: 1.0
    rr = WL.f32_to_bf16_bits(np.array([[1.5]], np.float32))
    gg = WL.f32_to_bf16_bits(np.array([-0.25], np.float32))
    assert O.epilogue_ref(np.array([[2.0]]), O.EPI_RESIDUAL_GATE, rr, gg)[0, 0] == 1.0
    # the gate indexes features (columns), not tokens
    gcol = WL.f32_to_bf16_bits(np.arange(8, dtype=np.float32))
    out = O.epilogue_ref(np.ones((5, 8)), O.EPI_RESIDUAL_GATE, WL.f32_to_bf16_bits(np.zeros((5, 8), np.float32)),
                         gcol)
    assert np.array_equal(out, np.broadcast_to(np.arange(8.0), (5, 8)))


def test_fused_reference_composes_the_plain_gemm():
    """qgemm_ref_epilogue is the plain reference followed by the epilogue."""
    X, W, bias = WL.random_case(41, 6, 64, 128, 4, with_bias=True)
    p, s, b = O.pack_ref(W, 4, 64)
    y = O.qgemm_ref(X, p, s, b, 4, 64, 128, bias)
    assert np.array_equal(O.qgemm_ref_epilogue(X, p, s, b, 4, 64, 128, bias, O.EPI_NONE), y)
    assert np.array_equal(O.qgemm_ref_epilogue(X, p, s, b, 4, 64, 128, bias, O.EPI_GELU_TANH), O.gelu_tanh_ref(y))
    with pytest.raises(ValueError):
        O.epilogue_ref(y, 7)


# ----------------------------------------------------------------------------
# the 1-bit format (Q1_0_g128)
# ----------------------------------------------------------------------------

def test_layout_hand_derived_1bit():
    # +1 at k = 0 (bit 0), k = 1 (bit 16), k = 30 (bit 15) and k = 31 (bit 31);
    # -1 elsewhere: word = 0x1 | 0x10000 | 0x8000 | 0x80000000 = 0x80018001
    c = -np.ones((1, 32), dtype=np.int64)
    c[0, [0, 1, 30, 31]] = 1
    assert O.pack_codes(c, 1).tolist() == [[0x01, 0x80, 0x01, 0x80]]
    with pytest.raises(ValueError):
        O.pack_codes(np.zeros((1, 32), dtype=np.int64), 1)   # 0 is not a 1-bit code


def test_1bit_pack_unpack_bijection_and_every_byte():
    g = np.random.default_rng(11)
    c = np.where(g.integers(0, 2, size=(7, 256)) == 1, 1, -1)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c, 1), 1, 256), c)
    raw = g.integers(0, 256, size=(5, 64), dtype=np.uint8)      # every byte pattern is valid
    assert np.array_equal(O.pack_codes(O.unpack_codes(raw, 1, 512), 1), raw)


def test_1bit_constructed_weights_round_trip_exactly():
    """W = s16 * c (signs, one fp16 scale per 128) packs back to c and s16."""
    W = WL.make_w(5, 1, 64, 3072, "binary", 128)
    packed, s16, b = O.pack_ref(W, 1, 128)
    assert b is None and packed.shape == (64, 3072 // 8)
    c = O.unpack_codes(packed, 1, 3072)
    recon = np.repeat(s16.T.astype(np.float32), 128, axis=1) * c
    assert np.array_equal(recon.astype(np.float32), W)


def test_1bit_scale_is_the_least_squares_one():
    """For fixed signs the squared error of s * sign(w) is minimised by the
    mean |w|; no neighbouring fp16 value of the stored scale does better, and
    the signs follow w (zero and -0 counted as +1)."""
    g = np.random.default_rng(12)
    w = (g.standard_normal((3, 256)) * 0.02).astype(np.float32)
    w[0, 5], w[1, 9] = 0.0, -0.0
    packed, s16, _ = O.pack_ref(w, 1, 128)
    c = O.unpack_codes(packed, 1, 256)
    assert np.array_equal(c, np.where(w >= 0, 1, -1))
    assert c[0, 5] == 1 and c[1, 9] == 1
    for n in range(3):
        for j in range(2):
            wg = w[n, 128 * j:128 * (j + 1)].astype(np.float64)
            cg = c[n, 128 * j:128 * (j + 1)]
            s = float(s16[j, n])
            err = lambda v: float(np.sum((wg - v * cg) ** 2))
            up = float(np.nextafter(np.float16(s), np.float16(np.inf)))
            down = float(np.nextafter(np.float16(s), np.float16(0)))
            assert err(s) <= err(up) and err(s) <= err(down)


def test_1bit_dequant_is_signed_scale_and_gemm_matches_triple_loop():
    g = np.random.default_rng(13)
    c = np.where(g.integers(0, 2, size=(6, 256)) == 1, 1, -1)
    s16 = g.uniform(0.01, 0.05, size=(6, 2)).astype(np.float16)
    packed = O.pack_codes(c, 1)
    bits = O.dequant_ref_bits(packed, np.ascontiguousarray(s16.T), None, 1, 128, 256)
    sb = torch.from_numpy(np.repeat(s16.astype(np.float32), 128, axis=1)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(O.bf16_bits_to_f64(bits), c * sb.astype(np.float64))
    X, W, bias = WL.random_case(2, 4, 5, 128, 1, with_bias=True)
    p, s, b = O.pack_ref(W, 1, 128)
    ref = O.qgemm_ref(X, p, s, b, 1, 128, 128, bias)
    brute = _naive(O.bf16_bits_to_f64(X), O.wq_exact(p, s, b, 1, 128, 128), O.bf16_bits_to_f64(bias))
    assert np.allclose(ref, brute, rtol=1e-12, atol=1e-14)
    assert O.format_bytes(12288, 3072, 1, 128) == 12288 * 3072 // 8 + 12288 * 24 * 2


def test_1bit_scale_is_the_exact_mean_rounded_once():
    """The 1-bit scale is the fp16 value nearest the exact mean of the
    group's |w| (ties to even), whatever order the weights come in. Groups
    whose exact means are derived by hand:

    * one weight of 1049088 (= 8196 * 128; 8196 is the tie between the fp16
      values 8192 and 8200) and 127 of 2^-38: the mean is 8196 + 127 * 2^-45,
      above the tie, so 8200 in either order (an fp64 running sum in k order
      swallows each tiny term and would land on the tie itself, giving 8192);
    * 1049088 and 127 zeros: exactly the tie, rounds to the even 8192;
    * 1049087.875 (the fp32 value just below) and 127 zeros: below the tie, 8192;
    * 1049088 + 2^-1 and 127 zeros: above the tie, 8200;
    * 128 weights of 2^-20: mean 2^-20, an fp16 subnormal (16 * 2^-24), exact;
    * 127 zeros and one 2^-17 * 3: mean 3 * 2^-24, the third subnormal;
    * 127 zeros and one 1.5 * 2^-17: mean 1.5 * 2^-24, a tie between the
      subnormals 1 and 2 (units of 2^-24), rounds to the even 2;
    * 128 weights of 65520: mean 65520, the fp16 overflow threshold: refused.
    """
    def scale(row):
        w = np.asarray(row, dtype=np.float32)[None, :]
        return float(O.pack_ref(w, 1, 128)[1][0, 0])

    tiny = [2.0 ** -38] * 127
    assert scale([1049088.0] + tiny) == 8200.0
    assert scale(tiny + [1049088.0]) == 8200.0
    assert scale(tiny[:60] + [1049088.0] + tiny[60:]) == 8200.0
    assert scale([1049088.0] + [0.0] * 127) == 8192.0
    assert np.float32(1049087.875) == 1049087.875
    assert scale([1049087.875] + [0.0] * 127) == 8192.0
    assert scale([1049088.5] + [0.0] * 127) == 8200.0
    assert scale([2.0 ** -20] * 128) == 2.0 ** -20
    assert scale([0.0] * 127 + [3 * 2.0 ** -17]) == 3 * 2.0 ** -24
    assert scale([0.0] * 127 + [1.5 * 2.0 ** -17]) == 2 * 2.0 ** -24
    with pytest.raises(OverflowError):
        O.pack_ref(np.full((1, 128), 65520.0, dtype=np.float32), 1, 128)
    assert scale([65504.0] * 128) == 65504.0
    # on ordinary groups the exact mean and an fp64 sum agree after rounding
    g = np.random.default_rng(13)
    wr = (g.standard_normal((4, 256)) * 0.02).astype(np.float32)
    _, s16g, _ = O.pack_ref(wr, 1, 128)
    for n in range(4):
        for j in range(2):
            assert s16g[j, n] == np.float16(np.abs(wr[n, 128 * j:128 * (j + 1)].astype(np.float64)).mean())


def test_fp16_rn_exact_on_rationals():
    """The exact-rational fp16 rounding on values derived by hand: the
    midpoint between 1 and 1 + 2^-10 rounds to 1 (even), a hair above it to
    1 + 2^-10, 1/3 to the fp16 value 0x3555, and the overflow threshold."""
    from fractions import Fraction as F
    assert O.fp16_rn_exact(F(2049, 2048)) == 1.0
    assert O.fp16_rn_exact(F(2049, 2048) + F(1, 10 ** 30)) == 1.0 + 2.0 ** -10
    assert O.fp16_rn_exact(F(2051, 2048)) == 1.0 + 2 * 2.0 ** -10     # tie of 1 + u and 1 + 2u: the even one
    assert int(np.array(O.fp16_rn_exact(F(1, 3))).view(np.uint16)) == 0x3555
    assert O.fp16_rn_exact(F(65519)) == 65504.0
    assert np.isinf(O.fp16_rn_exact(F(65520)))
    assert O.fp16_rn_exact(F(0)) == 0.0
    assert O.fp16_rn_exact(F(1, 2 ** 25)) == 0.0                        # half the smallest subnormal: even 0
    assert O.fp16_rn_exact(F(3, 2 ** 26)) == 2.0 ** -24                 # above half


def test_dense_ref_hand_worked_2x3():
    """dense_ref on a case worked by hand: W is rounded to bf16 first (1 + 2^-8
    is the tie between 1 and 1 + 2^-7 and goes to the even 1; 1 + 2^-8 +
    2^-10 goes up to 1 + 2^-7; fp32 0.1 = 0x3DCCCCCD rounds up to bf16
    0x3DCD = 0.10009765625), then X . bf16(W)^T + bias in exact arithmetic."""
    X = WL.f32_to_bf16_bits(np.array([[1.0, 2.0], [-1.0, 0.5]], dtype=np.float32))
    W = np.array([[1 + 2.0 ** -8, 3.0], [1 + 2.0 ** -8 + 2.0 ** -10, -2.0], [0.1, 0.0]], dtype=np.float32)
    bias = WL.f32_to_bf16_bits(np.array([0.5, -1.0, 0.25], dtype=np.float32))
    expect = np.array([[7.5, -3.9921875, 0.35009765625],
                       [1.0, -3.0078125, 0.14990234375]])
    assert np.array_equal(O.dense_ref(X, W, bias), expect)
    assert np.array_equal(O.dense_ref(X, W), expect - np.array([0.5, -1.0, 0.25])[None, :])


def test_dense_ref_equals_python_loop_over_torch_bf16_weights():
    """dense_ref against a pure-Python triple loop over W cast to bf16 by
    torch (not by the oracle's own rounding helper), with a bias."""
    X, W, bias = WL.random_case(21, 5, 7, 128, 4, with_bias=True, w_scale=0.3)
    Wb = torch.from_numpy(W).to(torch.bfloat16).double().numpy()
    Xf = WL.bf16_bits_to_f32(X).astype(np.float64)
    bf = WL.bf16_bits_to_f32(bias).astype(np.float64)
    ref = O.dense_ref(X, W, bias)
    for m in range(5):
        for n in range(7):
            acc = 0.0
            for k in range(128):
                acc += float(Xf[m, k]) * float(Wb[n, k])
            assert abs(ref[m, n] - (acc + float(bf[n]))) <= 1e-12 * (1 + abs(acc))
