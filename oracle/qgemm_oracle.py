"""Oracle for the weight-quantised GEMM: plain, slow, obviously correct CPU code.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library (no kernels, headers, tables or helpers); the
two meet only through the seeded inputs of ``workloads.py``.

What the method computes
------------------------
stable-diffusion.rs README (andreinknv), introduction: weights stay packed
in their quantised form and are expanded to full precision within the GEMM
kernel, tile by tile. The result it reaches is, up to rounding order, the plain
product of the activations with the dequantised weights, so this oracle is
that definition written out in fp64:

    out[M, N] = X[M, K] . Wq[N, K]^T (+ bias[N])

Formats (this library's definition; the pages give no bit layout, no scale
formula and no rounding rule):

* 4-bit and 8-bit group-wise affine, groups of 64 consecutive k in a row:
  ``w ~ s16 * q + b16`` with fp16 scale s16 and fp16 bias b16 per group,
  q in [0, 2^b - 1]. The two widths are the pages' (stable-diffusion.rs
  README, introduction: 4 bits for most linears, 8 for those whose output
  scales the residual stream).
* ternary {-1, 0, +1} with one fp16 scale per group of 128
  (pictor README, "Extreme quantization is first-class": TQ2_0_g128).
* 1-bit {-1, +1} with one fp16 scale per group of 128 (the same README's
  Q1_0_g128, named without a definition).

Packing is round-to-nearest (RTN) in fp64, ties to even:

* affine: lo = min, hi = max of the group; s16 = fp16(fl64((hi - lo) /
  (2^b - 1))), b16 = fp16(lo) (a zero minimum or maximum taken as +0, so the
  sign of a zero weight never decides a stored bit: a group of zeros stores
  +0 for both its scale and its bias); q = clamp(rint((w - b16) / s16), 0,
  2^b - 1), q = 0 where s16 == 0.
* ternary: s16 = fp16(max |w|); t = clamp(rint(w / s16), -1, 1), t = 0 where
  s16 == 0.
* 1-bit: s16 = fp16(mean |w|), the scale that minimises the squared error
  for fixed signs, rounded once (to nearest, ties to even) from the exact
  mean of the group's 128 magnitudes; c = +1 where w >= 0 (-0 included),
  else -1.

Bit layout, row-major over N with K contiguous, little-endian 32-bit words:

* 8-bit: byte k holds q[k].
* 4-bit: a word holds 8 consecutive k; offset j = 2i (even) sits in bits
  4i..4i+3 and offset j = 2i + 1 (odd) in bits 16+4i..19+4i.
* ternary: a word holds 16 consecutive k; offset j = 2i in bits 2i..2i+1 and
  j = 2i + 1 in bits 16+2i..17+2i. The 2-bit code is t in two's complement
  (0 -> 00, +1 -> 01, -1 -> 11); code 10 is invalid.
* 1-bit: a word holds 32 consecutive k; offset j = 2i in bit i and j = 2i + 1
  in bit 16 + i; bit 1 is +1, bit 0 is -1.
* scales and biases: fp16 [K / group, N], group-major (the scales of one
  group of k for all rows are contiguous).

Dequantised weight (the bit-exact contract of the dequant-tile entry point):

* affine: wdeq = bf16_rn( fl32(s16 * q + b16) ). s16 * q is exact in fp32
  (11 + 8 significant bits), so this equals one fp32 FMA followed by one
  round-to-nearest-even to bf16.
* ternary: wdeq = t * bf16_rn(fl32(s16)), with +0 for t = 0.
* 1-bit: wdeq = c * bf16_rn(fl32(s16)).

Numerics of the matmul: fp32 accumulation is what the kernels keep (pictor
README, numerics: accumulation stays in fp32, without reduced-precision TF32
or fp16 multiply-accumulate);
the oracle accumulates in fp64.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

AFFINE_BITS = (4, 8)
TERNARY_BITS = 2
BINARY_BITS = 1


# ----------------------------------------------------------------------------
# rounding helpers
# ----------------------------------------------------------------------------

def fp16_rn(x) -> np.ndarray:
    """fp64 -> fp16, round to nearest even, in one rounding (numpy's double->half).

    Pinned in the tests against CPython's own IEEE half packing
    (``struct.pack('e')``) on every fp16 value, every midpoint and random doubles.
    """
    with np.errstate(over="ignore"):    # overflow gives inf, which the callers refuse
        return np.asarray(x, dtype=np.float64).astype(np.float16)


def fp16_rn_exact(q: Fraction) -> np.float16:
    """The fp16 value nearest to the exact rational q >= 0, ties to the even
    encoding; +inf at and above 65520 (the largest finite fp16, 65504, plus
    half its spacing).

    Written from the definition: the nearest of the fp16 values that bracket
    q, found around a first guess and compared exactly.
    """
    if q >= 65520:
        return np.float16(np.inf)
    guess = np.float16(float(q))
    cands = {guess, np.nextafter(guess, np.float16(0)), np.nextafter(guess, np.float16(65504))}
    return min(cands, key=lambda c: (abs(Fraction(float(c)) - q), int(np.array(c).view(np.uint16)) & 1))


def mean_abs_fp16(values) -> np.float16:
    """fp16 of the exact mean of |values| (fp32 weights), rounded once.

    math.fsum gives the exact sum rounded once to fp64; dividing by the
    group size (a power of two) keeps that exact. Rounding that fp64 value to
    fp16 gives the same answer as rounding the exact mean, except where the
    fp64 neighbourhood of the mean straddles an fp16 rounding boundary; only
    then is the mean formed exactly (fractions.Fraction) and rounded from
    there.
    """
    a = [abs(float(v)) for v in values]
    n = len(a)
    v = math.fsum(a) / n
    lo, hi = np.nextafter(v, -np.inf), np.nextafter(v, np.inf)
    with np.errstate(over="ignore"):
        r = np.float16(v)
        if np.float16(lo) == r == np.float16(hi):
            return r
    return fp16_rn_exact(sum(Fraction(x) for x in a) / n)


def bf16_rn_bits(x32) -> np.ndarray:
    """fp32 -> bf16 storage bits, round to nearest even on the fp32 bit pattern.

    bf16 keeps the top 16 bits of an fp32. Rounding adds 0x7FFF plus the
    lowest kept bit (the tie-to-even correction) before truncating. NaN keeps
    its sign and top payload bits and is made quiet.
    """
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint32)
    nan = (u & np.uint64(0x7FFFFFFF)) > np.uint64(0x7F800000)
    r = np.where(nan, ((u >> np.uint64(16)) | np.uint64(0x40)).astype(np.uint32), r)
    return r.astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    """bf16 storage bits -> fp64 values (exact)."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# bit layout
# ----------------------------------------------------------------------------

def codes_per_word(bits: int) -> int:
    """Codes per little-endian 32-bit word of the packed layout (32 / bits). The pages give no
    bit layout; this is the layout the module header fixes."""
    return 32 // bits


def code_bit_position(bits: int, j: int) -> int:
    """Bit position, inside its 32-bit word, of the code for in-word offset j."""
    if bits == 8:
        return 8 * j
    i, odd = divmod(j, 2)
    return 16 * odd + bits * i


def pack_codes(codes, bits: int) -> np.ndarray:
    """Integer codes [N, K] -> packed bytes [N, K * bits / 8], in the bit
    layout the module header fixes (the pages give none).

    Affine codes are q in [0, 2^b - 1]; ternary codes are t in {-1, 0, +1}
    and are stored as 2-bit two's complement; 1-bit codes are c in {-1, +1},
    stored as 1 for +1 and 0 for -1.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    per = codes_per_word(bits)
    if K % per:
        raise ValueError("K must fill whole 32-bit words")
    mask = (1 << bits) - 1
    if bits == BINARY_BITS:
        if not np.all(np.abs(codes) == 1):
            raise ValueError("1-bit codes are -1 or +1")
        field = (codes > 0).astype(np.int64)
    else:
        field = codes.astype(np.int64) & mask           # two's complement for t = -1
    field = field.astype(np.uint32).reshape(N, K // per, per)
    words = np.zeros((N, K // per), dtype=np.uint32)
    for j in range(per):
        words |= field[:, :, j] << np.uint32(code_bit_position(bits, j))
    return words.astype("<u4").view(np.uint8).reshape(N, K * bits // 8)


def unpack_codes(packed, bits: int, K: int) -> np.ndarray:
    """Packed bytes [N, K * bits / 8] -> integer codes [N, K] (int32): the
    inverse of pack_codes.

    Raises ValueError on the invalid ternary code 10.
    """
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    per = codes_per_word(bits)
    words = packed.reshape(N, -1).view("<u4").astype(np.uint32)
    if words.shape[1] * per != K:
        raise ValueError("packed width does not match K")
    mask = np.uint32((1 << bits) - 1)
    out = np.empty((N, words.shape[1], per), dtype=np.int32)
    for j in range(per):
        out[:, :, j] = (words >> np.uint32(code_bit_position(bits, j))) & mask
    out = out.reshape(N, K)
    if bits == BINARY_BITS:
        return np.where(out == 1, 1, -1).astype(np.int32)
    if bits == TERNARY_BITS:
        if np.any(out == 2):
            raise ValueError("invalid ternary code 0b10")
        out = np.where(out == 3, -1, out)
    return out


# ----------------------------------------------------------------------------
# packing (RTN)
# ----------------------------------------------------------------------------

def check_format(bits: int, group: int, K: int) -> None:
    """The (bits, group) pairs the formats define: 64 for the affine widths the mixed policy uses
    (stable-diffusion.rs README, introduction), 128 for TQ2_0_g128 and Q1_0_g128 (pictor README,
    "Extreme quantization is first-class"); K a whole number of groups."""
    if bits in AFFINE_BITS:
        if group != 64:
            raise ValueError("affine formats use groups of 64")
    elif bits in (TERNARY_BITS, BINARY_BITS):
        if group != 128:
            raise ValueError("ternary and 1-bit use groups of 128")
    else:
        raise ValueError("bits must be 1, 2 (ternary), 4 or 8")
    if K % group:
        raise ValueError("K must be a multiple of the group size")


def pack_ref(W, bits: int, group: int):
    """RTN group quantisation of fp32 W [N, K]: the packing that keeps weights
    quantised in memory (stable-diffusion.rs README, introduction), with the
    scale, bias and rounding readings of the module header.

    Returns (packed uint8 [N, K*b/8], scales fp16 [K/g, N], biases fp16
    [K/g, N] or None for ternary), in the at-rest layout.
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    check_format(bits, group, K)
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    Wg = W.astype(np.float64).reshape(N, K // group, group)
    if bits in AFFINE_BITS:
        qmax = (1 << bits) - 1
        lo = Wg.min(axis=2) + 0.0      # a zero minimum is stored as +0, never -0
        hi = Wg.max(axis=2) + 0.0      # so a zero range gives a +0 scale, whichever zeros the group holds
        s16 = fp16_rn((hi - lo) / qmax)
        b16 = fp16_rn(lo)
        if not (np.all(np.isfinite(s16)) and np.all(np.isfinite(b16))):
            raise OverflowError("scale or bias overflows fp16")
        s = s16.astype(np.float64)[:, :, None]
        b = b16.astype(np.float64)[:, :, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.clip(np.rint((Wg - b) / s), 0, qmax)
        q = np.where(s == 0, 0, q)
        codes = q.reshape(N, K).astype(np.int64)
        return pack_codes(codes, bits), np.ascontiguousarray(s16.T), np.ascontiguousarray(b16.T)
    if bits == BINARY_BITS:
        # numpy's fp64 sum of 128 non-negative terms is within a relative
        # 127 * 2^-53 < 2^-46 of the exact sum; where fp16 rounding gives one
        # value over a relative 2^-40 either side, that is the fp16 of the exact
        # mean, and the few groups where it does not go through mean_abs_fp16
        v = np.abs(Wg).sum(axis=2) / group
        s16 = fp16_rn(v * (1.0 - 2.0 ** -40))
        for n, j in zip(*np.nonzero(s16 != fp16_rn(v * (1.0 + 2.0 ** -40)))):
            s16[n, j] = mean_abs_fp16(Wg[n, j])
        if not np.all(np.isfinite(s16)):
            raise OverflowError("scale overflows fp16")
        c = np.where(Wg >= 0, 1, -1)
        return pack_codes(c.reshape(N, K).astype(np.int64), bits), np.ascontiguousarray(s16.T), None
    s16 = fp16_rn(np.abs(Wg).max(axis=2))
    if not np.all(np.isfinite(s16)):
        raise OverflowError("scale overflows fp16")
    s = s16.astype(np.float64)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.clip(np.rint(Wg / s), -1, 1)
    t = np.where(s == 0, 0, t)
    return pack_codes(t.reshape(N, K).astype(np.int64), bits), np.ascontiguousarray(s16.T), None


# ----------------------------------------------------------------------------
# dequantisation
# ----------------------------------------------------------------------------

def _expand(groupwise, group: int) -> np.ndarray:
    """At-rest [K/g, N] per-group values -> fp64 [N, K], one per weight."""
    return np.repeat(np.asarray(groupwise, dtype=np.float16).T.astype(np.float64), group, axis=1)


def wq_exact(packed, scales, biases, bits: int, group: int, K: int) -> np.ndarray:
    """The quantised weight before any bf16 rounding, fp64 [N, K]: s16*q + b16 or s16*t (or s16*c):
    the weights the method multiplies by, exactly (stable-diffusion.rs README, introduction)."""
    codes = unpack_codes(packed, bits, K).astype(np.float64)
    s = _expand(scales, group)
    if bits in (TERNARY_BITS, BINARY_BITS):
        return s * codes
    return s * codes + _expand(biases, group)


def dequant_ref_bits(packed, scales, biases, bits: int, group: int, K: int) -> np.ndarray:
    """The dequantised weight as bf16 bits [N, K] (the bit-exact contract):
    the tile the method expands to inside the matmul (stable-diffusion.rs
    README, introduction), in the precision the module header fixes.

    affine: s16*q + b16 is exact in fp64 (at most 11+8 significant bits in the
    product and an fp16 addend; the sum spans under 53 bits), so casting it to
    fp32 rounds exactly once, like an fp32 FMA; bf16_rn then rounds again.
    ternary: t * bf16_rn(fp32(s16)), i.e. the sign bit flipped for t = -1 and
    +0 for t = 0.
    """
    codes = unpack_codes(packed, bits, K)
    s = _expand(scales, group)
    if bits in (TERNARY_BITS, BINARY_BITS):
        sb = bf16_rn_bits(s.astype(np.float32))
        out = np.where(codes < 0, sb | np.uint16(0x8000), sb)
        return np.where(codes == 0, np.uint16(0), out).astype(np.uint16)
    v = s * codes.astype(np.float64) + _expand(biases, group)
    return bf16_rn_bits(v.astype(np.float32))


def dequant_ref(packed, scales, biases, bits: int, group: int, K: int) -> np.ndarray:
    """The dequantised weight as fp64 values [N, K] (dequant_ref_bits, widened exactly)."""
    return bf16_bits_to_f64(dequant_ref_bits(packed, scales, biases, bits, group, K))


# ----------------------------------------------------------------------------
# the matmul
# ----------------------------------------------------------------------------

def qgemm_ref(X_bits, packed, scales, biases, bits: int, group: int, K: int,
              bias_bits=None) -> np.ndarray:
    """fp64 out[M, N] = X . Wq_exact^T (+ bias): the reference the kernels are checked against.
    The matmul against the dequantised weights (stable-diffusion.rs README, introduction), taken in
    fp64 where the kernels keep fp32 accumulation (pictor README, numerics)."""
    X = bf16_bits_to_f64(X_bits)
    out = X @ wq_exact(packed, scales, biases, bits, group, K).T
    if bias_bits is not None:
        out = out + bf16_bits_to_f64(bias_bits)[None, :]
    return out


def qgemm_ref_bf16w(X_bits, packed, scales, biases, bits: int, group: int, K: int,
                    bias_bits=None) -> np.ndarray:
    """fp64 out = X . wdeq^T (+ bias), with the bf16 dequantised weights: a tighter diagnostic."""
    X = bf16_bits_to_f64(X_bits)
    out = X @ dequant_ref(packed, scales, biases, bits, group, K).T
    if bias_bits is not None:
        out = out + bf16_bits_to_f64(bias_bits)[None, :]
    return out


def qgemm_ref_rows(rows, X_bits, packed, scales, biases, bits: int, group: int, K: int,
                   bias_bits=None) -> np.ndarray:
    """Reference for a subset of output rows (large shapes, sampled checking)."""
    rows = np.asarray(rows)
    return qgemm_ref(np.asarray(X_bits)[rows], packed, scales, biases, bits, group, K, bias_bits)


def dense_ref(X_bits, W, bias_bits=None) -> np.ndarray:
    """fp64 X . bf16_rn(W)^T (+ bias): the dense bf16 layer the quantised one replaces, the
    reference of the cosine the mixed policy is rated by (stable-diffusion.rs README, introduction)."""
    X = bf16_bits_to_f64(X_bits)
    Wb = bf16_bits_to_f64(bf16_rn_bits(np.asarray(W, dtype=np.float32)))
    out = X @ Wb.T
    if bias_bits is not None:
        out = out + bf16_bits_to_f64(bias_bits)[None, :]
    return out


# ----------------------------------------------------------------------------
# fused epilogues: the elementwise steps on either side of a FLUX block's
# linears (stable-diffusion.rs README, introduction, singles out the linears
# whose output scales the residual stream). The pages give no formula; the
# readings are FLUX's own: the MLP's up projection is followed by the
# tanh-approximate GELU, and a residual-writing linear's output y updates the
# stream as r + gate * y with one gate value per output feature.
# ----------------------------------------------------------------------------

EPI_NONE, EPI_GELU_TANH, EPI_RESIDUAL_GATE = 0, 1, 2


def gelu_tanh_ref(y) -> np.ndarray:
    """0.5 y (1 + tanh(sqrt(2 / pi) (y + 0.044715 y^3))), in fp64."""
    y = np.asarray(y, dtype=np.float64)
    return 0.5 * y * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (y + 0.044715 * y ** 3)))


def epilogue_ref(y, op: int, residual_bits=None, gate_bits=None) -> np.ndarray:
    """Applies the fused epilogue to y = X . Wq^T (+ bias), all in fp64."""
    y = np.asarray(y, dtype=np.float64)
    if op == EPI_NONE:
        return y
    if op == EPI_GELU_TANH:
        return gelu_tanh_ref(y)
    if op == EPI_RESIDUAL_GATE:
        r = bf16_bits_to_f64(residual_bits)
        g = bf16_bits_to_f64(gate_bits)
        return r + g[None, :] * y
    raise ValueError(f"unknown epilogue {op}")


def qgemm_ref_epilogue(X_bits, packed, scales, biases, bits: int, group: int, K: int, bias_bits, op: int,
                       residual_bits=None, gate_bits=None) -> np.ndarray:
    """fp64 epilogue(X . Wq_exact^T (+ bias)): the reference of the fused calls."""
    y = qgemm_ref(X_bits, packed, scales, biases, bits, group, K, bias_bits)
    return epilogue_ref(y, op, residual_bits, gate_bits)


# ----------------------------------------------------------------------------
# error metrics
# ----------------------------------------------------------------------------

REL_FROB_TOL = 5e-3      # ||Y - ref||_F / ||ref||_F
MAX_ABS_TOL = 3e-2       # max |Y - ref| / max |ref|


def rel_frobenius(y, ref) -> float:
    """||y - ref||_F / ||ref||_F: half of the parity gate applied to the kernels (<= REL_FROB_TOL)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / den) if den > 0 else float(np.linalg.norm(y))


def max_abs_rel(y, ref) -> float:
    """max |y - ref| / max |ref|: the other half of the parity gate (<= MAX_ABS_TOL)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref)) if ref.size else 0.0
    err = np.max(np.abs(y - ref)) if ref.size else 0.0
    return float(err / den) if den > 0 else float(err)


def cosine(a, b) -> float:
    """Cosine of two outputs, flattened: the accuracy measure the mixed policy is rated by, against
    the dense output (stable-diffusion.rs README, introduction)."""
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def within_tolerance(y, ref) -> bool:
    """Both halves of the parity gate at once."""
    return rel_frobenius(y, ref) <= REL_FROB_TOL and max_abs_rel(y, ref) <= MAX_ABS_TOL


def format_bytes(N: int, K: int, bits: int, group: int) -> int:
    """Bytes of one packed weight at rest: codes + fp16 scales (+ fp16 biases)."""
    per_group = 2 if bits in (TERNARY_BITS, BINARY_BITS) else 4
    return N * K * bits // 8 + N * (K // group) * per_group
