"""The tcgen05 small-M kernel (QGEMM_SMALL_TC=1: decoded weights in tensor
memory, tcgen05.mma with N = 16 tokens, one fp32 accumulator per scale group)
against the oracle in every format: ragged M and N, K of one ring stage, of
several and with a short last stage, every M of 1..16 on one shape, bias and
fused epilogues. QGEMM_SMALL_TC is read once per process, so the cases run in
a child process."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import numpy as np
import oracle as O
import weight_quantised_gemm_b200 as wq
import workloads as WL
from gpu_util import from_dev_bf16, gpu_qgemm, to_dev_bf16

SMALL = wq.QGEMM_PATH_SMALL_M
bad = []

def close(y, ref, what):
    y = O.bf16_bits_to_f64(y)
    rf, ma = O.rel_frobenius(y, ref), O.max_abs_rel(y, ref)
    if not (np.all(np.isfinite(y)) and rf <= O.REL_FROB_TOL and ma <= O.MAX_ABS_TOL):
        bad.append(f"{what}: rel_frob={rf:.3e} max_abs={ma:.3e}")

for bits in (1, 2, 4, 8):
    group = wq.GROUP_OF_BITS[bits]
    # ragged N (rows past N in the last 128-row CTA), K of part of a stage, one, several, a short last stage
    for M, N, K in [(1, 16, 256), (3, 144, 512), (16, 272, 1024), (5, 400, 2560), (9, 1040, 3072), (16, 128, 5376)]:
        X, W, bias = WL.random_case(M + N + bits, M, N, K, bits, with_bias=(M % 2 == 1))
        y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
        p, s, b = O.pack_ref(W, bits, group)
        close(y, O.qgemm_ref(X, p, s, b, bits, group, K, bias), f"bits={bits} M={M} N={N} K={K}")
    # every token count on one shape (4 tokens read back for M <= 4, 16 above)
    N, K = 256, 1536
    for M in range(1, 17):
        X, W, bias = WL.random_case(100 + M + bits, M, N, K, bits, with_bias=True)
        y, _ = gpu_qgemm(X, W, bias, bits, path=SMALL)
        p, s, b = O.pack_ref(W, bits, group)
        close(y, O.qgemm_ref(X, p, s, b, bits, group, K, bias), f"bits={bits} M={M}")
    # fused epilogues
    g = np.random.default_rng(5 + bits)
    for op in (wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE):
        M, N, K = 7, 400, 1024
        X, W, bias = WL.random_case(60 + op + bits, M, N, K, bits, with_bias=True)
        r = WL.f32_to_bf16_bits(g.standard_normal((M, N)).astype(np.float32))
        gt = WL.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
        dw = wq.qgemm_pack(W, bits).to_device()
        y = wq.qgemm_fused(to_dev_bf16(X), dw, op, bias=to_dev_bf16(bias), residual=to_dev_bf16(r),
                           gate=to_dev_bf16(gt), path=SMALL)
        wq.check_device_status()
        p, s, b = O.pack_ref(W, bits, group)
        close(from_dev_bf16(y), O.qgemm_ref_epilogue(X, p, s, b, bits, group, K, bias, op, r, gt),
              f"fused op={op} bits={bits}")
print("BAD" if bad else "OK", *bad, sep="\n")
"""


def test_small_m_tcgen05_kernel_parity():
    env = dict(os.environ, QGEMM_SMALL_TC="1", PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests")]))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.strip().splitlines()[0] == "OK", r.stdout[-3000:]
