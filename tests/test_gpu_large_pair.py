"""The large-M kernel's CTA-pair form (tcgen05.mma.cta_group::2: two CTAs of
a cluster share a 256-row x 256-token tile, each staging half of the tokens)
against the oracle, in every format and epilogue, and the single-CTA form on
the same cases. QGEMM_LARGE_PAIR (read once per process) picks the form, so
each setting runs in a child process on the same GPU, one after the other."""
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

LARGE = wq.QGEMM_PATH_LARGE_M
bad = []

def close(y, ref, what):
    y = O.bf16_bits_to_f64(y)
    rf, ma = O.rel_frobenius(y, ref), O.max_abs_rel(y, ref)
    if not (np.all(np.isfinite(y)) and rf <= O.REL_FROB_TOL and ma <= O.MAX_ABS_TOL):
        bad.append(f"{what}: rel_frob={rf:.3e} max_abs={ma:.3e}")

for bits in (1, 2, 4, 8):
    group = wq.GROUP_OF_BITS[bits]
    # ragged M and N (the odd CTA's rows or tokens partly or wholly outside), K of one stage and many
    for M, N, K in [(17, 144, 256), (255, 272, 384), (300, 400, 640), (600, 528, 1024), (513, 1040, 3072)]:
        X, W, bias = WL.random_case(M + N + bits, M, N, K, bits, with_bias=(M % 2 == 1))
        y, _ = gpu_qgemm(X, W, bias, bits, path=LARGE)
        p, s, b = O.pack_ref(W, bits, group)
        close(y, O.qgemm_ref(X, p, s, b, bits, group, K, bias), f"bits={bits} M={M} N={N} K={K}")
    # one-hot tokens: the output is the dequantised weight, bit for bit
    N, K, M = 528, 768, 300
    g = np.random.default_rng(9 + bits)
    _, W, _ = WL.random_case(7 + bits, 1, N, K, bits, with_bias=False)
    ks = g.choice(K, size=M)
    X = np.zeros((M, K), dtype=np.uint16)
    X[np.arange(M), ks] = 0x3F80
    y, _ = gpu_qgemm(X, W, None, bits, path=LARGE)
    p, s, b = O.pack_ref(W, bits, group)
    if not np.array_equal(y, O.dequant_ref_bits(p, s, b, bits, group, K)[:, ks].T):
        bad.append(f"one-hot bits={bits}")
    # fused epilogues
    for op in (wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE):
        M, N, K = 280, 784, 512
        X, W, bias = WL.random_case(40 + op + bits, M, N, K, bits, with_bias=True)
        r = WL.f32_to_bf16_bits(g.standard_normal((M, N)).astype(np.float32))
        gt = WL.f32_to_bf16_bits(g.standard_normal(N).astype(np.float32))
        dw = wq.qgemm_pack(W, bits).to_device()
        y = wq.qgemm_fused(to_dev_bf16(X), dw, op, bias=to_dev_bf16(bias), residual=to_dev_bf16(r),
                           gate=to_dev_bf16(gt), path=LARGE)
        wq.check_device_status()
        p, s, b = O.pack_ref(W, bits, group)
        close(from_dev_bf16(y), O.qgemm_ref_epilogue(X, p, s, b, bits, group, K, bias, op, r, gt),
              f"fused op={op} bits={bits}")
print("BAD" if bad else "OK", *bad, sep="\n")
"""


@pytest.mark.parametrize("mode", ["1", "0"])
def test_large_m_pair_and_single_forms(mode):
    env = dict(os.environ, QGEMM_LARGE_PAIR=mode, PYTHONPATH=os.pathsep.join([ROOT, os.path.join(ROOT, "tests")]))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.strip().splitlines()[0] == "OK", r.stdout[-3000:]
