"""The C ABI on the host: the library loads without a GPU, exports every entry
point include/qgemm.h declares, and rejects bad arguments with the documented
status before touching a device."""
import ctypes
import os
import pathlib
import re

import numpy as np
import pytest

import weight_quantised_gemm_b200 as wq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = pathlib.Path(ROOT, "include", "qgemm.h").read_text()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qgemm[a-z_]*)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(wq.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(wq.EXPORTED)


def test_status_strings_and_version():
    assert wq.qgemm_status_str(0) == "ok"
    for s in range(1, 7):
        assert wq.qgemm_status_str(s) not in ("ok", "unknown status")
    assert wq.qgemm_status_str(99) == "unknown status"
    assert "sm_100a" in wq.qgemm_version()


def test_pack_sizes():
    assert wq.qgemm_pack_sizes(9216, 3072, 4) == (9216 * 1536, 9216 * 48 * 2, 9216 * 48 * 2)
    assert wq.qgemm_pack_sizes(3072, 12288, 8) == (3072 * 12288, 3072 * 192 * 2, 3072 * 192 * 2)
    assert wq.qgemm_pack_sizes(12288, 3072, 2) == (12288 * 768, 12288 * 24 * 2, 0)
    assert wq.qgemm_pack_sizes(12288, 3072, 1) == (12288 * 384, 12288 * 24 * 2, 0)


@pytest.mark.parametrize("args,status", [
    ((16, 128, 3, 64), wq.QGEMM_ERR_UNSUPPORTED),
    ((16, 128, 4, 128), wq.QGEMM_ERR_UNSUPPORTED),
    ((16, 128, 2, 64), wq.QGEMM_ERR_UNSUPPORTED),
    ((16, 128, 1, 64), wq.QGEMM_ERR_UNSUPPORTED),
    ((16, 192, 4, 64), wq.QGEMM_ERR_UNSUPPORTED),     # K not a multiple of 128
    ((0, 128, 4, 64), wq.QGEMM_ERR_INVALID_ARG),
    ((16, -128, 4, 64), wq.QGEMM_ERR_INVALID_ARG),
    (((1 << 30) + 16, 128, 4, 64), wq.QGEMM_ERR_UNSUPPORTED),   # N above 2^30
    ((16, (1 << 30) + 128, 2, 128), wq.QGEMM_ERR_UNSUPPORTED),  # K above 2^30
])
def test_pack_sizes_rejects(args, status):
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_pack_sizes(*args)
    assert e.value.status == status


def test_pack_rejects_nonfinite_and_overflow():
    W = np.zeros((16, 128), dtype=np.float32)
    W[3, 7] = np.inf
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_pack(W, 4)
    assert e.value.status == wq.QGEMM_ERR_NONFINITE
    W[3, 7] = np.nan
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_pack(W, 2)
    assert e.value.status == wq.QGEMM_ERR_NONFINITE
    W[3, 7] = 0.0
    W[0, 0], W[0, 1] = -7e5, 7e5          # range / 15 overflows fp16
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_pack(W, 4)
    assert e.value.status == wq.QGEMM_ERR_UNSUPPORTED
    W[0, 0], W[0, 1] = 0.0, 7e5           # absmax overflows fp16
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_pack(W, 2)
    assert e.value.status == wq.QGEMM_ERR_UNSUPPORTED


def _desc(N=256, K=512, bits=4, group=64, packed=0x1000, scales=0x2000, biases=0x3000):
    return wq._Weights(N, K, bits, group, packed, scales, biases)


def _call(desc, X=0x10000, M=64, out=0x20000, bias=None, path=0):
    return wq._lib.qgemm_ex(X, M, ctypes.byref(desc) if desc is not None else None, out, bias, path, None)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=3), wq.QGEMM_ERR_UNSUPPORTED),
    (dict(bits=2, group=64), wq.QGEMM_ERR_UNSUPPORTED),
    (dict(K=192), wq.QGEMM_ERR_UNSUPPORTED),
    (dict(N=264), wq.QGEMM_ERR_UNSUPPORTED),         # N % 16 != 0
    (dict(N=0), wq.QGEMM_ERR_INVALID_ARG),
    (dict(packed=0), wq.QGEMM_ERR_INVALID_ARG),
    (dict(scales=0), wq.QGEMM_ERR_INVALID_ARG),
    (dict(biases=0), wq.QGEMM_ERR_INVALID_ARG),      # affine needs biases
    (dict(packed=0x1008), wq.QGEMM_ERR_ALIGNMENT),
    (dict(scales=0x2002), wq.QGEMM_ERR_ALIGNMENT),
    (dict(N=(1 << 30) + 16), wq.QGEMM_ERR_UNSUPPORTED),         # above the 2^30 limit
    (dict(K=(1 << 30) + 128), wq.QGEMM_ERR_UNSUPPORTED),
])
def test_qgemm_rejects_bad_weights_without_device(kw, status):
    assert _call(_desc(**kw)) == status


def test_qgemm_rejects_bad_operands_without_device():
    d = _desc()
    assert wq._lib.qgemm_ex(0x10000, 64, None, 0x20000, None, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert _call(d, M=-1) == wq.QGEMM_ERR_INVALID_ARG
    assert _call(d, X=0) == wq.QGEMM_ERR_INVALID_ARG
    assert _call(d, out=0) == wq.QGEMM_ERR_INVALID_ARG
    assert _call(d, X=0x10004) == wq.QGEMM_ERR_ALIGNMENT
    assert _call(d, out=0x20002) == wq.QGEMM_ERR_ALIGNMENT
    assert _call(d, bias=0x30001) == wq.QGEMM_ERR_ALIGNMENT
    assert _call(d, path=7) == wq.QGEMM_ERR_INVALID_ARG
    assert _call(d, path=wq.QGEMM_PATH_LARGE_M | 0x200) == wq.QGEMM_ERR_INVALID_ARG   # unknown flag bit
    assert _call(d, M=0, path=wq.QGEMM_PATH_SMALL_M | wq.QGEMM_FLAG_OVERLAP_PREVIOUS) == wq.QGEMM_OK
    assert _call(d, M=65, path=wq.QGEMM_PATH_SMALL_M) == wq.QGEMM_ERR_UNSUPPORTED      # small path: M <= 64
    assert _call(d, M=(1 << 30) + 1) == wq.QGEMM_ERR_UNSUPPORTED                      # above the 2^30 limit
    assert _call(d, M=(1 << 31) - 1) == wq.QGEMM_ERR_UNSUPPORTED
    # M = 0 is a no-op that never touches the device
    assert _call(d, M=0) == wq.QGEMM_OK
    # ternary needs no biases
    assert _call(_desc(bits=2, group=128, biases=0), M=0) == wq.QGEMM_OK


def test_dequant_tile_rejects_bad_windows_without_device():
    d = _desc()
    f = wq._lib.qgemm_dequant_tile
    assert f(ctypes.byref(d), 0, 0, 257, 64, 0x40000, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), 0, 4, 16, 64, 0x40000, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), 0, 0, 16, 60, 0x40000, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), 0, 0, 16, 64, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), 0, 0, 16, 64, 0x40008, None) == wq.QGEMM_ERR_ALIGNMENT
    assert f(ctypes.byref(d), 0, 0, 0, 0, 0x40000, None) == wq.QGEMM_OK


def test_select_path_table():
    # 1-bit rows need K % 256 == 0 on the small path; otherwise the large path
    assert wq.qgemm_select_path(1, 12288, 1152, 1) == wq.QGEMM_PATH_LARGE_M
    assert _call(_desc(bits=1, group=128, K=1152, biases=0), M=4, path=wq.QGEMM_PATH_SMALL_M) == \
        wq.QGEMM_ERR_UNSUPPORTED
    for bits in (1, 2, 4, 8):
        assert wq.qgemm_select_path(1, 12288, 3072, bits) == wq.QGEMM_PATH_SMALL_M
        assert wq.qgemm_select_path(4096, 9216, 3072, bits) == wq.QGEMM_PATH_LARGE_M
        # every (N, K) of the FLUX workloads: the measured table's choice at decode and prefill M
        for N, K in ((12288, 3072), (9216, 3072), (18432, 3072), (3072, 3072), (3072, 12288)):
            if N <= 3072:
                small_max = 64
            elif bits <= 2:
                small_max = 48 if N <= 9216 else 32
            else:
                small_max = 32 if N <= 9216 else 16
            for M in (1, 4, 8, 16, 17, 24, 32, 33, 48, 49, 64):
                want = wq.QGEMM_PATH_SMALL_M if M <= small_max else wq.QGEMM_PATH_LARGE_M
                assert wq.qgemm_select_path(M, N, K, bits) == want, (bits, N, K, M)
            for M in (65, 256, 4608):
                assert wq.qgemm_select_path(M, N, K, bits) == wq.QGEMM_PATH_LARGE_M, (bits, N, K, M)
        # narrow N below K = 3072 keeps the one-launch limits: the tiny 64 x 512 x 512 case on the tile path
        assert wq.qgemm_select_path(64, 512, 512, bits) == wq.QGEMM_PATH_LARGE_M
        assert wq.qgemm_select_path(32, 512, 512, bits) == wq.QGEMM_PATH_SMALL_M
    with pytest.raises(wq.QGemmError):
        wq.qgemm_select_path(1, 16, 128, 3)
    with pytest.raises(wq.QGemmError) as e:
        wq.qgemm_select_path((1 << 31) - 1, 16, 128, 4)
    assert e.value.status == wq.QGEMM_ERR_UNSUPPORTED


def test_missing_library_fails_loudly_on_first_call(tmp_path):
    """Without libqgemm.so the package still imports (so its build module can
    run on a fresh checkout) but every entry point raises: no CPU fallback."""
    import shutil
    import subprocess
    import sys
    pkg = tmp_path / "weight_quantised_gemm_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "weight_quantised_gemm_b200", "__init__.py"), pkg / "__init__.py")
    code = ("import weight_quantised_gemm_b200 as wq\n"
            "try:\n    wq.qgemm_version()\nexcept ImportError as e:\n    print('raised', 'not built' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "raised True"


def _fused(desc, op, residual=0x40000, gate=0x50000, M=64, path=0):
    epi = wq._Epilogue(op, residual, gate)
    return wq._lib.qgemm_fused(0x10000, M, ctypes.byref(desc), 0x20000, None, ctypes.byref(epi), path, None)


def test_fused_rejects_bad_epilogues_without_device():
    d = _desc()
    assert _fused(d, 3) == wq.QGEMM_ERR_INVALID_ARG
    assert _fused(d, -1) == wq.QGEMM_ERR_INVALID_ARG
    assert _fused(d, wq.QGEMM_EPI_RESIDUAL_GATE, residual=None) == wq.QGEMM_ERR_INVALID_ARG
    assert _fused(d, wq.QGEMM_EPI_RESIDUAL_GATE, gate=None) == wq.QGEMM_ERR_INVALID_ARG
    assert _fused(d, wq.QGEMM_EPI_RESIDUAL_GATE, residual=0x40008) == wq.QGEMM_ERR_ALIGNMENT
    assert _fused(d, wq.QGEMM_EPI_RESIDUAL_GATE, gate=0x50001) == wq.QGEMM_ERR_ALIGNMENT
    # valid descriptors with M = 0: a no-op that never touches the device
    for op in (wq.QGEMM_EPI_NONE, wq.QGEMM_EPI_GELU_TANH, wq.QGEMM_EPI_RESIDUAL_GATE):
        assert _fused(d, op, M=0) == wq.QGEMM_OK
    # a NULL epilogue is plain qgemm_ex
    assert wq._lib.qgemm_fused(0x10000, 0, ctypes.byref(d), 0x20000, None, None, 0, None) == wq.QGEMM_OK


def test_pack_device_rejects_bad_arguments_without_device():
    f = wq._lib.qgemm_pack_device
    ok = dict(W=0x1000, N=16, K=128, bits=4, group=64, p=0x2000, s=0x3000, b=0x4000)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["W"], a["N"], a["K"], a["bits"], a["group"], a["p"], a["s"], a["b"], None)
    assert call(bits=3) == wq.QGEMM_ERR_UNSUPPORTED
    assert call(K=192) == wq.QGEMM_ERR_UNSUPPORTED
    assert call(N=0) == wq.QGEMM_ERR_INVALID_ARG
    assert call(W=None) == wq.QGEMM_ERR_INVALID_ARG
    assert call(b=None) == wq.QGEMM_ERR_INVALID_ARG            # affine needs biases
    assert call(W=0x1004) == wq.QGEMM_ERR_ALIGNMENT
    assert call(s=0x3002) == wq.QGEMM_ERR_ALIGNMENT


def test_binding_device_check_is_host_logic():
    """The binding's same-device check (run before every launch) needs no GPU:
    a weight or output buffer on another device is refused by name."""
    import torch
    cpu = torch.zeros(4)
    W = wq.DeviceWeights(16, 128, 4, 64, cpu, cpu, cpu)
    with pytest.raises(ValueError, match="W.packed is on cpu"):
        wq._same_device(torch.device("cuda", 0), W)
    with pytest.raises(ValueError, match="out is on meta"):
        wq._same_device(torch.device("cpu"), W, out=torch.zeros(2, device="meta"))
    wq._same_device(torch.device("cpu"), W, out=cpu, bias=None)   # one device throughout: accepted


def test_path_variable_defers_to_the_table_where_its_path_cannot_go():
    """QGEMM_PATH=small (read once per process) forces the small path only
    where it can take the shape: qgemm_select_path and the dispatch agree,
    and a call past the small path's limits is not refused. Without a GPU a
    call that reaches a kernel launcher fails with QGEMM_ERR_CUDA (no device),
    which tells it apart from a refusal by the dispatch (UNSUPPORTED)."""
    import subprocess
    import sys
    code = r"""
import ctypes
import weight_quantised_gemm_b200 as wq
W = lambda **kw: wq._Weights(kw.get('N', 256), kw.get('K', 512), kw.get('bits', 4), kw.get('group', 64),
                             0x1000, 0x2000, kw.get('biases', 0x3000))
call = lambda d, M: wq._lib.qgemm_ex(0x10000, M, ctypes.byref(d), 0x20000, None, 0, None)
print(wq.qgemm_select_path(16, 256, 512, 4), wq.qgemm_select_path(65, 256, 512, 4),
      wq.qgemm_select_path(4, 256, 1152, 1), wq.qgemm_select_path(4, 256, 1024, 1))
print(call(W(), 33), call(W(bits=1, group=128, K=1152, biases=0), 4))
"""
    env = dict(os.environ, QGEMM_PATH="small", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    sel, disp = r.stdout.strip().splitlines()
    assert sel.split() == [str(wq.QGEMM_PATH_SMALL_M), str(wq.QGEMM_PATH_LARGE_M), str(wq.QGEMM_PATH_LARGE_M),
                           str(wq.QGEMM_PATH_SMALL_M)]
    assert disp.split() == [str(wq.QGEMM_ERR_CUDA)] * 2
    env["QGEMM_PATH"] = "large"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split()[:4] == [str(wq.QGEMM_PATH_LARGE_M)] * 4


def _grouped(problems, flags=0):
    arr = (wq._Problem * len(problems))(*problems)
    return wq._lib.qgemm_grouped(arr, len(problems), flags, None)


def _problem(M=4, X=0x10000, out=0x20000, bias=None, **kw):
    return wq._Problem(X, M, _desc(**kw), out, bias)


def test_grouped_rejects_bad_lists_without_device():
    ok = _problem()
    assert wq._lib.qgemm_grouped(None, 1, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert _grouped([ok], flags=0x400) == wq.QGEMM_ERR_INVALID_ARG
    # the one-launch flag is known: the call gets past the argument checks (and,
    # without a device, fails at the launch)
    assert _grouped([ok], flags=wq.QGEMM_FLAG_GROUPED_ONE_LAUNCH) == wq.QGEMM_ERR_CUDA
    arr = (wq._Problem * 17)(*([ok] * 17))
    assert wq._lib.qgemm_grouped(arr, 17, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert wq._lib.qgemm_grouped(arr, 0, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert _grouped([ok, _problem(bits=8)]) == wq.QGEMM_ERR_UNSUPPORTED            # one format per call
    assert _grouped([ok, _problem(M=17)]) == wq.QGEMM_ERR_UNSUPPORTED             # small-M only
    assert _grouped([ok, _problem(M=-1)]) == wq.QGEMM_ERR_UNSUPPORTED
    assert _grouped([_problem(bits=1, group=128, K=1152, biases=0)]) == wq.QGEMM_ERR_UNSUPPORTED
    assert _grouped([ok, _problem(X=0)]) == wq.QGEMM_ERR_INVALID_ARG
    assert _grouped([ok, _problem(out=0x20008)]) == wq.QGEMM_ERR_ALIGNMENT
    assert _grouped([ok, _problem(bias=0x30001)]) == wq.QGEMM_ERR_ALIGNMENT
    assert _grouped([ok, _problem(N=264)]) == wq.QGEMM_ERR_UNSUPPORTED           # the weights are checked too
    # every problem empty: a no-op that never touches the device
    assert _grouped([_problem(M=0, X=0, out=0), _problem(M=0)]) == wq.QGEMM_OK


def test_problem_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes mirror of qgemm_problem has the C layout."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc is not installed")
    src = tmp_path / "layout.c"
    src.write_text('#include <stddef.h>\n#include <stdio.h>\n#include "qgemm.h"\n'
                   'int main(void) { printf("%zu %zu %zu %zu %zu\\n", sizeof(qgemm_problem), '
                   'offsetof(qgemm_problem, M), offsetof(qgemm_problem, W), offsetof(qgemm_problem, out), '
                   'offsetof(qgemm_problem, bias)); return 0; }\n')
    exe = tmp_path / "layout"
    r = subprocess.run([gcc, "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    P = wq._Problem
    assert got == [ctypes.sizeof(P), P.M.offset, P.W.offset, P.out.offset, P.bias.offset]


def test_debug_stream_rejects_bad_arguments_without_device():
    d = _desc()
    f = wq._lib.qgemm_debug_stream
    assert f(0x10000, 65, ctypes.byref(d), 0, None) == wq.QGEMM_ERR_UNSUPPORTED       # small-M shapes only
    assert f(0x10000, -1, ctypes.byref(d), 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(0x10000, 4, ctypes.byref(d), 0x200, None) == wq.QGEMM_ERR_INVALID_ARG    # unknown flag
    assert f(None, 4, ctypes.byref(d), 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(0x10004, 4, ctypes.byref(d), 0, None) == wq.QGEMM_ERR_ALIGNMENT
    assert f(0x10000, 4, None, 0, None) == wq.QGEMM_ERR_INVALID_ARG
    assert f(0x10000, 0, ctypes.byref(d), 0, None) == wq.QGEMM_OK                    # M = 0: nothing to stream
