"""Helpers for the GPU tests: run the library through its Python binding on
seeded inputs and bring results back as bf16 bits."""
import numpy as np
import torch

import weight_quantised_gemm_b200 as wq


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def gpu_qgemm(X_bits, W, bias_bits, bits, path=wq.QGEMM_PATH_AUTO, stream=None):
    """Packs W with the library's packer, runs qgemm, returns (Y bf16 bits, device weights)."""
    dw = wq.qgemm_pack(W, bits).to_device("cuda")
    X = to_dev_bf16(X_bits)
    b = None if bias_bits is None else to_dev_bf16(bias_bits)
    y = wq.qgemm(X, dw, bias=b, path=path, stream=stream)
    wq.check_device_status(stream)
    return from_dev_bf16(y), dw


def gpu_qgemm_packed(X_bits, dw, bias_bits, path=wq.QGEMM_PATH_AUTO):
    X = to_dev_bf16(X_bits)
    b = None if bias_bits is None else to_dev_bf16(bias_bits)
    y = wq.qgemm(X, dw, bias=b, path=path)
    wq.check_device_status()
    return from_dev_bf16(y)
