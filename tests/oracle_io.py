"""Conversions between torch tensors and the oracle's raw numpy arrays.

Bit-level only: fp16 stays float16, bf16 becomes its uint16 bit patterns,
fp8 codes stay uint8. No arithmetic of the method happens here.
"""
import numpy as np
import torch


def raw(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float16:
        return t.numpy()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.uint8, torch.int32, torch.int64, torch.float32):
        return t.numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(t.dtype)


def kind_of(t: torch.Tensor) -> str:
    return {torch.float16: "f16", torch.bfloat16: "bf16", torch.uint8: "fp8_e4m3"}[t.dtype]
