"""Shared test helpers: moving seeded inputs to the device and outputs back."""
import numpy as np


def to_dev_bf16(x_bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_np(t):
    return t.detach().cpu().numpy()


def bf16_tensor_bits(t) -> np.ndarray:
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
