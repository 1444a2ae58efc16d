"""Helpers shared by the GPU tests: move seeded numpy inputs to the device and
run the CUDA path through the binding (which calls the C ABI)."""
import numpy as np
import torch

import bitlinear_w1_a8_03_b200 as bl
from bitlinear_w1_a8_03_b200 import synth


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def as_input(a_f32, dtype):
    """(device tensor, oracle array) of one input in `dtype` ('f32' or 'bf16')."""
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(a_f32)
        return dev_bf16(bits), bits
    return dev_f32(a_f32), np.ascontiguousarray(a_f32, dtype=np.float32)


def gpu_quantize_weights(Wd):
    packed, alpha = bl.bitlinear_quantize_weights(Wd)
    return packed, alpha


def gpu_forward(xd, packed, alpha, N, bias=None):
    xq, beta = bl.bitlinear_quantize_act(xd)
    acc = torch.empty((xd.shape[0], N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, bias=bias, acc_out=acc)
    return xq, beta, acc, y


def np_(t):
    return t.detach().cpu().numpy()
