"""Helpers for the GPU parity tests: move seeded cases to the device, unpack
device buffers for comparison with the oracle."""
import numpy as np

from oracle import nvfp4


def to_device(case):
    import torch
    dev = torch.device("cuda")
    x = torch.from_numpy(case.x).to(dev).to(torch.bfloat16)      # exact: values are bf16
    W = torch.from_numpy(case.W).to(dev).to(torch.bfloat16)
    s = torch.from_numpy(case.s).to(dev)
    V = torch.from_numpy(case.V).to(dev).contiguous() if case.r else None
    bias = torch.from_numpy(case.bias).to(dev).to(torch.bfloat16)
    return x, W, s, V, bias


def prepare(case, wd_out=False):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    x, W, s, V, bias = to_device(case)
    wd = torch.empty((case.N, case.K), dtype=torch.float32, device="cuda") if wd_out else None
    h = qw.prepare_weight(W, s, V, bias, case.b, wd_out=wd)
    return h, x, wd


def codes_of(packed_dev) -> np.ndarray:
    """Device packed codes [rows, K/2] -> unpacked numpy codes [rows, K]."""
    return nvfp4.unpack_nibbles(packed_dev.cpu().numpy())


def scales_of(tiled_dev, rows: int, K: int) -> np.ndarray:
    return nvfp4.unswizzle_scales(tiled_dev.cpu().numpy(), rows, K)


def bf16_to_np(t) -> np.ndarray:
    import torch
    return t.to(torch.float32).cpu().numpy().astype(np.float64)
