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


def prepare(case, wd_out=False, variant="deflated", fmt="nvfp4"):
    import torch
    from bit_w4a4_quantised_b200 import binding as qw
    x, W, s, V, bias = to_device(case)
    wd = torch.empty((case.N, case.K), dtype=torch.float32, device="cuda") if wd_out else None
    h = qw.prepare_weight(W, s, V, bias, case.b, wd_out=wd, variant=variant, fmt=fmt)
    return h, x, wd


def codes_of(packed_dev) -> np.ndarray:
    """Device packed codes [rows, K/2] -> unpacked numpy codes [rows, K]."""
    return nvfp4.unpack_nibbles(packed_dev.cpu().numpy())


def scales_of(tiled_dev, rows: int, K: int) -> np.ndarray:
    return nvfp4.unswizzle_scales(tiled_dev.cpu().numpy(), rows, K)


def bf16_to_np(t) -> np.ndarray:
    import torch
    return t.to(torch.float32).cpu().numpy().astype(np.float64)


def local_rel_errors(got, ref, block: int = 128):
    """Largest relative Frobenius error over single rows and over 128-column
    blocks (all rows): a wrong tile, a wrong ragged tail or one bad row shows
    here even when the whole-tensor error is small."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    d = got - ref
    row = np.linalg.norm(d, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    cols = [np.linalg.norm(d[:, j:j + block]) / max(np.linalg.norm(ref[:, j:j + block]), 1e-30)
            for j in range(0, ref.shape[1], block)]
    return float(row.max()), float(max(cols))


def device_operand_reference(case, h, x, rows=None, variant="deflated"):
    """float64 y from the device's own quantised operands: the activation codes,
    scales and g_x the prologue produced for x, the weight codes, scales and
    g_w of the handle, plus the exact float64 branch u (W~V)^T and the bias.
    Code flips against the float64 oracle (allowed: >= 99.9 % equal) drop out,
    so what remains between this and the device's y is the GEMM's fp32
    accumulation, the bf16 branch operands and the bf16 output rounding."""
    from bit_w4a4_quantised_b200 import binding as qw
    from oracle import asp
    d = qw.debug_prologue(x, h)
    w = qw.export_weight(h)
    rows = np.arange(case.M) if rows is None else np.asarray(rows)
    a_codes = codes_of(d["codes"])[rows]
    a_sc = scales_of(d["scales"], case.M, case.K)[rows]
    deq_a = nvfp4.dequantize(a_codes, a_sc, np.float32(d["g_x"].item()))
    deq_b = nvfp4.dequantize(codes_of(w["codes"]), scales_of(w["scales"], case.N, case.K), np.float32(h.g_w))
    y = asp.nvfp4_gemm(deq_a, deq_b)
    if case.r:
        u = asp.activation_prologue(case.x[rows], case.s, case.V, case.b, fp4=False)["u"]
        if variant == "shared":   # the branch weight of the shared arm: deq(stored weight) V
            L = deq_b @ np.asarray(case.V, dtype=np.float64)
        else:
            L = asp.prepare_weight(case.W, case.s, case.V, case.b, fp4=False)["L"]
        y = y + u @ L.T
    return y + np.asarray(case.bias, dtype=np.float64)[None, :]


def sample_rows(M: int, n: int = 48, seed: int = 7) -> np.ndarray:
    """Rows checked at full size: the first and last rows of the first, a middle
    and the last 128-row tiles, plus n seeded random rows."""
    rng = np.random.default_rng(seed)
    edge = [0, 1, 127, 128, 255, 256, M // 2, M - 129, M - 128, M - 2, M - 1]
    rows = np.concatenate([np.array(edge), rng.integers(0, M, n)])
    return np.unique(np.clip(rows, 0, M - 1))
