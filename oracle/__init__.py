"""Float64 CPU oracle for the ASP (deflated form) NVFP4 W4A4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA path (``bit_w4a4_quantised_b200/csrc``) and reads nothing the CUDA path
writes except where a test explicitly feeds it a GPU tensor to *check*.

Modules
-------
nvfp4
    E2M1 / E4M3 value tables, round-to-nearest-even encoders by brute-force
    table search, the fp32-exact two-level NVFP4 quantiser, dequantiser, nibble
    packing and the 128x4 scale-tile layout.
fp8
    The FP8 W8A8 arm's per-tensor E4M3 quantiser and its dequantisation.
int4
    The SVDQuant arm's INT4 group-64 quantiser (fp16 scales), its
    dequantisation and the exact integer group sums of its product.
asp
    Block Hadamard, smoothing, rank-r deflation and the full layer
    ``y = (x~V)(W~V)^T + NVFP4GEMM((I-VV^T)x~, W~(I-VV^T)) + bias`` in float64;
    the shared-weight arm's weight side; the FP8 arm (``fmt="fp8"``); the
    SVDQuant arm (``svdquant_linear``: no rotation, activation not deflated,
    INT4 group 64 on both sides).

Sources: "QuantWAMs: Calibrating at the Right Granularity for World Action
Models" (report), section "During inference" (FP8 W8A8 for the upgraded
Linears); "FastWAM UR3 3-task — 4-bit quantisations" (Hugging Face model card),
sections "What ASP is, and what the deflated form means" (the contract), the
top comparison table (numeric formats of both checkpoints), "Verification —
INT4 SVDQuant", "Files" (scale swizzle), and
"Verification — NVFP4 deflated ASP" (storage figures); "Q-WAM: 4-Bit Quantization
of World Action Models with Action-Subspace Protection", abstract (16-bit
low-rank branch, both sides as dense matmuls).

Parity status: every function here is pinned by a ``-m "not gpu"`` test in
``tests/test_oracle_*.py`` against closed forms, library routines, printed
figures or brute force; none is "parity unpinned".
"""
