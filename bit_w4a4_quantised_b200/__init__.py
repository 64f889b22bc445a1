"""ASP (deflated form) NVFP4 W4A4 linear layer for NVIDIA B200 (sm_100a).

The compute path lives in ``libqwam.so`` (C-ABI, ``include/qwam.h``); this
package is its thin Python binding plus the seeded input generators.

    from bit_w4a4_quantised_b200 import binding as qw
    h = qw.prepare_weight(W, s, V, bias, hadamard_block=128)
    y = qw.linear(x, h)

Importing the package does not load the library; the first binding call does,
and raises if the library has not been built.
"""
from . import workloads  # noqa: F401

__all__ = ["workloads", "binding"]


def __getattr__(name):
    if name == "binding":
        import importlib
        return importlib.import_module(__name__ + ".binding")
    raise AttributeError(name)
