"""Shared tolerance checks for GPU-vs-oracle parity.

Tolerances (fixed for this operator): bf16 outputs o within max-abs 2e-2 and
relative L2 5e-3 of the fp64 oracle; fp32 states within relative L2 1e-4.
The same thresholds apply to fp32 I/O.
"""
import numpy as np
import torch

O_MAX_ABS = 2e-2
O_REL_L2 = 5e-3
S_REL_L2 = 1e-4


def to64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rel_l2(x, ref):
    x, ref = to64(x), to64(ref)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return num / den if den > 0 else num


def max_abs(x, ref):
    x, ref = to64(x), to64(ref)
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def check_o(o_gpu, o_ref, what="o"):
    ra, rl = max_abs(o_gpu, o_ref), rel_l2(o_gpu, o_ref)
    assert ra <= O_MAX_ABS and rl <= O_REL_L2, f"{what}: max-abs {ra:.3e} rel-L2 {rl:.3e}"
    return ra, rl


def check_state(s_gpu, s_ref, what="state"):
    rl = rel_l2(s_gpu, s_ref)
    assert rl <= S_REL_L2, f"{what}: rel-L2 {rl:.3e}"
    return rl
