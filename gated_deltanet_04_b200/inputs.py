"""Seeded synthetic inputs for the gated delta rule.

This module is shared by the CUDA path's tests/benchmark and by the fp64
oracle's tests.  It holds none of the method's arithmetic: it only draws
random tensors with the workload's shapes and distributions and lays them out
in the library's token-major packed format.

Workloads (recipe; the model pages fix no kernel workload, so these shapes are
the hot path's own, for the "three DeltaNet, one attention" hybrid stack of
the pages "Layouts híbridos: três DeltaNet, uma attention" and "Qwen3.8-27B
架构深读", section 四):

* ``tiny``      N=1, T=64, Hqk=Hv=2, Dk=Dv=16, chunk 16, fp32 q/k/v.
* ``layer4k``   N=1, T=4096, Hqk=16, Hv=48, Dk=Dv=128, chunk 64, bf16 q/k/v.
* ``long256k``  as ``layer4k`` with T=262,144.
* ``decode256`` 256 sequences x 1 token, 48 layers, 48 v / 16 q-k heads,
                D=128, fp32 states ~ N(0, 0.05^2) updated in place.
* ``varlen32``  32 sequences, lengths uniform in [512, 16384], packed with
                cu_seqlens, fp32 initial states ~ N(0, 0.05^2), each sequence
                split at a uniform point in [1, L-1].

Distributions: q, k ~ N(0,1) then divided by their L2 norm over D per
(token, head) in fp32 and rounded to the I/O dtype; v ~ N(0,1);
beta = sigmoid(N(0,1)); g = -s * softplus(N(0,1)) with s = 1 for ``tiny`` and
s = -ln(0.97)/ln(2) otherwise, so that the median decay exp(g) is exactly 0.97
(softplus is monotone and softplus(0) = ln 2).  g and beta are fp32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# median(exp(g)) = 0.97 when g = -G_SCALE * softplus(x), x ~ N(0,1)
G_SCALE_097 = -math.log(0.97) / math.log(2.0)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    T: int
    Hqk: int
    Hv: int
    Dk: int
    Dv: int
    chunk: int
    io_dtype: torch.dtype
    g_scale: float
    s0_std: float  # 0 -> zero initial state
    seed: int
    layers: int = 1
    varlen: Optional[tuple] = None  # (min_len, max_len) when lengths are drawn


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 2, 2, 16, 16, 16, torch.float32, 1.0, 0.0, 1000),
    "layer4k": Workload("layer4k", 1, 4096, 16, 48, 128, 128, 64, torch.bfloat16,
                        G_SCALE_097, 0.0, 1001),
    "long256k": Workload("long256k", 1, 262144, 16, 48, 128, 128, 64, torch.bfloat16,
                         G_SCALE_097, 0.0, 1002),
    "decode256": Workload("decode256", 256, 256, 16, 48, 128, 128, 1, torch.bfloat16,
                          G_SCALE_097, 0.05, 1003, layers=48),
    "varlen32": Workload("varlen32", 32, -1, 16, 48, 128, 128, 64, torch.bfloat16,
                         G_SCALE_097, 0.05, 1004, varlen=(512, 16384)),
}


def _normal(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _l2_normalised(x):
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def draw_lengths(N, lo, hi, gen, device="cpu"):
    """Sequence lengths uniform in [lo, hi] (inclusive)."""
    return torch.randint(lo, hi + 1, (N,), generator=gen, device=device, dtype=torch.int64)


def cu_from_lengths(lengths):
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(torch.as_tensor(lengths, dtype=torch.int64), 0)
    return cu


def make_tokens(T, Hqk, Hv, Dk, Dv, io_dtype, g_scale, gen, device="cpu"):
    """q,k [T,Hqk,Dk], v [T,Hv,Dv] in io_dtype; g, beta [T,Hv] fp32."""
    q = _l2_normalised(_normal((T, Hqk, Dk), gen, device)).to(io_dtype)
    k = _l2_normalised(_normal((T, Hqk, Dk), gen, device)).to(io_dtype)
    v = _normal((T, Hv, Dv), gen, device).to(io_dtype)
    g = -g_scale * torch.nn.functional.softplus(_normal((T, Hv), gen, device))
    beta = torch.sigmoid(_normal((T, Hv), gen, device))
    return q, k, v, g.contiguous(), beta.contiguous()


def make_state(N, Hv, Dv, Dk, std, gen, device="cpu"):
    if std == 0.0:
        return torch.zeros((N, Hv, Dv, Dk), dtype=torch.float32, device=device)
    return std * _normal((N, Hv, Dv, Dk), gen, device)


def make_prefill(name_or_wl, device="cpu", seed=None, T=None):
    """Inputs of a prefill workload as a dict of tensors on ``device``.

    Keys: q, k, v, g, beta, s0 (None when the workload starts from zeros),
    cu_seqlens (int32, None for a single sequence), lengths, split (varlen
    only: per-sequence split points) and wl (the Workload).  ``T`` overrides
    the token count of a single-sequence workload (for reduced samples).
    """
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed if seed is None else seed)
    out = {"wl": wl}
    if wl.varlen is not None:
        lengths = draw_lengths(wl.N, wl.varlen[0], wl.varlen[1], gen, device).cpu()
        # split point of sequence n: uniform integer in [1, L_n - 1]
        split = torch.stack([torch.randint(1, int(L), (1,), generator=gen, device=device).cpu()[0]
                             for L in lengths])
        cu = cu_from_lengths(lengths)
        Ttot = int(cu[-1])
        out.update(lengths=lengths, split=split)
    else:
        Ttot = wl.T if T is None else T
        cu = None
        out.update(lengths=torch.tensor([Ttot]), split=None)
    q, k, v, g, beta = make_tokens(Ttot, wl.Hqk, wl.Hv, wl.Dk, wl.Dv, wl.io_dtype, wl.g_scale,
                                   gen, device)
    N = wl.N if wl.varlen is not None else 1
    s0 = make_state(N, wl.Hv, wl.Dv, wl.Dk, wl.s0_std, gen, device) if wl.s0_std else None
    out.update(q=q, k=k, v=v, g=g, beta=beta, s0=s0,
               cu_seqlens=None if cu is None else cu.to(torch.int32).to(device), T=Ttot, N=N)
    return out


def make_decode_layer(layer, device="cpu", seed=None, N=None, wl=None):
    """One layer of the batched decode workload: q,k [N,Hqk,Dk], v [N,Hv,Dv],
    g,beta [N,Hv] and the pre-existing state [N,Hv,Dv,Dk] fp32."""
    wl = wl or WORKLOADS["decode256"]
    N = wl.N if N is None else N
    gen = torch.Generator(device=device)
    gen.manual_seed((wl.seed if seed is None else seed) * 1000 + layer)
    q, k, v, g, beta = make_tokens(N, wl.Hqk, wl.Hv, wl.Dk, wl.Dv, wl.io_dtype, wl.g_scale,
                                   gen, device)
    state = make_state(N, wl.Hv, wl.Dv, wl.Dk, wl.s0_std, gen, device)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "state": state, "N": N, "wl": wl}


def split_packed(inp):
    """Split every sequence of a packed varlen batch at inp['split'][n].

    Returns (first, second): two dicts with q,k,v,g,beta and cu_seqlens (int64,
    host) for the leading and trailing parts of every sequence.  Pure
    re-indexing; no arithmetic of the method.
    """
    lengths = inp["lengths"].tolist()
    split = inp["split"].tolist()
    cu = cu_from_lengths(lengths).tolist()
    idx_a, idx_b = [], []
    for n, L in enumerate(lengths):
        s = split[n]
        idx_a.append(torch.arange(cu[n], cu[n] + s))
        idx_b.append(torch.arange(cu[n] + s, cu[n] + L))
    ia = torch.cat(idx_a)
    ib = torch.cat(idx_b)
    parts = []
    for idx, lens in ((ia, split), (ib, [L - s for L, s in zip(lengths, split)])):
        dev = inp["q"].device
        idx = idx.to(dev)
        parts.append({key: inp[key].index_select(0, idx) for key in ("q", "k", "v", "g", "beta")}
                     | {"cu_seqlens": cu_from_lengths(lens), "T": int(sum(lens))})
    return parts[0], parts[1]
