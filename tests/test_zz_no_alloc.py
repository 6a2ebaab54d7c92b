"""gdn_prefill_static_workspace: the cluster prefill with libgdn's own fixed
workspace array, called through the C ABI with ctypes.

Two calls in a row (different shapes, the second with an initial state and
cu_seqlens) are each compared bit for bit with gdn_prefill_ex(kernel=cluster)
given a caller-allocated workspace; the second call reuses the array the first
one left behind.  The file is named to be collected last, so the first call on
the device may come after every other test or, run alone, in a fresh process.
"""
import ctypes

import pytest
import torch

import gated_deltanet_04_b200 as gdn
from gated_deltanet_04_b200 import inputs

MAX_UNITS = 48  # GDN_STATIC_WORKSPACE_MAX_UNITS
UNSUPPORTED = 2


def _fn():
    from gated_deltanet_04_b200 import build
    build.build()
    lib = gdn.library()
    f = lib.gdn_prefill_static_workspace
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                  vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_rejects_more_units_than_the_array_holds():
    # returns before any CUDA call, so this runs without a GPU
    P = 0x10000
    f = _fn()
    args = [P, P + 0x1000, P + 0x2000, 0, P + 0x3000, P + 0x4000, None, P + 0x6000]
    assert f(*args, 2, 128, 16, 32, 128, 128, 64, P + 0x5000, None, None, None) == UNSUPPORTED
    assert f(*args[:7], None, 1, 128, 1, MAX_UNITS + 1, 128, 128, 64, P + 0x5000, None, None,
             None) == UNSUPPORTED
    assert f(*args[:7], None, 1, 128, 16, 48, 64, 64, 64, P + 0x5000, None, None,
             None) == UNSUPPORTED  # not a cluster-kernel shape


def _case(seed, T, Hqk, Hv, lengths=None, s0_std=0.0):
    gen = torch.Generator().manual_seed(seed)
    N = 1 if lengths is None else len(lengths)
    q, k, v, g, beta = inputs.make_tokens(T, Hqk, Hv, 128, 128, torch.bfloat16,
                                          inputs.G_SCALE_097, gen)
    s0 = inputs.make_state(N, Hv, 128, 128, s0_std, gen) if s0_std else None
    cu = None if lengths is None else inputs.cu_from_lengths(lengths).to(torch.int32)
    dev = torch.device("cuda:0")
    t = lambda x: None if x is None else x.to(dev).contiguous()
    return dict(q=t(q), k=t(k), v=t(v), g=t(g), beta=t(beta), s0=t(s0), cu=t(cu), N=N, T=T, Hqk=Hqk, Hv=Hv)


def _static(c):
    dev = c["q"].device
    o = torch.full((c["T"], c["Hv"], 128), float("nan"), dtype=torch.bfloat16, device=dev)
    sT = torch.full((c["N"], c["Hv"], 128, 128), float("nan"), dtype=torch.float32, device=dev)
    flag = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _fn()(_p(c["q"]), _p(c["k"]), _p(c["v"]), 0, _p(c["g"]), _p(c["beta"]), _p(c["s0"]),
               _p(c["cu"]), c["N"], c["T"], c["Hqk"], c["Hv"], 128, 128, 64, _p(o), _p(sT), _p(flag),
               stream)
    assert rc == 0, gdn.STATUS.get(rc, rc)
    return o, sT, flag


def _with_workspace(c):
    flag = torch.zeros(4, dtype=torch.int32, device=c["q"].device)
    o, sT = gdn.gdn_prefill(c["q"], c["k"], c["v"], c["g"], c["beta"], c["s0"], c["cu"],
                            chunk=64, kernel="cluster", error_flag=flag)
    return o, sT, flag


@pytest.mark.gpu
def test_static_workspace_matches_cluster_kernel_twice_in_a_row():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    cases = [
        _case(2101, 1000, 16, 48),                       # 48 units, ragged tail
        _case(2102, 1500, 4, 8, lengths=[700, 0, 63, 737, 0, 0], s0_std=0.05),  # varlen, state
    ]
    static = []
    for c in cases:  # both static calls back to back on the stream
        static.append(_static(c))
    torch.cuda.synchronize()
    for c, (o1, s1, f1) in zip(cases, static):
        o2, s2, f2 = _with_workspace(c)
        torch.cuda.synchronize()
        assert int(f1[0]) == 0 and int(f2[0]) == 0
        assert torch.equal(o1, o2), "o differs from gdn_prefill_ex(cluster)"
        assert torch.equal(s1, s2), "final state differs from gdn_prefill_ex(cluster)"
