"""The bounded-wait timeout path of the pool prefill kernel, on the GPU.

gdn_debug_prefill_pool_stall runs the pool kernel with one (sequence, head)
unit that its producers never prepare and a short limit on every spin on a
hand-off flag.  The skipped unit's chain then waits for a chunk that never
comes (a spin on a flag in global memory, with no copy in flight into its
shared memory) until the limit expires.  The test checks that the expired wait
is reported as GDN_ERR_TIMEOUT through the device flag, that the launch
returns, and that a normal call right after it on the same context still
matches the oracle.  Nothing here faults, traps or hangs the GPU: every wait
in the kernel is bounded, and the one that runs out is a flag spin.
"""
import ctypes

import pytest
import torch

import gated_deltanet_04_b200 as gdn
from tests.helpers import check_o, check_state
from tests.test_prefill_gpu import DEV, run_gpu, run_oracle, synth

pytestmark = pytest.mark.gpu
TIMEOUT = 4


def _stall_fn():
    from gated_deltanet_04_b200 import build
    build.build()
    f = gdn.library().gdn_debug_prefill_pool_stall
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i32, i64, i32, i32, i32, i32, i32,
                  vp, vp, vp, ctypes.c_size_t, vp, vp, i32, i64]
    f.restype = ctypes.c_int
    return f


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_stalled_unit_reports_timeout_and_the_context_stays_usable():
    T, Hqk, Hv = 640, 2, 6  # 10 chunks x 6 units
    inp, s0 = synth(T, Hqk, Hv, 128, torch.bfloat16, seed=2500, s0_std=0.05)
    d = {k_: v_.to(DEV).contiguous() for k_, v_ in inp.items()}
    s0d = s0.to(DEV)
    o = torch.empty_like(d["v"])
    sT = torch.empty_like(s0d)
    nbytes = gdn.gdn_prefill_workspace_bytes(1, T, Hqk, Hv, 128, 128, 64, "pool")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    f = _stall_fn()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = f(_p(d["q"]), _p(d["k"]), _p(d["v"]), 0, _p(d["g"]), _p(d["beta"]), _p(s0d), None, 1, T,
           Hqk, Hv, 128, 128, 64, _p(o), _p(sT), _p(ws), nbytes, _p(flag), stream, 4, 1 << 22)
    assert rc == 0
    torch.cuda.synchronize()  # the launch returns
    assert int(flag[0]) == TIMEOUT
    # the same context, right after: a normal call matches the oracle
    o2, s2 = run_gpu(inp, s0, kernel="pool")
    o_ref, s_ref = run_oracle(inp, s0)
    check_o(o2, o_ref)
    check_state(s2, s_ref)

