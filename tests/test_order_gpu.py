"""GPU parity of the recall-first step order (the page's per-head step function
takes the recall S k before the decay; section 三 of "Qwen3.8-27B 架构深读:
Gated DeltaNet 混合线性注意力与 262K 长上下文") against the oracle's flagged
variant, through gdn_prefill_order and gdn_decode_step_order.

In the chunked kernels the order only moves the decay of the recall terms from
Gamma_r to Gamma_{r-1}, so the chunked kernels, the token-recurrent kernel and
the oracle are compared on ragged packed batches, on decays strong enough to
take the kernels' exponent-difference path, and with a = 1, where both orders
are the same rule.  Tolerances: tests/helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_04_b200 as gdn
from gated_deltanet_04_b200 import inputs
from tests.helpers import check_o, check_state

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
KERNELS = ["pool", "cluster", "single_cta", "recurrent"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_deltanet_04_b200 import build
    build.build()


def synth(T, Hqk, Hv, seed, N=1, s0_std=0.05, g_scale=inputs.G_SCALE_097):
    gen = torch.Generator().manual_seed(seed)
    q, k, v, g, beta = inputs.make_tokens(T, Hqk, Hv, 128, 128, torch.bfloat16, g_scale, gen)
    s0 = inputs.make_state(N, Hv, 128, 128, s0_std, gen) if s0_std else None
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta}, s0


def run(inp, s0, cu, kernel, order):
    t = lambda x: None if x is None else x.to(DEV).contiguous()
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    o, sT = gdn.gdn_prefill(t(inp["q"]), t(inp["k"]), t(inp["v"]), t(inp["g"]), t(inp["beta"]),
                            t(s0), None if cu is None else cu.to(torch.int32).to(DEV),
                            kernel=kernel, order=order, error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag[0]) == 0, f"device error {gdn.STATUS.get(int(flag[0]))}"
    return o.cpu(), sT.cpu()


def oracle_rf(inp, s0, cu=None):
    return oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], s0,
                            None if cu is None else cu.to(torch.int64),
                            order=oracle.ORDER_ILLUSTRATIVE)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_recall_first_packed(kernel):
    lengths = [0, 65, 64, 1, 200, 130]
    cu = inputs.cu_from_lengths(lengths)
    inp, s0 = synth(int(cu[-1]), 2, 6, seed=900, N=len(lengths))
    o, sT = run(inp, s0, cu, kernel, "recall_first")
    o_ref, s_ref = oracle_rf(inp, s0, cu)
    check_o(o, o_ref)
    check_state(sT, s_ref)
    # and it is not the standard order: the two differ by b (1 - a) (S k) k^T per step
    o_std, _ = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], s0,
                                cu.to(torch.int64))
    assert np.abs(o_std - o_ref).max() > 1e-3


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("case", ["strong_decay", "decay_1", "b1"])
def test_prefill_recall_first_gates(case, kernel):
    """Strong decays (|gamma| past the kernels' 60 bound) take the
    exponent-difference path for A; b = 1 writes hardest."""
    inp, s0 = synth(130, 1, 3, seed=910)
    if case == "strong_decay":
        inp["g"].fill_(-30.0)
    elif case == "decay_1":
        inp["g"].fill_(-1.0)
    elif case == "b1":
        inp["beta"].fill_(1.0)
    o, sT = run(inp, s0, None, kernel, "recall_first")
    o_ref, s_ref = oracle_rf(inp, s0)
    check_o(o, o_ref)
    check_state(sT, s_ref)


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_orders_agree_without_decay(kernel):
    """a = 1: both orders are the same rule, so the GPU gives the same result."""
    inp, s0 = synth(200, 2, 6, seed=920)
    inp["g"].zero_()
    o1, s1 = run(inp, s0, None, kernel, "standard")
    o2, s2 = run(inp, s0, None, kernel, "recall_first")
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_prefill_recall_first_layer4k():
    inp = inputs.make_prefill("layer4k")
    o, sT = run(inp, None, None, "auto", "recall_first")
    o_ref, s_ref = oracle_rf(inp, None)
    check_o(o, o_ref)
    check_state(sT, s_ref)


@pytest.mark.parametrize("D,N,Hqk,Hv", [(64, 9, 2, 6), (128, 9, 2, 6), (128, 38, 2, 4)])
def test_decode_recall_first(D, N, Hqk, Hv):
    gen = torch.Generator().manual_seed(930 + D + N)
    q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, D, D, torch.bfloat16, inputs.G_SCALE_097, gen)
    state = 0.05 * torch.randn(N, Hv, D, D, generator=gen)
    o_ref, s_ref = oracle.decode_step(q, k, v, g, beta, state, order=oracle.ORDER_ILLUSTRATIVE)
    st = state.to(DEV)
    o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st,
                            order="recall_first")
    torch.cuda.synchronize()
    check_o(o.cpu(), o_ref)
    check_state(st.cpu(), s_ref)
