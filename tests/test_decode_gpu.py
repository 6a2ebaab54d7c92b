"""GPU parity of gdn_decode_step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_04_b200 as gdn
from gated_deltanet_04_b200 import inputs
from tests.helpers import check_o, check_state

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_deltanet_04_b200 import build
    build.build()


def oracle_step(layer):
    return oracle.decode_step(layer["q"], layer["k"], layer["v"], layer["g"], layer["beta"],
                              layer["state"])


@pytest.mark.parametrize("Dk,Dv,dtype", [(16, 16, torch.float32), (16, 12, torch.bfloat16),
                                         (32, 40, torch.float32), (64, 64, torch.bfloat16),
                                         (128, 128, torch.bfloat16), (128, 7, torch.float32)])
def test_decode_small_shapes(Dk, Dv, dtype):
    gen = torch.Generator().manual_seed(Dk * 1000 + Dv)
    N, Hqk, Hv = 9, 2, 6
    q, k, _, g, beta = inputs.make_tokens(N, Hqk, Hv, Dk, Dk, dtype, inputs.G_SCALE_097, gen)
    v = torch.randn(N, Hv, Dv, generator=gen).to(dtype)
    state = 0.05 * torch.randn(N, Hv, Dv, Dk, generator=gen)
    layer = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "state": state}
    o_ref, s_ref = oracle_step(layer)
    st = state.to(DEV)
    o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st)
    torch.cuda.synchronize()
    check_o(o.cpu(), o_ref)
    check_state(st.cpu(), s_ref)


@pytest.mark.parametrize("N,Hqk,Hv", [(1, 1, 1), (37, 2, 4), (38, 2, 4), (75, 2, 4),
                                       (8, 16, 48)])
def test_decode_staged_unit_counts(N, Hqk, Hv):
    """The D = 128 kernel splits N * Hv units into one contiguous range per CTA
    (one CTA per SM) and spreads the units % grid left over as single rows over
    all CTAs.  Unit counts below, at and just past a 148-SM grid, and 2.6 grids
    with 88 left over, must all match the oracle."""
    gen = torch.Generator().manual_seed(N * 100 + Hv)
    q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, 128, 128, torch.bfloat16,
                                          inputs.G_SCALE_097, gen)
    state = 0.05 * torch.randn(N, Hv, 128, 128, generator=gen)
    layer = {"q": q, "k": k, "v": v, "g": g, "beta": beta, "state": state}
    o_ref, s_ref = oracle_step(layer)
    st = state.to(DEV)
    o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st)
    torch.cuda.synchronize()
    check_o(o.cpu(), o_ref)
    check_state(st.cpu(), s_ref)


def test_decode_repeated_steps_track_recurrence():
    """Eight decode steps in a row equal one 8-token prefill of each sequence."""
    gen = torch.Generator().manual_seed(77)
    N, Hqk, Hv, D, steps = 4, 2, 6, 128, 8
    q, k, v, g, beta = inputs.make_tokens(N * steps, Hqk, Hv, D, D, torch.bfloat16,
                                          inputs.G_SCALE_097, gen)
    s0 = 0.05 * torch.randn(N, Hv, D, D, generator=gen)
    # token t of sequence n sits at row n*steps + t of the packed prefill layout
    cu = torch.arange(N + 1, dtype=torch.int64) * steps
    o_ref, s_ref = oracle.recurrent(q, k, v, g, beta, s0, cu)
    st = s0.to(DEV)
    outs = []
    for t in range(steps):
        rows = torch.arange(N) * steps + t
        o = gdn.gdn_decode_step(q[rows].to(DEV), k[rows].to(DEV), v[rows].to(DEV),
                                g[rows].to(DEV), beta[rows].to(DEV), st)
        outs.append(o.cpu())
    torch.cuda.synchronize()
    o_all = torch.stack(outs, 1).reshape(N * steps, Hv, D)
    check_o(o_all, o_ref)
    check_state(st.cpu(), s_ref)


def test_decode256_all_layers_sampled():
    """The batched-decode workload as the bench runs it: 256 sequences, 48 layers,
    each with its own 768 MiB fp32 state, updated in place; layers 0, 23 and 47
    are compared in full with the oracle."""
    wl = inputs.WORKLOADS["decode256"]
    check_layers = {0, 23, 47}
    for layer_id in range(wl.layers):
        layer = inputs.make_decode_layer(layer_id, device="cuda")
        pre = {key: layer[key].cpu() for key in ("q", "k", "v", "g", "beta", "state")} \
            if layer_id in check_layers else None
        o = gdn.gdn_decode_step(layer["q"], layer["k"], layer["v"], layer["g"], layer["beta"],
                                layer["state"])
        torch.cuda.synchronize()
        if pre is not None:
            o_ref, s_ref = oracle_step(pre)
            check_o(o.cpu(), o_ref, f"layer {layer_id} o")
            check_state(layer["state"].cpu(), s_ref, f"layer {layer_id} state")
        del layer
