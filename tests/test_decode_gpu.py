"""GPU parity of gdn_decode_step against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_04_b200 as gdn
from gated_deltanet_04_b200 import inputs
from tests.helpers import Guarded, check_o, check_state

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
    gst = Guarded(state.shape, torch.float32, DEV, fill=state)
    go = Guarded((N, Hv, v.shape[2]), v.dtype, DEV)
    st = gst.t
    o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st, o=go.t)
    torch.cuda.synchronize()
    gst.check("state")
    go.check("o")
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
    gst = Guarded(state.shape, torch.float32, DEV, fill=state)
    go = Guarded((N, Hv, v.shape[2]), v.dtype, DEV)
    st = gst.t
    o = gdn.gdn_decode_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st, o=go.t)
    torch.cuda.synchronize()
    gst.check("state")
    go.check("o")
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


# ---- bfloat16 state storage ----------------------------------------------------
# The kernel widens each stored bfloat16 element to fp32, steps in fp32 and
# rounds the new state once to bfloat16 (nearest even); the oracle steps in
# fp64 and rounds its result the same way.  Rounding moves an element by at
# most half a bfloat16 ulp, 2^-8 of its magnitude in the worst case, so the
# state's rel-L2 against the oracle's unrounded fp64 state is bounded by 2^-8
# (plus fp32 arithmetic error, ~1e-6).  Element by element, the kernel's value
# is the oracle's rounded value or a neighbour, the two rounding different
# inputs (an fp32 and an fp64 value) that can straddle a rounding boundary --
# up to fp32 error: a S + u k^T rounds its terms (|a S|, |u k| up to a few
# times max|S'|) at 2^-24, which for an element that nearly cancels can be
# several of its own (tiny) ulps, hence an absolute slack of 2^-22 max|S'|.

BF16_STATE_REL_L2 = 2.0 ** -8


def bf16_ulp(x):
    _, e = np.frexp(np.asarray(x, dtype=np.float64))
    return np.ldexp(1.0, e - 8)


def check_bf16_state(s_gpu, s_new64, s_rounded):
    g64 = s_gpu.double().numpy()
    rl = np.linalg.norm((g64 - s_new64).ravel()) / np.linalg.norm(s_new64.ravel())
    assert rl <= BF16_STATE_REL_L2, f"bf16 state rel-L2 {rl:.3e}"
    diff = np.abs(g64 - s_rounded)
    slack = 2.0 ** -22 * np.max(np.abs(s_new64))
    assert np.all(diff <= bf16_ulp(s_rounded) * 1.0000001 + slack), \
        "bf16 state off by more than 1 ulp plus fp32 error"
    same = float(np.mean(diff == 0))
    assert same >= 0.99, f"only {same:.4f} of the bf16 state equals the oracle's rounding"
    return rl, same


@pytest.mark.parametrize("N,Hqk,Hv,dtype", [(1, 1, 1, torch.bfloat16), (38, 2, 4, torch.bfloat16),
                                            (8, 16, 48, torch.bfloat16), (9, 2, 6, torch.float32)])
def test_decode_bf16_state(N, Hqk, Hv, dtype):
    gen = torch.Generator().manual_seed(5000 + N * 10 + Hv)
    q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, 128, 128, dtype, inputs.G_SCALE_097, gen)
    state = (0.05 * torch.randn(N, Hv, 128, 128, generator=gen)).to(torch.bfloat16)
    o_ref, s_new, s_rounded = oracle.decode_step_bf16_state(q, k, v, g, beta, state)
    st = state.to(DEV)
    o = gdn.gdn_decode_step_bf16_state(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), st)
    torch.cuda.synchronize()
    check_o(o.cpu(), o_ref)
    check_bf16_state(st.cpu(), s_new, s_rounded)


def test_decode_bf16_state_repeated_steps():
    """Eight bfloat16-state steps against eight oracle bfloat16-state steps.  Each
    side rounds its own state every step; a 1-ulp difference at one step is
    carried (and contracted) by the next, so after m steps the state's rel-L2 is
    within m half-ulps: 8 * 2^-9."""
    gen = torch.Generator().manual_seed(6001)
    N, Hqk, Hv, steps = 4, 2, 6, 8
    state = (0.05 * torch.randn(N, Hv, 128, 128, generator=gen)).to(torch.bfloat16)
    s_ref = state
    st = state.to(DEV)
    for t in range(steps):
        q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, 128, 128, torch.bfloat16,
                                              inputs.G_SCALE_097, gen)
        o_ref, _, s_ref = oracle.decode_step_bf16_state(q, k, v, g, beta, s_ref)
        o = gdn.gdn_decode_step_bf16_state(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV),
                                           beta.to(DEV), st)
        torch.cuda.synchronize()
        check_o(o.cpu(), o_ref, what=f"o step {t}")
    g64 = st.cpu().double().numpy()
    rl = np.linalg.norm((g64 - s_ref).ravel()) / np.linalg.norm(s_ref.ravel())
    assert rl <= steps * 2.0 ** -9, f"state rel-L2 after {steps} steps {rl:.3e}"


def test_decode_bf16_state_decode256_layer():
    """The decode workload's shape (256 sequences x 48 heads) with a bfloat16
    state: the full layer against the oracle."""
    wl = inputs.WORKLOADS["decode256"]
    layer = inputs.make_decode_layer(0, device="cpu")
    state = layer["state"].to(torch.bfloat16)
    o_ref, s_new, s_rounded = oracle.decode_step_bf16_state(layer["q"], layer["k"], layer["v"],
                                                             layer["g"], layer["beta"], state)
    st = state.to(DEV)
    o = gdn.gdn_decode_step_bf16_state(layer["q"].to(DEV), layer["k"].to(DEV), layer["v"].to(DEV),
                                       layer["g"].to(DEV), layer["beta"].to(DEV), st)
    torch.cuda.synchronize()
    assert o.shape == (wl.N, wl.Hv, wl.Dv)
    check_o(o.cpu(), o_ref)
    check_bf16_state(st.cpu(), s_new, s_rounded)


# ---- continuous batching: states in a pool of slots ----------------------------

def run_slots(q, k, v, g, beta, pool, idx, reset, flag=None):
    t = lambda x: None if x is None else x.to(DEV).contiguous()
    pd = pool.to(DEV)
    o = torch.full(v.shape, 7.0, dtype=v.dtype, device=DEV)
    gdn.gdn_decode_step_slots(t(q), t(k), t(v), t(g), t(beta), pd,
                              torch.as_tensor(idx, dtype=torch.int32).to(DEV),
                              None if reset is None else torch.as_tensor(reset, dtype=torch.int32).to(DEV),
                              o=o, error_flag=flag)
    torch.cuda.synchronize()
    return o.cpu(), pd.cpu()


@pytest.mark.parametrize("D,N,S,Hqk,Hv", [(128, 7, 20, 2, 6), (64, 7, 20, 2, 6),
                                          (128, 256, 300, 16, 48)])
def test_decode_slots(D, N, S, Hqk, Hv):
    """Entries scattered over a pool in shuffled order, about one in five
    starting a new request: o and every named slot match the oracle, and the
    slots nobody names come back bit for bit."""
    gen = torch.Generator().manual_seed(7000 + D + N)
    q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, D, D, torch.bfloat16, inputs.G_SCALE_097, gen)
    pool = 0.05 * torch.randn(S, Hv, D, D, generator=gen)
    idx = torch.randperm(S, generator=gen)[:N]
    reset = (torch.rand(N, generator=gen) < 0.2).to(torch.int32)
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    o, pd = run_slots(q, k, v, g, beta, pool, idx, reset, flag)
    assert int(flag[0]) == 0
    o_ref, pool_ref = oracle.decode_step_slots(q, k, v, g, beta, pool, idx, reset)
    check_o(o, o_ref)
    check_state(pd[idx], pool_ref[idx.numpy()])
    untouched = torch.ones(S, dtype=torch.bool)
    untouched[idx] = False
    assert torch.equal(pd[untouched], pool[untouched])


@pytest.mark.parametrize("D", [128, 64])
def test_decode_slots_bad_index_sets_flag_and_writes_nothing(D):
    gen = torch.Generator().manual_seed(7100 + D)
    N, S, Hqk, Hv = 5, 8, 2, 4
    q, k, v, g, beta = inputs.make_tokens(N, Hqk, Hv, D, D, torch.bfloat16, inputs.G_SCALE_097, gen)
    pool = 0.05 * torch.randn(S, Hv, D, D, generator=gen)
    idx = torch.tensor([3, 8, 0, -1, 6])  # entries 1 and 3 name no slot
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    o, pd = run_slots(q, k, v, g, beta, pool, idx, None, flag)
    assert int(flag[0]) == 6  # GDN_ERR_BAD_SLOT
    good = [0, 2, 4]
    o_ref, pool_ref = oracle.decode_step_slots(q[good], k[good], v[good], g[good], beta[good],
                                               pool, idx[good])
    check_o(o[good], o_ref)
    check_state(pd[idx[good]], pool_ref[idx[good].numpy()])
    assert torch.all(o[[1, 3]] == 7.0)           # the bad entries wrote no output
    others = [s for s in range(S) if s not in idx[good].tolist()]
    assert torch.equal(pd[others], pool[others])  # ... and no state
