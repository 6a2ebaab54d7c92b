"""gdn_prefill_slots: packed prefill whose sequences start from, and end in,
slots of a state pool (reset = a new request from zeros), against the oracle's
prefill_slots; then a decode step on the same pool."""
import numpy as np
import pytest
import torch

import gated_deltanet_04_b200 as gdn
import oracle
from gated_deltanet_04_b200 import inputs
from tests.helpers import check_o, check_state
from tests.test_prefill_gpu import DEV, synth

pytestmark = pytest.mark.gpu


def _case(lengths, Hqk, Hv, D, dtype, S, seed):
    cu = inputs.cu_from_lengths(lengths)
    inp, _ = synth(int(cu[-1]), Hqk, Hv, D, dtype, seed)
    gen = torch.Generator().manual_seed(seed + 7)
    pool = 0.05 * torch.randn(S, Hv, D, D, generator=gen)
    return inp, cu, pool


def _run(inp, cu, pool, idx, reset):
    t = lambda x: x.to(DEV).contiguous()
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    dpool = t(pool)
    o = gdn.gdn_prefill_slots(t(inp["q"]), t(inp["k"]), t(inp["v"]), t(inp["g"]), t(inp["beta"]),
                              dpool, t(torch.tensor(idx, dtype=torch.int32)),
                              None if reset is None else t(torch.tensor(reset, dtype=torch.int32)),
                              t(cu.to(torch.int32)), error_flag=flag)
    torch.cuda.synchronize()
    return o.cpu(), dpool.cpu(), int(flag[0])


def _oracle(inp, cu, pool, idx, reset):
    return oracle.prefill_slots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], pool,
                                np.array(idx), None if reset is None else np.array(reset),
                                cu.to(torch.int64))


def _check_slots(new, ref, pool, idx):
    for s in idx:
        check_state(new[s][None], torch.from_numpy(ref[s][None]), f"slot {s}")
    untouched = [s for s in range(pool.shape[0]) if s not in idx]
    assert torch.equal(new[untouched], pool[untouched]), "a slot nobody names changed"


@pytest.mark.parametrize("lengths,Hv,idx,reset", [
    ([0, 64, 200, 1, 333], 6, [7, 2, 5, 0, 3], [0, 1, 0, 1, 0]),   # pool kernel (30 units)
    ([97] * 16, 6, list(range(15, -1, -1)), [i % 3 == 0 for i in range(16)]),  # single CTA (96 units)
])
def test_prefill_slots_against_oracle(lengths, Hv, idx, reset):
    S = max(idx) + 3
    inp, cu, pool = _case(lengths, 2, Hv, 128, torch.bfloat16, S, seed=9500 + len(lengths))
    reset = [int(r) for r in reset]
    o, new, err = _run(inp, cu, pool, idx, reset)
    assert err == 0
    o_ref, ref = _oracle(inp, cu, pool, idx, reset)
    check_o(o, o_ref)
    _check_slots(new, ref, pool, idx)


def test_prefill_slots_fp32_recurrent_no_reset():
    inp, cu, pool = _case([50, 0, 129], 1, 2, 32, torch.float32, 4, seed=9600)
    idx = [3, 0, 2]
    o, new, err = _run(inp, cu, pool, idx, None)
    assert err == 0
    o_ref, ref = _oracle(inp, cu, pool, idx, None)
    check_o(o, o_ref)
    _check_slots(new, ref, pool, idx)


def test_prefill_slots_bad_index_is_reported_and_not_stored():
    """An out-of-range slot raises GDN_ERR_BAD_SLOT; that sequence runs from
    zeros and stores nothing; the others are unaffected."""
    inp, cu, pool = _case([70, 40], 2, 6, 128, torch.bfloat16, 3, seed=9700)
    o, new, err = _run(inp, cu, pool, [1, 3], None)
    assert gdn.STATUS.get(err) == "GDN_ERR_BAD_SLOT"
    o_ref, ref = _oracle(inp, cu, pool, [1, 2], [0, 1])  # sequence 1 as a reset into a spare slot
    check_o(o, o_ref)
    check_state(new[1][None], torch.from_numpy(ref[1][None]), "slot 1")
    assert torch.equal(new[[0, 2]], pool[[0, 2]])


def test_prefill_then_decode_on_the_same_pool():
    """Continuous batching: prefill three requests into their slots, then one
    decode step of all three from those slots, against the oracle's two calls."""
    lengths, idx = [150, 64, 3], [4, 0, 2]
    inp, cu, pool = _case(lengths, 2, 6, 128, torch.bfloat16, 5, seed=9800)
    _, new, err = _run(inp, cu, pool, idx, [1, 0, 1])
    assert err == 0
    _, ref = _oracle(inp, cu, pool, idx, [1, 0, 1])
    dec, _ = synth(3, 2, 6, 128, torch.bfloat16, seed=9801)
    t = lambda x: x.to(DEV).contiguous()
    dpool = t(new)
    od = gdn.gdn_decode_step_slots(t(dec["q"]), t(dec["k"]), t(dec["v"]), t(dec["g"]),
                                   t(dec["beta"]), dpool, t(torch.tensor(idx, dtype=torch.int32)))
    torch.cuda.synchronize()
    od_ref, ref2 = oracle.decode_step_slots(dec["q"], dec["k"], dec["v"], dec["g"], dec["beta"],
                                            ref, np.array(idx))
    check_o(od.cpu(), od_ref)
    for s in idx:
        check_state(dpool.cpu()[s][None], torch.from_numpy(ref2[s][None]), f"slot {s}")
