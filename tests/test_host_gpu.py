"""gdn_prefill_host: one sequence from host memory, streamed through the device
in segments that carry the state, against the oracle and one device call."""
import pytest
import torch

import gated_deltanet_04_b200 as gdn
from tests.helpers import check_o, check_state
from tests.test_prefill_gpu import DEV, run_gpu, run_oracle, synth

pytestmark = pytest.mark.gpu


def _host(inp, s0=None, pin=True, **kw):
    h = lambda x: None if x is None else (x.contiguous().pin_memory() if pin else x.contiguous())
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    o, sT = gdn.gdn_prefill_host(h(inp["q"]), h(inp["k"]), h(inp["v"]), h(inp["g"]), h(inp["beta"]),
                                 h(s0), error_flag=flag, device=DEV, **kw)
    torch.cuda.synchronize()
    assert int(flag[0]) == 0, gdn.STATUS.get(int(flag[0]))
    return o, sT


@pytest.mark.parametrize("T,seg", [(5000, 1024), (4096, 1024), (700, 64), (64, 0), (1, 0)])
def test_segments_match_oracle_and_one_call(T, seg):
    """Ragged last segments, exact multiples, one-chunk segments, one segment:
    the streamed result against the oracle and against one gdn_prefill call on
    device buffers (pool kernel, 6 heads)."""
    inp, s0 = synth(T, 2, 6, 128, torch.bfloat16, seed=9100 + T, s0_std=0.05)
    s0 = s0[0]
    o, sT = _host(inp, s0, segment_tokens=seg)
    o_ref, s_ref = run_oracle(inp, s0[None])
    check_o(o, o_ref)
    check_state(sT[None], s_ref)
    o1, s1 = run_gpu(inp, s0[None])
    check_o(o, o1.double(), "streamed vs one call")
    check_state(sT[None], s1.double(), "streamed vs one call")


def test_layer_head_shape_no_initial_state():
    """The benchmark's head shape (16 q/k heads, 48 v-heads) over 8,192 tokens in
    four segments, no initial state."""
    inp, _ = synth(8192, 16, 48, 128, torch.bfloat16, seed=9200)
    o, sT = _host(inp, segment_tokens=2048)
    o_ref, s_ref = run_oracle(inp)
    check_o(o, o_ref)
    check_state(sT[None], s_ref)


def test_pageable_memory_and_fp32_recurrent():
    """Pageable host tensors (serialised copies) and the fp32 recurrent kernel
    (D = 32) give the same result as the oracle."""
    inp, s0 = synth(900, 1, 2, 32, torch.float32, seed=9300, s0_std=0.1)
    o, sT = _host(inp, s0[0], pin=False, segment_tokens=256)
    o_ref, s_ref = run_oracle(inp, s0)
    check_o(o, o_ref)
    check_state(sT[None], s_ref)


def test_empty_sequence_and_validation():
    """T = 0 returns the initial state; a segment length that is not a multiple
    of 64 and a short scratch are rejected."""
    inp, s0 = synth(0, 2, 6, 128, torch.bfloat16, seed=9400, s0_std=0.05)
    o, sT = _host(inp, s0[0])
    assert o.shape == (0, 6, 128)
    assert torch.equal(sT, s0[0])
    inp, _ = synth(300, 2, 6, 128, torch.bfloat16, seed=9401)
    with pytest.raises(gdn.GdnError) as e:
        _host(inp, segment_tokens=100)
    assert e.value.code == 1
    need = gdn.gdn_prefill_host_scratch_bytes(300, 2, 6, 128, 128, segment_tokens=128)
    short = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(gdn.GdnError) as e:
        _host(inp, segment_tokens=128, scratch=short)
    assert e.value.code == 1
