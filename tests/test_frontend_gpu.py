"""GPU parity of gdn_short_conv_norm, the mixer's kernel-4 causal convolution
with per-head q/k normalisation (page "Layouts híbridos: três DeltaNet, uma
attention", section 01), against the fp64 oracle, and of the front end
followed by the prefill.

The kernel computes in fp32 and rounds once to the io dtype; the oracle
computes in fp64.  Compared after the rounding: bf16 outputs equal the
oracle's rounding of its own result for at least 99% of elements and are
within one bf16 ulp plus fp32 error everywhere (the two round values that
differ by fp32 arithmetic error, which can straddle a rounding boundary).
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


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from gated_deltanet_04_b200 import build
    build.build()


def make(T, Hqk, Hv, seed, dtype=torch.bfloat16, N_state=None):
    gen = torch.Generator().manual_seed(seed)
    D = 128
    xq = torch.randn(T, Hqk, D, generator=gen).to(dtype)
    xk = torch.randn(T, Hqk, D, generator=gen).to(dtype)
    xv = torch.randn(T, Hv, D, generator=gen).to(dtype)
    wq = 0.5 * torch.randn(Hqk * D, 4, generator=gen)
    wk = 0.5 * torch.randn(Hqk * D, 4, generator=gen)
    wv = 0.5 * torch.randn(Hv * D, 4, generator=gen)
    st = None
    if N_state:
        st = torch.randn(N_state, 3, (2 * Hqk + Hv) * D, generator=gen).to(dtype).float()
    return xq, xk, xv, wq, wk, wv, st


def check_rounded(gpu, ref64, what):
    """bf16 output against the fp64 oracle value."""
    g = gpu.double().numpy()
    want = oracle.round_bf16(ref64)
    _, e = np.frexp(want)
    ulp = np.ldexp(1.0, e - 8)
    slack = 2.0 ** -20 * np.max(np.abs(ref64))
    diff = np.abs(g - want)
    assert np.all(diff <= ulp * 1.0000001 + slack), f"{what}: more than 1 ulp off"
    same = float(np.mean(diff == 0))
    assert same >= 0.99, f"{what}: only {same:.4f} identical"


def run(xq, xk, xv, wq, wk, wv, cu, st, out_state=True):
    t = lambda x: None if x is None else x.to(DEV).contiguous()
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    res = gdn.gdn_short_conv_norm(t(xq), t(xk), t(xv), t(wq), t(wk), t(wv),
                                  None if cu is None else cu.to(torch.int32).to(DEV), t(st),
                                  output_conv_state=out_state, error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag[0]) == 0
    return [None if r is None else r.cpu() for r in res]


@pytest.mark.parametrize("with_state", [False, True])
def test_short_conv_norm_packed(with_state):
    lengths = [0, 1, 2, 3, 70, 129]
    cu = inputs.cu_from_lengths(lengths)
    T = int(cu[-1])
    xq, xk, xv, wq, wk, wv, st = make(T, 2, 6, seed=8000, N_state=len(lengths) if with_state else None)
    q, k, v, s_out = run(xq, xk, xv, wq, wk, wv, cu, st)
    q_ref, k_ref, v_ref, s_ref = oracle.short_conv_norm(xq, xk, xv, wq, wk, wv, cu, st)
    check_rounded(q, q_ref, "q")
    check_rounded(k, k_ref, "k")
    check_rounded(v, v_ref, "v")
    assert torch.equal(s_out, torch.from_numpy(s_ref).float())  # raw inputs: exact


def test_short_conv_norm_split_and_carry_equals_one_shot():
    xq, xk, xv, wq, wk, wv, _ = make(200, 2, 6, seed=8100)
    full = run(xq, xk, xv, wq, wk, wv, None, None)
    for cut in (1, 2, 64, 131):
        a = run(xq[:cut], xk[:cut], xv[:cut], wq, wk, wv, None, None)
        b = run(xq[cut:], xk[cut:], xv[cut:], wq, wk, wv, None, a[3])
        for i in range(3):
            assert torch.equal(torch.cat([a[i], b[i]]), full[i]), (cut, i)
        assert torch.equal(b[3], full[3])


def test_short_conv_norm_fp32():
    xq, xk, xv, wq, wk, wv, st = make(100, 2, 6, seed=8200, dtype=torch.float32, N_state=1)
    q, k, v, _ = run(xq, xk, xv, wq, wk, wv, None, st)
    q_ref, k_ref, v_ref, _ = oracle.short_conv_norm(xq, xk, xv, wq, wk, wv, None, st)
    for g_, r_ in ((q, q_ref), (k, k_ref), (v, v_ref)):
        rel = np.linalg.norm(g_.double().numpy() - r_) / np.linalg.norm(r_)
        assert rel <= 1e-6, rel


def test_front_end_then_prefill_layer_shape():
    """Front end, then the prefill (pool kernel), on a 4096-token layer of the
    benchmark's head shape, against the oracle's front end (rounded to bf16 as
    the GPU stores it) followed by the oracle's recurrence."""
    T, Hqk, Hv = 4096, 16, 48
    xq, xk, xv, wq, wk, wv, _ = make(T, Hqk, Hv, seed=8300)
    gen = torch.Generator().manual_seed(8301)
    g = -inputs.G_SCALE_097 * torch.nn.functional.softplus(torch.randn(T, Hv, generator=gen))
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen))
    q, k, v = run(xq, xk, xv, wq, wk, wv, None, None, out_state=False)
    o, sT = gdn.gdn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV))
    torch.cuda.synchronize()
    q_ref, k_ref, v_ref, _ = oracle.short_conv_norm(xq, xk, xv, wq, wk, wv)
    r = lambda a: torch.from_numpy(oracle.round_bf16(a))
    o_ref, s_ref = oracle.recurrent(r(q_ref), r(k_ref), r(v_ref), g, beta)
    check_o(o.cpu(), o_ref)
    check_state(sT.cpu(), s_ref)


# ---- the front end fused into the pool prefill (gdn_prefill_conv) ----

def _fused_inputs(lengths, Hqk, Hv, seed, with_state):
    cu = inputs.cu_from_lengths(lengths)
    T = int(cu[-1])
    xq, xk, xv, wq, wk, wv, st = make(T, Hqk, Hv, seed=seed,
                                      N_state=len(lengths) if with_state else None)
    gen = torch.Generator().manual_seed(seed + 1)
    g = -inputs.G_SCALE_097 * torch.nn.functional.softplus(torch.randn(T, Hv, generator=gen))
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen))
    s0 = 0.05 * torch.randn(len(lengths), Hv, 128, 128, generator=gen) if with_state else None
    return cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0


def _fused(cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0):
    t = lambda x: None if x is None else x.to(DEV).contiguous()
    flag = torch.zeros(4, dtype=torch.int32, device=DEV)
    o, sT, st_out = gdn.gdn_prefill_conv(t(xq), t(xk), t(xv), t(wq), t(wk), t(wv), t(g), t(beta),
                                         t(s0), None if cu is None else cu.to(torch.int32).to(DEV),
                                         t(st), output_conv_state=True, error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag[0]) == 0, gdn.STATUS.get(int(flag[0]))
    return o.cpu(), sT.cpu(), st_out.cpu()


def _oracle_chain(cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0):
    q_ref, k_ref, v_ref, st_ref = oracle.short_conv_norm(xq, xk, xv, wq, wk, wv, cu, st)
    r = lambda a: torch.from_numpy(oracle.round_bf16(a))
    o_ref, s_ref = oracle.recurrent(r(q_ref), r(k_ref), r(v_ref), g, beta, s0,
                                    None if cu is None else cu.to(torch.int64))
    return o_ref, s_ref, st_ref


@pytest.mark.parametrize("with_state", [False, True])
def test_fused_front_end_prefill_packed(with_state):
    """Packed sequences (an empty one, a single chunk, ragged tails, chunks past
    the first) with and without carried conv and recurrent states, against the
    oracle's front end (rounded to bf16) then its recurrence."""
    args = _fused_inputs([0, 64, 200, 1, 777, 130], 2, 6, 8400, with_state)
    o, sT, st_out = _fused(*args)
    o_ref, s_ref, st_ref = _oracle_chain(*args)
    check_o(o, o_ref)
    check_state(sT, s_ref)
    assert torch.equal(st_out, torch.from_numpy(st_ref).float())  # raw inputs: exact


@pytest.mark.parametrize("Hqk,Hv", [(3, 3), (2, 4), (1, 5)])
def test_fused_front_end_other_group_sizes(Hqk, Hv):
    """Producer items of one and of two v-heads per q/k head (the group sizes
    other than 3 that the pool kernel uses: 3 heads share q/k with 1, 4 heads
    over 2 with 2, 5 over 1 with 1), packed sequences with carried states."""
    args = _fused_inputs([130, 1, 64, 257], Hqk, Hv, 8800 + 10 * Hqk + Hv, True)
    o, sT, st_out = _fused(*args)
    o_ref, s_ref, st_ref = _oracle_chain(*args)
    check_o(o, o_ref)
    check_state(sT, s_ref)
    assert torch.equal(st_out, torch.from_numpy(st_ref).float())


def test_fused_front_end_split_and_carry():
    """Each sequence split in two calls that carry the conv state and the
    recurrent state: matches the one-shot call and the oracle."""
    lengths = [300, 129, 64, 1000]
    split = [100, 64, 1, 555]
    cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0 = _fused_inputs(lengths, 2, 6, 8500, True)
    o1, s1, c1 = _fused(cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0)
    o_ref, s_ref, _ = _oracle_chain(cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0)
    check_o(o1, o_ref, "one-shot o")
    check_state(s1, s_ref, "one-shot state")
    pieces = [[], []]
    for n, L in enumerate(lengths):
        b = int(cu[n])
        pieces[0].append((b, b + split[n]))
        pieces[1].append((b + split[n], b + L))
    idx = lambda part: torch.cat([torch.arange(a, e) for a, e in part])
    lens = lambda part: [e - a for a, e in part]
    sel = lambda x, part: x[idx(part)]
    ia, ib = pieces
    cua, cub = inputs.cu_from_lengths(lens(ia)), inputs.cu_from_lengths(lens(ib))
    oa, sa, ca = _fused(cua, sel(xq, ia), sel(xk, ia), sel(xv, ia), wq, wk, wv, st, sel(g, ia),
                        sel(beta, ia), s0)
    ob, sb, cb = _fused(cub, sel(xq, ib), sel(xk, ib), sel(xv, ib), wq, wk, wv, ca, sel(g, ib),
                        sel(beta, ib), sa)
    o2 = torch.empty_like(o1)
    o2[idx(ia)] = oa
    o2[idx(ib)] = ob
    check_o(o2, o_ref, "segmented o")
    check_state(sb, s_ref, "segmented state")
    assert torch.equal(cb, c1)


def test_fused_front_end_layer_shape_matches_separate_calls():
    """The 4096-token layer of the benchmark's head shape: the fused call
    against the separate front end then prefill (pool kernel), and against
    the oracle chain."""
    T, Hqk, Hv = 4096, 16, 48
    xq, xk, xv, wq, wk, wv, _ = make(T, Hqk, Hv, seed=8600)
    gen = torch.Generator().manual_seed(8601)
    g = -inputs.G_SCALE_097 * torch.nn.functional.softplus(torch.randn(T, Hv, generator=gen))
    beta = torch.sigmoid(torch.randn(T, Hv, generator=gen))
    o, sT, _ = _fused(None, xq, xk, xv, wq, wk, wv, None, g, beta, None)
    q, k, v = run(xq, xk, xv, wq, wk, wv, None, None, out_state=False)
    o2, s2 = gdn.gdn_prefill(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), beta.to(DEV), kernel="pool")
    torch.cuda.synchronize()
    check_o(o, o2.cpu().double(), "fused vs separate o")
    check_state(sT, s2.cpu().double(), "fused vs separate state")
    o_ref, s_ref, _ = _oracle_chain(None, xq, xk, xv, wq, wk, wv, None, g, beta, None)
    check_o(o, o_ref)
    check_state(sT, s_ref)


def test_fused_front_end_rejects_small_workspace_and_fp32():
    """gdn_prefill_conv validates before launching: a workspace one byte short
    of gdn_prefill_conv_workspace_bytes, and fp32 inputs (the pool kernel is
    bf16 only), are errors and leave the output untouched."""
    args = _fused_inputs([200], 2, 6, 8700, False)
    cu, xq, xk, xv, wq, wk, wv, st, g, beta, s0 = args
    T = xq.shape[0]
    t = lambda x: x.to(DEV).contiguous()
    need = gdn.gdn_prefill_conv_workspace_bytes(1, T, 2, 6, 128, 128)
    assert need > 0
    ws = torch.empty(need - 1, dtype=torch.uint8, device=DEV)
    o = torch.full((T, 6, 128), 3.0, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_prefill_conv(t(xq), t(xk), t(xv), t(wq), t(wk), t(wv), t(g), t(beta), o=o,
                             workspace=ws)
    assert e.value.code == 1
    with pytest.raises(gdn.GdnError) as e:
        gdn.gdn_prefill_conv(t(xq).float(), t(xk).float(), t(xv).float(), t(wq), t(wk), t(wv),
                             t(g), t(beta))
    assert e.value.code == 2
    torch.cuda.synchronize()
    assert bool((o == 3.0).all())
