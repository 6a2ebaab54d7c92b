"""Randomised properties of the oracle (hypothesis), over shapes, packings,
chunk lengths and both step orders: the chunk-parallel form equals the token
recurrence; splitting sequences and carrying the state is bit-identical to one
call; packing sequences together changes nothing; the state-slot prefill is
the recurrence on gathered states.  Small sizes, a bounded number of examples,
CPU only."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from oracle import ORDER_STANDARD

ORDERS = [ORDER_STANDARD, 1]  # standard, recall-first


def _case(seed, lengths, Hqk, G, D, strong):
    r = np.random.default_rng(seed)
    T = int(sum(lengths))
    Hv = Hqk * G

    def unit(x):
        n = np.linalg.norm(x, axis=-1, keepdims=True)
        return x / np.where(n > 0, n, 1.0)

    q = unit(r.standard_normal((T, Hqk, D)))
    k = unit(r.standard_normal((T, Hqk, D)))
    v = r.standard_normal((T, Hv, D))
    g = -r.uniform(0.0, 4.0 if strong else 0.5, (T, Hv))
    b = r.uniform(0.0, 1.0, (T, Hv))
    s0 = 0.5 * r.standard_normal((len(lengths), Hv, D, D))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, g, b, s0, cu


shapes = st.tuples(
    st.integers(0, 2**31 - 1),                              # seed
    st.lists(st.integers(0, 40), min_size=1, max_size=4),   # sequence lengths
    st.sampled_from([1, 2]),                                # Hqk
    st.sampled_from([1, 2, 3]),                             # v-heads per q/k head
    st.sampled_from([4, 8]),                                # D
    st.booleans(),                                          # strong decay
)


@settings(max_examples=40, deadline=None)
@given(shapes, st.sampled_from([1, 3, 8, 16, 64]), st.sampled_from(ORDERS))
def test_chunked_equals_recurrent(shape, C, order):
    q, k, v, g, b, s0, cu = _case(*shape)
    o1, s1 = oracle.recurrent(q, k, v, g, b, s0, cu, order=order)
    o2, s2 = oracle.chunked(q, k, v, g, b, s0, cu, chunk=C, order=order)
    scale = max(1.0, float(np.abs(o1).max()) if o1.size else 1.0)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-11 * scale)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-11 * max(1.0, float(np.abs(s1).max())))


@settings(max_examples=40, deadline=None)
@given(shapes, st.data(), st.sampled_from(ORDERS))
def test_split_and_carry_is_bitwise(shape, data, order):
    q, k, v, g, b, s0, cu = _case(*shape)
    lengths = np.diff(cu)
    o, sT = oracle.recurrent(q, k, v, g, b, s0, cu, order=order)
    for n, L in enumerate(lengths):
        p = data.draw(st.integers(0, int(L)))
        a, e = int(cu[n]), int(cu[n + 1])
        sl = lambda x, lo, hi: x[lo:hi]
        oa, sa = oracle.recurrent(sl(q, a, a + p), sl(k, a, a + p), sl(v, a, a + p),
                                  sl(g, a, a + p), sl(b, a, a + p), s0[n:n + 1], order=order)
        ob, sb = oracle.recurrent(sl(q, a + p, e), sl(k, a + p, e), sl(v, a + p, e),
                                  sl(g, a + p, e), sl(b, a + p, e), sa, order=order)
        assert np.array_equal(np.concatenate([oa, ob]), o[a:e])
        assert np.array_equal(sb[0], sT[n])


@settings(max_examples=25, deadline=None)
@given(shapes, st.randoms(use_true_random=False))
def test_prefill_slots_is_the_recurrence_on_gathered_states(shape, rnd):
    q, k, v, g, b, _, cu = _case(*shape)
    N = len(cu) - 1
    S = N + 3
    pool = np.random.default_rng(shape[0] + 1).standard_normal((S, v.shape[1], v.shape[2],
                                                                 q.shape[2]))
    idx = np.array(rnd.sample(range(S), N))
    reset = np.array([rnd.randint(0, 1) for _ in range(N)])
    o, new = oracle.prefill_slots(q, k, v, g, b, pool, idx, reset, cu)
    start = pool[idx].copy()
    start[reset != 0] = 0.0
    o_ref, s_ref = oracle.recurrent(q, k, v, g, b, start, cu)
    assert np.array_equal(o, o_ref)
    assert np.array_equal(new[idx], s_ref)
    others = np.setdiff1d(np.arange(S), idx)
    assert np.array_equal(new[others], pool[others])
