"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

None of these re-types the oracle's formula: each checks a property that a
plausible mistake in it (a dropped decay, a wrong sign, a transposed state,
recall taken from the wrong state, a mis-indexed head group, a wrong mask)
would break.  Source of the rule: page "Qwen3.8-27B 架构深读: Gated DeltaNet
混合线性注意力与 262K 长上下文", section 三.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import GATE_LINEAR, GATE_LOG, ORDER_ILLUSTRATIVE, ORDER_STANDARD

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed):
    return np.random.default_rng(seed)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def make(seed, T=24, Hqk=2, Hv=4, Dk=8, Dv=6, N=1, s0_std=0.5):
    r = rnd(seed)
    q = unit_rows(r.standard_normal((T, Hqk, Dk)))
    k = unit_rows(r.standard_normal((T, Hqk, Dk)))
    v = r.standard_normal((T, Hv, Dv))
    g = -np.log1p(np.exp(r.standard_normal((T, Hv))))
    beta = 1 / (1 + np.exp(-r.standard_normal((T, Hv))))
    s0 = s0_std * r.standard_normal((N, Hv, Dv, Dk)) if s0_std else None
    return q, k, v, g, beta, s0


def fro(x):
    return float(np.sqrt(np.sum(x * x)))


# ---------------------------------------------------------------- golden ---

def load_worked():
    toks, illus = [], None
    with open(os.path.join(GOLDEN, "worked_2x2.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, state, out = (p.split() for p in line.split("|"))
            if head[0] == "token":
                vals = [float(x) for x in head[2:]]
                toks.append((vals, [float(x) for x in state], [float(x) for x in out]))
            else:
                illus = ([float(x) for x in state], [float(x) for x in out])
    return toks, illus


@pytest.mark.parametrize("gate_kind", [GATE_LINEAR, GATE_LOG])
def test_golden_worked_example(gate_kind):
    toks, illus = load_worked()
    T = len(toks)
    a = np.array([t[0][0] for t in toks])
    b = np.array([t[0][1] for t in toks])
    k = np.array([t[0][2:4] for t in toks]).reshape(T, 1, 2)
    v = np.array([t[0][4:6] for t in toks]).reshape(T, 1, 2)
    q = np.array([t[0][6:8] for t in toks]).reshape(T, 1, 2)
    gate = a if gate_kind == GATE_LINEAR else np.log(a)
    tol = 1e-15 if gate_kind == GATE_LINEAR else 1e-14
    # step by step, carrying the state, so every intermediate state is checked
    s = None
    for t in range(T):
        sl = slice(t, t + 1)
        o, s = oracle.recurrent(q[sl], k[sl], v[sl], gate[sl].reshape(1, 1), b[sl].reshape(1, 1),
                                s, gate_kind=gate_kind)
        np.testing.assert_allclose(s.reshape(4), toks[t][1], rtol=0, atol=tol)
        np.testing.assert_allclose(o.reshape(2), toks[t][2], rtol=0, atol=tol)
    # the page's illustrative order differs only at token 4
    s = None
    for t in range(T):
        sl = slice(t, t + 1)
        o, s = oracle.recurrent(q[sl], k[sl], v[sl], gate[sl].reshape(1, 1), b[sl].reshape(1, 1),
                                s, gate_kind=gate_kind, order=ORDER_ILLUSTRATIVE)
        want_s = toks[t][1] if t < 3 else illus[0]
        want_o = toks[t][2] if t < 3 else illus[1]
        np.testing.assert_allclose(s.reshape(4), want_s, rtol=0, atol=tol)
        np.testing.assert_allclose(o.reshape(2), want_o, rtol=0, atol=tol)
    # and the chunked form reaches the same sequence of outputs
    if gate_kind == GATE_LOG:
        for C in (1, 2, 3, 4):
            o, s = oracle.chunked(q, k, v, gate.reshape(T, 1), b.reshape(T, 1), chunk=C)
            np.testing.assert_allclose(o.reshape(T, 2), [t[2] for t in toks], atol=1e-14)
            np.testing.assert_allclose(s.reshape(4), toks[-1][1], atol=1e-14)


def test_accounting_pins_workload_shapes():
    vals = {}
    with open(os.path.join(GOLDEN, "accounting.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, val = line.split()
                vals[name] = int(val)
    from gated_deltanet_04_b200.inputs import WORKLOADS
    wl = WORKLOADS["long256k"]
    # 48 layers of fp32 state per sequence == about 144 MiB (exactly, with these heads)
    assert 48 * wl.Hv * wl.Dv * wl.Dk * 4 == vals["gdn_state_48_layers_fp32"] == 144 * 2**20
    assert 16 * wl.T * 2 * 4 * 256 * 2 == vals["attention_kv_16_layers_262144"] == 16 * 2**30
    d = WORKLOADS["decode256"]
    assert d.N * d.Hv * d.Dv * d.Dk * 4 == vals["decode_state_per_layer_256_seqs"]
    assert d.layers == 48 and wl.Hv // wl.Hqk == 3


# ----------------------------------------------------------- invariants ---

def test_P1_identity_step_keeps_state():
    """a = 1, b = 0: S unchanged (bitwise) and o_t = S0 q_t."""
    q, k, v, g, beta, s0 = make(1)
    g[:] = 0.0
    beta[:] = 0.0
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    assert np.array_equal(sT, s0)
    G = 2
    for h in range(4):
        want = np.einsum("ed,td->te", s0[0, h], q[:, h // G])
        np.testing.assert_allclose(o[:, h], want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("a_val", [1.0, 0.7, 0.05])
def test_P2_erase_then_write_unit_key(a_val):
    """|k| = 1 exactly and b = 1: after the step, S_t k_t = v_t (erase-then-write)."""
    r = rnd(2)
    Dk, Dv = 16, 5
    k = (r.integers(0, 2, (1, 1, Dk)) * 2 - 1) / 4.0  # entries +-1/4 -> |k|^2 = 1 exactly
    q = unit_rows(r.standard_normal((1, 1, Dk)))
    v = r.standard_normal((1, 1, Dv))
    s0 = r.standard_normal((1, 1, Dv, Dk))
    _, s1 = oracle.recurrent(q, k, v, np.full((1, 1), a_val), np.ones((1, 1)), s0,
                             gate_kind=GATE_LINEAR)
    np.testing.assert_allclose(s1[0, 0] @ k[0, 0], v[0, 0], rtol=0, atol=1e-14)
    # basis key: only column j is rewritten, the rest only decays
    e = np.zeros((1, 1, Dk)); e[0, 0, 3] = 1.0
    _, s2 = oracle.recurrent(q, e, v, np.full((1, 1), a_val), np.ones((1, 1)), s0,
                             gate_kind=GATE_LINEAR)
    np.testing.assert_allclose(s2[0, 0][:, 3], v[0, 0], rtol=0, atol=1e-15)
    others = [d for d in range(Dk) if d != 3]
    assert np.array_equal(s2[0, 0][:, others], a_val * s0[0, 0][:, others])


def test_P3_zero_decay_erases_history():
    """a = 0: S_t = b_t v_t k_t^T and o_t = b_t (k_t . q_t) v_t, whatever came before."""
    q, k, v, g, beta, s0 = make(3, T=5)
    a = np.full_like(g, 0.0)
    o, sT = oracle.recurrent(q, k, v, a, beta, s0, gate_kind=GATE_LINEAR)
    for h in range(4):
        kt, qt = k[-1, h // 2], q[-1, h // 2]
        np.testing.assert_allclose(sT[0, h], beta[-1, h] * np.outer(v[-1, h], kt), atol=1e-15)
        for t in range(5):
            want = beta[t, h] * np.dot(k[t, h // 2], q[t, h // 2]) * v[t, h]
            np.testing.assert_allclose(o[t, h], want, atol=1e-14)


def test_P4_linear_in_v_and_state():
    """At fixed k, b, g the map (S0, V) -> (O, S_T) is linear: superposition holds."""
    q, k, v, g, beta, s0 = make(4)
    o_full, s_full = oracle.recurrent(q, k, v, g, beta, s0)
    o_s0, s_s0 = oracle.recurrent(q, k, np.zeros_like(v), g, beta, s0)
    o_v, s_v = oracle.recurrent(q, k, v, g, beta, None)
    np.testing.assert_allclose(o_full, o_s0 + o_v, atol=1e-12)
    np.testing.assert_allclose(s_full, s_s0 + s_v, atol=1e-12)
    o_2v, s_2v = oracle.recurrent(q, k, 2.5 * v, g, beta, None)
    np.testing.assert_allclose(o_2v, 2.5 * o_v, atol=1e-12)
    np.testing.assert_allclose(s_2v, 2.5 * s_v, atol=1e-12)


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_P5_chunked_equals_recurrent(C):
    q, k, v, g, beta, s0 = make(5, T=150, Dk=16, Dv=16)
    o1, s1 = oracle.recurrent(q, k, v, g, beta, s0)
    o2, s2 = oracle.chunked(q, k, v, g, beta, s0, chunk=C)
    scale = max(1.0, np.abs(o1).max())
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(s2, s1, rtol=0, atol=1e-12)


def test_P5_chunked_equals_recurrent_tiny_workload():
    from gated_deltanet_04_b200.inputs import make_prefill
    inp = make_prefill("tiny")
    o1, s1 = oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"])
    o2, s2 = oracle.chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], chunk=16)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(s2, s1, atol=1e-12)


def test_P6_split_and_carry_is_bitwise_and_packing_is_independent():
    q, k, v, g, beta, s0 = make(6, T=40)
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    for p in (1, 7, 16, 39):
        oa, sa = oracle.recurrent(q[:p], k[:p], v[:p], g[:p], beta[:p], s0)
        ob, sb = oracle.recurrent(q[p:], k[p:], v[p:], g[p:], beta[p:], sa)
        assert np.array_equal(np.concatenate([oa, ob]), o)
        assert np.array_equal(sb, sT)
    # three sequences packed with cu_seqlens == three separate runs
    cu = np.array([0, 9, 9, 40])
    s03 = np.concatenate([s0, 0.3 * s0, -s0])
    op, sp = oracle.recurrent(q, k, v, g, beta, s03, cu)
    for n in range(3):
        a, b = cu[n], cu[n + 1]
        on, sn = oracle.recurrent(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], s03[n:n + 1])
        assert np.array_equal(op[a:b], on)
        assert np.array_equal(sp[n], sn[0])
    assert np.array_equal(sp[1], s03[1])  # an empty sequence leaves its state alone


def orthonormal_keys(seed, T, Dk):
    r = rnd(seed)
    Qm, _ = np.linalg.qr(r.standard_normal((Dk, Dk)))
    return Qm[:T]  # rows orthonormal


def test_P7_linear_attention_closed_form():
    """Orthonormal keys, a = b = 1, S0 = 0: S_T = sum_i v_i k_i^T (linear attention)."""
    T, Dk, Dv = 10, 12, 7
    kk = orthonormal_keys(7, T, Dk)
    r = rnd(70)
    v = r.standard_normal((T, 1, Dv))
    q = unit_rows(r.standard_normal((T, 1, Dk)))
    o, sT = oracle.recurrent(q, kk.reshape(T, 1, Dk), v, np.zeros((T, 1)), np.ones((T, 1)))
    np.testing.assert_allclose(sT[0, 0], v[:, 0].T @ kk, atol=1e-13)
    for t in range(T):
        np.testing.assert_allclose(o[t, 0], (v[: t + 1, 0].T @ kk[: t + 1]) @ q[t, 0], atol=1e-13)


def test_P8_orthogonal_keys_brute_force_decay_mask():
    """Orthonormal keys, general a, b, S0 = 0:
    o_t = sum_{i<=t} (Gamma_t / Gamma_i) b_i (k_i . q_t) v_i   (O(T^2) brute force)."""
    T, Dk, Dv = 16, 16, 5
    kk = orthonormal_keys(8, T, Dk)
    r = rnd(80)
    v = r.standard_normal((T, 1, Dv))
    q = r.standard_normal((T, 1, Dk))
    g = -r.uniform(0.0, 1.5, (T, 1))
    b = r.uniform(0.0, 1.0, (T, 1))
    o, sT = oracle.recurrent(q, kk.reshape(T, 1, Dk), v, g, b)
    gam = np.cumsum(g[:, 0])
    for t in range(T):
        want = np.zeros(Dv)
        for i in range(t + 1):
            want += math.exp(gam[t] - gam[i]) * b[i, 0] * np.dot(kk[i], q[t, 0]) * v[i, 0]
        np.testing.assert_allclose(o[t, 0], want, atol=1e-13)
    want_S = sum(math.exp(gam[-1] - gam[i]) * b[i, 0] * np.outer(v[i, 0], kk[i]) for i in range(T))
    np.testing.assert_allclose(sT[0, 0], want_S, atol=1e-13)


def test_P9_repeated_key_overwrites():
    """A key written twice with b = 1 recalls only the latest value (any decay)."""
    T, Dk, Dv = 6, 8, 3
    r = rnd(9)
    key = unit_rows(r.standard_normal(Dk))
    k = np.tile(key, (T, 1)).reshape(T, 1, Dk)
    v = r.standard_normal((T, 1, Dv))
    q = np.tile(key, (T, 1)).reshape(T, 1, Dk)
    g = -r.uniform(0, 1, (T, 1))
    o, sT = oracle.recurrent(q, k, v, g, np.ones((T, 1)), r.standard_normal((1, 1, Dv, Dk)))
    # querying with the key itself returns exactly the latest value
    np.testing.assert_allclose(o[:, 0], v[:, 0], atol=1e-13)
    np.testing.assert_allclose(sT[0, 0] @ key, v[-1, 0], atol=1e-13)


def test_P10_householder_norm():
    """b = 2, |k| = 1, v = 0: S (I - 2 k k^T) is a reflection, |S|_F is kept;
    with decay, |S_t|_F = Gamma_t |S_0|_F."""
    T, Dk, Dv = 12, 8, 5
    q, k, v, g, beta, s0 = make(10, T=T, Hqk=1, Hv=1, Dk=Dk, Dv=Dv)
    v[:] = 0.0
    beta[:] = 2.0
    _, sT = oracle.recurrent(q, k, v, np.zeros_like(g), beta, s0)
    assert abs(fro(sT) - fro(s0)) < 1e-12 * fro(s0)
    _, sT = oracle.recurrent(q, k, v, g, beta, s0)
    assert abs(fro(sT) - math.exp(g.sum()) * fro(s0)) < 1e-12 * fro(s0)


def test_P11_contractive_when_v_zero():
    T = 20
    q, k, v, g, beta, s0 = make(11, T=T, Hqk=1, Hv=1)
    v[:] = 0.0
    s = s0
    prev = fro(s)
    for t in range(T):
        sl = slice(t, t + 1)
        _, s = oracle.recurrent(q[sl], k[sl], v[sl], g[sl], beta[sl], s)
        cur = fro(s)
        assert cur <= prev * (1 + 1e-15)
        assert cur <= math.exp(g[t, 0]) * prev * (1 + 1e-15)
        prev = cur


def test_P13_illustrative_order_difference():
    """illustrative - standard = -b (1 - a) (S_{t-1} k) k^T for one step; equal when a = 1 or b = 0."""
    q, k, v, g, beta, s0 = make(13, T=1, Hqk=1, Hv=1)
    _, s_std = oracle.recurrent(q, k, v, g, beta, s0)
    _, s_ill = oracle.recurrent(q, k, v, g, beta, s0, order=ORDER_ILLUSTRATIVE)
    a, b = math.exp(g[0, 0]), beta[0, 0]
    kt = k[0, 0]
    diff = -b * (1 - a) * np.outer(s0[0, 0] @ kt, kt)
    np.testing.assert_allclose(s_ill - s_std, diff.reshape(s_std.shape), atol=1e-14)
    _, s_std = oracle.recurrent(q, k, v, np.zeros_like(g), beta, s0)
    _, s_ill = oracle.recurrent(q, k, v, np.zeros_like(g), beta, s0, order=ORDER_ILLUSTRATIVE)
    assert np.array_equal(s_std, s_ill)


def test_head_grouping_is_contiguous():
    """v-heads h and h' read the same q/k head iff h // G == h' // G."""
    q, k, v, g, beta, s0 = make(14, Hqk=2, Hv=4)
    v[:, 1] = v[:, 0]; g[:, 1] = g[:, 0]; beta[:, 1] = beta[:, 0]; s0[:, 1] = s0[:, 0]
    v[:, 2] = v[:, 0]; g[:, 2] = g[:, 0]; beta[:, 2] = beta[:, 0]; s0[:, 2] = s0[:, 0]
    o, sT = oracle.recurrent(q, k, v, g, beta, s0)
    assert np.array_equal(o[:, 0], o[:, 1])            # same group -> identical
    assert not np.allclose(o[:, 0], o[:, 2])           # other group -> different keys


def test_state_orientation_recall():
    """The state maps keys to values: after one write from S0 = 0 with b = 1,
    S k = v, i.e. S is Dv x Dk (not its transpose)."""
    Dk, Dv = 6, 3
    r = rnd(15)
    k = unit_rows(r.standard_normal((1, 1, Dk)))
    v = r.standard_normal((1, 1, Dv))
    _, s = oracle.recurrent(k, k, v, np.zeros((1, 1)), np.ones((1, 1)))
    assert s.shape == (1, 1, Dv, Dk)
    np.testing.assert_allclose(s[0, 0] @ k[0, 0], v[0, 0], atol=1e-15)


def test_decode_step_is_length_one_recurrence():
    r = rnd(16)
    N, Hqk, Hv, D = 5, 2, 4, 8
    q = unit_rows(r.standard_normal((N, Hqk, D)))
    k = unit_rows(r.standard_normal((N, Hqk, D)))
    v = r.standard_normal((N, Hv, D))
    g = -r.uniform(0, 1, (N, Hv))
    b = r.uniform(0, 1, (N, Hv))
    S = r.standard_normal((N, Hv, D, D))
    o, S1 = oracle.decode_step(q, k, v, g, b, S)
    for n in range(N):
        on, sn = oracle.recurrent(q[n:n + 1], k[n:n + 1], v[n:n + 1], g[n:n + 1], b[n:n + 1],
                                  S[n:n + 1])
        assert np.array_equal(o[n], on[0]) and np.array_equal(S1[n], sn[0])


def test_bad_seqlens_rejected():
    q, k, v, g, beta, s0 = make(17, T=8)
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, g, beta, None, np.array([0, 5, 3, 8]))
    with pytest.raises(ValueError):
        oracle.recurrent(q, k, v, g, beta, None, np.array([0, 9]))


# ---- bfloat16 state storage for decode ----------------------------------------

def test_round_bf16_agrees_with_torch_on_fp32_values():
    """torch rounds fp32 -> bfloat16 to nearest, ties to even; on values that are
    exactly fp32 the oracle's one-step rounding from fp64 must agree bit for bit
    (random normals, powers of two, and values right at rounding boundaries)."""
    import torch
    r = rnd(21)
    x = r.standard_normal(200000).astype(np.float32)
    ulp = np.float32(2.0 ** -7)
    edges = (np.float32(1.0) + np.arange(-64, 64, dtype=np.float32) * ulp / 2).astype(np.float32)
    x = np.concatenate([x, edges, -edges, np.float32(2.0) ** np.arange(-60, 60, dtype=np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64)), want)


def test_round_bf16_ties_to_even_and_error_bound():
    one = 1.0
    # halfway between 1 and 1 + 2^-7 -> 1 (even); between 1 + 2^-7 and 1 + 2^-6 -> 1 + 2^-6
    assert oracle.round_bf16(np.array([one + 2.0 ** -8]))[0] == one
    assert oracle.round_bf16(np.array([one + 3 * 2.0 ** -8]))[0] == one + 2.0 ** -6
    assert oracle.round_bf16(np.array([one + 2.0 ** -8 + 2.0 ** -40]))[0] == one + 2.0 ** -7
    x = rnd(22).standard_normal(100000) * 10.0 ** rnd(23).uniform(-20, 20, 100000)
    y = oracle.round_bf16(x)
    _, e = np.frexp(x)                                           # x = m 2^e, 0.5 <= |m| < 1
    assert np.all(np.abs(y - x) <= np.ldexp(1.0, e - 9))          # half an ulp (ulp = 2^(e-8))
    assert np.array_equal(oracle.round_bf16(y), y)                # idempotent
    with pytest.raises(ValueError):
        oracle.round_bf16(np.array([1e-39]))


def test_decode_bf16_state_identity_step_keeps_bf16_state():
    """a = 1, b = 0 leaves the state unchanged, so a bfloat16 state comes back
    bit-identical and o = S q (P1 through the bfloat16 storage)."""
    r = rnd(24)
    N, Hqk, Hv, D = 3, 2, 4, 8
    q = unit_rows(r.standard_normal((N, Hqk, D)))
    k = unit_rows(r.standard_normal((N, Hqk, D)))
    v = r.standard_normal((N, Hv, D))
    S = oracle.round_bf16(r.standard_normal((N, Hv, D, D)))
    o, s_new, s_bf16 = oracle.decode_step_bf16_state(q, k, v, np.zeros((N, Hv)), np.zeros((N, Hv)), S)
    assert np.array_equal(s_bf16, S) and np.array_equal(s_new, S)
    heads = np.arange(Hv) // (Hv // Hqk)
    assert np.allclose(o, np.einsum("nhij,nhj->nhi", S, q[:, heads]), rtol=1e-13, atol=1e-13)
    with pytest.raises(ValueError):
        oracle.decode_step_bf16_state(q, k, v, np.zeros((N, Hv)), np.zeros((N, Hv)), S + 2.0 ** -20)


# ---- decode over a pool of state slots -----------------------------------------

def _slots_case(seed, N=5, S=9, Hqk=2, Hv=4, D=8):
    r = rnd(seed)
    q = unit_rows(r.standard_normal((N, Hqk, D)))
    k = unit_rows(r.standard_normal((N, Hqk, D)))
    v = r.standard_normal((N, Hv, D))
    g = -r.uniform(0, 1, (N, Hv))
    b = r.uniform(0, 1, (N, Hv))
    pool = r.standard_normal((S, Hv, D, D))
    return q, k, v, g, b, pool


def test_slots_identity_mapping_is_decode_step():
    q, k, v, g, b, pool = _slots_case(31, N=5, S=5)
    o, new = oracle.decode_step_slots(q, k, v, g, b, pool, np.arange(5))
    o_ref, s_ref = oracle.decode_step(q, k, v, g, b, pool)
    assert np.array_equal(o, o_ref) and np.array_equal(new, s_ref)


def test_slots_gather_scatter_and_untouched_slots():
    """Entries read and write only their own slots, in any order; slots nobody
    names come back bit for bit; permuting the batch permutes only o."""
    q, k, v, g, b, pool = _slots_case(32)
    idx = np.array([7, 2, 5, 0, 3])
    o, new = oracle.decode_step_slots(q, k, v, g, b, pool, idx)
    o_ref, s_ref = oracle.decode_step(q, k, v, g, b, pool[idx])
    assert np.array_equal(o, o_ref) and np.array_equal(new[idx], s_ref)
    untouched = np.setdiff1d(np.arange(pool.shape[0]), idx)
    assert np.array_equal(new[untouched], pool[untouched])
    perm = np.array([3, 0, 4, 1, 2])
    o_p, new_p = oracle.decode_step_slots(q[perm], k[perm], v[perm], g[perm], b[perm], pool, idx[perm])
    assert np.array_equal(o_p, o[perm]) and np.array_equal(new_p, new)


def test_slots_reset_starts_from_zero():
    """A reset entry ignores its slot: with S = 0 the step is S' = b v k^T and
    o = b (k . q) v (the rule from a zero state)."""
    q, k, v, g, b, pool = _slots_case(33)
    idx = np.array([4, 1, 8, 6, 0])
    reset = np.array([0, 1, 0, 1, 0])
    o, new = oracle.decode_step_slots(q, k, v, g, b, pool, idx, reset)
    heads = np.arange(v.shape[1]) // (v.shape[1] // q.shape[1])
    for n in np.nonzero(reset)[0]:
        kk, qq = k[n, heads], q[n, heads]                       # [Hv, D]
        want_s = b[n][:, None, None] * v[n][:, :, None] * kk[:, None, :]
        assert np.allclose(new[idx[n]], want_s, rtol=1e-13, atol=1e-14)
        want_o = (b[n] * np.sum(kk * qq, axis=1))[:, None] * v[n]
        assert np.allclose(o[n], want_o, rtol=1e-12, atol=1e-13)
    keep = np.nonzero(reset == 0)[0]
    o_k, new_k = oracle.decode_step_slots(q[keep], k[keep], v[keep], g[keep], b[keep], pool, idx[keep])
    assert np.array_equal(o[keep], o_k) and np.array_equal(new[idx[keep]], new_k[idx[keep]])


def test_slots_reject_bad_indices():
    q, k, v, g, b, pool = _slots_case(34)
    for bad in ([0, 1, 2, 3, 9], [0, 1, 2, 3, -1], [0, 1, 2, 2, 4]):
        with pytest.raises(ValueError):
            oracle.decode_step_slots(q, k, v, g, b, pool, np.array(bad))


# ---- prefill over a pool of state slots ----------------------------------------

def _pslots_case(seed, lengths=(3, 1, 5), S=7, Hqk=2, Hv=4, D=8):
    r = rnd(seed)
    T = sum(lengths)
    q = unit_rows(r.standard_normal((T, Hqk, D)))
    k = unit_rows(r.standard_normal((T, Hqk, D)))
    v = r.standard_normal((T, Hv, D))
    g = -r.uniform(0, 1, (T, Hv))
    b = r.uniform(0, 1, (T, Hv))
    pool = r.standard_normal((S, Hv, D, D))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    return q, k, v, g, b, pool, cu


def test_prefill_slots_identity_mapping_is_recurrent():
    q, k, v, g, b, pool, cu = _pslots_case(41, S=3)
    o, new = oracle.prefill_slots(q, k, v, g, b, pool, np.arange(3), cu_seqlens=cu)
    o_ref, s_ref = oracle.recurrent(q, k, v, g, b, pool, cu)
    assert np.array_equal(o, o_ref) and np.array_equal(new, s_ref)


def test_prefill_slots_gather_scatter_untouched_and_permuted():
    """Sequences read and write only their own slots; slots nobody names come
    back bit for bit; reordering the packed sequences (tokens and slot list
    together) reorders only o."""
    lengths = (3, 1, 5)
    q, k, v, g, b, pool, cu = _pslots_case(42, lengths)
    idx = np.array([5, 1, 3])
    o, new = oracle.prefill_slots(q, k, v, g, b, pool, idx, cu_seqlens=cu)
    o_ref, s_ref = oracle.recurrent(q, k, v, g, b, pool[idx], cu)
    assert np.array_equal(o, o_ref) and np.array_equal(new[idx], s_ref)
    untouched = np.setdiff1d(np.arange(pool.shape[0]), idx)
    assert np.array_equal(new[untouched], pool[untouched])
    perm = [2, 0, 1]
    tok = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in perm])
    cu_p = np.concatenate([[0], np.cumsum([lengths[n] for n in perm])]).astype(np.int64)
    o_p, new_p = oracle.prefill_slots(q[tok], k[tok], v[tok], g[tok], b[tok], pool, idx[perm],
                                      cu_seqlens=cu_p)
    assert np.array_equal(o_p, o[tok]) and np.array_equal(new_p, new)


def test_prefill_slots_reset_starts_from_zero():
    """A reset sequence ignores its slot: one token from S = 0 gives
    S' = b v k^T and o = b (k . q) v; a longer reset sequence equals the same
    sequence started from a slot that holds zeros."""
    lengths = (1, 4, 2)
    q, k, v, g, b, pool, cu = _pslots_case(43, lengths)
    idx = np.array([6, 2, 0])
    reset = np.array([1, 1, 0])
    o, new = oracle.prefill_slots(q, k, v, g, b, pool, idx, reset, cu)
    heads = np.arange(v.shape[1]) // (v.shape[1] // q.shape[1])
    kk, qq = k[0, heads], q[0, heads]
    want_s = b[0][:, None, None] * v[0][:, :, None] * kk[:, None, :]
    assert np.allclose(new[6], want_s, rtol=1e-13, atol=1e-14)
    want_o = (b[0] * np.sum(kk * qq, axis=1))[:, None] * v[0]
    assert np.allclose(o[0], want_o, rtol=1e-12, atol=1e-13)
    zeroed = pool.copy()
    zeroed[[6, 2]] = 0.0
    o_z, new_z = oracle.prefill_slots(q, k, v, g, b, zeroed, idx, None, cu)
    assert np.array_equal(o, o_z) and np.array_equal(new[idx], new_z[idx])


def test_prefill_slots_reject_bad_indices():
    q, k, v, g, b, pool, cu = _pslots_case(44)
    for bad in ([0, 1, 7], [0, -1, 2], [3, 3, 4]):
        with pytest.raises(ValueError):
            oracle.prefill_slots(q, k, v, g, b, pool, np.array(bad), cu_seqlens=cu)


# ---- front end: kernel-4 causal short convolution and per-head L2 norm ---------

def test_short_conv_taps_are_delays():
    """A filter with a single 1 in tap j delays the input by 3 - j tokens, with
    zeros (no conv state) before each sequence start."""
    r = rnd(41)
    T, C = 11, 5
    x = r.standard_normal((T, C))
    cu = np.array([0, 4, 4, 11])              # an empty sequence in the middle
    for j in range(4):
        w = np.zeros((C, 4))
        w[:, j] = 1.0
        y, _ = oracle.short_conv(x, w, cu)
        d = 3 - j
        for a, b in ((0, 4), (4, 11)):
            for t in range(a, b):
                want = x[t - d] if t - d >= a else np.zeros(C)
                assert np.array_equal(y[t], want)


def test_short_conv_carry_equals_one_shot():
    """Splitting a sequence anywhere and passing the conv state gives the
    one-shot result, for every split point (including shorter than 3)."""
    r = rnd(42)
    T, C = 13, 4
    x = r.standard_normal((T, C))
    w = r.standard_normal((C, 4))
    y_all, s_all = oracle.short_conv(x, w)
    for cut in range(0, T + 1):
        y1, s1 = oracle.short_conv(x[:cut], w)
        y2, s2 = oracle.short_conv(x[cut:], w, conv_state=s1)
        assert np.allclose(np.concatenate([y1, y2]), y_all, rtol=0, atol=1e-14)
        assert np.array_equal(s2, s_all)


def test_short_conv_is_linear_and_brute_force():
    r = rnd(43)
    T, C = 9, 3
    x, x2 = r.standard_normal((T, C)), r.standard_normal((T, C))
    w = r.standard_normal((C, 4))
    s0 = r.standard_normal((1, 3, C))
    y, _ = oracle.short_conv(x, w, conv_state=s0)
    ext = np.concatenate([s0[0], x])
    brute = np.array([[sum(w[c, j] * ext[t + j, c] for j in range(4)) for c in range(C)]
                      for t in range(T)])
    assert np.allclose(y, brute, rtol=1e-14, atol=1e-14)
    ya, _ = oracle.short_conv(x + 2.0 * x2, w)
    yb, _ = oracle.short_conv(x, w)
    yc, _ = oracle.short_conv(x2, w)
    assert np.allclose(ya, yb + 2.0 * yc, rtol=1e-13, atol=1e-13)


def test_short_conv_norm_heads_are_unit_and_v_is_not_normalised():
    r = rnd(44)
    T, Hqk, Hv, D = 7, 2, 4, 8
    xq, xk = r.standard_normal((T, Hqk, D)), r.standard_normal((T, Hqk, D))
    xv = r.standard_normal((T, Hv, D))
    wq, wk, wv = (r.standard_normal((Hqk * D, 4)), r.standard_normal((Hqk * D, 4)),
                  r.standard_normal((Hv * D, 4)))
    q, k, v, st = oracle.short_conv_norm(xq, xk, xv, wq, wk, wv)
    assert np.allclose(np.linalg.norm(q, axis=-1), 1.0, rtol=1e-14)
    assert np.allclose(np.linalg.norm(k, axis=-1), 1.0, rtol=1e-14)
    yv, _ = oracle.short_conv(xv.reshape(T, -1), wv)
    assert np.array_equal(v, yv.reshape(T, Hv, D))
    yq, _ = oracle.short_conv(xq.reshape(T, -1), wq)
    yq = yq.reshape(T, Hqk, D)
    assert np.allclose(q * np.linalg.norm(yq, axis=-1, keepdims=True), yq, rtol=1e-13, atol=1e-14)
    assert st.shape == (1, 3, 2 * Hqk * D + Hv * D)
    assert np.array_equal(st[0, :, :Hqk * D], xq[-3:].reshape(3, -1))
    assert np.array_equal(st[0, :, 2 * Hqk * D:], xv[-3:].reshape(3, -1))


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunked_recall_first_equals_recurrent(C):
    """The chunked form in the recall-first order (Gamma_{r-1} in A and W)
    reaches the recall-first recurrence, with an entering state, packed
    sequences and decays from weak to strong; and differs from the standard
    order."""
    q, k, v, g, beta, s0 = make(51, T=70, N=2, s0_std=0.5)
    cu = np.array([0, 33, 70])
    g = g * 3.0  # stronger decay: the two orders differ more
    o_r, s_r = oracle.recurrent(q, k, v, g, beta, s0, cu, order=ORDER_ILLUSTRATIVE)
    o_c, s_c = oracle.chunked(q, k, v, g, beta, s0, cu, chunk=C, order=ORDER_ILLUSTRATIVE)
    assert np.allclose(o_c, o_r, rtol=1e-10, atol=1e-11)
    assert np.allclose(s_c, s_r, rtol=1e-10, atol=1e-11)
    o_std, _ = oracle.chunked(q, k, v, g, beta, s0, cu, chunk=C)
    assert np.abs(o_std - o_r).max() > 1e-3


# ---- a chunk step as an affine map of the entering state (for a scan) ---------

def test_chunk_state_maps_reproduce_the_recurrence():
    """Applying each chunk's affine map S -> S A_c + B_c in turn gives the
    recurrence's final state, for ragged chunks and an entering state."""
    q, k, v, g, beta, s0 = make(61, T=70, Hqk=1, Hv=2, N=1, s0_std=0.5)
    _, s_ref = oracle.recurrent(q, k, v, g, beta, s0)
    for h in range(2):
        for C in (1, 7, 16, 64):
            S = s0[0, h].copy()
            for A, B in oracle.chunk_state_maps(k, v, g, beta, chunk=C, head_k=0, head_v=h):
                S = S @ A + B
            assert np.allclose(S, s_ref[0, h], rtol=1e-10, atol=1e-11), (h, C)


def test_chunk_state_maps_compose_associatively():
    """Composing the maps pairwise in a tree (as a parallel scan would) equals
    composing them left to right, and equals the one-step map of the whole
    sequence as a single chunk."""
    q, k, v, g, beta, s0 = make(62, T=48, Hqk=1, Hv=1, N=1, s0_std=0.5)
    maps = oracle.chunk_state_maps(k, v, g, beta, chunk=6)
    seq = maps[0]
    for m in maps[1:]:
        seq = oracle.compose_state_maps(seq, m)
    level = maps
    while len(level) > 1:
        level = [oracle.compose_state_maps(level[i], level[i + 1]) if i + 1 < len(level) else level[i]
                 for i in range(0, len(level), 2)]
    whole = oracle.chunk_state_maps(k, v, g, beta, chunk=48)[0]
    for A, B in (level[0], whole):
        assert np.allclose(A, seq[0], rtol=1e-10, atol=1e-11)
        assert np.allclose(B, seq[1], rtol=1e-10, atol=1e-11)
