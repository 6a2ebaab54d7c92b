"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (``libgdn`` and its
binding ``gated_deltanet_04_b200``) never imports, links or calls it, and the
two share no code: the oracle is plain C (``gdn_oracle.c``) compiled with gcc,
driven here through ctypes on numpy float64 arrays.

Method (page "Qwen3.8-27B 架构深读 ...", section 三): the gated delta rule
    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,   o_t = S_t q_t,
with a_t = exp(g_t), b_t = beta_t, plus the page's illustrative step order
(recall S k taken before the decay) as a flagged variant, and an fp64
chunk-parallel form used only to cross-check the recurrence.

Every function is pinned by tests/test_oracle_pins.py (invariants, closed
forms, brute force) and tests/golden/ (hand-worked example).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None

ORDER_STANDARD = 0
ORDER_ILLUSTRATIVE = 1
GATE_LOG = 0
GATE_LINEAR = 1


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (fp64, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            i64p = ctypes.POINTER(ctypes.c_int64)
            i64 = ctypes.c_int64
            lib.gdn_oracle_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, i64p, i64, i64, i64, i64,
                                                 i64, i64, ctypes.c_int, ctypes.c_int,
                                                 ctypes.c_void_p, dp, dp]
            lib.gdn_oracle_recurrent.restype = ctypes.c_int
            lib.gdn_oracle_chunked.argtypes = [dp, dp, dp, dp, dp, dp, i64p, i64, i64, i64, i64,
                                               i64, i64, i64, ctypes.c_int, dp, dp]
            lib.gdn_oracle_chunked.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor -> exact fp64 copy on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a, ctype=ctypes.c_double):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _prep(q, k, v, gate, beta, s0, cu_seqlens):
    q, k, v, gate, beta, s0 = (_f64(x) for x in (q, k, v, gate, beta, s0))
    T, Hqk, Dk = q.shape
    Hv, Dv = v.shape[1], v.shape[2]
    assert k.shape == q.shape and v.shape[0] == T
    assert gate.shape == (T, Hv) and beta.shape == (T, Hv)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        if hasattr(cu_seqlens, "detach"):
            cu_seqlens = cu_seqlens.detach().cpu().numpy()
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    if s0 is not None:
        assert s0.shape == (N, Hv, Dv, Dk)
    return q, k, v, gate, beta, s0, cu, N, T, Hqk, Hv, Dk, Dv


def recurrent(q, k, v, gate, beta, s0=None, cu_seqlens=None, *, order=ORDER_STANDARD,
              gate_kind=GATE_LOG, heads=None, want_o=True):
    """Token-by-token fp64 recurrence.

    Shapes: q,k [T,Hqk,Dk]; v [T,Hv,Dv]; gate,beta [T,Hv]; s0 [N,Hv,Dv,Dk] or None;
    cu_seqlens [N+1] or None (one sequence).  ``gate`` is g (a = exp(g)) for
    GATE_LOG, or a itself for GATE_LINEAR.  ``heads``: optional iterable of
    v-heads to compute (others are left as zeros).
    Returns (o [T,Hv,Dv] or None, final_state [N,Hv,Dv,Dk]) in float64.
    """
    lib = _load()
    q, k, v, gate, beta, s0, cu, N, T, Hqk, Hv, Dk, Dv = _prep(q, k, v, gate, beta, s0, cu_seqlens)
    o = np.zeros((T, Hv, Dv), dtype=np.float64) if want_o else None
    sT = np.zeros((N, Hv, Dv, Dk), dtype=np.float64)
    mask = None
    if heads is not None:
        m = np.zeros(Hv, dtype=np.uint8)
        m[list(heads)] = 1
        mask = m
    rc = lib.gdn_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(s0),
                                  _ptr(cu, ctypes.c_int64), N, T, Hqk, Hv, Dk, Dv, order,
                                  gate_kind, None if mask is None else mask.ctypes.data,
                                  _ptr(o), _ptr(sT))
    if rc != 0:
        raise ValueError(f"gdn_oracle_recurrent failed with code {rc}")
    return o, sT


def chunked(q, k, v, g, beta, s0=None, cu_seqlens=None, *, chunk=64, order=ORDER_STANDARD):
    """fp64 chunk-parallel form (log gate), in either step order: the
    recall-first order moves token r's recall decay from Gamma_r to
    Gamma_{r-1} in A and W.  Same shapes as recurrent()."""
    lib = _load()
    q, k, v, g, beta, s0, cu, N, T, Hqk, Hv, Dk, Dv = _prep(q, k, v, g, beta, s0, cu_seqlens)
    o = np.zeros((T, Hv, Dv), dtype=np.float64)
    sT = np.zeros((N, Hv, Dv, Dk), dtype=np.float64)
    rc = lib.gdn_oracle_chunked(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
                                _ptr(cu, ctypes.c_int64), N, T, Hqk, Hv, Dk, Dv, int(chunk),
                                int(order), _ptr(o), _ptr(sT))
    if rc != 0:
        raise ValueError(f"gdn_oracle_chunked failed with code {rc}")
    return o, sT


def decode_step(q, k, v, g, beta, state, *, order=ORDER_STANDARD):
    """One-token update of N independent sequences: q,k [N,Hqk,Dk], v [N,Hv,Dv],
    g,beta [N,Hv], state [N,Hv,Dv,Dk].  Returns (o [N,Hv,Dv], new_state).
    This is the recurrence with every sequence of length one."""
    N = q.shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return recurrent(q, k, v, g, beta, state, cu, order=order)


def round_bf16(x):
    """Round float64 values to the nearest bfloat16, ties to even, in one step.

    bfloat16 is the upper half of an IEEE-754 binary32 (sign, 8 exponent bits,
    7 stored fraction bits): 8 significant bits.  With x = m 2^e, 0.5 <= |m| < 1
    (frexp), the nearest such value is rint(m 2^8) 2^(e-8), rint rounding
    halfway cases to the even integer.  Normal range only: a nonzero |x| below
    2^-126 (bfloat16 subnormals) or above the largest finite bfloat16 raises.
    Returns float64 arrays holding bfloat16 values exactly.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    if np.any((ax != 0) & (ax < 2.0 ** -126)) or np.any(ax > 3.3895313892515355e38):
        raise ValueError("round_bf16: value outside the normal bfloat16 range")
    m, e = np.frexp(x)
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


def decode_step_bf16_state(q, k, v, g, beta, state, *, order=ORDER_STANDARD):
    """decode_step for a state stored in bfloat16 between steps.

    The stored values are exact in fp64; the step runs in fp64 as decode_step
    does, and the new state is stored by rounding each element once to
    bfloat16 (nearest, ties to even).  ``state`` holds bfloat16 values (a torch
    bfloat16 tensor, or float64 values that are all bfloat16-representable).
    Returns (o [N,Hv,Dv], new state before rounding, new state rounded), all
    float64.
    """
    s = _f64(state)
    if not np.array_equal(round_bf16(s), s):
        raise ValueError("decode_step_bf16_state: state is not bfloat16-representable")
    o, s_new = decode_step(q, k, v, g, beta, s, order=order)
    return o, s_new, round_bf16(s_new)


def _gather_slots(pool, slot_idx, reset, what):
    """The batch/reset rule of a state pool: a copy of the pool (fp64), the
    slot of each entry, and each entry's starting state -- its slot's, or
    zeros when reset[n] is nonzero.  Slot indices must be distinct and in
    range."""
    pool = _f64(pool).copy()
    idx = np.asarray(slot_idx.detach().cpu().numpy() if hasattr(slot_idx, "detach") else slot_idx,
                     dtype=np.int64)
    S = pool.shape[0]
    if idx.ndim != 1 or np.any(idx < 0) or np.any(idx >= S) or len(set(idx.tolist())) != idx.size:
        raise ValueError(f"{what}: slot indices must be distinct and in range")
    states = pool[idx].copy()
    if reset is not None:
        rs = np.asarray(reset.detach().cpu().numpy() if hasattr(reset, "detach") else reset)
        states[rs != 0] = 0.0
    return pool, idx, states


def _scatter_slots(pool, idx, new):
    """Each entry's final state back into its slot; other slots unchanged."""
    pool[idx] = new
    return pool


def decode_step_slots(q, k, v, g, beta, pool, slot_idx, reset=None, *, order=ORDER_STANDARD):
    """One decode step of N batch entries whose states live in a pool of slots
    (continuous batching): entry n uses pool[slot_idx[n]]; when reset[n] is
    nonzero it starts from a zero state instead (a new request), whatever the
    slot held.  The updated states are written back to their slots; slots no
    entry names are left as they are.  slot_idx must hold distinct values in
    [0, num_slots).

    Shapes: q,k [N,Hqk,Dk], v [N,Hv,Dv], g,beta [N,Hv], pool [S,Hv,Dv,Dk],
    slot_idx [N] int, reset [N] or None.  Returns (o [N,Hv,Dv], new pool) in
    float64.
    """
    pool, idx, states = _gather_slots(pool, slot_idx, reset, "decode_step_slots")
    o, new = decode_step(q, k, v, g, beta, states, order=order)
    return o, _scatter_slots(pool, idx, new)


def prefill_slots(q, k, v, g, beta, pool, slot_idx, reset=None, cu_seqlens=None, *,
                  order=ORDER_STANDARD):
    """A prefill of N packed sequences whose states live in a pool of slots
    (continuous batching, page "Hybrid · kết hợp…", section 3: state updates
    with batch and reset rules): sequence n starts from pool[slot_idx[n]], or
    from zeros when reset[n] is nonzero (a new request), and its final state is
    written back to that slot; slots no sequence names are left as they are.
    slot_idx must hold distinct values in [0, num_slots).

    Shapes as ``recurrent`` with N sequences; pool [S,Hv,Dv,Dk], slot_idx [N]
    int, reset [N] or None.  Returns (o [T,Hv,Dv], new pool) in float64.
    """
    pool, idx, states = _gather_slots(pool, slot_idx, reset, "prefill_slots")
    o, new = recurrent(q, k, v, g, beta, states, cu_seqlens, order=order)
    return o, _scatter_slots(pool, idx, new)


def short_conv(x, w, cu_seqlens=None, conv_state=None):
    """Causal depthwise convolution with 4 taps along time, the DeltaNet
    mixer's "kernel 4" convolution (page "Layouts híbridos: três DeltaNet, uma
    attention", section 01), one filter per channel:

        y[t, c] = w[c, 0] x[t-3, c] + w[c, 1] x[t-2, c] + w[c, 2] x[t-1, c] + w[c, 3] x[t, c]

    x [T, C] packed over sequences (cu_seqlens [N+1], or None for one); w [C, 4].
    Inputs before a sequence's first token come from conv_state [N, 3, C] (the
    three inputs that preceded it, oldest first) or are zero when it is None.
    Returns (y [T, C], new conv state [N, 3, C]: each sequence's last three
    inputs, reaching into the old state when the sequence is shorter than 3).
    All float64.
    """
    x, w = _f64(x), _f64(w)
    T, C = x.shape
    assert w.shape == (C, 4)
    if cu_seqlens is None:
        cu = np.array([0, T], dtype=np.int64)
    else:
        cu = np.asarray(cu_seqlens.detach().cpu().numpy() if hasattr(cu_seqlens, "detach")
                        else cu_seqlens, dtype=np.int64)
    N = cu.shape[0] - 1
    st = np.zeros((N, 3, C)) if conv_state is None else _f64(conv_state)
    y = np.zeros((T, C))
    new_state = np.zeros((N, 3, C))
    for n in range(N):
        # the sequence's inputs with its three predecessors in front
        ext = np.concatenate([st[n], x[cu[n]:cu[n + 1]]], axis=0)
        for t in range(cu[n + 1] - cu[n]):
            for j in range(4):
                y[cu[n] + t] += w[:, j] * ext[t + j]
        new_state[n] = ext[ext.shape[0] - 3:]
    return y, new_state


def l2_normalise_heads(y, H, D):
    """Each (token, head) row of y [T, H*D] divided by its Euclidean norm (a
    zero row stays zero).  Returns [T, H, D] float64."""
    y = _f64(y).reshape(-1, H, D)
    nrm = np.sqrt(np.sum(y * y, axis=-1, keepdims=True))
    return np.divide(y, nrm, out=np.zeros_like(y), where=nrm > 0)


def short_conv_norm(xq, xk, xv, wq, wk, wv, cu_seqlens=None, conv_state=None):
    """The front end of the DeltaNet mixer before the delta rule: the kernel-4
    causal convolution on the q, k and v channels, then q and k normalised per
    head.  xq, xk [T, Hqk, Dk], xv [T, Hv, Dv]; wq, wk [Hqk*Dk, 4], wv [Hv*Dv, 4];
    conv_state [N, 3, 2*Hqk*Dk + Hv*Dv] (q, k, v channels in that order) or
    None.  Returns (q, k, v, new conv state), float64."""
    xq, xk, xv = _f64(xq), _f64(xk), _f64(xv)
    T, Hqk, Dk = xq.shape
    Hv, Dv = xv.shape[1], xv.shape[2]
    Cq, Cv = Hqk * Dk, Hv * Dv
    cs = None if conv_state is None else _f64(conv_state)
    parts = [(xq, wq, 0, Cq), (xk, wk, Cq, Cq), (xv, wv, 2 * Cq, Cv)]
    ys, states = [], []
    for x, w, off, C in parts:
        y, s = short_conv(x.reshape(T, C), w, cu_seqlens, None if cs is None else cs[:, :, off:off + C])
        ys.append(y)
        states.append(s)
    q = l2_normalise_heads(ys[0], Hqk, Dk)
    k = l2_normalise_heads(ys[1], Hqk, Dk)
    v = ys[2].reshape(T, Hv, Dv)
    return q, k, v, np.concatenate(states, axis=2)


def chunk_state_maps(k, v, g, beta, *, chunk=64, head_k=0, head_v=0):
    """The chunk step of one (sequence, head) as an affine map of the entering
    state, for a context-parallel scan over a sequence's chunks.

    With the chunk quantities of chunked() (T = (I + A)^-1, W = T diag(b Gamma) K,
    U~ = T diag(b) V, e_C = Gamma_C / Gamma), the state leaving a chunk is
        S' = Gamma_C S + (U~ - W S^T)^T diag(e_C) K = S A_c + B_c,
        A_c = Gamma_C I - W^T diag(e_C) K   (Dk x Dk),
        B_c = U~^T diag(e_C) K              (Dv x Dk).
    k [T,Hqk,Dk], v [T,Hv,Dv], g, beta [T,Hv] of one sequence; head_k / head_v
    pick the heads.  Returns a list of (A_c, B_c), float64, one per chunk.
    """
    k, v, g, beta = _f64(k)[:, head_k], _f64(v)[:, head_v], _f64(g)[:, head_v], _f64(beta)[:, head_v]
    T, Dk = k.shape
    maps = []
    for c0 in range(0, T, chunk):
        K, V = k[c0:c0 + chunk], v[c0:c0 + chunk]
        gg, b = g[c0:c0 + chunk], beta[c0:c0 + chunk]
        L = K.shape[0]
        gam = np.cumsum(gg)
        M = np.tril(np.exp(gam[:, None] - gam[None, :]))
        A = np.tril(b[:, None] * (K @ K.T) * M, -1)
        Tm = np.linalg.solve(np.eye(L) + A, np.eye(L))
        W = Tm @ ((b * np.exp(gam))[:, None] * K)
        Ut = Tm @ (b[:, None] * V)
        eC = np.exp(gam[-1] - gam)
        Ac = np.exp(gam[-1]) * np.eye(Dk) - W.T @ (eC[:, None] * K)
        Bc = Ut.T @ (eC[:, None] * K)
        maps.append((Ac, Bc))
    return maps


def compose_state_maps(first, second):
    """The map of running chunk map `first`, then `second`:
    S -> (S A1 + B1) A2 + B2 = S (A1 A2) + (B1 A2 + B2).  Associative, so a
    sequence's chunk maps can be combined by a parallel scan."""
    (A1, B1), (A2, B2) = first, second
    return A1 @ A2, B1 @ A2 + B2
